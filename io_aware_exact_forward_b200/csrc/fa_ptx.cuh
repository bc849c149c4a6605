// fa_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA tensor loads (never multicast), tcgen05 (TMEM allocation, MMA,
// commit, TMEM loads/stores) and the shared-memory matrix descriptors that
// tcgen05.mma reads.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "fa_status.h"

namespace fa {

// ---------------------------------------------------------------------------
// Device status word and bounded waits
// ---------------------------------------------------------------------------

// Set by any kernel whose bounded wait expires; read and cleared by fa_check().
// (libfa is a single translation unit, so the definition lives here.)
__device__ int g_fa_status = 0;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// try_wait with the default suspend-time limit.  (A short explicit hint
// halves the hand-off latency between two otherwise idle warps, but the
// extra polling slowed the backward kernel, where most warps wait at once.)
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA abort flag in shared memory plus the wait limit.  Every wait polls
// the barrier; every 256 polls it checks the clock and the CTA's abort flag.
// On expiry it records FA_ERR_TIMEOUT in g_fa_status, raises the abort flag
// so that the CTA's other roles stop too, and returns false.  It never traps.
struct WaitCtl {
  volatile int* abort_flag;  // shared memory
  uint64_t limit_ns;
};

__device__ __forceinline__ void raise_abort(const WaitCtl& w) {
  *w.abort_flag = 1;
  atomicCAS(&g_fa_status, 0, (int)FA_ERR_TIMEOUT);
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) return false;
    if (globaltimer_ns() - t0 > w.limit_ns) {
      raise_abort(w);
      return false;
    }
  }
}

// Bounded wait used while draining in-flight work on an abort path: ignores
// the abort flag and records nothing.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit_ns) return false;
  return true;
}

// Move this warpgroup's per-thread register budget down / up to N (a
// multiple of 8 in [24, 256]).  Every warp of the warpgroup executes it; an
// increase waits until other warpgroups of the block have released enough
// of the registers the block was launched with.
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Named barrier among `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// TMA (tensor loads into this CTA's shared memory; no multicast)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, loads and stores
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T-as-described, kind::f16.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with the A operand read from tensor memory (K-major, bf16 pairs per column).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f8f6f4 forms of the two MMAs above (8-bit A and B of the formats the
// instruction descriptor names; K = 32 elements, 32 bytes, per instruction).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// A from tensor memory: four 8-bit values per 32-bit column, K-major.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

#define FA_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                 "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FA_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                 "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : FA_R8(0)
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), FA_W8(0)
               : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp gets
// lane (addr.lane + t), columns addr.col .. addr.col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : FA_R8(0), FA_R8(8)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      FA_W8(0), FA_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FA_W8(0), FA_W8(8), FA_W8(16), FA_W8(24)
      : "memory");
}

#undef FA_R8
#undef FA_W8

// ---------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor (tcgen05 format, version 1) for a tile
// stored with the 128-byte swizzle: 8-row x 128-byte atoms (1024 B).
//   start: byte address of the first element (atoms 1024-byte aligned)
//   lbo:   leading byte offset (MN-major: stride between 64-element column
//          blocks; unused for K-major swizzled layouts)
//   sbo:   stride byte offset (stride between consecutive 8-row groups)
// The descriptor as two 32-bit words.  Low: start (bits 0-13, 16-byte
// units) and lbo (bits 16-29).  High: sbo (bits 0-13), the version (bit 14)
// and the layout (bits 29-31: 2 = 128-byte swizzle).
__device__ __forceinline__ uint32_t sw128_lo(uint32_t start, uint32_t lbo) {
  return ((start >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t sw128_hi(uint32_t sbo) {
  return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t lo, uint32_t hi) {
  return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
  return sw128_desc(sw128_lo(start, lbo), sw128_hi(sbo));
}
// The MMA loops keep the low word of an operand's first K slice and add the
// slice's byte offset / 16: one integer add per MMA instead of rebuilding the
// descriptor.  The MMA-issuing thread shares its sub-partition with busy
// softmax warps, so its instruction count sets how fast it can feed the
// tensor core.  (Shared-memory addresses stay below 2^18 bytes, so the
// 14-bit start field never carries into the lbo field.)

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
//   a_mn / b_mn: 1 if that operand is MN-major (transposed) in shared memory.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                              // D format: f32
         | (1u << 7)                            // A format: bf16
         | (1u << 10)                           // B format: bf16
         | ((uint32_t)a_mn << 15)               // A major
         | ((uint32_t)b_mn << 16)               // B major
         | ((uint32_t)(N >> 3) << 17)           // N / 8
         | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0)
// and fp32 accumulation; a_mn / b_mn as above (MN-major is allowed for the
// 8-bit formats E4M3 and E5M2).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                              // D format: f32
         | (0u << 7)                            // A format: E4M3
         | (0u << 10)                           // B format: E4M3
         | ((uint32_t)a_mn << 15)
         | ((uint32_t)b_mn << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Small math helpers
// ---------------------------------------------------------------------------

// max(a, b, c) in one instruction (three-input form of max.f32).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair of floats on the FMA pipe instead of the MUFU unit.
// Cody-Waite range reduction: x = n + f with n = round(x) (from the bits of
// x + 1.5*2^23) and f in [-1/2, 1/2]; 2^f by the degree-3 minimax polynomial
// of fit_exp2_poly.py (Remez exchange on relative error, 7.5e-5 at most);
// 2^n added into the exponent bits.  x is clamped below at -126 (a lower
// clamp would wrap the exponent field of p < 1 into the sign bit), so inputs
// under -126 (including -inf) give a denormal near 2^-126, not 0: callers
// that need exact zeros (masked entries) must select them.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(kMagic, kMagic));
  const float2 n = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                        make_float2(0.2426111251115799f, 0.2426111251115799f));
  p = __ffma2_rn(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
  p = __ffma2_rn(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  // the low mantissa bits of t hold n; shifting them to the exponent field
  // multiplies by 2^n (the magic's own bits vanish in the shift)
  return make_float2(__int_as_float(__float_as_int(p.x) + (int)((uint32_t)__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (int)((uint32_t)__float_as_int(t.y) << 23)));
}

// ---------------------------------------------------------------------------
// Dropout mask: Philox-4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
// random numbers: as easy as 1, 2, 3", SC 2011), one block per 4 x 4 block of
// (query, key) pairs
// ---------------------------------------------------------------------------

// Ten rounds: multiply words 0 and 2 by the round constants into (hi, lo)
// pairs, mix with words 1 and 3 and the key, bump the key by the Weyl
// increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u, kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kW0;
      k1 += kW1;
    }
    // one 32 x 32 -> 64-bit product per multiplier gives both halves
    const uint64_t p0 = (uint64_t)kM0 * c.x, p1 = (uint64_t)kM1 * c.z;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
  }
  return c;
}

// Bit 7 of each byte of the result is set iff that byte of b is below t
// (every byte of tt is t; the other bits are zero).  Per byte, with the top
// bits set aside, (b | 0x80) - (t & 0x7F) cannot borrow from the next byte
// and its bit 7 says (b & 0x7F) >= (t & 0x7F); then b < t iff b7 < t7, or
// b7 == t7 and the low seven bits are below.
__device__ __forceinline__ uint32_t bytes_below(uint32_t b, uint32_t tt) {
  const uint32_t x = (b | 0x80808080u) - (tt & 0x7F7F7F7Fu);
  return ((~b & tt) | (~(b ^ tt) & ~x)) & 0x80808080u;
}

// Bits 7, 15, 23 and 31 of m (all other bits zero) as bits 0..3: the
// product puts each at bit 28 + its byte, and no two partial products share
// a bit.
__device__ __forceinline__ uint32_t gather_msb4(uint32_t m) { return (m * 0x00204081u) >> 28; }

// Keep bits of query row `row` for the 128 keys key0 .. key0 + 127 (key0 a
// multiple of 16): bit k of mask[k >> 5] is key key0 + k.  The block of rows
// 4a..4a+3 and keys 4c..4c+3 is Philox at counter (a, c, bh, offset); its
// word w is row 4a + w, byte j of that word key 4c + j, kept iff the byte is
// below t (1 <= t <= 255).  The four lanes of a quad hold rows 4a..4a+3 (row
// & 3 == lane & 3) and share blocks: lane q computes key groups 4m + q and
// passes each quad-mate its row's word.
__device__ __forceinline__ void dropout_keep_128(uint32_t (&mask)[4], int row, int key0, uint32_t bh,
                                                 uint32_t offset, uint32_t k0, uint32_t k1, uint32_t t) {
  const int lane = threadIdx.x & 31;
  const int q = lane & 3;
  const uint32_t tt = t * 0x01010101u;
#pragma unroll
  for (int i = 0; i < 4; ++i) mask[i] = 0u;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint4 wv = philox4x32_10(make_uint4((uint32_t)row >> 2, (uint32_t)(key0 >> 2) + 4 * m + q, bh, offset), k0, k1);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int src = (q + s) & 3;       // lane of the quad whose block this is
      const int want = (q - s) & 3;      // the word the receiving lane needs
      const uint32_t send = want == 0 ? wv.x : want == 1 ? wv.y : want == 2 ? wv.z : wv.w;
      const uint32_t got = s == 0 ? send : __shfl_sync(0xffffffffu, send, (lane & ~3) | src);
      const uint32_t bits = gather_msb4(bytes_below(got, tt));  // bit j: byte j below t
      // keys 4 * (4m + src) .. + 3 of the tile: word m / 2, bits 16 (m & 1) + 4 src
      mask[m >> 1] |= bits << (16 * (m & 1) + 4 * src);
    }
  }
}

// Two floats to two E4M3 bytes (round to nearest even, saturating to +-448),
// `lo` in bits 0-7 and `hi` in bits 8-15.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace fa
