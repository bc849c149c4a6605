// fa_bwd.cuh -- backward kernels: dQ, dK, dV of L = sum(dO * O), with S and
// P recomputed tile by tile from the forward's log-sum-exp instead of being
// stored ("FlashAttention" interview track, follow-up on recomputation; the
// products dV = P^T dO, dP = dO V^T, dS = P*(dP - D), dQ = scale dS K,
// dK = scale dS^T Q of "Efficient attention: memory-bound", section "Real
// code moves even more").
//
// Three kernels:
//   preprocess   D_i = sum_c dO_ic O_ic (fp32), LSE in log2 units (+inf for a
//                row that saw no key, so that its P is exactly 0), dQ
//                accumulator zeroed (unless dq_acc is null). (memory-bound)
//   dkdv         one work item per (128-key tile, KV head, batch).  K and V
//                stay in shared memory; the item walks the query tiles of
//                every query head of its GQA group.  Per tile:
//                  S^T = K Q^T, dP^T = V dO^T          (SS MMAs, TMEM)
//                  P^T = 2^{S^T*scale*log2e - LSE2}   (P warps, bf16 into
//                        the S^T columns)
//                  dV += P^T dO                         (TS MMA, P^T from TMEM)
//                  dS = P^T * (dP^T - D)               (dS warps, bf16 into
//                        a swizzled shared-memory tile: key rows, query
//                        columns)
//                  dK += dS^T Q                         (SS MMA, the tile
//                        read K-major)
//                  dQ_tile = dS K                       (SS MMA, the tile
//                        read MN-major)
//                At d = 64 (two S^T buffers) the next tile's S^T is issued
//                ahead and its dP^T as soon as the dS warps have read this
//                tile's; at d = 128 (one S^T buffer) the next S^T follows dV
//                once the dS warps hold this tile's P^T in registers, and
//                dQ_tile lands in the dP^T columns, so the next dP^T follows
//                the dQ read-out.  A sliding window is a separate
//                instantiation (its masking costs registers).
//                dQ_tile is read by a second warpgroup, staged in shared
//                memory and added into an fp32 accumulator in global memory
//                with bulk tensor reduce-adds (every KV tile contributes to
//                every query row it sees).  dK and dV are summed over the
//                group's heads in tensor memory, so the GQA sum needs no
//                atomics.
//   dq_convert   dq = bf16(accumulator).
// Warp roles in dkdv: 0-7 P^T and, at an item's end, dK/dV out; 8-15 dS
// (two warps per TMEM lane quarter, one per half of the 128 query columns);
// 16-19 dQ read-out and reduce-adds (one query row per thread); 20 MMA
// issuer; 21 TMA producer; with dropout at d = 64, 22-23 make the keep bits.
// The deterministic backward builds dkdv without dQ (DQ = false: no dQ
// product, warps 16-19 idle) and takes dQ from the pass in fa_bwd_dq.cuh.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

// ---------------------------------------------------------------------------
// preprocess
// ---------------------------------------------------------------------------
// Dv and lse2 rows have a pitch of Tq_pad = Tq rounded up to 128, so that
// every 128-row slice starts 16-byte aligned for a bulk copy; the padding
// entries hold D = 0 and LSE2 = +inf (P = 0).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ Dv, float* __restrict__ lse2,
    float* __restrict__ dq_acc, int B, int Hq, int Tq, int Tq_pad) {
  constexpr int LPR = D / 8;  // lanes per row, 8 elements (16 bytes) each
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gid / LPR;            // row index in [B][Tq][Hq] order
  const int sub = (int)(gid % LPR);
  const long long nrows = (long long)B * Tq * Hq;
  float dot = 0.f;
  if (row < nrows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + sub * 8);
    const uint4 c = *reinterpret_cast<const uint4*>(dO + row * D + sub * 8);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(a2[e]);
      const float2 y = __bfloat1622float2(c2[e]);
      dot = fmaf(x.x, y.x, dot);
      dot = fmaf(x.y, y.y, dot);
    }
    if (dq_acc) {
      float4* z = reinterpret_cast<float4*>(dq_acc + row * D + sub * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (row < nrows && sub == 0) {
    const int h = (int)(row % Hq);
    const long long bt = row / Hq;
    const int t = (int)(bt % Tq);
    const int b = (int)(bt / Tq);
    const long long bh = (long long)b * Hq + h;
    Dv[bh * Tq_pad + t] = dot;
    const float l = lse[bh * Tq + t];
    lse2[bh * Tq_pad + t] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
  }
  const int npad = Tq_pad - Tq;
  if (npad > 0 && gid < (long long)B * Hq * npad) {
    const long long bh = gid / npad;
    const long long idx = bh * Tq_pad + Tq + gid % npad;
    Dv[idx] = 0.f;
    lse2[idx] = INFINITY;
  }
}

// ---------------------------------------------------------------------------
// dq convert
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                __nv_bfloat16* __restrict__ dq,
                                                                long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  uint4 out;
  out.x = pack_bf16x2(a.x, a.y);
  out.y = pack_bf16x2(a.z, a.w);
  out.z = pack_bf16x2(b.x, b.y);
  out.w = pack_bf16x2(b.z, b.w);
  reinterpret_cast<uint4*>(dq)[i] = out;
}

// ---------------------------------------------------------------------------
// dK / dV (+ dQ contributions)
// ---------------------------------------------------------------------------
struct BwdParams {
  CUtensorMap tm_q;    // [B][Tq][Hq][d] bf16, box {64,1,128,1}, 128-byte swizzle
  CUtensorMap tm_do;
  CUtensorMap tm_k;    // [B][Tk][Hkv][d]
  CUtensorMap tm_v;
  CUtensorMap tm_dq;   // fp32 accumulator [B][Tq][Hq][d], box {32,1,128,1}, 128-byte swizzle
  const float* lse2;   // [B][Hq][Tq]
  const float* Dv;     // [B][Hq][Tq]
  float* dq_acc;       // [B][Tq][Hq][d], receives scale * dS K
  __nv_bfloat16* dk;   // [B][Tk][Hkv][d]
  __nv_bfloat16* dv;
  int B, Hq, Hkv, Tq, Tk, causal;
  int window;          // > 0: sliding window of that many keys (implies causal)
  int Tq_pad;          // row pitch of lse2 / Dv
  float scale, scale_log2;
  int n_kv_tiles;
  int n_items;         // n_kv_tiles * B * Hkv
  // dropout on P (the DROP instantiation): keep iff the Philox byte < drop_t
  // (1..255), kept values scaled by drop_scale = 256 / drop_t; Philox key
  // (seed_lo, seed_hi) and counter word 3 drop_offset, as in the forward
  uint32_t drop_t, seed_lo, seed_hi, drop_offset;
  float drop_scale;
  unsigned long long wait_limit_ns;
};

// Bulk tensor reduce-add of a shared-memory tile into global memory (fp32).
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* m, uint32_t src, int c0, int c1,
                                                  int c2, int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int D, bool DROP = false, bool DQ = true>
struct BwdCfg {
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = 128 * 128;
  static constexpr int TILE = NBOX * BOX_BYTES;         // 128 rows x D bf16
  // d = 64: two S^T buffers in tensor memory, two K/V buffers and three
  // Q/dO stages in shared memory (the next item's K/V load overlaps this
  // item) and one 32-column fp32 box for staging dQ.  d = 128: one S^T
  // buffer and one K/V buffer (tensor and shared memory are full), two Q
  // stages but a single dO buffer with its own barriers (the next dO is
  // loaded between this tile's dV and the next tile's dP^T), which leaves
  // room for two dQ staging boxes.  The staged boxes go out with bulk
  // tensor reduce-adds.  Without dQ (DQ = false) the staging boxes' room
  // holds a second dO buffer instead, and dO travels with Q in each stage.
  static constexpr int NSBUF = (D == 64) ? 2 : 1;
  static constexpr int NKV = (D == 64) ? 2 : 1;
  static constexpr bool SPLIT_DO = (D == 128) && DQ;
  static constexpr int NQ = (D == 64) ? 3 : 2;          // Q / LSE2 / D (and dO) stages
  static constexpr int NDO = SPLIT_DO ? 1 : NQ;         // dO buffers
  static constexpr int NDQS = (D == 128) ? 2 : 1;       // dQ staging boxes (none allocated without dQ)
  static constexpr int OFF_K = 0;                       // NKV buffers of (K, V)
  static constexpr int OFF_Q = 2 * NKV * TILE;          // NQ stages
  static constexpr int OFF_DO = OFF_Q + NQ * TILE;      // NDO buffers
  static constexpr int OFF_DS = OFF_DO + NDO * TILE;    // 128 x 128 bf16, 2 boxes
  // fp32 staging of 32 dQ columns per box (128-byte swizzle), reused across
  // the boxes of the tile
  static constexpr int OFF_DQS = OFF_DS + 2 * BOX_BYTES;
  static constexpr int DQS_BYTES = DQ ? NDQS * 128 * 32 * 4 : 0;
  static constexpr int OFF_LSE = OFF_DQS + DQS_BYTES;   // [NQ][128] f32
  static constexpr int OFF_DD = OFF_LSE + NQ * 128 * 4; // [NQ][128] f32
  // Dropout at d = 64: warps 22-23 make each query tile's keep bits ahead
  // of the P^T warps, into two buffers of [128 keys][2 query halves] x 64
  // bits; the P^T warps load their key's 8 bytes.  (At d = 128 shared
  // memory is full and the P^T warps make their own.)
  static constexpr bool MASKW = DROP && D == 64;
  static constexpr int OFF_MASK = OFF_DD + NQ * 128 * 4;
  static constexpr int MASK_BYTES = MASKW ? 2 * 128 * 2 * 8 : 0;
  static constexpr int OFF_BAR = OFF_MASK + MASK_BYTES;
  // kv_full[2], kv_empty[2], qdo_full[3], qdo_empty[3], s_full[2], p_full[2],
  // dp_full, ds_full, dq_full[2], dq_free[2], dkdv_done, mma_done, dp_free,
  // do_full, p_read, do_empty (, mask_full[2], mask_empty[2])
  static constexpr int NBAR = 26 + (MASKW ? 4 : 0);
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  // warps 0-7 P^T (two per TMEM lane quarter, one per half of the query
  // columns), 8-15 dS, 16-19 dQ, 20 MMA issuer, 21 TMA producer
  static constexpr int THREADS = MASKW ? 768 : 704;
  static constexpr int MMA_WARP = 20;
  static constexpr int LOAD_WARP = 21;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_DV = 0;
  static constexpr int TM_DK = D;
  static constexpr int TM_S0 = 2 * D;                   // S^T buffers; dQ reuses them
  static constexpr int TM_DP = 2 * D + 128 * NSBUF;
  static constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t IDESC_TS = idesc_bf16_f32(128, D, 0, 1);
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 1, 1);
  static_assert(TM_DP + 128 <= TMEM_COLS, "tensor memory overflow");
  static_assert(OFF_DQS % 1024 == 0 && OFF_DS % 1024 == 0 && OFF_DO % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
  static_assert(NQ <= 3, "barrier slots");
};

// One work item: the 128-key tile kt of KV head hkv of batch b, against
// every query tile (of every query head of the GQA group) that sees it.
struct BwdItem {
  int b, hkv, j0, qt_begin, nq, n_it;
};

__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p, int item) {
  BwdItem it;
  // Key tiles of one (batch, KV head) are adjacent in item order, so the
  // head's dQ accumulator rows and Q/dO tiles stay in L2 while they run.
  const int kt = item % p.n_kv_tiles;
  const int hb = item / p.n_kv_tiles;
  it.b = hb / p.Hkv;
  it.hkv = hb % p.Hkv;
  it.j0 = kt * 128;
  const int n_qt = (p.Tq + 127) / 128;
  it.qt_begin = 0;
  int qt_end = n_qt;
  if (p.causal) {
    const int qmin = it.j0 - (p.Tk - p.Tq);   // first query that sees key j0
    it.qt_begin = qmin <= 0 ? 0 : min(n_qt, qmin / 128);
    if (p.window > 0) {
      // last query whose window still holds the tile's last key
      const long long qmax = (long long)it.j0 + 127 - (p.Tk - p.Tq) + p.window - 1;
      qt_end = qmax < 0 ? 0 : (int)min((long long)n_qt, qmax / 128 + 1);
    }
  }
  it.nq = max(0, qt_end - it.qt_begin);
  it.n_it = (p.Hq / p.Hkv) * it.nq;
  return it;
}

// Keep bits of key row `key` for the 64 queries q0 .. q0 + 63 (q0 a multiple
// of 16) under the forward's dropout mask: bit i of mask[i >> 5] is query
// q0 + i.  The block of queries 4a..4a+3 and keys 4c..4c+3 is Philox at
// counter (a, c, bh, offset); word w is query 4a + w, byte j key 4c + j.
// The four lanes of a quad hold keys 4c..4c+3 (key & 3 == lane & 3): lane q
// computes the blocks of query groups 4m + q, transposes each block's 4 x 4
// bytes so that word r holds key 4c + r's bytes, and passes word r to
// quad-mate r.
__device__ __forceinline__ void dropout_keep_keyrow_64(uint32_t (&mask)[2], int key, int q0, uint32_t bh,
                                                       uint32_t offset, uint32_t k0, uint32_t k1, uint32_t t) {
  const int lane = threadIdx.x & 31;
  const int q = lane & 3;
  const uint32_t tt = t * 0x01010101u;
  mask[0] = mask[1] = 0u;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 wv = philox4x32_10(make_uint4((uint32_t)(q0 >> 2) + 4 * m + q, (uint32_t)key >> 2, bh, offset), k0, k1);
    // 4 x 4 byte transpose: x[r] = byte r of words 0..3
    const uint32_t lo01 = __byte_perm(wv.x, wv.y, 0x5140), hi01 = __byte_perm(wv.x, wv.y, 0x7362);
    const uint32_t lo23 = __byte_perm(wv.z, wv.w, 0x5140), hi23 = __byte_perm(wv.z, wv.w, 0x7362);
    const uint32_t x[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                           __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int src = (q + s) & 3;       // lane whose block (query group 4m + src) arrives now
      const int want = (q - s) & 3;      // the key (quad-mate) this lane sends to
      const uint32_t send = want == 0 ? x[0] : want == 1 ? x[1] : want == 2 ? x[2] : x[3];
      const uint32_t got = s == 0 ? send : __shfl_sync(0xffffffffu, send, (lane & ~3) | src);
      const uint32_t bits = gather_msb4(bytes_below(got, tt));  // bit j: byte j below t
      // queries 4 (4m + src) .. + 3 of the 64: word m / 2, bits 16 (m & 1) + 4 src
      mask[m >> 1] |= bits << (16 * (m & 1) + 4 * src);
    }
  }
}

// WIN: sliding-window masking compiled in (a separate instantiation, so
// that the plain path keeps its registers).  DQ = false: no dQ product,
// read-out or reduce-adds (warps 16-19 idle); dQ then comes from the
// separate, deterministic pass of fa_bwd_dq.cuh.  DROP: dropout on P, with the
// keep mask of the forward regenerated per key row; the P^T warps write the
// dropped P^T (the dV operand) and the undropped P^T side by side, 8 columns
// each per 16-query chunk, and the dS warps read the keep bits off the
// dropped copy's zeros:
//   dV += (P*Z)^T dO * s,   dS = P * (Z * s * dP - D),   s = 256 / t.
template <int D, bool WIN, bool DROP = false, bool DQ = true>
__global__ void __maxnreg__(80) fa_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D, DROP, DQ>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the layout needs 1024-byte aligned swizzle atoms
    if (threadIdx.x == 0) atomicCAS(&g_fa_status, 0, (int)FA_ERR_CUDA);
    return;
  }
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar_kv_full = [&](int k) { return bar0 + 8u * k; };
  auto bar_kv_empty = [&](int k) { return bar0 + 8u * (2 + k); };
  auto bar_qdo_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto bar_qdo_empty = [&](int s) { return bar0 + 8u * (7 + s); };
  auto bar_s_full = [&](int b) { return bar0 + 8u * (10 + b); };
  auto bar_p_full = [&](int b) { return bar0 + 8u * (12 + b); };
  const uint32_t bar_dp_full = bar0 + 8u * 14;
  const uint32_t bar_ds_full = bar0 + 8u * 15;
  auto bar_dq_full = [&](int b) { return bar0 + 8u * (16 + b); };
  auto bar_dq_free = [&](int b) { return bar0 + 8u * (18 + b); };
  const uint32_t bar_dkdv_done = bar0 + 8u * 20;
  const uint32_t bar_mma_done = bar0 + 8u * 21;
  const uint32_t bar_dp_free = bar0 + 8u * 22;
  const uint32_t bar_do_full = bar0 + 8u * 23;   // single dO buffer (d = 128)
  const uint32_t bar_p_read = bar0 + 8u * 24;    // the dS warps hold this tile's P^T
  const uint32_t bar_do_empty = bar0 + 8u * 25;
  // dropout keep bits of query tile gi in buffer gi & 1: written by the mask
  // warps, read by every P^T thread
  auto bar_mask_full = [&](int b) { return bar0 + 8u * (26 + b); };
  auto bar_mask_empty = [&](int b) { return bar0 + 8u * (28 + b); };
  // Q/dO stage of global iteration g and the parity of its use of that stage.
  auto stg = [&](int g) { return g % C::NQ; };
  auto stg_par = [&](int g) { return (uint32_t)((g / C::NQ) & 1); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* stop_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  float* lse_s = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* dd_s = reinterpret_cast<float*>(smem + C::OFF_DD);
  auto aK = [&](int kvb) { return sbase + C::OFF_K + (2 * kvb) * C::TILE; };
  auto aV = [&](int kvb) { return sbase + C::OFF_K + (2 * kvb + 1) * C::TILE; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  WaitCtl wc{abort_flag, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *stop_flag = 0;
    for (int s = 0; s < C::NQ; ++s) {
      mbar_init(bar_qdo_full(s), 1);
      mbar_init(bar_qdo_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
      mbar_init(bar_s_full(s), 1);
      mbar_init(bar_p_full(s), 256);
      mbar_init(bar_dq_full(s), 1);
      mbar_init(bar_dq_free(s), DQ ? 128 : 256);
    }
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_dp_free, 256);
    mbar_init(bar_ds_full, 256);
    mbar_init(bar_dkdv_done, 1);
    mbar_init(bar_mma_done, 1);
    mbar_init(bar_do_full, 1);
    mbar_init(bar_do_empty, 1);
    mbar_init(bar_p_read, 256);
    if (C::MASKW) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar_mask_full(b), 64);
        mbar_init(bar_mask_empty(b), 512);  // the P^T and the dS warps read each buffer
      }
    }
    fence_barrier_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::LOAD_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_do);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      bool ok = true;
      int gi = 0, ki = 0, issued_kv = 0, n_do = 0;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const BwdItem I = bwd_item(p, item);
        if (I.n_it == 0) continue;
        const int kvb = ki % C::NKV;
        if (ki >= C::NKV) ok = mbar_wait(bar_kv_empty(kvb), ((ki / C::NKV) - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kv_full(kvb), 2 * C::TILE);
        for (int kb = 0; kb < C::NBOX; ++kb) {
          tma_load_4d(aK(kvb) + kb * C::BOX_BYTES, &p.tm_k, bar_kv_full(kvb), kb * 64, I.hkv, I.j0, I.b);
          tma_load_4d(aV(kvb) + kb * C::BOX_BYTES, &p.tm_v, bar_kv_full(kvb), kb * 64, I.hkv, I.j0, I.b);
        }
        ++issued_kv;
        for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
          const int s = stg(gi);
          const int h = I.hkv * G + it / I.nq;
          const int q0 = (I.qt_begin + it % I.nq) * 128;
          if (gi >= C::NQ) ok = mbar_wait(bar_qdo_empty(s), stg_par(gi) ^ 1u, wc);
          if (!ok) break;
          const size_t rbase = ((size_t)I.b * p.Hq + h) * p.Tq_pad + q0;
          mbar_arrive_expect_tx(bar_qdo_full(s), (C::SPLIT_DO ? 1 : 2) * C::TILE + 2 * 512);
          for (int kb = 0; kb < C::NBOX; ++kb) {
            tma_load_4d(sbase + C::OFF_Q + s * C::TILE + kb * C::BOX_BYTES, &p.tm_q, bar_qdo_full(s), kb * 64, h,
                        q0, I.b);
            if (!C::SPLIT_DO)
              tma_load_4d(sbase + C::OFF_DO + s * C::TILE + kb * C::BOX_BYTES, &p.tm_do, bar_qdo_full(s),
                          kb * 64, h, q0, I.b);
          }
          bulk_load(sbase + C::OFF_LSE + s * 512, p.lse2 + rbase, 512, bar_qdo_full(s));
          bulk_load(sbase + C::OFF_DD + s * 512, p.Dv + rbase, 512, bar_qdo_full(s));
          if (C::SPLIT_DO) {
            // the single dO buffer: free once the previous tile's dV is done
            if (gi >= 1) ok = mbar_wait(bar_do_empty, (gi - 1) & 1, wc);
            if (!ok) break;
            mbar_arrive_expect_tx(bar_do_full, C::TILE);
            for (int kb = 0; kb < C::NBOX; ++kb)
              tma_load_4d(sbase + C::OFF_DO + kb * C::BOX_BYTES, &p.tm_do, bar_do_full, kb * 64, h, q0, I.b);
            ++n_do;
          }
        }
        ++ki;
      }
      if (!ok) {
        for (int k = max(0, issued_kv - C::NKV); k < issued_kv; ++k)
          mbar_wait_drain(bar_kv_full(k % C::NKV), (k / C::NKV) & 1, p.wait_limit_ns);
        for (int g = max(0, gi - C::NQ); g <= gi; ++g)
          mbar_wait_drain(bar_qdo_full(stg(g)), stg_par(g), p.wait_limit_ns);
        if (n_do > 0) mbar_wait_drain(bar_do_full, (n_do - 1) & 1, p.wait_limit_ns);
      }
    }
  } else if (C::MASKW && warp >= 22) {
    // ------------------------------------------------------------ dropout mask
    // Thread mt makes the keep bits of keys 4 (mt >> 1) .. + 3 of the tile for
    // query half mt & 1 of every query tile: the 16 Philox blocks of those
    // keys and 64 queries (the layout the P^T warps' own generator uses:
    // counter (query / 4, key / 4, bh, offset), word = query, byte = key),
    // each key's bits gathered into two 32-query words.
    const int mt = threadIdx.x - 704;
    const int cl = mt >> 1, half = mt & 1;
    const uint32_t tt = p.drop_t * 0x01010101u;
    uint2* mbuf = reinterpret_cast<uint2*>(smem + C::OFF_MASK);
    bool ok = true;
    int gi = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const BwdItem I = bwd_item(p, item);
      const uint32_t cg = (uint32_t)(I.j0 >> 2) + (uint32_t)cl;
      for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
        const int mb = gi & 1;
        if (gi >= 2) ok = mbar_wait(bar_mask_empty(mb), ((gi >> 1) - 1) & 1, wc);
        if (!ok) break;
        const uint32_t bh = (uint32_t)(I.b * p.Hq + I.hkv * G + it / I.nq);
        const uint32_t a0 = (uint32_t)((I.qt_begin + it % I.nq) * 128 + 64 * half) >> 2;
        uint32_t kw[4][2];  // [key of the group][32-query word]
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
#pragma unroll
          for (int r = 0; r < 4; ++r) kw[r][w2] = 0u;
          // rolled: unrolled, the blocks' states would not fit 80 registers
#pragma unroll 1
          for (int al = 0; al < 8; ++al) {
            const uint4 wv = philox4x32_10(make_uint4(a0 + 8 * w2 + al, cg, bh, p.drop_offset), p.seed_lo, p.seed_hi);
            // 4 x 4 byte transpose: x[r] = byte r (key 4 cg + r) of words 0..3
            // (queries)
            const uint32_t lo01 = __byte_perm(wv.x, wv.y, 0x5140), hi01 = __byte_perm(wv.x, wv.y, 0x7362);
            const uint32_t lo23 = __byte_perm(wv.z, wv.w, 0x5140), hi23 = __byte_perm(wv.z, wv.w, 0x7362);
            const uint32_t x[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                                   __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
#pragma unroll
            for (int r = 0; r < 4; ++r) kw[r][w2] |= gather_msb4(bytes_below(x[r], tt)) << (4 * al);
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) mbuf[(mb * 128 + 4 * cl + r) * 2 + half] = make_uint2(kw[r][0], kw[r][1]);
        mbar_arrive(bar_mask_full(mb));
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tDP = tmem + C::TM_DP, tDV = tmem + C::TM_DV, tDK = tmem + C::TM_DK;
      auto tS = [&](int buf) { return tmem + C::TM_S0 + 128 * buf; };
      const uint32_t aDS = sbase + C::OFF_DS;
      auto aQ = [&](int g) { return sbase + C::OFF_Q + stg(g) * C::TILE; };
      auto aDO = [&](int g) { return sbase + C::OFF_DO + (C::SPLIT_DO ? 0 : stg(g) * C::TILE); };
      auto wait_do = [&](int g) { return !C::SPLIT_DO || mbar_wait(bar_do_full, g & 1, wc); };
      // Descriptors: the low word of the tile's first slice plus the slice
      // offset / 16 (the tile's low word is common to the unrolled slices).
      constexpr uint32_t HI = sw128_hi(1024);
      auto kdesc = [&](uint32_t base, int k) {  // K-major tile, k-th 16-element slice of d
        return sw128_desc(sw128_lo(base, 16) + (((k >> 2) * C::BOX_BYTES + (k & 3) * 32) >> 4), HI);
      };
      auto mndesc = [&](uint32_t base, int k) {  // MN-major view, k-th 16-row slice
        return sw128_desc(sw128_lo(base, C::BOX_BYTES) + ((k * 16 * 128) >> 4), HI);
      };
      auto issue_s = [&](int g, int kvb) {
        const int buf = g % C::NSBUF;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) mma_ss(tS(buf), kdesc(aK(kvb), k), kdesc(aQ(g), k), C::IDESC_SS, k > 0);
        mma_commit(bar_s_full(buf));
      };
      auto issue_dp = [&](int g, int kvb) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) mma_ss(tDP, kdesc(aV(kvb), k), kdesc(aDO(g), k), C::IDESC_SS, k > 0);
        mma_commit(bar_dp_full);
      };
      bool ok = true;
      int gi = 0, ki = 0;
      bool started = false;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const BwdItem I = bwd_item(p, item);
        if (I.n_it == 0) continue;
        const int kvb = ki % C::NKV;
        if (!started) {
          ok = mbar_wait(bar_kv_full(kvb), (ki / C::NKV) & 1, wc);
          if (ok) ok = mbar_wait(bar_qdo_full(stg(0)), stg_par(0), wc);
          if (ok) ok = wait_do(0);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, kvb);
          issue_dp(0, kvb);
          started = true;
        }
        const bool has_next_item = item + (int)gridDim.x < p.n_items;
        for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
          const int buf = gi % C::NSBUF;
          const bool last = it + 1 == I.n_it;
          const bool has_next = !last || has_next_item;
          // K/V buffer of the next iteration; waits for it when it belongs
          // to the next item.
          const int kvb_next = last ? (ki + 1) % C::NKV : kvb;
          auto wait_next_operands = [&]() -> bool {
            if (!mbar_wait(bar_qdo_full(stg(gi + 1)), stg_par(gi + 1), wc)) return false;
            if (last && !mbar_wait(bar_kv_full(kvb_next), ((ki + 1) / C::NKV) & 1, wc)) return false;
            return true;
          };
          if (C::NSBUF == 2 && has_next) {
            // S^T of the next iteration into the other buffer, which dQ of
            // the previous iteration used.  Without dQ the buffer's dq_free
            // barrier is arrived on by the dS warps once they hold that
            // iteration's P^T (its dV, issued earlier, reads P^T ahead of
            // the new S^T in the tensor pipe's order); a barrier per buffer,
            // so that the awaited phase is never two behind.
            ok = wait_next_operands();
            if (ok && gi >= 1) ok = mbar_wait(bar_dq_free((gi + 1) & 1), ((gi - 1) >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_s(gi + 1, kvb_next);
          }
          // P^T of query half h sits in columns [64h, 64h+32) of the S^T
          // buffer; with dropout the dropped P^T of chunk c (16 queries) in
          // columns 64h + 16c .. + 7.
          auto p_col = [](int k) {
            return DROP ? ((k < 4) ? k * 16 : 64 + (k - 4) * 16) : ((k < 4) ? k * 8 : 64 + (k - 4) * 8);
          };
          ok = mbar_wait(bar_p_full(buf), (gi / C::NSBUF) & 1, wc);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts(tDV, tS(buf) + p_col(k), mndesc(aDO(gi), k), C::IDESC_TS, it > 0 || k > 0);
          if (C::SPLIT_DO) mma_commit(bar_do_empty);
          if (C::NSBUF == 2 && has_next) {
            // dP^T of the next tile as soon as the dS warps have read this one.
            ok = mbar_wait(bar_dp_free, gi & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_dp(gi + 1, kvb_next);
          }
          if (C::NSBUF == 1 && has_next) {
            // With one S^T buffer the next S^T follows dV (queued behind it)
            // once the dS warps hold this tile's P^T in registers.
            ok = wait_next_operands();
            if (ok) ok = mbar_wait(bar_p_read, gi & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_s(gi + 1, kvb_next);
          }
          ok = mbar_wait(bar_ds_full, gi & 1, wc);
          if (!ok) break;
          tc_fence_after();
          // dK += dS^T Q with dS^T read from the shared dS tile (key rows,
          // query columns: K-major for this product); its completion frees
          // the Q stage.  dQ = dS K: with two S^T buffers (d = 64) into this
          // tile's (P^T was read above); with one (d = 128), into the dP^T
          // columns, which the dS warps have read (the S^T buffer already
          // holds the next S^T).  At d = 64 dQ goes first, so that its
          // read-out, which the next-but-one S^T waits for, starts one
          // product earlier (measured 6% faster), and dK's commit, which
          // frees the Q stage, also frees the dS tile (the dS warps wait on
          // the stage's barrier); at d = 128 dK first measured faster, and
          // dQ's completion frees the tile.
          const uint32_t tDQ = C::NSBUF == 1 ? tDP : tS(buf);
          if constexpr (D == 64) {
            if constexpr (DQ) {
#pragma unroll
              for (int k = 0; k < 8; ++k) mma_ss(tDQ, mndesc(aDS, k), mndesc(aK(kvb), k), C::IDESC_DQ, k > 0);
              mma_commit(bar_dq_full(buf));
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ss(tDK, kdesc(aDS, k), mndesc(aQ(gi), k), C::IDESC_TS, it > 0 || k > 0);
            mma_commit(bar_qdo_empty(stg(gi)));
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ss(tDK, kdesc(aDS, k), mndesc(aQ(gi), k), C::IDESC_TS, it > 0 || k > 0);
            mma_commit(bar_qdo_empty(stg(gi)));
            if constexpr (DQ) {
#pragma unroll
              for (int k = 0; k < 8; ++k) mma_ss(tDQ, mndesc(aDS, k), mndesc(aK(kvb), k), C::IDESC_DQ, k > 0);
              mma_commit(bar_dq_full(buf));
            }
          }
          if (last) {
            mma_commit(bar_kv_empty(kvb));
            mma_commit(bar_dkdv_done);
          }
          if (C::NSBUF == 1 && has_next) {
            // The next dP^T reuses the dQ columns: after the dQ read-out
            // (without dQ, once the dS warps have read this dP^T).
            ok = DQ ? mbar_wait(bar_dq_free(0), gi & 1, wc) : mbar_wait(bar_dp_free, gi & 1, wc);
            if (ok) ok = wait_do(gi + 1);
            if (!ok) break;
            tc_fence_after();
            issue_dp(gi + 1, kvb_next);
          }
        }
        ++ki;
      }
      mma_commit(bar_mma_done);
      mbar_wait_drain(bar_mma_done, 0, p.wait_limit_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T (WG-A)
    const int lq = warp & 3, half = warp >> 2;  // TMEM lane quarter, query half
    const int j = lq * 32 + lane;               // key row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(lq * 32) << 16;
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    bool ok = true;
    int gi = 0, ki = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const BwdItem I = bwd_item(p, item);
      const int key = I.j0 + j;
      const int qmin = key - (p.Tk - p.Tq);  // causal: first query that sees this key
      const bool key_ok = key < p.Tk;
      for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
        const int s = stg(gi), buf = gi % C::NSBUF;
        const int q0 = (I.qt_begin + it % I.nq) * 128;
        const uint32_t tS = tmem + C::TM_S0 + 128 * buf + lane_off + 64 * half;
        // dropout: this key's keep bits for the warp's 64 queries, made while
        // the tensor core computes S^T
        uint32_t keep[2] = {0u, 0u};
        if constexpr (C::MASKW) {
          // this key's keep bits for the warp's 64 queries, from the mask warps
          const int mb = gi & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_mask_full(mb), (gi >> 1) & 1, wc));
          if (!ok) break;
          const uint2 kv = reinterpret_cast<const uint2*>(smem + C::OFF_MASK)[(mb * 128 + j) * 2 + half];
          keep[0] = kv.x;
          keep[1] = kv.y;
          mbar_arrive(bar_mask_empty(mb));
        } else if constexpr (DROP) {
          dropout_keep_keyrow_64(keep, key, q0 + 64 * half, (uint32_t)(I.b * p.Hq + I.hkv * G + it / I.nq),
                                 p.drop_offset, p.seed_lo, p.seed_hi, p.drop_t);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar_qdo_full(s), stg_par(gi), wc));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(buf), (gi / C::NSBUF) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        const float* lrow = lse_s + s * 128 + 64 * half;
        const int cmin = p.causal ? qmin - q0 - 64 * half : 0;  // columns < cmin are masked
        // and, with a window, columns >= cmax (queries past this key's window)
        const int cmax = WIN ? qmin + p.window - q0 - 64 * half : (1 << 30);
        const bool masked = __any_sync(0xffffffffu, !key_ok || cmin > 0 || (WIN && cmax < 64));
        // 64 query columns in four 16-column chunks; the load of chunk c+1
        // overlaps the exponentials of chunk c.  P^T (bf16 pairs) goes to
        // the first 32 columns of this warp's 64, never ahead of its loads.
        uint32_t sv[2][16];
        tmem_ld16(tS, sv[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_wait_ld();
          if (c + 1 < 4) tmem_ld16(tS + (c + 1) * 16, sv[(c + 1) & 1]);
          const uint32_t* cur = sv[c & 1];
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = c * 16 + 2 * e;
            const float2 l2 = *reinterpret_cast<const float2*>(lrow + col);
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(cur[2 * e]), __uint_as_float(cur[2 * e + 1])),
                                        sl2, make_float2(-l2.x, -l2.y));
            float p0 = ex2_approx(x.x);
            float p1 = ex2_approx(x.y);
            if (masked) {
              if (!key_ok || col < cmin || (WIN && col >= cmax)) p0 = 0.f;
              if (!key_ok || col + 1 < cmin || (WIN && col + 1 >= cmax)) p1 = 0.f;
            }
            pk[e] = pack_bf16x2(p0, p1);
          }
          if constexpr (DROP) {
            // undropped P^T beside the dropped one, both over this chunk's
            // own (already loaded) S^T columns
            tmem_st8(tS + c * 16 + 8, pk);
            const uint32_t kb = keep[c >> 1] >> (16 * (c & 1));
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pk[e] &= ((kb >> (2 * e)) & 1u ? 0x0000FFFFu : 0u) | ((kb >> (2 * e + 1)) & 1u ? 0xFFFF0000u : 0u);
            tmem_st8(tS + c * 16, pk);
          } else {
            tmem_st8(tS + c * 8, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_full(buf));
      }
      if (!ok) break;
      // ---------------------------------------------------------- dK, dV out
      const bool have = I.n_it > 0;
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_dkdv_done, ki & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tsrc = tmem + (which ? C::TM_DK : C::TM_DV) + lane_off + half * (D / 2);
        const float mul = which ? p.scale : (DROP ? p.drop_scale : 1.f);
        __nv_bfloat16* dst = (which ? p.dk : p.dv) +
                             (((size_t)I.b * p.Tk + (key < p.Tk ? key : 0)) * p.Hkv + I.hkv) * D + half * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tsrc + c * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pw[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
          if (key < p.Tk) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = pk[i];
          }
        }
      }
      // dK/dV have been read: the next item's first dV/dK MMAs (which
      // overwrite them) wait for this warp's next p_full arrival.
      tc_fence_before();
      if (have) ++ki;
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------ dS (WG-B)
    const int w8 = warp - 8;
    const int lq = w8 & 3, half = w8 >> 2;
    const int j = lq * 32 + lane;               // key row == TMEM lane
    const uint32_t lane_off = (uint32_t)(lq * 32) << 16;
    const uint32_t tDP = tmem + C::TM_DP + lane_off + 64 * half;
    uint8_t* ds_row = smem + C::OFF_DS + half * C::BOX_BYTES + j * 128;
    bool ok = true;
    int gi = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const BwdItem I = bwd_item(p, item);
      for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
        const int s = stg(gi), buf = gi % C::NSBUF;
        const uint32_t tP = tmem + C::TM_S0 + 128 * buf + lane_off + 64 * half;  // P^T (bf16 pairs)
        ok = __all_sync(0xffffffffu, mbar_wait(bar_qdo_full(s), stg_par(gi), wc));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_p_full(buf), (gi / C::NSBUF) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        // P^T of this warp's 64 query columns into registers at once, so
        // that the S^T buffer can take the next S^T.
        uint32_t pp[32];
        uint32_t keep[2] = {0u, 0u};
        if constexpr (C::MASKW) {
          // undropped P^T, and this key's keep bits from the mask warps'
          // buffer (as the P^T warps read them)
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld8(tP + 16 * c + 8, pp + 8 * c);
          const int mb = gi & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_mask_full(mb), (gi >> 1) & 1, wc));
          if (!ok) break;
          const uint2 kv = reinterpret_cast<const uint2*>(smem + C::OFF_MASK)[(mb * 128 + j) * 2 + half];
          keep[0] = kv.x;
          keep[1] = kv.y;
          mbar_arrive(bar_mask_empty(mb));
        } else if constexpr (DROP) {
          // undropped P^T, and the keep bits from the dropped copy's zeros
          // (a kept entry whose P rounds to 0 has dS = 0 either way)
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld8(tP + 16 * c + 8, pp + 8 * c);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pd[8];
            tmem_ld8(tP + 16 * c, pd);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              keep[c >> 1] |= (((pd[e] & 0xFFFFu) != 0u ? 1u : 0u) | ((pd[e] >> 16) != 0u ? 2u : 0u))
                              << (16 * (c & 1) + 2 * e);
          }
        } else {
          tmem_ld32(tP, pp);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_p_read);
        if constexpr (!DQ && C::NSBUF == 2) mbar_arrive(bar_dq_free(buf));
        ok = __all_sync(0xffffffffu, mbar_wait(bar_dp_full, gi & 1, wc));
        if (!ok) break;
        tc_fence_after();
        const float* drow = dd_s + s * 128 + 64 * half;
        // Four chunks of 16 query columns; dS overwrites P in pp.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t dp[16];
          tmem_ld16(tDP + 16 * c, dp);
          tmem_wait_ld();
          if (c == 3) {
            // every dP^T column of this warp has been read
            tc_fence_before();
            mbar_arrive(bar_dp_free);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pp[8 * c + e]));
            const float2 dd = *reinterpret_cast<const float2*>(drow + 16 * c + 2 * e);
            float2 t;
            if constexpr (DROP) {
              // Z * s * dP - D
              const uint32_t kb = keep[c >> 1] >> (16 * (c & 1) + 2 * e);
              const float2 zs = make_float2(kb & 1u ? p.drop_scale : 0.f, kb & 2u ? p.drop_scale : 0.f);
              t = __ffma2_rn(make_float2(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])), zs,
                             make_float2(-dd.x, -dd.y));
            } else {
              t = __fadd2_rn(make_float2(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                             make_float2(-dd.x, -dd.y));
            }
            const float2 r = __fmul2_rn(pf, t);
            pp[8 * c + e] = pack_bf16x2(r.x, r.y);
          }
          if (c == 0 && gi > 0) {
            // The shared dS tile is still an operand of the previous tile's
            // dK and dQ MMAs until they complete (this tile's dP^T can
            // complete before them).
            ok = __all_sync(0xffffffffu,
                            (D == 64 || !DQ) ? mbar_wait(bar_qdo_empty(stg(gi - 1)), stg_par(gi - 1), wc)
                                    : mbar_wait(bar_dq_full((gi - 1) % C::NSBUF), ((gi - 1) / C::NSBUF) & 1, wc));
            if (!ok) break;
          }
          // dS into shared memory: row j of box `half`, 16-byte chunks 2c and
          // 2c+1, 128-byte swizzle (chunk ^ (row % 8)).
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int chunk = 2 * c + q;
            *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (j & 7)) << 4)) =
                make_uint4(pp[8 * c + 4 * q], pp[8 * c + 4 * q + 1], pp[8 * c + 4 * q + 2], pp[8 * c + 4 * q + 3]);
          }
        }
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_ds_full);
      }
    }
  } else if (DQ && warp < 20) {
    // ------------------------------------------------------------ dQ (WG-C)
    const int r = threadIdx.x - 512;         // query row in the tile == TMEM lane
    const int lead = 512;                    // thread that issues the bulk reduces
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    int gi = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const BwdItem I = bwd_item(p, item);
      for (int it = 0; it < I.n_it && ok; ++it, ++gi) {
        const int buf = gi % C::NSBUF;
        const int h = I.hkv * G + it / I.nq;
        const int q0 = (I.qt_begin + it % I.nq) * 128;
        const uint32_t tDQ = tmem + (C::NSBUF == 1 ? C::TM_DP : C::TM_S0 + 128 * buf) + lane_off;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_dq_full(buf), (gi / C::NSBUF) & 1, wc));
        // The four warps meet at named barriers below: after an expired wait
        // they still pass them, and all stop together at the end.
        if (ok) tc_fence_after();
        // Passes of BPP 32-column boxes: TMEM loads, then staging and bulk
        // reduce-adds; the columns are released after the last pass's
        // loads.  d = 64 takes one box per pass (fewer live registers, no
        // spills); d = 128 two, which releases its four boxes sooner.
        constexpr int BPP = (D == 64) ? 1 : 2;
#pragma unroll
        for (int pr = 0; pr < D / 32 / BPP; ++pr) {
          uint32_t v[BPP][32];
          if (ok) {
#pragma unroll
            for (int b = 0; b < BPP; ++b) tmem_ld32(tDQ + 32 * (pr * BPP + b), v[b]);
            tmem_wait_ld();
            if (pr + 1 == D / 32 / BPP) {
              tc_fence_before();
              mbar_arrive(bar_dq_free(buf));
            }
          } else {
#pragma unroll
            for (int b = 0; b < BPP; ++b)
#pragma unroll
              for (int i = 0; i < 32; ++i) v[b][i] = 0u;  // a stopped warp adds nothing
          }
#pragma unroll
          for (int b = 0; b < BPP; ++b) {
            const int bx = pr * BPP + b;
            // Before a staging box is refilled, the bulk reduce that last
            // read it must have finished reading.
            const uint32_t slot = C::OFF_DQS + (bx % C::NDQS) * C::BOX_BYTES;
            if (bx % C::NDQS == 0) {
              if (threadIdx.x == lead) bulk_wait_group_read0();
              named_bar_sync(2, 128);
            }
#pragma unroll
            for (int chunk = 0; chunk < 8; ++chunk) {
              *reinterpret_cast<float4*>(smem + slot + r * 128 + ((chunk ^ (r & 7)) << 4)) =
                  make_float4(__uint_as_float(v[b][4 * chunk]) * p.scale,
                              __uint_as_float(v[b][4 * chunk + 1]) * p.scale,
                              __uint_as_float(v[b][4 * chunk + 2]) * p.scale,
                              __uint_as_float(v[b][4 * chunk + 3]) * p.scale);
            }
            fence_proxy_async_smem();
            if (bx + 1 == D / 32 && threadIdx.x == lead) *stop_flag = *abort_flag;
            named_bar_sync(2, 128);
            if (threadIdx.x == lead && !*stop_flag) {
              tma_reduce_add_4d(&p.tm_dq, sbase + slot, bx * 32, h, q0, I.b);
              bulk_commit_group();
            }
          }
        }
        if (*stop_flag) {
          ok = false;
          break;
        }
      }
    }
    if (threadIdx.x == lead) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

static int bwd_setup() {
  const void* kernels[10] = {reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<64, false>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<64, true>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<128, false>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<128, true>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<64, false, true>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<128, false, true>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<64, false, false, false>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<64, true, false, false>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<128, false, false, false>),
                            reinterpret_cast<const void*>(fa_bwd_dkdv_kernel<128, true, false, false>)};
  const int bytes[10] = {BwdCfg<64>::SMEM_BYTES,
                         BwdCfg<64>::SMEM_BYTES,
                         BwdCfg<128>::SMEM_BYTES,
                         BwdCfg<128>::SMEM_BYTES,
                         BwdCfg<64, true>::SMEM_BYTES,
                         BwdCfg<128, true>::SMEM_BYTES,
                         BwdCfg<64, false, false>::SMEM_BYTES,
                         BwdCfg<64, false, false>::SMEM_BYTES,
                         BwdCfg<128, false, false>::SMEM_BYTES,
                         BwdCfg<128, false, false>::SMEM_BYTES};
  for (int i = 0; i < 10; ++i)
    if (cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize, bytes[i]) != cudaSuccess)
      return FA_ERR_CUDA;
  return FA_OK;
}

}  // namespace fa
