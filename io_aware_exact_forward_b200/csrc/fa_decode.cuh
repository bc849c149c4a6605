// fa_decode.cuh -- split-KV decode: one query token per sequence against a
// long KV cache.  The cache of every (sequence, KV head) is cut into chunks
// that separate work items process (FlashDecoding, "FlashAttention"
// interview track, section "In practice"); each item writes its chunk's
// normalised output O_c and log-sum-exp LSE_c, and a second kernel merges
// them:
//   LSE = log sum_c e^{LSE_c},  O = sum_c e^{LSE_c - LSE} O_c
// -- the same rescaling algebra as the online softmax of "Flash Attention:
// Why Memory Traffic, Not Compute, Is the Bottleneck", section "Softmax
// Looks Like an Obstacle".
//
// Decode reads every cached key and value once and does ~4*G FLOPs per
// cached bf16 element pair, so it is bound by HBM bandwidth ("Efficient
// attention: memory-bound", the decoding paragraph).  The kernel is built to
// keep loads in flight and to spend little issue time per byte:
//   * persistent CTAs (two per SM); a producer warp streams 64-key K and V
//     tiles (K_0, V_0, K_1, V_1, ...) with TMA and the 128-byte swizzle into a
//     ring of shared-memory stages, continuously across work items;
//   * four compute warps, each owning 16 keys of every tile, run the dot
//     products on the tensor cores with mma.sync (the G query rows of a GQA
//     group padded to 16), keep an online softmax of their keys, and merge
//     with the other warps by log-sum-exp at the end of the chunk.  A group
//     has only G = 4 rows, far too few for a tcgen05 tile; mma.sync with
//     padding costs a few instructions per 16 keys, so issue time stays far
//     below the memory time.
// Merging the chunks inside the split kernel (the last item of a sequence
// to finish merging all of them) was measured 2.7x slower than the
// separate merge kernel: the merging CTA stops streaming.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct DecodeParams {
  CUtensorMap tm_k;          // cache [B][Tk_max][Hkv][d], box {64, 1, 64, 1}, 128-byte swizzle
  CUtensorMap tm_v;
  const __nv_bfloat16* q;    // [B][Hq][d]
  const int* seqlens;        // [B]
  float* ws_o;               // [B][Hq][nchunk][d]
  float* ws_lse;             // [B][Hq][nchunk]
  __nv_bfloat16* o;          // [B][Hq][d]
  float* o32;                // non-null: O goes here in fp32 [B][Hq][d] instead of to `o`
  float* lse;                // [B][Hq]
  int B, Hq, Hkv, Tk_max, chunk, nchunk;
  int n_items;               // B * Hkv * nchunk (items past a sequence's end are skipped)
  int window;                // > 0: the query sees only the last `window` keys of its sequence
  float scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D, int G>
struct DecCfg {
  static constexpr int SUB = 64;                   // keys per TMA tile
  static constexpr int NBOX = D / 64;              // 64-column swizzle boxes per tile
  static constexpr int BOX_BYTES = SUB * 128;
  static constexpr int STAGE_BYTES = NBOX * BOX_BYTES;
  static constexpr int NSTAGE = (D == 128) ? (G >= 8 ? 5 : 6) : 10;  // two CTAs per SM
  static constexpr int NWARP = 4;                  // compute warps, 16 keys of each tile each
  static constexpr int THREADS = (NWARP + 1) * 32;
  static constexpr int SEQ_CACHE = 1024;           // seqlens cached in shared memory
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int Q_STRIDE = (Q_BYTES + 127) / 128 * 128;
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_Q = NSTAGE * STAGE_BYTES;                 // 2 stages
  static constexpr int OFF_SEQ = OFF_Q + 2 * Q_STRIDE;
  static constexpr int OFF_MRG = OFF_SEQ + SEQ_CACHE * 4;            // [NWARP][G][D] fp32
  static constexpr int OFF_ML = OFF_MRG + NWARP * G * D * 4;         // m, l: [NWARP][G] each
  static constexpr int OFF_BAR = OFF_ML + 2 * NWARP * G * 4;
  static constexpr int NBAR = 2 * NSTAGE + 4;
  static constexpr int OFF_FLAG = OFF_BAR + NBAR * 8;                // abort, stop flags
  static constexpr int SMEM_BYTES = OFF_FLAG + 16 + 1024;            // + alignment slack
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.x4.m8n8.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.x4.trans.m8n8.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D(16x8 fp32) += A(16x16 bf16) * B(16x8 bf16)
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `ch` (0 .. D/8-1) of row `key` in a stage made
// of 64-column boxes with the 128-byte swizzle (chunk ^ row % 8).
__device__ __forceinline__ uint32_t swz_off(int key, int ch) {
  return (uint32_t)((ch >> 3) * 64 * 128 + key * 128 + (((ch & 7) ^ (key & 7)) << 4));
}

// A sequence length as every decode kernel reads it: clamped to
// [0, Tk_max], so that a length outside the cache's extent can neither send
// the split kernel past its chunk count nor the merge past the partials the
// split kernel wrote.
__device__ __forceinline__ int clamp_seqlen(const DecodeParams& p, int n) { return min(max(n, 0), p.Tk_max); }

// Item k covers chunk k % nchunk of (sequence, KV head) k / nchunk.
template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D, G>::THREADS)
fa_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecCfg<D, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int* seq_s = reinterpret_cast<int*>(smem + C::OFF_SEQ);
  float* mrg = reinterpret_cast<float*>(smem + C::OFF_MRG);
  float* m_s = reinterpret_cast<float*>(smem + C::OFF_ML);
  float* l_s = m_s + C::NWARP * G;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  volatile int* stop_flag = abort_flag + 1;
  auto bar_full = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
  auto bar_empty = [&](int s) { return sbase + C::OFF_BAR + 8u * (C::NSTAGE + s); };
  auto bar_qfull = [&](int s) { return sbase + C::OFF_BAR + 8u * (2 * C::NSTAGE + s); };
  auto bar_qempty = [&](int s) { return sbase + C::OFF_BAR + 8u * (2 * C::NSTAGE + 2 + s); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.wait_limit_ns};

  for (int i = threadIdx.x; i < min(p.B, C::SEQ_CACHE); i += blockDim.x) seq_s[i] = clamp_seqlen(p, p.seqlens[i]);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *stop_flag = 0;
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), C::NWARP);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), C::NWARP);
    }
    fence_barrier_init();
  }
  __syncthreads();
  auto seqlen_of = [&](int b) { return b < C::SEQ_CACHE ? seq_s[b] : clamp_seqlen(p, p.seqlens[b]); };

  if (warp == C::NWARP) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      bool ok = true;
      int t = 0, qi = 0;  // ring slot counter and item counter, continuous across items
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const int c = item % p.nchunk;
        const int bh = item / p.nchunk;
        const int b = bh / p.Hkv, hkv = bh % p.Hkv;
        const int k0 = c * p.chunk;
        const int seqlen = seqlen_of(b);
        if (k0 >= seqlen || (p.window > 0 && k0 + p.chunk <= seqlen - p.window)) continue;
        const int nsub = (min(p.chunk, seqlen - k0) + C::SUB - 1) / C::SUB;
        // the G query rows of the group are contiguous: one bulk copy
        const int qs = qi & 1;
        if (qi >= 2) ok = mbar_wait(bar_qempty(qs), ((qi >> 1) - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_qfull(qs), C::Q_BYTES);
        bulk_load(sbase + C::OFF_Q + qs * C::Q_STRIDE, p.q + ((size_t)b * p.Hq + hkv * G) * D, C::Q_BYTES,
                  bar_qfull(qs));
        ++qi;
        // K_0, V_0, K_1, V_1, ... -- the order the compute warps consume
        for (int i = 0; i < 2 * nsub && ok; ++i, ++t) {
          const int s = t % C::NSTAGE;
          const int round = t / C::NSTAGE;
          if (round > 0) ok = mbar_wait(bar_empty(s), (round - 1) & 1, wc);
          if (!ok) break;
          mbar_arrive_expect_tx(bar_full(s), C::STAGE_BYTES);
          for (int kb = 0; kb < C::NBOX; ++kb)
            tma_load_4d(sbase + C::OFF_RING + s * C::STAGE_BYTES + kb * C::BOX_BYTES, (i & 1) ? &p.tm_v : &p.tm_k,
                        bar_full(s), kb * 64, hkv, k0 + (i >> 1) * C::SUB, b);
        }
      }
      if (!ok) {
        for (int k = max(0, t - C::NSTAGE); k < t; ++k)
          mbar_wait_drain(bar_full(k % C::NSTAGE), (k / C::NSTAGE) & 1, p.wait_limit_ns);
        for (int k = max(0, qi - 2); k < qi; ++k) mbar_wait_drain(bar_qfull(k & 1), (k >> 1) & 1, p.wait_limit_ns);
      }
    }
    // the producer warp takes part in no named barrier below
    return;
  }

  // ------------------------------------------------------------ compute
  // mma.sync fragment coordinates: row g = lane / 4 (query head of the group
  // when g < G; rows G..15 are padding), column pair 2t, 2t+1 with t = lane % 4.
  const int g = lane >> 2, t4 = lane & 3;
  const bool real_row = g < G;
  const int kw = warp * 16;                // this warp's 16 keys of every tile
  bool ok = true;
  int t = 0, qi = 0;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    const int c = item % p.nchunk;
    const int bh = item / p.nchunk;
    const int b = bh / p.Hkv, hkv = bh % p.Hkv;
    const int k0 = c * p.chunk;
    const int seqlen = seqlen_of(b);
    if (k0 >= seqlen || (p.window > 0 && k0 + p.chunk <= seqlen - p.window)) continue;
    const int nkeys = min(p.chunk, seqlen - k0);
    // keys of the chunk before this bound are outside the window
    const int klo = p.window > 0 ? seqlen - p.window - k0 : -(1 << 30);
    const int nsub = (nkeys + C::SUB - 1) / C::SUB;

    // Q as the A operand (rows >= G are zero); scaling is applied to the
    // fp32 scores, so the bf16 inputs enter the MMA unrounded.
    uint32_t qa[D / 16][2];
    {
      const int qs = qi & 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_qfull(qs), (qi >> 1) & 1, wc));
      const uint32_t* qrow =
          reinterpret_cast<const uint32_t*>(smem + C::OFF_Q + qs * C::Q_STRIDE + (real_row ? g : 0) * D * 2);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qa[ks][0] = real_row ? qrow[ks * 8 + t4] : 0u;       // cols 16ks + 2t, +1
        qa[ks][1] = real_row ? qrow[ks * 8 + 4 + t4] : 0u;   // cols 16ks + 8 + 2t, +1
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_qempty(qs));
      ++qi;
    }

    // Online softmax over this warp's keys of the chunk (log2 units).
    float m_run = -INFINITY, l_part = 0.f;
    float oacc[D / 8][4];
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[nb][e] = 0.f;

    for (int i = 0; i < nsub; ++i) {
      // ---- K tile: scores of keys kw .. kw+15 of this 64-key tile
      const int sK = t % C::NSTAGE;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_full(sK), (t / C::NSTAGE) & 1, wc));
      ++t;
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) {
        const uint32_t st = sbase + C::OFF_RING + sK * C::STAGE_BYTES;
        // matrices: (keys +0..7, cols +0..7), (+0..7, +8..15), (+8..15, +0..7), (+8..15, +8..15)
        const int mrow = kw + ((lane >> 4) << 3) + (lane & 7);
        const int mcol = (lane >> 3) & 1;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(st + swz_off(mrow, 2 * ks + mcol), b0, b1, b2, b3);
          mma_16816(s0, qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
          mma_16816(s1, qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(sK));
      // this lane's keys: kw + 2t, +1 (s0) and kw + 8 + 2t, +1 (s1)
      const int kb0 = i * C::SUB + kw + 2 * t4;
      float sc[4] = {s0[0], s0[1], s1[0], s1[1]};
      const int kk[4] = {kb0, kb0 + 1, kb0 + 8, kb0 + 9};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sc[e] = (kk[e] < nkeys && kk[e] >= klo && real_row) ? sc[e] * p.scale_log2 : -INFINITY;
      float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      // Lazy rescale: move the reference only when the maximum grew by more
      // than the threshold; l and O always share the reference.
      if (mx > m_run + C::RESCALE_THRESHOLD || (m_run == -INFINITY && mx != -INFINITY)) {
        const float alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mx);
        l_part *= alpha;
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb) {
          oacc[nb][0] *= alpha;
          oacc[nb][1] *= alpha;
        }
        m_run = mx;
      }
      const float ref = (m_run == -INFINITY) ? 0.f : m_run;
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pv[e] = ex2_approx(sc[e] - ref);
        l_part += pv[e];
      }
      const uint32_t pa0 = pack_bf16x2(pv[0], pv[1]);   // row g, keys kw + 2t, +1
      const uint32_t pa2 = pack_bf16x2(pv[2], pv[3]);   // row g, keys kw + 8 + 2t, +1

      // ---- V tile: O += P V over the same 16 keys
      const int sV = t % C::NSTAGE;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_full(sV), (t / C::NSTAGE) & 1, wc));
      ++t;
      if (ok) {
        const uint32_t st = sbase + C::OFF_RING + sV * C::STAGE_BYTES;
        // transposed matrices: (keys +0..7, d 8nb..), (keys +8..15, d 8nb..),
        // (keys +0..7, d 8nb+8..), (keys +8..15, d 8nb+8..)
        const int vrow = kw + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int vcol = lane >> 4;
#pragma unroll
        for (int nb = 0; nb < D / 8; nb += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(st + swz_off(vrow, nb + vcol), b0, b1, b2, b3);
          mma_16816(oacc[nb], pa0, 0u, pa2, 0u, b0, b1);
          mma_16816(oacc[nb + 1], pa0, 0u, pa2, 0u, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(sV));
    }

    // ---- merge the four warps by log-sum-exp
    float l_row = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_row += __shfl_xor_sync(0xffffffffu, l_row, 2);
    if (real_row) {
      if (t4 == 0) {
        m_s[warp * G + g] = m_run;
        l_s[warp * G + g] = l_row;
      }
#pragma unroll
      for (int nb = 0; nb < D / 8; ++nb)
        *reinterpret_cast<float2*>(&mrg[(warp * G + g) * D + nb * 8 + 2 * t4]) =
            make_float2(oacc[nb][0], oacc[nb][1]);
    }
    named_bar_sync(1, C::NWARP * 32);
    for (int idx = threadIdx.x; idx < G * D; idx += C::NWARP * 32) {
      const int gg = idx / D, dd = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::NWARP; ++w) M = fmaxf(M, m_s[w * G + gg]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < C::NWARP; ++w) {
        const float mw = m_s[w * G + gg];
        const float f = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
        L = fmaf(f, l_s[w * G + gg], L);
        O = fmaf(f, mrg[(w * G + gg) * D + dd], O);
      }
      const size_t row = (size_t)b * p.Hq + hkv * G + gg;
      p.ws_o[(row * p.nchunk + c) * D + dd] = O / L;
      if (dd == 0) p.ws_lse[row * p.nchunk + c] = (M + log2f(L)) * 0.69314718055994531f;
    }
    // The merge scratch is reused by the next item only after this barrier.
    // After an expired wait every compute warp has still passed the same
    // named barriers; thread 0 samples the abort flag before the barrier so
    // that all of them stop here together.
    if (threadIdx.x == 0) *stop_flag = *abort_flag;
    named_bar_sync(1, C::NWARP * 32);
    if (*stop_flag) break;
  }
}

// One output row of D values, D/32 consecutive ones per lane: bf16 into `o`,
// or fp32 into `o32` when the caller asked for partials to merge later.
template <int D>
__device__ __forceinline__ void store_row(const DecodeParams& p, int row, int lane, const float (&acc)[D / 32]) {
  constexpr int E = D / 32;
  if (p.o32) {
    float* dst = p.o32 + (size_t)row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<float2*>(dst + e) = make_float2(acc[e], acc[e + 1]);
  } else {
    __nv_bfloat16* dst = p.o + (size_t)row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
  }
}

// Separate merge of the chunk partials: one warp per (sequence, query head).
template <int D>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq;
  const int seqlen = clamp_seqlen(p, p.seqlens[b]);
  const int nch = (seqlen + p.chunk - 1) / p.chunk;
  if (nch == 0) return;  // written by fa_decode_empty_kernel
  // with a window the chunks before the first visible key were skipped
  const int c_lo = p.window > 0 ? max(0, seqlen - p.window) / p.chunk : 0;
  constexpr int E = D / 32;
  const float* lse_c = p.ws_lse + (size_t)gw * p.nchunk;
  const float* o_c = p.ws_o + (size_t)gw * p.nchunk * D;
  float mx = -INFINITY;
  for (int cc = c_lo + lane; cc < nch; cc += 32) mx = fmaxf(mx, lse_c[cc]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  for (int cc = c_lo + lane; cc < nch; cc += 32) sum += ex2_approx((lse_c[cc] - mx) * 1.4426950408889634f);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse = mx + logf(sum);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  int cc = c_lo;
  for (; cc + 4 <= nch; cc += 4) {
    float wgt[4], vals[4][E];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      wgt[u] = lse_c[cc + u];
#pragma unroll
      for (int e = 0; e < E; ++e) vals[u][e] = o_c[(size_t)(cc + u) * D + lane * E + e];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float w = ex2_approx((wgt[u] - lse) * 1.4426950408889634f);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(w, vals[u][e], acc[e]);
    }
  }
  for (; cc < nch; ++cc) {
    const float w = ex2_approx((lse_c[cc] - lse) * 1.4426950408889634f);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(w, o_c[(size_t)cc * D + lane * E + e], acc[e]);
  }
  if (lane == 0) p.lse[gw] = lse;
  store_row<D>(p, gw, lane, acc);
}

// Sequences with no cached key (seqlen <= 0) get O = 0 and LSE = -inf; every
// other (sequence, head) is written by the merge kernel.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_empty_kernel(const __grid_constant__ DecodeParams p) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq;
  if (clamp_seqlen(p, p.seqlens[b]) > 0) return;
  float zero[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) zero[e] = 0.f;
  store_row<D>(p, gw, lane, zero);
  if (lane == 0) p.lse[gw] = -INFINITY;
}

// Merge of per-device partials (context-parallel decode): device r decoded
// its own share of every sequence's keys into a normalised fp32 O_r and
// LSE_r; the full result is
//   LSE = log sum_r e^{LSE_r},  O = sum_r e^{LSE_r - LSE} O_r,
// the chunk merge above with devices in place of chunks.  A device whose
// share of a sequence is empty contributes LSE_r = -inf and is skipped; a
// row no device saw a key of gets O = 0 and LSE = -inf.
struct MergeParams {
  const float* o_parts;    // [R] blocks of [rows][d], `o_stride` floats apart
  const float* lse_parts;  // [R] blocks of [rows], `lse_stride` floats apart
  size_t o_stride, lse_stride;
  __nv_bfloat16* o;        // [rows][d]
  float* lse;              // [rows]
  int R, rows;
};

template <int D>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const __grid_constant__ MergeParams p) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  constexpr int E = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  float mx = -INFINITY;
  for (int r = lane; r < p.R; r += 32) mx = fmaxf(mx, p.lse_parts[(size_t)r * p.lse_stride + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (mx == -INFINITY) {
    __nv_bfloat16* dst = p.o + (size_t)row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = 0u;
    if (lane == 0) p.lse[row] = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int r = lane; r < p.R; r += 32) sum += ex2_approx((p.lse_parts[(size_t)r * p.lse_stride + row] - mx) * kLog2e);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse = mx + logf(sum);
  for (int r = 0; r < p.R; ++r) {
    const float l = p.lse_parts[(size_t)r * p.lse_stride + row];
    if (l == -INFINITY) continue;  // same value in every lane: no divergence
    const float w = ex2_approx((l - lse) * kLog2e);
    const float* src = p.o_parts + (size_t)r * p.o_stride + (size_t)row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float2 x = *reinterpret_cast<const float2*>(src + e);
      acc[e] = fmaf(w, x.x, acc[e]);
      acc[e + 1] = fmaf(w, x.y, acc[e + 1]);
    }
  }
  if (lane == 0) p.lse[row] = lse;
  __nv_bfloat16* dst = p.o + (size_t)row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
}

}  // namespace fa
