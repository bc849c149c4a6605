// fa_decode.cuh -- split-KV decode: one query token per sequence against a
// long KV cache.  The cache of every (sequence, KV head) is cut into chunks
// that separate thread blocks process (FlashDecoding, "FlashAttention"
// interview track, section "In practice"); each block writes its chunk's
// normalised output O_c and log-sum-exp LSE_c, and a second kernel merges
// them: LSE = log sum_c e^{LSE_c}, O = sum_c e^{LSE_c - LSE} O_c -- the same
// rescaling algebra as the online softmax of "Flash Attention: Why Memory
// Traffic, Not Compute, Is the Bottleneck", section "Softmax Looks Like an
// Obstacle".
//
// Decode reads every cached key and value once and does ~4*G FLOPs per
// cached bf16 element pair, so it is bound by HBM bandwidth ("Efficient
// attention: memory-bound", the decoding paragraph).  The kernel therefore
// uses CUDA cores (a GQA group has only G query rows, too few for a useful
// tensor-core tile) and spends its effort on keeping loads in flight: a
// producer warp streams 64-key K and V tiles with TMA into a ring of shared-
// memory stages while four compute warps consume them.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct DecodeParams {
  CUtensorMap tm_k;          // cache [B][Tk_max][Hkv][d], box {d, 1, 64, 1}, no swizzle
  CUtensorMap tm_v;
  const __nv_bfloat16* q;    // [B][Hq][d]
  const int* seqlens;        // [B]
  float* ws_o;               // [B][Hq][nchunk][d]
  float* ws_lse;             // [B][Hq][nchunk]
  __nv_bfloat16* o;          // [B][Hq][d]
  float* lse;                // [B][Hq]
  int B, Hq, Hkv, Tk_max, chunk, nchunk;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D, int G>
struct DecCfg {
  static constexpr int SUB = 64;                   // keys per TMA tile
  static constexpr int STAGE_BYTES = SUB * D * 2;
  static constexpr int NSTAGE = (D == 128) ? 4 : 8;
  static constexpr int LPK = D / 8;                // lanes per key row (16 bytes each)
  static constexpr int KPS = 32 / LPK;             // keys per warp step
  static constexpr int NWARP = 4;                  // compute warps
  static constexpr int THREADS = (NWARP + 1) * 32;
  static constexpr int MAX_CHUNK = 4096 / G;       // scores buffer: G * chunk floats
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_SCORE = NSTAGE * STAGE_BYTES;
  static constexpr int OFF_RED = OFF_SCORE + G * MAX_CHUNK * 4;      // [NWARP][G][D] fp32
  static constexpr int OFF_STAT = OFF_RED + NWARP * G * D * 4;       // m[G], l[G]
  static constexpr int OFF_BAR = OFF_STAT + 2 * G * 4;
  static constexpr int OFF_FLAG = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int SMEM_BYTES = OFF_FLAG + 16 + 128;
};

template <int D, int G>
__global__ void __launch_bounds__(DecCfg<D, G>::THREADS)
fa_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecCfg<D, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t sbase = smem_u32(smem);
  float* score = reinterpret_cast<float*>(smem + C::OFF_SCORE);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* stat = reinterpret_cast<float*>(smem + C::OFF_STAT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  auto bar_full = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
  auto bar_empty = [&](int s) { return sbase + C::OFF_BAR + 8u * (C::NSTAGE + s); };

  const int c = blockIdx.x;        // chunk index
  const int hkv = blockIdx.y;
  const int b = blockIdx.z;
  const int seqlen = p.seqlens[b];
  const int k0 = c * p.chunk;
  if (k0 >= seqlen) return;        // chunk past this sequence's end: nothing to do
  const int nkeys = min(p.chunk, seqlen - k0);
  const int nsub = (nkeys + C::SUB - 1) / C::SUB;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), C::NWARP);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == C::NWARP) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int t = 0; t < 2 * nsub && ok; ++t) {
        const int s = t % C::NSTAGE;
        const int round = t / C::NSTAGE;
        if (round > 0) ok = mbar_wait(bar_empty(s), (round - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_full(s), C::STAGE_BYTES);
        const int sub = t < nsub ? t : t - nsub;
        tma_load_4d(sbase + C::OFF_RING + s * C::STAGE_BYTES, t < nsub ? &p.tm_k : &p.tm_v,
                    bar_full(s), 0, hkv, k0 + sub * C::SUB, b);
        ++issued;
      }
      if (!ok)
        for (int t = max(0, issued - C::NSTAGE); t < issued; ++t)
          mbar_wait_drain(bar_full(t % C::NSTAGE), (t / C::NSTAGE) & 1, p.wait_limit_ns);
    }
    // the producer warp takes part in no named barrier below
    return;
  }

  // ------------------------------------------------------------ compute
  const int kl = lane / C::LPK;            // key slot within a warp step
  const int dl = (lane % C::LPK) * 8;      // first of this lane's 8 d-elements
  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + hkv * G + g) * D + dl);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      qf[g][2 * e] = f.x * p.scale_log2;
      qf[g][2 * e + 1] = f.y * p.scale_log2;
    }
  }

  bool ok = true;
  // Phase 1: scores (log2 units) for every key of the chunk.
  for (int t = 0; t < nsub; ++t) {
    const int s = t % C::NSTAGE;
    ok = __all_sync(0xffffffffu, mbar_wait(bar_full(s), (t / C::NSTAGE) & 1, wc));
    if (!ok) break;
    const uint8_t* stage = smem + C::OFF_RING + s * C::STAGE_BYTES;
#pragma unroll
    for (int st = 0; st < 16 / C::KPS; ++st) {
      const int kk = warp * 16 + st * C::KPS + kl;   // key within the 64-key tile
      const uint4 raw = *reinterpret_cast<const uint4*>(stage + kk * D * 2 + dl * 2);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float kf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        kf[2 * e] = f.x;
        kf[2 * e + 1] = f.y;
      }
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qf[g][e], kf[e], a);
        acc[g] = a;
      }
#pragma unroll
      for (int off = C::LPK / 2; off > 0; off >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], off);
      const int key = t * C::SUB + kk;               // key within the chunk
      if ((lane % C::LPK) == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) score[g * C::MAX_CHUNK + key] = key < nkeys ? acc[g] : -INFINITY;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty(s));
  }
  named_bar_sync(1, C::NWARP * 32);

  // Phase 2: softmax statistics per query head of the group; p = 2^{s - m}.
  if (ok) {
    for (int g = warp; g < G; g += C::NWARP) {
      float mx = -INFINITY;
      for (int k = lane; k < nkeys; k += 32) mx = fmaxf(mx, score[g * C::MAX_CHUNK + k]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      float sum = 0.f;
      for (int k = lane; k < nsub * C::SUB; k += 32) {
        const float e = k < nkeys ? ex2_approx(score[g * C::MAX_CHUNK + k] - mx) : 0.f;
        score[g * C::MAX_CHUNK + k] = e;
        sum += e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        stat[g] = mx;
        stat[G + g] = sum;
      }
    }
  }
  named_bar_sync(1, C::NWARP * 32);

  // Phase 3: O_c = sum_k p_k V_k over the chunk's V tiles.
  float acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  for (int t = nsub; t < 2 * nsub && ok; ++t) {
    const int s = t % C::NSTAGE;
    ok = __all_sync(0xffffffffu, mbar_wait(bar_full(s), (t / C::NSTAGE) & 1, wc));
    if (!ok) break;
    const uint8_t* stage = smem + C::OFF_RING + s * C::STAGE_BYTES;
#pragma unroll
    for (int st = 0; st < 16 / C::KPS; ++st) {
      const int kk = warp * 16 + st * C::KPS + kl;
      const int key = (t - nsub) * C::SUB + kk;
      const uint4 raw = *reinterpret_cast<const uint4*>(stage + kk * D * 2 + dl * 2);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float vf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        vf[2 * e] = f.x;
        vf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pg = score[g * C::MAX_CHUNK + key];   // 0 for keys past the end
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty(s));
  }
  // Sum the key slots of the warp, then the warps, through shared memory.
#pragma unroll
  for (int off = 16; off >= C::LPK; off >>= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], off);
  if (lane < C::LPK) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[(warp * G + g) * D + dl + e] = acc[g][e];
  }
  named_bar_sync(1, C::NWARP * 32);
  if (!ok) return;
  for (int i = threadIdx.x; i < G * D; i += C::NWARP * 32) {
    const int g = i / D, dd = i % D;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < C::NWARP; ++w) v += red[(w * G + g) * D + dd];
    const int h = hkv * G + g;
    p.ws_o[(((size_t)b * p.Hq + h) * p.nchunk + c) * D + dd] = v / stat[G + g];
  }
  if (threadIdx.x < G) {
    const int g = threadIdx.x;
    const int h = hkv * G + g;
    // natural-log LSE of the chunk: (m + log2 l) * ln 2
    p.ws_lse[((size_t)b * p.Hq + h) * p.nchunk + c] = (stat[g] + log2f(stat[G + g])) * 0.69314718055994531f;
  }
}

// One warp per (sequence, query head): merge the chunk partials by LSE.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq;
  const int seqlen = p.seqlens[b];
  const int nch = (seqlen + p.chunk - 1) / p.chunk;
  const float* lse_c = p.ws_lse + (size_t)gw * p.nchunk;
  const float* o_c = p.ws_o + (size_t)gw * p.nchunk * D;
  constexpr int E = D / 32;  // elements per lane
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  if (nch == 0) {
    if (lane == 0) p.lse[gw] = -INFINITY;
  } else {
    float mx = -INFINITY;
    for (int c = lane; c < nch; c += 32) mx = fmaxf(mx, lse_c[c]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
    for (int c = lane; c < nch; c += 32) sum += ex2_approx((lse_c[c] - mx) * 1.4426950408889634f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float lse = mx + logf(sum);
    for (int c = 0; c < nch; ++c) {
      const float wgt = ex2_approx((lse_c[c] - lse) * 1.4426950408889634f);
      const float* src = o_c + (size_t)c * D + lane * E;
      if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
        acc[2] = fmaf(wgt, v.z, acc[2]);
        acc[3] = fmaf(wgt, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
      }
    }
    if (lane == 0) p.lse[gw] = lse;
  }
  __nv_bfloat16* dst = p.o + (size_t)gw * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2)
    *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
}

}  // namespace fa
