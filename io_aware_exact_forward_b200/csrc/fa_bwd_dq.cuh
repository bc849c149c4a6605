// fa_bwd_dq.cuh -- the backward's dQ as a pass of its own: one work item per
// (128-query tile, query head, batch), which walks the KV tiles its rows see
// and recomputes S and dP for them ("FlashAttention" interview track,
// follow-up on recomputation; the products of "Efficient attention:
// memory-bound", section "Real code moves even more"):
//   S  = Q K_j^T,  dP = dO V_j^T                 (SS MMAs into tensor memory)
//   P  = 2^{S*scale*log2e - LSE2},  dS = P*(dP - D)   (compute warps, dS as
//        bf16 into tensor memory)
//   dQ += dS K_j                                  (TS MMA, fp32 in tensor memory)
// and writes dQ = scale * dQ once, at the end of the item.  Each dQ row is
// summed in one fixed order, so the result is the same from run to run, and
// no fp32 accumulator goes through global memory.  It is the deterministic
// backward's dQ (fa_backward_deterministic, with the dK/dV kernel built
// without dQ); the default backward keeps the fused dQ, which measured faster:
// this pass issues 24 MMAs per tile against the 16 of the forward's pair of
// products, and the single issuing thread, sharing its sub-partition with two
// compute warps, takes ~160 cycles per MMA.
//
// Warp roles (320 threads): 0-7 compute (two warps per TMEM lane quarter,
// one per half of the 128 key columns; one query row per lane), 8 MMA issuer,
// 9 TMA producer.  Tensor memory: S [0,128), dP [128,256), dQ [256,256+d),
// two dS buffers (bf16 pairs) [256+d, 384+d).  Shared memory: Q and dO (one tile each)
// and a ring of two (K_j, V_j) stages.  S_{j+1} and dP_{j+1} are issued as
// soon as the compute warps have loaded S_j and dP_j, so the products of the
// next tile overlap the exponentials of this one.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct DqParams {
  CUtensorMap tm_q;    // [B][Tq][Hq][d] bf16, box {64,1,128,1}, 128-byte swizzle
  CUtensorMap tm_do;
  CUtensorMap tm_k;    // [B][Tk][Hkv][d]
  CUtensorMap tm_v;
  const float* lse2;   // [B][Hq][Tq_pad]: LSE in log2 units (+inf: the row saw no key)
  const float* Dv;     // [B][Hq][Tq_pad]: D_i = sum_c dO_ic O_ic
  float* dq_acc;       // fp32 [B][Tq][Hq][d], written when dq is null
  __nv_bfloat16* dq;   // bf16 [B][Tq][Hq][d], or null
  int B, Hq, Hkv, Tq, Tk, causal;
  int window;          // > 0: sliding window of that many keys (implies causal)
  int Tq_pad;
  float scale, scale_log2;
  int n_qt;            // ceil(Tq / 128)
  int n_items;         // B * Hq * n_qt
  unsigned long long wait_limit_ns;
};

template <int D>
struct DqCfg {
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = 128 * 128;
  static constexpr int TILE = NBOX * BOX_BYTES;   // 128 rows x D bf16
  static constexpr int NST = 2;                   // (K, V) stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  // qdo_full, kv_full[NST], kv_empty[NST], s_full, s_free, ds_full[2],
  // ds_free[2], dq_done, mma_done
  static constexpr int NBAR = 1 + 2 * NST + 8;
  static constexpr int OFF_BAR = OFF_RING + NST * 2 * TILE;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // tmem base (u32), abort flag (int)
  // + alignment slack; at least 120 KB, so that two CTAs never share an SM
  // (each allocates all 512 tensor-memory columns)
  static constexpr int SMEM_BYTES = (OFF_MISC + 16 + 1024) > 122880 ? (OFF_MISC + 16 + 1024) : 122880;
  static constexpr int THREADS = 320;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_S = 0;
  static constexpr int TM_DP = 128;
  static constexpr int TM_DQ = 256;
  static constexpr int TM_DS = 256 + D;            // two dS buffers of 64 columns
  static constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 0, 1);   // dS from TMEM, K MN-major
  static_assert(TM_DS + 128 <= TMEM_COLS, "tensor memory overflow");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
};

// One work item: query tile [q0, q0 + 128) of head h of batch b against KV
// tiles kt0 .. kt0 + n_kv - 1.
struct DqItem {
  int b, h, hkv, q0, kt0, n_kv;
};

__device__ __forceinline__ DqItem dq_item(const DqParams& p, int item) {
  DqItem it;
  // The query tiles of one (batch, head) are adjacent in item order, so
  // the CTAs running at one time share that head's K and V through L2
  // (and the heads of a GQA group, adjacent too, share them as well);
  // within a head the heaviest causal tile (the last one) comes first.
  const int bh = item / p.n_qt;
  const int qt = p.causal ? p.n_qt - 1 - item % p.n_qt : item % p.n_qt;
  it.b = bh / p.Hq;
  it.h = bh % p.Hq;
  it.hkv = it.h / (p.Hq / p.Hkv);
  it.q0 = qt * 128;
  const int n_kv_all = (p.Tk + 127) / 128;
  it.kt0 = 0;
  int kt_end = n_kv_all;
  if (p.causal) {
    const int last_row = min(it.q0 + 128, p.Tq) - 1;
    const int kmax = last_row + (p.Tk - p.Tq);  // last key any row of the tile sees
    kt_end = kmax < 0 ? 0 : min(n_kv_all, kmax / 128 + 1);
    if (p.window > 0) {
      const int kmin = it.q0 + (p.Tk - p.Tq) - p.window + 1;  // first key of the first row's window
      it.kt0 = kmin <= 0 ? 0 : min(kt_end, kmin / 128);
    }
  }
  it.n_kv = kt_end - it.kt0;
  return it;
}

template <int D, bool WIN>
__global__ void __launch_bounds__(320, 1) fa_bwd_dq_kernel(const __grid_constant__ DqParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_qdo_full = bar0;
  auto bar_kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_kv_empty = [&](int s) { return bar0 + 8u * (1 + C::NST + s); };
  const uint32_t bar_s_full = bar0 + 8u * (1 + 2 * C::NST);   // S_j and dP_j in tensor memory
  const uint32_t bar_s_free = bar0 + 8u * (2 + 2 * C::NST);   // the compute warps hold them
  // dS of tile j in buffer j & 1; a barrier pair per buffer, so that no
  // wait is ever for a phase two behind
  auto bar_ds_full = [&](int b) { return bar0 + 8u * (3 + 2 * C::NST + b); };  // dS_j in tensor memory
  auto bar_ds_free = [&](int b) { return bar0 + 8u * (5 + 2 * C::NST + b); };  // dQ += dS_j K_j has read it
  const uint32_t bar_dq_done = bar0 + 8u * (7 + 2 * C::NST);
  const uint32_t bar_mma_done = bar0 + 8u * (8 + 2 * C::NST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t aQ = sbase + C::OFF_Q, aDO = sbase + C::OFF_DO;
  auto aK = [&](int s) { return sbase + C::OFF_RING + (2 * s) * C::TILE; };
  auto aV = [&](int s) { return sbase + C::OFF_RING + (2 * s + 1) * C::TILE; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.wait_limit_ns};
  const DqItem it = dq_item(p, blockIdx.x);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_qdo_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 256);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_ds_full(b), 256);
      mbar_init(bar_ds_free(b), 1);
    }
    mbar_init(bar_dq_done, 1);
    mbar_init(bar_mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && it.n_kv > 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_do);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar_qdo_full, 2 * C::TILE);
      for (int kb = 0; kb < C::NBOX; ++kb) {
        tma_load_4d(aQ + kb * C::BOX_BYTES, &p.tm_q, bar_qdo_full, kb * 64, it.h, it.q0, it.b);
        tma_load_4d(aDO + kb * C::BOX_BYTES, &p.tm_do, bar_qdo_full, kb * 64, it.h, it.q0, it.b);
      }
      bool ok = true;
      int j = 0;
      for (; j < it.n_kv; ++j) {
        const int s = j % C::NST;
        if (j >= C::NST) ok = mbar_wait(bar_kv_empty(s), ((j / C::NST) - 1) & 1, wc);
        if (!ok) break;
        const int k0 = (it.kt0 + j) * 128;
        mbar_arrive_expect_tx(bar_kv_full(s), 2 * C::TILE);
        for (int kb = 0; kb < C::NBOX; ++kb) {
          tma_load_4d(aK(s) + kb * C::BOX_BYTES, &p.tm_k, bar_kv_full(s), kb * 64, it.hkv, k0, it.b);
          tma_load_4d(aV(s) + kb * C::BOX_BYTES, &p.tm_v, bar_kv_full(s), kb * 64, it.hkv, k0, it.b);
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        mbar_wait_drain(bar_qdo_full, 0, p.wait_limit_ns);
        for (int k = max(0, j - C::NST); k < j; ++k)
          mbar_wait_drain(bar_kv_full(k % C::NST), (k / C::NST) & 1, p.wait_limit_ns);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tmem + C::TM_S, tDP = tmem + C::TM_DP, tDQ = tmem + C::TM_DQ, tDS = tmem + C::TM_DS;
      constexpr uint32_t HI = sw128_hi(1024);
      auto kdesc = [&](uint32_t base, int k) {  // K-major tile, k-th 16-element slice of d
        return sw128_desc(sw128_lo(base, 16) + (((k >> 2) * C::BOX_BYTES + (k & 3) * 32) >> 4), HI);
      };
      auto mndesc = [&](uint32_t base, int k) {  // MN-major view (keys down), k-th 16-key slice
        return sw128_desc(sw128_lo(base, C::BOX_BYTES) + ((k * 16 * 128) >> 4), HI);
      };
      bool ok = true;
      if (it.n_kv > 0) {
        ok = mbar_wait(bar_qdo_full, 0, wc);
        for (int j = 0; j <= it.n_kv && ok; ++j) {
          if (j < it.n_kv) {
            // S_j and dP_j once K_j, V_j have landed and the compute warps
            // have loaded S_{j-1} and dP_{j-1}
            const int s = j % C::NST;
            ok = mbar_wait(bar_kv_full(s), (j / C::NST) & 1, wc);
            if (ok && j > 0) ok = mbar_wait(bar_s_free, (j - 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k) mma_ss(tS, kdesc(aQ, k), kdesc(aK(s), k), C::IDESC_SS, k > 0);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) mma_ss(tDP, kdesc(aDO, k), kdesc(aV(s), k), C::IDESC_SS, k > 0);
            mma_commit(bar_s_full);
          }
          if (j > 0) {
            // dQ += dS_{j-1} K_{j-1}, then the stage and the dS columns are free
            const int s = (j - 1) % C::NST;
            ok = mbar_wait(bar_ds_full((j - 1) & 1), ((j - 1) >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ts(tDQ, tDS + 64 * ((j - 1) & 1) + 8 * k, mndesc(aK(s), k), C::IDESC_DQ, j > 1 || k > 0);
            mma_commit(bar_ds_free((j - 1) & 1));
            mma_commit(bar_kv_empty(s));
          }
        }
        if (ok) mma_commit(bar_dq_done);
      }
      // Wait until every MMA issued above has completed before teardown.
      mma_commit(bar_mma_done);
      mbar_wait_drain(bar_mma_done, 0, p.wait_limit_ns);
    }
  } else {
    // ------------------------------------------------------------ compute
    const int lq = warp & 3, hc = warp >> 2;   // TMEM lane quarter, key half
    const int r = lq * 32 + lane;              // query row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(lq * 32) << 16;
    const int row = it.q0 + r;
    const size_t rb = ((size_t)it.b * p.Hq + it.h) * p.Tq_pad + row;  // row < Tq_pad
    const float lse2 = p.lse2[rb];
    const float dd = p.Dv[rb];
    // keys < key_limit are visible to this row, and, with a window, keys >= key_lo
    const int key_limit = p.causal ? min(p.Tk, row + (p.Tk - p.Tq) + 1) : p.Tk;
    const int key_lo = WIN ? row + (p.Tk - p.Tq) - p.window + 1 : 0;
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 nl2 = make_float2(-lse2, -lse2);
    const float2 ndd = make_float2(-dd, -dd);
    const uint32_t tS = tmem + C::TM_S + lane_off + 64 * hc;
    const uint32_t tDP = tmem + C::TM_DP + lane_off + 64 * hc;
    const uint32_t tDS = tmem + C::TM_DS + lane_off + 32 * hc;
    bool ok = true;
    for (int j = 0; j < it.n_kv && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full, j & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld32(tS, sv);
      tmem_ld32(tS + 32, sv + 32);
      tmem_ld32(tDP, dv);
      tmem_ld32(tDP + 32, dv + 32);
      tmem_wait_ld();
      // S_j and dP_j are in registers: the next tile's products may overwrite them
      tc_fence_before();
      mbar_arrive(bar_s_free);
      const int kbase = (it.kt0 + j) * 128 + 64 * hc;
      const int nvalid = key_limit - kbase;  // columns >= nvalid are masked
      const int nlo = key_lo - kbase;        // and columns < nlo
      const bool masked = __any_sync(0xffffffffu, nvalid < 64 || (WIN && nlo > 0));
      uint32_t ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sl2, nl2);
        float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        if (masked) {
          if (2 * e >= nvalid || (WIN && 2 * e < nlo)) pr.x = 0.f;
          if (2 * e + 1 >= nvalid || (WIN && 2 * e + 1 < nlo)) pr.y = 0.f;
        }
        const float2 t = __fadd2_rn(make_float2(__uint_as_float(dv[2 * e]), __uint_as_float(dv[2 * e + 1])), ndd);
        const float2 g = __fmul2_rn(pr, t);
        ds[e] = pack_bf16x2(g.x, g.y);
      }
      // dS buffer j & 1 is free once the dQ product of tile j - 2 has read it
      if (j > 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_ds_free(j & 1), ((j - 2) >> 1) & 1, wc));
        if (!ok) break;
      }
      tc_fence_after();
      tmem_st32(tDS + 64 * (j & 1), ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ds_full(j & 1));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && it.n_kv > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_dq_done, 0, wc));
      if (ok) tc_fence_after();
    }
    // The tensor-memory loads are warp-collective: every lane takes them
    // (ok and n_kv are warp-uniform); only the stores depend on the row.
    if (ok) {
      const bool in_range = row < p.Tq;
      const size_t obase = (((size_t)it.b * p.Tq + (in_range ? row : 0)) * p.Hq + it.h) * D + hc * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        if (it.n_kv > 0) {
          tmem_ld32(tmem + C::TM_DQ + lane_off + hc * (D / 2) + 32 * c, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (in_range && p.dq) {
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pw[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * p.scale, __uint_as_float(v[2 * i + 1]) * p.scale);
          uint4* d4 = reinterpret_cast<uint4*>(p.dq + obase + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = pk[i];
        } else if (in_range) {
          float4* d4 = reinterpret_cast<float4*>(p.dq_acc + obase + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(v[4 * i]) * p.scale, __uint_as_float(v[4 * i + 1]) * p.scale,
                                __uint_as_float(v[4 * i + 2]) * p.scale, __uint_as_float(v[4 * i + 3]) * p.scale);
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

static int bwd_dq_setup() {
  const void* kernels[4] = {reinterpret_cast<const void*>(fa_bwd_dq_kernel<64, false>),
                            reinterpret_cast<const void*>(fa_bwd_dq_kernel<64, true>),
                            reinterpret_cast<const void*>(fa_bwd_dq_kernel<128, false>),
                            reinterpret_cast<const void*>(fa_bwd_dq_kernel<128, true>)};
  const int bytes[4] = {DqCfg<64>::SMEM_BYTES, DqCfg<64>::SMEM_BYTES, DqCfg<128>::SMEM_BYTES,
                        DqCfg<128>::SMEM_BYTES};
  for (int i = 0; i < 4; ++i)
    if (cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize, bytes[i]) != cudaSuccess)
      return FA_ERR_CUDA;
  return FA_OK;
}

}  // namespace fa
