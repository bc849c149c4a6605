// fa_fwd.cuh -- forward kernel: O = softmax(scale QK^T [+ causal or
// sliding-window mask]) V and one fp32 log-sum-exp per row, tile by tile with
// the online softmax.  (The sliding window, named next to GQA in the
// "FlashAttention" interview track's "In practice" section, is read as a
// causal window of the W most recent keys; tiles wholly outside it are not
// loaded.)
//
// Method: "Flash Attention: Why Memory Traffic, Not Compute, Is the
// Bottleneck", sections "Flash Attention Uses Tiles" (Q/K/V tiles in on-chip
// memory, S never written out), "Softmax Looks Like an Obstacle" (running m,
// l, u; rescale both l and u by e^{m-m'} when the maximum grows), "Causal
// Masks Still Apply"; "FlashAttention" (interview track), "Softmax without
// seeing the whole row" (keep m and l as one log-sum-exp per row).
//
// B200 mapping.  The kernel is persistent: one CTA per SM walks a list of
// work items, each two 128-row query tiles of one (batch, head), so that one
// item's set-up (Q load, first K/V tiles) and epilogue overlap the next
// item's MMAs instead of leaving the SM idle.
//   warp 9      TMA producer: Q0, Q1 of each item into one of two Q buffers,
//               then K_j, V_j tiles into a ring of shared-memory stages
//               (128-byte swizzle, 64-column boxes), running ahead across
//               items.
//   warp 8      MMA issuer (one thread): S_w = Q_w K_j^T into tensor memory,
//               O_w += P_w V_j with P_w read from tensor memory.
//   warps 10-11 no role (they complete the third warpgroup, whose registers
//               go to the softmax warpgroups).
//   warps 12-15 with dropout at d = 64 only: each KV tile's keep bits for the
//               softmax, one warp per SM sub-partition.
//   warps 0-3   softmax for query tile 0 (TMEM lanes 0..127, one row per
//   warps 4-7   thread) and for query tile 1.  Each thread keeps m and l of
//               its row in registers, writes P (bf16) over its S columns, and
//               rescales its O row in tensor memory when its reference
//               maximum moves; then the epilogue writes O = u / l and LSE.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0, O1 after that.
// Registers: the block is launched with 168 per thread; the MMA/TMA
// warpgroup gives all but 72 of them to the two softmax warpgroups (216
// each), so that a thread holds its whole S row without spilling.  The two
// softmax warpgroups share each SM sub-partition; per pair of columns the
// exponentials, the bf16 pack and the two FP32x2 operations cost about 16
// issue cycles, which bounds the d = 64 kernel.
//
// O is normalised by the sum of the P values the P V product actually
// multiplies (P rounded to bf16), so that O stays a convex combination of
// V rows however nearly one-hot a row is; LSE uses the sum of the unrounded
// p.
//
// FP8 variant (F8 = true, d = 128): Q, K and V are E4M3 with one dequantising
// factor per tensor, the two products run as kind::f8f6f4 MMAs (twice the bf16
// rate), and P is rounded to E4M3 for P V (32 tensor-memory columns over S),
// as FlashAttention-3's low-precision forward does ("FlashAttention",
// interview track, "In practice").  The q and k factors fold into the
// exponent's scale, the v factor into the epilogue's 1 / l; l itself sums the
// unrounded fp32 p.  P goes to shared memory (16 KB per query tile), so that
// the next S overlaps the softmax as in the d = 64 kernel.
//
// Dropout variant (DROP = true, bf16): P is multiplied by a keep mask before
// P V ("Efficient attention: memory-bound", "Real code moves even more", puts
// dropout on the probabilities before the final product); the mask is
// regenerated from Philox-4x32-10 for each tile (at d = 64 by a fourth
// warpgroup, warps 12-15, into shared memory; at d = 128 by the softmax
// threads themselves), l sums the undropped P, and the epilogue
// scales O by 256 / t.
//
// The rescale is lazy: a row keeps its reference maximum until the running
// maximum exceeds it by more than 8 (log2 units), so exponentials stay below
// 2^8.  l and u always share one reference, so the result is the same
// exact softmax (the pages' requirement that both are rescaled together).
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct FwdParams {
  CUtensorMap tm_q;   // [B][Tq][Hq][d] bf16 (E4M3), box {64 (128), 1, 128, 1}, 128-byte swizzle
  CUtensorMap tm_k;   // [B][Tk][Hkv][d]
  CUtensorMap tm_v;
  __nv_bfloat16* o;   // [B][Tq][Hq][d]
  float* lse;         // [B][Hq][Tq]
  int B, Hq, Hkv, Tq, Tk;
  int causal;
  int window;         // > 0: sliding window of that many keys (implies causal)
  float scale_log2;   // scale * log2(e) (times the q and k factors for E4M3 inputs)
  float o_scale;      // multiplies O = u / l: 1, the v factor for E4M3 inputs, or 256 / t with dropout
  uint32_t drop_t;    // dropout: keep iff the Philox byte < drop_t (1..255)
  uint32_t seed_lo, seed_hi, drop_offset;  // dropout: Philox key and counter word 3
  int n_mblocks;      // ceil(Tq / 256): work items per (batch, head)
  int n_items;        // B * Hq * n_mblocks
  unsigned long long wait_limit_ns;
};

template <int D, bool F8 = false, bool DROP = false>
struct FwdCfg {
  static constexpr int BM = 128;                 // rows per query tile
  static constexpr int BN = 128;                 // keys per KV tile
  static constexpr int ELT = F8 ? 1 : 2;         // bytes per element
  static constexpr int BOX_ELEMS = 128 / ELT;    // elements per 128-byte swizzle row
  static constexpr int NBOX = D / BOX_ELEMS;     // swizzle boxes along d
  static constexpr int BOX_BYTES = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  static constexpr int KSTEP = 32 / ELT;         // K elements per MMA instruction (32 bytes)
  static constexpr int NSTAGE = F8 ? 8 : (D == 64) ? 6 : 3;
  static constexpr int OFF_Q = 0;                // 2 buffers x (Q0, Q1)
  static constexpr int OFF_RING = 4 * TILE_BYTES;
  // E4M3: P0, P1 (128 rows x 128 one-byte keys each) in shared memory
  static constexpr int P_BYTES = BM * BN;
  static constexpr int OFF_P = OFF_RING + NSTAGE * TILE_BYTES;
  // Dropout at d = 64: warps 12-15 make each KV tile's keep bits ahead of
  // the softmax, into two buffers of
  // [2 query tiles][128 rows] x 128 bits; the softmax threads load their
  // row's 16 bytes.  (At d = 128 shared memory is full and the softmax
  // threads make their own.)
  static constexpr bool MASKW = DROP && D == 64 && !F8;
  static constexpr int OFF_MASK = OFF_P + (F8 ? 2 * P_BYTES : 0);
  static constexpr int MASK_BYTES = MASKW ? 2 * 2 * 128 * 16 : 0;
  static constexpr int OFF_BAR = OFF_MASK + MASK_BYTES;
  // q_full[2], q_empty[2], kv_full[NSTAGE], kv_empty[NSTAGE], s_full[2],
  // p_full[2], o_final[2], mma_done, s_free[2], p_free[2] (, mask_full[2],
  // mask_empty[2])
  static constexpr int NBAR = 4 + 2 * NSTAGE + 2 + 2 + 2 + 1 + 4 + (MASKW ? 4 : 0);
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (u32), abort flag (int)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  // With the keep-bit warps a fourth warpgroup (warps 12-15) makes the bits,
  // one warp on each SM sub-partition.
  static constexpr int THREADS = MASKW ? 512 : 384;
  static constexpr int MASK_THREADS = 128;
  // setmaxnreg split of the launch's registers (384 x 168, or 512 x 128 with
  // the keep-bit warpgroup): two softmax warpgroups at REG_SOFTMAX, the
  // MMA/TMA warpgroup (and the keep-bit one) at REG_OTHER.
  static constexpr int REG_LAUNCH = MASKW ? 128 : 168;
  static constexpr int REG_SOFTMAX = MASKW ? 208 : 216;
  static constexpr int REG_OTHER = MASKW ? 48 : 72;
  static_assert(128 * (2 * REG_SOFTMAX + (THREADS / 128 - 2) * REG_OTHER) <= THREADS * REG_LAUNCH,
                "register split exceeds the launch");
  static constexpr int TMEM_COLS = 512;
  // P apart from S, so that the next S can be computed as soon as the softmax
  // has loaded this one, overlapping the softmax: at d = 64 (bf16) in its own
  // tensor-memory columns after S0, S1, O0, O1; with E4M3 (d = 128, tensor
  // memory full) in shared memory, where one-byte P takes 16 KB per tile.
  // bf16 at d = 128 has room in neither and writes P over S.
  static constexpr bool SEP_P = (D == 64) || F8;
  // With SEP_P the ring holds (K_j, V_j) pairs with one barrier pair each.
  static constexpr int NPAIR = NSTAGE / 2;
  static constexpr int TM_P = 256 + 2 * D;       // P0, P1: 64 columns each (SEP_P)
  static constexpr uint32_t IDESC_S = F8 ? idesc_e4m3_f32(128, BN, 0, 0) : idesc_bf16_f32(128, BN, 0, 0);
  static constexpr uint32_t IDESC_O = F8 ? idesc_e4m3_f32(128, D, 0, 1) : idesc_bf16_f32(128, D, 0, 1);
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  // Pairs of S columns whose exponentials would use exp2_poly2 on the FMA
  // pipe instead of the MUFU unit.  None: per pair of columns the bf16 pack,
  // the two FP32x2 sums and the scale cost about as many sub-partition
  // cycles as the two MUFU exponentials, so moving exponentials to the FMA
  // pipe slows the softmax at both head sizes (measured 0 < 1/8 < 2/8 < 3/8
  // of the pairs).
  static constexpr bool poly_pair(int) { return false; }
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
  static_assert(!F8 || D == 128, "the E4M3 forward is built for d = 128");
};

// One work item: two query tiles [m0, m0 + 256) of head h of batch b,
// against KV tiles kv0 .. kv0 + n_kv - 1.
struct FwdItem {
  int b, h, hkv, m0, kv0, n_kv;
};

template <int D>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int item) {
  using C = FwdCfg<D>;  // BM and BN are the same for both element types
  FwdItem it;
  // Query blocks of one (batch, head) are adjacent in item order, so they
  // share that head's K/V tiles through L2; within a head the heaviest
  // causal block (the last one) comes first.
  const int bh = item / p.n_mblocks;
  it.b = bh / p.Hq;
  it.h = bh % p.Hq;
  it.hkv = it.h / (p.Hq / p.Hkv);
  it.m0 = (p.n_mblocks - 1 - item % p.n_mblocks) * 2 * C::BM;
  const int n_kv_all = (p.Tk + C::BN - 1) / C::BN;
  it.kv0 = 0;
  it.n_kv = n_kv_all;
  if (p.causal) {
    const int last_row = min(it.m0 + 2 * C::BM, p.Tq) - 1;
    const int kmax = last_row + (p.Tk - p.Tq);  // last visible key (inclusive)
    it.n_kv = kmax < 0 ? 0 : min(n_kv_all, kmax / C::BN + 1);
    if (p.window > 0) {
      // the first row's window starts at its first visible key; tiles
      // before it are skipped
      const int kmin = it.m0 + (p.Tk - p.Tq) - p.window + 1;
      it.kv0 = kmin <= 0 ? 0 : min(it.n_kv, kmin / C::BN);
      it.n_kv -= it.kv0;
    }
  }
  return it;
}

template <int D, bool F8 = false, bool DROP = false>
__global__ void __launch_bounds__(FwdCfg<D, F8, DROP>::THREADS, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D, F8, DROP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_base = sbase + C::OFF_BAR;
  auto bar_q_full = [&](int q) { return bar_base + 8u * q; };
  auto bar_q_empty = [&](int q) { return bar_base + 8u * (2 + q); };
  auto bar_kv_full = [&](int s) { return bar_base + 8u * (4 + s); };
  auto bar_kv_empty = [&](int s) { return bar_base + 8u * (4 + C::NSTAGE + s); };
  auto bar_s_full = [&](int w) { return bar_base + 8u * (4 + 2 * C::NSTAGE + w); };
  auto bar_p_full = [&](int w) { return bar_base + 8u * (6 + 2 * C::NSTAGE + w); };
  auto bar_o_final = [&](int w) { return bar_base + 8u * (8 + 2 * C::NSTAGE + w); };
  const uint32_t bar_mma_done = bar_base + 8u * (10 + 2 * C::NSTAGE);
  auto bar_s_free = [&](int w) { return bar_base + 8u * (11 + 2 * C::NSTAGE + w); };  // softmax loaded S
  auto bar_p_free = [&](int w) { return bar_base + 8u * (13 + 2 * C::NSTAGE + w); };  // PV read P, wrote O
  // dropout keep bits of KV tile t in buffer t & 1: written / read by every row
  auto bar_mask_full = [&](int b) { return bar_base + 8u * (15 + 2 * C::NSTAGE + b); };
  auto bar_mask_empty = [&](int b) { return bar_base + 8u * (17 + 2 * C::NSTAGE + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto q_addr = [&](int qb, int w) { return sbase + C::OFF_Q + (2 * qb + w) * C::TILE_BYTES; };
  auto stage_addr = [&](int s) { return sbase + C::OFF_RING + s * C::TILE_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl wc{abort_flag, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_q_full(q), 1);
      mbar_init(bar_q_empty(q), 1);
    }
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar_s_full(w), 1);
      mbar_init(bar_p_full(w), 128);
      mbar_init(bar_o_final(w), 1);
      mbar_init(bar_s_free(w), 128);
      mbar_init(bar_p_free(w), 1);
      if (C::MASKW) {
        mbar_init(bar_mask_full(w), C::MASK_THREADS);
        mbar_init(bar_mask_empty(w), 256);
      }
    }
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
  // Each role runs inside the branch that set its register budget, so that
  // the compiler allocates that budget for it.
  if (warp >= 8) {
   setmaxnreg_dec<C::REG_OTHER>();
   if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      bool ok = true;
      int qi = 0;         // items with work, in this CTA's order
      int idx = 0;        // K/V ring slot counter
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const FwdItem it = fwd_item<D>(p, item);
        if (it.n_kv == 0) continue;
        const int qb = qi & 1;
        if (qi >= 2) ok = mbar_wait(bar_q_empty(qb), ((qi >> 1) - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_q_full(qb), 2 * C::TILE_BYTES);
        for (int kb = 0; kb < C::NBOX; ++kb) {
          tma_load_4d(q_addr(qb, 0) + kb * C::BOX_BYTES, &p.tm_q, bar_q_full(qb), kb * C::BOX_ELEMS, it.h, it.m0,
                      it.b);
          tma_load_4d(q_addr(qb, 1) + kb * C::BOX_BYTES, &p.tm_q, bar_q_full(qb), kb * C::BOX_ELEMS, it.h,
                      it.m0 + C::BM, it.b);
        }
        for (int j = 0; j < it.n_kv && ok; ++j) {
          if constexpr (C::SEP_P) {
            // K_j and V_j share one stage pair and one full/empty barrier
            const int gp = idx >> 1, pi = gp % C::NPAIR, round = gp / C::NPAIR;
            if (round > 0) ok = mbar_wait(bar_kv_empty(pi), (round - 1) & 1, wc);
            if (!ok) break;
            mbar_arrive_expect_tx(bar_kv_full(pi), 2 * C::TILE_BYTES);
            for (int kb = 0; kb < C::NBOX; ++kb) {
              tma_load_4d(stage_addr(2 * pi) + kb * C::BOX_BYTES, &p.tm_k, bar_kv_full(pi), kb * 64, it.hkv,
                          (it.kv0 + j) * C::BN, it.b);
              tma_load_4d(stage_addr(2 * pi + 1) + kb * C::BOX_BYTES, &p.tm_v, bar_kv_full(pi), kb * 64, it.hkv,
                          (it.kv0 + j) * C::BN, it.b);
            }
            idx += 2;
          } else {
            for (int which = 0; which < 2 && ok; ++which, ++idx) {
              const int s = idx % C::NSTAGE;
              const int round = idx / C::NSTAGE;
              if (round > 0) ok = mbar_wait(bar_kv_empty(s), (round - 1) & 1, wc);
              if (!ok) break;
              mbar_arrive_expect_tx(bar_kv_full(s), C::TILE_BYTES);
              const CUtensorMap* tm = which ? &p.tm_v : &p.tm_k;
              for (int kb = 0; kb < C::NBOX; ++kb)
                tma_load_4d(stage_addr(s) + kb * C::BOX_BYTES, tm, bar_kv_full(s), kb * C::BOX_ELEMS, it.hkv,
                            (it.kv0 + j) * C::BN, it.b);
            }
          }
        }
        ++qi;
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        for (int q = max(0, qi - 1); q <= qi; ++q) mbar_wait_drain(bar_q_full(q & 1), (q >> 1) & 1, p.wait_limit_ns);
        if constexpr (C::SEP_P) {
          for (int k = max(0, (idx >> 1) - C::NPAIR); k < (idx >> 1); ++k)
            mbar_wait_drain(bar_kv_full(k % C::NPAIR), (k / C::NPAIR) & 1, p.wait_limit_ns);
        } else {
          for (int k = max(0, idx - C::NSTAGE); k < idx; ++k)
            mbar_wait_drain(bar_kv_full(k % C::NSTAGE), (k / C::NSTAGE) & 1, p.wait_limit_ns);
        }
      }
    }
  } else if (C::MASKW && warp >= 12) {
    // ------------------------------------------------------------ dropout mask
    // Thread mt makes rows 4 a .. 4 a + 3 (a = (mt >> 1) & 31) of query tile
    // mt >> 6 against key half mt & 1: for each of that half's 16 key groups
    // the Philox block of those four rows (the layout the softmax's own
    // generator uses: counter (row / 4, key / 4, bh, offset), word = row,
    // byte = key), each row's keep bits gathered into its two 32-key words
    // of the half.
    const int mt = threadIdx.x - 384;
    const int wq = mt >> 6, a_loc = (mt >> 1) & 31, kh = mt & 1;
    const uint32_t tt = p.drop_t * 0x01010101u;
    uint4* mbuf = reinterpret_cast<uint4*>(smem + C::OFF_MASK);
    bool ok = true;
    int g = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const FwdItem it = fwd_item<D>(p, item);
      if (it.n_kv == 0) continue;
      const uint32_t a_glob = (uint32_t)((it.m0 + wq * C::BM) >> 2) + (uint32_t)a_loc;
      const uint32_t bh = (uint32_t)(it.b * p.Hq + it.h);
      for (int j = 0; j < it.n_kv && ok; ++j) {
        const int t = g + j, buf = t & 1;
        if (t >= 2) ok = mbar_wait(bar_mask_empty(buf), ((t >> 1) - 1) & 1, wc);
        if (!ok) break;
        const uint32_t c0 = (uint32_t)((it.kv0 + j) * C::BN) >> 2;
        uint32_t* mw = reinterpret_cast<uint32_t*>(mbuf + (buf * 2 + wq) * 128 + 4 * a_loc);
#pragma unroll
        for (int k = 2 * kh; k < 2 * kh + 2; ++k) {  // keys 32k .. 32k + 31: eight Philox blocks
          uint32_t rw[4] = {0u, 0u, 0u, 0u};  // one word per row of the group
          // not unrolled: fully unrolled, the blocks' states spill at this
          // warpgroup's 72 registers (measured 1.37 against 1.19 ms)
#pragma unroll 1
          for (int cl = 8 * k; cl < 8 * k + 8; ++cl) {
            const uint4 v = philox4x32_10(make_uint4(a_glob, c0 + cl, bh, p.drop_offset), p.seed_lo, p.seed_hi);
            const int sh = 4 * (cl & 7);
            rw[0] |= gather_msb4(bytes_below(v.x, tt)) << sh;
            rw[1] |= gather_msb4(bytes_below(v.y, tt)) << sh;
            rw[2] |= gather_msb4(bytes_below(v.z, tt)) << sh;
            rw[3] |= gather_msb4(bytes_below(v.w, tt)) << sh;
          }
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) mw[4 * w4 + k] = rw[w4];
        }
        mbar_arrive(bar_mask_full(buf));
      }
      g += it.n_kv;
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
      // Descriptors: the low word of the tile's first K slice plus the slice
      // offset / 16 (the high word is the same for every operand here).
      constexpr uint32_t HI = sw128_hi(1024);
      auto issue_s = [&](int w, uint32_t qa, int sK) {
        const uint32_t a0 = sw128_lo(qa, 16), b0 = sw128_lo(stage_addr(sK), 16);
#pragma unroll
        for (int k = 0; k < D / C::KSTEP; ++k) {
          const uint32_t o = ((k >> 2) * C::BOX_BYTES + (k & 3) * 32) >> 4;
          const uint64_t da = sw128_desc(a0 + o, HI), db = sw128_desc(b0 + o, HI);
          if constexpr (F8) mma_ss_f8(tS[w], da, db, C::IDESC_S, k > 0);
          else mma_ss(tS[w], da, db, C::IDESC_S, k > 0);
        }
      };
      // P (over S's first columns) times V_j: each MMA takes KSTEP keys, 32
      // bytes of P per row (8 columns) and KSTEP rows of the V tile.
      auto issue_pv = [&](int w, int sV, bool first) {
        const uint32_t v0 = sw128_lo(stage_addr(sV), C::BOX_BYTES);
#pragma unroll
        for (int k = 0; k < C::BN / C::KSTEP; ++k) {
          const uint64_t db = sw128_desc(v0 + ((k * C::KSTEP * 128) >> 4), HI);
          if constexpr (F8) mma_ts_f8(tO[w], tS[w] + k * 8, db, C::IDESC_O, (!first) || k > 0);
          else mma_ts(tO[w], tS[w] + k * 8, db, C::IDESC_O, (!first) || k > 0);
        }
      };
      bool ok = true;
      int qi = 0, g = 0;  // items with work, global KV tile counter
      if constexpr (C::SEP_P) {
        // P lives in its own columns: for every KV tile j, S_0(j) and S_1(j)
        // are issued as soon as the softmax warpgroups have loaded S(j-1)
        // (s_free), and PV_w(j-1) once P_w(j-1) is written (p_full); each PV
        // commits p_free, which releases the P columns and O to the softmax.
        const uint32_t tP[2] = {tmem + C::TM_P, tmem + C::TM_P + 64};
        auto issue_pv_p = [&](int w, int sV, bool first) {
          const uint32_t v0 = sw128_lo(stage_addr(sV), C::BOX_BYTES);
          const uint32_t p0 = sw128_lo(sbase + C::OFF_P + w * C::P_BYTES, 16);
#pragma unroll
          for (int k = 0; k < C::BN / C::KSTEP; ++k) {
            const uint64_t db = sw128_desc(v0 + ((k * C::KSTEP * 128) >> 4), HI);
            if constexpr (F8) {
              // P_w in shared memory: K-major, 128-byte rows, 128-byte swizzle
              const uint64_t da = sw128_desc(p0 + ((k * 32) >> 4), HI);
              mma_ss_f8(tO[w], da, db, C::IDESC_O, (!first) || k > 0);
            } else {
              mma_ts(tO[w], tP[w] + k * 8, db, C::IDESC_O, (!first) || k > 0);
            }
          }
        };
        for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
          const FwdItem it = fwd_item<D>(p, item);
          if (it.n_kv == 0) continue;
          const int qb = qi & 1;
          ok = mbar_wait(bar_q_full(qb), (qi >> 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          for (int j = 0; j <= it.n_kv && ok; ++j) {
            const int gt = g + j;
            if (j < it.n_kv) {
              const int pi = gt % C::NPAIR;
              ok = mbar_wait(bar_kv_full(pi), (gt / C::NPAIR) & 1, wc);  // K_j and V_j
#pragma unroll
              for (int w = 0; w < 2; ++w) {
                if (ok && gt > 0) ok = mbar_wait(bar_s_free(w), (gt - 1) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                issue_s(w, q_addr(qb, w), 2 * pi);
                mma_commit(bar_s_full(w));
              }
              if (!ok) break;
            }
            if (j > 0) {
              // PV of the previous tile (its V arrived with its K)
              const int pi = (gt - 1) % C::NPAIR, sV = 2 * pi + 1;
              const bool last = j == it.n_kv;
#pragma unroll
              for (int w = 0; w < 2; ++w) {
                if (ok) ok = mbar_wait(bar_p_full(w), (gt - 1) & 1, wc);
                if (!ok) break;
                tc_fence_after();
                issue_pv_p(w, sV, j == 1);
                mma_commit(bar_p_free(w));
                if (last) mma_commit(bar_o_final(w));
              }
              if (!ok) break;
              mma_commit(bar_kv_empty(pi));
            }
          }
          if (!ok) break;
          mma_commit(bar_q_empty(qb));
          g += it.n_kv;
          ++qi;
        }
      } else {
        for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
          const FwdItem it = fwd_item<D>(p, item);
          if (it.n_kv == 0) continue;
          const int qb = qi & 1;
          ok = mbar_wait(bar_q_full(qb), (qi >> 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          int sV_prev = 0;
          for (int j = 0; j < it.n_kv && ok; ++j) {
            const int gt = g + j;
            const int iK = 2 * gt, iV = 2 * gt + 1;
            const int sK = iK % C::NSTAGE, sV = iV % C::NSTAGE;
            ok = mbar_wait(bar_kv_full(sK), (iK / C::NSTAGE) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_s(0, q_addr(qb, 0), sK);
            mma_commit(bar_s_full(0));
            if (j > 0) {
              ok = mbar_wait(bar_p_full(1), (gt - 1) & 1, wc);
              if (!ok) break;
              tc_fence_after();
              issue_pv(1, sV_prev, j - 1 == 0);
              mma_commit(bar_kv_empty(sV_prev));
            }
            issue_s(1, q_addr(qb, 1), sK);
            mma_commit(bar_s_full(1));
            mma_commit(bar_kv_empty(sK));
            ok = mbar_wait(bar_p_full(0), gt & 1, wc);
            if (!ok) break;
            ok = mbar_wait(bar_kv_full(sV), (iV / C::NSTAGE) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_pv(0, sV, j == 0);
            sV_prev = sV;
          }
          if (!ok) break;
          mma_commit(bar_o_final(0));
          ok = mbar_wait(bar_p_full(1), (g + it.n_kv - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, sV_prev, it.n_kv - 1 == 0);
          mma_commit(bar_kv_empty(sV_prev));
          mma_commit(bar_o_final(1));
          mma_commit(bar_q_empty(qb));
          g += it.n_kv;
          ++qi;
        }
      }
      // Wait until every MMA issued above has completed before teardown.
      mma_commit(bar_mma_done);
      mbar_wait_drain(bar_mma_done, 0, p.wait_limit_ns);
    }
  }
  } else {
    setmaxnreg_inc<C::REG_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;                 // query tile 0 or 1
    const int r = threadIdx.x & 127;         // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + w * 128 + lane_off;
    const uint32_t tO = tmem + 256 + w * D + lane_off;
    const uint32_t tP = tmem + C::TM_P + w * 64 + lane_off;  // P's own columns (SEP_P)
    bool ok = true;
    int qi = 0, g = 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const FwdItem it = fwd_item<D>(p, item);
      const int row = it.m0 + w * C::BM + r;
      const int key_limit = p.causal ? min(p.Tk, row + (p.Tk - p.Tq) + 1) : p.Tk;  // keys < limit visible
      const int key_lo = p.window > 0 ? row + (p.Tk - p.Tq) - p.window + 1 : 0;     // and keys >= key_lo
      float m_ref = -INFINITY;  // reference maximum, log2 units of scaled scores
      float l = 0.f;            // sum of the p (the LSE's)
      float l_r = 0.f;          // sum of the p as rounded for P V (O's normaliser; bf16)
      for (int j = 0; j < it.n_kv; ++j) {
        // dropout: this tile's keep bits, made while the tensor core computes S
        uint32_t keep[4];
        if constexpr (C::MASKW) {
          // this row's keep bits from the mask warps
          const int t = g + j, mb = t & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_mask_full(mb), (t >> 1) & 1, wc));
          if (!ok) break;
          const uint4 kv = reinterpret_cast<const uint4*>(smem + C::OFF_MASK)[(mb * 2 + w) * 128 + r];
          keep[0] = kv.x;
          keep[1] = kv.y;
          keep[2] = kv.z;
          keep[3] = kv.w;
          mbar_arrive(bar_mask_empty(mb));
        } else if constexpr (DROP) {
          dropout_keep_128(keep, row, (it.kv0 + j) * C::BN, (uint32_t)(it.b * p.Hq + it.h), p.drop_offset,
                           p.seed_lo, p.seed_hi, p.drop_t);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(w), (g + j) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        uint32_t su[128];  // S row, then P (bf16 pairs) packed in place
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, su + c * 32);
        tmem_wait_ld();
        if constexpr (C::SEP_P) {
          // S is in registers: the next S may overwrite its columns
          tc_fence_before();
          mbar_arrive(bar_s_free(w));
        }
        const int nvalid = key_limit - (it.kv0 + j) * C::BN;  // columns >= nvalid are masked
        const int nlo = key_lo - (it.kv0 + j) * C::BN;         // and columns < nlo
        const bool masked = __any_sync(0xffffffffu, nvalid < C::BN || nlo > 0);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nvalid || c < nlo) su[c] = __float_as_uint(-INFINITY);
        }
        // Row maximum: eight independent chains of three-input maxima (two
        // new columns per step), then a short tree.
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmax3(__uint_as_float(su[i]), __uint_as_float(su[8 + i]),
                                                  __uint_as_float(su[16 + i]));
#pragma unroll
        for (int c = 24; c < 120; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], __uint_as_float(su[c + i]), __uint_as_float(su[c + 8 + i]));
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], __uint_as_float(su[120 + i]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_tile = mx * p.scale_log2;
        // Lazy rescale: move the reference only when the maximum grew by more
        // than the threshold (or there was no reference yet).
        const bool move = (m_tile > m_ref + C::RESCALE_THRESHOLD) || (m_ref == -INFINITY && m_tile != -INFINITY);
        float alpha = 1.f;
        if (move) {
          alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_tile);
          m_ref = m_tile;
          l *= alpha;
          l_r *= alpha;
        }
        const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nref = make_float2(-ref, -ref);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 acc_r[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if constexpr (C::SEP_P) {
          // P's columns (E4M3: P's shared-memory tile) and O are free once
          // the previous tile's PV completed (normally long since): bf16 P is
          // stored in two halves as the loop below produces it.  Waiting here
          // rather than after the loop measured 12% faster for E4M3 (1444
          // against 1292 TFLOP/s on the 32k causal GQA workload).
          if (g + j > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_p_free(w), (g + j - 1) & 1, wc));
            if (!ok) break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(su[2 * c]), __uint_as_float(su[2 * c + 1])), sl2, nref);
          // Part of the exponentials go to the FMA pipe so that the MUFU
          // unit, shared by both softmax warpgroups, is not the bottleneck.
          float2 pr = C::poly_pair(c) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          if (C::poly_pair(c) && masked) {
            if (2 * c >= nvalid || 2 * c < nlo) pr.x = 0.f;
            if (2 * c + 1 >= nvalid || 2 * c + 1 < nlo) pr.y = 0.f;
          }
          acc[c & 3] = __fadd2_rn(acc[c & 3], pr);   // l sums the undropped p
          if constexpr (F8) {
            if constexpr (DROP) {
              const uint32_t kb = keep[c >> 4] >> ((2 * c) & 31);
              pr.x = (kb & 1u) ? pr.x : 0.f;
              pr.y = (kb & 2u) ? pr.y : 0.f;
            }
            // four E4M3 values per column; su[c >> 1] was consumed at step c >> 2
            const uint32_t h = pack_e4m3x2(pr.x, pr.y);
            su[c >> 1] = (c & 1) ? (su[c >> 1] | (h << 16)) : h;
          } else {
            uint32_t pk = pack_bf16x2(pr.x, pr.y);
            // l_r sums the undropped p as rounded (bf16 to fp32 is a shift)
            acc_r[c & 1] = __fadd2_rn(acc_r[c & 1], make_float2(__uint_as_float(pk << 16),
                                                                 __uint_as_float(pk & 0xFFFF0000u)));
            if constexpr (DROP) {
              const uint32_t kb = keep[c >> 4] >> ((2 * c) & 31);
              pk &= ((kb & 1u) ? 0x0000FFFFu : 0u) | ((kb & 2u) ? 0xFFFF0000u : 0u);
            }
            su[c] = pk;
            // each half of P (32 columns) goes to tensor memory while the
            // next half is computed: P's own columns (d = 64) or, at d = 128,
            // the S columns already in registers
            if (c == 31 || c == 63) tmem_st32((C::SEP_P ? tP : tS) + (c == 63 ? 32 : 0), su + (c == 63 ? 32 : 0));
          }
        }
        const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l += a.x + a.y;
        const float2 ar = __fadd2_rn(acc_r[0], acc_r[1]);
        l_r += ar.x + ar.y;
        if constexpr (F8) {
          {
            // row r of P_w: eight 16-byte chunks, chunk c stored at c ^ (r & 7)
            // (the 128-byte swizzle the MMA's descriptor names)
            uint8_t* prow = smem + C::OFF_P + w * C::P_BYTES + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
                  make_uint4(su[4 * c], su[4 * c + 1], su[4 * c + 2], su[4 * c + 3]);
            fence_proxy_async_smem();
          }
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // O row *= alpha.  The PV of the previous tile has completed (with
          // P over S, the commit behind s_full tracks every MMA issued before
          // it; with P apart, p_free was awaited above), and the PV of this
          // tile waits for p_full below.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_full(w));
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (it.n_kv > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_final(w), qi & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
      const bool in_range = row < p.Tq;
      const float l_o = F8 ? l : l_r;
      const float inv_l = (l_o > 0.f) ? p.o_scale / l_o : 0.f;
      __nv_bfloat16* orow = p.o + (((size_t)it.b * p.Tq + (in_range ? row : 0)) * p.Hq + it.h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (it.n_kv > 0) {
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint4 packed[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pw[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = packed[i];
        }
      }
      if (in_range) {
        const float lse = (l > 0.f) ? (m_ref * 0.69314718055994531f + logf(l)) : -INFINITY;
        p.lse[((size_t)it.b * p.Hq + it.h) * p.Tq + row] = lse;
      }
      // O has been read: the next item's first PV (which overwrites O) is
      // issued only after this warpgroup's next p_full arrival.
      tc_fence_before();
      if (it.n_kv > 0) {
        g += it.n_kv;
        ++qi;
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

}  // namespace fa
