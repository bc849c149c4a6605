// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument
// checks, TMA descriptor set-up and kernel launches.  Every kernel of the
// library is compiled in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <initializer_list>
#include <mutex>

#include "fa_status.h"
#include "fa_ptx.cuh"
#include "fa_fwd.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd_dq.cuh"
#include "fa_decode.cuh"

namespace fa {

// Limit for every bounded wait inside the kernels.  Far above any legitimate
// wait (the longest kernels run for tens of milliseconds).
static constexpr unsigned long long kWaitLimitNs = 4000000000ull;

// ---------------------------------------------------------------------------
// Driver entry point for TMA descriptors (resolved through the runtime, so
// the library links no driver stub and loads on machines without a GPU).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 4-D bf16 tensor [n3][n2][n1][n0] (n0 contiguous) with box {64, 1, box_rows, 1}
// along (n0, n1, n2, n3) and the 128-byte swizzle, or no swizzle when
// `swizzle` is false (then box_inner elements along n0).
// elt = 2: bf16 elements; elt = 1: 8-bit (E4M3) elements.
static int make_tmap_4d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                        uint64_t n3, uint32_t box_inner, uint32_t box_rows, bool swizzle, int elt = 2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {n0, n1, n2, n3};
  const cuuint64_t strides[3] = {n0 * elt, n0 * n1 * elt, n0 * n1 * n2 * elt};
  const cuuint32_t box[4] = {box_inner, 1, box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, elt == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 4-D fp32 tensor [n3][n2][n1][n0] with box {32, 1, 128, 1} and the 128-byte
// swizzle (the dQ accumulator, written by bulk tensor reduce-add).
static int make_tmap_f32_4d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                            uint64_t n3) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {n0, n1, n2, n3};
  const cuuint64_t strides[3] = {n0 * 4, n0 * n1 * 4, n0 * n1 * n2 * 4};
  const cuuint32_t box[4] = {32, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Per-device set-up: architecture check and shared-memory opt-in, once.
// ---------------------------------------------------------------------------
static constexpr int kMaxDevices = 64;

template <typename Fn>
static int set_smem(Fn* kernel, int bytes) {
  return cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

// The forward kernels move registers between warpgroups with setmaxnreg;
// the split adds up only if the block is launched with exactly the per-thread
// count it was planned for (an increase beyond the launch's pool would wait
// forever), so a build that came out differently is refused, not launched.
template <int D, bool F8, bool DROP>
static int fwd_setup_one() {
  using C = FwdCfg<D, F8, DROP>;
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, reinterpret_cast<const void*>(fa_fwd_kernel<D, F8, DROP>)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (a.numRegs != C::REG_LAUNCH) return FA_ERR_UNSUPPORTED;
  return set_smem(fa_fwd_kernel<D, F8, DROP>, C::SMEM_BYTES);
}

template <int D, int G>
static int decode_setup_one() {
  int st = set_smem(fa_decode_split_kernel<D, G>, DecCfg<D, G>::SMEM_BYTES);
  return st;
}

static int decode_setup() {
  int st = FA_OK;
  if (!st) st = decode_setup_one<64, 1>();
  if (!st) st = decode_setup_one<64, 2>();
  if (!st) st = decode_setup_one<64, 4>();
  if (!st) st = decode_setup_one<64, 8>();
  if (!st) st = decode_setup_one<128, 1>();
  if (!st) st = decode_setup_one<128, 2>();
  if (!st) st = decode_setup_one<128, 4>();
  if (!st) st = decode_setup_one<128, 8>();
  return st;
}

static int device_setup_impl() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
  int st = FA_OK;
  if (!st) st = fwd_setup_one<64, false, false>();
  if (!st) st = fwd_setup_one<128, false, false>();
  if (!st) st = fwd_setup_one<128, true, false>();
  if (!st) st = fwd_setup_one<64, false, true>();
  if (!st) st = fwd_setup_one<128, false, true>();
  if (!st) st = bwd_setup();
  if (!st) st = bwd_dq_setup();
  if (!st) st = decode_setup();
  return st;
}

static int device_setup() {
  static int state[kMaxDevices];  // 0 = not done, else status + 1
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (state[dev] == 0) state[dev] = device_setup_impl() + 1;
  return state[dev] - 1;
}

// Persistent decode grid: CTAs per SM.
static constexpr int kDecodeCtasPerSm = 2;

// Number of SMs of the current device (persistent grids use one CTA per SM).
static int sm_count(int* n) {
  static int cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return FA_ERR_CUDA;
    cache[dev] = v;
  }
  *n = cache[dev];
  return FA_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int launch_status() {
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Checks shared by the prefill entry points.
static int check_prefill(int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Tq < 0 || Tk < 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // Tensor-map extents are 32-bit and row/item indices are int; (batch, KV
  // head) pairs index the backward's second grid dimension (at most 65535).
  if ((int64_t)Tq > (1 << 30) || (int64_t)Tk > (1 << 30) || (int64_t)B * Hq > 65535 ||
      (int64_t)B * Hq * ((Tq + 255) / 256) > (1ll << 30))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_version(void) { return 100; }

}  // extern "C"

// Dropout keep threshold t = round(256 (1 - p)) clamped to [1, 256]; 256
// means no dropout.  Returns 0 for a rate outside [0, 1).
static uint32_t keep_threshold(float p_drop) {
  if (!(p_drop >= 0.f && p_drop < 1.f)) return 0;
  long t = lrintf(256.f * (1.f - p_drop));
  return (uint32_t)(t < 1 ? 1 : (t > 256 ? 256 : t));
}

// window > 0: sliding window of that many keys (the caller passes causal = 1).
// f8: q, k, v are E4M3; `qk_factor` multiplies the scores' scale and
// `o_scale` the output (the dequantising factors).  drop_t in 1..255: dropout
// on P with keep threshold drop_t (o_scale is then 256 / drop_t), Philox key
// (seed_lo, seed_hi) and counter word `drop_offset`.
static int forward_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                        int Hkv, int Tq, int Tk, int d, float scale, int causal, int window, void* stream,
                        bool f8 = false, float qk_factor = 1.f, float o_scale = 1.f, uint32_t drop_t = 256,
                        uint32_t seed_lo = 0, uint32_t seed_hi = 0, uint32_t drop_offset = 0) {
  const bool drop = drop_t < 256;
  int st = check_prefill(B, Hq, Hkv, Tq, Tk, d, scale, causal);
  if (st) return st;
  if (window < 0 || window > (1 << 30)) return FA_ERR_INVALID_ARG;
  if (f8 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Tq == 0) return FA_OK;
  if (!q || !o || !lse || (Tk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || (Tk > 0 && (!aligned16(k) || !aligned16(v))))
    return FA_ERR_ALIGNMENT;
  st = device_setup();
  if (st) return st;
  FwdParams p;
  memset(&p, 0, sizeof(p));
  const int elt = f8 ? 1 : 2, box_inner = 128 / elt;  // one 128-byte swizzle row per box
  st = make_tmap_4d(&p.tm_q, q, d, Hq, Tq, B, box_inner, 128, true, elt);
  if (!st && Tk > 0) st = make_tmap_4d(&p.tm_k, k, d, Hkv, Tk, B, box_inner, 128, true, elt);
  if (!st && Tk > 0) st = make_tmap_4d(&p.tm_v, v, d, Hkv, Tk, B, box_inner, 128, true, elt);
  if (st) return st;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Tq = Tq; p.Tk = Tk;
  p.causal = causal;
  p.window = window;
  p.scale_log2 = scale * qk_factor * 1.4426950408889634f;
  p.o_scale = o_scale;
  p.drop_t = drop_t;
  p.seed_lo = seed_lo;
  p.seed_hi = seed_hi;
  p.drop_offset = drop_offset;
  p.n_mblocks = (Tq + 255) / 256;
  p.n_items = B * Hq * p.n_mblocks;
  p.wait_limit_ns = kWaitLimitNs;
  // Uniform (non-causal or sliding-window) items: persistent, one CTA per
  // SM.  Causal items differ in cost: one CTA per item, heaviest first,
  // balanced by the block scheduler.
  int nsm = 0;
  if ((st = sm_count(&nsm))) return st;
  // Sliding-window items are about equally long: persistent as well.
  dim3 grid(causal && window == 0 ? p.n_items : std::min(p.n_items, nsm));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (f8)
    fa_fwd_kernel<128, true><<<grid, FwdCfg<128, true>::THREADS, FwdCfg<128, true>::SMEM_BYTES, s>>>(p);
  else if (drop && d == 64)
    fa_fwd_kernel<64, false, true><<<grid, FwdCfg<64, false, true>::THREADS, FwdCfg<64, false, true>::SMEM_BYTES, s>>>(p);
  else if (drop)
    fa_fwd_kernel<128, false, true><<<grid, FwdCfg<128, false, true>::THREADS, FwdCfg<128, false, true>::SMEM_BYTES, s>>>(p);
  else if (d == 64)
    fa_fwd_kernel<64><<<grid, FwdCfg<64>::THREADS, FwdCfg<64>::SMEM_BYTES, s>>>(p);
  else
    fa_fwd_kernel<128><<<grid, FwdCfg<128>::THREADS, FwdCfg<128>::SMEM_BYTES, s>>>(p);
  return launch_status();
}

extern "C" {

int fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Tq, int Tk, int d, float scale, int causal, void* stream) {
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0, stream);
}

int fa_forward_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                      int Hkv, int Tq, int Tk, int d, float scale, int window, void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, d, scale, 1, window, stream);
}

int fa_forward_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                       int Hkv, int Tq, int Tk, int d, float scale, int causal, float p_drop,
                       unsigned long long seed, unsigned int offset, void* stream) {
  const uint32_t t = keep_threshold(p_drop);
  if (!t) return FA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0, stream, false, 1.f,
                      256.f / (float)t, (uint32_t)t, (uint32_t)(seed & 0xFFFFFFFFull), (uint32_t)(seed >> 32),
                      offset);
}

int fa_forward_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                   float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                   float scale, int causal, void* stream) {
  for (float f : {q_descale, k_descale, v_descale})
    if (!(f > 0.f) || !isfinite(f)) return FA_ERR_INVALID_ARG;
  if (!isfinite(scale * q_descale * k_descale)) return FA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0, stream, true,
                      q_descale * k_descale, v_descale);
}

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

static int tq_pad(int Tq) { return (Tq + 127) / 128 * 128; }

size_t fa_backward_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int d) {
  (void)Hkv; (void)Tk;
  if (B < 0 || Hq < 1 || Tq < 0 || (d != 64 && d != 128)) return 0;
  return round256((size_t)B * Tq * Hq * d * 4) + 2 * round256((size_t)B * Hq * tq_pad(Tq) * 4);
}

// Workspace pieces of the backward pass.
struct BwdWs {
  float* dq_acc;
  float* Dv;
  float* lse2;
};
static BwdWs bwd_ws(void* ws, int B, int Hq, int Tq, int d) {
  BwdWs w;
  w.dq_acc = reinterpret_cast<float*>(ws);
  w.Dv = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + round256((size_t)B * Tq * Hq * d * 4));
  w.lse2 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(w.Dv) + round256((size_t)B * Hq * tq_pad(Tq) * 4));
  return w;
}

static int check_ws(void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d) {
  const size_t need = fa_backward_workspace_bytes(B, Hq, Hkv, Tq, Tk, d);
  if (!ws || ws_bytes < need || !aligned16(ws)) return FA_ERR_WORKSPACE;
  return FA_OK;
}

static int check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* ptr : ptrs) {
    if (!ptr) return FA_ERR_INVALID_ARG;
    if (!aligned16(ptr)) return FA_ERR_ALIGNMENT;
  }
  return FA_OK;
}

// zero_acc = false leaves the fp32 dQ accumulator alone (a backward whose dQ
// pass writes dq directly does not read it).
static int preprocess_impl(const void* o, const float* lse, const void* dO, void* ws, size_t ws_bytes, int B,
                           int Hq, int Hkv, int Tq, int Tk, int d, void* stream, bool zero_acc) {
  int st = check_prefill(B, Hq, Hkv, Tq, Tk, d, 1.f, 0);
  if (st) return st;
  if (B == 0 || Tq == 0) return FA_OK;
  if ((st = check_ptrs({o, lse, dO}))) return st;
  if ((st = check_ws(ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d))) return st;
  if ((st = device_setup())) return st;
  const BwdWs w = bwd_ws(ws, B, Hq, Tq, d);
  const int Tp = tq_pad(Tq);
  const long long threads = std::max((long long)B * Tq * Hq * (d / 8), (long long)B * Hq * (Tp - Tq));
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const __nv_bfloat16* o16 = reinterpret_cast<const __nv_bfloat16*>(o);
  const __nv_bfloat16* do16 = reinterpret_cast<const __nv_bfloat16*>(dO);
  float* acc = zero_acc ? w.dq_acc : nullptr;
  if (d == 64)
    fa_bwd_preprocess_kernel<64><<<blocks, 256, 0, s>>>(o16, do16, lse, w.Dv, w.lse2, acc, B, Hq, Tq, Tp);
  else
    fa_bwd_preprocess_kernel<128><<<blocks, 256, 0, s>>>(o16, do16, lse, w.Dv, w.lse2, acc, B, Hq, Tq, Tp);
  return launch_status();
}

int fa_backward_preprocess(const void* o, const float* lse, const void* dO, void* ws, size_t ws_bytes,
                           int B, int Hq, int Hkv, int Tq, int Tk, int d, void* stream) {
  return preprocess_impl(o, lse, dO, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, stream, true);
}

}  // extern "C"

// drop_t in 1..255: dropout on P with that keep threshold and Philox key
// (seed_lo, seed_hi), counter word drop_offset (the forward's mask).
// det: dQ from the separate, deterministic pass (fa_bwd_dq.cuh) after the
// dK/dV kernel built without dQ, into the fp32 accumulator or, when dq_out
// is given, as bf16 straight into dq_out (no dropout).
static int dkdv_impl(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, void* ws,
                     size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal,
                     int window, void* stream, uint32_t drop_t = 256, uint32_t seed_lo = 0, uint32_t seed_hi = 0,
                     uint32_t drop_offset = 0, bool det = false, void* dq_out = nullptr) {
  const bool drop = drop_t < 256;
  int st = check_prefill(B, Hq, Hkv, Tq, Tk, d, scale, causal);
  if (st) return st;
  if (window < 0 || window > (1 << 30)) return FA_ERR_INVALID_ARG;
  if (B == 0 || Tk == 0) return FA_OK;
  if ((st = check_ptrs({k, v, dk, dv}))) return st;
  if (Tq > 0 && (st = check_ptrs({q, dO}))) return st;
  if ((st = check_ws(ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d))) return st;
  if ((st = device_setup())) return st;
  const BwdWs w = bwd_ws(ws, B, Hq, Tq, d);
  BwdParams p;
  memset(&p, 0, sizeof(p));
  if (Tq > 0) {
    st = make_tmap_4d(&p.tm_q, q, d, Hq, Tq, B, 64, 128, true);
    if (!st) st = make_tmap_4d(&p.tm_do, dO, d, Hq, Tq, B, 64, 128, true);
  }
  if (!st) st = make_tmap_4d(&p.tm_k, k, d, Hkv, Tk, B, 64, 128, true);
  if (!st) st = make_tmap_4d(&p.tm_v, v, d, Hkv, Tk, B, 64, 128, true);
  if (!st && Tq > 0) st = make_tmap_f32_4d(&p.tm_dq, w.dq_acc, d, Hq, Tq, B);
  if (st) return st;
  p.lse2 = w.lse2;
  p.Dv = w.Dv;
  p.dq_acc = w.dq_acc;
  p.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Tq = Tq; p.Tk = Tk; p.causal = causal;
  p.window = window;
  p.Tq_pad = tq_pad(Tq);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_kv_tiles = (Tk + 127) / 128;
  p.n_items = p.n_kv_tiles * B * Hkv;
  p.drop_t = drop_t;
  p.seed_lo = seed_lo;
  p.seed_hi = seed_hi;
  p.drop_offset = drop_offset;
  p.drop_scale = 256.f / (float)drop_t;
  p.wait_limit_ns = kWaitLimitNs;
  // Non-causal d = 64: one persistent CTA per SM, whose next item's K/V
  // load overlaps the current item (two K/V buffers); items are all the
  // same length there.  Causal: one CTA per item, since items differ in
  // length and the hardware scheduler balances them.
  int nsm = 0;
  if ((st = sm_count(&nsm))) return st;
  const bool persistent = d == 64 && !causal;
  dim3 grid(persistent ? std::min(p.n_items, nsm) : p.n_items);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (drop && (window > 0 || det)) return FA_ERR_UNSUPPORTED;
  if (drop) {
    if (d == 64)
      fa_bwd_dkdv_kernel<64, false, true><<<grid, BwdCfg<64, true>::THREADS, BwdCfg<64, true>::SMEM_BYTES, s>>>(p);
    else
      fa_bwd_dkdv_kernel<128, false, true><<<grid, BwdCfg<128, true>::THREADS, BwdCfg<128, true>::SMEM_BYTES, s>>>(p);
    return launch_status();
  }
  if (!det) {
    if (d == 64 && window > 0)
      fa_bwd_dkdv_kernel<64, true><<<grid, BwdCfg<64>::THREADS, BwdCfg<64>::SMEM_BYTES, s>>>(p);
    else if (d == 64)
      fa_bwd_dkdv_kernel<64, false><<<grid, BwdCfg<64>::THREADS, BwdCfg<64>::SMEM_BYTES, s>>>(p);
    else if (window > 0)
      fa_bwd_dkdv_kernel<128, true><<<grid, BwdCfg<128>::THREADS, BwdCfg<128>::SMEM_BYTES, s>>>(p);
    else
      fa_bwd_dkdv_kernel<128, false><<<grid, BwdCfg<128>::THREADS, BwdCfg<128>::SMEM_BYTES, s>>>(p);
    return launch_status();
  }
  // deterministic: dK/dV without dQ, then the dQ pass
  using C64 = BwdCfg<64, false, false>;
  using C128 = BwdCfg<128, false, false>;
  if (d == 64 && window > 0)
    fa_bwd_dkdv_kernel<64, true, false, false><<<grid, C64::THREADS, C64::SMEM_BYTES, s>>>(p);
  else if (d == 64)
    fa_bwd_dkdv_kernel<64, false, false, false><<<grid, C64::THREADS, C64::SMEM_BYTES, s>>>(p);
  else if (window > 0)
    fa_bwd_dkdv_kernel<128, true, false, false><<<grid, C128::THREADS, C128::SMEM_BYTES, s>>>(p);
  else
    fa_bwd_dkdv_kernel<128, false, false, false><<<grid, C128::THREADS, C128::SMEM_BYTES, s>>>(p);
  if ((st = launch_status())) return st;
  if (Tq == 0) return FA_OK;
  DqParams qp;
  memset(&qp, 0, sizeof(qp));
  qp.tm_q = p.tm_q;
  qp.tm_do = p.tm_do;
  qp.tm_k = p.tm_k;
  qp.tm_v = p.tm_v;
  qp.lse2 = w.lse2;
  qp.Dv = w.Dv;
  qp.dq_acc = w.dq_acc;
  qp.dq = reinterpret_cast<__nv_bfloat16*>(dq_out);
  qp.B = B; qp.Hq = Hq; qp.Hkv = Hkv; qp.Tq = Tq; qp.Tk = Tk; qp.causal = causal;
  qp.window = window;
  qp.Tq_pad = p.Tq_pad;
  qp.scale = scale;
  qp.scale_log2 = p.scale_log2;
  qp.n_qt = (Tq + 127) / 128;
  const long long n_items = (long long)B * Hq * qp.n_qt;
  if (n_items > 0x7FFFFFFFll) return FA_ERR_INVALID_ARG;
  qp.n_items = (int)n_items;
  qp.wait_limit_ns = kWaitLimitNs;
  const unsigned nblk = (unsigned)qp.n_items;
  if (d == 64 && window > 0)
    fa_bwd_dq_kernel<64, true><<<nblk, DqCfg<64>::THREADS, DqCfg<64>::SMEM_BYTES, s>>>(qp);
  else if (d == 64)
    fa_bwd_dq_kernel<64, false><<<nblk, DqCfg<64>::THREADS, DqCfg<64>::SMEM_BYTES, s>>>(qp);
  else if (window > 0)
    fa_bwd_dq_kernel<128, true><<<nblk, DqCfg<128>::THREADS, DqCfg<128>::SMEM_BYTES, s>>>(qp);
  else
    fa_bwd_dq_kernel<128, false><<<nblk, DqCfg<128>::THREADS, DqCfg<128>::SMEM_BYTES, s>>>(qp);
  return launch_status();
}

extern "C" {

int fa_backward_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                     void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                     float scale, int causal, void* stream) {
  return dkdv_impl(q, k, v, dO, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0, stream);
}

int fa_backward_dkdv_window(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                            void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                            float scale, int window, void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return dkdv_impl(q, k, v, dO, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, 1, window, stream);
}

int fa_backward_dkdv_dropout(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                             void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                             float scale, int causal, float p_drop, unsigned long long seed, unsigned int offset,
                             void* stream) {
  const uint32_t t = keep_threshold(p_drop);
  if (!t) return FA_ERR_INVALID_ARG;
  return dkdv_impl(q, k, v, dO, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0, stream, t,
                   (uint32_t)(seed & 0xFFFFFFFFull), (uint32_t)(seed >> 32), offset);
}

int fa_backward_dq_finalize(void* dq, void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk,
                            int d, void* stream) {
  int st = check_prefill(B, Hq, Hkv, Tq, Tk, d, 1.f, 0);
  if (st) return st;
  if (B == 0 || Tq == 0) return FA_OK;
  if ((st = check_ptrs({dq}))) return st;
  if ((st = check_ws(ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d))) return st;
  if ((st = device_setup())) return st;
  const BwdWs w = bwd_ws(ws, B, Hq, Tq, d);
  const long long n8 = (long long)B * Tq * Hq * d / 8;
  fa_bwd_dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      w.dq_acc, reinterpret_cast<__nv_bfloat16*>(dq), n8);
  return launch_status();
}

}  // extern "C"

static int backward_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B, int Hq,
                         int Hkv, int Tq, int Tk, int d, float scale, int causal, int window, void* stream,
                         uint32_t drop_t = 256, uint32_t seed_lo = 0, uint32_t seed_hi = 0,
                         uint32_t drop_offset = 0, bool det = false) {
  int st = check_prefill(B, Hq, Hkv, Tq, Tk, d, scale, causal);
  if (st) return st;
  if (window < 0 || window > (1 << 30)) return FA_ERR_INVALID_ARG;
  if (B == 0 || (Tq == 0 && Tk == 0)) return FA_OK;
  if (Tq > 0 && (st = check_ptrs({q, o, lse, dO, dq}))) return st;
  if (Tk > 0 && (st = check_ptrs({k, v, dk, dv}))) return st;
  if ((st = check_ws(ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d))) return st;
  // deterministic: the dQ pass writes dq itself (when there are keys; with
  // none, dq is the zeroed accumulator converted)
  const bool direct = det && Tq > 0 && Tk > 0;
  if ((st = preprocess_impl(o, lse, dO, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, stream, !direct))) return st;
  if ((st = dkdv_impl(q, k, v, dO, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, window, stream,
                      drop_t, seed_lo, seed_hi, drop_offset, det, direct ? dq : nullptr)))
    return st;
  if (direct) return FA_OK;
  return fa_backward_dq_finalize(dq, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, stream);
}

extern "C" {

int fa_backward(const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B,
                int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal, void* stream) {
  return backward_impl(q, k, v, o, lse, dO, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0,
                       stream);
}

int fa_backward_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B, int Hq,
                        int Hkv, int Tq, int Tk, int d, float scale, int causal, float p_drop,
                        unsigned long long seed, unsigned int offset, void* stream) {
  const uint32_t t = keep_threshold(p_drop);
  if (!t) return FA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, o, lse, dO, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, 0,
                       stream, t, (uint32_t)(seed & 0xFFFFFFFFull), (uint32_t)(seed >> 32), offset);
}

int fa_backward_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B,
                       int Hq, int Hkv, int Tq, int Tk, int d, float scale, int window, void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, o, lse, dO, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, 1, window,
                       stream);
}

int fa_backward_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B,
                              int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal, int window,
                              void* stream) {
  if (window < 0 || (window > 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, o, lse, dO, dq, dk, dv, ws, ws_bytes, B, Hq, Hkv, Tq, Tk, d, scale, causal, window,
                       stream, 256, 0, 0, 0, true);
}

static size_t decode_nchunk(int Tk_max, int chunk) { return ((size_t)Tk_max + chunk - 1) / chunk; }

size_t fa_decode_workspace_bytes(int B, int Hq, int Tk_max, int d, int chunk) {
  if (B < 0 || Hq < 1 || Tk_max < 0 || chunk < 1 || (d != 64 && d != 128)) return 0;
  const size_t n = decode_nchunk(Tk_max, chunk);
  return round256((size_t)B * Hq * n * d * 4) + round256((size_t)B * Hq * n * 4);
}

}  // extern "C"

// `o` receives bf16 O, or, when `o32` is non-null instead, fp32 O.
static int decode_impl(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k, void* o,
                       float* o32, float* lse, void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tk_max,
                       int d, float scale, int chunk, int window, void* stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Tk_max < 0 || Hq % Hkv != 0 || !isfinite(scale))
    return FA_ERR_INVALID_ARG;
  if (window < 0 || window > (1 << 30)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FA_ERR_UNSUPPORTED;
  if (chunk < 64 || chunk % 64 != 0 || chunk * G > 4096) return FA_ERR_INVALID_ARG;
  // one warp per (sequence, head) row in the merge kernels: 32 * B * Hq
  // threads must stay below 2^31
  if ((int64_t)Tk_max > (1 << 30) || (int64_t)B * Hq > (1 << 26)) return FA_ERR_INVALID_ARG;
  if (B == 0) return FA_OK;
  if (!q || !seqlens_k || (!o == !o32) || !lse || (Tk_max > 0 && (!k_cache || !v_cache)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o ? o : o32) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(seqlens_k) & 3u) ||
      (Tk_max > 0 && (!aligned16(k_cache) || !aligned16(v_cache))))
    return FA_ERR_ALIGNMENT;
  const size_t need = fa_decode_workspace_bytes(B, Hq, Tk_max, d, chunk);
  if (!ws || ws_bytes < need || !aligned16(ws)) return FA_ERR_WORKSPACE;
  int st = device_setup();
  if (st) return st;
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  const size_t n = decode_nchunk(Tk_max, chunk);
  if (Tk_max > 0) {
    st = make_tmap_4d(&p.tm_k, k_cache, d, Hkv, Tk_max, B, 64, 64, true);
    if (!st) st = make_tmap_4d(&p.tm_v, v_cache, d, Hkv, Tk_max, B, 64, 64, true);
    if (st) return st;
  }
  if ((size_t)B * Hkv * n > (size_t)(1 << 30)) return FA_ERR_INVALID_ARG;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.seqlens = seqlens_k;
  p.ws_o = reinterpret_cast<float*>(ws);
  p.ws_lse = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + round256((size_t)B * Hq * n * d * 4));
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.o32 = o32;
  p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Tk_max = Tk_max; p.chunk = chunk; p.nchunk = (int)n;
  p.n_items = (int)((size_t)B * Hkv * n);
  p.window = window;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = kWaitLimitNs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (Tk_max > 0) {
    int nsm = 0;
    if ((st = sm_count(&nsm))) return st;
    // persistent: two CTAs per SM walk the (sequence, KV head, chunk) items
    dim3 grid((unsigned)std::min<long long>(p.n_items, (long long)kDecodeCtasPerSm * nsm));
#define FA_DEC_LAUNCH(DD, GG) \
    fa_decode_split_kernel<DD, GG><<<grid, DecCfg<DD, GG>::THREADS, DecCfg<DD, GG>::SMEM_BYTES, s>>>(p)
    if (d == 64) {
      if (G == 1) FA_DEC_LAUNCH(64, 1); else if (G == 2) FA_DEC_LAUNCH(64, 2);
      else if (G == 4) FA_DEC_LAUNCH(64, 4); else FA_DEC_LAUNCH(64, 8);
    } else {
      if (G == 1) FA_DEC_LAUNCH(128, 1); else if (G == 2) FA_DEC_LAUNCH(128, 2);
      else if (G == 4) FA_DEC_LAUNCH(128, 4); else FA_DEC_LAUNCH(128, 8);
    }
#undef FA_DEC_LAUNCH
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  const int warps = B * Hq;
  const int blocks = (warps * 32 + 255) / 256;
  if (Tk_max > 0) {
    if (d == 64)
      fa_decode_combine_kernel<64><<<blocks, 256, 0, s>>>(p);
    else
      fa_decode_combine_kernel<128><<<blocks, 256, 0, s>>>(p);
  }
  if (d == 64)
    fa_decode_empty_kernel<64><<<blocks, 256, 0, s>>>(p);
  else
    fa_decode_empty_kernel<128><<<blocks, 256, 0, s>>>(p);
  return launch_status();
}

extern "C" {

int fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k,
                      void* o, float* lse, void* ws, size_t ws_bytes, int B, int Hq, int Hkv,
                      int Tk_max, int d, float scale, int chunk, void* stream) {
  return decode_impl(q, k_cache, v_cache, seqlens_k, o, nullptr, lse, ws, ws_bytes, B, Hq, Hkv, Tk_max, d, scale,
                     chunk, 0, stream);
}

int fa_decode_splitkv_partial(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k,
                              float* o, float* lse, void* ws, size_t ws_bytes, int B, int Hq, int Hkv,
                              int Tk_max, int d, float scale, int chunk, void* stream) {
  return decode_impl(q, k_cache, v_cache, seqlens_k, nullptr, o, lse, ws, ws_bytes, B, Hq, Hkv, Tk_max, d, scale,
                     chunk, 0, stream);
}

int fa_decode_merge(const float* o_parts, size_t o_stride, const float* lse_parts, size_t lse_stride, void* o,
                    float* lse, int R, int B, int Hq, int d, void* stream) {
  if (R < 1 || R > (1 << 20) || B < 0 || Hq < 1 || (int64_t)B * Hq > (1 << 26)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const size_t rows = (size_t)B * Hq;
  if (rows == 0) return FA_OK;
  if (!o_parts || !lse_parts || !o || !lse) return FA_ERR_INVALID_ARG;
  if (R > 1 && (o_stride < rows * d || lse_stride < rows)) return FA_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o) || (o_stride & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_parts) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGNMENT;
  int st = device_setup();
  if (st) return st;
  MergeParams p;
  p.o_parts = o_parts;
  p.lse_parts = lse_parts;
  p.o_stride = o_stride;
  p.lse_stride = lse_stride;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.R = R;
  p.rows = (int)rows;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
  if (d == 64)
    fa_decode_merge_kernel<64><<<blocks, 256, 0, s>>>(p);
  else
    fa_decode_merge_kernel<128><<<blocks, 256, 0, s>>>(p);
  return launch_status();
}

int fa_decode_splitkv_window(const void* q, const void* k_cache, const void* v_cache, const int* seqlens_k,
                             void* o, float* lse, void* ws, size_t ws_bytes, int B, int Hq, int Hkv,
                             int Tk_max, int d, float scale, int chunk, int window, void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return decode_impl(q, k_cache, v_cache, seqlens_k, o, nullptr, lse, ws, ws_bytes, B, Hq, Hkv, Tk_max, d, scale,
                     chunk, window, stream);
}

int fa_check(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"

namespace fa {
// One block, one thread waits on a barrier that nothing completes.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl w{&abort_flag, limit_ns};
    mbar_wait(smem_u32(&bar), 0, w);
  }
  __syncthreads();
}
}  // namespace fa

namespace fa {
__global__ void selftest_exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 out = exp2_poly2(in);
  y[i] = out.x;
  if (i + 1 < n) y[i + 1] = out.y;
}
}  // namespace fa

extern "C" int fa_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  int st = device_setup();
  if (st) return st;
  const int pairs = (n + 1) / 2;
  selftest_exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

extern "C" int fa_selftest_bounded_wait(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return FA_ERR_INVALID_ARG;
  int st = device_setup();
  if (st) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_us * 1000ull);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Split-KV decode without caller-provided workspace.
//
// For callers that cannot allocate device memory at the call site --
// plug-in interfaces that hand over only the input and output tensors and
// no allocator, or latency-critical loops where cudaMalloc's implicit
// device synchronisation is not acceptable.  The chunk partials live in one
// file-scope device array that every GPU loading this library keeps until
// the process exits.
// ---------------------------------------------------------------------------
namespace fa {

static constexpr size_t kDecodeScratchBytes = 32u << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

// Device address of g_decode_scratch for the current device, looked up once
// per device (host code may not use the symbol itself as an address).
static int decode_scratch_ptr(void** out) {
  static void* cache[kMaxDevices];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return FA_ERR_CUDA;
    cache[dev] = ptr;
  }
  *out = cache[dev];
  return FA_OK;
}

}  // namespace fa

extern "C" int fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv,
                                         int Tk_max, int d, float scale, int chunk, void* stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Tk_max < 0 || chunk < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // The partials of this call must fit in the built-in scratch array.
  if (fa_decode_workspace_bytes(B, Hq, Tk_max, d, chunk) > kDecodeScratchBytes) return FA_ERR_WORKSPACE;
  // No rows: the workspace entry point checks the remaining arguments the
  // same way and returns before it touches the (empty) workspace.
  if (B == 0)
    return fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, o, lse, nullptr, 0, B, Hq, Hkv, Tk_max, d, scale, chunk,
                             stream);
  void* scratch = nullptr;
  const int st = decode_scratch_ptr(&scratch);
  if (st) return st;
  // Every partial the combine step reads is written first by the split step
  // of the same call, so nothing in the scratch needs clearing.
  return fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, o, lse, scratch, kDecodeScratchBytes, B, Hq, Hkv,
                           Tk_max, d, scale, chunk, stream);
}
