/*
 * fa.h -- C ABI of libfa: exact, IO-aware scaled-dot-product attention for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (all entry points compute the same function):
 *   S = scale * Q K^T (+ causal mask), P = softmax(S) row by row, O = P V,
 *   LSE_i = ln sum_j exp(S_ij).
 * It is computed tile by tile with the online softmax, never writing S or P
 * to device memory.  Sources, cited by page title and section:
 *   - "Flash Attention: Why Memory Traffic, Not Compute, Is the Bottleneck",
 *     sections "Flash Attention Uses Tiles", "Softmax Looks Like an Obstacle",
 *     "Causal Masks Still Apply", "We Usually Call It Through an API";
 *   - "Efficient attention: memory-bound", sections "Standard attention,
 *     kernel by kernel" and "Real code moves even more" (the backward
 *     products), "The obstacle, a normalizer that needs the whole row";
 *   - "FlashAttention" (interview track), sections "Softmax without seeing
 *     the whole row" (one fp32 log-sum-exp per row kept for the backward
 *     pass, recomputation instead of storing P) and "In practice" (GQA,
 *     causal masks, FlashDecoding's split of the KV cache).
 *
 * Conventions shared by every entry point
 *   - Element types: bf16 = IEEE bfloat16 stored as uint16_t bit patterns;
 *     float = IEEE fp32.  Accumulation is fp32.
 *   - Layouts are dense, row-major "BTHD":
 *       q, o, dO, dq   : [B, Tq, Hq, d]
 *       k, v, dk, dv   : [B, Tk, Hkv, d]
 *       lse            : [B, Hq, Tq]   (natural-log units of the scaled scores)
 *   - d must be 64 or 128; Hq % Hkv == 0; B * Hq <= 65535 for the prefill
 *     entry points and B * Hq <= 2^26 for the decode ones (larger sizes are
 *     FA_ERR_INVALID_ARG).  Query head h reads KV head h / (Hq / Hkv)
 *     (contiguous groups).
 *   - Causal rule: key j is visible to query i iff j <= i + (Tk - Tq)
 *     (bottom-right aligned; for Tq == Tk this is j <= i).  A row that sees
 *     no key gets O = 0, LSE = -inf and zero gradients.
 *   - All pointers are DEVICE pointers of the current CUDA device, 16-byte
 *     aligned.  The caller owns every buffer, including workspaces; the
 *     library never allocates or frees device memory (except where an entry
 *     point says otherwise).
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t passed
 *     as void*; NULL = legacy default stream).  Nothing synchronises.
 *   - Inputs are never modified.
 *   - Return value: FA_OK or one of the fa_status codes.  Argument errors are
 *     detected on the host before anything is launched.  A kernel whose
 *     bounded wait expires records FA_ERR_TIMEOUT in a device status word,
 *     which fa_check() reports.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* bad size, null pointer, Hq % Hkv != 0, ... */
  FA_ERR_UNSUPPORTED = 2,  /* head dim other than 64/128, device not sm_100 */
  FA_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,    /* workspace pointer null or smaller than required */
  FA_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
  FA_ERR_TIMEOUT = 6       /* a kernel's bounded wait expired (see fa_check) */
} fa_status;

/* Human-readable name of a status code (static string). */
const char* fa_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int fa_version(void);

/*
 * fa_forward -- O and LSE of exact attention.
 * ("Flash Attention: Why Memory Traffic...", "Flash Attention Uses Tiles" and
 *  "Softmax Looks Like an Obstacle"; LSE as in "FlashAttention",
 *  "Softmax without seeing the whole row".)
 *   q [B,Tq,Hq,d], k/v [B,Tk,Hkv,d]  bf16 in
 *   o [B,Tq,Hq,d] bf16 out; lse [B,Hq,Tq] fp32 out
 *   scale: multiplies QK^T before the softmax (usually 1/sqrt(d))
 *   causal: 0 or 1
 * Tq == 0 is a no-op.  Tk == 0 writes O = 0 and LSE = -inf.
 */
int fa_forward(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal,
               void* stream);

/*
 * fa_forward_window -- fa_forward with a sliding-window mask: query i sees
 * key j iff i + (Tk - Tq) - window < j <= i + (Tk - Tq), i.e. its own
 * (bottom-right aligned) diagonal key and the window - 1 keys before it.
 * ("FlashAttention", "In practice", names sliding windows next to GQA and
 * causal masks without defining them; this causal local window is the
 * reading used here.)  window >= Tk gives the causal result; window < 1 or
 * above 2^30 is FA_ERR_INVALID_ARG.  Other arguments as fa_forward.  Key
 * tiles wholly outside every window of a query tile are not read.
 */
int fa_forward_window(const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int window,
                      void* stream);

/*
 * fa_forward_dropout -- fa_forward with dropout on P fused into the kernel
 * ("Efficient attention: memory-bound", "Real code moves even more", lists
 * dropout among the elementwise steps on P before the final product):
 *   O = (P * Z) V / (t / 256),  LSE that of the undropped P,
 * where Z_ij keeps (i, j) with probability t / 256, t = round(256 (1 - p_drop))
 * clamped to 1..256 (p_drop is used to the nearest 1/256).  Z is regenerated
 * from Philox-4x32-10 (Salmon et al., SC 2011): the block of rows 4a..4a+3 and
 * keys 4c..4c+3 of head h of batch b uses counter (a, c, b * Hq + h, offset)
 * and key (seed mod 2^32, seed >> 32); word w of its output is row 4a + w and
 * byte j of that word key 4c + j, kept iff the byte < t.  The same (seed,
 * offset) always gives the same mask.
 *   p_drop in [0, 1) (else FA_ERR_INVALID_ARG); p_drop = 0 gives fa_forward.
 *   Other arguments and errors as fa_forward.  bf16 only; no window.
 */
int fa_forward_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                       int Hkv, int Tq, int Tk, int d, float scale, int causal, float p_drop,
                       unsigned long long seed, unsigned int offset, void* stream);

/*
 * fa_forward_fp8 -- fa_forward with 8-bit inputs: the low-precision forward
 * that "FlashAttention" (interview track, "In practice") lists for FA3, here
 * on B200's kind::f8f6f4 tensor-core MMAs.
 *   q, k, v   E4M3 (OCP FP8: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 *             bits), one byte per element, layouts as fa_forward.
 *   q_descale, k_descale, v_descale  the factor that turns each tensor's
 *             codes into its values (value = code * descale), finite and > 0.
 *   o, lse    as fa_forward (bf16 O, fp32 LSE of the scaled scores).
 * The result is attention on the dequantised inputs, with P rounded to E4M3
 * before P V (the row sums l use the unrounded P); that rounding makes O
 * differ from exact attention by up to a few percent on rows with few keys
 * (3 mantissa bits), much less on long rows.  d must be 128
 * (FA_ERR_UNSUPPORTED otherwise); other arguments and errors as fa_forward.
 */
int fa_forward_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                   float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                   float scale, int causal, void* stream);

/*
 * Bytes of device workspace fa_backward needs: an fp32 dQ accumulator
 * [B,Tq,Hq,d], the fp32 row terms D_i = sum_c dO_ic O_ic and the LSE in log2
 * units, each [B,Hq,Tq_pad] with Tq_pad = Tq rounded up to 128; every piece
 * rounded up to 256 bytes.  Returns 0 for invalid sizes.
 */
size_t fa_backward_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int d);

/*
 * fa_backward -- dQ, dK, dV of L = sum(dO * O) for the forward above, with
 * S and P recomputed tile by tile from the saved LSE ("FlashAttention",
 * follow-up on recomputing instead of storing P; the products dV = P^T dO,
 * dP = dO V^T, dS = P*(dP - D), dQ = scale dS K, dK = scale dS^T Q from
 * "Efficient attention: memory-bound", "Real code moves even more").
 *   q, k, v, o (the forward's output), lse (the forward's LSE), dO  in
 *   dq [B,Tq,Hq,d], dk/dv [B,Tk,Hkv,d] bf16 out.  For GQA, dk/dv sum over the
 *   query heads of each group.
 *   ws/ws_bytes: device workspace of at least fa_backward_workspace_bytes();
 *   its contents on entry do not matter.
 */
int fa_backward(const void* q, const void* k, const void* v, const void* o,
                const float* lse, const void* dO, void* dq, void* dk, void* dv,
                void* ws, size_t ws_bytes,
                int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int causal,
                void* stream);

/*
 * fa_backward_window -- gradients of fa_forward_window (same window rule;
 * o and lse must come from fa_forward_window with the same window).  Other
 * arguments, the workspace and the errors as fa_backward.
 */
int fa_backward_window(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dO, void* dq, void* dk, void* dv,
                       void* ws, size_t ws_bytes,
                       int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale, int window,
                       void* stream);

/*
 * fa_backward_deterministic -- the gradients of fa_backward (causal = 0 or 1,
 * window = 0) or of fa_backward_window (causal = 1, window >= 1), with dQ
 * the same bit for bit from run to run.  fa_backward adds every KV tile's
 * share of dQ into an fp32 accumulator with bulk reduce-adds, whose order
 * varies between runs; here the dK/dV pass leaves dQ out and a second pass,
 * one work item per (128-query tile, head, batch), recomputes S and dP for
 * the tile's KV tiles, keeps dQ in tensor memory and writes it once
 * ("FlashAttention", follow-up on recomputing instead of storing P).  dK and
 * dV are those of fa_backward, bit for bit.  It costs more time: the second
 * pass recomputes the two products S and dP.  Arguments, workspace and
 * errors as fa_backward; window < 0, or window > 0 without causal = 1, is
 * FA_ERR_INVALID_ARG.  bf16, d = 64 or 128, no dropout.
 */
int fa_backward_deterministic(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dO, void* dq, void* dk, void* dv,
                              void* ws, size_t ws_bytes,
                              int B, int Hq, int Hkv, int Tq, int Tk, int d, float scale,
                              int causal, int window, void* stream);

/*
 * The three steps fa_backward runs, in this order on one stream, exposed so
 * that a caller can schedule or time them separately.  They share the
 * workspace of fa_backward_workspace_bytes() and its layout; arguments mean
 * what they mean for fa_backward.
 *   fa_backward_preprocess   D_i = sum_c dO_ic O_ic and the LSE in log2
 *                            units into the workspace; zeroes the fp32 dQ
 *                            accumulator.
 *   fa_backward_dkdv         one pass over (key tile, KV head, batch): dK and
 *                            dV written, scale*dS*K added into the dQ
 *                            accumulator.  Needs the preprocess step first.
 *   fa_backward_dq_finalize  dq = bf16(accumulator).
 */
int fa_backward_preprocess(const void* o, const float* lse, const void* dO, void* ws, size_t ws_bytes,
                           int B, int Hq, int Hkv, int Tq, int Tk, int d, void* stream);
int fa_backward_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                     void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                     float scale, int causal, void* stream);

/* fa_backward_dkdv with the sliding window of fa_forward_window (window >= 1). */
int fa_backward_dkdv_window(const void* q, const void* k, const void* v, const void* dO, void* dk,
                            void* dv, void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq,
                            int Tk, int d, float scale, int window, void* stream);

int fa_backward_dq_finalize(void* dq, void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk,
                            int d, void* stream);

/*
 * fa_backward_dropout -- gradients of L = sum(dO * O) for fa_forward_dropout
 * with the same p_drop, seed and offset ("Efficient attention: memory-bound",
 * "Real code moves even more": dropout on P before the final product; the
 * products are those of fa_backward with the keep mask Z in them):
 *   dV = s (P*Z)^T dO,  dP = s (dO V^T) * Z,  dS = P * (dP - D),
 *   dQ = scale dS K,    dK = scale dS^T Q,    s = 256 / t,
 * with D_i = sum_c dO_ic O_ic of the dropout forward's O (equal to
 * sum_j P_ij dP_ij) and P recomputed from its (undropped) LSE.  Z is not
 * stored: the kernel regenerates the forward's Philox-4x32-10 mask block by
 * block, so o and lse must come from fa_forward_dropout with the same
 * (p_drop, seed, offset).  p_drop = 0 gives fa_backward.  Arguments,
 * workspace, layouts and errors as fa_backward; p_drop outside [0, 1) is
 * FA_ERR_INVALID_ARG.  bf16 only; no window.
 *
 * fa_backward_dkdv_dropout -- its dK/dV step alone (after
 * fa_backward_preprocess, before fa_backward_dq_finalize).
 */
int fa_backward_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int B, int Hq,
                        int Hkv, int Tq, int Tk, int d, float scale, int causal, float p_drop,
                        unsigned long long seed, unsigned int offset, void* stream);
int fa_backward_dkdv_dropout(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                             void* ws, size_t ws_bytes, int B, int Hq, int Hkv, int Tq, int Tk, int d,
                             float scale, int causal, float p_drop, unsigned long long seed, unsigned int offset,
                             void* stream);

/*
 * Bytes of device workspace fa_decode_splitkv needs: fp32 partial outputs
 * [B,Hq,nchunk,d] and partial LSEs [B,Hq,nchunk], nchunk = ceil(Tk_max/chunk).
 */
size_t fa_decode_workspace_bytes(int B, int Hq, int Tk_max, int d, int chunk);

/*
 * fa_decode_splitkv -- one query token per sequence against a KV cache,
 * split into chunks of `chunk` keys processed by separate thread blocks and
 * merged by their log-sum-exp ("FlashAttention", "In practice":
 * FlashDecoding).
 *   q [B,Hq,d] bf16; k_cache/v_cache [B,Tk_max,Hkv,d] bf16;
 *   seqlens_k: DEVICE int32 [B], each in [0, Tk_max] (sequence b attends to
 *   its first seqlens_k[b] cached keys, no mask); a value outside that range
 *   is read as the nearer end of it (below 0 as 0, above Tk_max as Tk_max);
 *   o [B,Hq,d] bf16 out; lse [B,Hq] fp32 out;
 *   ws/ws_bytes: at least fa_decode_workspace_bytes(); contents on entry do
 *   not matter.  chunk must be a positive multiple of 64.
 *   Hq/Hkv must be 1, 2, 4 or 8 and chunk * (Hq/Hkv) at most 4096.
 */
int fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                      const int* seqlens_k, void* o, float* lse, void* ws, size_t ws_bytes,
                      int B, int Hq, int Hkv, int Tk_max, int d, float scale, int chunk,
                      void* stream);

/*
 * fa_decode_splitkv_window -- fa_decode_splitkv with the sliding window of
 * fa_forward_window: the query (the sequence's last position) sees only the
 * last `window` cached keys, min(window, seqlens_k[b]) of them.  Chunks that
 * hold none of them are skipped.  window >= 1; other arguments, workspace
 * and errors as fa_decode_splitkv.
 */
int fa_decode_splitkv_window(const void* q, const void* k_cache, const void* v_cache,
                             const int* seqlens_k, void* o, float* lse, void* ws, size_t ws_bytes,
                             int B, int Hq, int Hkv, int Tk_max, int d, float scale, int chunk,
                             int window, void* stream);

/*
 * fa_decode_splitkv_noalloc -- fa_decode_splitkv for callers that cannot
 * allocate device memory where they call it: a plug-in interface of a
 * serving engine that hands the kernel its input and output tensors but no
 * allocator, or a latency-critical decode loop that cannot afford
 * cudaMalloc's implicit device synchronisation.  The pages have no
 * counterpart; this is a deployment convenience around the same kernels.
 *   Arguments as for fa_decode_splitkv, without ws/ws_bytes.  The chunk
 *   partials live in a 32 MiB array inside the library (every GPU that loads
 *   the library holds it until the process exits), so
 *   fa_decode_workspace_bytes(B, Hq, Tk_max, d, chunk) must be at most
 *   33554432; larger calls return FA_ERR_WORKSPACE before any launch.
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   The first call on a device looks up the array's device address and sets
 *   kernel attributes for that device; make that first call outside any
 *   stream capture.
 *   All calls share the one array: calls whose kernels overlap on the GPU
 *   (different streams, or different host threads, without ordering) race
 *   and produce wrong results.  Calls ordered on one stream are safe; the
 *   array keeps the last call's contents, which no later call relies on.
 */
int fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int* seqlens_k, void* o, float* lse,
                              int B, int Hq, int Hkv, int Tk_max, int d, float scale, int chunk,
                              void* stream);

/*
 * Context-parallel decode: one sequence's KV cache spread over several GPUs.
 * Each GPU decodes its own share of the keys with fa_decode_splitkv_partial,
 * the GPUs exchange their (O_r, LSE_r) rows (an all-gather, the caller's
 * collective), and fa_decode_merge combines them.  This is FlashDecoding's
 * split of the KV cache ("FlashAttention", interview track, section "In
 * practice") taken across devices: the merge is the chunk merge of
 * fa_decode_splitkv with devices in place of chunks,
 *   LSE = log sum_r e^{LSE_r},  O = sum_r e^{LSE_r - LSE} O_r.
 * Keys may be shared out in any way (the unmasked softmax does not depend on
 * key order); no window is offered because the window of the full sequence is
 * not a window of each share.
 *
 * fa_decode_splitkv_partial -- fa_decode_splitkv over this GPU's share, with
 * the normalised output written in fp32 so that the merge does not round
 * twice.
 *   o     fp32 [B][Hq][d], 16-byte aligned;  lse fp32 [B][Hq].
 *   A sequence whose share is empty (seqlens_k[b] == 0) gets O = 0 and
 *   LSE = -inf, which the merge ignores.  Everything else (arguments,
 *   workspace, errors, asynchrony) as fa_decode_splitkv.
 */
int fa_decode_splitkv_partial(const void* q, const void* k_cache, const void* v_cache,
                              const int* seqlens_k, float* o, float* lse, void* ws, size_t ws_bytes,
                              int B, int Hq, int Hkv, int Tk_max, int d, float scale, int chunk,
                              void* stream);

/*
 * fa_decode_merge -- combines R partial decodes of the same B x Hq rows.
 *   o_parts     device fp32; partial r is the [B][Hq][d] block starting at
 *               o_parts + r * o_stride.  16-byte aligned.
 *   o_stride    floats between consecutive O blocks: a multiple of 4 and,
 *               when R > 1, at least B * Hq * d.
 *   lse_parts   device fp32; partial r is the [B][Hq] block starting at
 *               lse_parts + r * lse_stride.  4-byte aligned.
 *   lse_stride  floats between consecutive LSE blocks; when R > 1, at least
 *               B * Hq.  (O and LSE of one partial may share one packed
 *               block: O first, LSE after it, both strides the block size.)
 *   o           device bf16 [B][Hq][d] (16-byte aligned); lse device fp32 [B][Hq].
 *   R           number of partials, 1 .. 2^20.   d in {64, 128}.
 * A row with LSE_r = -inf in every partial gets O = 0 and LSE = -inf.
 * Errors: FA_ERR_INVALID_ARG (sizes, null pointers, short stride),
 * FA_ERR_UNSUPPORTED (d), FA_ERR_ALIGNMENT, FA_ERR_CUDA (launch), all before
 * or at launch; B == 0 is a no-op.  Asynchronous on `stream`; nothing is
 * allocated and the inputs are not modified.
 */
int fa_decode_merge(const float* o_parts, size_t o_stride, const float* lse_parts, size_t lse_stride,
                    void* o, float* lse, int R, int B, int Hq, int d, void* stream);

/*
 * fa_check -- synchronise `stream`, then read and clear the device status
 * word that kernels set when a bounded wait expires.  Returns FA_OK,
 * FA_ERR_TIMEOUT, or FA_ERR_CUDA if the synchronisation itself failed.
 */
int fa_check(void* stream);

/*
 * fa_selftest_bounded_wait -- launch one block that waits on a barrier that
 * nothing will ever complete, with a wait limit of `limit_us` microseconds
 * (1..1000000).  The kernel gives up, records FA_ERR_TIMEOUT in the status
 * word and returns normally; fa_check() then reports it.  Used to test the
 * failure path without faulting or hanging the GPU.
 */
int fa_selftest_bounded_wait(int limit_us, void* stream);

/*
 * fa_selftest_exp2_poly -- evaluate, on n device floats x, the 2^x that the
 * softmax kernels compute on the FMA pipe (Cody-Waite range reduction plus a
 * degree-3 minimax polynomial), writing y.  Relative error below 1e-4 for x
 * in [-125, 16]; x below -126 gives a non-negative value under 2^-125.
 * Exposed so the approximation can be checked against a reference.  No
 * counterpart on the pages: an implementation detail of the kernels.
 */
int fa_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
