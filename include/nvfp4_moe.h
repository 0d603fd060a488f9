/*
 * nvfp4_moe.h -- C ABI of the NVFP4 routed-expert MoE library (sm_100a).
 *
 * What the library computes is defined on page "GLM-5-NVFP4-MTP":
 *   "Model Description" -- the expert weights are NVFP4: 4-bit values with one FP8 scale per
 *                          16 consecutive elements; each MoE layer has 256 experts, 8 active
 *                          per token.
 *   "What's quantized"  -- only the routed experts' gate, up and down projections are NVFP4.
 * The format is fixed as: E2M1 elements, E4M3 ("FN", finite) block scales, one fp32 global
 * scale g per tensor, block scale = (block amax / 6) / g rounded to E4M3 (nearest, ties to
 * even, saturating at 448), g = tensor amax / (6 * 448) (1 for an all-zero tensor).
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers owned by the caller unless a parameter says "host".
 *     The library never allocates or frees memory; scratch comes from a caller workspace
 *     sized by the matching *_workspace_size() query, except for moe_nvfp4_forward_static,
 *     which uses one fixed array per device compiled into the library.
 *   - Calls are asynchronous on `stream`: they enqueue kernels and return without waiting.
 *   - The return value is a status: NVFP4_OK (0) on success.  On a negative status nothing
 *     was enqueued (argument checks run before any launch), except NVFP4_ECUDA, which reports
 *     a failed launch; nvfp4_last_cuda_error() then names the CUDA error.
 *   - Layouts are row-major.  A packed row stores element 2j in the LOW nibble of byte j and
 *     element 2j+1 in the HIGH nibble.  Block scales run along the contiguous dimension.
 *   - The library keeps no global state apart from a per-thread copy of the last CUDA error,
 *     the fixed array of moe_nvfp4_forward_static and a cache of per-kernel launch
 *     attributes (occupancy); calls on different streams may run concurrently if their
 *     workspaces differ.
 */
#ifndef NVFP4_MOE_H
#define NVFP4_MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status codes */
#define NVFP4_OK 0
#define NVFP4_EINVAL -1      /* null pointer, negative or zero dimension, bad path value */
#define NVFP4_ESHAPE -2      /* a dimension that must be a multiple of 16/32 is not, or a
                                size above a documented limit */
#define NVFP4_EWORKSPACE -3  /* workspace pointer null or smaller than the query says */
#define NVFP4_ECUDA -4       /* a kernel launch failed; see nvfp4_last_cuda_error() */

/* Human-readable name of a status code (static string). */
NVFP4_API const char *nvfp4_status_string(int status);

/* Text of the last CUDA error seen by a call on this host thread ("no error" if none). */
NVFP4_API const char *nvfp4_last_cuda_error(void);

/* ---------------------------------------------------------------- codec */

/* Bytes of workspace nvfp4_quantize needs: an error word, a per-tensor amax accumulator and
 * a per-tensor count of merged amax shares.  After the call, the first int32 of the
 * workspace is 0, or has bit 1 set if a device-side wait gave up (the outputs are then
 * invalid); it can be read with moe_nvfp4_read_error_flag. */
NVFP4_API size_t nvfp4_quantize_workspace_size(int64_t n_tensors, int64_t rows, int64_t cols);

/* Quantize n_tensors bf16 tensors of shape [rows, cols] to NVFP4 (page "GLM-5-NVFP4-MTP",
 * "Model Description": 4-bit values, one FP8 scale per 16 elements).
 *   x            [n_tensors, rows, cols] bf16
 *   packed       [n_tensors, rows, cols/2] E2M1 codes, two per byte (low nibble first)
 *   scales       [n_tensors, rows, cols/16] E4M3 codes
 *   global_scale [n_tensors] fp32, g = amax / 2688 (1.0 for an all-zero tensor)
 * Per 16-element block: s = (amax_b / 6) / g -> E4M3 (nearest, ties to even, saturating);
 * d = decoded s * g; code_i = E2M1(x_i / d) (nearest, ties to even, saturating at 6, sign
 * kept, so a small negative value gives 0x8); all codes 0 when d == 0.  Every step is an
 * IEEE fp32 operation rounded to nearest even, so results are reproducible bit for bit.
 * One cooperative kernel reads each tensor from HBM once: the quantize pass of a tensor
 * follows its amax pass while the tensor is still in L2.
 * Requires cols % 32 == 0.  NaN/Inf inputs give unspecified codes.
 * Alignment: x 16 bytes, packed 8 bytes, global_scale and workspace 4 bytes.
 * Errors: EINVAL (null pointer, dimension <= 0, misaligned pointer), ESHAPE (cols % 32 != 0),
 * EWORKSPACE (ws_bytes < nvfp4_quantize_workspace_size). */
NVFP4_API int nvfp4_quantize(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows, int64_t cols,
                   uint8_t *packed, uint8_t *scales, float *global_scale,
                   void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Dequantize NVFP4 to bf16 (page "GLM-5-NVFP4-MTP", "Model Description": each weight is a
 * 4-bit value times the FP8 scale of its 16-element block, times the tensor's fp32 scale):
 * out = bf16( fp32(e2m1 * e4m3) * g ), the first product exact, the multiply by g rounded
 * once in fp32, then rounded to bf16 (nearest even).
 * Shapes as in nvfp4_quantize; requires cols % 32 == 0.  Alignment: packed and out 16
 * bytes, scales 2 bytes.  Errors: EINVAL (null or misaligned pointer), ESHAPE. */
NVFP4_API int nvfp4_dequantize(const uint8_t *packed, const uint8_t *scales, const float *global_scale,
                     int64_t n_tensors, int64_t rows, int64_t cols, __nv_bfloat16 *out,
                     cudaStream_t stream);

/* Calibrated (static) global scales (page "GLM-5-NVFP4-MTP", "Calibration dataset":
 * several calibration passes, merged by element-wise max).
 *
 * nvfp4_amax: amax[t] = max |x| over tensor t of x [n_tensors, rows, cols] bf16 (exact).
 * With merge == 0 amax is overwritten; with merge != 0 it becomes the element-wise max of
 * its current value and this pass's, so one call per calibration pass on the same array
 * leaves the merged amax.  amax: [n_tensors] fp32, device.  Requires cols % 32 == 0.
 * Alignment: x 16 bytes, amax 4 bytes.  Errors: EINVAL, ESHAPE, ECUDA. */
NVFP4_API int nvfp4_amax(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows, int64_t cols,
                         float *amax, int merge, cudaStream_t stream);

/* nvfp4_quantize with the tensor amax given (e.g. from nvfp4_amax over calibration data)
 * instead of measured on x: g[t] = amax[t] / 2688 (1.0 for 0), written to global_scale,
 * then every block exactly as nvfp4_quantize takes it.  Data beyond the calibrated range
 * saturates (a block scale above 448 is stored as 448, an element above 6 * d as 6).
 * One read of x; no workspace.  amax[t] must be finite and >= 0 (other values give
 * unspecified codes).  Shapes, layout and alignment as nvfp4_quantize (x 16 bytes, packed
 * 8 bytes, amax and global_scale 4 bytes).
 * Errors: EINVAL, ESHAPE, ECUDA. */
NVFP4_API int nvfp4_quantize_with_amax(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows,
                                       int64_t cols, const float *amax, uint8_t *packed,
                                       uint8_t *scales, float *global_scale,
                                       cudaStream_t stream);

/* Scalar format casts, element by element, exactly as the quantizer takes them:
 * e4m3[i] = E4M3(in[i]) and e2m1[i] = E2M1(in[i]) (nearest, ties to even, saturating,
 * sign kept; one code per byte in the low nibble for E2M1).  Either output may be NULL.
 * Errors: EINVAL (in NULL or n <= 0). */
NVFP4_API int nvfp4_cast_f32(const float *in, int64_t n, uint8_t *e4m3, uint8_t *e2m1,
                   cudaStream_t stream);

/* ---------------------------------------------------------------- MoE layer */

/* Routed-expert MoE MLP of one layer, run directly from NVFP4 expert weights (page
 * "GLM-5-NVFP4-MTP", "Model Description": 256 experts, 8 active per token; "What's
 * quantized": gate, up and down projections are NVFP4).  For token t:
 *   out[t] = sum over k = 0..K-1 of topk_w[t,k] * y_k, with e = topk_ids[t,k] and
 *   a   = g_gu[e] * (W_gu[e] x_t)        2I values: rows 0..I-1 gate, rows I..2I-1 up
 *   h_j = bf16( silu(a_j) * a_{I+j} )     SwiGLU, rounded to bf16
 *   y_k = g_dn[e] * (W_dn[e] h)           H values
 * where each weight is its exact NVFP4 value e2m1 * e4m3 (products accumulate in fp32).
 * Ids outside [0, E) contribute nothing and set the workspace error flag
 * (moe_nvfp4_read_error_flag).  A repeated id within a token counts once per slot.
 *   x        [T, H] bf16            topk_ids [T, K] int32      topk_w [T, K] fp32
 *   w_gu     [E, 2I, H/2] u8        s_gu [E, 2I, H/16] E4M3    g_gu [E] fp32
 *   w_dn     [E, H, I/2] u8         s_dn [E, H, I/16] E4M3     g_dn [E] fp32
 *   out      [T, H] bf16
 * Limits: H % 64 == 0, I % 64 == 0, 1 <= K <= 16, E <= 1024, T*K < 2^31.
 * Alignment: x, w_gu, s_gu, w_dn, s_dn, out and workspace 16 bytes (EINVAL /
 * EWORKSPACE otherwise).
 * Workspace: caller-owned device memory of moe_nvfp4_workspace_size bytes.  Its first
 * NVFP4_WORKSPACE_ZERO_BYTES bytes hold the error flag and two work counters of the
 * one-token kernels; they must be zero before the workspace's first call (cudaMemset), and
 * every call leaves the counters zero again.  The rest needs no initialisation.  Calls that
 * share a workspace must not overlap in time.
 * The call picks a memory-bound GEMV path for small T and a tensor-core grouped GEMM path
 * otherwise; both compute the same function.  It never synchronises with the host and
 * may be captured in a CUDA graph.
 * Errors: EINVAL, ESHAPE, EWORKSPACE (ws_bytes < moe_nvfp4_workspace_size), ECUDA. */
#define NVFP4_WORKSPACE_ZERO_BYTES 512
NVFP4_API size_t moe_nvfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int64_t K);

NVFP4_API int moe_nvfp4_forward(const __nv_bfloat16 *x, const int32_t *topk_ids, const float *topk_w,
                      int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                      const uint8_t *w_gu, const uint8_t *s_gu, const float *g_gu,
                      const uint8_t *w_dn, const uint8_t *s_dn, const float *g_dn,
                      __nv_bfloat16 *out, void *workspace, size_t ws_bytes,
                      cudaStream_t stream);

/* Paths of moe_nvfp4_forward_path. */
#define NVFP4_PATH_AUTO 0     /* what moe_nvfp4_forward does */
#define NVFP4_PATH_GEMV 1     /* dequant-fused grouped GEMV (CUDA cores at T = 1, mma.sync for
                                 T >= 2); T*K <= 1024, H <= 6144, I <= 6144 (3072 at T = 1) */
#define NVFP4_PATH_GEMM 2     /* dequant-to-shared-memory grouped GEMM (tcgen05), any T */

/* moe_nvfp4_forward with the path chosen by the caller (same arguments, same result up
 * to fp32 summation order).  Errors as moe_nvfp4_forward, plus EINVAL for a bad path and
 * ESHAPE for a shape outside the GEMV limits when that path is asked for. */
NVFP4_API int moe_nvfp4_forward_path(const __nv_bfloat16 *x, const int32_t *topk_ids,
                           const float *topk_w, int64_t T, int64_t H, int64_t I, int64_t E,
                           int64_t K, const uint8_t *w_gu, const uint8_t *s_gu,
                           const float *g_gu, const uint8_t *w_dn, const uint8_t *s_dn,
                           const float *g_dn, __nv_bfloat16 *out, void *workspace,
                           size_t ws_bytes, int path, cudaStream_t stream);

/* moe_nvfp4_forward_path with timing marks, for measurement.  stage_events points to five
 * cudaEvent_t (created by the caller, timing enabled) that are recorded on `stream`:
 * [0] before the route step, [1] after it, [2] after the gate/up + SwiGLU step, [3] after
 * the down step, [4] after the combine.  The events sit between the kernels, so the
 * kernels do not overlap their neighbours as they do in an unmarked call.  Under stream
 * capture the marks are recorded as external events, so they time each graph replay.
 * Errors as moe_nvfp4_forward_path, plus EINVAL for a null event. */
NVFP4_API int moe_nvfp4_forward_profiled(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                         const float *topk_w, int64_t T, int64_t H, int64_t I,
                                         int64_t E, int64_t K, const uint8_t *w_gu,
                                         const uint8_t *s_gu, const float *g_gu,
                                         const uint8_t *w_dn, const uint8_t *s_dn,
                                         const float *g_dn, __nv_bfloat16 *out,
                                         void *workspace, size_t ws_bytes, int path,
                                         void *const *stage_events, cudaStream_t stream);

/* ---------------------------------------------------------------- router */

/* The router's decision for each token (page "GLM-5-NVFP4-MTP", "Model Description":
 * 256 experts, 8 active per token; the router stays BF16 / fp32 per "What's quantized").
 * The pages do not state its function; the one computed is: p = softmax(logits[t, :]),
 * the K largest p in descending order with the lower expert index first among equal
 * values, and their weights p_k / (sum of the K selected p).  The selection compares the
 * fp32 logits themselves (softmax preserves their order), so it is exact; the weights are
 * fp32, exp(l_k - l_max) / sum of exp(l_j - l_max) over the selected j.
 *   logits    [T, E] fp32, finite (NaN or infinite logits give unspecified results)
 *   topk_ids  [T, K] int32 out: slot k = the k-th largest logit's expert
 *   topk_w    [T, K] fp32 out: positive, summing to 1 over a token's K slots
 * Limits: 1 <= K <= min(16, E), E <= 1024, T*K < 2^31.  Pointers 4-byte aligned.
 * Errors: EINVAL, ESHAPE, ECUDA. */
NVFP4_API int moe_nvfp4_router(const float *logits, int64_t T, int64_t E, int64_t K,
                               int32_t *topk_ids, float *topk_w, cudaStream_t stream);

/* moe_nvfp4_forward_path from router logits: the router above, then the layer on its
 * decisions (one stream-ordered chain, no host round trip).  topk_ids_out / topk_w_out
 * ([T, K], may be NULL) receive the decisions; when NULL they stay in the workspace.
 * Arguments, layouts, limits and errors otherwise as moe_nvfp4_forward_path (plus ESHAPE
 * for K > E). */
NVFP4_API int moe_nvfp4_forward_logits(const __nv_bfloat16 *x, const float *router_logits,
                                       int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                                       const uint8_t *w_gu, const uint8_t *s_gu,
                                       const float *g_gu, const uint8_t *w_dn,
                                       const uint8_t *s_dn, const float *g_dn,
                                       __nv_bfloat16 *out, int32_t *topk_ids_out,
                                       float *topk_w_out, void *workspace, size_t ws_bytes,
                                       int path, cudaStream_t stream);

/* ---------------------------------------------------------------- shared expert, layer */

/* The shared expert: a dense SwiGLU MLP in BF16 that every token passes through beside the
 * routed experts (page "GLM-5-NVFP4-MTP", "What's quantized": only the routed experts are
 * NVFP4; the rest of the model, shared experts included, stays BF16).  For every token t:
 *   h[t, j]   = bf16( silu(w_gu[j] . x_t) * (w_gu[Is + j] . x_t) )      j < Is
 *   out[t, n] = bf16( routed[t, n] + w_dn[n] . h[t] )                     n < H
 * with exact bf16 products and fp32 sums (the order of the fp32 sums is the kernel's).
 *   x       [T, H] bf16              w_gu [2 Is, H] bf16 (gate rows, then up rows)
 *   w_dn    [H, Is] bf16             routed [T, H] fp32, or NULL for 0 (e.g. the partial
 *                                    of moe_nvfp4_forward_ep, or a reduced sum of them)
 *   out     [T, H] bf16
 * Limits: H % 64 == 0, Is % 64 == 0, H and Is <= 65536; with T <= 8 the tokens' rows must
 * fit one CTA's shared memory (T * max(H, Is) * 2 bytes <= 227 KB, else ESHAPE).
 * Alignment: x, w_gu, w_dn, out and workspace 16 bytes; routed 4 bytes.
 * Workspace: moe_nvfp4_shared_workspace_size(T, Is) bytes (holds h), no initialisation.
 * Errors: EINVAL, ESHAPE, EWORKSPACE, ECUDA. */
NVFP4_API size_t moe_nvfp4_shared_workspace_size(int64_t T, int64_t Is);
NVFP4_API int moe_nvfp4_shared_expert(const __nv_bfloat16 *x, int64_t T, int64_t H, int64_t Is,
                                      const __nv_bfloat16 *w_gu, const __nv_bfloat16 *w_dn,
                                      const float *routed, __nv_bfloat16 *out, void *workspace,
                                      size_t ws_bytes, cudaStream_t stream);

/* The whole MoE layer in one stream-ordered call: the router on router_logits
 * (moe_nvfp4_router), the routed NVFP4 experts summed in fp32 (moe_nvfp4_forward_logits
 * before its rounding), and the shared expert added to that sum before the single rounding
 * to bf16:  out[t] = bf16( sum_k w[t,k] y_k(t) + shared(x_t) ).
 * Arguments as moe_nvfp4_forward_logits plus shared_gu [2 Is, H] / shared_dn [H, Is] bf16
 * and Is; limits of both.  Workspace: moe_nvfp4_layer_workspace_size bytes whose first
 * NVFP4_WORKSPACE_ZERO_BYTES are zero before its first use (the error flag, read with
 * moe_nvfp4_read_error_flag, is its first word).  Errors: EINVAL, ESHAPE, EWORKSPACE,
 * ECUDA. */
NVFP4_API size_t moe_nvfp4_layer_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E,
                                                int64_t K, int64_t Is);
NVFP4_API int moe_nvfp4_layer(const __nv_bfloat16 *x, const float *router_logits, int64_t T,
                              int64_t H, int64_t I, int64_t E, int64_t K, const uint8_t *w_gu,
                              const uint8_t *s_gu, const float *g_gu, const uint8_t *w_dn,
                              const uint8_t *s_dn, const float *g_dn,
                              const __nv_bfloat16 *shared_gu, const __nv_bfloat16 *shared_dn,
                              int64_t Is, __nv_bfloat16 *out, int32_t *topk_ids_out,
                              float *topk_w_out, void *workspace, size_t ws_bytes, int path,
                              cudaStream_t stream);

/* Copy the workspace error flag to *host_flag (host pointer) and wait for it:
 * 0 = no error, bit 0 = an id outside [0, E) was met, bit 1 = a device-side wait gave up.
 * The flag is cleared by the next moe_nvfp4_forward on that workspace.  Synchronises
 * `stream`.  Errors: EINVAL, ECUDA. */
NVFP4_API int moe_nvfp4_read_error_flag(const void *workspace, int32_t *host_flag, cudaStream_t stream);

/* The token permutation step on its own (the first step of moe_nvfp4_forward):
 *   counts[e]  = number of (t, k) with topk_ids[t,k] == e                  [E]
 *   offsets    = exclusive prefix sum of counts                             [E+1]
 *   perm       = flat pair indices t*K+k grouped by expert, ascending within
 *                an expert; entries past offsets[E] are left unwritten      [T*K]
 *   inv[t*K+k] = position of that pair in perm, -1 for an out-of-range id  [T*K]
 *   error_flag = bit 0 set when an id is out of range (may be NULL)         [1]
 * Limits: E <= 1024, 1 <= K <= 16, T*K < 2^31.  Errors: EINVAL, ESHAPE, ECUDA. */
NVFP4_API int moe_nvfp4_route(const int32_t *topk_ids, int64_t T, int64_t K, int64_t E,
                    int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                    int32_t *error_flag, cudaStream_t stream);

/* ---------------------------------------------------------------- expert parallelism */

/* Page "GLM-5-NVFP4-MTP", "How to Run", serves the model across several GPUs.  The routed
 * experts shard by expert: rank r of G ("ep_size") owns the experts e in [0, E) with
 * e mod G == r and stores expert e at local index e / G.  Every rank runs
 * moe_nvfp4_forward_ep on the same tokens and routing; the layer output is
 * bf16(sum over ranks of their fp32 partials), which moe_nvfp4_ep_reduce forms (over
 * peer-mapped partials, or as the rounding step after a library reduction of them). */
#define NVFP4_EP_MAX_PARTS 16

/* Number of experts rank ep_rank owns: ceil((E - ep_rank) / ep_size); 0 for E <= 0,
 * ep_size <= 0 or ep_rank outside [0, ep_size). */
NVFP4_API int64_t moe_nvfp4_ep_local_experts(int64_t E, int64_t ep_size, int64_t ep_rank);

/* The forward of rank ep_rank's experts only.  Arguments as moe_nvfp4_forward_path, except:
 *   E            the layer's expert count; topk_ids hold ids in [0, E)
 *   ep_size      ranks sharing the experts, 1 <= ep_size <= E
 *   ep_rank      this rank, 0 <= ep_rank < ep_size
 *   w_gu .. g_dn this rank's experts, local index l = expert l * ep_size + ep_rank:
 *                [E_loc, ...] with E_loc = moe_nvfp4_ep_local_experts(E, ep_size, ep_rank)
 *   out_partial  [T, H] fp32, 16-byte aligned: for every token the sum, over its slots k
 *                in ascending order whose expert this rank owns, of topk_w[t,k] * y(t,k),
 *                with y as in moe_nvfp4_forward; 0 for a token with none.
 * Slots routed to another rank's expert are skipped without error; ids outside [0, E) are
 * skipped and set bit 0 of the workspace error flag, as in moe_nvfp4_forward.  Workspace:
 * moe_nvfp4_workspace_size(T, H, I, E_loc, K) bytes (the size for E covers it).
 * With ep_size 1 the call computes moe_nvfp4_forward's sum before its bf16 rounding.
 * Errors: EINVAL (also ep_size / ep_rank out of range, null out_partial), ESHAPE,
 * EWORKSPACE, ECUDA. */
NVFP4_API int moe_nvfp4_forward_ep(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                   const float *topk_w, int64_t T, int64_t H, int64_t I,
                                   int64_t E, int64_t K, int64_t ep_size, int64_t ep_rank,
                                   const uint8_t *w_gu, const uint8_t *s_gu, const float *g_gu,
                                   const uint8_t *w_dn, const uint8_t *s_dn, const float *g_dn,
                                   float *out_partial, void *workspace, size_t ws_bytes,
                                   int path, cudaStream_t stream);

/* out = bf16_RN(partials[0] + partials[1] + ... + partials[n_parts-1]), elementwise, in
 * fp32 and in that order (deterministic whichever rank finished first).
 *   partials  HOST array of n_parts device pointers, each [rows, cols] fp32 row-major,
 *             16-byte aligned; a pointer may be another GPU's memory that this device can
 *             read (peer access enabled, or an IPC / virtual-memory mapping)
 *   out       [rows, cols] bf16, 8-byte aligned, on this device; must not overlap a partial
 * Limits: 1 <= n_parts <= NVFP4_EP_MAX_PARTS, cols % 4 == 0.  rows == 0 enqueues nothing.
 * The caller orders the call after every partial is complete (an event or a barrier across
 * ranks) and keeps the partials unchanged until it has run.
 * Errors: EINVAL (null or misaligned pointer, n_parts <= 0, rows < 0, cols <= 0), ESHAPE,
 * ECUDA. */
NVFP4_API int moe_nvfp4_ep_reduce(const float *const *partials, int64_t n_parts, int64_t rows,
                                  int64_t cols, __nv_bfloat16 *out, cudaStream_t stream);

/* ---------------------------------------------------------------- W4A4 (FP4 tensor cores) */

/* The routed layer on the block-scaled FP4 tensor cores (tcgen05.mma kind::mxf4nvf4).  Page
 * "GLM-5-NVFP4-MTP", "How to Run", serves the NVFP4 checkpoint with ModelOpt FP4 quantization
 * and FP4 MoE kernels.  The activations are quantized to NVFP4 on the fly.  Each activation
 * row (a token's x for gate/up, a routed pair's bf16 h for down) is quantized as a tensor of
 * its own: global scale amax(row) / 2688, E4M3 scale per 16, E2M1 codes, exactly as
 * nvfp4_quantize.  Its exact NVFP4 values multiply the exact NVFP4 weights with fp32
 * accumulation.  This computes a different function from moe_nvfp4_forward, whose
 * activations stay bf16; the pages fix no activation format.
 *
 * The tensor cores take block scales in their own layout.  nvfp4_w4a4_prepare_scales
 * rearranges a weight tensor's E4M3 scales ([n, rows, cols/16], as nvfp4_quantize writes
 * them) into it, once per weight: one 512-byte atom per 128 rows and 64 columns, row r's four
 * scales in the 32-bit word at byte 16 (r % 32) + 4 (r / 32).  gate_rows = I for a fused
 * gate/up weight [2I, cols], whose atom group m then holds gate rows 64m.. and up rows
 * I + 64m..; gate_rows = 0 for a plain weight (group m = rows 128m..).  out has the size of
 * scales.  Limits: rows % 128 == 0, cols % 64 == 0; 4-byte aligned pointers.
 * Errors: EINVAL, ESHAPE, ECUDA. */
NVFP4_API int nvfp4_w4a4_prepare_scales(const uint8_t *scales, int64_t n_tensors, int64_t rows,
                                        int64_t cols, int64_t gate_rows, uint8_t *out,
                                        cudaStream_t stream);

/* The W4A4 forward.  Arguments as moe_nvfp4_forward, except that sf_gu / sf_dn are the
 * prepared scales (nvfp4_w4a4_prepare_scales with gate_rows I, resp. 0).  Runs the
 * tensor-core path for any T.  Limits: H % 256 == 0, I % 256 == 0, K <= 16, E <= 1024.
 * Workspace: moe_nvfp4_w4a4_workspace_size bytes, first NVFP4_WORKSPACE_ZERO_BYTES zero
 * before first use (the error flag is its first word, as for moe_nvfp4_forward).
 * Errors: EINVAL, ESHAPE, EWORKSPACE, ECUDA. */
NVFP4_API size_t moe_nvfp4_w4a4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E,
                                               int64_t K);
NVFP4_API int moe_nvfp4_forward_w4a4(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                     const float *topk_w, int64_t T, int64_t H, int64_t I,
                                     int64_t E, int64_t K, const uint8_t *w_gu,
                                     const uint8_t *sf_gu, const float *g_gu,
                                     const uint8_t *w_dn, const uint8_t *sf_dn,
                                     const float *g_dn, __nv_bfloat16 *out, void *workspace,
                                     size_t ws_bytes, cudaStream_t stream);

/* moe_nvfp4_forward_w4a4 with timing marks: five caller events recorded on `stream` before
 * the route step, after the x quantization, after the gate/up GEMM, after the h quantization
 * and down GEMM, and after the combine.  Errors as moe_nvfp4_forward_w4a4, plus EINVAL for a
 * null event. */
NVFP4_API int moe_nvfp4_forward_w4a4_profiled(
    const __nv_bfloat16 *x, const int32_t *topk_ids, const float *topk_w, int64_t T, int64_t H,
    int64_t I, int64_t E, int64_t K, const uint8_t *w_gu, const uint8_t *sf_gu, const float *g_gu,
    const uint8_t *w_dn, const uint8_t *sf_dn, const float *g_dn, __nv_bfloat16 *out,
    void *workspace, size_t ws_bytes, void *const *stage_events, cudaStream_t stream);

/* ---------------------------------------------------------------- fixed-scratch forward */

/* Bytes of the fixed scratch of moe_nvfp4_forward_static: it holds 256 bytes of counters,
 * T*K rows of I bf16 values (rounded up to 256 bytes) and T*K rows of H fp32 values, so a
 * call needs 256 + roundup256(2*T*K*I) + 4*T*K*H <= 4 MiB (at H = 6144, I = 2048, K = 8:
 * T <= 18). */
#define NVFP4_STATIC_SCRATCH_BYTES 4194304

/* The small-batch forward of moe_nvfp4_forward (its GEMV path: same kernels, same result)
 * without a caller workspace.  The pages have no counterpart to this call: it exists for
 * callers that cannot hand the library any device memory, such as a decode loop that has
 * committed all free memory to its KV-cache pool and holds only the layer's tensors.
 * Arguments, layouts, alignment and the computed function are those of moe_nvfp4_forward,
 * except:
 *   error_flag  [1] int32, may be NULL: receives what the workspace flag of
 *               moe_nvfp4_forward would (0, bit 0 = an id outside [0, E), bit 1 = a
 *               device-side wait gave up); overwritten by every call; 4-byte aligned.
 * Scratch: one array of NVFP4_STATIC_SCRATCH_BYTES per device, inside the library; no
 * call allocates or frees memory.  Only its first 8 bytes (the work counters of the
 * one-token kernels) must be zero at a call: they are zero when the library loads and every
 * call leaves them zero.  It keeps the last call's intermediate values after that call
 * ends.  All calls on a device share it, so calls that can overlap in time (different
 * streams, or different host threads, on the same device) race; calls on one stream are
 * ordered and safe.  The first call on each device looks the array's address up
 * (cudaGetSymbolAddress): make that first call before any stream capture begins on that
 * device.
 * Errors: EINVAL (null or misaligned pointer, dimension <= 0), ESHAPE (the limits of
 * moe_nvfp4_forward, a batch whose h and y do not fit NVFP4_STATIC_SCRATCH_BYTES, or a
 * shape the GEMV path does not take: T*K > 1024, H > 6144, I > 6144, or I > 3072 with
 * T = 1), ECUDA. */
NVFP4_API int moe_nvfp4_forward_static(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                       const float *topk_w, int64_t T, int64_t H, int64_t I,
                                       int64_t E, int64_t K, const uint8_t *w_gu,
                                       const uint8_t *s_gu, const float *g_gu,
                                       const uint8_t *w_dn, const uint8_t *s_dn,
                                       const float *g_dn, __nv_bfloat16 *out,
                                       int32_t *error_flag, cudaStream_t stream);

/* ---------------------------------------------------------------- test hook */

/* Runs the device-side failure path on purpose (the pages have no counterpart; this
 * is test infrastructure for the library's bounded waits).  One kernel waits, with nothing
 * to complete the wait, for
 *   kind 0: an mbarrier phase that no thread arrives at;
 *   kind 1: the bytes a barrier arrival announced, from a copy that is never issued;
 *   kind 2: a global counter that no CTA advances,
 * each bounded by limit_ns nanoseconds of %globaltimer instead of the kernels' 2 s.  When
 * the limit runs out the kernel ORs bit 1 (NVFP4 "a device-side wait gave up") into *flag
 * and returns; nothing faults and the CUDA context stays usable.  flag is a device int32
 * (e.g. the first word of a forward workspace, so moe_nvfp4_read_error_flag reads it and the
 * next forward on that workspace clears it), 4-byte aligned.
 * Errors: EINVAL (null or misaligned flag, kind outside 0..2, limit_ns outside
 * 1..1000000000), ECUDA. */
NVFP4_API int nvfp4_selftest_wait_timeout(int32_t *flag, int kind, int64_t limit_ns,
                                          cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_MOE_H */
