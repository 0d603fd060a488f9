// moe.cuh -- arguments and workspace layout shared by the MoE forward kernels.
#pragma once
#include "route.cuh"

namespace nvfp4 {

// Everything one forward call needs on the device.  Weight pointers are the caller's;
// the int32 / bf16 / fp32 scratch arrays live in the caller's workspace.
struct MoeArgs {
  // inputs
  const __nv_bfloat16 *x;     // [T, H]
  const int32_t *ids;         // [T, K]
  const float *w;             // [T, K]
  const uint8_t *w_gu;        // [E, 2I, H/2]
  const uint8_t *s_gu;        // [E, 2I, H/16]
  const float *g_gu;          // [E]
  const uint8_t *w_dn;        // [E, H, I/2]
  const uint8_t *s_dn;        // [E, H, I/16]
  const float *g_dn;          // [E]
  __nv_bfloat16 *out;         // [T, H]
  float *out_f32;             // [T, H] fp32 partial output instead of out (expert parallel),
                              //   or null
  int64_t T, H, I, E, K;      // E: experts on this device (the length of the weight arrays)
  ExpertMap map;              // routed (global) id -> local expert
  // workspace
  int32_t *flag;              // [1] error bits
  int32_t *work;              // [2] work counters of the one-token gate/up kernel (zero)
  int32_t *n_active;          // [1]
  int32_t *counts;            // [E]
  int32_t *offsets;           // [E+1]
  int32_t *active;            // [E]
  int32_t *tile_prefix;       // [E+1]
  int32_t *perm;              // [T*K]  pair index t*K+k, grouped by expert
  int32_t *inv;               // [T*K]  position of pair t*K+k in perm
  __nv_bfloat16 *h;           // [T*K, I]   SwiGLU output, rows in perm order
  float *y;                   // [T*K, H]   w * g_dn * (W_dn h), rows in perm order
  __half *xs;                 // [T*K + pad, H]  x gathered in perm order, f16, row r
                              //   scaled by 1/xscale[r] (GEMM path)
  float *xscale;              // [T*K]  2^-p of each gathered row (GEMM path)
};

// Workspace carve-up (byte offsets, each 256-aligned).
struct WorkspaceLayout {
  size_t flag, work, n_active, counts, offsets, active, tile_prefix, perm, inv, h, y, xs, xscale,
      rids, rw, route_blk, total;
};
WorkspaceLayout workspace_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t K);
constexpr int kGatherPadRows = 256;

// GEMV path (decode.cu): routing fused into both kernels, combine fused into the second
bool gemv_supported(int64_t T, int64_t H, int64_t I, int64_t K);
int launch_gemv_gateup(const MoeArgs &a, cudaStream_t s);
int launch_gemv_down(const MoeArgs &a, cudaStream_t s);
bool gemv_fused_combine(int64_t T);   // the GEMV down kernel also combines (no combine launch)
// The routed layer from router logits with its fp32 sum (before the bf16 rounding) written
// to out_f32 (api.cu); the shared expert's down step adds to it and rounds.
int forward_logits_partial(const __nv_bfloat16 *x, const float *logits, int64_t T, int64_t H,
                           int64_t I, int64_t E, int64_t K, const uint8_t *w_gu,
                           const uint8_t *s_gu, const float *g_gu, const uint8_t *w_dn,
                           const uint8_t *s_dn, const float *g_dn, float *out_f32,
                           int32_t *ids_out, float *w_out, void *workspace, size_t ws_bytes,
                           int path, cudaStream_t stream);
// router (router.cu): top-K of each token's E logits, renormalised softmax weights
int launch_router(const float *logits, int64_t T, int64_t E, int64_t K, int32_t *ids, float *w,
                  cudaStream_t s);
// combine of the GEMM path (combine.cu)
int launch_combine(const MoeArgs &a, cudaStream_t s);
int launch_combine_pairs(const MoeArgs &a, cudaStream_t s);   // y indexed by pair (GEMV path)
// GEMM path (gemm.cu)
int launch_gemm_gateup(const MoeArgs &a, cudaStream_t s);   // gather + gate/up + SwiGLU
int launch_gemm_down(const MoeArgs &a, cudaStream_t s);
int gemm_tile_n();

// SM count of the current device, and blocks of kernel `fn` that fit on one SM with this
// block size and dynamic shared memory (after raising the kernel's shared-memory limit to at
// least `smem`); both cached per device.  resident_blocks returns -1 on a CUDA error.
int num_sms();
int resident_blocks_fn(const void *fn, int threads, size_t smem);
template <typename Kern>
int resident_blocks(Kern k, int threads, size_t smem) {
  return resident_blocks_fn(reinterpret_cast<const void *>(k), threads, smem);
}

// Launch with programmatic dependent launch enabled (the kernel must call pdl_wait()
// before it reads what the previous kernel wrote).
template <typename Kern, typename... Args>
int launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

}  // namespace nvfp4
