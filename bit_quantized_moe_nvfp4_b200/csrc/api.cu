// api.cu -- status handling, workspace layout and the moe_nvfp4_forward entry points.
//
// The forward runs the routed-expert MoE MLP of page "GLM-5-NVFP4-MTP" ("Model
// Description": 256 experts, 8 active per token, NVFP4 expert weights) as a chain of
// stream-ordered kernels:
//   route (histogram + scan + stable scatter) -> gate/up + SwiGLU -> down -> combine
// with either the GEMV kernels (decode.cu) or the tensor-core GEMM kernels (gemm.cu) for
// the two projections.  Every kernel after the first is launched with programmatic
// dependent launch, so its prologue overlaps the previous kernel's tail.
#include <cstdio>
#include <cstring>

#include "moe.cuh"

namespace nvfp4 {

static thread_local char g_last_error[256] = "no error";

void set_last_cuda_error(cudaError_t e) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}

int check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

WorkspaceLayout workspace_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t K) {
  WorkspaceLayout L = {};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += align256(bytes);
    return at;
  };
  const size_t TK = (size_t)(T * K);
  L.flag = take(4);
  L.work = take(8);   // zero before first use; every call leaves it zero
  L.n_active = take(4);
  L.counts = take(4 * (size_t)E);
  L.offsets = take(4 * (size_t)(E + 1));
  L.active = take(4 * (size_t)E);
  L.tile_prefix = take(4 * (size_t)(E + 1));
  L.perm = take(4 * TK);
  L.inv = take(4 * TK);
  L.h = take(2 * (TK + kGatherPadRows) * (size_t)I);   // rows past T*K: tile overhang
  L.y = take(4 * TK * (size_t)H);
  L.xs = take(2 * (TK + kGatherPadRows) * (size_t)H);
  L.xscale = take(4 * TK);
  L.rids = take(4 * TK);   // router decisions when the call starts from logits
  L.rw = take(4 * TK);
  L.route_blk = take(4 * (size_t)route_scratch_ints(T * K, (int)E));   // many-CTA route
  L.total = o;
  return L;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Token count at or below which the GEMV kernels run (few tokens per expert).
constexpr int64_t kGemvMaxTokens = 64;

}  // namespace nvfp4

using namespace nvfp4;

extern "C" const char *nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_EINVAL: return "NVFP4_EINVAL: null pointer, bad dimension or bad path";
    case NVFP4_ESHAPE: return "NVFP4_ESHAPE: dimension not a required multiple or above a limit";
    case NVFP4_EWORKSPACE: return "NVFP4_EWORKSPACE: workspace missing or too small";
    case NVFP4_ECUDA: return "NVFP4_ECUDA: CUDA launch failed (see nvfp4_last_cuda_error)";
    default: return "unknown status";
  }
}

extern "C" const char *nvfp4_last_cuda_error(void) { return g_last_error; }

extern "C" size_t moe_nvfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E,
                                           int64_t K) {
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0) return 0;
  return workspace_layout(T, H, I, E, K).total;
}

// Record a timing mark.  Under stream capture an event record becomes a graph node only
// when recorded as an external event.
static int record(cudaEvent_t const *ev, int i, cudaStream_t s) {
  if (!ev) return NVFP4_OK;
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &st);
  if (e == cudaSuccess)
    e = (st == cudaStreamCaptureStatusActive)
            ? cudaEventRecordWithFlags(ev[i], s, cudaEventRecordExternal)
            : cudaEventRecord(ev[i], s);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}

// Experts of rank `rank` of `size` under the e mod size partition (0 for bad arguments).
static int64_t local_experts(int64_t E, int64_t size, int64_t rank) {
  if (E <= 0 || size <= 0 || rank < 0 || rank >= size) return 0;
  return (E - rank + size - 1) / size;
}

// Where the routing of a forward call comes from: the caller's ids and weights, or the
// router run on the caller's logits (its decisions written to ids_out / w_out, or to the
// workspace where those are null).
struct Routing {
  const int32_t *ids;
  const float *w;
  const float *logits;
  int32_t *ids_out;
  float *w_out;
};

// One forward call.  E is the layer's expert count; `ep_size` > 1 runs the experts of rank
// `ep_rank` only (the weight arrays then hold those experts) and writes the fp32 partial
// out_f32 instead of out.
static int forward_impl(const __nv_bfloat16 *x, const Routing &rt, int64_t T, int64_t H,
                        int64_t I, int64_t E, int64_t K, int64_t ep_size, int64_t ep_rank,
                        const uint8_t *w_gu, const uint8_t *s_gu, const float *g_gu,
                        const uint8_t *w_dn, const uint8_t *s_dn, const float *g_dn,
                        __nv_bfloat16 *out, float *out_f32, void *workspace, size_t ws_bytes,
                        int path, cudaEvent_t const *ev, cudaStream_t stream) {
  if (!x || (!rt.logits && (!rt.ids || !rt.w)) || !w_gu || !s_gu || !g_gu || !w_dn || !s_dn ||
      !g_dn || (!out && !out_f32))
    return NVFP4_EINVAL;
  if (rt.logits && (K > E || ((reinterpret_cast<uintptr_t>(rt.logits) |
                               reinterpret_cast<uintptr_t>(rt.ids_out) |
                               reinterpret_cast<uintptr_t>(rt.w_out)) & 3)))
    return K > E ? NVFP4_ESHAPE : NVFP4_EINVAL;
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0) return NVFP4_EINVAL;
  if (ep_size < 1 || ep_rank < 0 || ep_rank >= ep_size || ep_size > E) return NVFP4_EINVAL;
  if (path != NVFP4_PATH_AUTO && path != NVFP4_PATH_GEMV && path != NVFP4_PATH_GEMM)
    return NVFP4_EINVAL;
  if (H % 64 || I % 64 || K > 16 || E > kMaxExperts || T * K >= (int64_t(1) << 31))
    return NVFP4_ESHAPE;
  if (!aligned16(x) || !aligned16(w_gu) || !aligned16(w_dn) || !aligned16(out) ||
      !aligned16(out_f32) || !aligned16(s_gu) || !aligned16(s_dn))
    return NVFP4_EINVAL;
  const int64_t E_loc = local_experts(E, ep_size, ep_rank);
  const WorkspaceLayout L = workspace_layout(T, H, I, E_loc, K);
  if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return NVFP4_EWORKSPACE;

  char *ws = static_cast<char *>(workspace);
  MoeArgs a = {};
  a.x = x;
  a.ids = rt.ids;
  a.w = rt.w;
  int32_t *r_ids = nullptr;   // router output, when the call starts from logits
  float *r_w = nullptr;
  if (rt.logits) {
    r_ids = rt.ids_out ? rt.ids_out : reinterpret_cast<int32_t *>(ws + L.rids);
    r_w = rt.w_out ? rt.w_out : reinterpret_cast<float *>(ws + L.rw);
    a.ids = r_ids;
    a.w = r_w;
  }
  a.w_gu = w_gu;
  a.s_gu = s_gu;
  a.g_gu = g_gu;
  a.w_dn = w_dn;
  a.s_dn = s_dn;
  a.g_dn = g_dn;
  a.out = out;
  a.out_f32 = out_f32;
  a.T = T;
  a.H = H;
  a.I = I;
  a.E = E_loc;
  a.K = K;
  a.map = ExpertMap{(int)E, (int)ep_size, (int)ep_rank};
  a.flag = reinterpret_cast<int32_t *>(ws + L.flag);
  a.work = reinterpret_cast<int32_t *>(ws + L.work);
  a.n_active = reinterpret_cast<int32_t *>(ws + L.n_active);
  a.counts = reinterpret_cast<int32_t *>(ws + L.counts);
  a.offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
  a.active = reinterpret_cast<int32_t *>(ws + L.active);
  a.tile_prefix = reinterpret_cast<int32_t *>(ws + L.tile_prefix);
  a.perm = reinterpret_cast<int32_t *>(ws + L.perm);
  a.inv = reinterpret_cast<int32_t *>(ws + L.inv);
  a.h = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);
  a.y = reinterpret_cast<float *>(ws + L.y);
  a.xs = reinterpret_cast<__half *>(ws + L.xs);
  a.xscale = reinterpret_cast<float *>(ws + L.xscale);

  if (path == NVFP4_PATH_AUTO)
    path = (T <= kGemvMaxTokens && gemv_supported(T, H, I, K)) ? NVFP4_PATH_GEMV
                                                               : NVFP4_PATH_GEMM;
  if (path == NVFP4_PATH_GEMV && !gemv_supported(T, H, I, K)) return NVFP4_ESHAPE;

  if (int s = record(ev, 0, stream)) return s;
  if (rt.logits)
    if (int s = launch_router(rt.logits, T, E, K, r_ids, r_w, stream)) return s;
  if (path == NVFP4_PATH_GEMV) {
    // routing is recomputed inside each projection kernel, so there is no route launch
    if (int s = record(ev, 1, stream)) return s;
    if (int s = launch_gemv_gateup(a, stream)) return s;
    if (int s = record(ev, 2, stream)) return s;
    if (int s = launch_gemv_down(a, stream)) return s;
    if (int s = record(ev, 3, stream)) return s;
    if (!gemv_fused_combine(T))
      if (int s = launch_combine_pairs(a, stream)) return s;
    return record(ev, 4, stream);
  }

  RouteArgs r = {};
  r.ids = a.ids;
  r.n_pairs = T * K;
  r.E = (int)E_loc;
  r.map = a.map;
  r.counts = a.counts;
  r.offsets = a.offsets;
  r.perm = a.perm;
  r.inv = a.inv;
  r.flag = a.flag;
  r.active = a.active;
  r.n_active = a.n_active;
  r.tile_prefix = a.tile_prefix;
  r.tile_n = gemm_tile_n();
  if (int s = launch_route(r, stream, true, reinterpret_cast<int32_t *>(ws + L.route_blk)))
    return s;
  if (int s = record(ev, 1, stream)) return s;
  if (int s = launch_gemm_gateup(a, stream)) return s;
  if (int s = record(ev, 2, stream)) return s;
  if (int s = launch_gemm_down(a, stream)) return s;
  if (int s = record(ev, 3, stream)) return s;
  if (int s = launch_combine(a, stream)) return s;
  return record(ev, 4, stream);
}

namespace nvfp4 {
int forward_logits_partial(const __nv_bfloat16 *x, const float *logits, int64_t T, int64_t H,
                           int64_t I, int64_t E, int64_t K, const uint8_t *w_gu,
                           const uint8_t *s_gu, const float *g_gu, const uint8_t *w_dn,
                           const uint8_t *s_dn, const float *g_dn, float *out_f32,
                           int32_t *ids_out, float *w_out, void *workspace, size_t ws_bytes,
                           int path, cudaStream_t stream) {
  if (!logits || !out_f32) return NVFP4_EINVAL;
  const Routing rt = {nullptr, nullptr, logits, ids_out, w_out};
  return forward_impl(x, rt, T, H, I, E, K, 1, 0, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, nullptr,
                      out_f32, workspace, ws_bytes, path, nullptr, stream);
}
}  // namespace nvfp4

extern "C" int moe_nvfp4_forward_path(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                      const float *topk_w, int64_t T, int64_t H, int64_t I,
                                      int64_t E, int64_t K, const uint8_t *w_gu,
                                      const uint8_t *s_gu, const float *g_gu,
                                      const uint8_t *w_dn, const uint8_t *s_dn,
                                      const float *g_dn, __nv_bfloat16 *out, void *workspace,
                                      size_t ws_bytes, int path, cudaStream_t stream) {
  const Routing rt = {topk_ids, topk_w, nullptr, nullptr, nullptr};
  return forward_impl(x, rt, T, H, I, E, K, 1, 0, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, out,
                      nullptr, workspace, ws_bytes, path, nullptr, stream);
}

extern "C" int moe_nvfp4_forward_profiled(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                          const float *topk_w, int64_t T, int64_t H, int64_t I,
                                          int64_t E, int64_t K, const uint8_t *w_gu,
                                          const uint8_t *s_gu, const float *g_gu,
                                          const uint8_t *w_dn, const uint8_t *s_dn,
                                          const float *g_dn, __nv_bfloat16 *out,
                                          void *workspace, size_t ws_bytes, int path,
                                          void *const *stage_events, cudaStream_t stream) {
  if (!stage_events) return NVFP4_EINVAL;
  for (int i = 0; i < 5; ++i)
    if (!stage_events[i]) return NVFP4_EINVAL;
  const Routing rt = {topk_ids, topk_w, nullptr, nullptr, nullptr};
  return forward_impl(x, rt, T, H, I, E, K, 1, 0, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, out,
                      nullptr, workspace, ws_bytes, path,
                      reinterpret_cast<cudaEvent_t const *>(stage_events), stream);
}

extern "C" int moe_nvfp4_forward(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                 const float *topk_w, int64_t T, int64_t H, int64_t I, int64_t E,
                                 int64_t K, const uint8_t *w_gu, const uint8_t *s_gu,
                                 const float *g_gu, const uint8_t *w_dn, const uint8_t *s_dn,
                                 const float *g_dn, __nv_bfloat16 *out, void *workspace,
                                 size_t ws_bytes, cudaStream_t stream) {
  return moe_nvfp4_forward_path(x, topk_ids, topk_w, T, H, I, E, K, w_gu, s_gu, g_gu, w_dn,
                                s_dn, g_dn, out, workspace, ws_bytes, NVFP4_PATH_AUTO, stream);
}

extern "C" int64_t moe_nvfp4_ep_local_experts(int64_t E, int64_t ep_size, int64_t ep_rank) {
  return local_experts(E, ep_size, ep_rank);
}

extern "C" int moe_nvfp4_forward_ep(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                    const float *topk_w, int64_t T, int64_t H, int64_t I,
                                    int64_t E, int64_t K, int64_t ep_size, int64_t ep_rank,
                                    const uint8_t *w_gu, const uint8_t *s_gu, const float *g_gu,
                                    const uint8_t *w_dn, const uint8_t *s_dn, const float *g_dn,
                                    float *out_partial, void *workspace, size_t ws_bytes,
                                    int path, cudaStream_t stream) {
  if (!out_partial) return NVFP4_EINVAL;
  const Routing rt = {topk_ids, topk_w, nullptr, nullptr, nullptr};
  return forward_impl(x, rt, T, H, I, E, K, ep_size, ep_rank, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn,
                      nullptr, out_partial, workspace, ws_bytes, path, nullptr, stream);
}

extern "C" int moe_nvfp4_forward_logits(const __nv_bfloat16 *x, const float *router_logits,
                                        int64_t T, int64_t H, int64_t I, int64_t E, int64_t K,
                                        const uint8_t *w_gu, const uint8_t *s_gu,
                                        const float *g_gu, const uint8_t *w_dn,
                                        const uint8_t *s_dn, const float *g_dn,
                                        __nv_bfloat16 *out, int32_t *topk_ids_out,
                                        float *topk_w_out, void *workspace, size_t ws_bytes,
                                        int path, cudaStream_t stream) {
  if (!router_logits) return NVFP4_EINVAL;
  const Routing rt = {nullptr, nullptr, router_logits, topk_ids_out, topk_w_out};
  return forward_impl(x, rt, T, H, I, E, K, 1, 0, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, out,
                      nullptr, workspace, ws_bytes, path, nullptr, stream);
}

extern "C" int moe_nvfp4_read_error_flag(const void *workspace, int32_t *host_flag,
                                         cudaStream_t stream) {
  if (!workspace || !host_flag) return NVFP4_EINVAL;
  cudaError_t e = cudaMemcpyAsync(host_flag, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                  stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return NVFP4_OK;
}
