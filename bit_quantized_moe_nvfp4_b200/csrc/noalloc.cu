// noalloc.cu -- moe_nvfp4_forward_static: the small-batch (GEMV) forward with a fixed,
// library-owned scratch instead of a caller workspace.
//
// The pages define the MoE layer, not its memory management: this entry point has no
// counterpart there.  It exists for callers that cannot hand the library any device memory
// -- e.g. a decode loop that has committed every free byte of HBM to its KV-cache pool and
// holds only the layer's own tensors, so it can neither allocate a workspace nor carve one
// out of a buffer it owns.  The kernels are the ones moe_nvfp4_forward runs on its GEMV
// path; only the scratch they write differs:
//   work [2] int32      work counters of the one-token gate/up kernel -> g_static_scratch
//   h   [T*K, I] bf16   SwiGLU outputs, one row per routed pair    -> g_static_scratch + 256
//   y   [T*K, H] fp32   weighted expert outputs before the combine -> after h
//   flag                error bits                                 -> the caller's pointer
// Of the scratch only the two work counters at its start (read by the one-token gate/up
// kernel) have to be zero: they are zero when the library loads, and every call leaves them
// zero.  Nothing else has to start at zero: the gate/up kernel writes every h row the down
// kernel reads, the down kernel every y row the combine reads, and the flag is overwritten
// by each call.  The array keeps the rows of the last call after it ends.  There is ONE
// array per device, shared by every call on that device: calls on one stream are ordered
// and safe; calls that can overlap (different streams or host threads on the same device)
// race on it.
#include <mutex>

#include "moe.cuh"

namespace nvfp4 {
namespace {

constexpr int64_t kStaticBytes = NVFP4_STATIC_SCRATCH_BYTES;   // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

std::mutex g_lookup_mu;
void *g_static_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device.
// The lookup may load this library's device code, which is why the first call on a device
// has to come before any stream capture on it begins.
int static_scratch(unsigned char **base) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_EINVAL;
  std::lock_guard<std::mutex> lock(g_lookup_mu);
  if (!g_static_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      set_last_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return NVFP4_ECUDA;
    }
    g_static_addr[dev] = p;
  }
  *base = static_cast<unsigned char *>(g_static_addr[dev]);
  return NVFP4_OK;
}

// Bytes of the counter block and of h (each rounded up to 256): h and y follow the counters.
constexpr int64_t kStaticHead = 256;
int64_t static_h_bytes(int64_t pairs, int64_t I) { return (pairs * I * 2 + 255) & ~int64_t(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" int moe_nvfp4_forward_static(const __nv_bfloat16 *x, const int32_t *topk_ids,
                                        const float *topk_w, int64_t T, int64_t H, int64_t I,
                                        int64_t E, int64_t K, const uint8_t *w_gu,
                                        const uint8_t *s_gu, const float *g_gu,
                                        const uint8_t *w_dn, const uint8_t *s_dn,
                                        const float *g_dn, __nv_bfloat16 *out,
                                        int32_t *error_flag, cudaStream_t stream) {
  if (!x || !topk_ids || !topk_w || !w_gu || !s_gu || !g_gu || !w_dn || !s_dn || !g_dn || !out)
    return NVFP4_EINVAL;
  if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0) return NVFP4_EINVAL;
  if (H % 64 || I % 64 || K > 16 || E > kMaxExperts || T * K >= (int64_t(1) << 31))
    return NVFP4_ESHAPE;
  if (!aligned16(x) || !aligned16(w_gu) || !aligned16(w_dn) || !aligned16(out) ||
      !aligned16(s_gu) || !aligned16(s_dn) ||
      (reinterpret_cast<uintptr_t>(error_flag) & 3))
    return NVFP4_EINVAL;
  // the fixed scratch bounds the batch: counters, h (T*K*I bf16) and y (T*K*H fp32)
  if (!gemv_supported(T, H, I, K)) return NVFP4_ESHAPE;
  if (kStaticHead + static_h_bytes(T * K, I) + T * K * H * 4 > kStaticBytes) return NVFP4_ESHAPE;

  unsigned char *base = nullptr;
  if (int s = static_scratch(&base)) return s;

  MoeArgs a = {};
  a.x = x;
  a.ids = topk_ids;
  a.w = topk_w;
  a.w_gu = w_gu;
  a.s_gu = s_gu;
  a.g_gu = g_gu;
  a.w_dn = w_dn;
  a.s_dn = s_dn;
  a.g_dn = g_dn;
  a.out = out;
  a.T = T;
  a.H = H;
  a.I = I;
  a.E = E;
  a.K = K;
  a.map = whole_layer(E);
  a.flag = error_flag;   // may be NULL: the kernels then skip the flag writes
  a.work = reinterpret_cast<int32_t *>(base);
  a.h = reinterpret_cast<__nv_bfloat16 *>(base + kStaticHead);
  a.y = reinterpret_cast<float *>(base + kStaticHead + static_h_bytes(T * K, I));
  if (int s = launch_gemv_gateup(a, stream)) return s;
  if (int s = launch_gemv_down(a, stream)) return s;
  return gemv_fused_combine(T) ? NVFP4_OK : launch_combine_pairs(a, stream);
}
