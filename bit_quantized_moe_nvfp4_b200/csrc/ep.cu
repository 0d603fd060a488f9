// ep.cu -- the exchange step of the expert-parallel forward: sum the ranks' fp32 partial
// outputs and round once to the bf16 layer output.
//
// Page "GLM-5-NVFP4-MTP", "How to Run": the model is served across several GPUs at once.
// The routed experts shard by expert: rank g of G owns the experts e with e mod G == g, and
// its forward (moe_nvfp4_forward_ep) leaves out_g[t] = sum over its own pairs (t, k), k
// ascending, of w[t,k] * y[t,k] in fp32.  The layer output is bf16(sum over g of out_g).
// This kernel takes that sum over any number of partial arrays in index order, so the
// result does not depend on which rank finished first.  A partial may be another GPU's
// memory mapped into this one (peer access): the loads are plain global loads, never a
// multicast copy.  With one partial it is the rounding step after a library reduction
// (e.g. a reduce-scatter) has already summed the ranks.
#include "moe.cuh"

namespace nvfp4 {
namespace {

struct Parts {
  const float *p[NVFP4_EP_MAX_PARTS];
  int n;
};

__global__ void __launch_bounds__(256) ep_reduce_kernel(Parts parts, int64_t n4,
                                                         __nv_bfloat16 *out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4 *>(parts.p[0])[i];
    for (int j = 1; j < parts.n; ++j) {
      const float4 v = reinterpret_cast<const float4 *>(parts.p[j])[i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2 *>(out)[i] = o;
  }
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" int moe_nvfp4_ep_reduce(const float *const *partials, int64_t n_parts, int64_t rows,
                                   int64_t cols, __nv_bfloat16 *out, cudaStream_t stream) {
  if (!partials || !out || n_parts <= 0 || rows < 0 || cols <= 0) return NVFP4_EINVAL;
  if (n_parts > NVFP4_EP_MAX_PARTS || cols % 4) return NVFP4_ESHAPE;
  if (rows > (int64_t(1) << 40) / cols) return NVFP4_ESHAPE;
  if (reinterpret_cast<uintptr_t>(out) & 7) return NVFP4_EINVAL;
  Parts parts = {};
  parts.n = (int)n_parts;
  for (int64_t j = 0; j < n_parts; ++j) {
    if (!partials[j] || (reinterpret_cast<uintptr_t>(partials[j]) & 15)) return NVFP4_EINVAL;
    parts.p[j] = partials[j];
  }
  const int64_t n4 = rows * cols / 4;
  if (n4 == 0) return NVFP4_OK;
  const int sms = num_sms();
  if (sms <= 0) return NVFP4_ECUDA;
  int64_t blocks = ceil_div(n4, 256);
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  ep_reduce_kernel<<<(unsigned)blocks, 256, 0, stream>>>(parts, n4, out);
  return check_launch();
}
