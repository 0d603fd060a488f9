// router.cu -- the router's decision for each token: top-K experts and their weights.
//
// Page "GLM-5-NVFP4-MTP", "Model Description": 256 experts, 8 active per token; the router
// itself stays in BF16 / fp32 ("What's quantized": only the routed experts are NVFP4).  The
// pages do not spell out the router's function; the one taken here is softmax over the E
// logits, the K largest probabilities (the lower expert index first among equal ones), and
// those K renormalised to sum to 1.  Softmax is increasing in the logit, so the selection is
// made on the fp32 logits themselves (exact comparisons), and the renormalised weight of a
// selected expert is exp(l_k - l_max) / sum over the selected j of exp(l_j - l_max): the
// softmax denominator over all E cancels.
//
// One warp per token.  Lane i holds logits i, i + 32, i + 64, ...; each of the K rounds
// takes the lane-local best of the untaken ones and then the warp-wide best by shuffles,
// ordered by (logit descending, index ascending).  Slot k of the output is the k-th pick.
#include "moe.cuh"

namespace nvfp4 {
namespace {

// (v, e) beats (w, f): larger logit, or the same logit and a lower index.
__device__ __forceinline__ bool better(float v, int e, float w, int f) {
  return v > w || (v == w && e < f);
}

template <int PER>   // logits per lane: E <= 32 * PER
__global__ void __launch_bounds__(256) router_kernel(const float *__restrict__ logits,
                                                     int64_t T, int E, int K,
                                                     int32_t *__restrict__ ids,
                                                     float *__restrict__ w) {
  pdl_wait();   // the logits may come from the previous kernel
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t < T) {
    const float *row = logits + t * E;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < E ? __ldg(row + e) : -INFINITY;
    }
    uint32_t taken = 0;   // bit i: logit lane + 32 i already picked (or past E)
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i >= E) taken |= 1u << i;
    float my_v = 0.f;     // lane k < K: the k-th pick
    int my_e = 0;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int be = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        if (!(taken >> i & 1u) && better(v[i], e, bv, be)) {
          bv = v[i];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
        if (better(ov, oe, bv, be)) {
          bv = ov;
          be = oe;
        }
      }
      if (be < E && (be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == k) {
        my_v = bv;
        my_e = be;
      }
    }
    const float top = __shfl_sync(0xFFFFFFFFu, my_v, 0);   // the largest logit
    const float p = lane < K ? expf(my_v - top) : 0.f;
    float s = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane < K) {
      ids[t * K + lane] = my_e;
      w[t * K + lane] = p / s;
    }
  }
  pdl_launch_dependents();
}

template <int PER>
int launch(const float *logits, int64_t T, int E, int K, int32_t *ids, float *w,
           cudaStream_t s) {
  const int64_t blocks = ceil_div(T * 32, 256);
  return launch_pdl(router_kernel<PER>, dim3((unsigned)blocks), dim3(256), 0, s, logits, T, E,
                    K, ids, w);
}

}  // namespace

int launch_router(const float *logits, int64_t T, int64_t E, int64_t K, int32_t *ids, float *w,
                  cudaStream_t s) {
  const int e = (int)E, k = (int)K;
  if (E <= 32) return launch<1>(logits, T, e, k, ids, w, s);
  if (E <= 64) return launch<2>(logits, T, e, k, ids, w, s);
  if (E <= 128) return launch<4>(logits, T, e, k, ids, w, s);
  if (E <= 256) return launch<8>(logits, T, e, k, ids, w, s);
  if (E <= 512) return launch<16>(logits, T, e, k, ids, w, s);
  return launch<32>(logits, T, e, k, ids, w, s);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int moe_nvfp4_router(const float *logits, int64_t T, int64_t E, int64_t K,
                                int32_t *topk_ids, float *topk_w, cudaStream_t stream) {
  if (!logits || !topk_ids || !topk_w || T <= 0 || E <= 0 || K <= 0) return NVFP4_EINVAL;
  if (E > kMaxExperts || K > 16 || K > E || T * K >= (int64_t(1) << 31) ||
      T >= (int64_t(1) << 31) / 32)
    return NVFP4_ESHAPE;
  if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(topk_ids) |
       reinterpret_cast<uintptr_t>(topk_w)) & 3)
    return NVFP4_EINVAL;
  return launch_router(logits, T, E, K, topk_ids, topk_w, stream);
}
