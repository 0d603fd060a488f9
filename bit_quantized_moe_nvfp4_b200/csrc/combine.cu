// combine.cu -- weighted top-k combine of the expert outputs of each token.
//
// Page "GLM-5-NVFP4-MTP", "Model Description": each token is served by 8 experts; its layer
// output is the routing-weighted sum of their outputs.  The down-projection kernels leave
// y[r] = w * g_dn * (W_dn h_r) for every routed pair r (in expert-grouped order), so here
// out[t] = bf16( sum over k = 0..K-1, ascending, of y[inv[t*K+k]] ) in fp32.  The fixed k
// order makes the result independent of which expert finished first.
#include "moe.cuh"

namespace nvfp4 {

namespace {

__global__ void __launch_bounds__(256) combine_kernel(MoeArgs a) {
  pdl_wait();
  const int64_t H = a.H, K = a.K;
  const int64_t n4 = H / 4;
  const int64_t total = a.T * n4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / n4, c = (i % n4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t k = 0; k < K; ++k) {
      const int pos = __ldg(a.inv + t * K + k);
      if (pos < 0) continue;
      const float4 v = __ldg(reinterpret_cast<const float4 *>(a.y + (int64_t)pos * H + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(a.out + t * H + c) = o;
  }
  pdl_launch_dependents();
}

// The GEMV path leaves y indexed by pair (t*K + k) rather than by slot; pairs whose id is
// out of range have no y row and are skipped.
__global__ void __launch_bounds__(256) combine_pairs_kernel(MoeArgs a) {
  pdl_wait();
  const int64_t H = a.H, K = a.K;
  const int64_t n4 = H / 4;
  const int64_t total = a.T * n4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / n4, c = (i % n4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t k = 0; k < K; ++k) {
      const int e = __ldg(a.ids + t * K + k);
      if (e < 0 || e >= a.E) continue;
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.y + (t * K + k) * H + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(a.out + t * H + c) = o;
  }
  pdl_launch_dependents();
}

}  // namespace

int launch_combine_pairs(const MoeArgs &a, cudaStream_t s) {
  const int64_t total = a.T * (a.H / 4);
  int64_t blocks = ceil_div(total, 256);
  if (blocks > kNumSMs * 8) blocks = kNumSMs * 8;
  return launch_pdl(combine_pairs_kernel, dim3((unsigned)blocks), dim3(256), 0, s, a);
}

int launch_combine(const MoeArgs &a, cudaStream_t s) {
  const int64_t total = a.T * (a.H / 4);
  int64_t blocks = ceil_div(total, 256);
  if (blocks > kNumSMs * 8) blocks = kNumSMs * 8;
  return launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(256), 0, s, a);
}

}  // namespace nvfp4
