// combine.cu -- weighted top-k combine of the expert outputs of each token.
//
// Page "GLM-5-NVFP4-MTP", "Model Description": each token is served by 8 experts; its layer
// output is the routing-weighted sum of their outputs.  The down-projection kernels leave
// y[r] = w * g_dn * (W_dn h_r) for every routed pair r (in expert-grouped order), so here
// out[t] = bf16( sum over k = 0..K-1, ascending, of y[inv[t*K+k]] ) in fp32.  The fixed k
// order makes the result independent of which expert finished first.  Under expert
// parallelism the sum runs over this device's pairs only and stays fp32 (out_f32).
#include "moe.cuh"

namespace nvfp4 {

namespace {

// Four outputs of a token: bf16 (the layer output), or the fp32 partial of this device's
// experts under expert parallelism.
__device__ __forceinline__ void store_out(const MoeArgs &a, int64_t at, float4 acc) {
  if (a.out_f32) {
    *reinterpret_cast<float4 *>(a.out_f32 + at) = acc;
  } else {
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(a.out + at) = o;
  }
}

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
    store_out(a, t * H + c, acc);
  }
  pdl_launch_dependents();
}

// The GEMV path leaves y indexed by pair (t*K + k) rather than by slot; pairs this device
// does not serve (id out of range, or another rank's expert) have no y row and are skipped.
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
      if (a.map.local(__ldg(a.ids + t * K + k)) < 0) continue;
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.y + (t * K + k) * H + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    store_out(a, t * H + c, acc);
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
