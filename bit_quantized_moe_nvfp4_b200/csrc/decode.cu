// decode.cu -- memory-bound GEMV path of the NVFP4 MoE layer (small token counts).
//
// Page "GLM-5-NVFP4-MTP", "Model Description": experts are NVFP4 (4-bit values, one FP8
// scale per 16 elements), 8 of 256 active per token.  With few tokens per expert the layer
// is a stream of packed expert bytes, so these kernels read every needed weight byte once
// with 16-byte loads, decode E2M1 / E4M3 in registers with the hardware converts, and
// accumulate in fp32 (packed FFMA2).  Each warp owns a contiguous range of equal-sized
// work units (one gate/up row pair, or one or two down rows, of one active expert), so
// the bytes are spread evenly over all warps of a persistent grid.
//
//   gate/up: a_j = g_gu * sum_h W[j,h] x[h] for the gate row j and the up row I+j together,
//            then h_j = bf16(silu(gate) * up)  (SwiGLU fused, both rows in one warp)
//   down:    y[r, n] = w[r] * g_dn * sum_i W[n,i] h[r,i]   for the expert's rows r
// The combine over the K slots of a token runs afterwards (combine.cu).
#include "moe.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// 8 E2M1 codes (one 32-bit word) -> 4 float2 (elements 2p, 2p+1), exact.
__device__ __forceinline__ void decode8(uint32_t word, float2 (&q)[4]) {
  uint32_t h[4];
  e2m1x8_to_f16x2x4(word, h);
#pragma unroll
  for (int p = 0; p < 4; ++p) q[p] = __half22float2(*reinterpret_cast<__half2 *>(&h[p]));
}

// 8 bf16 (one uint4) -> 4 float2, exact.
__device__ __forceinline__ void bf16x8(uint4 v, float2 (&f)[4]) {
  f[0] = make_float2(bf16_lo(v.x), bf16_hi(v.x));
  f[1] = make_float2(bf16_lo(v.y), bf16_hi(v.y));
  f[2] = make_float2(bf16_lo(v.z), bf16_hi(v.z));
  f[3] = make_float2(bf16_lo(v.w), bf16_hi(v.w));
}

// Dot product of one 32-element chunk (16 packed bytes, 2 block scales) with 32 fp32
// activations given as 4 uint4 of bf16; returns acc + s0 * dot(block 0) + s1 * dot(block 1).
__device__ __forceinline__ float2 chunk_dot(uint4 q, float s0, float s1, const uint4 (&xv)[4],
                                            float2 acc) {
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float2 part = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      float2 qf[4], xf[4];
      decode8(words[2 * b + w], qf);
      bf16x8(xv[2 * b + w], xf);
#pragma unroll
      for (int p = 0; p < 4; ++p) part = ffma2(qf[p], xf[p], part);
    }
    const float s = b ? s1 : s0;
    acc = ffma2(part, make_float2(s, s), acc);
  }
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ void load_x_chunk(const __nv_bfloat16 *row, int c, uint4 (&xv)[4]) {
  const uint4 *p = reinterpret_cast<const uint4 *>(row + 32 * c);
#pragma unroll
  for (int i = 0; i < 4; ++i) xv[i] = __ldg(p + i);
}

__device__ __forceinline__ void scales2(const uint8_t *srow, int c, float &s0, float &s1) {
  const uint32_t two = __ldg(reinterpret_cast<const unsigned short *>(srow) + c);
  const uint32_t h = e4m3x2_to_f16x2(two);
  s0 = f16_lo(h);
  s1 = f16_hi(h);
}

// ------------------------------------------------------------------ gate/up + SwiGLU
template <int NT>
__global__ void __launch_bounds__(kThreads) gemv_gateup_kernel(MoeArgs a) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * kWarps;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t I = a.I, H = a.H, K = a.K;
  const int64_t units = (int64_t)(*a.n_active) * I;
  const int64_t u0 = units * gw / warps_total, u1 = units * (gw + 1) / warps_total;
  const int nchunks = (int)(H / 32);

  for (int64_t u = u0; u < u1; ++u) {
    const int e = a.active[u / I];
    const int64_t j = u % I;
    const int off = a.offsets[e], cnt = a.counts[e];
    const uint8_t *pg = a.w_gu + ((int64_t)e * 2 * I + j) * (H / 2);
    const uint8_t *pu = pg + I * (H / 2);
    const uint8_t *sg = a.s_gu + ((int64_t)e * 2 * I + j) * (H / 16);
    const uint8_t *su = sg + I * (H / 16);
    const float g = __ldg(a.g_gu + e);
    for (int t0 = 0; t0 < cnt; t0 += NT) {
      const int nt = min(NT, cnt - t0);
      const __nv_bfloat16 *xr[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i)
        xr[i] = a.x + (int64_t)(a.perm[off + t0 + min(i, nt - 1)] / K) * H;
      float2 ag[NT], au[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) ag[i] = au[i] = make_float2(0.f, 0.f);
#pragma unroll 2
      for (int c = lane; c < nchunks; c += 32) {
        const uint4 qg = ldg_stream(pg + 16 * c);
        const uint4 qu = ldg_stream(pu + 16 * c);
        float sg0, sg1, su0, su1;
        scales2(sg, c, sg0, sg1);
        scales2(su, c, su0, su1);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          if (i < nt) {
            uint4 xv[4];
            load_x_chunk(xr[i], c, xv);
            ag[i] = chunk_dot(qg, sg0, sg1, xv, ag[i]);
            au[i] = chunk_dot(qu, su0, su1, xv, au[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        if (i < nt) {
          const float gate = warp_sum(ag[i].x + ag[i].y) * g;
          const float up = warp_sum(au[i].x + au[i].y) * g;
          if (lane == 0) {
            const float hv = silu_f32(gate) * up;
            a.h[(int64_t)(off + t0 + i) * I + j] = __float2bfloat16_rn(hv);
          }
        }
      }
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ down
// Work unit = two consecutive output rows of one expert (H is even).
template <int NT>
__global__ void __launch_bounds__(kThreads) gemv_down_kernel(MoeArgs a) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * kWarps;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t I = a.I, H = a.H;
  const int64_t per_expert = H / 2;
  const int64_t units = (int64_t)(*a.n_active) * per_expert;
  const int64_t u0 = units * gw / warps_total, u1 = units * (gw + 1) / warps_total;
  const int nchunks = (int)(I / 32);

  for (int64_t u = u0; u < u1; ++u) {
    const int e = a.active[u / per_expert];
    const int64_t n = (u % per_expert) * 2;
    const int off = a.offsets[e], cnt = a.counts[e];
    const uint8_t *p0 = a.w_dn + ((int64_t)e * H + n) * (I / 2);
    const uint8_t *p1 = p0 + I / 2;
    const uint8_t *s0r = a.s_dn + ((int64_t)e * H + n) * (I / 16);
    const uint8_t *s1r = s0r + I / 16;
    const float g = __ldg(a.g_dn + e);
    for (int t0 = 0; t0 < cnt; t0 += NT) {
      const int nt = min(NT, cnt - t0);
      const __nv_bfloat16 *hr[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) hr[i] = a.h + (int64_t)(off + t0 + min(i, nt - 1)) * I;
      float2 a0[NT], a1[NT];
#pragma unroll
      for (int i = 0; i < NT; ++i) a0[i] = a1[i] = make_float2(0.f, 0.f);
#pragma unroll 2
      for (int c = lane; c < nchunks; c += 32) {
        const uint4 q0 = ldg_stream(p0 + 16 * c);
        const uint4 q1 = ldg_stream(p1 + 16 * c);
        float s00, s01, s10, s11;
        scales2(s0r, c, s00, s01);
        scales2(s1r, c, s10, s11);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          if (i < nt) {
            uint4 hv[4];
            load_x_chunk(hr[i], c, hv);
            a0[i] = chunk_dot(q0, s00, s01, hv, a0[i]);
            a1[i] = chunk_dot(q1, s10, s11, hv, a1[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        if (i < nt) {
          const float d0 = warp_sum(a0[i].x + a0[i].y);
          const float d1 = warp_sum(a1[i].x + a1[i].y);
          if (lane == 0) {
            const int r = off + t0 + i;
            const float wk = __ldg(a.w + a.perm[r]) * g;
            *reinterpret_cast<float2 *>(a.y + (int64_t)r * H + n) = make_float2(wk * d0, wk * d1);
          }
        }
      }
    }
  }
  pdl_launch_dependents();
}

int gemv_grid() { return kNumSMs * 4; }

}  // namespace

int launch_gemv_gateup(const MoeArgs &a, cudaStream_t s) {
  const dim3 grid(gemv_grid()), block(kThreads);
  if (a.T <= 1) return launch_pdl(gemv_gateup_kernel<1>, grid, block, 0, s, a);
  if (a.T <= 16) return launch_pdl(gemv_gateup_kernel<2>, grid, block, 0, s, a);
  return launch_pdl(gemv_gateup_kernel<4>, grid, block, 0, s, a);
}

int launch_gemv_down(const MoeArgs &a, cudaStream_t s) {
  const dim3 grid(gemv_grid()), block(kThreads);
  if (a.T <= 1) return launch_pdl(gemv_down_kernel<1>, grid, block, 0, s, a);
  if (a.T <= 16) return launch_pdl(gemv_down_kernel<2>, grid, block, 0, s, a);
  return launch_pdl(gemv_down_kernel<4>, grid, block, 0, s, a);
}

}  // namespace nvfp4
