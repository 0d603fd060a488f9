// codec.cu -- NVFP4 quantize / dequantize kernels and their C ABI.
//
// Format: page "GLM-5-NVFP4-MTP", "Model Description" (4-bit values, one FP8 scale per 16
// elements), with E2M1 elements, E4M3 block scales and one fp32 global scale per tensor:
//   g = amax / (6 * 448)  (1 for an all-zero tensor)
//   s = (amax_b / 6) / g  -> E4M3, nearest even, saturating
//   code_i = E2M1(x_i / (dec(s) * g)), nearest even, saturating, sign kept; 0 if the
//   divisor is 0.
// The codes and scales are exactly those of the IEEE fp32 operations written (no contraction):
// the kernels reach them through reciprocal multiplies checked against the rounding
// boundaries, and divide wherever that check cannot decide (below).  The kernels stream HBM
// with 16-byte accesses.
#include "pipeline.cuh"
#include "quant.cuh"

namespace nvfp4 {

// ------------------------------------------------------------------ quantize
// Workspace of nvfp4_quantize: [0] error flag, [4..4+n) amax bits, [4+n..4+2n) number of
// CTAs whose amax share of tensor t is merged.
constexpr int kQwsHeader = 4;

// Bounded wait (one thread) until *p >= want; a wait that gives up sets bit 1 of ws[0].
__device__ __forceinline__ bool wait_count(const uint32_t *p, uint32_t want, uint32_t *ws,
                                           volatile int *abort) {
  if (wait_geq(p, want, abort)) return true;
  if (!*abort) {
    atomicOr(ws, (uint32_t)kFlagWaitTimeout);
    *abort = 1;
  }
  return false;
}

// Quantize n tensors with one cooperative launch.  Warps 0-1 of every CTA take the amax of
// tensor p over the CTA's share while warps 2-7 quantize the CTA's share of tensor p - 1,
// which may start once every CTA has merged its amax of that tensor.  The amax warps wait
// for their own CTA's quantize warps to finish tensor p - 2 before reading tensor p, so at
// most about three tensors are in flight: a gate/up tensor of the layer is 50 MB, and the
// quantize pass finds it in L2 right after the amax pass brought it in.  Each input byte
// crosses HBM once.
constexpr int kDeqUnits = 4;   // 8-element units per dequantize thread per pass
constexpr int kAmaxWarps = 2;
constexpr int kAmaxThreads = 32 * kAmaxWarps;
constexpr int kQuantThreads = 256 - kAmaxThreads;
constexpr int kAmaxLoads = 16;   // 16-byte loads in flight per amax thread

// L2 eviction-priority policies for the two reads of a tensor: the amax pass marks lines to
// be kept (the quantize pass comes back for them), the quantize pass marks them as last use.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_l2_hint(const void *ptr, uint64_t policy) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr), "l"(policy));
  return r;
}

__global__ void __launch_bounds__(256) quantize_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t per_tensor, int n_tensors,
    uint32_t *__restrict__ ws, uint8_t *__restrict__ packed, uint8_t *__restrict__ scales,
    float *__restrict__ global_scale) {
  __shared__ int s_abort;
  __shared__ int s_qdone;          // tensors this CTA has quantized
  __shared__ uint32_t s_red[kAmaxWarps];
  if (threadIdx.x == 0) {
    s_abort = 0;
    s_qdone = 0;
  }
  __syncthreads();
  volatile int *abort = &s_abort;
  uint32_t *amax_bits = ws + kQwsHeader;
  uint32_t *merged = amax_bits + n_tensors;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nvec = per_tensor / 8;                    // 16-byte vectors = half blocks
  const int64_t v0 = nvec * blockIdx.x / gridDim.x, v1 = nvec * (blockIdx.x + 1) / gridDim.x;

  if (warp < kAmaxWarps) {
    const uint64_t keep = l2_policy_evict_last();
    for (int p = 0; p < n_tensors; ++p) {
      if (threadIdx.x == 0 && p >= 2) {   // keep the tensors in flight few
        const uint64_t t0 = global_timer_ns();
        while (*(volatile int *)&s_qdone < p - 1 && !*abort) {
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(ws, (uint32_t)kFlagWaitTimeout);
            *abort = 1;
          }
        }
      }
      named_sync(1, kAmaxThreads);
      const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)p * per_tensor);
      uint32_t m = 0;   // max of |bf16| bit patterns (same order as the values)
      int64_t i = v0 + threadIdx.x;
      for (; i + (kAmaxLoads - 1) * kAmaxThreads < v1; i += kAmaxLoads * kAmaxThreads) {
        uint4 v[kAmaxLoads];
#pragma unroll
        for (int k = 0; k < kAmaxLoads; ++k) v[k] = ld_l2_hint(src + i + k * kAmaxThreads, keep);
#pragma unroll
        for (int k = 0; k < kAmaxLoads; ++k) {
          const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
        }
      }
      for (; i < v1; i += kAmaxThreads) {
        const uint4 v = ld_l2_hint(src + i, keep);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (lane == 0) s_red[warp] = m;
      named_sync(1, kAmaxThreads);
      if (threadIdx.x == 0) {
        for (int w = 1; w < kAmaxWarps; ++w) m = max(m, s_red[w]);
        if (m) atomicMax(amax_bits + p, m << 16);   // bf16 bits << 16 = fp32 bits
        __threadfence();
        atomicAdd(merged + p, 1u);
      }
    }
    return;
  }

  // ---- quantize: one thread per 16-element block, two blocks per thread per pass
  const uint64_t last_use = l2_policy_evict_first();
  const int qt = threadIdx.x - kAmaxThreads;
  // the share boundaries are made even, so both halves of a block fall in one share
  const int64_t b0 = (v0 & ~int64_t(1)) / 2;
  const int64_t b1 = blockIdx.x + 1 == gridDim.x ? nvec / 2 : (v1 & ~int64_t(1)) / 2;
  for (int t = 0; t < n_tensors; ++t) {
    if (qt == 0) wait_count(merged + t, gridDim.x, ws, abort);
    named_sync(2, kQuantThreads);
    const float g = global_scale_from_amax(__ldcg(amax_bits + t));
    const BlockScaleConsts bc = block_scale_consts(g);
    if (blockIdx.x == 0 && qt == 0) global_scale[t] = g;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)t * per_tensor);
    uint2 *dst = reinterpret_cast<uint2 *>(packed) + (int64_t)t * (nvec / 2);
    uint8_t *sdst = scales + (int64_t)t * (nvec / 2);
    for (int64_t i0 = b0 + qt; i0 < b1; i0 += 2 * kQuantThreads) {
      uint4 v[2][2];
      bool act[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t b = i0 + k * kQuantThreads;
        act[k] = b < b1;
        v[k][0] = act[k] ? ld_l2_hint(src + 2 * b, last_use) : make_uint4(0u, 0u, 0u, 0u);
        v[k][1] = act[k] ? ld_l2_hint(src + 2 * b + 1, last_use) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t b = i0 + k * kQuantThreads;
        if (act[k]) {
          uint32_t sc;
          dst[b] = quantize_block16(v[k][0], v[k][1], g, bc.c, bc.fast, &sc);
          sdst[b] = (uint8_t)sc;
        }
      }
    }
    named_sync(2, kQuantThreads);
    if (qt == 0) *(volatile int *)&s_qdone = t + 1;
  }
}

// ------------------------------------------------------------------ dequantize
// One thread per 32 elements: 16 packed bytes + 2 scale codes -> 64 bytes of bf16.
__global__ void __launch_bounds__(256) dequantize_kernel(
    const uint8_t *__restrict__ packed, const uint8_t *__restrict__ scales,
    const float *__restrict__ global_scale, int64_t per_tensor, int64_t n_units,
    __nv_bfloat16 *__restrict__ out) {
  // A unit is 8 consecutive elements: 4 packed bytes in, one 16-byte store out, so a warp's
  // loads and stores are each one contiguous run.  kDeqUnits units per thread are loaded
  // before any is converted.
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // tensor of element e: a double-precision estimate of e / per_tensor, corrected by one
  const double inv_per = 1.0 / (double)per_tensor;
  auto tensor_of = [&](int64_t e) -> int64_t {
    int64_t t = (int64_t)((double)e * inv_per);
    if (t * per_tensor > e) --t;
    else if ((t + 1) * per_tensor <= e) ++t;
    return t;
  };
  for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u0 < n_units;
       u0 += stride * kDeqUnits) {
    uint32_t q[kDeqUnits], sc[kDeqUnits];
    float g[kDeqUnits];
#pragma unroll
    for (int k = 0; k < kDeqUnits; ++k) {
      const int64_t u = u0 + k * stride;
      if (u < n_units) {
        q[k] = __ldg(reinterpret_cast<const uint32_t *>(packed) + u);
        sc[k] = __ldg(scales + (u >> 1));
        g[k] = __ldg(global_scale + tensor_of(u * 8));
      }
    }
#pragma unroll
    for (int k = 0; k < kDeqUnits; ++k) {
      const int64_t u = u0 + k * stride;
      if (u >= n_units) break;
      const uint32_t s16 = e4m3x2_to_f16x2(sc[k] | (sc[k] << 8));   // (s, s) as f16
      uint32_t h[4], o[4];
      e2m1x8_to_f16x2x4(q[k], h);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        // q * s is exact in f16 (at most 6 significant bits, within f16's range)
        __half2 qs = __hmul2(*reinterpret_cast<__half2 *>(&h[p]),
                             *reinterpret_cast<const __half2 *>(&s16));
        const uint32_t qsu = *reinterpret_cast<uint32_t *>(&qs);
        o[p] = pack_bf16x2(__fmul_rn(f16_lo(qsu), g[k]), __fmul_rn(f16_hi(qsu), g[k]));
      }
      stg_stream(reinterpret_cast<uint4 *>(out) + u, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// ------------------------------------------------------------------ calibrated scales
// Page "GLM-5-NVFP4-MTP", "Calibration dataset": static scales from several calibration
// passes, merged by element-wise max.  amax_kernel folds max |x| of each tensor into amax
// (fp32 bits of a non-negative value order like the value, so an integer max merges them);
// quantize_amax_kernel is the quantizer with that amax given, one read of the input.
constexpr int kStreamLoads = 8;      // 16-byte loads in flight per thread (amax)
constexpr int kQuantPerThread = 2;   // blocks per thread per pass (static quantizer)

// CTA b takes the vectors [W b / G, W (b+1) / G) of all n tensors together (W vectors of 8
// elements in all), tensor by tensor where its range crosses a boundary.
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16 *__restrict__ x,
                                                   int64_t per_vec, int n_tensors,
                                                   uint32_t *__restrict__ amax_bits) {
  __shared__ uint32_t s_red[8];
  const int64_t W = per_vec * n_tensors;
  const int64_t v0 = W * blockIdx.x / gridDim.x, v1 = W * (blockIdx.x + 1) / gridDim.x;
  const uint4 *src = reinterpret_cast<const uint4 *>(x);
  for (int64_t seg = v0; seg < v1;) {
    const int t = (int)(seg / per_vec);
    const int64_t end = min(v1, (int64_t)(t + 1) * per_vec);
    uint32_t m = 0;   // max of |bf16| bit patterns (same order as the values)
    int64_t i = seg + threadIdx.x;
    for (; i + (kStreamLoads - 1) * 256 < end; i += kStreamLoads * 256) {
      uint4 v[kStreamLoads];
#pragma unroll
      for (int k = 0; k < kStreamLoads; ++k) v[k] = ldg_stream(src + i + k * 256);
#pragma unroll
      for (int k = 0; k < kStreamLoads; ++k) {
        const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
      }
    }
    for (; i < end; i += 256) {
      const uint4 v = ldg_stream(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < 8; ++w) m = max(m, s_red[w]);
      if (m) atomicMax(amax_bits + t, m << 16);   // bf16 bits << 16 = fp32 bits
    }
    __syncthreads();
    seg = end;
  }
}

// One thread per 16-element block (32 bytes in, 8 bytes of codes and a scale byte out),
// kQuantPerThread blocks per thread per pass.  g = amax / 2688 (1 for an amax of 0), IEEE
// division.
__global__ void __launch_bounds__(256) quantize_amax_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t per_blk, int64_t n_blk,
    const float *__restrict__ amax, uint8_t *__restrict__ packed,
    uint8_t *__restrict__ scales, float *__restrict__ global_scale) {
  const uint4 *src = reinterpret_cast<const uint4 *>(x);
  uint2 *dst = reinterpret_cast<uint2 *>(packed);
  const int64_t span = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x * kQuantPerThread + threadIdx.x;
       i0 < n_blk; i0 += span * kQuantPerThread) {
    uint4 v[kQuantPerThread][2];
    bool act[kQuantPerThread];
#pragma unroll
    for (int k = 0; k < kQuantPerThread; ++k) {
      const int64_t b = i0 + (int64_t)k * blockDim.x;
      act[k] = b < n_blk;
      v[k][0] = act[k] ? ldg_stream(src + 2 * b) : make_uint4(0u, 0u, 0u, 0u);
      v[k][1] = act[k] ? ldg_stream(src + 2 * b + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
    // the tensor of the thread's first block and its constants (a later block past the end
    // of that tensor steps to the next one)
    int t = (int)(i0 / per_blk);
    float am = __ldg(amax + t);
    float g = am == 0.0f ? 1.0f : __fdiv_rn(am, 2688.0f);
    BlockScaleConsts bc = block_scale_consts(g);
#pragma unroll
    for (int k = 0; k < kQuantPerThread; ++k) {
      const int64_t b = i0 + (int64_t)k * blockDim.x;
      if (!act[k]) continue;
      if (b >= (int64_t)(t + 1) * per_blk) {
        while (b >= (int64_t)(t + 1) * per_blk) ++t;
        am = __ldg(amax + t);
        g = am == 0.0f ? 1.0f : __fdiv_rn(am, 2688.0f);
        bc = block_scale_consts(g);
      }
      uint32_t sc;
      dst[b] = quantize_block16(v[k][0], v[k][1], g, bc.c, bc.fast, &sc);
      scales[b] = (uint8_t)sc;
      if (b == (int64_t)t * per_blk) global_scale[t] = g;
    }
  }
}

// ------------------------------------------------------------------ scalar casts
__global__ void cast_kernel(const float *__restrict__ in, int64_t n, uint8_t *__restrict__ e4m3,
                            uint8_t *__restrict__ e2m1) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = in[i];
    if (e4m3) e4m3[i] = (uint8_t)f32_to_e4m3(v);
    if (e2m1) e2m1[i] = (uint8_t)f32_to_e2m1(v);
  }
}

static int grid_for(int64_t work_items, int threads) {
  int64_t b = ceil_div(work_items, threads);
  const int64_t cap = (int64_t)kNumSMs * 16;
  return (int)(b < cap ? (b > 0 ? b : 1) : cap);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_quantize_workspace_size(int64_t n_tensors, int64_t, int64_t) {
  if (n_tensors <= 0) return 0;
  return (size_t)ceil_div((kQwsHeader + 2 * n_tensors) * 4, 256) * 256;
}

extern "C" int nvfp4_quantize(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows,
                              int64_t cols, uint8_t *packed, uint8_t *scales,
                              float *global_scale, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
  if (!x || !packed || !scales || !global_scale || n_tensors <= 0 || rows <= 0 || cols <= 0)
    return NVFP4_EINVAL;
  if (cols % 32 != 0) return NVFP4_ESHAPE;
  if (n_tensors >= (int64_t(1) << 24)) return NVFP4_ESHAPE;
  // 16-byte loads of x, 8-byte stores of packed codes
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(packed) & 7) ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3))
    return NVFP4_EINVAL;
  if (!workspace || ws_bytes < nvfp4_quantize_workspace_size(n_tensors, rows, cols) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3))
    return NVFP4_EWORKSPACE;
  const int64_t per = rows * cols;
  uint32_t *ws = static_cast<uint32_t *>(workspace);
  cudaError_t e =
      cudaMemsetAsync(ws, 0, sizeof(uint32_t) * (kQwsHeader + 2 * n_tensors), stream);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  // a cooperative launch: every CTA is resident, so no CTA waits on one that has not started
  int dev = 0, sms = kNumSMs, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_kernel, 256, 0);
  if (e != cudaSuccess || per_sm <= 0) {
    set_last_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
    return NVFP4_ECUDA;
  }
  const int ctas = sms * (per_sm < 4 ? per_sm : 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, quantize_kernel, x, per, (int)n_tensors, ws, packed, scales,
                         global_scale);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  return check_launch();
}

extern "C" int nvfp4_dequantize(const uint8_t *packed, const uint8_t *scales,
                                const float *global_scale, int64_t n_tensors, int64_t rows,
                                int64_t cols, __nv_bfloat16 *out, cudaStream_t stream) {
  if (!packed || !scales || !global_scale || !out || n_tensors <= 0 || rows <= 0 || cols <= 0)
    return NVFP4_EINVAL;
  if (cols % 32 != 0) return NVFP4_ESHAPE;
  // the kernel stores bf16 in 16-byte pieces; packed and scales keep the alignment the header
  // states (16 and 2 bytes)
  if ((reinterpret_cast<uintptr_t>(packed) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(scales) & 1))
    return NVFP4_EINVAL;
  const int64_t per = rows * cols;
  const int64_t n_units = n_tensors * per / 8;
  dequantize_kernel<<<grid_for(ceil_div(n_units, kDeqUnits), 256), 256, 0, stream>>>(
      packed, scales, global_scale, per, n_units, out);
  return check_launch();
}

extern "C" int nvfp4_cast_f32(const float *in, int64_t n, uint8_t *e4m3, uint8_t *e2m1,
                              cudaStream_t stream) {
  if (!in || n <= 0) return NVFP4_EINVAL;
  cast_kernel<<<grid_for(n, 256), 256, 0, stream>>>(in, n, e4m3, e2m1);
  return check_launch();
}

extern "C" int nvfp4_amax(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows, int64_t cols,
                          float *amax, int merge, cudaStream_t stream) {
  if (!x || !amax || n_tensors <= 0 || rows <= 0 || cols <= 0) return NVFP4_EINVAL;
  if (cols % 32 != 0 || n_tensors >= (int64_t(1) << 24)) return NVFP4_ESHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(amax) & 3))
    return NVFP4_EINVAL;
  if (!merge) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * n_tensors, stream);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return NVFP4_ECUDA;
    }
  }
  const int64_t per_vec = rows * cols / 8;
  const int64_t W = per_vec * n_tensors;
  const int grid = (int)min((int64_t)kNumSMs * 8, max((int64_t)1, ceil_div(W, 256 * 32)));
  amax_kernel<<<grid, 256, 0, stream>>>(x, per_vec, (int)n_tensors,
                                        reinterpret_cast<uint32_t *>(amax));
  return check_launch();
}

extern "C" int nvfp4_quantize_with_amax(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows,
                                        int64_t cols, const float *amax, uint8_t *packed,
                                        uint8_t *scales, float *global_scale,
                                        cudaStream_t stream) {
  if (!x || !amax || !packed || !scales || !global_scale || n_tensors <= 0 || rows <= 0 ||
      cols <= 0)
    return NVFP4_EINVAL;
  if (cols % 32 != 0 || n_tensors >= (int64_t(1) << 24)) return NVFP4_ESHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(packed) & 7) ||
      (reinterpret_cast<uintptr_t>(amax) & 3) || (reinterpret_cast<uintptr_t>(global_scale) & 3))
    return NVFP4_EINVAL;
  const int64_t per_blk = rows * cols / 16;
  const int64_t n_blk = per_blk * n_tensors;
  const int grid = grid_for(ceil_div(n_blk, kQuantPerThread), 256);
  quantize_amax_kernel<<<grid, 256, 0, stream>>>(x, per_blk, n_blk, amax, packed, scales,
                                                 global_scale);
  return check_launch();
}
