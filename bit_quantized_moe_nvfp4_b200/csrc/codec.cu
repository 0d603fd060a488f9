// codec.cu -- NVFP4 quantize / dequantize kernels and their C ABI.
//
// Format: page "GLM-5-NVFP4-MTP", "Model Description" (4-bit values, one FP8 scale per 16
// elements), with E2M1 elements, E4M3 block scales and one fp32 global scale per tensor:
//   g = amax / (6 * 448)  (1 for an all-zero tensor)
//   s = (amax_b / 6) / g  -> E4M3, nearest even, saturating
//   code_i = E2M1(x_i / (dec(s) * g)), nearest even, saturating, sign kept; 0 if the
//   divisor is 0.
// Every step is the IEEE fp32 operation written (no reciprocal, no contraction), so the
// bits are reproducible.  All three kernels stream HBM with 16-byte accesses.
#include "common.cuh"

namespace nvfp4 {

// ------------------------------------------------------------------ amax
// Per-tensor max |x| as fp32 bits, merged with atomicMax (non-negative floats order like
// their bit patterns).  grid = (blocks per tensor, n_tensors).
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16 *__restrict__ x,
                                                   int64_t per_tensor,
                                                   uint32_t *__restrict__ amax_bits) {
  const int t = blockIdx.y;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)t * per_tensor);
  const int64_t nvec = per_tensor / 8;
  uint32_t m = 0;  // max of |bf16| bit patterns (sign cleared) -- same order as values
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 v = ldg_stream(src + i);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, w[j] & 0x7FFFu);
      m = max(m, (w[j] >> 16) & 0x7FFFu);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = max(m, red[w]);
    // bf16 bits << 16 are the fp32 bits of the same value
    atomicMax(amax_bits + t, m << 16);
  }
}

// g = amax / 2688, IEEE division, 1 for an all-zero tensor.
__device__ __forceinline__ float global_scale_from_amax(uint32_t amax_bits) {
  float amax = __uint_as_float(amax_bits);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// ------------------------------------------------------------------ quantize
// One thread per 8 elements (half a block); lanes 2i and 2i+1 share a block.
__global__ void __launch_bounds__(256) quantize_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t per_tensor, int64_t n_half_blocks,
    const uint32_t *__restrict__ amax_bits, uint8_t *__restrict__ packed,
    uint8_t *__restrict__ scales, float *__restrict__ global_scale) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  // Warp-uniform loop so the pair shuffle always runs with all 32 lanes; lanes past the
  // end compute on zeros and store nothing.  n_half_blocks is even, so both lanes of a
  // pair are in range together.
  for (int64_t hb0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
       hb0 < n_half_blocks; hb0 += stride) {
    const int64_t hb = hb0 + lane;
    const bool active = hb < n_half_blocks;
    const int64_t e0 = (active ? hb : hb0) * 8;   // first element
    const int t = (int)(e0 / per_tensor);           // tensor index
    const float g = global_scale_from_amax(__ldg(amax_bits + t));
    if (active && e0 == (int64_t)t * per_tensor) global_scale[t] = g;

    uint4 v = active ? ldg_stream(x + e0) : make_uint4(0, 0, 0, 0);
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));

    const float s = __fdiv_rn(__fdiv_rn(amax, 6.0f), g);
    const uint32_t sc = f32_to_e4m3(s);
    const float d = __fmul_rn(e4m3_to_f32(sc), g);
    uint32_t word = 0;
    if (d != 0.0f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= f32_to_e2m1(__fdiv_rn(f[i], d)) << (4 * i);
    }
    if (active) {
      reinterpret_cast<uint32_t *>(packed)[hb] = word;
      if ((hb & 1) == 0) scales[hb >> 1] = (uint8_t)sc;
    }
  }
}

// ------------------------------------------------------------------ dequantize
// One thread per 32 elements: 16 packed bytes + 2 scale codes -> 64 bytes of bf16.
__global__ void __launch_bounds__(256) dequantize_kernel(
    const uint8_t *__restrict__ packed, const uint8_t *__restrict__ scales,
    const float *__restrict__ global_scale, int64_t per_tensor, int64_t n_chunks,
    __nv_bfloat16 *__restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n_chunks; c += stride) {
    const int64_t e0 = c * 32;
    const int t = (int)(e0 / per_tensor);
    const float g = __ldg(global_scale + t);
    const uint4 q = ldg_stream(packed + c * 16);
    const uint32_t sc2 = __ldg(reinterpret_cast<const unsigned short *>(scales) + c);
    const uint32_t s16 = e4m3x2_to_f16x2(sc2);          // two block scales as f16
    const uint32_t s_lo = __byte_perm(s16, 0, 0x1010);   // (s0, s0)
    const uint32_t s_hi = __byte_perm(s16, 0, 0x3232);   // (s1, s1)
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[16];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t h[4];
      e2m1x8_to_f16x2x4(words[w], h);
      const uint32_t s = (w < 2) ? s_lo : s_hi;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        // q * s is exact in f16 (at most 6 significant bits, within f16's range)
        __half2 qs = __hmul2(*reinterpret_cast<__half2 *>(&h[p]),
                             *reinterpret_cast<const __half2 *>(&s));
        uint32_t qsu = *reinterpret_cast<uint32_t *>(&qs);
        o[w * 4 + p] = pack_bf16x2(__fmul_rn(f16_lo(qsu), g), __fmul_rn(f16_hi(qsu), g));
      }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + e0);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      stg_stream(dst + i, make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
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
  return (size_t)ceil_div(n_tensors * 4, 256) * 256;
}

extern "C" int nvfp4_quantize(const __nv_bfloat16 *x, int64_t n_tensors, int64_t rows,
                              int64_t cols, uint8_t *packed, uint8_t *scales,
                              float *global_scale, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
  if (!x || !packed || !scales || !global_scale || n_tensors <= 0 || rows <= 0 || cols <= 0)
    return NVFP4_EINVAL;
  if (cols % 32 != 0) return NVFP4_ESHAPE;
  // 16-byte loads of x, 4-byte stores of packed codes
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(packed) & 3) ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3))
    return NVFP4_EINVAL;
  if (!workspace || ws_bytes < nvfp4_quantize_workspace_size(n_tensors, rows, cols) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3))
    return NVFP4_EWORKSPACE;
  const int64_t per = rows * cols;
  uint32_t *amax = static_cast<uint32_t *>(workspace);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t) * n_tensors, stream);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return NVFP4_ECUDA;
  }
  // blocks per tensor: enough to fill the GPU a few times over in total
  int64_t bpt = ceil_div(per / 8, 256 * 8);
  int64_t want = ceil_div((int64_t)kNumSMs * 8, n_tensors);
  if (bpt > want) bpt = want;
  if (bpt < 1) bpt = 1;
  amax_kernel<<<dim3((unsigned)bpt, (unsigned)n_tensors), 256, 0, stream>>>(x, per, amax);
  if (int s = check_launch()) return s;
  const int64_t n_hb = n_tensors * per / 8;
  quantize_kernel<<<grid_for(n_hb, 256), 256, 0, stream>>>(x, per, n_hb, amax, packed, scales,
                                                            global_scale);
  return check_launch();
}

extern "C" int nvfp4_dequantize(const uint8_t *packed, const uint8_t *scales,
                                const float *global_scale, int64_t n_tensors, int64_t rows,
                                int64_t cols, __nv_bfloat16 *out, cudaStream_t stream) {
  if (!packed || !scales || !global_scale || !out || n_tensors <= 0 || rows <= 0 || cols <= 0)
    return NVFP4_EINVAL;
  if (cols % 32 != 0) return NVFP4_ESHAPE;
  // 16-byte loads of packed codes and stores of bf16, 2-byte loads of scale pairs
  if ((reinterpret_cast<uintptr_t>(packed) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(scales) & 1))
    return NVFP4_EINVAL;
  const int64_t per = rows * cols;
  const int64_t n_chunks = n_tensors * per / 32;
  dequantize_kernel<<<grid_for(n_chunks, 256), 256, 0, stream>>>(packed, scales, global_scale,
                                                                 per, n_chunks, out);
  return check_launch();
}

extern "C" int nvfp4_cast_f32(const float *in, int64_t n, uint8_t *e4m3, uint8_t *e2m1,
                              cudaStream_t stream) {
  if (!in || n <= 0) return NVFP4_EINVAL;
  cast_kernel<<<grid_for(n, 256), 256, 0, stream>>>(in, n, e4m3, e2m1);
  return check_launch();
}
