// common.cuh -- device helpers shared by the NVFP4 MoE kernels (sm_100a only).
//
// Format (page "GLM-5-NVFP4-MTP", "Model Description": 4-bit values with one FP8 scale per
// 16 elements): E2M1 elements, E4M3 block scales, one fp32 global scale per tensor.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4_moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is written for sm_100a only"
#endif

namespace nvfp4 {

// Error flag bits written into the forward workspace.
constexpr int32_t kFlagBadId = 1;
constexpr int32_t kFlagWaitTimeout = 2;

// Records the CUDA error of the calling host thread (see nvfp4_last_cuda_error).
void set_last_cuda_error(cudaError_t e);
int check_launch();  // NVFP4_OK or NVFP4_ECUDA after a launch

constexpr int kNumSMs = 148;

// ------------------------------------------------------------------ bf16 / f16 bits
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two fp32 -> packed bf16x2 (lo in bits 0..15), each rounded to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------ E2M1 / E4M3 decode
// Two E2M1 codes (one byte: element 2j low nibble, 2j+1 high nibble) -> f16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(r) : "r"(byte_in_low8));
  return r;
}

// Four E2M1 pairs of one 32-bit word -> four f16x2 (pair p holds elements 2p, 2p+1).
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}

// Two E4M3 codes (low 16 bits) -> f16x2, exact (E4M3 fits f16's range and precision).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t r;
  asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}"
      : "=r"(r) : "r"(two_codes));
  return r;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h = e4m3x2_to_f16x2(code & 0xFFu);
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

__device__ __forceinline__ float f16_lo(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)(h >> 16)));
}

// ------------------------------------------------------------------ encoders
// fp32 -> E4M3 code, round to nearest even, saturating to +-448 (hardware conversion).
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Two fp32 -> two E2M1 codes in one byte (lo in bits 0..3, hi in bits 4..7), by the
// hardware convert: round to nearest, ties to the even code, saturating at +-6, sign kept
// (so -0.1 -> 0x8).
__device__ __forceinline__ uint32_t e2m1x2_rn_sat(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// fp32 -> E2M1 code (low nibble), rounded as e2m1x2_rn_sat rounds.
__device__ __forceinline__ uint32_t f32_to_e2m1(float v) { return e2m1x2_rn_sat(v, 0.0f) & 0xFu; }

// ------------------------------------------------------------------ memory
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void stg_stream(void *p, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};"
               :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its prologue,
// and wait for the previous kernel's results before touching them.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------ f16 activation scaling
// Activations enter f16 tensor/FMA operands after scaling by 2^p with p = 14 - floor(log2 m),
// m the row's largest magnitude, so m * 2^p lies in [2^14, 2^15).  bf16 has 8 significant
// bits and f16 11, so the rounding to f16 is exact for every element above 2^-31 * m.
__device__ __forceinline__ float exp2i(int p) { return __uint_as_float((uint32_t)(p + 127) << 23); }

__device__ __forceinline__ int prescale_exponent(float m) {
  if (!(m > 0.0f)) return 0;
  const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;  // floor(log2 m) for normals
  int p = 14 - e;
  p = max(-100, min(100, p));
  return p;
}

}  // namespace nvfp4
