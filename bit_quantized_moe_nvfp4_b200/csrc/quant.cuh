// quant.cuh -- the NVFP4 quantizer's per-block arithmetic, shared by the codec kernels and the
// W4A4 path's activation quantizer, so both make the same decisions.
//
// Format: page "GLM-5-NVFP4-MTP", "Model Description" (4-bit values, one FP8 scale per 16
// elements): g = amax / 2688 per tensor (1 for an all-zero tensor), block scale
// E4M3(RN(RN(amax_b / 6) / g)), element codes E2M1(RN(x / (dec(s) * g))).
#pragma once
#include "common.cuh"

namespace nvfp4 {

// The element codes without a division per element.  The code of x is E2M1(q) with
// q = RN(x / d), the IEEE quotient.  With r = RN(1/d), the product q' = RN(x * r) is within
// 1.5 ulp of q (each of the two roundings is half an ulp, the reciprocal's error is carried
// by the product once more), so q lies between q' * (1 - 2^-21) and q' * (1 + 2^-21), an
// interval of +-4 ulp.  E2M1 rounding is monotone, so when the hardware convert
// (round to nearest, ties to the even code, saturating, sign kept) gives the same code at
// both ends, that is the code of q; only when a rounding midpoint of the E2M1 grid lies
// inside the interval -- rare outside data placed on the midpoints -- is q formed by IEEE
// division and converted.  The codes are therefore those of dividing every element by d.
// (For d below 2^-100 the reciprocal could overflow, and every element is divided.)
__device__ __forceinline__ uint32_t e2m1_pair_code(float x0, float x1, float d, float r) {
  const float2 q = __fmul2_rn(make_float2(x0, x1), make_float2(r, r));
  constexpr float kBelow = 1.0f - 0x1p-21f, kAbove = 1.0f + 0x1p-21f;
  const float2 lo = __fmul2_rn(q, make_float2(kBelow, kBelow));
  const float2 hi = __fmul2_rn(q, make_float2(kAbove, kAbove));
  const uint32_t a = e2m1x2_rn_sat(lo.x, lo.y), b = e2m1x2_rn_sat(hi.x, hi.y);
  if (a == b) return a;
  return e2m1x2_rn_sat(__fdiv_rn(x0, d), __fdiv_rn(x1, d));
}

// The block scale code E4M3(RN(RN(amax_b / 6) / g)) the same way: with c = RN(1 / RN(6 g)),
// RN(amax_b * c) is within 5 ulp of the twice-rounded quotient (five roundings of at most
// half an ulp each), so when the E4M3 convert (nearest even, saturating) gives one code at
// both ends of +-16 ulp around it, that is the code; otherwise the two divisions are taken.
// `fast` is false for g below 2^-100, where c could overflow.
__device__ __forceinline__ uint32_t block_scale_code(float amax_b, float g, float c, bool fast) {
  if (fast) {
    const float sp = __fmul_rn(amax_b, c);
    const float2 e = __fmul2_rn(make_float2(sp, sp),
                                make_float2(1.0f - 0x1p-20f, 1.0f + 0x1p-20f));
    const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(e, __NV_SATFINITE, __NV_E4M3);
    if ((two & 0xFFu) == (two >> 8)) return two & 0xFFu;
  }
  return f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax_b, 6.0f), g));
}

// One 16-element block (two 16-byte words of bf16: element 2k in the low half of word k)
// -> 8 bytes of codes (element 2j in the low nibble of byte j) and its scale code.
// Four E2M1 code pairs (8 codes, element 2j in the low nibble of byte j) of the values
// q[0..7] as one 32-bit word: the hardware convert of each pair, the four bytes packed by one
// move.
__device__ __forceinline__ uint32_t e2m1x8_rn_sat(const float (&q)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return r;
}

// The codes of 8 elements (four bf16 pairs w[0..3]) for divisor d with r = RN(1/d): the
// interval test of e2m1_pair_code made for four pairs at once (the lower and the upper ends
// converted and compared as whole words); a word that differs is decided pair by pair.
__device__ __forceinline__ uint32_t e2m1_codes8(const uint32_t *w, float d, float r) {
  constexpr float kBelow = 1.0f - 0x1p-21f, kAbove = 1.0f + 0x1p-21f;
  float lo[8], hi[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 q = __fmul2_rn(make_float2(bf16_lo(w[k]), bf16_hi(w[k])), make_float2(r, r));
    const float2 a = __fmul2_rn(q, make_float2(kBelow, kBelow));
    const float2 b = __fmul2_rn(q, make_float2(kAbove, kAbove));
    lo[2 * k] = a.x;
    lo[2 * k + 1] = a.y;
    hi[2 * k] = b.x;
    hi[2 * k + 1] = b.y;
  }
  const uint32_t A = e2m1x8_rn_sat(lo), B = e2m1x8_rn_sat(hi);
  if (A == B) return A;
  uint32_t out = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    out |= e2m1_pair_code(bf16_lo(w[k]), bf16_hi(w[k]), d, r) << (8 * k);
  return out;
}

__device__ __forceinline__ uint2 quantize_block16(const uint4 &v0, const uint4 &v1, float g,
                                                  float c, bool fast, uint32_t *sc_out) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  // max of |bf16| bit patterns (same order as the values), two halves at a time
  uint32_t m2 = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t a = w[k] & 0x7FFF7FFFu;
    asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(a));
  }
  const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  const uint32_t sc = block_scale_code(__uint_as_float(m << 16), g, c, fast);
  const float d = __fmul_rn(e4m3_to_f32(sc), g);
  uint32_t out[2] = {0u, 0u};
  if (d >= 0x1p-100f) {
    const float r = __frcp_rn(d);
    out[0] = e2m1_codes8(w, d, r);
    out[1] = e2m1_codes8(w + 4, d, r);
  } else if (d != 0.0f) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      out[k >> 2] |= e2m1x2_rn_sat(__fdiv_rn(bf16_lo(w[k]), d), __fdiv_rn(bf16_hi(w[k]), d))
                     << (8 * (k & 3));
  }
  *sc_out = sc;
  return make_uint2(out[0], out[1]);
}

// The per-tensor constants of quantize_block16: c = RN(1 / RN(6 g)), and whether the fast
// scale path applies.
struct BlockScaleConsts {
  float c;
  bool fast;
};
__device__ __forceinline__ BlockScaleConsts block_scale_consts(float g) {
  return {__frcp_rn(__fmul_rn(6.0f, g)), g >= 0x1p-100f};
}

// g = amax / 2688, IEEE division, 1 for an all-zero tensor.
__device__ __forceinline__ float global_scale_from_amax(uint32_t amax_bits) {
  float amax = __uint_as_float(amax_bits);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

}  // namespace nvfp4
