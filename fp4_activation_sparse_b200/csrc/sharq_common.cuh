// Shared device helpers for the SharQ kernels (sm_100a only).
//
// Conversions use the sm_100a FP4/FP8 cvt instructions: round to nearest even,
// satfinite, the first source operand lands in the upper nibble/byte. E2M1 codes
// are stored two per byte with the lower K index in the low nibble.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "SharQ kernels are written for sm_100a (B200) only"
#endif

namespace sharq {

constexpr int kFmtNV = 0;  // NVFP4: 16-element blocks, E4M3 scales, float32 second-level scale
constexpr int kFmtMX = 1;  // MXFP4: 32-element blocks, E8M0 scales

// ---------------------------------------------------------------------------------
// layouts shared by the producer kernels (prep, pack) and the GEMM
// ---------------------------------------------------------------------------------
// Byte offset of scale (row r, index s) in a 128x4-atom scale tensor with
// `spr` scales per row (spr % 4 == 0).
__host__ __device__ __forceinline__ size_t atom_offset(int r, int s, int spr) {
  return ((size_t)(r >> 7) * (spr >> 2) + (s >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (s & 3);
}

__host__ __device__ __forceinline__ int round_up(int a, int b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------------------------
// FP4 / FP8 conversions
// ---------------------------------------------------------------------------------
// Two float32 -> one byte of E2M1 codes: lo in bits 0..3, hi in bits 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
      : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

// Eight float32 -> four bytes of E2M1 codes (v0 in the low nibble of byte 0).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                              float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// Four bytes of E2M1 codes -> four half2 (exact); byte j -> h[j], low nibble in .x.
__device__ __forceinline__ void cvt_e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

// One byte of two E2M1 codes -> half2 (exact), low nibble in .x.
__device__ __forceinline__ uint32_t cvt_e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
  return out;
}

// float32 -> E4M3 code (RNE, satfinite to 448) in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// E4M3 code -> float32 (exact, via f16).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t in = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h2) {
  __half2 h = *reinterpret_cast<__half2 *>(&h2);
  return __half22float2(h);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Correctly rounded 1/d for normal d whose reciprocal is normal: the hardware approximation
// refined by one fused multiply-add step (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990: with y faithful to 1/d,
// the residual e = 1 - d*y is exact and RN(y + y*e) = RN(1/d)). tests/cuda/rcp_check.cu checks
// it bit for bit against the correctly rounded reciprocal over every such float32.
__device__ __forceinline__ float rcp_rn(float d) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
  const float e = __fmaf_rn(-d, y, 1.0f);
  return __fmaf_rn(y, e, y);
}

// max(|a|, |b|, |c|) in one instruction
__device__ __forceinline__ float max3abs(float a, float b, float c) {
  float d;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^(e-127) as float32 (e in 0..254; e = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  return e == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// Exact squares of a word's two bf16 values added to a float64 sum (low half first), without
// conversion instructions: the bf16 exponent and mantissa bits of |x|, moved to the top of a
// float64 high word, encode a = |x| * 2^-896 exactly (zero and subnormal values included);
// the same bits with 1792 added to the exponent field encode b = |x| * 2^896 for every normal
// x, so a*b = x^2 exactly (16 significant bits) and zero contributes exactly 0. (A subnormal
// bf16, |x| < 2^-126, contributes below 2^-252 instead of x^2: far below the float64 rounding
// of any row sum the contract admits.)
__device__ __forceinline__ double add_squares_exact(uint32_t w, double ss) {
  const uint32_t al = (w & 0x7FFFu) << 13, ah = (w >> 3) & 0x0FFFE000u;  // low / high value
  constexpr uint32_t kUp = 1792u << 20;
  const double a0 = __hiloint2double((int)al, 0), b0 = __hiloint2double((int)(al + kUp), 0);
  const double a1 = __hiloint2double((int)ah, 0), b1 = __hiloint2double((int)(ah + kUp), 0);
  return __fma_rn(a1, b1, __fma_rn(a0, b0, ss));
}

}  // namespace sharq
