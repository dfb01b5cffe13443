// Block quantizers shared by the preparation kernel and the weight packer.
#pragma once

#include "sharq_common.cuh"

namespace sharq {

// ---------------------------------------------------------------- block quantizers
// NVFP4 block of N values: returns the E4M3 scale code, writes N/2 code bytes and
// (optionally) the dequantized values fp32(fp32(dec(q)*dec(sb))*s).
template <int N, bool DEQ>
__device__ __forceinline__ uint32_t quant_nv(const float *v, float s_x, float g_x, uint32_t *bytes,
                                             float *deq) {
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) am = fmaxf(am, fabsf(v[i]));
  const uint32_t sb = cvt_e4m3(__fmul_rn(am, g_x));
  const float sbd = e4m3_to_f32(sb);
  const float d = __fmul_rn(sbd, s_x);
  if (d == 0.f) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) bytes[i] = 0u;
    if (DEQ) {
#pragma unroll
      for (int i = 0; i < N; ++i) deq[i] = 0.f;
    }
    return sb;
  }
  const float inv = __fdiv_rn(1.f, d);
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    bytes[i] = cvt_e2m1x2(__fmul_rn(v[2 * i], inv), __fmul_rn(v[2 * i + 1], inv));
    if (DEQ) {
      const float2 q = half2_bits_to_float2(cvt_e2m1x2_to_f16x2(bytes[i]));
      deq[2 * i] = __fmul_rn(__fmul_rn(q.x, sbd), s_x);
      deq[2 * i + 1] = __fmul_rn(__fmul_rn(q.y, sbd), s_x);
    }
  }
  return sb;
}

// MXFP4 block of N values: E8M0 exponent e = clamp(floor(log2 amax) - 2 + 127, 0, 254),
// codes E2M1(v * 2^(127-e)) (the scaling is exact).
template <int N, bool DEQ>
__device__ __forceinline__ uint32_t quant_mx(const float *v, uint32_t *bytes, float *deq) {
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) am = fmaxf(am, fabsf(v[i]));
  if (am == 0.f) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) bytes[i] = 0u;
    if (DEQ) {
#pragma unroll
      for (int i = 0; i < N; ++i) deq[i] = 0.f;
    }
    return 0u;
  }
  const int ef = (int)(__float_as_uint(am) >> 23);
  const uint32_t e = (uint32_t)max(ef - 2, 0);
  const float mult = __uint_as_float((254u - e) << 23);  // 2^(127-e), exact scaling
  const float sc = e8m0_to_f32(e);
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    bytes[i] = cvt_e2m1x2(__fmul_rn(v[2 * i], mult), __fmul_rn(v[2 * i + 1], mult));
    if (DEQ) {
      const float2 q = half2_bits_to_float2(cvt_e2m1x2_to_f16x2(bytes[i]));
      deq[2 * i] = __fmul_rn(q.x, sc);
      deq[2 * i + 1] = __fmul_rn(q.y, sc);
    }
  }
  return e;
}

__device__ __forceinline__ uint32_t pack4(const uint32_t *b) {
  return b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
}

}  // namespace sharq
