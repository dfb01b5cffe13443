// Fused SharQ preparation operator (K2) and the dense FP4 activation quantizer.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference",
// Abstract: "a fused preparation kernel absorbs mask generation, residual
// construction, and layer normalization into one operator"; the residual is
// defined "relative to the quantized sparse backbone rather than the
// unquantized sparse values".
//
// One pass over the bf16 activations. A team of threads owns one token row; each
// thread owns chunks of 64 consecutive K elements (128 bytes of input). The row's
// sum of squares (RMSNorm, float64) and amax (second-level scale) are team
// reductions; everything else is local to the chunk:
//   mask (per group of 8 for pairs / 4 for elements) -> 32 stored values ->
//   backbone blocks (2 x 16 NVFP4 / 1 x 32 MXFP4) -> dequantized backbone ->
//   residual -> residual blocks (4 x 16 / 2 x 32).
// The outputs go straight to the layouts the GEMM's TMA and tensor-core scale copies
// read, so no re-layout pass follows. Float32 operations use explicit _rn
// intrinsics so no contraction changes a rounding.
#include "sharq_common.cuh"
#include "sharq_internal.h"
#include "sharq_quant.cuh"

namespace sharq {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// mask of kept units (bit i = unit i kept) -> metadata nibble i0 | i1 << 2
constexpr unsigned long long kNibbleLut =
    (4ull << (3 * 4)) | (8ull << (5 * 4)) | (9ull << (6 * 4)) | (12ull << (9 * 4)) |
    (13ull << (10 * 4)) | (14ull << (12 * 4));

// Top-2 of four keys, ties to the lower index: the two units whose rank
// (#keys strictly above + #equal keys at lower index) is below 2.
__device__ __forceinline__ uint32_t top2_of_4(float k0, float k1, float k2, float k3) {
  int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
  if (k0 >= k1) ++r1; else ++r0;
  if (k0 >= k2) ++r2; else ++r0;
  if (k0 >= k3) ++r3; else ++r0;
  if (k1 >= k2) ++r2; else ++r1;
  if (k1 >= k3) ++r3; else ++r1;
  if (k2 >= k3) ++r3; else ++r2;
  const uint32_t m = (r0 < 2) | ((r1 < 2) << 1) | ((r2 < 2) << 2) | ((r3 < 2) << 3);
  return (uint32_t)(kNibbleLut >> (m * 4)) & 0xFu;
}

__device__ __forceinline__ float sel4(uint32_t i, float a, float b, float c, float d) {
  return i == 0 ? a : (i == 1 ? b : (i == 2 ? c : d));
}

// ---------------------------------------------------------------- team reductions
// Butterfly reductions: every lane ends with the identical result (each step adds
// the same two operands), so all threads of a row derive bit-identical scales.
template <typename V>
__device__ __forceinline__ V team_sum(V v, int TS, V *sm) {
  const int lim = TS < 32 ? TS : 32;
  for (int o = lim >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (TS > 32) {
    const int w = threadIdx.x >> 5, nw = TS >> 5;
    if ((threadIdx.x & 31) == 0) sm[w] = v;
    __syncthreads();
    v = sm[0];
    for (int i = 1; i < nw; ++i) v += sm[i];
    __syncthreads();
  }
  return v;
}

__device__ __forceinline__ float team_max(float v, int TS, float *sm) {
  const int lim = TS < 32 ? TS : 32;
  for (int o = lim >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  if (TS > 32) {
    const int w = threadIdx.x >> 5, nw = TS >> 5;
    if ((threadIdx.x & 31) == 0) sm[w] = v;
    __syncthreads();
    v = sm[0];
    for (int i = 1; i < nw; ++i) v = fmaxf(v, sm[i]);
    __syncthreads();
  }
  return v;
}

// ---------------------------------------------------------------- chunk I/O
__device__ __forceinline__ void load_bf16x64(const uint16_t *src, float *v) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 q = __ldg(s + i);
    v[8 * i + 0] = bf16lo(q.x); v[8 * i + 1] = bf16hi(q.x);
    v[8 * i + 2] = bf16lo(q.y); v[8 * i + 3] = bf16hi(q.y);
    v[8 * i + 4] = bf16lo(q.z); v[8 * i + 5] = bf16hi(q.z);
    v[8 * i + 6] = bf16lo(q.w); v[8 * i + 7] = bf16hi(q.w);
  }
}

__device__ __forceinline__ void apply_norm(float *v, const uint16_t *gamma, float rstd) {
  const uint4 *g = reinterpret_cast<const uint4 *>(gamma);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 q = __ldg(g + i);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = __fmul_rn(__fmul_rn(v[8 * i + 2 * j], rstd), bf16lo(w[j]));
      v[8 * i + 2 * j + 1] = __fmul_rn(__fmul_rn(v[8 * i + 2 * j + 1], rstd), bf16hi(w[j]));
    }
  }
}

// ---------------------------------------------------------------- one chunk
// Quantizes the 64 values v[] (already normalized) of chunk `c` of row `row`.
template <int FMT, int UNIT, bool DENSE>
__device__ __forceinline__ void process_chunk(const PrepParams &p, float *v, int row, int c, float s_x,
                                              float g_x) {
  uint32_t rb[32];  // residual code bytes (64 codes)
  if (!DENSE) {
    // ---- mask: 32 stored values and their metadata
    float sv[32];
    uint32_t nib[16];
    if (UNIT == 2) {
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float *e = v + 8 * g;
        const float k0 = fmaxf(fabsf(e[0]), fabsf(e[1])), k1 = fmaxf(fabsf(e[2]), fabsf(e[3]));
        const float k2 = fmaxf(fabsf(e[4]), fabsf(e[5])), k3 = fmaxf(fabsf(e[6]), fabsf(e[7]));
        const uint32_t n = top2_of_4(k0, k1, k2, k3);
        const uint32_t i0 = n & 3u, i1 = n >> 2;
        nib[g] = n;
        sv[4 * g + 0] = sel4(i0, e[0], e[2], e[4], e[6]);
        sv[4 * g + 1] = sel4(i0, e[1], e[3], e[5], e[7]);
        sv[4 * g + 2] = sel4(i1, e[0], e[2], e[4], e[6]);
        sv[4 * g + 3] = sel4(i1, e[1], e[3], e[5], e[7]);
      }
    } else {
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const float *e = v + 4 * g;
        const uint32_t n = top2_of_4(fabsf(e[0]), fabsf(e[1]), fabsf(e[2]), fabsf(e[3]));
        nib[g] = n;
        sv[2 * g + 0] = sel4(n & 3u, e[0], e[1], e[2], e[3]);
        sv[2 * g + 1] = sel4(n >> 2, e[0], e[1], e[2], e[3]);
      }
    }
    // ---- backbone quantization (32 stored values)
    uint32_t sb[16];
    float dq[32];
    uint32_t sc_sp;
    if (FMT == kFmtNV) {
      const uint32_t s0 = quant_nv<16, true>(sv, s_x, g_x, sb, dq);
      const uint32_t s1 = quant_nv<16, true>(sv + 16, s_x, g_x, sb + 8, dq + 16);
      sc_sp = s0 | (s1 << 8);
    } else {
      sc_sp = quant_mx<32, true>(sv, sb, dq);
    }
    // ---- residual against the quantized backbone: r = xh - deq at kept positions
    if (UNIT == 2) {
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const uint32_t i0 = nib[g] & 3u, i1 = nib[g] >> 2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float d0 = (i0 == (uint32_t)j) ? dq[4 * g + 0] : ((i1 == (uint32_t)j) ? dq[4 * g + 2] : 0.f);
          const float d1 = (i0 == (uint32_t)j) ? dq[4 * g + 1] : ((i1 == (uint32_t)j) ? dq[4 * g + 3] : 0.f);
          v[8 * g + 2 * j] = __fsub_rn(v[8 * g + 2 * j], d0);
          v[8 * g + 2 * j + 1] = __fsub_rn(v[8 * g + 2 * j + 1], d1);
        }
      }
    } else {
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const uint32_t i0 = nib[g] & 3u, i1 = nib[g] >> 2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float d = (i0 == (uint32_t)j) ? dq[2 * g] : ((i1 == (uint32_t)j) ? dq[2 * g + 1] : 0.f);
          v[4 * g + j] = __fsub_rn(v[4 * g + j], d);
        }
      }
    }
    // ---- store backbone codes, metadata and scales
    uint4 *spc = reinterpret_cast<uint4 *>(p.sp_codes + (size_t)row * (p.K / 4) + (size_t)c * 16);
    *spc = make_uint4(pack4(sb), pack4(sb + 4), pack4(sb + 8), pack4(sb + 12));
    if (UNIT == 2) {
      uint32_t m = 0;
#pragma unroll
      for (int g = 0; g < 8; ++g) m |= nib[g] << (4 * g);
      uint32_t *dst = reinterpret_cast<uint32_t *>(p.meta + ((size_t)(c >> 2) * p.T_pad + row) * 16 + (c & 3) * 4);
      *dst = m;
    } else {
      uint32_t m0 = 0, m1 = 0;
#pragma unroll
      for (int g = 0; g < 8; ++g) { m0 |= nib[g] << (4 * g); m1 |= nib[g + 8] << (4 * g); }
      uint2 *dst = reinterpret_cast<uint2 *>(p.meta + ((size_t)(c >> 1) * p.T_pad + row) * 16 + (c & 1) * 8);
      *dst = make_uint2(m0, m1);
    }
    if (FMT == kFmtNV) {
      *reinterpret_cast<uint16_t *>(p.sp_scales + atom_offset(row, 2 * c, p.n_sf_sp)) = (uint16_t)sc_sp;
    } else {
      p.sp_scales[atom_offset(row, c, p.n_sf_sp)] = (uint8_t)sc_sp;
    }
  }
  // ---- residual (or, for the dense quantizer, xh itself) in dense blocks
  uint32_t sc_res;
  if (FMT == kFmtNV) {
    uint32_t s[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) s[b] = quant_nv<16, false>(v + 16 * b, s_x, g_x, rb + 8 * b, nullptr);
    sc_res = s[0] | (s[1] << 8) | (s[2] << 16) | (s[3] << 24);
    *reinterpret_cast<uint32_t *>(p.res_scales + atom_offset(row, 4 * c, p.n_sf_res)) = sc_res;
  } else {
    const uint32_t e0 = quant_mx<32, false>(v, rb, nullptr);
    const uint32_t e1 = quant_mx<32, false>(v + 32, rb + 16, nullptr);
    *reinterpret_cast<uint16_t *>(p.res_scales + atom_offset(row, 2 * c, p.n_sf_res)) = (uint16_t)(e0 | (e1 << 8));
  }
  uint4 *rc = reinterpret_cast<uint4 *>(p.res_codes + (size_t)row * (p.K / 2) + (size_t)c * 32);
  rc[0] = make_uint4(pack4(rb), pack4(rb + 4), pack4(rb + 8), pack4(rb + 12));
  rc[1] = make_uint4(pack4(rb + 16), pack4(rb + 20), pack4(rb + 24), pack4(rb + 28));
}

// Zero scale / metadata bytes of chunk c for a padding row (rows T..T_pad-1), so the
// GEMM reads defined values there.
template <int FMT, int UNIT, bool DENSE>
__device__ __forceinline__ void zero_pad_chunk(const PrepParams &p, int row, int c) {
  if (!DENSE) {
    if (UNIT == 2)
      *reinterpret_cast<uint32_t *>(p.meta + ((size_t)(c >> 2) * p.T_pad + row) * 16 + (c & 3) * 4) = 0u;
    else
      *reinterpret_cast<uint2 *>(p.meta + ((size_t)(c >> 1) * p.T_pad + row) * 16 + (c & 1) * 8) = make_uint2(0u, 0u);
    if (FMT == kFmtNV) *reinterpret_cast<uint16_t *>(p.sp_scales + atom_offset(row, 2 * c, p.n_sf_sp)) = 0;
    else p.sp_scales[atom_offset(row, c, p.n_sf_sp)] = 0;
  }
  if (FMT == kFmtNV) *reinterpret_cast<uint32_t *>(p.res_scales + atom_offset(row, 4 * c, p.n_sf_res)) = 0u;
  else *reinterpret_cast<uint16_t *>(p.res_scales + atom_offset(row, 2 * c, p.n_sf_res)) = 0;
}

__device__ __forceinline__ void row_scales(int fmt, float amax, float &s_x, float &g_x) {
  if (fmt == kFmtMX) { s_x = 1.f; g_x = 1.f; return; }
  if (amax == 0.f) { s_x = 1.f; g_x = 0.f; return; }
  s_x = __fdiv_rn(amax, 2688.f);  // 448 (E4M3 max) * 6 (E2M1 max)
  g_x = __fdiv_rn(448.f, amax);   // = 1 / (6 s_x)
}

__device__ __forceinline__ float rstd_from(double ss, int K, float eps) {
  const float ms = __double2float_rn(__ddiv_rn(ss, (double)K));
  return __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(ms, eps)));
}

// ---------------------------------------------------------------- kernels
// Every thread owns at most one 64-element chunk (K <= 64*256) and keeps it in registers.
template <int FMT, int UNIT, bool NORM, bool DENSE>
__global__ void __launch_bounds__(256) prep_kernel(PrepParams p) {
  __shared__ double sm_d[8];
  __shared__ float sm_f[8];
  const int TS = p.TS;
  const int team = threadIdx.x / TS;
  const int c = threadIdx.x - team * TS;
  const int row = blockIdx.x * (blockDim.x / TS) + team;
  const bool live = row < p.T && c < p.C;

  float v[64];
  if (live) load_bf16x64(p.x + (size_t)row * p.K + (size_t)c * 64, v);
  else {
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = 0.f;
  }
  if (NORM) {
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 64; ++i) ss = __fma_rn((double)v[i], (double)v[i], ss);
    ss = team_sum<double>(ss, TS, sm_d);
    const float rstd = rstd_from(ss, p.K, p.eps);
    if (live) apply_norm(v, p.gamma + (size_t)c * 64, rstd);
  }
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) am = fmaxf(am, fabsf(v[i]));
  am = team_max(am, TS, sm_f);
  float s_x, g_x;
  row_scales(FMT, am, s_x, g_x);
  if (live) {
    process_chunk<FMT, UNIT, DENSE>(p, v, row, c, s_x, g_x);
    if (c == 0) p.row_scale[row] = s_x;
  } else if (row >= p.T && row < p.T_pad && c < p.C) {
    zero_pad_chunk<FMT, UNIT, DENSE>(p, row, c);
  }
}

// Rows longer than 256 chunks: 256 threads per row, chunks strided by 256, and the
// input re-read (from L2) in each of the three passes instead of held in registers.
template <int FMT, int UNIT, bool NORM, bool DENSE>
__global__ void __launch_bounds__(256) prep_kernel_long(PrepParams p) {
  __shared__ double sm_d[8];
  __shared__ float sm_f[8];
  const int row = blockIdx.x;
  const int TS = 256;
  float v[64];
  float rstd = 1.f;
  if (row >= p.T) {
    if (row < p.T_pad)
      for (int c = threadIdx.x; c < p.C; c += TS) zero_pad_chunk<FMT, UNIT, DENSE>(p, row, c);
    return;
  }
  const uint16_t *xr = p.x + (size_t)row * p.K;
  if (NORM) {
    double ss = 0.0;
    for (int c = threadIdx.x; c < p.C; c += TS) {
      load_bf16x64(xr + (size_t)c * 64, v);
#pragma unroll
      for (int i = 0; i < 64; ++i) ss = __fma_rn((double)v[i], (double)v[i], ss);
    }
    ss = team_sum<double>(ss, TS, sm_d);
    rstd = rstd_from(ss, p.K, p.eps);
  }
  float am = 0.f;
  for (int c = threadIdx.x; c < p.C; c += TS) {
    load_bf16x64(xr + (size_t)c * 64, v);
    if (NORM) apply_norm(v, p.gamma + (size_t)c * 64, rstd);
#pragma unroll
    for (int i = 0; i < 64; ++i) am = fmaxf(am, fabsf(v[i]));
  }
  am = team_max(am, TS, sm_f);
  float s_x, g_x;
  row_scales(FMT, am, s_x, g_x);
  for (int c = threadIdx.x; c < p.C; c += TS) {
    load_bf16x64(xr + (size_t)c * 64, v);
    if (NORM) apply_norm(v, p.gamma + (size_t)c * 64, rstd);
    process_chunk<FMT, UNIT, DENSE>(p, v, row, c, s_x, g_x);
  }
  if (threadIdx.x == 0) p.row_scale[row] = s_x;
}

template <int FMT, int UNIT, bool NORM, bool DENSE>
cudaError_t launch_t(const PrepParams &p, cudaStream_t st) {
  if (p.C > 256) {
    prep_kernel_long<FMT, UNIT, NORM, DENSE><<<p.T_pad, 256, 0, st>>>(p);
  } else {
    const int block = p.TS <= 32 ? 256 : p.TS;
    const int rows_per_block = block / p.TS;
    const int grid = (p.T_pad + rows_per_block - 1) / rows_per_block;
    prep_kernel<FMT, UNIT, NORM, DENSE><<<grid, block, 0, st>>>(p);
  }
  return cudaGetLastError();
}

template <int FMT, int UNIT, bool DENSE>
cudaError_t launch_n(const PrepParams &p, bool norm, cudaStream_t st) {
  return norm ? launch_t<FMT, UNIT, true, DENSE>(p, st) : launch_t<FMT, UNIT, false, DENSE>(p, st);
}

}  // namespace

// Team size: chunks per row rounded up to a power of two within a warp, or to whole
// warps beyond; rows with more than 256 chunks use the 256-thread strided kernel.
int prep_team_size(int chunks) {
  if (chunks > 256) return 256;
  if (chunks <= 32) {
    int t = 1;
    while (t < chunks) t <<= 1;
    return t;
  }
  return (chunks + 31) / 32 * 32;
}

cudaError_t launch_prep(PrepParams p, int fmt, int unit, bool norm, bool dense, cudaStream_t st) {
  p.C = p.K / 64;
  p.TS = prep_team_size(p.C);
  if (dense) {
    return fmt == kFmtNV ? launch_n<kFmtNV, 2, true>(p, norm, st) : launch_n<kFmtMX, 2, true>(p, norm, st);
  }
  if (fmt == kFmtNV)
    return unit == 2 ? launch_n<kFmtNV, 2, false>(p, norm, st) : launch_n<kFmtNV, 1, false>(p, norm, st);
  return unit == 2 ? launch_n<kFmtMX, 2, false>(p, norm, st) : launch_n<kFmtMX, 1, false>(p, norm, st);
}

}  // namespace sharq
