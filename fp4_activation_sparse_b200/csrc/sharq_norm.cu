// Stand-alone RMSNorm: the separate normalization pass of the dense-FP4 baseline pipeline
// (normalize into a bf16 tensor, then quantize it densely, then the dense FP4 GEMM). The
// SharQ preparation operator performs the same normalization inside its single pass; this
// kernel exists so the pipeline it replaces can be measured with the library's own code.
//
// One CTA per row: every thread loads 16-byte units (8 bf16) of the row into registers, the
// float64 sum of the exact squares is reduced over the CTA, and the row is written back as
// y = bf16_RNE(fp32(fp32(x * rstd) * gamma)), rstd = 1/sqrt(fp32(sum/K) + eps) -- the same
// normalized value the preparation operator quantizes, rounded to bf16 as an unfused pipeline
// would hand it to the next kernel.
#include "sharq_common.cuh"
#include "sharq_internal.h"

namespace sharq {
namespace {

constexpr int kUnitsPerThread = 4;  // up to 32 bf16 per thread: K <= 32768 with 1024 threads

__device__ __forceinline__ void ld128(const void *p, uint32_t (&r)[4]) {
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "l"(p));
}

__global__ void __launch_bounds__(1024) rmsnorm_kernel(const uint16_t *x, const uint16_t *gamma, float eps, int K,
                                                       uint16_t *y) {
  __shared__ double red[32];
  __shared__ float rstd_s;
  const size_t row = blockIdx.x;
  const int units = K / 8;
  uint32_t w[kUnitsPerThread][4];
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < kUnitsPerThread; ++i) {
    const int u = threadIdx.x + i * blockDim.x;
    if (u < units) {
      ld128(x + row * K + (size_t)u * 8, w[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) ss = add_squares_exact(w[i][j], ss);
    }
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    rstd_s = __frcp_rn(__fsqrt_rn(__fadd_rn(__double2float_rn(__ddiv_rn(t, (double)K)), eps)));
  }
  __syncthreads();
  const float rstd = rstd_s;
#pragma unroll
  for (int i = 0; i < kUnitsPerThread; ++i) {
    const int u = threadIdx.x + i * blockDim.x;
    if (u < units) {
      uint32_t g[4];
      ld128(gamma + (size_t)u * 8, g);
      uint4 o;
      uint32_t *op = &o.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = __fmul_rn(__fmul_rn(bf16lo(w[i][j]), rstd), bf16lo(g[j]));
        const float b = __fmul_rn(__fmul_rn(bf16hi(w[i][j]), rstd), bf16hi(g[j]));
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        op[j] = *reinterpret_cast<const uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(y + row * K + (size_t)u * 8) = o;
    }
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int T, int K, uint16_t *y,
                           cudaStream_t st) {
  const int units = K / 8;
  int threads = (units + kUnitsPerThread - 1) / kUnitsPerThread;
  threads = (threads + 31) / 32 * 32;
  if (threads > 1024) return cudaErrorInvalidValue;
  if (threads < 64) threads = 64;
  rmsnorm_kernel<<<T, threads, 0, st>>>(x, gamma, eps, K, y);
  return cudaGetLastError();
}

}  // namespace sharq
