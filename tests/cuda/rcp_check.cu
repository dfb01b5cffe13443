// Exhaustive check of the library's rcp_rn (sharq_common.cuh) against the correctly rounded
// reciprocal __frcp_rn over every positive and negative normal float32 whose reciprocal is
// normal. Prints the mismatch count; exit status 0 when the run itself succeeded.
#include <cstdio>
#include "../../fp4_activation_sparse_b200/csrc/sharq_common.cuh"

__device__ unsigned long long g_bad;
__device__ unsigned int g_first;

__global__ void check(unsigned int lo, unsigned int hi) {
  for (unsigned long long i = lo + blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; i < hi;
       i += (unsigned long long)gridDim.x * blockDim.x) {
    for (unsigned int sign = 0; sign < 2; ++sign) {
      const float x = __uint_as_float((unsigned int)i | (sign << 31));
      if (fabsf(x) > 8.5e37f) continue;  // 1/x below the normal range
      if (__float_as_uint(sharq::rcp_rn(x)) != __float_as_uint(__frcp_rn(x))) {
        atomicAdd(&g_bad, 1ull);
        atomicMin(&g_first, (unsigned int)i);
      }
    }
  }
}

int main() {
  unsigned long long zero = 0;
  unsigned int first = ~0u;
  cudaMemcpyToSymbol(g_bad, &zero, sizeof zero);
  cudaMemcpyToSymbol(g_first, &first, sizeof first);
  check<<<148 * 16, 256>>>(0x00800000u, 0x7F800000u);  // every normal magnitude
  cudaError_t e = cudaDeviceSynchronize();
  unsigned long long bad = 0;
  cudaMemcpyFromSymbol(&bad, g_bad, sizeof bad);
  cudaMemcpyFromSymbol(&first, g_first, sizeof first);
  printf("status=%s mismatches=%llu first=0x%08x\n", cudaGetErrorString(e), bad, first);
  return e == cudaSuccess ? 0 : 1;
}
