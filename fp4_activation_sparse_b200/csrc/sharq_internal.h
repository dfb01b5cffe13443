// Internal launch interfaces between the C ABI (sharq_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sharq {

struct PrepParams {
  const uint16_t *x;      // [T][K] bf16
  const uint16_t *gamma;  // [K] bf16 or null
  float eps;
  int T, K, T_pad;
  int C;   // 64-element chunks per row
  int TS;  // threads per row team
  uint8_t *sp_codes, *meta, *sp_scales, *res_codes, *res_scales;
  float *row_scale;
  int n_sf_sp, n_sf_res;  // scales per row of the backbone / residual
};

struct PackParams {
  const uint16_t *w;  // [N][K] bf16
  int N, K, N_pad;
  uint8_t *codes, *sc_sparse, *sc_dense;
  float *tensor_scale;  // [0] s_w, [1] amax
};

struct GemmParams {
  // activation operands
  const uint8_t *a_res;       // [T][K/2]
  const uint8_t *a_sp;        // [T][K/4] (null for the dense-only GEMM)
  const uint8_t *meta;        // slabs [K/256][T_pad][16]
  const uint8_t *sfa_res;     // atoms, K/B per row
  const uint8_t *sfa_sp;      // atoms, K/(2B) per row
  const float *row_scale;     // [T]
  // weight operands
  const uint8_t *b;           // [N][K/2]
  const uint8_t *sfb_dense;   // atoms, K/B per row
  const uint8_t *sfb_sparse;  // atoms, K/(2B) per row
  const float *tensor_scale;  // [0] = s_w
  void *y;                    // [T][N]
  int T, N, K, T_pad, N_pad;
  int fmt, out_f32, sparse;
  long long wait_limit;
};

cudaError_t launch_prep(PrepParams p, int fmt, int unit, bool norm, bool dense, cudaStream_t st);
cudaError_t launch_pack(PackParams p, int fmt, cudaStream_t st);
cudaError_t launch_gemm(const GemmParams &p, cudaStream_t st, const char **why);
cudaError_t read_and_clear_device_status(int *status, cudaStream_t st);

}  // namespace sharq
