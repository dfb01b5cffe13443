// Internal launch interfaces between the C ABI (sharq_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sharq {

// ---------------------------------------------------------------- tiled operands
// Activations and weights are stored as chunks of 128 rows x 256 K, one contiguous chunk
// per (128-row block, 256-K step), chunk-major [row block][K step]. A chunk is the exact
// shared-memory image the GEMM's tensor-core descriptors and scale copies read, so one
// bulk copy moves it. Offsets inside a chunk (bytes):
//   activation, SharQ prep:  res  128 x 128 B residual codes, 128-byte swizzle
//                            sp   128 x 64 B backbone codes (kept values), 64-byte swizzle
//                            meta 128 x 16 B metadata (pair unit; element unit: two slabs
//                                 of 128 x 16 B, 4096 B)
//                            sf_sp / sf_res  backbone / residual scales as 128x4 atoms
//   activation, dense quantizer: res codes + sf_res only
//   weight (128 rows = one half of a 256-row block): b 128 x 128 B codes, 128-byte swizzle;
//                            sf_sp / sf_res the scales of the whole 256-row block (the
//                            rows of both halves, block-half-major), so each half's chunk
//                            carries what a CTA pair's MMA reads for its 256 columns.
// Chunk sizes are multiples of 1024 bytes.
struct ActTile {
  int res, sp, meta, sf_sp, sf_res, bytes;
};
struct WTile {
  int b, sf_sp, sf_res, bytes;
};
__host__ __device__ constexpr int tile_round(int a) { return (a + 1023) / 1024 * 1024; }
// scale atoms (512 B, 4 scales x 128 rows) per 256-K step for 128 rows; fmt 0 = NVFP4, 1 = MXFP4
__host__ __device__ constexpr int atoms_res(int fmt) { return fmt == 0 ? 4 : 2; }  // one scale per B
__host__ __device__ constexpr int atoms_sp(int fmt) { return fmt == 0 ? 2 : 1; }   // one scale per 2B
// Mask pattern codes (the `unit` argument of the layout and the preparation's templates):
// 2 = two of four pairs, 1 = two of four elements, kPat48 = four of eight elements.
constexpr int kPat48 = 3;
// metadata bytes per chunk: 128 rows x 16 B (pairs: 4-bit entries per 8 elements), x 32 B
// (elements 2:4: 4 bits per 4), x 48 B (elements 4:8: 12 bits per 8)
__host__ __device__ constexpr int meta_bytes(int unit) { return unit == 2 ? 2048 : unit == 1 ? 4096 : 6144; }
__host__ __device__ constexpr ActTile act_tile(int fmt, int unit, bool sparse) {
  return sparse ? ActTile{0, 16384, 24576, 24576 + meta_bytes(unit),
                          24576 + meta_bytes(unit) + 512 * atoms_sp(fmt),
                          tile_round(24576 + meta_bytes(unit) + 512 * (atoms_sp(fmt) + atoms_res(fmt)))}
                : ActTile{0, 0, 0, 0, 16384, tile_round(16384 + 512 * atoms_res(fmt))};
}
__host__ __device__ constexpr WTile w_tile(int fmt) {
  return WTile{0, 16384, 16384 + 1024 * atoms_sp(fmt), 16384 + 1024 * (atoms_sp(fmt) + atoms_res(fmt))};
}
// byte offset of (row r in 0..127, scale s of the K step) inside a run of 128x4 atoms
__host__ __device__ constexpr int atom_pos(int r, int s) { return (s >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (s & 3); }

struct PrepParams {
  const uint16_t *x;      // [T][x_stride] bf16: the activation, or [g | u] for the gated form
  const uint16_t *gamma;  // [K] bf16 or null
  int x_stride;           // elements per input row: K, or 2K for the gated form
  float eps;
  int T, K, T_pad;
  int KS;  // 256-K steps per row
  int TS;  // warps per row team
  uint8_t *tiles;         // activation chunks (act_tile layout)
  float *row_scale;       // [T]
};

struct PackParams {
  const uint16_t *w;  // [N][K] bf16
  int N, K, N_pad;
  uint8_t *tiles;       // weight chunks (w_tile layout)
  float *tensor_scale;  // [0] s_w, [1] amax
};

// One GEMM problem of a (possibly grouped) launch: Y_g = A_g . W_g^T.
struct GemmGroup {
  const uint8_t *a_tiles;     // activation chunks: SharQ prep (sparse) or dense quantizer
  const float *row_scale;     // [T]
  const uint8_t *w_tiles;     // weight chunks
  const float *tensor_scale;  // [0] = s_w
  void *y;                    // [T][N]
  int T, T_pad;
  int tile_begin, num_m;      // first pair tile of this group in the launch, its 256-row blocks
  int k0, num_k;              // the group's K steps (of 256): k0 .. k0 + num_k - 1 (split K);
                              // num_k = 0 means all of K
};

// groups per launch of the grouped GEMM: its tensor maps (3 x 128 B per group) and group table
// travel in the kernel parameters, which hold up to 32764 bytes
constexpr int kMaxGroups = 64;

struct GemmParams {
  GemmGroup grp[kMaxGroups];
  int n_groups, num_tiles;    // num_tiles: pair tiles over all groups
  int N, K, N_pad;            // shared by every group
  int fmt, out_f32, sparse;
  int single;                 // one CTA per 128 x 256 tile (set by launch_gemm), else CTA pairs
  long long wait_limit;
};

cudaError_t launch_prep(PrepParams p, int fmt, int unit, bool norm, bool dense, bool swiglu, cudaStream_t st);
cudaError_t launch_prep_tensor_scale(PrepParams p, int unit, bool norm, void *workspace, unsigned long long limit_ns,
                                     cudaStream_t st);
int prep_tensor_groups(int tokens, int k);
cudaError_t launch_prep_tensor_scale_static(PrepParams p, int unit, bool norm, unsigned long long limit_ns,
                                            cudaStream_t st, size_t *needed, size_t *capacity);
cudaError_t read_and_clear_prep_status(uint32_t *status);
cudaError_t launch_pack(PackParams p, int fmt, cudaStream_t st);
cudaError_t launch_gemm(GemmParams p, cudaStream_t st, const char **why);
cudaError_t read_and_clear_device_status(int *status, cudaStream_t st);
cudaError_t launch_mma_peak(int mode, int fmt, int iters, int clusters, cudaStream_t st);
int sm_count();
int gemm_split_count(int tokens, int n_out, int k);
cudaError_t launch_splitk_reduce(const float *ws, int S, int T, int N, void *y, int out_f32, cudaStream_t st);
cudaError_t launch_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int T, int K, uint16_t *y,
                           cudaStream_t st);

}  // namespace sharq
