// Weight packer (K1): one FP4 weight payload with path-specific scale views.
//
// Per "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference"
// (Abstract), the sparse and the dense path read one set of FP4 weight codes, each with
// scales laid out for its own MMA. The weight is quantized once, in blocks of 2B consecutive K
// positions (B = 16 NVFP4 / 32 MXFP4): that is the K span one scale covers in the
// structured-sparse block-scaled MMA, whose scale vector counts stored values of a
// 50%-dense operand. The dense MMA needs one scale per B positions, so its view
// repeats each sparse-view scale twice. Both views decode to the same weight.
//
// Launch 1 reduces amax|W| into tensor_scale[1] (float bits of a non-negative value
// order like unsigned integers, so atomicMax on the bits is a float max). Launch 2
// quantizes: one thread per (row, 64-element piece), writing the tiled weight operand
// (chunks of 128 rows x 256 K: 128-byte-swizzled codes plus both scale views of the
// 256-row block, stored in the chunks of both of its halves). Rows N..N_pad-1 are zeroed.
#include "sharq_common.cuh"
#include "sharq_internal.h"
#include "sharq_quant.cuh"

namespace sharq {
namespace {

__global__ void __launch_bounds__(256) amax_kernel(const uint16_t *w, size_t n_vec8, uint32_t *amax_bits) {
  const uint4 *src = reinterpret_cast<const uint4 *>(w);
  uint32_t m = 0;  // max of |bf16| bit patterns (sign cleared), as uint
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_vec8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 q = __ldg(src + i);
    const uint32_t ws[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m = max(m, (ws[j] << 16) & 0x7FFF0000u);
      m = max(m, ws[j] & 0x7FFF0000u);
    }
  }
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t sm[8];
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = max(m, sm[i]);
    atomicMax(amax_bits, m);
  }
}

// Scale bytes of one 64-K piece: `sp` (2 NVFP4 / 1 MXFP4 bytes) at sparse-view index s0
// and `dn` (4 / 2 bytes) at dense-view index d0 of the K step, written for row n into the
// chunks of both halves of its 256-row block.
template <int FMT>
__device__ __forceinline__ void store_scales(const PackParams &p, int n, int ks, int s0, int d0, uint32_t sp,
                                             uint32_t dn) {
  constexpr WTile L = w_tile(FMT);
  const int KS = p.K / 256, r = n & 127, half = (n >> 7) & 1;
  for (int h = 0; h < 2; ++h) {
    uint8_t *chunk = p.tiles + ((size_t)(((n >> 8) << 1) + h) * KS + ks) * L.bytes;
    uint8_t *sp_at = chunk + L.sf_sp + half * 512 * atoms_sp(FMT) + atom_pos(r, s0);
    uint8_t *dn_at = chunk + L.sf_res + half * 512 * atoms_res(FMT) + atom_pos(r, d0);
    if (FMT == kFmtNV) {
      *reinterpret_cast<uint16_t *>(sp_at) = (uint16_t)sp;
      *reinterpret_cast<uint32_t *>(dn_at) = dn;
    } else {
      *sp_at = (uint8_t)sp;
      *reinterpret_cast<uint16_t *>(dn_at) = (uint16_t)dn;
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(128) pack_kernel(PackParams p) {
  constexpr WTile L = w_tile(FMT);
  const int C = p.K / 64;
  const size_t gid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (gid >= (size_t)p.N_pad * C) return;
  const int n = (int)(gid / C), c = (int)(gid % C);
  const int ks = c >> 2, c4 = c & 3, r = n & 127;
  // sparse view: NVFP4 2 scales (of 32 K) per piece, MXFP4 1 (of 64 K); dense view twice as many
  const int s0 = FMT == kFmtNV ? 2 * c4 : c4, d0 = 2 * s0;
  uint4 *dst = reinterpret_cast<uint4 *>(p.tiles + ((size_t)(n >> 7) * (p.K / 256) + ks) * L.bytes + L.b + r * 128);
  const int u0 = 2 * c4;  // 16-byte units u0, u0+1 of the 128-byte row, swizzled with row bits 0..2
  if (n >= p.N) {  // padding rows
    store_scales<FMT>(p, n, ks, s0, d0, 0u, 0u);
    dst[u0 ^ (r & 7)] = make_uint4(0u, 0u, 0u, 0u);
    dst[(u0 + 1) ^ (r & 7)] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  float v[64];
  const uint4 *src = reinterpret_cast<const uint4 *>(p.w + (size_t)n * p.K + (size_t)c * 64);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 q = __ldg(src + i);
    v[8 * i + 0] = bf16lo(q.x); v[8 * i + 1] = bf16hi(q.x);
    v[8 * i + 2] = bf16lo(q.y); v[8 * i + 3] = bf16hi(q.y);
    v[8 * i + 4] = bf16lo(q.z); v[8 * i + 5] = bf16hi(q.z);
    v[8 * i + 6] = bf16lo(q.w); v[8 * i + 7] = bf16hi(q.w);
  }
  uint32_t bytes[32];
  if (FMT == kFmtNV) {
    const float amax = p.tensor_scale[1];
    const float s_w = amax == 0.f ? 1.f : __fdiv_rn(amax, 2688.f);
    const float g_w = amax == 0.f ? 0.f : __fdiv_rn(448.f, amax);
    if (gid == 0) p.tensor_scale[0] = s_w;
    const uint32_t e0 = quant_nv<32, false>(v, s_w, g_w, bytes, nullptr);
    const uint32_t e1 = quant_nv<32, false>(v + 32, s_w, g_w, bytes + 16, nullptr);
    store_scales<FMT>(p, n, ks, s0, d0, e0 | (e1 << 8), e0 | (e0 << 8) | (e1 << 16) | (e1 << 24));
  } else {
    if (gid == 0) p.tensor_scale[0] = 1.f;
    const uint32_t e = quant_mx<64, false>(v, bytes, nullptr);
    store_scales<FMT>(p, n, ks, s0, d0, e, e | (e << 8));
  }
  dst[u0 ^ (r & 7)] = make_uint4(pack4(bytes), pack4(bytes + 4), pack4(bytes + 8), pack4(bytes + 12));
  dst[(u0 + 1) ^ (r & 7)] = make_uint4(pack4(bytes + 16), pack4(bytes + 20), pack4(bytes + 24), pack4(bytes + 28));
}

}  // namespace

cudaError_t launch_pack(PackParams p, int fmt, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(p.tensor_scale, 0, 2 * sizeof(float), st);
  if (e != cudaSuccess) return e;
  const size_t n_vec8 = (size_t)p.N * p.K / 8;
  const int blocks = (int)((n_vec8 + 255) / 256 < 148 * 8 ? (n_vec8 + 255) / 256 : 148 * 8);
  amax_kernel<<<blocks, 256, 0, st>>>(p.w, n_vec8, reinterpret_cast<uint32_t *>(p.tensor_scale + 1));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t threads = (size_t)p.N_pad * (p.K / 64);
  const int grid = (int)((threads + 127) / 128);
  if (fmt == kFmtNV) pack_kernel<kFmtNV><<<grid, 128, 0, st>>>(p);
  else pack_kernel<kFmtMX><<<grid, 128, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sharq
