// Weight packer (K1): one FP4 weight payload with path-specific scale views.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference",
// Abstract: "The two paths share a single FP4 weight payload with path-specific
// scale views." The weight is quantized once, in blocks of 2B consecutive K
// positions (B = 16 NVFP4 / 32 MXFP4): that is the K span one scale covers in the
// structured-sparse block-scaled MMA, whose scale vector counts stored values of a
// 50%-dense operand. The dense MMA needs one scale per B positions, so its view
// repeats each sparse-view scale twice. Both views decode to the same weight.
//
// Launch 1 reduces amax|W| into tensor_scale[1] (float bits of a non-negative value
// order like unsigned integers, so atomicMax on the bits is a float max). Launch 2
// quantizes: one thread per (row, 64-element chunk).
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

template <int FMT>
__global__ void __launch_bounds__(128) pack_kernel(PackParams p) {
  const int C = p.K / 64;
  const size_t gid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (gid >= (size_t)p.N_pad * C) return;
  const int n = (int)(gid / C), c = (int)(gid % C);
  const int spr_dense = FMT == kFmtNV ? p.K / 16 : p.K / 32;
  const int spr_sparse = spr_dense / 2;
  if (n >= p.N) {  // padding rows of the scale atoms
    if (FMT == kFmtNV) {
      *reinterpret_cast<uint16_t *>(p.sc_sparse + atom_offset(n, 2 * c, spr_sparse)) = 0;
      *reinterpret_cast<uint32_t *>(p.sc_dense + atom_offset(n, 4 * c, spr_dense)) = 0u;
    } else {
      p.sc_sparse[atom_offset(n, c, spr_sparse)] = 0;
      *reinterpret_cast<uint16_t *>(p.sc_dense + atom_offset(n, 2 * c, spr_dense)) = 0;
    }
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
    const uint32_t s0 = quant_nv<32, false>(v, s_w, g_w, bytes, nullptr);
    const uint32_t s1 = quant_nv<32, false>(v + 32, s_w, g_w, bytes + 16, nullptr);
    *reinterpret_cast<uint16_t *>(p.sc_sparse + atom_offset(n, 2 * c, spr_sparse)) = (uint16_t)(s0 | (s1 << 8));
    *reinterpret_cast<uint32_t *>(p.sc_dense + atom_offset(n, 4 * c, spr_dense)) =
        s0 | (s0 << 8) | (s1 << 16) | (s1 << 24);
  } else {
    if (gid == 0) p.tensor_scale[0] = 1.f;
    const uint32_t e = quant_mx<64, false>(v, bytes, nullptr);
    p.sc_sparse[atom_offset(n, c, spr_sparse)] = (uint8_t)e;
    *reinterpret_cast<uint16_t *>(p.sc_dense + atom_offset(n, 2 * c, spr_dense)) = (uint16_t)(e | (e << 8));
  }
  uint4 *dst = reinterpret_cast<uint4 *>(p.codes + (size_t)n * (p.K / 2) + (size_t)c * 32);
  dst[0] = make_uint4(pack4(bytes), pack4(bytes + 4), pack4(bytes + 8), pack4(bytes + 12));
  dst[1] = make_uint4(pack4(bytes + 16), pack4(bytes + 20), pack4(bytes + 24), pack4(bytes + 28));
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
