// Fused SharQ preparation operator (K2) and the dense FP4 activation quantizer.
//
// Per "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference"
// (Abstract), one kernel performs the normalization, the choice of the mask and the
// construction of the residual; the residual is taken against the backbone after its FP4
// rounding, not against the backbone's unrounded values.
//
// One read of the bf16 activations. A team of W warps owns one token row (W = K/4096
// rounded up); every lane owns "double pieces" of 16 consecutive K elements (one 256-bit
// load), consecutive lanes owning consecutive pieces, and keeps its whole share of the
// row in registers. Passes over those registers: sum of squares (RMSNorm, float64), row
// amax (second-level scale), then per double piece:
//   mask (2 groups of 4 pairs / 4 groups of 4 elements; a tournament picks the two
//   largest keys) -> backbone block amax (the largest element of a group is always kept,
//   so it is the max of the group maxima) -> backbone codes for every element with the
//   backbone block scale; the kept bytes are stored, the dropped ones zeroed ->
//   dequantized backbone -> residual r = xh - deq -> residual block scale and codes.
// Blocks spanning lanes reduce with warp shuffles. Every output goes straight into the
// tiled activation operand (chunks of 128 rows x 256 K holding swizzled codes, metadata
// and 128x4 scale atoms: the GEMM's shared-memory image); rows T..T_pad-1 are zeroed. The RMSNorm weight is staged once
// per block in shared memory as float32. Float32 arithmetic uses explicit
// round-to-nearest operations so that no contraction changes a rounding: scalar mul.rn /
// sub.rn, or the packed f32x2 forms, which round each lane exactly like the scalar ones
// (checked bitwise on B200 over random finite operands, subnormals, signed zeros and
// infinities) but which the assembler may fuse into a packed FMA when a packed product
// feeds a packed add. So a packed product never feeds an addition here: products that do
// (x*rstd*gamma and the dequantized backbone, both subtracted for the residual) are scalar.
#include <mutex>

#include "sharq_common.cuh"
#include "sharq_internal.h"

namespace sharq {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kMaxDP = 8;  // double pieces (16 elements) per lane, at most

// The two largest of four keys, ties to the lower index, as a metadata nibble i0 | i1 << 2
// (i0 < i1); also returns the largest key. Tournament: winners and losers of (0,1) and
// (2,3), the overall winner, then the runner-up among the winner's pair loser and the other
// pair's winner (on equal keys the lower index wins every comparison).
__device__ __forceinline__ uint32_t top2_of_4(float k0, float k1, float k2, float k3, float &kmax) {
  const bool c01 = k0 >= k1, c23 = k2 >= k3;
  const float hi01 = fmaxf(k0, k1), lo01 = fminf(k0, k1), hi23 = fmaxf(k2, k3), lo23 = fminf(k2, k3);
  const uint32_t ih01 = c01 ? 0u : 1u, il01 = ih01 ^ 1u, ih23 = c23 ? 2u : 3u, il23 = ih23 ^ 1u;
  const bool cw = hi01 >= hi23;
  const uint32_t first = cw ? ih01 : ih23;
  const uint32_t second = cw ? (lo01 >= hi23 ? il01 : ih23) : (hi01 >= lo23 ? ih01 : il23);
  kmax = fmaxf(hi01, hi23);
  return min(first, second) | (max(first, second) << 2);
}

// The four largest of eight keys, ties to the lower index, as a bit mask (bit i: key i kept).
// Key i is kept when fewer than four keys beat it: key j beats key i when it is larger, or
// equal with j < i. Each of the 28 pairs is compared once.
__device__ __forceinline__ uint32_t top4_of_8(const float *a) {
  int beaten[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = i + 1; j < 8; ++j) {
      const int jb = a[j] > a[i] ? 1 : 0;  // the higher index wins only when strictly larger
      beaten[i] += jb;
      beaten[j] += 1 - jb;
    }
  uint32_t keep = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) keep |= (beaten[i] < 4 ? 1u : 0u) << i;
  return keep;
}

// ---------------------------------------------------------------- I/O
__device__ __forceinline__ void ld256(const void *p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

// Packed float32 pairs: (a, b) op= (c, d), each lane rounded to nearest even.
__device__ __forceinline__ void mul2(float &a, float &b, float c, float d) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tmul.rn.f32x2 z, x, y;\n\t"
      "mov.b64 {%0, %1}, z;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(c), "f"(d));
}
__device__ __forceinline__ void sub2(float &a, float &b, float c, float d) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tsub.rn.f32x2 z, x, y;\n\t"
      "mov.b64 {%0, %1}, z;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(c), "f"(d));
}

// Exact squares of a word's two bf16 values added to a float64 sum (low half first).
__device__ __forceinline__ double add_squares(uint32_t w, double ss) {
  double lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f64.bf16 %0, l;\n\tcvt.f64.bf16 %1, h;\n\t}"
      : "=d"(lo), "=d"(hi)
      : "r"(w));
  return __fma_rn(hi, hi, __fma_rn(lo, lo, ss));
}

// ---------------------------------------------------------------- gated activation
// x = bf16_RNE(fp32(silu(g) * u)) with silu(g) = fp32(g * sigma(g)), sigma(g) = 1/(1+e) for
// g >= 0 and e/(1+e) for g < 0, e = exp(-|g|) -- the down projection's input computed inside
// the preparation operator. exp by range reduction with Cody and Waite's two-part ln 2 and a
// degree-7 Taylor polynomial of e^x on |x| <= ln2/2 (W. J. Cody and W. Waite, "Software
// Manual for the Elementary Functions", 1980): every step a separate round-to-nearest
// float32 operation, the division correctly rounded, no fused multiply-add, so the result
// is a fixed function of g (|g| log2 e >= 126 gives e = 0).
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2Hi = 0.693145751953125f;  // 15 significant bits: n * kLn2Hi is exact for n <= 126
constexpr float kLn2Lo = (float)(0.6931471805599453 - 0.693145751953125);

__device__ __forceinline__ float exp_neg_abs(float g) {
  const float a = fabsf(g);
  const float t = __fmul_rn(a, kLog2e);
  const float n = rintf(fminf(t, 126.f));
  const float r = __fsub_rn(__fsub_rn(a, __fmul_rn(n, kLn2Hi)), __fmul_rn(n, kLn2Lo));
  const float x = -r;
  float q = (float)(1.0 / 5040.0);
  q = __fadd_rn(__fmul_rn(q, x), (float)(1.0 / 720.0));
  q = __fadd_rn(__fmul_rn(q, x), (float)(1.0 / 120.0));
  q = __fadd_rn(__fmul_rn(q, x), (float)(1.0 / 24.0));
  q = __fadd_rn(__fmul_rn(q, x), (float)(1.0 / 6.0));
  q = __fadd_rn(__fmul_rn(q, x), 0.5f);
  q = __fadd_rn(__fmul_rn(q, x), 1.f);
  q = __fadd_rn(__fmul_rn(q, x), 1.f);
  const float e = __fmul_rn(q, __int_as_float((127 - (int)n) << 23));  // * 2^-n, exact scale
  return t >= 126.f ? 0.f : e;
}

__device__ __forceinline__ float gated(float g, float u) {
  const float e = exp_neg_abs(g);
  const float sigma = __fdiv_rn(g >= 0.f ? 1.f : e, __fadd_rn(1.f, e));
  return __fmul_rn(__fmul_rn(g, sigma), u);
}

// 16 gated activations from a 256-bit word group of g and one of u, as packed bf16 (RNE)
__device__ __forceinline__ void gated16(const uint32_t (&g)[8], const uint32_t (&u)[8], uint32_t (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(gated(bf16lo(g[i]), bf16lo(u[i])), gated(bf16hi(g[i]), bf16hi(u[i])));
    x[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
}

__device__ __forceinline__ void unpack16(const uint32_t (&w)[8], float *v) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16lo(w[i]);
    v[2 * i + 1] = bf16hi(w[i]);
  }
}

// Float offset of element k of the RMSNorm weight in shared memory: [dp / 32][chunk][lane][4]
// with dp = k / 16, chunk = (k % 16) / 4, so a warp's 32 lanes read 32 consecutive 16-byte
// chunks (no bank conflicts).
__device__ __forceinline__ int gamma_smem_index(int k) {
  const int dp = k >> 4, c = (k >> 2) & 3;
  return ((((dp >> 5) << 2) + c) * 32 + (dp & 31)) * 4 + (k & 3);
}

// xh = fp32(fp32(x * rstd) * gamma) for the 16 values of a double piece whose staged weights
// start at g4 (this lane's chunk 0; chunk c at g4 + 32 c). PACKED_GAMMA: the gamma product
// may be packed (its result feeds no addition: the row-amax pass).
template <bool PACKED_GAMMA>
__device__ __forceinline__ void normalize16(float *v, const float4 *g4, float rstd) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 g = g4[32 * c];
    mul2(v[4 * c + 0], v[4 * c + 1], rstd, rstd);
    mul2(v[4 * c + 2], v[4 * c + 3], rstd, rstd);
    if (PACKED_GAMMA) {
      mul2(v[4 * c + 0], v[4 * c + 1], g.x, g.y);
      mul2(v[4 * c + 2], v[4 * c + 3], g.z, g.w);
    } else {
      v[4 * c + 0] = __fmul_rn(v[4 * c + 0], g.x);
      v[4 * c + 1] = __fmul_rn(v[4 * c + 1], g.y);
      v[4 * c + 2] = __fmul_rn(v[4 * c + 2], g.z);
      v[4 * c + 3] = __fmul_rn(v[4 * c + 3], g.w);
    }
  }
}

// max over m and the 16 values |v[i]| (a tree of three-input maxima)
__device__ __forceinline__ float amax16(const float *v, float m) {
  const float t0 = max3abs(v[0], v[1], v[2]), t1 = max3abs(v[3], v[4], v[5]), t2 = max3abs(v[6], v[7], v[8]);
  const float t3 = max3abs(v[9], v[10], v[11]), t4 = max3abs(v[12], v[13], v[14]);
  const float u0 = max3abs(t0, t1, t2), u1 = max3abs(t3, t4, v[15]);
  return max3abs(m, u0, u1);
}

// ---------------------------------------------------------------- block scales
// NVFP4: E4M3 code of fp32(amax*g); d = fp32(dec*s); inv = 1/d (0 when d = 0).
struct NvScale {
  uint32_t code;
  float dec;  // decoded E4M3 scale
  float inv;  // 1/d
  bool zero;  // d == 0: all codes of the block are zero
};
__device__ __forceinline__ NvScale nv_scale(float amax, float s_x, float g_x) {
  NvScale s;
  s.code = cvt_e4m3(__fmul_rn(amax, g_x));
  s.dec = e4m3_to_f32(s.code);
  const float d = __fmul_rn(s.dec, s_x);
  s.zero = d == 0.f;
  s.inv = s.zero ? 0.f : rcp_rn(d);  // d normal: the row-scale contract
  return s;
}

// MXFP4: E8M0 exponent e; multiplier 2^(127-e) (exact); decoded scale 2^(e-127).
struct MxScale {
  uint32_t code;
  float mult, dec;
  bool zero;
};
__device__ __forceinline__ MxScale mx_scale(float amax) {
  MxScale s;
  s.zero = amax == 0.f;
  const int ef = (int)(__float_as_uint(amax) >> 23);
  s.code = s.zero ? 0u : (uint32_t)max(ef - 2, 0);
  s.mult = __uint_as_float((254u - s.code) << 23);
  s.dec = e8m0_to_f32(s.code);
  return s;
}

// Codes of 16 values scaled by `mult` -> two words (lower K in the low nibble).
__device__ __forceinline__ void codes16(const float *v, float mult, uint32_t &w0, uint32_t &w1) {
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    t[i] = v[i];
    t[i + 1] = v[i + 1];
    mul2(t[i], t[i + 1], mult, mult);
  }
  w0 = cvt_e2m1x8(t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]);
  w1 = cvt_e2m1x8(t[8], t[9], t[10], t[11], t[12], t[13], t[14], t[15]);
}

// Dequantized values of one word of codes (8 values): NVFP4 fp32(fp32(q*dec)*s_x) with the
// exact product q*dec taken in half precision; MXFP4 q*dec (exact).
template <int FMT>
__device__ __forceinline__ void deq8(uint32_t w, float dec, float s_x, float *o) {
  uint32_t h[4];
  cvt_e2m1x8_to_f16x2(w, h);
  if (FMT == kFmtNV) {
    const __half2 d2 = __float2half2_rn(dec);  // E4M3 values are exact in half precision
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 q = __hmul2(*reinterpret_cast<const __half2 *>(&h[j]), d2);  // exact (<= 6 significant bits)
      const float2 f = __half22float2(q);  // scalar products: they feed the residual subtraction
      o[2 * j] = __fmul_rn(f.x, s_x);
      o[2 * j + 1] = __fmul_rn(f.y, s_x);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = half2_bits_to_float2(h[j]);
      o[2 * j] = __fmul_rn(f.x, dec);
      o[2 * j + 1] = __fmul_rn(f.y, dec);
    }
  }
}

// Where a lane's double pieces land in the tiled operand. A lane's pieces dp = i*32W + 32wt +
// lane all have the same position j = dp % 16 inside their 256-K step (32W and 32 are
// multiples of 16) and the same row, so every offset inside a chunk is fixed per lane; only
// the chunk changes from piece to piece.
struct Spot {
  int res, sp, meta, sf_sp, sf_res;  // byte offsets inside a chunk (sf_*: -1 = no scale byte here)
  int mb;                            // elements 4:8: first metadata byte of the lane in its row
};
template <int FMT, int UNIT, bool DENSE>
__device__ __forceinline__ Spot lane_spot(int row, int lane) {
  constexpr ActTile L = act_tile(FMT, UNIT, !DENSE);
  const int r = row & 127, j = lane & 15;
  Spot o;
  // 128-byte rows, 16-byte unit j/2 swizzled with row bits 0..2
  o.res = L.res + r * 128 + (((j >> 1) ^ (r & 7)) << 4) + (j & 1) * 8;
  // 64-byte rows, 16-byte unit j/4 swizzled with row bits 1..2
  o.sp = L.sp + r * 64 + (((j >> 2) ^ ((r >> 1) & 3)) << 4) + (j & 3) * 4;
  // pairs: byte j of the row's 16; elements 2:4: 2 bytes at 2j of 32 (halves of 16 B 2048 apart);
  // elements 4:8: 3 bytes from 3j of 48 (thirds of 16 B 2048 apart; store16 places each byte)
  o.meta = UNIT == 2 ? L.meta + r * 16 + j
                     : UNIT == 1 ? L.meta + (j >> 3) * 2048 + r * 16 + (j & 7) * 2 : L.meta + r * 16;
  o.mb = 3 * j;
  if (FMT == kFmtNV) {  // one backbone scale per 2 pieces, one residual scale per piece
    o.sf_sp = (j & 1) == 0 ? L.sf_sp + atom_pos(r, j >> 1) : -1;
    o.sf_res = L.sf_res + atom_pos(r, j);
  } else {  // one backbone scale per 4 pieces, one residual scale per 2
    o.sf_sp = (j & 3) == 0 ? L.sf_sp + atom_pos(r, j >> 2) : -1;
    o.sf_res = (j & 1) == 0 ? L.sf_res + atom_pos(r, j >> 1) : -1;
  }
  return o;
}

// Store the results of one double piece into its chunk: backbone codes (4 bytes: 8 kept
// values), metadata (pair unit 8 bits, element unit 16 bits), the backbone block scale (first
// lane of its block), residual codes (8 bytes) and the residual block scale.
template <int FMT, int UNIT, bool DENSE>
__device__ __forceinline__ void store16(uint8_t *chunk, const Spot &o, uint32_t kept, uint32_t meta, uint32_t sc_sp,
                                        uint32_t r0, uint32_t r1, uint32_t sc_res) {
  if (!DENSE) {
    *reinterpret_cast<uint32_t *>(chunk + o.sp) = kept;
    if (UNIT == 2) {
      chunk[o.meta] = (uint8_t)meta;
    } else if (UNIT == 1) {
      *reinterpret_cast<uint16_t *>(chunk + o.meta) = (uint16_t)meta;
    } else {
#pragma unroll
      for (int b = 0; b < 3; ++b) {
        const int mb = o.mb + b;
        chunk[o.meta + (mb >> 4) * 2048 + (mb & 15)] = (uint8_t)(meta >> (8 * b));
      }
    }
    if (o.sf_sp >= 0) chunk[o.sf_sp] = (uint8_t)sc_sp;
  }
  *reinterpret_cast<uint2 *>(chunk + o.res) = make_uint2(r0, r1);
  if (o.sf_res >= 0) chunk[o.sf_res] = (uint8_t)sc_res;
}

// ---------------------------------------------------------------- one double piece
// 16 normalized values of double piece `dp` (lane-aligned: dp % 32 == lane).
template <int FMT, int UNIT, bool DENSE>
__device__ __forceinline__ void process16(uint8_t *chunk, const Spot &o, float *v, bool live, float s_x,
                                          float g_x) {
  uint32_t kept = 0u, meta = 0u, sc_sp = 0u;
  if (!DENSE) {
    // ---- mask
    uint32_t nib[4];
    float gmax = 0.f;
    if (UNIT == 2) {
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const float *e = v + 8 * g;
        float km;
        nib[g] = top2_of_4(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])),
                           fmaxf(fabsf(e[4]), fabsf(e[5])), fmaxf(fabsf(e[6]), fabsf(e[7])), km);
        gmax = fmaxf(gmax, km);
      }
    } else if (UNIT == 1) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float *e = v + 4 * g;
        float km;
        nib[g] = top2_of_4(fabsf(e[0]), fabsf(e[1]), fabsf(e[2]), fabsf(e[3]), km);
        gmax = fmaxf(gmax, km);
      }
    } else {
      // elements 4:8: nib[g] holds group g's keep mask (8 bits, four set); the group maximum
      // is always kept, so the backbone block amax is the amax of all 16 values
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fabsf(v[8 * g + i]);
        nib[g] = top4_of_8(a);
      }
      gmax = amax16(v, 0.f);
    }
    // ---- backbone block amax: 16 stored (NVFP4) = 2 lanes, 32 stored (MXFP4) = 4 lanes
    gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 1));
    if (FMT == kFmtMX) gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 2));
    float mult, dec;
    bool zero;
    if (FMT == kFmtNV) {
      const NvScale s = nv_scale(gmax, s_x, g_x);
      sc_sp = s.code; mult = s.inv; dec = s.dec; zero = s.zero;
    } else {
      const MxScale s = mx_scale(gmax);
      sc_sp = s.code; mult = s.mult; dec = s.dec; zero = s.zero;
    }
    // ---- backbone codes of all 16 values; keep the selected ones
    uint32_t w0, w1;
    codes16(v, mult, w0, w1);
    if (zero) { w0 = 0u; w1 = 0u; }
    if (UNIT == 2) {
      // group g = word g: byte j = pair j; kept bytes i0, i1
      const uint32_t n0 = nib[0], n1 = nib[1];
      const uint32_t k0 = __byte_perm(w0, 0u, (n0 & 3u) | ((n0 >> 2) << 4));
      const uint32_t k1 = __byte_perm(w1, 0u, (n1 & 3u) | ((n1 >> 2) << 4));
      kept = __byte_perm(k0, k1, 0x5410);
      w0 &= (0xFFu << (8 * (n0 & 3u))) | (0xFFu << (8 * (n0 >> 2)));
      w1 &= (0xFFu << (8 * (n1 & 3u))) | (0xFFu << (8 * (n1 >> 2)));
      meta = n0 | (n1 << 4);
    } else if (UNIT == kPat48) {
      // group g = word g: keep the four selected nibbles in index order (16 bits), zero the
      // others; metadata: the four indices, 3 bits each, ascending (12 bits per group)
      kept = 0u;
      meta = 0u;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t &w = g == 0 ? w0 : w1;
        const uint32_t keep = nib[g];
        uint32_t q = 0u, m = 0u, nmask = 0u;
        int pos = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((keep >> i) & 1u) {
            q |= ((w >> (4 * i)) & 0xFu) << (4 * pos);
            m |= (uint32_t)i << (3 * pos);
            nmask |= 0xFu << (4 * i);
            ++pos;
          }
        }
        w &= nmask;
        kept |= q << (16 * g);
        meta |= m << (12 * g);
      }
    } else {
      // group g = 16 bits (4 nibbles) of the words; kept nibbles i0, i1 -> one byte
      kept = 0u;
      meta = 0u;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t &w = g < 2 ? w0 : w1;
        const int sh = 16 * (g & 1);
        const uint32_t n = nib[g], i0 = n & 3u, i1 = n >> 2;
        const uint32_t q = w >> sh;
        kept |= (((q >> (4 * i0)) & 0xFu) | (((q >> (4 * i1)) & 0xFu) << 4)) << (8 * g);
        w &= ~(0xFFFFu << sh) | (((0xFu << (4 * i0)) | (0xFu << (4 * i1))) << sh);
        meta |= n << (4 * g);
      }
    }
    // ---- residual against the dequantized backbone (dropped codes were zeroed: +0)
    float dq[16];
    deq8<FMT>(w0, dec, s_x, dq);
    deq8<FMT>(w1, dec, s_x, dq + 8);
#pragma unroll
    for (int i = 0; i < 16; i += 2) sub2(v[i], v[i + 1], dq[i], dq[i + 1]);
  }
  // ---- residual (or xh itself for the dense quantizer): dense blocks
  float am = amax16(v, 0.f);
  uint32_t r0, r1, sc_res;
  if (FMT == kFmtNV) {  // block = this lane's 16 values
    const NvScale s = nv_scale(am, s_x, g_x);
    codes16(v, s.inv, r0, r1);
    if (s.zero) { r0 = 0u; r1 = 0u; }
    sc_res = s.code;
  } else {  // block of 32 = 2 lanes
    am = fmaxf(am, __shfl_xor_sync(kFull, am, 1));
    const MxScale s = mx_scale(am);
    codes16(v, s.mult, r0, r1);
    if (s.zero) { r0 = 0u; r1 = 0u; }
    sc_res = s.code;
  }
  if (live) store16<FMT, UNIT, DENSE>(chunk, o, kept, meta, sc_sp, r0, r1, sc_res);
}

// ---------------------------------------------------------------- team reductions
// Butterfly within the warp (every lane ends with the identical value), then the W warps of
// a team combine their partials in a fixed order through shared memory.
__device__ __forceinline__ double team_sum(double v, int W, int team, int wt, double *sm) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (W > 1) {
    if ((threadIdx.x & 31) == 0) sm[team * 8 + wt] = v;
    __syncthreads();
    v = sm[team * 8];
    for (int i = 1; i < W; ++i) v += sm[team * 8 + i];
    __syncthreads();
  }
  return v;
}

__device__ __forceinline__ float team_max(float v, int W, int team, int wt, float *sm) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  if (W > 1) {
    if ((threadIdx.x & 31) == 0) sm[team * 8 + wt] = v;
    __syncthreads();
    v = sm[team * 8];
    for (int i = 1; i < W; ++i) v = fmaxf(v, sm[team * 8 + i]);
    __syncthreads();
  }
  return v;
}

__device__ __forceinline__ void row_scales(int fmt, float amax, float &s_x, float &g_x) {
  if (fmt == kFmtMX) { s_x = 1.f; g_x = 1.f; return; }
  if (amax == 0.f) { s_x = 1.f; g_x = 0.f; return; }
  s_x = __fdiv_rn(amax, 2688.f);  // 448 (E4M3 max) * 6 (E2M1 max)
  g_x = __fdiv_rn(448.f, amax);   // = 1 / (6 s_x)
}

// ---------------------------------------------------------------- kernel
// Kernel modes. kRow: one second-level scale per row (written to row_scale). kSwiglu: as kRow,
// the input formed as SiLU(g)*u from [g | u].
constexpr int kRow = 0, kSwiglu = 1;

// UNROLLED: the branch-free piece loop for rows whose every piece is live, in its own
// instantiation (the other instantiations hold only the per-piece loop). Two blocks per SM:
// the register cap keeps 16 warps per SM (the branch-free loop alone would take ~142
// registers; capped, a few bytes spill).
template <int FMT, int UNIT, bool NORM, bool DENSE, int MODE, int DP, bool UNROLLED>
__global__ void __launch_bounds__(256, 2) prep_kernel(PrepParams p) {
  extern __shared__ float4 gamma_smem4[];  // NORM: the RMSNorm weight as float32 (K rounded up to 512)
  __shared__ double sm_d[64];
  __shared__ float sm_f[64];
  float *gs = reinterpret_cast<float *>(gamma_smem4);  // [dp/32][chunk][lane][4] (gamma_smem_index)
  const int W = p.TS;  // warps per row team
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int team = warp / W, wt = warp - team * W;
  const int row = blockIdx.x * ((blockDim.x >> 5) / W) + team;
  const int ndp_row = p.K >> 4;  // double pieces per row
  const int stride = 32 * W;
  const bool live_row = row < p.T;

  // A GEMM launched after this kernel as its programmatic dependent may start its prologue on
  // SMs this grid leaves; it reads our outputs only after this grid has completed.
  asm volatile("griddepcontrol.launch_dependents;");
  uint32_t xr[DP][8];
#pragma unroll
  for (int i = 0; i < DP; ++i) {
    const int dp = i * stride + wt * 32 + lane;
    if (live_row && dp < ndp_row) {
      const uint16_t *src = p.x + (size_t)row * p.x_stride + (size_t)dp * 16;
      ld256(src, xr[i]);
      if (MODE == kSwiglu) {  // xr holds g; u sits K columns further
        uint32_t u[8];
        ld256(src + p.K, u);
        gated16(xr[i], u, xr[i]);
      }
    }
  }

  float rstd = 1.f;
  if (NORM) {
    // stage gamma (bf16 -> float32) once per block while the row loads are in flight
    for (int k = 2 * threadIdx.x; k < p.K; k += 2 * blockDim.x) {
      const uint32_t g2 = *reinterpret_cast<const uint32_t *>(p.gamma + k);
      gs[gamma_smem_index(k)] = bf16lo(g2);
      gs[gamma_smem_index(k + 1)] = bf16hi(g2);
    }
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < DP; ++i) {
      const int dp = i * stride + wt * 32 + lane;
      if (live_row && dp < ndp_row) {
        // float64: bf16 squares are exact and the sum keeps ~2^-53 relative accuracy, so
        // fp32(sum/K) does not depend on the summation order in practice
#pragma unroll
        for (int w = 0; w < 8; ++w) ss = add_squares(xr[i][w], ss);
      }
    }
    __syncthreads();  // gamma staged
    ss = team_sum(ss, W, team, wt, sm_d);
    const float ms = __double2float_rn(__ddiv_rn(ss, (double)p.K));
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, p.eps)));
  }
  // staged weights of this lane's piece i: chunk c at g_lane + i*128W + 32c (see gamma_smem_index)
  const float4 *g_lane = gamma_smem4 + wt * 128 + lane;

  float am = 0.f;
#pragma unroll
  for (int i = 0; i < DP; ++i) {
    const int dp = i * stride + wt * 32 + lane;
    if (live_row && dp < ndp_row) {
      float v[16];
      unpack16(xr[i], v);
      if (NORM) normalize16<true>(v, g_lane + i * 128 * W, rstd);
      am = amax16(v, am);
    }
  }
  am = team_max(am, W, team, wt, sm_f);
  float s_x, g_x;
  row_scales(FMT, am, s_x, g_x);

  constexpr int kChunk = act_tile(FMT, UNIT, !DENSE).bytes;
  const Spot o = lane_spot<FMT, UNIT, DENSE>(row, lane);
  // chunk of piece i: row block, then K step i*2W + 2wt + lane/16
  uint8_t *chunk0 = p.tiles + ((size_t)(row >> 7) * p.KS + 2 * wt + (lane >> 4)) * kChunk;
  const size_t chunk_step = (size_t)2 * W * kChunk;
  const bool pad_row = !live_row && row < p.T_pad;
  if (UNROLLED && live_row && ndp_row == DP * stride) {
    // Every piece of the row is live (K a multiple of 512 W): no per-piece control flow, so
    // the compiler may interleave pieces (8 % faster at 16384 rows). The loop's code is
    // larger, so a launch of one wave, whose blocks all start with a cold instruction cache,
    // keeps the loop below (the same speed in the benchmark's step at 2048 rows).
#pragma unroll
    for (int i = 0; i < DP; ++i) {
      float v[16];
      unpack16(xr[i], v);
      if (NORM) normalize16<false>(v, g_lane + i * 128 * W, rstd);
      process16<FMT, UNIT, DENSE>(chunk0 + i * chunk_step, o, v, true, s_x, g_x);
    }
    if (wt == 0 && lane == 0) p.row_scale[row] = s_x;
    return;
  }
#pragma unroll
  for (int i = 0; i < DP; ++i) {
    const int base = i * stride + wt * 32;  // warp-uniform
    if (base >= ndp_row) break;
    const int dp = base + lane;
    const bool live = live_row && dp < ndp_row;
    uint8_t *chunk = chunk0 + i * chunk_step;
    if (live_row) {
      float v[16];
      if (live) {
        unpack16(xr[i], v);
        if (NORM) normalize16<false>(v, g_lane + i * 128 * W, rstd);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
      }
      process16<FMT, UNIT, DENSE>(chunk, o, v, live, s_x, g_x);
    } else if (pad_row && dp < ndp_row) {
      store16<FMT, UNIT, DENSE>(chunk, o, 0u, 0u, 0u, 0u, 0u, 0u);
    }
  }
  if (live_row && wt == 0 && lane == 0) p.row_scale[row] = s_x;
}

// ---------------------------------------------------------------- one scale per tensor
// NVFP4 with one second-level scale for the whole tensor needs the tensor amax before any code
// is formed. One cooperative launch (every block resident at once): a block's teams take the
// row groups blockIdx.x, blockIdx.x + G, ... Phase 1 loads each of its rows, forms rstd and the
// normalized row amax; rstd waits in row_scale[row] for phase 2, except the last row's, which
// stays in registers with the row itself. Each block writes its maximum to the workspace, a
// grid barrier follows (an arrival counter the host cleared, a bounded wait), and every block
// takes the maximum of all block maxima. Phase 2 quantizes the last row from registers and
// re-reads the others, the most recently read first (L2 may still hold them); when every row
// fits on chip (one row group per team) x is read once. Finally row_scale gets the tensor's
// scale. Workspace words: [0] arrival counter, [1] barrier generation, [4 + b] block b's
// maximum (float). The last block to arrive zeroes the counter and advances the generation,
// so a call leaves the workspace ready for the next one (it starts from zeros).
__device__ uint32_t g_prep_status = 0;  // bit 0: the grid barrier's wait gave up

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t *a) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

template <int UNIT, bool NORM, int DP>
__global__ void __launch_bounds__(256, 2) prep_tensor_kernel(PrepParams p, uint32_t *ws, int groups,
                                                          unsigned long long limit_ns) {
  extern __shared__ float4 gamma_smem4[];
  __shared__ double sm_d[64];
  __shared__ float sm_f[64];
  __shared__ float tensor_amax;
  __shared__ int barrier_ok;
  float *gs = reinterpret_cast<float *>(gamma_smem4);
  const int W = p.TS;
  const int teams = (blockDim.x >> 5) / W;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int team = warp / W, wt = warp - team * W;
  const int ndp_row = p.K >> 4;
  const int stride = 32 * W;
  const int G = gridDim.x;
  const int J = (groups - (int)blockIdx.x + G - 1) / G;  // >= 1: G <= groups
  const float4 *g_lane = gamma_smem4 + wt * 128 + lane;

  if (NORM) {
    for (int k = 2 * threadIdx.x; k < p.K; k += 2 * blockDim.x) {
      const uint32_t g2 = *reinterpret_cast<const uint32_t *>(p.gamma + k);
      gs[gamma_smem_index(k)] = bf16lo(g2);
      gs[gamma_smem_index(k + 1)] = bf16hi(g2);
    }
    __syncthreads();
  }
  uint32_t xr[DP][8];
  auto load_row = [&](int row) {
#pragma unroll
    for (int i = 0; i < DP; ++i) {
      const int dp = i * stride + wt * 32 + lane;
      if (row < p.T && dp < ndp_row) ld256(p.x + (size_t)row * p.x_stride + (size_t)dp * 16, xr[i]);
    }
  };

  // ---- phase 1: rstd and the normalized amax of every row of this block
  float rstd = 1.f, am = 0.f;
  for (int j = 0; j < J; ++j) {
    const int row = ((int)blockIdx.x + j * G) * teams + team;
    const bool live_row = row < p.T;
    load_row(row);
    if (NORM) {
      double ss = 0.0;
#pragma unroll
      for (int i = 0; i < DP; ++i) {
        const int dp = i * stride + wt * 32 + lane;
        if (live_row && dp < ndp_row) {
#pragma unroll
          for (int w = 0; w < 8; ++w) ss = add_squares(xr[i][w], ss);
        }
      }
      ss = team_sum(ss, W, team, wt, sm_d);
      const float ms = __double2float_rn(__ddiv_rn(ss, (double)p.K));
      rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, p.eps)));
      if (j < J - 1 && live_row && wt == 0 && lane == 0) p.row_scale[row] = rstd;
    }
#pragma unroll
    for (int i = 0; i < DP; ++i) {
      const int dp = i * stride + wt * 32 + lane;
      if (live_row && dp < ndp_row) {
        float v[16];
        unpack16(xr[i], v);
        if (NORM) normalize16<true>(v, g_lane + i * 128 * W, rstd);
        am = amax16(v, am);
      }
    }
  }

  // ---- block maximum, grid barrier, tensor maximum
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(kFull, am, o));
  if (lane == 0) sm_f[warp] = am;
  __syncthreads();
  float *bmax = reinterpret_cast<float *>(ws + 4);
  if (threadIdx.x == 0) {
    float m = sm_f[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, sm_f[w]);
    // generation read before arriving: it advances only after every block has arrived
    const uint32_t gen = ld_relaxed_gpu(ws + 1);
    bmax[blockIdx.x] = m;
    __threadfence();
    bool ok = true;
    if (atomicAdd(ws, 1u) == (uint32_t)G - 1u) {
      // the last block: reset the counter for the next call, then release the others
      atomicExch(ws, 0u);
      __threadfence();
      atomicAdd(ws + 1, 1u);
    } else if (ld_acquire_gpu(ws + 1) == gen) {
      ok = false;
      const uint64_t t0 = global_ns();
      for (uint32_t i = 1;; ++i) {
        if (ld_acquire_gpu(ws + 1) != gen) { ok = true; break; }
        if ((i & 31u) == 0 && global_ns() - t0 > limit_ns) break;
      }
    }
    if (!ok) atomicOr(&g_prep_status, 1u);
    barrier_ok = ok ? 1 : 0;
  }
  __syncthreads();
  if (!barrier_ok) return;  // outputs undefined; the status word reports it
  // the maximum of the G block maxima, read by the whole block at once
  float t = 0.f;
  for (int b = threadIdx.x; b < G; b += blockDim.x) t = fmaxf(t, __ldcg(bmax + b));
  for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(kFull, t, o));
  __syncthreads();  // sm_f's block maxima have been read
  if (lane == 0) sm_f[warp] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = sm_f[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, sm_f[w]);
    tensor_amax = m;
  }
  __syncthreads();
  float s_x, g_x;
  row_scales(kFmtNV, tensor_amax, s_x, g_x);

  // ---- phase 2: quantize, the row still in registers first
  constexpr int kChunk = act_tile(kFmtNV, UNIT, true).bytes;
  for (int j = J - 1; j >= 0; --j) {
    const int row = ((int)blockIdx.x + j * G) * teams + team;
    const bool live_row = row < p.T;
    if (j < J - 1) {
      load_row(row);
      if (NORM) rstd = live_row ? __ldcg(p.row_scale + row) : 1.f;
    }
    const Spot o = lane_spot<kFmtNV, UNIT, false>(row, lane);
    uint8_t *chunk0 = p.tiles + ((size_t)(row >> 7) * p.KS + 2 * wt + (lane >> 4)) * kChunk;
    const size_t chunk_step = (size_t)2 * W * kChunk;
    const bool pad_row = !live_row && row < p.T_pad;
    // every piece live and several row groups per block (the instruction cache warm after the
    // first): branch-free, as prep_kernel's multi-wave launches
    if (J > 1 && live_row && ndp_row == DP * stride) {
#pragma unroll
      for (int i = 0; i < DP; ++i) {
        float v[16];
        unpack16(xr[i], v);
        if (NORM) normalize16<false>(v, g_lane + i * 128 * W, rstd);
        process16<kFmtNV, UNIT, false>(chunk0 + i * chunk_step, o, v, true, s_x, g_x);
      }
      continue;
    }
#pragma unroll
    for (int i = 0; i < DP; ++i) {
      const int base = i * stride + wt * 32;  // warp-uniform
      if (base >= ndp_row) break;
      const int dp = base + lane;
      const bool live = live_row && dp < ndp_row;
      uint8_t *chunk = chunk0 + i * chunk_step;
      if (live_row) {
        float v[16];
        if (live) {
          unpack16(xr[i], v);
          if (NORM) normalize16<false>(v, g_lane + i * 128 * W, rstd);
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = 0.f;
        }
        process16<kFmtNV, UNIT, false>(chunk, o, v, live, s_x, g_x);
      } else if (pad_row && dp < ndp_row) {
        store16<kFmtNV, UNIT, false>(chunk, o, 0u, 0u, 0u, 0u, 0u, 0u);
      }
    }
  }
  __syncthreads();  // every warp of a team has read its rows' rstd before the entries change
  for (int j = 0; j < J; ++j) {
    const int row = ((int)blockIdx.x + j * G) * teams + team;
    if (row < p.T && wt == 0 && lane == 0) p.row_scale[row] = s_x;
  }
}

int prep_sm_count() {
  static std::once_flag once[64];
  static int sms[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::call_once(once[dev], [dev] {
    if (cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms[dev] = 148;
  });
  return sms[dev];
}

template <int FMT, int UNIT, bool NORM, bool DENSE, int MODE, int DP, bool UNROLLED>
cudaError_t launch_u(const PrepParams &p, cudaStream_t st) {
  const int W = p.TS;
  const int teams = W >= 8 ? 1 : 8 / W;
  const int block = teams * W * 32;
  const int grid = (p.T_pad + teams - 1) / teams;
  const PrepParams &q = p;
  // the staging layout reserves 512 floats per 32 double pieces: round K up to 512
  const size_t smem = NORM ? (size_t)((p.K + 511) / 512 * 512) * sizeof(float) : 0;
  if (smem > 48 * 1024) {
    // opt in once per device to the largest staging size (K = 32768)
    static std::once_flag once[64];
    static cudaError_t err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
      err[dev] = cudaFuncSetAttribute(prep_kernel<FMT, UNIT, NORM, DENSE, MODE, DP, UNROLLED>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      32768 * (int)sizeof(float));
    });
    if (err[dev] != cudaSuccess) return err[dev];
  }
  prep_kernel<FMT, UNIT, NORM, DENSE, MODE, DP, UNROLLED><<<grid, block, smem, st>>>(q);
  return cudaGetLastError();
}

// The branch-free instantiation for the executed mask (pairs, sparse) when every piece of a
// row is live and the launch has several waves (grid >= 4 x the SM count: the instruction
// cache is warm after the first blocks; a one-wave launch starts every block cold and the
// larger loop then costs as much as it saves).
template <int FMT, int UNIT, bool NORM, bool DENSE, int MODE, int DP>
cudaError_t launch_k(const PrepParams &p, cudaStream_t st) {
  const int W = p.TS;
  const int teams = W >= 8 ? 1 : 8 / W;
  const int grid = (p.T_pad + teams - 1) / teams;
  const bool full = (p.K >> 4) == DP * 32 * W;
  if constexpr (UNIT == 2 && !DENSE) {
    if (full && grid >= 4 * prep_sm_count()) return launch_u<FMT, UNIT, NORM, DENSE, MODE, DP, true>(p, st);
  }
  return launch_u<FMT, UNIT, NORM, DENSE, MODE, DP, false>(p, st);
}

// A single-warp row of at most 2048 elements needs 4 pieces per lane: the smaller register
// array leaves room for more resident warps.
template <int FMT, int UNIT, bool NORM, bool DENSE, int MODE = kRow>
cudaError_t launch_t(const PrepParams &p, cudaStream_t st) {
  if (p.TS == 1 && p.K / 16 <= 32 * 4) return launch_k<FMT, UNIT, NORM, DENSE, MODE, 4>(p, st);
  return launch_k<FMT, UNIT, NORM, DENSE, MODE, kMaxDP>(p, st);
}

template <int FMT, int UNIT, bool DENSE>
cudaError_t launch_n(const PrepParams &p, bool norm, cudaStream_t st) {
  return norm ? launch_t<FMT, UNIT, true, DENSE>(p, st) : launch_t<FMT, UNIT, false, DENSE>(p, st);
}

}  // namespace

// Warps per row: each lane holds at most kMaxDP double pieces (16 elements each).
int prep_team_warps(int k) { return (k / 16 + 32 * kMaxDP - 1) / (32 * kMaxDP); }

cudaError_t launch_prep(PrepParams p, int fmt, int unit, bool norm, bool dense, bool swiglu, cudaStream_t st) {
  p.KS = p.K / 256;
  p.TS = prep_team_warps(p.K);
  if (p.TS > 8) return cudaErrorInvalidValue;  // k > 32768: outside the supported range
  if (dense) {
    return fmt == kFmtNV ? launch_n<kFmtNV, 2, true>(p, norm, st) : launch_n<kFmtMX, 2, true>(p, norm, st);
  }
  if (swiglu) {  // the gated activation of a down projection (no normalization)
    if (fmt == kFmtNV)
      return unit == 2 ? launch_t<kFmtNV, 2, false, false, kSwiglu>(p, st)
                       : launch_t<kFmtNV, 1, false, false, kSwiglu>(p, st);
    return unit == 2 ? launch_t<kFmtMX, 2, false, false, kSwiglu>(p, st) : launch_t<kFmtMX, 1, false, false, kSwiglu>(p, st);
  }
  if (unit == kPat48)  // four of eight elements (sharq_prepare only)
    return fmt == kFmtNV ? launch_n<kFmtNV, kPat48, false>(p, norm, st) : launch_n<kFmtMX, kPat48, false>(p, norm, st);
  if (fmt == kFmtNV)
    return unit == 2 ? launch_n<kFmtNV, 2, false>(p, norm, st) : launch_n<kFmtNV, 1, false>(p, norm, st);
  return unit == 2 ? launch_n<kFmtMX, 2, false>(p, norm, st) : launch_n<kFmtMX, 1, false>(p, norm, st);
}

// Row groups of the per-tensor launch: teams of TS warps, 8 warps per block.
int prep_tensor_groups(int tokens, int k) {
  const int ts = prep_team_warps(k);
  const int teams = ts >= 8 ? 1 : 8 / ts;
  return (round_up(tokens, 256) + teams - 1) / teams;
}

namespace {
template <int UNIT, bool NORM, int DP>
cudaError_t launch_tensor_t(PrepParams p, uint32_t *ws, unsigned long long limit_ns, cudaStream_t st) {
  auto kern = prep_tensor_kernel<UNIT, NORM, DP>;
  static std::once_flag once[64];
  static cudaError_t err[64];
  static int sms[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev, kern] {
    err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 * (int)sizeof(float));
    if (err[dev] == cudaSuccess) err[dev] = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  });
  if (err[dev] != cudaSuccess) return err[dev];
  const int W = p.TS;
  const int teams = W >= 8 ? 1 : 8 / W;
  const int block = teams * W * 32;
  const size_t smem = NORM ? (size_t)((p.K + 511) / 512 * 512) * sizeof(float) : 0;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, block, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  int groups = (p.T_pad + teams - 1) / teams;
  const int grid = groups < per_sm * sms[dev] ? groups : per_sm * sms[dev];
  void *args[] = {&p, &ws, &groups, &limit_ns};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(grid), dim3(block), args, smem, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int UNIT, bool NORM>
cudaError_t launch_tensor_dp(const PrepParams &p, uint32_t *ws, unsigned long long limit_ns, cudaStream_t st) {
  if (p.TS == 1 && p.K / 16 <= 32 * 4) return launch_tensor_t<UNIT, NORM, 4>(p, ws, limit_ns, st);
  return launch_tensor_t<UNIT, NORM, kMaxDP>(p, ws, limit_ns, st);
}
}  // namespace

// NVFP4 with one second-level scale for the whole tensor: one cooperative launch.
cudaError_t launch_prep_tensor_scale(PrepParams p, int unit, bool norm, void *workspace, unsigned long long limit_ns,
                                     cudaStream_t st) {
  p.KS = p.K / 256;
  p.TS = prep_team_warps(p.K);
  if (p.TS > 8) return cudaErrorInvalidValue;
  uint32_t *ws = static_cast<uint32_t *>(workspace);
  if (unit == 2)
    return norm ? launch_tensor_dp<2, true>(p, ws, limit_ns, st) : launch_tensor_dp<2, false>(p, ws, limit_ns, st);
  return norm ? launch_tensor_dp<1, true>(p, ws, limit_ns, st) : launch_tensor_dp<1, false>(p, ws, limit_ns, st);
}

// ---------------------------------------------------------------- per-tensor scale, no caller memory
// The per-tensor preparation for callers that cannot hand the library a workspace: code that
// runs where it may not allocate device memory at all (inside a memory budget owned by a host
// framework or an inference server that pre-assigns every byte, or a plugin ABI that passes
// only its tensors), or where cudaMalloc's implicit device synchronization would stall a
// latency-critical path. The grid barrier's words and block maxima live in this file-scope
// array instead, loaded with the library and held by every GPU that loads it until exit.
// One array per device, shared by every call on that device: calls whose launches may overlap
// on the GPU (different streams, no ordering between them) race on it.
namespace {
constexpr size_t kStaticScratchBytes = 8192;  // barrier words + up to 2044 block maxima
static __device__ __align__(256) uint32_t g_static_scratch[kStaticScratchBytes / 4];
}  // namespace

cudaError_t launch_prep_tensor_scale_static(PrepParams p, int unit, bool norm, unsigned long long limit_ns,
                                            cudaStream_t st, size_t *needed, size_t *capacity) {
  // Once per device, with that device current: the array's device address. In host code the
  // array's name is only a host-side stand-in, never a pointer a kernel may be given.
  static std::once_flag once[64];
  static cudaError_t err[64];
  static void *addr[64];
  static int sms[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev] {
    err[dev] = cudaGetSymbolAddress(&addr[dev], g_static_scratch);
    if (err[dev] == cudaSuccess) err[dev] = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  });
  if (err[dev] != cudaSuccess) return err[dev];
  // the launch uses at most one block slot per row group and at most 8 resident blocks of 256
  // threads per SM
  const int groups = prep_tensor_groups(p.T, p.K);
  const int max_grid = 8 * sms[dev];
  *needed = 16 + 4 * (size_t)(groups < max_grid ? groups : max_grid);
  *capacity = kStaticScratchBytes;
  if (*needed > kStaticScratchBytes) return cudaErrorInvalidValue;
  // the array keeps the previous call's contents: the counter and generation start at zero
  if ((e = cudaMemsetAsync(addr[dev], 0, 2 * sizeof(uint32_t), st)) != cudaSuccess) return e;
  return launch_prep_tensor_scale(p, unit, norm, addr[dev], limit_ns, st);
}

cudaError_t read_and_clear_prep_status(uint32_t *status) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(status, g_prep_status, sizeof *status);
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_prep_status, &zero, sizeof zero);
}

}  // namespace sharq
