"""Plain CPU oracle of SharQ's online sparse-dense FP4 linear layer.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA library and never calls it.

What the method computes ("SharQ: Bridging Activation Sparsity and FP4
Quantization for LLM Inference", Abstract): for each activation tensor,

1. optional layer normalization (RMSNorm; the README's "--disable_rmsnorm_fusion"
   flag, section "Evaluation"),
2. an N:M mask chosen from the activation itself, which pulls the outliers
   into a sparse backbone,
3. FP4 quantization of that backbone,
4. a dense residual defined against the *quantized* backbone (not the
   unquantized sparse values), quantized densely to FP4,
5. a sparse FP4 GEMM on the backbone plus a dense FP4 GEMM on the residual,
   both against one FP4 weight payload with path-specific scale views,
   summed into one output.

The pages define none of these numerically. The readings taken here (each
one is listed with its reason in the repository's design notes):

* RMSNorm: ss = sum(x^2) in float64; rstd = 1/sqrt(fp32(ss/K) + eps) in
  float32 with correctly rounded sqrt and divide; xh = fp32(fp32(x*rstd)*gamma).
  ``gamma is None`` means no normalization: xh = x.
* Mask: the K axis is cut into units of ``unit`` consecutive elements (1 = an
  element, 2 = an aligned pair), and into aligned groups of M units. In each
  group the N units with the largest key are kept; a unit's key is the largest
  |xh| inside it; equal keys go to the lower unit index.
* Second-level scale (NVFP4): one float32 scale per token row,
  s_x = fp32(amax_row/2688) with g_x = fp32(448/amax_row), shared by the
  backbone and the residual of that row (so both GEMMs add into one
  accumulator). A zero row has s_x = 1 and g_x = 0. MXFP4 has none (s_x = 1).
* NVFP4 block (E4M3 scale): sb = E4M3(fp32(amax_b*g_x)); d = fp32(dec(sb)*s_x);
  d == 0 gives all-zero codes; otherwise code = E2M1(fp32(v*fp32(1/d))).
* MXFP4 block (E8M0 scale): amax_b == 0 gives e = 0 and zero codes; otherwise
  e = clamp(floor(log2 amax_b) - 2 + 127, 0, 254) and code = E2M1(v*2^(127-e)).
* Block membership: the residual uses 16 (NVFP4) / 32 (MXFP4) consecutive K
  positions; the backbone uses 16 / 32 consecutive *stored* values; the weight
  is quantized in blocks matching the sparse path's K span (2x the dense
  block at 50% density), and its dense-path view repeats each scale over the
  dense blocks it covers, so both views decode to the same weight.
* Backbone value used for the residual: fp32(fp32(dec(code)*dec(sb))*s_x);
  residual r = fp32(xh - that) at kept positions, r = xh elsewhere.

Everything that decides a code is float32 arithmetic written out with numpy
float32 operands (IEEE correctly rounded), in the order stated above; the GEMM
is float64 on exactly dequantized operands.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, e8m0_decode

NVFP4 = "nvfp4"
MXFP4 = "mxfp4"

F32 = np.float32
_E4M3_TIMES_E2M1_MAX = F32(448.0 * 6.0)  # 2688: amax maps to the top of E4M3 x E2M1
_E4M3_MAX = F32(448.0)


def block_size(fmt: str) -> int:
    """Elements per block scale: 16 for NVFP4 (E4M3 scale), 32 for MXFP4 (E8M0 scale)."""
    if fmt == NVFP4:
        return 16
    if fmt == MXFP4:
        return 32
    raise ValueError(f"unknown format {fmt!r}")


# --------------------------------------------------------------------------------------
# step a1: RMSNorm
# --------------------------------------------------------------------------------------
def rmsnorm(x: np.ndarray, gamma: np.ndarray | None, eps: float) -> np.ndarray:
    """Layer normalization fused into the preparation operator.

    The abstract lists layer normalization among the steps folded into the fused
    preparation kernel; the README mirror (section "Benchmarks") calls it RMSNorm fusion.
    ``x`` holds the bf16 activations as float32 [T, K]; ``gamma`` the bf16
    weight as float32 [K] or None (no normalization).
    """
    x = np.asarray(x, dtype=F32)
    if gamma is None:
        return x.copy()
    gamma = np.asarray(gamma, dtype=F32)
    T, K = x.shape
    ss = np.sum(x.astype(np.float64) ** 2, axis=1)                 # float64 sum of squares
    ms = (ss / np.float64(K)).astype(F32)                          # fp32(ss / K)
    v = ms + F32(eps)                                              # fp32 add
    rstd = F32(1.0) / np.sqrt(v)                                   # fp32 sqrt, fp32 divide
    return ((x * rstd[:, None]).astype(F32) * gamma[None, :]).astype(F32)


# --------------------------------------------------------------------------------------
# step a2: input-adaptive N:M mask
# --------------------------------------------------------------------------------------
def nm_select(xh: np.ndarray, n: int, m: int, unit: int) -> np.ndarray:
    """Indices of the kept units: int array [T, G, n], ascending within each group.

    Per the abstract, a mask chosen from the input itself (N of every M) pulls
    out a sparse backbone that carries the outliers. A group is M consecutive units of
    ``unit`` elements along K; the N units of largest key survive, key = the
    largest |xh| inside the unit, ties to the lower unit index.
    """
    T, K = xh.shape
    span = m * unit
    if K % span:
        raise ValueError("K must be a multiple of M*unit")
    key = np.abs(xh.reshape(T, K // unit, unit)).max(axis=2)       # [T, K/unit]
    key = key.reshape(T, K // span, m)
    order = np.argsort(-key, axis=2, kind="stable")                # descending, stable on ties
    return np.sort(order[:, :, :n], axis=2)


def keep_mask(idx: np.ndarray, k: int, m: int, unit: int) -> np.ndarray:
    """Boolean [T, K] mask of the kept elements from unit indices [T, G, n]."""
    T, G, n = idx.shape
    mask_units = np.zeros((T, G, m), dtype=bool)
    np.put_along_axis(mask_units, idx, True, axis=2)
    return np.repeat(mask_units.reshape(T, G * m), unit, axis=1).reshape(T, k)


def gather_kept(xh: np.ndarray, idx: np.ndarray, m: int, unit: int) -> np.ndarray:
    """Kept values in storage order [T, K*n/m]: groups in K order, kept units ascending."""
    T, K = xh.shape
    G, n = idx.shape[1], idx.shape[2]
    units = xh.reshape(T, G, m, unit)
    kept = np.take_along_axis(units, idx[:, :, :, None], axis=2)   # [T, G, n, unit]
    return kept.reshape(T, G * n * unit)


def scatter_kept(stored: np.ndarray, idx: np.ndarray, k: int, m: int, unit: int) -> np.ndarray:
    """Inverse of gather_kept: dense [T, K] with zeros at dropped positions."""
    T = stored.shape[0]
    G, n = idx.shape[1], idx.shape[2]
    out = np.zeros((T, G, m, unit), dtype=stored.dtype)
    np.put_along_axis(out, idx[:, :, :, None], stored.reshape(T, G, n, unit), axis=2)
    return out.reshape(T, k)


# --------------------------------------------------------------------------------------
# steps a3 / a5: block quantization
# --------------------------------------------------------------------------------------
def row_scale(xh: np.ndarray, fmt: str, per_tensor: bool = False):
    """Second-level scale s_x and its encode factor g_x = 1/(6*s_x) (NVFP4), one per row.

    per_tensor: one scale for the whole tensor (amax over every row), repeated per row -- the
    stricter reading of NVFP4's "fp32 tensor scale". MXFP4 has no second-level scale:
    s_x = 1, g_x unused (returned as 1).
    """
    T = xh.shape[0]
    if fmt == MXFP4:
        return np.ones(T, dtype=F32), np.ones(T, dtype=F32)
    amax = np.abs(xh).max(axis=1).astype(F32)
    if per_tensor:
        amax = np.full(T, amax.max() if T else F32(0.0), dtype=F32)
    zero = amax == 0
    safe = np.where(zero, F32(1.0), amax).astype(F32)
    s_x = np.where(zero, F32(1.0), safe / _E4M3_TIMES_E2M1_MAX).astype(F32)
    g_x = np.where(zero, F32(0.0), _E4M3_MAX / safe).astype(F32)
    return s_x, g_x


def quantize_blocks_nvfp4(vals: np.ndarray, s_x: np.ndarray, g_x: np.ndarray):
    """NVFP4 block quantization of ``vals`` [T, nb, 16] with row scales [T].

    Returns (codes uint8 [T, nb, 16], sb uint8 E4M3 [T, nb]).
    """
    vals = np.asarray(vals, dtype=F32)
    amax = np.abs(vals).max(axis=2).astype(F32)                    # [T, nb]
    q = (amax * g_x[:, None]).astype(F32)
    sb = e4m3_encode(q)
    d = (e4m3_decode(sb).astype(F32) * s_x[:, None]).astype(F32)
    zero = d == 0
    inv = (F32(1.0) / np.where(zero, F32(1.0), d)).astype(F32)
    v = (vals * inv[:, :, None]).astype(F32)
    codes = e2m1_encode(v)
    codes = np.where(zero[:, :, None], np.uint8(0), codes).astype(np.uint8)
    return codes, sb


def dequant_blocks_nvfp4(codes: np.ndarray, sb: np.ndarray, s_x: np.ndarray) -> np.ndarray:
    """fp32(fp32(dec(code)*dec(sb))*s_x) for codes [T, nb, B], sb [T, nb] (float32 result)."""
    prod = (e2m1_decode(codes).astype(F32) * e4m3_decode(sb).astype(F32)[:, :, None]).astype(F32)
    return (prod * s_x[:, None, None]).astype(F32)


def mx_exponent(amax: np.ndarray) -> np.ndarray:
    """E8M0 scale code per block: floor(log2 amax) - 2 + 127 clamped to [0, 254]; 0 for amax 0."""
    amax = np.asarray(amax, dtype=np.float64)
    mant, ex = np.frexp(amax)                                      # amax = mant * 2^ex, mant in [0.5, 1)
    e = np.clip(ex - 1 - 2 + 127, 0, 254)
    return np.where(amax == 0, 0, e).astype(np.uint8)


def quantize_blocks_mxfp4(vals: np.ndarray):
    """MXFP4 block quantization of ``vals`` [T, nb, 32]: (codes [T, nb, 32], e uint8 [T, nb])."""
    vals = np.asarray(vals, dtype=F32)
    amax = np.abs(vals).max(axis=2)
    e = mx_exponent(amax)
    scaled = np.ldexp(vals.astype(np.float64), 127 - e.astype(np.int64)[:, :, None]).astype(F32)
    codes = e2m1_encode(scaled)
    codes = np.where((amax == 0)[:, :, None], np.uint8(0), codes).astype(np.uint8)
    return codes, e


def dequant_blocks_mxfp4(codes: np.ndarray, e: np.ndarray) -> np.ndarray:
    """dec(code) * 2^(e-127) (exact), as float32 [T, nb, B]."""
    return (e2m1_decode(codes) * e8m0_decode(e)[:, :, None]).astype(F32)


def _quantize(vals2d: np.ndarray, fmt: str, s_x, g_x):
    """Quantize a [T, L] array in consecutive blocks; returns (codes [T,L], scales [T,L/B], deq [T,L])."""
    T, L = vals2d.shape
    B = block_size(fmt)
    if L % B:
        raise ValueError("length must be a multiple of the block size")
    blocks = vals2d.reshape(T, L // B, B)
    if fmt == NVFP4:
        codes, sc = quantize_blocks_nvfp4(blocks, s_x, g_x)
        deq = dequant_blocks_nvfp4(codes, sc, s_x)
    else:
        codes, sc = quantize_blocks_mxfp4(blocks)
        deq = dequant_blocks_mxfp4(codes, sc)
    return codes.reshape(T, L), sc, deq.reshape(T, L)


# --------------------------------------------------------------------------------------
# the preparation operator (steps a1-a5)
# --------------------------------------------------------------------------------------
def prepare(x, gamma, eps: float, n: int, m: int, unit: int, fmt: str, per_tensor: bool = False) -> dict:
    """SharQ's fused preparation operator, written out step by step.

    Order of the abstract: mask -> backbone -> FP4 backbone -> residual taken
    against the backbone after quantization (not against its exact values) ->
    dense FP4 of that residual.

    Returns canonical (unpacked, unswizzled) arrays:
      xh [T,K] f32, idx [T,G,n], sp_codes [T,K*n/m] u8, sp_scales [T,nb_sp] u8,
      res_codes [T,K] u8, res_scales [T,nb_res] u8, row_scale [T] f32,
      sp_deq [T,K*n/m] f32, resid [T,K] f32.

    per_tensor: one second-level scale for the whole activation tensor instead of one per
    row (NVFP4; the variant of the reading "fp32 tensor scale"), shared by both paths.
    """
    x = np.asarray(x, dtype=F32)
    T, K = x.shape
    xh = rmsnorm(x, gamma, eps)
    s_x, g_x = row_scale(xh, fmt, per_tensor)
    idx = nm_select(xh, n, m, unit)
    stored = gather_kept(xh, idx, m, unit)
    sp_codes, sp_scales, sp_deq = _quantize(stored, fmt, s_x, g_x)
    deq_dense = scatter_kept(sp_deq, idx, K, m, unit)              # +0 at dropped positions
    resid = (xh - deq_dense).astype(F32)
    res_codes, res_scales, _ = _quantize(resid, fmt, s_x, g_x)
    return dict(xh=xh, idx=idx, sp_codes=sp_codes, sp_scales=sp_scales,
                res_codes=res_codes, res_scales=res_scales, row_scale=s_x,
                sp_deq=sp_deq, resid=resid, n=n, m=m, unit=unit, fmt=fmt)


# --------------------------------------------------------------------------------------
# SwiGLU fused into the preparation operator (down-projection input)
# --------------------------------------------------------------------------------------
# The abstract folds the steps in front of the quantizer into the one preparation kernel;
# for a down projection that step is the gated activation x = SiLU(g) * u of
# the gate/up projection's output [g | u]. Reading (the pages give no formula): the
# activation the unfused pipeline hands to the down projection is bf16, so
#   x = bf16_RNE(fp32(silu(g) * u)),  silu(g) = fp32(g * sigma(g)),
#   sigma(g) = 1 / (1 + e) for g >= 0 and e / (1 + e) for g < 0, with e = exp(-|g|),
# each step a float32 round-to-nearest operation (division correctly rounded). exp is
# evaluated by range reduction with Cody and Waite's two-part ln 2 (W. J. Cody and W. Waite,
# "Software Manual for the Elementary Functions", 1980) and a Taylor polynomial:
#   a = |g|; t = fp32(a * log2(e)); t >= 126 gives e = 0 (below the normal range);
#   n = rint(t); r = fp32(fp32(a - fp32(n * LN2_HI)) - fp32(n * LN2_LO)), |r| <~ ln2 / 2
#   (n * LN2_HI is exact: LN2_HI has 15 significant bits, n at most 7);
#   e^-r by Horner on the Taylor coefficients 1/k!, k = 7 .. 0, at -r, one rounding per
#   multiply and per add (no fused multiply-add); e = fp32(p * 2^-n).
# Written as separate correctly rounded float32 operations, the CUDA kernel reproduces
# every bit of it.
_LOG2E = F32(1.4426950408889634)
_LN2_HI = F32(0.693145751953125)            # 0x3F317200
_LN2_LO = F32(0.6931471805599453 - 0.693145751953125)
_EXP_TAYLOR = [F32(1.0 / np.prod(np.arange(1, k + 1, dtype=np.float64))) for k in range(8)]


def exp_neg_abs(g) -> np.ndarray:
    """exp(-|g|) in float32: Cody-Waite reduction to r in [-ln2/2, ln2/2] plus degree-7 Taylor."""
    a = np.abs(np.asarray(g, dtype=F32))
    with np.errstate(over="ignore", invalid="ignore"):  # |g| beyond the range: masked at the end
        t = (a * _LOG2E).astype(F32)
        n = np.rint(np.minimum(t, F32(126.0))).astype(F32)       # 0 .. 126, ties to even
        r = ((a - (n * _LN2_HI).astype(F32)).astype(F32) - (n * _LN2_LO).astype(F32)).astype(F32)
        x = (-r).astype(F32)
        p = np.full_like(x, _EXP_TAYLOR[7])
        for k in range(6, -1, -1):
            p = ((p * x).astype(F32) + _EXP_TAYLOR[k]).astype(F32)
        scale = np.ldexp(F32(1.0), -n.astype(np.int32)).astype(F32)  # 2^-n, exact
        e = (p * scale).astype(F32)
    return np.where(t >= F32(126.0), F32(0.0), e).astype(F32)


def silu(g) -> np.ndarray:
    """SiLU(g) = g * sigmoid(g) in float32 (reading above)."""
    g = np.asarray(g, dtype=F32)
    e = exp_neg_abs(g)
    den = (F32(1.0) + e).astype(F32)
    num = np.where(g >= F32(0.0), F32(1.0), e).astype(F32)
    sigma = (num / den).astype(F32)
    return (g * sigma).astype(F32)


def round_bf16(v) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32 values."""
    b = np.ascontiguousarray(v, dtype=F32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(F32)


def swiglu(gate_up) -> np.ndarray:
    """x [T, K] = bf16_RNE(fp32(silu(g) * u)) from gate_up [T, 2K] = [g | u]."""
    gu = np.asarray(gate_up, dtype=F32)
    K = gu.shape[1] // 2
    prod = (silu(gu[:, :K]) * gu[:, K:]).astype(F32)
    return round_bf16(prod)


def prepare_swiglu(gate_up, n: int, m: int, unit: int, fmt: str) -> dict:
    """The preparation operator on the gated activation of a down projection (no RMSNorm)."""
    return prepare(swiglu(gate_up), None, 0.0, n, m, unit, fmt)


def quantize_dense(x, gamma, eps: float, fmt: str) -> dict:
    """The plain dense FP4 activation quantizer (the README mirror's dense-only NVFP4 mode).

    Same row scale and block rule as the residual path, applied to xh itself.
    """
    xh = rmsnorm(np.asarray(x, dtype=F32), gamma, eps)
    s_x, g_x = row_scale(xh, fmt)
    codes, scales, _ = _quantize(xh, fmt, s_x, g_x)
    return dict(xh=xh, codes=codes, scales=scales, row_scale=s_x, fmt=fmt)


# --------------------------------------------------------------------------------------
# step a6: the weight payload and its two scale views
# --------------------------------------------------------------------------------------
def pack_weight(w, fmt: str, density_den: int = 2) -> dict:
    """One FP4 weight payload with path-specific scale views (Abstract: both GEMM
    paths read the same FP4 weight codes, each with scales laid out for that path).

    The weight [N, K] (bf16 values as float32) is quantized once in blocks of
    ``density_den * B`` consecutive K positions, the K span one backbone block
    covers at density 1/density_den. The sparse view holds one scale per such
    block; the dense view repeats it for each of the B-wide dense blocks inside.
    NVFP4 adds a per-tensor float32 scale s_w = amax(W)/2688.
    """
    w = np.asarray(w, dtype=F32)
    N, K = w.shape
    B = block_size(fmt)
    Bw = density_den * B
    if K % Bw:
        raise ValueError("K must be a multiple of the weight block")
    if fmt == NVFP4:
        amax = F32(np.abs(w).max())
        if amax == 0:
            s_w, g_w = F32(1.0), F32(0.0)
        else:
            s_w, g_w = F32(amax / _E4M3_TIMES_E2M1_MAX), F32(_E4M3_MAX / amax)
        codes, sb = quantize_blocks_nvfp4(w.reshape(N, K // Bw, Bw),
                                         np.full(N, s_w, F32), np.full(N, g_w, F32))
    else:
        s_w = F32(1.0)
        codes, sb = quantize_blocks_mxfp4(w.reshape(N, K // Bw, Bw))
    return dict(codes=codes.reshape(N, K), scales_sparse=sb,
                scales_dense=np.repeat(sb, density_den, axis=1),
                tensor_scale=s_w, fmt=fmt, block_sparse=Bw, block_dense=B)


def dequant_weight(wp: dict, view: str = "sparse") -> np.ndarray:
    """W_deq [N, K] in float64 (exact) from codes and one scale view, s_w included."""
    codes = wp["codes"]
    N, K = codes.shape
    if view == "sparse":
        sc, B = wp["scales_sparse"], wp["block_sparse"]
    else:
        sc, B = wp["scales_dense"], wp["block_dense"]
    vals = e2m1_decode(codes).reshape(N, K // B, B)
    dec = e4m3_decode(sc) if wp["fmt"] == NVFP4 else e8m0_decode(sc)
    return (vals * dec[:, :, None]).reshape(N, K) * np.float64(wp["tensor_scale"])


# --------------------------------------------------------------------------------------
# steps a7-a9: the two GEMMs into one output
# --------------------------------------------------------------------------------------
def dequant_prep(p: dict):
    """(A_sp, A_res) as exact float64 [T, K]: backbone scattered with zeros, residual; s_x included."""
    fmt, n, m, unit = p["fmt"], p["n"], p["m"], p["unit"]
    T, K = p["res_codes"].shape
    B = block_size(fmt)
    dec = e4m3_decode if fmt == NVFP4 else e8m0_decode
    s_x = p["row_scale"].astype(np.float64)[:, None, None]
    sp = e2m1_decode(p["sp_codes"]).reshape(T, -1, B) * dec(p["sp_scales"])[:, :, None]
    sp = (sp * s_x).reshape(T, -1)
    res = e2m1_decode(p["res_codes"]).reshape(T, -1, B) * dec(p["res_scales"])[:, :, None]
    res = (res * s_x).reshape(T, K)
    return scatter_kept(sp, p["idx"], K, m, unit), res


def linear(p: dict, wp: dict) -> np.ndarray:
    """Y [T, Nout] float64 = A_sp . W_sparse_view^T + A_res . W_dense_view^T.

    Abstract: the backbone goes through a sparse FP4 GEMM, the residual through a
    dense FP4 GEMM that restores what the mask dropped and the backbone's
    quantization error. Every dequantized value is exact in float64, so the
    only rounding is the float64 sum.
    """
    a_sp, a_res = dequant_prep(p)
    return a_sp @ dequant_weight(wp, "sparse").T + a_res @ dequant_weight(wp, "dense").T


def linear_dense(q: dict, wp: dict) -> np.ndarray:
    """Y of the dense FP4 baseline: dequant(Q(xh)) . W_dense_view^T in float64."""
    fmt = q["fmt"]
    T, K = q["codes"].shape
    B = block_size(fmt)
    dec = e4m3_decode if fmt == NVFP4 else e8m0_decode
    a = e2m1_decode(q["codes"]).reshape(T, -1, B) * dec(q["scales"])[:, :, None]
    a = (a * q["row_scale"].astype(np.float64)[:, None, None]).reshape(T, K)
    return a @ dequant_weight(wp, "dense").T
