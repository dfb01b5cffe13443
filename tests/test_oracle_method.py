"""Pins for the oracle's mask, quantizers, preparation operator, weight views and GEMM.

Every check ties the oracle to something other than its own code: brute force over
all subsets or codes, library routines (torch rms_norm, ml_dtypes, frexp/log2),
hand-derived fixtures (tests/golden) and closed-form invariants.
"""
import itertools
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from oracle.formats import e2m1_decode, e4m3_decode, e8m0_decode
from tests.golden_io import load

F32 = np.float32


# ------------------------------------------------------------------ mask
def _brute_force_keep(keys, n):
    """All n-subsets S such that every kept key beats every dropped key, ties going to the
    lower index. Exactly one subset qualifies; returned sorted."""
    m = len(keys)
    winners = []
    for s in itertools.combinations(range(m), n):
        ok = True
        for i in s:
            for j in range(m):
                if j in s:
                    continue
                if keys[i] < keys[j] or (keys[i] == keys[j] and i > j):
                    ok = False
        if ok:
            winners.append(list(s))
    assert len(winners) == 1, (keys, winners)
    return winners[0]


@pytest.mark.parametrize("n,m,unit", [(2, 4, 1), (2, 4, 2), (4, 8, 1), (1, 2, 1), (1, 4, 2), (3, 4, 1)])
def test_mask_brute_force(n, m, unit):
    rng = np.random.default_rng(10 + n * 7 + m + unit)
    # few distinct magnitudes and both signs -> many ties, including +x / -x pairs
    pool = np.float32([0, 0.5, 1, 1, 2, 3, -1, -2, -0.5])
    T, G = 40, 6
    xh = rng.choice(pool, size=(T, G * m * unit)).astype(F32)
    idx = O.nm_select(xh, n, m, unit)
    for t in range(T):
        for g in range(G):
            seg = xh[t, g * m * unit:(g + 1) * m * unit].reshape(m, unit)
            keys = [float(np.max(np.abs(seg[u]))) for u in range(m)]
            assert list(idx[t, g]) == _brute_force_keep(keys, n)


def test_mask_ties_go_to_lower_index():
    xh = np.float32([[1, -1, 1, -1, 2, 2, 2, 2]])
    assert O.nm_select(xh, 2, 4, 1).tolist() == [[[0, 1], [0, 1]]]
    assert O.nm_select(xh, 2, 4, 2).tolist() == [[[2, 3]]]
    # pair keys tie (both 1): lower pair kept
    xh = np.float32([[1, 0, 0, -1, 0, 0, 0, 0]])
    assert O.nm_select(xh, 1, 4, 2).tolist() == [[[0]]]


def test_mask_keeps_exactly_n_and_dominates():
    lin = wl.tiny()
    xh = O.rmsnorm(wl.bf16_bits_to_f32(lin.x), wl.bf16_bits_to_f32(lin.gamma), lin.eps)
    for n, m, unit in [(2, 4, 1), (2, 4, 2), (4, 8, 1)]:
        idx = O.nm_select(xh, n, m, unit)
        keep = O.keep_mask(idx, xh.shape[1], m, unit)
        assert keep.sum() == xh.size * n // m
        g = keep.reshape(xh.shape[0], -1, m * unit)
        a = np.abs(xh).reshape(g.shape)
        # largest element of every group is always kept, so the row amax lies in the backbone
        assert np.all(np.take_along_axis(g, a.argmax(axis=2)[..., None], axis=2))


# ------------------------------------------------------------------ RMSNorm
def test_rmsnorm_matches_torch_float64():
    lin = wl.llama_qkv(T=64)
    x = wl.bf16_bits_to_f32(lin.x)
    g = wl.bf16_bits_to_f32(lin.gamma)
    ours = O.rmsnorm(x, g, 1e-6).astype(np.float64)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (x.shape[1],),
                                       torch.from_numpy(g).double(), eps=1e-6).numpy()
    assert np.max(np.abs(ours - ref) / np.maximum(np.abs(ref), 1e-30)) < 2.0 ** -21


def test_rmsnorm_unit_rms_and_identity():
    rng = np.random.default_rng(3)
    x = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.standard_normal((8, 512)).astype(F32) * 7))
    y = O.rmsnorm(x, np.ones(512, F32), 0.0).astype(np.float64)
    assert np.allclose(np.mean(y ** 2, axis=1), 1.0, rtol=1e-6)
    assert np.array_equal(O.rmsnorm(x, None, 1e-6), x)


# ------------------------------------------------------------------ quantizers
def test_nvfp4_codes_are_nearest_grid_points():
    """Away from rounding midpoints, each code is the E2M1 value nearest to v/d (exact arithmetic),
    and the block scale is the E4M3 value nearest to amax*g_x (torch's float8 cast)."""
    rng = np.random.default_rng(5)
    vals = (rng.standard_normal((16, 8, 16)) * rng.uniform(0.01, 30, (16, 8, 1))).astype(F32)
    s_x, g_x = O.row_scale(vals.reshape(16, -1), O.NVFP4)
    codes, sb = O.quantize_blocks_nvfp4(vals, s_x, g_x)
    amax = np.abs(vals).max(axis=2)
    lib_sb = torch.from_numpy((amax * g_x[:, None]).astype(F32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(sb, lib_sb)
    d = e4m3_decode(sb) * s_x[:, None].astype(np.float64)
    ratio = vals.astype(np.float64) / d[:, :, None]
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mag = np.abs(ratio)
    nearest = np.abs(mag[..., None] - grid).argmin(axis=-1)
    nearest = np.where(mag >= 6, 7, nearest)
    mids = (grid[1:] + grid[:-1]) / 2
    far = np.min(np.abs(mag[..., None] - mids), axis=-1) > 1e-5
    assert far.mean() > 0.99
    assert np.array_equal((codes & 7)[far], nearest[far])
    assert np.array_equal((codes >> 3)[ratio != 0], np.signbit(ratio[ratio != 0]).astype(np.uint8))


def test_row_scale_closed_form():
    xh = np.float32([[2.625, -1.0, 0.0, 0.5], [0, 0, 0, 0], [-448 * 6, 1, 1, 1]])
    s_x, g_x = O.row_scale(xh, O.NVFP4)
    assert s_x.tolist() == [2.0 ** -10, 1.0, 1.0]
    assert g_x[1] == 0 and g_x[2] == np.float32(448 / 2688)


def test_mx_exponent_matches_log2():
    rng = np.random.default_rng(6)
    a = np.exp(rng.uniform(-60, 60, 5000)).astype(F32)
    a = np.concatenate([a, np.float32([1, 2, 4, 6, 8, 0.5, 0.75, 1.5, 3, 2.0 ** -126])])
    want = np.clip(np.array([math.floor(math.log2(float(v))) for v in a]) + 125, 0, 254)
    assert np.array_equal(O.mx_exponent(a).astype(int), want)
    assert O.mx_exponent(np.float32([0]))[0] == 0


def test_mxfp4_power_of_two_closed_form():
    """With an E8M0 scale the scaling is exact, so the codes equal ml_dtypes' E2M1 cast of x/2^(e-127)."""
    rng = np.random.default_rng(7)
    vals = (rng.standard_normal((8, 4, 32)) * 10).astype(F32)
    codes, e = O.quantize_blocks_mxfp4(vals)
    scaled = (vals.astype(np.float64) / e8m0_decode(e)[:, :, None]).astype(F32)
    lib = scaled.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(codes, lib)
    # the block amax scales into [4, 8): the largest element saturates or lands on 4 or 6
    top = np.abs(scaled).max(axis=2)
    assert np.all((top >= 4) & (top < 8))


def test_zero_block_gives_zero_codes_and_scale():
    vals = np.zeros((1, 2, 16), F32)
    codes, sb = O.quantize_blocks_nvfp4(vals, np.float32([2.0 ** -10]), np.float32([170.0]))
    assert np.all(codes == 0) and np.all(sb == 0)
    codes, e = O.quantize_blocks_mxfp4(np.zeros((1, 2, 32), F32))
    assert np.all(codes == 0) and np.all(e == 0)


# ------------------------------------------------------------------ preparation: golden rows
@pytest.mark.parametrize("name", ["nvfp4_pair24_row.txt", "nvfp4_elem24_row.txt", "mxfp4_pair24_row.txt",
                                  "mxfp4_elem48_row.txt"])
def test_prepare_matches_hand_derived_row(name):
    g = load(name)
    x = (np.array(g["x_over_D"], dtype=np.float64) * g["D"]).astype(F32)[None, :]
    assert np.array_equal(wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x)), x)
    p = O.prepare(x, None, 1e-6, g["n"], g["m"], g["unit"], g["fmt"])
    assert p["idx"].reshape(-1).tolist() == g["idx"]
    assert p["sp_codes"].reshape(-1).tolist() == g["sp_codes"]
    assert np.atleast_1d(p["sp_scales"].reshape(-1)).tolist() == np.atleast_1d(g["sp_scales"]).tolist()
    assert p["res_codes"].reshape(-1).tolist() == g["res_codes"]
    assert p["res_scales"].reshape(-1).tolist() == np.atleast_1d(g["res_scales"]).tolist()
    assert float(p["row_scale"][0]) == float(g["row_scale"])


# ------------------------------------------------------------------ preparation: invariants
@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
@pytest.mark.parametrize("n,m,unit", [(2, 4, 2), (2, 4, 1)])
def test_residual_is_defined_against_quantized_backbone(fmt, n, m, unit):
    lin = wl.tiny()
    x, gm = wl.bf16_bits_to_f32(lin.x), wl.bf16_bits_to_f32(lin.gamma)
    p = O.prepare(x, gm, 1e-6, n, m, unit, fmt)
    K = x.shape[1]
    deq = O.scatter_kept(p["sp_deq"], p["idx"], K, m, unit).astype(np.float64)
    xh, r = p["xh"].astype(np.float64), p["resid"].astype(np.float64)
    # r = fl(xh - deq): the only error is one float32 rounding of the subtraction
    err = np.abs((xh - deq) - r)
    half_ulp = np.spacing(np.abs(p["resid"])).astype(np.float64) / 2
    assert np.all(err <= half_ulp)
    keep = O.keep_mask(p["idx"], K, m, unit)
    assert np.array_equal(r[~keep], xh[~keep])
    # reconstruction error is bounded by the residual's own quantization step
    a_sp, a_res = O.dequant_prep(p)
    B = O.block_size(fmt)
    dec = e4m3_decode if fmt == O.NVFP4 else e8m0_decode
    step = (dec(p["res_scales"]) * p["row_scale"].astype(np.float64)[:, None])   # value of one E2M1 "1.0"
    step = np.repeat(step, B, axis=1)
    rq = np.abs(r - a_res)
    # E2M1 half-gaps: 0.25 below 2, 0.5 in [2,4), 1 in [4,6]; beyond 6*step the value saturates
    bound = np.where(np.abs(r) <= 6 * step, step * (1.0 + 1e-6), np.abs(r) - 6 * step + step * 1e-6)
    assert np.all(rq <= bound + 1e-30)
    # a_sp is the exact product; the residual was formed against its float32 rounding
    deq32 = O.scatter_kept(p["sp_deq"], p["idx"], K, m, unit)
    half_ulp_deq = np.spacing(np.abs(deq32)).astype(np.float64) / 2
    assert np.all(np.abs(xh - a_sp - a_res) <= bound + half_ulp + half_ulp_deq + 1e-30)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
def test_n_equals_m_degenerates_to_dense_fp4(fmt):
    lin = wl.tiny()
    x, gm = wl.bf16_bits_to_f32(lin.x), wl.bf16_bits_to_f32(lin.gamma)
    p = O.prepare(x, gm, 1e-6, 4, 4, 1, fmt)
    q = O.quantize_dense(x, gm, 1e-6, fmt)
    assert np.array_equal(p["sp_codes"], q["codes"])
    assert np.array_equal(p["sp_scales"], q["scales"])
    assert np.array_equal(p["row_scale"], q["row_scale"])
    # the residual is the dense quantization error, quantized again
    a_sp, a_res = O.dequant_prep(p)
    assert np.array_equal(a_sp, O.dequant_prep(dict(p, sp_codes=q["codes"]))[0])
    assert np.max(np.abs(p["xh"] - a_sp - a_res)) < np.max(np.abs(p["xh"] - a_sp))


# ------------------------------------------------------------------ weight payload
@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
def test_weight_views_decode_identically(fmt):
    lin = wl.tiny()
    w = wl.bf16_bits_to_f32(lin.w)
    wp = O.pack_weight(w, fmt)
    assert np.array_equal(O.dequant_weight(wp, "sparse"), O.dequant_weight(wp, "dense"))
    assert wp["scales_dense"].shape[1] == 2 * wp["scales_sparse"].shape[1]
    err = np.abs(O.dequant_weight(wp) - w)
    assert np.max(err) <= np.max(np.abs(w)) / 6 * (1 if fmt == O.NVFP4 else 2)


# ------------------------------------------------------------------ GEMM
def _decode_lib(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _scale_lib(sc, fmt):
    t = torch.from_numpy(np.ascontiguousarray(sc, dtype=np.uint8))
    d = torch.float8_e4m3fn if fmt == O.NVFP4 else torch.float8_e8m0fnu
    return t.view(d).double().numpy()


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
@pytest.mark.parametrize("unit", [1, 2])
def test_linear_matches_triple_loop(fmt, unit):
    """Brute force: decode every code with library codecs and sum in Python, one output at a time."""
    rng = np.random.default_rng(11)
    T, K, N = 3, 128, 5
    x = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(F32) * 3))
    x[:, 7] *= 40
    w = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(F32) * 0.02))
    p = O.prepare(x, None, 1e-6, 2, 4, unit, fmt)
    wp = O.pack_weight(w, fmt)
    Y = O.linear(p, wp)
    B = O.block_size(fmt)
    sp_vals = _decode_lib(p["sp_codes"])
    sp_sc = _scale_lib(p["sp_scales"], fmt)
    rs_vals = _decode_lib(p["res_codes"])
    rs_sc = _scale_lib(p["res_scales"], fmt)
    w_vals = _decode_lib(wp["codes"])
    w_sc_sp = _scale_lib(wp["scales_sparse"], fmt)
    w_sc_dn = _scale_lib(wp["scales_dense"], fmt)
    s_w = float(wp["tensor_scale"])
    for t in range(T):
        s_x = float(p["row_scale"][t])
        # logical K position of each stored backbone value
        pos = []
        for g in range(K // (4 * unit)):
            for u in p["idx"][t, g]:
                pos.extend(g * 4 * unit + u * unit + j for j in range(unit))
        for n_ in range(N):
            acc = 0.0
            for s, k in enumerate(pos):
                a = sp_vals[t, s] * sp_sc[t, s // B] * s_x
                acc += a * w_vals[n_, k] * w_sc_sp[n_, k // (2 * B)] * s_w
            for k in range(K):
                a = rs_vals[t, k] * rs_sc[t, k // B] * s_x
                acc += a * w_vals[n_, k] * w_sc_dn[n_, k // B] * s_w
            assert math.isclose(acc, Y[t, n_], rel_tol=1e-12, abs_tol=1e-12)


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
def test_linear_dense_matches_triple_loop(fmt):
    """Brute force for the dense FP4 baseline: every activation code, its block scale and the
    row scale, every weight code with its dense-view scale and s_w, decoded by library codecs
    and summed in Python one output at a time (fused RMSNorm on, outlier channels present)."""
    rng = np.random.default_rng(12)
    T, K, N = 3, 128, 5
    x = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.standard_normal((T, K)).astype(F32) * 3))
    x[:, 5] *= 60
    x[1] *= 1e-3                                            # rows with very different scales
    gamma = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(F32)))
    w = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(F32) * 0.02))
    q = O.quantize_dense(x, gamma, 1e-6, fmt)
    wp = O.pack_weight(w, fmt)
    Y = O.linear_dense(q, wp)
    B = O.block_size(fmt)
    a_vals = _decode_lib(q["codes"])
    a_sc = _scale_lib(q["scales"], fmt)
    w_vals = _decode_lib(wp["codes"])
    w_sc = _scale_lib(wp["scales_dense"], fmt)
    s_w = float(wp["tensor_scale"])
    assert len({float(s) for s in q["row_scale"]}) == (T if fmt == O.NVFP4 else 1)
    for t in range(T):
        s_x = float(q["row_scale"][t])
        for n_ in range(N):
            acc = 0.0
            for k in range(K):
                acc += (a_vals[t, k] * a_sc[t, k // B] * s_x) * (w_vals[n_, k] * w_sc[n_, k // B] * s_w)
            assert math.isclose(acc, Y[t, n_], rel_tol=1e-12, abs_tol=1e-300)


def test_sharq_error_below_dense_nvfp4_on_outlier_inputs():
    """Method sanity: against the bf16 product xh.W^T, SharQ's output error is below dense NVFP4's
    (the abstract's accuracy claim, checked as an inequality on synthetic outlier inputs)."""
    for lin in (wl.tiny(), wl.llama_qkv(T=64)):
        x = wl.bf16_bits_to_f32(lin.x)
        gm = None if lin.gamma is None else wl.bf16_bits_to_f32(lin.gamma)
        w = wl.bf16_bits_to_f32(lin.w)
        if lin.w.shape[0] > 512:
            w = w[:512]
        wp = O.pack_weight(w, O.NVFP4)
        p = O.prepare(x, gm, lin.eps, 2, 4, 2, O.NVFP4)
        q = O.quantize_dense(x, gm, lin.eps, O.NVFP4)
        xh_bf16 = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(p["xh"])).astype(np.float64)
        ref = xh_bf16 @ w.astype(np.float64).T
        e_sharq = np.linalg.norm(O.linear(p, wp) - ref)
        e_dense = np.linalg.norm(O.linear_dense(q, wp) - ref)
        assert e_sharq < e_dense


# ---------------------------------------------------------------- per-tensor activation scale
def test_per_tensor_scale_single_row_equals_per_row():
    """With one token row the tensor amax is the row amax: both readings coincide."""
    x = wl.bf16_bits_to_f32(wl.outlier_activations(np.random.default_rng(21), 1, 512, 4, 20.0, 100.0, 0.5))
    a = O.prepare(x, None, 1e-6, 2, 4, 2, O.NVFP4)
    b = O.prepare(x, None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True)
    for k in ("sp_codes", "res_codes", "sp_scales", "res_scales", "row_scale", "idx"):
        assert np.array_equal(a[k], b[k]), k


def test_per_tensor_scale_is_the_largest_row_scale():
    x = wl.bf16_bits_to_f32(wl.outlier_activations(np.random.default_rng(22), 32, 512, 4, 20.0, 100.0, 0.5))
    a = O.prepare(x, None, 1e-6, 2, 4, 2, O.NVFP4)
    b = O.prepare(x, None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True)
    assert np.all(b["row_scale"] == a["row_scale"].max())
    # the row holding the tensor amax is quantized exactly as with its own row scale
    r = int(np.argmax(a["row_scale"]))
    for k in ("sp_codes", "res_codes", "sp_scales", "res_scales"):
        assert np.array_equal(a[k][r], b[k][r]), k
    # other rows use a larger scale: their block scales can only shrink
    others = np.arange(32) != r
    assert np.all(e4m3_decode(b["sp_scales"][others]) <= e4m3_decode(a["sp_scales"][others]))


def test_per_tensor_scale_power_of_two_invariance():
    """Scaling X by 2^k scales s_x by 2^k and leaves every code and block scale unchanged."""
    x = wl.bf16_bits_to_f32(wl.outlier_activations(np.random.default_rng(23), 16, 256, 2, 20.0, 100.0, 0.5))
    a = O.prepare(x, None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True)
    b = O.prepare(x * np.float32(8.0), None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True)
    for k in ("sp_codes", "res_codes", "sp_scales", "res_scales", "idx"):
        assert np.array_equal(a[k], b[k]), k
    assert np.array_equal(b["row_scale"], a["row_scale"] * np.float32(8.0))
