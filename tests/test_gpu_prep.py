"""Parity of the fused preparation kernel and the dense quantizer with the CPU oracle.

Without RMSNorm (the normalized input held fixed) metadata, codes and scales must be
bit-exact. With fused RMSNorm the GPU sums the squares in float64 in a different order from the
oracle, so a row's rstd may (rarely) differ by one float32 ulp: at most 1e-4 of the codes
may then differ, each by one E2M1 step.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FMT_NAME, code_steps, f32, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def run_prep(S, lin, fmt, unit, use_norm, rows=None):
    x_bits = lin.x if rows is None else lin.x[rows]
    x = to_dev_bf16(x_bits)
    g = to_dev_bf16(lin.gamma) if (use_norm and lin.gamma is not None) else None
    p = S.sharq_prepare(x, g, lin.eps, 2, 4, unit, fmt)
    torch.cuda.synchronize()
    got = hw.read_prep(p, O.block_size(FMT_NAME[fmt]))
    ref = O.prepare(f32(x_bits), f32(lin.gamma) if g is not None else None, lin.eps, 2, 4, unit, FMT_NAME[fmt])
    return got, ref


def assert_exact(got, ref):
    for key in ("idx", "sp_codes", "sp_scales", "res_codes", "res_scales", "row_scale"):
        a, b = got[key], ref[key]
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{key}: {len(bad)} mismatches, first at {bad[:5].tolist()}: "
                                 f"got {a[tuple(bad[0])]} want {b[tuple(bad[0])]}")


_KEYS = ("idx", "sp_codes", "sp_scales", "res_codes", "res_scales", "row_scale")


def _row_with_rstd_step(x, gamma, eps, ref, r, step):
    """The oracle's row r quantized from xh built with rstd moved by `step` float32 ulps.

    Diagnostic only: the GPU and the oracle sum x^2 in float64 in different orders, so
    fp32(sum/K) -- hence rstd -- may differ by one ulp on rare rows. A differing row is
    accounted for when it equals the oracle's result under such a neighbouring rstd."""
    x = np.asarray(x[r:r + 1], np.float32)
    K = x.shape[1]
    ss = np.sum(x.astype(np.float64) ** 2, axis=1)
    rstd = np.float32(1.0) / np.sqrt((ss / np.float64(K)).astype(np.float32) + np.float32(eps))
    rstd = np.nextafter(rstd, np.float32(np.inf) if step > 0 else np.float32(0))
    xh = ((x * rstd[:, None]).astype(np.float32) * np.asarray(gamma, np.float32)[None, :]).astype(np.float32)
    return O.prepare(xh, None, 0.0, ref["n"], ref["m"], ref["unit"], ref["fmt"])


def assert_close_norm(got, ref, x=None, gamma=None, eps=None):
    """Fused-RMSNorm parity: at most 1e-4 of the codes differ, each by one E2M1 step. Mask
    flips and block-scale flips are counted and bounded on their own (each <= 1e-4 of its
    entries), and when the inputs are given every row that differs at all must equal the
    oracle's row under an rstd one float32 ulp away."""
    counts = {}
    for key in ("sp_codes", "res_codes"):
        diff = got[key] != ref[key]
        counts[key] = int(diff.sum())
        assert diff.mean() <= 1e-4, (key, diff.mean())
        if diff.any():
            assert code_steps(got[key][diff], ref[key][diff]).max() <= 1
    counts["mask_flips"] = int((got["idx"] != ref["idx"]).any(axis=2).sum())
    assert counts["mask_flips"] <= 1e-4 * ref["idx"].shape[0] * ref["idx"].shape[1], counts
    for key in ("sp_scales", "res_scales"):
        counts[key] = int((got[key] != ref[key]).sum())
        assert counts[key] <= 1e-4 * got[key].size, counts
    np.testing.assert_allclose(got["row_scale"], ref["row_scale"], rtol=2 ** -22)
    rows = sorted({int(r) for key in _KEYS for r in np.argwhere(
        (got[key] != ref[key]).reshape(got[key].shape[0], -1).any(axis=1)).ravel()})
    if rows:
        print(f"fused-RMSNorm rows differing from the oracle: {rows}; counts {counts}")
    if x is not None:
        for r in rows:
            ok = False
            for step in (-1, 1):
                alt = _row_with_rstd_step(x, gamma, eps, ref, r, step)
                if all(np.array_equal(got[k][r:r + 1], alt[k]) for k in _KEYS):
                    ok = True
                    break
            assert ok, f"row {r} differs from the oracle beyond a one-ulp rstd"


CASES = [  # (workload, rows) -- tiny: 64x256; ragged: 200 rows (not a multiple of 128)
    ("tiny", None),
    ("qkv", np.arange(200)),
]


def workload(name):
    return {"tiny": wl.tiny, "qkv": lambda: wl.llama_qkv(T=256)}[name]()


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("unit", [2, 1])
@pytest.mark.parametrize("name,rows", CASES)
def test_prep_bit_exact_without_norm(fmt, unit, name, rows):
    S = require_gpu()
    got, ref = run_prep(S, workload(name), fmt, unit, use_norm=False, rows=rows)
    assert_exact(got, ref)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("unit", [2, 1])
@pytest.mark.parametrize("name,rows", CASES)
def test_prep_with_fused_rmsnorm(fmt, unit, name, rows):
    S = require_gpu()
    lin = workload(name)
    got, ref = run_prep(S, lin, fmt, unit, use_norm=True, rows=rows)
    x = f32(lin.x if rows is None else lin.x[rows])
    assert_close_norm(got, ref, x, f32(lin.gamma), lin.eps)


@pytest.mark.parametrize("fmt", [0, 1])
def test_prep_hand_derived_rows(fmt):
    """The golden rows of tests/golden run through the kernel (tiled to a valid K)."""
    from tests.golden_io import load
    S = require_gpu()
    name = "nvfp4_pair24_row.txt" if fmt == 0 else "mxfp4_pair24_row.txt"
    g = load(name)
    row = (np.array(g["x_over_D"], dtype=np.float64) * g["D"]).astype(np.float32)
    x = np.tile(row, 256 // row.size)[None, :].repeat(3, axis=0)
    lin = wl.Linear("golden", wl.f32_to_bf16_bits(x), None, wl.f32_to_bf16_bits(np.zeros((16, 256), np.float32)))
    got, ref = run_prep(S, lin, fmt, 2, use_norm=False)
    assert_exact(got, ref)
    n_sp = len(g["sp_codes"])
    assert got["sp_codes"][0, :n_sp].tolist() == g["sp_codes"]
    assert got["res_codes"][0, :len(g["res_codes"])].tolist() == g["res_codes"]


def test_prep_edge_values():
    """Zero rows, all-equal groups (ties), +-x pairs, huge and tiny values, one-token input."""
    S = require_gpu()
    rng = np.random.default_rng(123)
    K = 512
    rows = [np.zeros(K), np.ones(K), np.tile([1, -1, 1, -1], K // 4), rng.standard_normal(K) * 1e-30,
            rng.standard_normal(K) * 3e4, np.tile([0, 0, 0, 5, 0, 0, 0, -5], K // 8),
            np.where(np.arange(K) % 16 == 3, 300.0, 1e-3)]
    x = wl.f32_to_bf16_bits(np.array(rows, dtype=np.float32))
    gamma = wl.f32_to_bf16_bits(np.linspace(0.5, 1.5, K).astype(np.float32))
    for fmt in (0, 1):
        for unit in (1, 2):
            lin = wl.Linear("edge", x, None, x)
            got, ref = run_prep(S, lin, fmt, unit, use_norm=False)
            assert_exact(got, ref)
            lin1 = wl.Linear("one", x[4:5], gamma, x)
            got, ref = run_prep(S, lin1, fmt, unit, use_norm=True)
            assert_close_norm(got, ref, f32(x[4:5]), f32(gamma), lin1.eps)


@pytest.mark.parametrize("fmt", [0, 1])
def test_dense_quantizer_matches_oracle(fmt):
    S = require_gpu()
    lin = wl.llama_qkv(T=200)
    x = to_dev_bf16(lin.x)
    q = S.sharq_quantize_dense(x, None, lin.eps, fmt)
    torch.cuda.synchronize()
    B = O.block_size(FMT_NAME[fmt])
    T, K = lin.x.shape
    ref = O.quantize_dense(f32(lin.x), None, lin.eps, FMT_NAME[fmt])
    got = hw.read_dense(q, B)
    assert np.array_equal(got["codes"], ref["codes"])
    assert np.array_equal(got["scales"], ref["scales"])
    assert np.array_equal(got["row_scale"], ref["row_scale"])


@pytest.mark.parametrize("which,T", [("qkv", 2048), ("down", 4096), ("qwen_down", 300), ("qwen_qkv", 130)])
def test_prep_full_size_sampled_rows(which, T):
    """Full-size workloads in the benchmark's launch configuration (and the widest K, 18944,
    which spreads a row over five warps); rows are independent, so the oracle checks a sample
    of them one by one."""
    S = require_gpu()
    lin = {"qkv": lambda: wl.llama_qkv(T=T), "down": lambda: wl.llama_down(T=T),
           "qwen_down": lambda: wl.qwen("down", T), "qwen_qkv": lambda: wl.qwen("qkv", T)}[which]()
    x = to_dev_bf16(lin.x)
    g = to_dev_bf16(lin.gamma) if lin.gamma is not None else None
    p = S.sharq_prepare(x, g, lin.eps, 2, 4, 2, 0)
    torch.cuda.synchronize()
    got = hw.read_prep(p, 16)
    rows = np.random.default_rng(0).choice(T, min(T, 48), replace=False)
    rows = np.concatenate([rows, [0, T - 1]])
    ref = O.prepare(f32(lin.x[rows]), f32(lin.gamma), lin.eps, 2, 4, 2, O.NVFP4)
    sub = {k: v[rows] for k, v in got.items()}
    if g is not None:
        assert_close_norm(sub, ref, f32(lin.x[rows]), f32(lin.gamma), lin.eps)
    else:
        assert_exact(sub, ref)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("unit", [2, 1])
@pytest.mark.parametrize("use_norm", [False, True])
def test_prep_multiwave_full_rows_sampled(fmt, unit, use_norm):
    """A launch of several waves (6000 rows of K=2048: 750 blocks for 148 SMs) with every piece
    of a row live takes the branch-free piece loop; sampled rows against the oracle."""
    S = require_gpu()
    rng = np.random.default_rng(60 + fmt + 2 * unit)
    T, K = 6000, 2048
    x_bits = wl.outlier_activations(rng, T, K, K // 100, 20.0, 100.0, 0.5)
    g_bits = wl.rms_gamma(rng, K)
    p = S.sharq_prepare(to_dev_bf16(x_bits), to_dev_bf16(g_bits) if use_norm else None, 1e-6, 2, 4, unit, fmt)
    torch.cuda.synchronize()
    got_all = hw.read_prep(p, O.block_size(FMT_NAME[fmt]))
    rows = np.unique(np.concatenate([[0, 127, 128, T - 1], rng.choice(T, 40, replace=False)]))
    got = {k: v[rows] for k, v in got_all.items()}
    ref = O.prepare(f32(x_bits[rows]), f32(g_bits) if use_norm else None, 1e-6, 2, 4, unit, FMT_NAME[fmt])
    if use_norm:
        assert_close_norm(got, ref, f32(x_bits[rows]), f32(g_bits), 1e-6)
    else:
        assert_exact(got, ref)
