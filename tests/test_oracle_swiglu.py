"""Pins of the oracle's gated activation (SiLU(g) * u fused into the preparation operator).

Each check ties the float32 restatement to something other than itself: numpy's float64
exp, torch's float64 SiLU, torch's bf16 rounding, closed forms and planted mistakes.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O

F32 = np.float32


def _ulp(x):
    return np.spacing(np.abs(x).astype(F32)).astype(np.float64)


def test_exp_neg_abs_against_float64_exp():
    g = np.concatenate([np.linspace(-87, 87, 1_000_001, dtype=F32),
                        np.random.default_rng(0).standard_normal(200_000).astype(F32) * 4])
    e = O.exp_neg_abs(g).astype(np.float64)
    ref = np.exp(-np.abs(g.astype(np.float64)))
    ok = ref >= 2.0 ** -126                   # below that the reading flushes to zero
    err = np.abs(e[ok] - ref[ok]) / _ulp(ref[ok].astype(F32))
    assert err.max() <= 3.0, err.max()
    assert np.all(np.diff(O.exp_neg_abs(np.linspace(0, 80, 100_001, dtype=F32))) <= 0)  # monotone


def test_exp_neg_abs_special_values():
    assert O.exp_neg_abs(np.array([0.0], F32))[0] == F32(1.0)
    assert O.exp_neg_abs(np.array([-0.0], F32))[0] == F32(1.0)
    # t = |g| log2(e) >= 126: below the normal range, flushed to zero by the reading
    assert np.all(O.exp_neg_abs(np.array([88.0, -88.0, 1e4, -3e38], F32)) == 0)
    # symmetric in the sign of g
    g = np.random.default_rng(1).standard_normal(1000).astype(F32)
    assert np.array_equal(O.exp_neg_abs(g), O.exp_neg_abs(-g))


def test_silu_against_torch_float64():
    g = np.concatenate([np.linspace(-40, 40, 400_001, dtype=F32),
                        np.random.default_rng(2).standard_normal(100_000).astype(F32) * 3])
    s = O.silu(g).astype(np.float64)
    ref = torch.nn.functional.silu(torch.from_numpy(g.astype(np.float64))).numpy()
    ok = np.abs(ref) > 1e-30
    err = np.abs(s[ok] - ref[ok]) / _ulp(ref[ok].astype(F32))
    assert err.max() <= 8.0, err.max()


def test_silu_closed_forms():
    assert O.silu(np.array([0.0], F32))[0] == 0 and not np.signbit(O.silu(np.array([0.0], F32))[0])
    assert np.signbit(O.silu(np.array([-0.0], F32))[0])
    big = np.linspace(17, 1e4, 1000, dtype=F32)  # e < 2^-24: 1 + e rounds to 1, sigma = 1
    assert np.array_equal(O.silu(big), big)
    # odd-ish symmetry: silu(g) - silu(-g) = g up to float32 rounding
    g = np.linspace(-8, 8, 10_001, dtype=F32)
    d = O.silu(g).astype(np.float64) - O.silu(-g).astype(np.float64)
    assert np.max(np.abs(d - g)) <= 4 * np.max(_ulp(g))


def test_round_bf16_matches_torch():
    v = np.random.default_rng(3).standard_normal(1_000_000).astype(F32) * np.float32(1e3)
    v = np.concatenate([v, np.array([0.0, -0.0, 1.00390625, 1.01171875, -1.00390625], F32)])  # ties
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(O.round_bf16(v).view(np.uint32), ref.view(np.uint32))


def test_swiglu_against_float64_reference():
    rng = np.random.default_rng(4)
    gu_bits = wl.gate_up_activations(rng, 64, 512)
    gu = wl.bf16_bits_to_f32(gu_bits)
    x = O.swiglu(gu)
    g, u = gu[:, :512].astype(np.float64), gu[:, 512:].astype(np.float64)
    ref = torch.from_numpy(torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u).to(torch.float32)
    ref = ref.to(torch.bfloat16).to(torch.float32).numpy()
    diff = x != ref
    assert diff.mean() <= 1e-3, diff.mean()             # float32 steps vs one float64 rounding
    if diff.any():                                       # and never by more than one bf16 step
        bits = np.abs(x[diff].view(np.int32).astype(np.int64) - ref[diff].view(np.int32).astype(np.int64))
        assert bits.max() <= 1 << 16
    assert x.shape == (64, 512)


def test_swiglu_planted_mistakes_fail():
    gu = wl.bf16_bits_to_f32(wl.gate_up_activations(np.random.default_rng(5), 16, 256))
    x = O.swiglu(gu)
    swapped = O.swiglu(np.concatenate([gu[:, 256:], gu[:, :256]], axis=1))  # silu(u) * g
    assert not np.array_equal(x, swapped)
    no_gate = O.round_bf16((gu[:, :256] * gu[:, 256:]).astype(F32))         # g * u without SiLU
    assert not np.array_equal(x, no_gate)


def test_prepare_swiglu_is_prepare_of_swiglu():
    gu = wl.bf16_bits_to_f32(wl.gate_up_activations(np.random.default_rng(6), 8, 256))
    a = O.prepare_swiglu(gu, 2, 4, 2, O.NVFP4)
    b = O.prepare(O.swiglu(gu), None, 0.0, 2, 4, 2, O.NVFP4)
    for k in ("sp_codes", "res_codes", "sp_scales", "res_scales", "row_scale", "idx"):
        assert np.array_equal(a[k], b[k])
