"""The 4:8 element pattern (four of every eight consecutive values along K kept) of the fused
preparation operator, against oracle.prepare(..., 4, 8, 1): bit-exact without RMSNorm
(metadata as four ascending indices per group, backbone codes and scales, residual codes and
scales, row scales), the one-ulp rstd allowance with it, ties resolved to the lower index, and
the pattern kept out of the calls that cannot take it (no sparse FP4 MMA of sm_100a executes
element-level 4:8, so sharq_linear rejects it; the gated, per-tensor and no-allocation
preparations are 2:4 only)."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FMT_NAME, f32, require_gpu, to_dev_bf16
from tests.test_gpu_prep import assert_close_norm, assert_exact

pytestmark = pytest.mark.gpu


def prep48(S, x_bits, g_bits, fmt, eps=1e-6):
    x = to_dev_bf16(x_bits)
    g = to_dev_bf16(g_bits) if g_bits is not None else None
    p = S.sharq_prepare(x, g, eps, 4, 8, 1, fmt)
    torch.cuda.synchronize()
    got = hw.read_prep(p, O.block_size(FMT_NAME[fmt]))
    ref = O.prepare(f32(x_bits), f32(g_bits) if g_bits is not None else None, eps, 4, 8, 1, FMT_NAME[fmt])
    return p, got, ref


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("T,K", [(64, 256), (200, 768), (130, 4096), (3, 14336)])
def test_prep48_bit_exact_without_norm(fmt, T, K):
    S = require_gpu()
    rng = np.random.default_rng(T + K + fmt)
    x_bits = wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5)
    _, got, ref = prep48(S, x_bits, None, fmt)
    assert got["idx"].shape == (T, K // 8, 4)
    assert_exact(got, ref)


@pytest.mark.parametrize("fmt", [0, 1])
def test_prep48_with_rmsnorm(fmt):
    S = require_gpu()
    lin = wl.llama_qkv(T=256)
    _, got, ref = prep48(S, lin.x, lin.gamma, fmt, lin.eps)
    assert_close_norm(got, ref, f32(lin.x), f32(lin.gamma), lin.eps)


def test_prep48_ties_and_zeros():
    """Rows of equal magnitudes (mixed signs), all zeros, and one large value per group: the
    kept indices are the lowest ones among equals, exactly as the oracle's stable order."""
    S = require_gpu()
    K = 256
    rows = [np.full(K, 1.5, np.float32), np.zeros(K, np.float32),
            np.tile(np.array([1, -1, 1, -1, 2, 2, -2, 2], np.float32), K // 8),
            np.tile(np.array([0, 0, 0, 7, 0, 0, 0, 0], np.float32), K // 8)]
    x_bits = wl.f32_to_bf16_bits(np.stack(rows))
    for fmt in (0, 1):
        _, got, ref = prep48(S, x_bits, None, fmt)
        assert_exact(got, ref)
    assert np.array_equal(got["idx"][0, 0], [0, 1, 2, 3])
    assert np.array_equal(got["idx"][2, 0], [4, 5, 6, 7])
    assert np.array_equal(got["idx"][3, 0], [0, 1, 2, 3])


def test_prep48_not_executed_or_taken_elsewhere():
    S = require_gpu()
    rng = np.random.default_rng(5)
    x = to_dev_bf16(wl.outlier_activations(rng, 64, 256, 3, 20.0, 100.0, 0.5))
    p = S.sharq_prepare(x, None, 1e-6, 4, 8, 1, 0)
    wp = S.sharq_pack_weight(to_dev_bf16(wl.weight(rng, 32, 256)), 0)
    with pytest.raises(S.SharqError) as e:
        S.sharq_linear(p, wp)
    assert e.value.status == S.SHARQ_ERR_UNSUPPORTED
    gu = to_dev_bf16(wl.gate_up_activations(rng, 64, 256))
    for call in (lambda: S.sharq_prepare_swiglu(gu, 4, 8, 1),
                 lambda: S.sharq_prepare_tensor_scale(x, None, 1e-6, 4, 8, 1),
                 lambda: S.sharq_prepare_tensor_scale_noalloc(x, None, 1e-6, 4, 8, 1)):
        with pytest.raises(S.SharqError) as e:
            call()
        assert e.value.status == S.SHARQ_ERR_UNSUPPORTED


def test_prep48_hand_derived_row():
    """The hand-derived MXFP4 4:8 row of tests/golden through the kernel (tiled to K=256)."""
    from tests.golden_io import load
    S = require_gpu()
    g = load("mxfp4_elem48_row.txt")
    row = (np.array(g["x_over_D"], dtype=np.float64) * g["D"]).astype(np.float32)
    x_bits = wl.f32_to_bf16_bits(np.tile(row, 256 // row.size)[None, :].repeat(3, axis=0))
    _, got, ref = prep48(S, x_bits, None, 1)
    assert_exact(got, ref)
    assert got["idx"][0, :8].reshape(-1).tolist() == g["idx"]
    assert got["sp_codes"][0, :len(g["sp_codes"])].tolist() == g["sp_codes"]
    assert got["res_codes"][0, :len(g["res_codes"])].tolist() == g["res_codes"]
    assert got["sp_scales"][0, :1].tolist() == [g["sp_scales"]]
    assert got["res_scales"][0, :2].tolist() == g["res_scales"]
