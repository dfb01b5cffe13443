"""Parity of the per-tensor second-level scale variant (one NVFP4 scale for the whole activation
tensor) with the CPU oracle: bit-exact without RMSNorm; with RMSNorm the same one-ulp rstd
allowance as the per-row preparation."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FMT_NAME, FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu

KEYS = ("idx", "sp_codes", "sp_scales", "res_codes", "res_scales", "row_scale")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("unit", [2, 1])
@pytest.mark.parametrize("T,K", [(64, 256), (300, 768), (130, 4096)])
def test_tensor_scale_bit_exact(fmt, unit, T, K):
    S = require_gpu()
    rng = np.random.default_rng(T * 3 + K + unit)
    x_bits = wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5)
    p = S.sharq_prepare_tensor_scale(to_dev_bf16(x_bits), None, 1e-6, 2, 4, unit, fmt)
    torch.cuda.synchronize()
    got = hw.read_prep(p, O.block_size(FMT_NAME[fmt]))
    ref = O.prepare(f32(x_bits), None, 1e-6, 2, 4, unit, FMT_NAME[fmt], per_tensor=True)
    for key in KEYS:
        assert np.array_equal(got[key], ref[key]), key
    if fmt == 0:
        assert np.all(got["row_scale"] == got["row_scale"][0])


def test_tensor_scale_with_rmsnorm():
    S = require_gpu()
    lin = wl.llama_qkv(T=256)
    p = S.sharq_prepare_tensor_scale(to_dev_bf16(lin.x), to_dev_bf16(lin.gamma), lin.eps)
    torch.cuda.synchronize()
    got = hw.read_prep(p, 16)
    ref = O.prepare(f32(lin.x), f32(lin.gamma), lin.eps, 2, 4, 2, O.NVFP4, per_tensor=True)
    assert np.all(got["row_scale"] == got["row_scale"][0])
    # the tensor scale equals the oracle's, or is one float32 step away (rstd of the amax row)
    assert abs(int(got["row_scale"][0].view(np.int32)) - int(ref["row_scale"][0].view(np.int32))) <= 1
    for key in ("sp_codes", "res_codes"):
        assert np.mean(got[key] != ref[key]) <= 1e-4, key


def test_linear_on_tensor_scale_prep():
    S = require_gpu()
    rng = np.random.default_rng(31)
    T, K, N = 300, 768, 640
    x_bits = wl.outlier_activations(rng, T, K, 8, 20.0, 100.0, 0.5)
    w_bits = wl.weight(rng, N, K)
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), 0)
    p = S.sharq_prepare_tensor_scale(to_dev_bf16(x_bits))
    y = S.sharq_linear(p, wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.linear(O.prepare(f32(x_bits), None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True),
                   O.pack_weight(f32(w_bits), O.NVFP4))
    max_abs, frob = gemm_errors(y.cpu().numpy(), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)


def test_zero_tensor():
    S = require_gpu()
    x = torch.zeros(40, 512, dtype=torch.bfloat16, device="cuda")
    p = S.sharq_prepare_tensor_scale(x)
    torch.cuda.synchronize()
    got = hw.read_prep(p, 16)
    assert np.all(got["row_scale"] == 1.0)
    assert not got["sp_codes"].any() and not got["res_codes"].any()


@pytest.mark.parametrize("T,K,norm", [(5000, 256, False), (1500, 8192, False), (3000, 4096, True)])
def test_tensor_scale_several_row_groups_per_block(T, K, norm):
    """More row groups than resident blocks: phase 2 re-reads rows (and their parked rstd)."""
    S = require_gpu()
    rng = np.random.default_rng(T + K)
    x_bits = wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5)
    g_bits = wl.rms_gamma(rng, K) if norm else None
    ws = torch.zeros(S.sharq_tensor_scale_workspace_size(T, K), dtype=torch.uint8, device="cuda")
    x = to_dev_bf16(x_bits)
    g = to_dev_bf16(g_bits) if norm else None
    p = S.sharq_prepare_tensor_scale(x, g, 1e-6, workspace=ws)
    p2 = S.sharq_prepare_tensor_scale(x, g, 1e-6, workspace=ws)  # the same workspace again
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0  # the counter is left at zero
    assert int(ws[4:8].view(torch.int32).item()) == 2  # two barrier generations
    assert S.sharq_device_status() == S.SHARQ_OK
    assert torch.equal(p.tiles, p2.tiles) and torch.equal(p.row_scale, p2.row_scale)
    got = hw.read_prep(p, 16)
    ref = O.prepare(f32(x_bits), f32(g_bits) if norm else None, 1e-6, 2, 4, 2, O.NVFP4, per_tensor=True)
    assert np.all(got["row_scale"] == got["row_scale"][0])
    if not norm:
        for key in KEYS:
            assert np.array_equal(got[key], ref[key]), key
    else:
        assert abs(int(got["row_scale"][0].view(np.int32)) - int(ref["row_scale"][0].view(np.int32))) <= 1
        for key in ("sp_codes", "res_codes", "idx"):
            assert np.mean(got[key] != ref[key]) <= 1e-4, key


def test_tensor_scale_benchmark_launch():
    """The benchmark's per-tensor launch (Llama-3.1-8B QKV input, 2048 x 4096, fused RMSNorm):
    the whole tensor against the oracle (the one-ulp rstd allowance of the per-row operator)."""
    S = require_gpu()
    lin = wl.llama_qkv(T=2048)
    ws = torch.zeros(S.sharq_tensor_scale_workspace_size(2048, 4096), dtype=torch.uint8, device="cuda")
    p = S.sharq_prepare_tensor_scale(to_dev_bf16(lin.x), to_dev_bf16(lin.gamma), lin.eps, workspace=ws)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    got = hw.read_prep(p, 16)
    ref = O.prepare(f32(lin.x), f32(lin.gamma), lin.eps, 2, 4, 2, O.NVFP4, per_tensor=True)
    assert np.all(got["row_scale"] == got["row_scale"][0])
    assert abs(int(got["row_scale"][0].view(np.int32)) - int(ref["row_scale"][0].view(np.int32))) <= 1
    for key in ("sp_codes", "res_codes", "idx", "sp_scales", "res_scales"):
        assert np.mean(got[key] != ref[key]) <= 1e-4, key
