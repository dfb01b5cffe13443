"""Parity of the preparation operator fed by a gate/up output (x = SiLU(g) * u formed in the
kernel) with the CPU oracle: metadata, codes and scales bit-exact, because both sides evaluate
the gated activation with the same correctly rounded float32 steps."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FMT_NAME, FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu

KEYS = ("idx", "sp_codes", "sp_scales", "res_codes", "res_scales", "row_scale")


def check_exact(got, ref, rows=None):
    for key in KEYS:
        a = got[key] if rows is None else got[key][rows]
        b = ref[key]
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{key}: {len(bad)} mismatches, first at {bad[:5].tolist()}")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("unit", [2, 1])
@pytest.mark.parametrize("T,K", [(64, 256), (200, 768), (130, 4096)])
def test_prepare_swiglu_bit_exact(fmt, unit, T, K):
    S = require_gpu()
    gu_bits = wl.gate_up_activations(np.random.default_rng(T + K + unit), T, K)
    p = S.sharq_prepare_swiglu(to_dev_bf16(gu_bits), 2, 4, unit, fmt)
    torch.cuda.synchronize()
    got = hw.read_prep(p, O.block_size(FMT_NAME[fmt]))
    ref = O.prepare_swiglu(f32(gu_bits), 2, 4, unit, FMT_NAME[fmt])
    check_exact(got, ref)


def test_prepare_swiglu_edge_values():
    """Large |g| (sigma saturates or exp leaves the normal range), signed zeros, subnormal and
    tiny inputs, a zero row."""
    S = require_gpu()
    T, K = 8, 512
    rng = np.random.default_rng(7)
    g = rng.standard_normal((T, K)).astype(np.float32)
    u = rng.standard_normal((T, K)).astype(np.float32)
    g[0, :64] = np.linspace(-120, 120, 64)
    g[1, :8] = [0.0, -0.0, 87.0, -87.0, 87.5, -87.5, 1e-38, -1e-38]
    u[2, :] = 0.0
    g[3, :] = 0.0
    g[4, :32] = np.float32(3e-39)  # bf16 subnormals after rounding
    u[5, :] *= np.float32(1e-30)
    gu_bits = wl.f32_to_bf16_bits(np.concatenate([g, u], axis=1))
    for fmt in (0, 1):
        p = S.sharq_prepare_swiglu(to_dev_bf16(gu_bits), 2, 4, 2, fmt)
        torch.cuda.synchronize()
        check_exact(hw.read_prep(p, O.block_size(FMT_NAME[fmt])), O.prepare_swiglu(f32(gu_bits), 2, 4, 2,
                                                                                       FMT_NAME[fmt]))


def test_prepare_swiglu_full_size_sampled_rows():
    """Llama-3.1-8B down projection, T=2048, K=14336 (four warps per row): sampled rows."""
    S = require_gpu()
    gu_bits, _ = wl.llama_down_gate_up(T=2048)
    p = S.sharq_prepare_swiglu(to_dev_bf16(gu_bits))
    torch.cuda.synchronize()
    got = hw.read_prep(p, 16)
    rows = np.concatenate([np.random.default_rng(0).choice(2048, 24, replace=False), [0, 2047]])
    check_exact(got, O.prepare_swiglu(f32(gu_bits[rows]), 2, 4, 2, O.NVFP4), rows)


def test_linear_on_swiglu_prep():
    S = require_gpu()
    rng = np.random.default_rng(11)
    T, K, N = 200, 1024, 384
    gu_bits = wl.gate_up_activations(rng, T, K)
    w_bits = wl.weight(rng, N, K)
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), 0)
    p = S.sharq_prepare_swiglu(to_dev_bf16(gu_bits))
    y = S.sharq_linear(p, wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.linear(O.prepare_swiglu(f32(gu_bits), 2, 4, 2, O.NVFP4), O.pack_weight(f32(w_bits), O.NVFP4))
    max_abs, frob = gemm_errors(y.cpu().numpy(), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)


def test_prepare_swiglu_rejects_bad_arguments():
    S = require_gpu()
    gu = torch.zeros(16, 2 * 4000, dtype=torch.bfloat16, device="cuda")  # k not a multiple of 256
    with pytest.raises(S.SharqError):
        S.sharq_prepare_swiglu(gu)
