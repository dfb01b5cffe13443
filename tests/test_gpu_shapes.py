"""GEMM parity at the configured model shapes beyond the benchmark's own, each in the launch
configuration the benchmark times (full-size activation, full weight, one prepare and one
linear): the Llama-3.1-8B MLP (gate_up N=28672, down K=14336), the Qwen2.5-7B down projection
(K=18944) and its small-token launches (T=1, 16), MXFP4 at the QKV shape, the 8192^3 square and
the video-DiT 32760x5120x5120 linears, and the mixture-of-experts grouped GEMM at its K=2048.

Rows are independent, so the oracle checks sampled activation rows against sampled weight rows
(output columns); the weight's largest |value| is planted in the first sampled weight row, so
packing the sampled rows alone gives the oracle the full weight's per-tensor scale. Prep without
RMSNorm (bit-exact), then max |Y - Y64| <= 1e-4 max|Y64| and relative Frobenius <= 1e-5."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests.test_gpu_grouped import _experts
from tests.gpu_common import FMT_NAME, FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def planted(w_bits: np.ndarray, row: int) -> np.ndarray:
    w = w_bits.copy()
    w[row, 7] = wl.f32_to_bf16_bits(np.array([[0.375]], np.float32))[0, 0]  # > every N(0, 0.02) draw
    return w


def check_shape(S, x_bits, w_bits, fmt, n_rows=24, n_cols=192, seed=0):
    T, K = x_bits.shape
    N = w_bits.shape[0]
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, T - 1], rng.choice(T, min(T, n_rows), replace=False)]))
    cols = rng.choice(N, min(N, n_cols), replace=False)
    cols = np.concatenate([[cols[0]], np.sort(cols[1:])])
    w_bits = planted(w_bits, int(cols[0]))
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), fmt)
    p = S.sharq_prepare(to_dev_bf16(x_bits), None, 1e-6, 2, 4, 2, fmt)
    y = S.sharq_linear(p, wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy()
    del y, p, wp
    name = FMT_NAME[fmt]
    ref = O.linear(O.prepare(f32(x_bits[rows]), None, 1e-6, 2, 4, 2, name), O.pack_weight(f32(w_bits[cols]), name))
    max_abs, frob = gemm_errors(got, ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)
    return max_abs, frob


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_llama_mlp(which):
    S = require_gpu()
    lin = wl.llama_gate_up(T=4096) if which == "gate_up" else wl.llama_down(T=4096)
    print(which, check_shape(S, lin.x, lin.w, 0))


@pytest.mark.parametrize("which,T", [("down", 2048), ("o", 1), ("o", 16), ("qkv", 128)])
def test_qwen_linears(which, T):
    S = require_gpu()
    lin = wl.qwen(which, T)
    print(which, T, check_shape(S, lin.x, lin.w, 0))


def test_mxfp4_full_size_qkv():
    S = require_gpu()
    lin = wl.llama_qkv(T=2048)
    print(check_shape(S, lin.x, lin.w, 1))


@pytest.mark.parametrize("fmt", [0, 1])
def test_square_8192(fmt):
    S = require_gpu()
    lin = wl.square()
    print(fmt, check_shape(S, lin.x, lin.w, fmt))


def test_dit_linear():
    S = require_gpu()
    lin = wl.dit()
    print(check_shape(S, lin.x, lin.w, 0))


@pytest.mark.parametrize("counts,fmt", [([130, 0, 256, 77, 300], 0), ([5, 128, 0, 77, 64, 100, 1, 128], 0),
                                        ([5, 128, 0, 77, 64, 100, 1, 128] * 3, 1)])
def test_moe_grouped_at_expert_shape(counts, fmt):
    """Qwen3-30B-A3B experts (K=2048, N=2*768): ragged and empty experts in one grouped launch;
    the second set (every expert at most 128 rows) runs on single-CTA 128-row tiles."""
    S = require_gpu()
    K, N = wl.QWEN3_MOE["hidden"], 2 * wl.QWEN3_MOE["moe_intermediate"]
    preps, wps, refs = _experts(S, np.random.default_rng(77), counts, K, N, fmt)
    ys = [torch.empty(max(t, 1), N, dtype=torch.float32, device="cuda") for t in counts]
    S.sharq_linear_grouped(preps, wps, ys)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    for e, t in enumerate(counts):
        if t:
            max_abs, frob = gemm_errors(ys[e][:t].cpu().numpy(), refs[e])
            assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (e, max_abs, frob)
