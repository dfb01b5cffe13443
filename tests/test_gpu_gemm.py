"""Parity of the weight packer and of the sparse+dense FP4 GEMM with the CPU oracle.

Packed weights must be bit-exact. GEMM outputs are compared with the oracle's float64
GEMM on the same quantized operands (the activation's prep is bit-exact without
RMSNorm, which these tests use so that both sides see identical operands):
max |Y - Y64| <= 1e-4 * max|Y64| and relative Frobenius error <= 1e-5. bf16 outputs
must equal the round-to-nearest-even of the fp32 output.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import (FMT_NAME, FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("N,K", [(256, 256), (208, 512), (384, 1024)])
def test_pack_weight_bit_exact(fmt, N, K):
    S = require_gpu()
    rng = np.random.default_rng(N + K)
    w_bits = wl.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    w = to_dev_bf16(w_bits)
    wp = S.sharq_pack_weight(w, fmt)
    torch.cuda.synchronize()
    B = O.block_size(FMT_NAME[fmt])
    got = hw.read_wpack(wp, B)
    ref = O.pack_weight(f32(w_bits), FMT_NAME[fmt])
    for key in ("codes", "scales_sparse", "scales_dense"):
        assert np.array_equal(got[key], ref[key]), key
    assert got["tensor_scale"] == ref["tensor_scale"]
    # both halves of a 256-row block carry the block's scales
    for half in ("lo", "hi"):
        cp = hw.read_wpack(wp, B, half)
        assert np.array_equal(cp["scales_sparse"], ref["scales_sparse"]), half
        assert np.array_equal(cp["scales_dense"], ref["scales_dense"]), half


def run_linear(S, x_bits, w_bits, fmt, out_dtype=torch.float32):
    x = to_dev_bf16(x_bits)
    w = to_dev_bf16(w_bits)
    wp = S.sharq_pack_weight(w, fmt)
    p = S.sharq_prepare(x, None, 1e-6, 2, 4, 2, fmt)
    y = S.sharq_linear(p, wp, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    return y, p, wp


def oracle_linear(x_bits, w_bits, fmt):
    p = O.prepare(f32(x_bits), None, 1e-6, 2, 4, 2, FMT_NAME[fmt])
    wp = O.pack_weight(f32(w_bits), FMT_NAME[fmt])
    return O.linear(p, wp)


SHAPES = [  # (T, K, N): one tile; ragged T; several tiles with ragged T and N % 256 != 0; long K
    (64, 256, 256),
    (200, 512, 256),
    (300, 768, 640),
    (128, 4096, 512),
]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("T,K,N", SHAPES)
def test_linear_matches_oracle(fmt, T, K, N):
    S = require_gpu()
    rng = np.random.default_rng(T * 7 + K + N)
    x_bits = wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5)
    w_bits = wl.weight(rng, N, K)
    y, _, _ = run_linear(S, x_bits, w_bits, fmt)
    ref = oracle_linear(x_bits, w_bits, fmt)
    max_abs, frob = gemm_errors(hw.to_np(y), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)


def test_linear_tiny_config_and_bf16_output():
    """BASELINE's tiny config (64 x 256 -> 256, NVFP4, 2:4 pairs); bf16 output = RNE(fp32 output)."""
    S = require_gpu()
    lin = wl.tiny()
    y32, p, wp = run_linear(S, lin.x, lin.w, 0, torch.float32)
    y16 = S.sharq_linear(p, wp, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ref = oracle_linear(lin.x, lin.w, 0)
    max_abs, frob = gemm_errors(hw.to_np(y32), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("fmt", [0, 1])
def test_dense_baseline_gemm_matches_oracle(fmt):
    S = require_gpu()
    rng = np.random.default_rng(5)
    T, K, N = 200, 1024, 384
    x_bits = wl.outlier_activations(rng, T, K, 10, 20.0, 100.0, 0.5)
    w_bits = wl.weight(rng, N, K)
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), fmt)
    q = S.sharq_quantize_dense(to_dev_bf16(x_bits), None, 1e-6, fmt)
    y = S.sharq_linear_dense(q, wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.linear_dense(O.quantize_dense(f32(x_bits), None, 1e-6, FMT_NAME[fmt]),
                         O.pack_weight(f32(w_bits), FMT_NAME[fmt]))
    max_abs, frob = gemm_errors(hw.to_np(y), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)


def test_sharq_beats_dense_nvfp4_on_device():
    """Method sanity on the GPU outputs: SharQ's error against the bf16 product is below the
    library's dense NVFP4 path on outlier activations."""
    S = require_gpu()
    lin = wl.llama_qkv(T=256)
    w_bits = lin.w[:512]
    x = to_dev_bf16(lin.x)
    g = to_dev_bf16(lin.gamma)
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), 0)
    y_sharq = S.sharq_linear(S.sharq_prepare(x, g, lin.eps, 2, 4, 2, 0), wp, out_dtype=torch.float32)
    y_dense = S.sharq_linear_dense(S.sharq_quantize_dense(x, g, lin.eps, 0), wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    xh = O.rmsnorm(f32(lin.x), f32(lin.gamma), lin.eps)
    ref = f32(wl.f32_to_bf16_bits(xh)).astype(np.float64) @ f32(w_bits).astype(np.float64).T
    e_s = np.linalg.norm(hw.to_np(y_sharq) - ref)
    e_d = np.linalg.norm(hw.to_np(y_dense) - ref)
    assert e_s < e_d, (e_s, e_d)


@pytest.mark.parametrize("which", ["qkv"])
def test_linear_full_size_sampled_outputs(which):
    """Llama-3.1-8B QKV at prefill (2048 x 4096 -> 6144), the benchmark's launch; the oracle
    recomputes sampled outputs (rows and columns of Y are independent)."""
    S = require_gpu()
    lin = wl.llama_qkv(T=2048)
    T, K, N = lin.shape
    x = to_dev_bf16(lin.x)
    wp = S.sharq_pack_weight(to_dev_bf16(lin.w), 0)
    p = S.sharq_prepare(x, None, lin.eps, 2, 4, 2, 0)
    y = S.sharq_linear(p, wp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(T, 32, replace=False))
    cols = np.sort(rng.choice(N, 64, replace=False))
    op = O.prepare(f32(lin.x[rows]), None, lin.eps, 2, 4, 2, O.NVFP4)
    full = O.pack_weight(f32(lin.w), O.NVFP4)   # per-tensor scale needs the whole weight
    sub = dict(full, codes=full["codes"][cols], scales_sparse=full["scales_sparse"][cols],
               scales_dense=full["scales_dense"][cols])
    ref = O.linear(op, sub)
    got = hw.to_np(y)[np.ix_(rows, cols)]
    max_abs, frob = gemm_errors(got, ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)


def test_linear_full_size_every_output():
    """The benchmark's GEMM launch (Llama-3.1-8B QKV, 2048 x 4096 -> 6144: 192 pair tiles on
    every SM pair) against the oracle on all 12.6 M outputs, float32 and bf16: every tile of
    every wave, including tiles whose scale buffers were handed between the two CTAs of a
    pair thousands of times."""
    S = require_gpu()
    lin = wl.llama_qkv(T=2048)
    x = to_dev_bf16(lin.x)
    wp = S.sharq_pack_weight(to_dev_bf16(lin.w), 0)
    p = S.sharq_prepare(x, None, lin.eps, 2, 4, 2, 0)
    y32 = S.sharq_linear(p, wp, out_dtype=torch.float32)
    y16 = S.sharq_linear(p, wp)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    ref = O.linear(O.prepare(f32(lin.x), None, lin.eps, 2, 4, 2, O.NVFP4), O.pack_weight(f32(lin.w), O.NVFP4))
    got = hw.to_np(y32)
    max_abs, frob = gemm_errors(got, ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)
    # per-tile check: no 256 x 256 output tile may carry a large share of the error
    tile_err = np.abs(got - ref).reshape(8, 256, 24, 256).max(axis=(1, 3)) / np.abs(ref).max()
    assert tile_err.max() <= MAX_ABS_TOL, np.argwhere(tile_err > MAX_ABS_TOL)[:5]
    assert torch.equal(y16, y32.to(torch.bfloat16))
