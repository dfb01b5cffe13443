"""Out-of-bounds evidence without a sanitizer: every device buffer a call writes is placed between
two 4 KiB guard regions filled with a canary byte, and the guards must be intact after the call
(and the guarded results equal the unguarded ones). Ragged token and output counts, a single
token, both formats and both mask units. Also: the library's calls issued on a non-default
stream behind a slow producer kernel that writes their input (the linear waits for the
preparation through programmatic dependent launch)."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


class Guarded:
    def __init__(self, nbytes: int):
        self.n = nbytes
        self.full = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.view = self.full[GUARD:GUARD + nbytes]

    def as_type(self, dtype, shape):
        return self.view.view(dtype).view(shape)

    def intact(self) -> bool:
        f = self.full.cpu().numpy()
        return bool((f[:GUARD] == CANARY).all() and (f[GUARD + self.n:] == CANARY).all())


def guarded_prep(S, T, K, unit, fmt):
    s = S.sharq_prep_buffer_sizes(T, K, 2, 4, unit, fmt)
    gt, gr = Guarded(s[0]), Guarded(s[1])
    return S.Prep(gt.view, gr.as_type(torch.float32, (T,)), T, K, 2, 4, unit, S._fmt(fmt)), (gt, gr)


def guarded_wpack(S, N, K, fmt):
    s = S.sharq_wpack_buffer_sizes(N, K, fmt)
    gt, gs = Guarded(s[0]), Guarded(s[1])
    return S.WPack(gt.view, gs.as_type(torch.float32, (s[1] // 4,)), N, K, S._fmt(fmt)), (gt, gs)


CASES = [(1, 256, 16), (200, 512, 272), (129, 768, 48)]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("T,K,N", CASES)
def test_no_writes_outside_buffers(fmt, T, K, N):
    S = require_gpu()
    rng = np.random.default_rng(T + K + N)
    x_bits = wl.outlier_activations(rng, T, K, 3, 20.0, 100.0, 0.5)
    w_bits = wl.weight(rng, N, K)
    g_bits = wl.rms_gamma(rng, K)
    x, w, g = to_dev_bf16(x_bits), to_dev_bf16(w_bits), to_dev_bf16(g_bits)
    guards = []
    wp, gw = guarded_wpack(S, N, K, fmt)
    S.sharq_pack_weight(w, fmt, out=wp)
    guards += gw
    for unit in (2, 1):
        p, gp = guarded_prep(S, T, K, unit, fmt)
        S.sharq_prepare(x, g, 1e-6, 2, 4, unit, fmt, out=p)
        guards += gp
        ref = hw.read_prep(S.sharq_prepare(x, g, 1e-6, 2, 4, unit, fmt), O.block_size(O.NVFP4 if fmt == 0 else O.MXFP4))
        got = hw.read_prep(p, O.block_size(O.NVFP4 if fmt == 0 else O.MXFP4))
        for key in ("idx", "sp_codes", "sp_scales", "res_codes", "res_scales", "row_scale"):
            assert np.array_equal(got[key], ref[key]), key
        if unit == 2:
            for dt, esz in ((torch.float32, 4), (torch.bfloat16, 2)):
                gy = Guarded(T * N * esz)
                y = gy.as_type(dt, (T, N))
                S.sharq_linear(p, wp, y=y)
                guards.append(gy)
                y0 = S.sharq_linear(p, wp, out_dtype=dt)
                torch.cuda.synchronize()
                assert torch.equal(y, y0)
    # gated input, per-tensor scale, dense baseline, separate RMSNorm
    gu = to_dev_bf16(wl.gate_up_activations(rng, T, K))
    p, gp = guarded_prep(S, T, K, 2, fmt)
    S.sharq_prepare_swiglu(gu, 2, 4, 2, fmt, out=p)
    guards += gp
    p, gp = guarded_prep(S, T, K, 2, fmt)
    gw = Guarded(S.sharq_tensor_scale_workspace_size(T, K))
    gw.view.zero_()
    S.sharq_prepare_tensor_scale(x, g, 1e-6, 2, 4, 2, fmt, out=p, workspace=gw.view)
    guards += list(gp) + [gw]
    s = S.sharq_dense_buffer_sizes(T, K, fmt)
    gt, gr = Guarded(s[0]), Guarded(s[1])
    q = S.DenseQ(gt.view, gr.as_type(torch.float32, (T,)), T, K, S._fmt(fmt))
    S.sharq_quantize_dense(x, g, 1e-6, fmt, out=q)
    gy = Guarded(T * N * 2)
    S.sharq_linear_dense(q, wp, y=gy.as_type(torch.bfloat16, (T, N)))
    guards += [gt, gr, gy]
    gn = Guarded(T * K * 2)
    S.sharq_rmsnorm(x, g, 1e-6, out=gn.as_type(torch.bfloat16, (T, K)))
    guards.append(gn)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    assert all(gd.intact() for gd in guards), [i for i, gd in enumerate(guards) if not gd.intact()]


def test_side_stream_after_slow_producer():
    S = require_gpu()
    lin = wl.llama_qkv(T=512)
    lin = wl.Linear("qkv_512x4096x1024", lin.x, None, lin.w[:1024])
    x_src = to_dev_bf16(lin.x)
    x = torch.zeros_like(x_src)
    wp = S.sharq_pack_weight(to_dev_bf16(lin.w), 0)
    p = S.alloc_prep(512, 4096)
    y = torch.empty(512, 1024, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        torch.cuda._sleep(20_000_000)  # a producer still running when the library's kernels are queued
        x.copy_(x_src)                 # ... which then writes their input
        S.sharq_prepare(x, None, 1e-6, out=p, stream=st)
        S.sharq_linear(p, wp, y=y, stream=st)
    st.synchronize()
    assert S.sharq_device_status(st) == S.SHARQ_OK
    ref = O.linear(O.prepare(f32(lin.x), None, 1e-6, 2, 4, 2, O.NVFP4), O.pack_weight(f32(lin.w), O.NVFP4))
    max_abs, frob = gemm_errors(y.cpu().numpy(), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)
