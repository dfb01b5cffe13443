"""The split-K form of the SharQ linear (sharq_linear_split) for launches with few output tiles:
against the oracle on sampled output columns (planted weight amax as in the shape tests), against
the plain launch (float32 rounding order only), the bf16 output rounded once after the sum, the
workspace size rule, the fallback when no slicing is called for, and guard bytes around the
workspace and the output."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests.gpu_common import FMT_NAME, FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16
from tests.test_gpu_canary import Guarded
from tests.test_gpu_shapes import planted

pytestmark = pytest.mark.gpu


def _problem(S, T, K, N, fmt, seed):
    rng = np.random.default_rng(seed)
    x_bits = wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5)
    cols = np.sort(rng.choice(N, min(N, 96), replace=False))
    w_bits = planted(wl.weight(rng, N, K), int(cols[0]))
    wp = S.sharq_pack_weight(to_dev_bf16(w_bits), fmt)
    p = S.sharq_prepare(to_dev_bf16(x_bits), None, 1e-6, 2, 4, 2, fmt)
    ref = O.linear(O.prepare(f32(x_bits), None, 1e-6, 2, 4, 2, FMT_NAME[fmt]),
                   O.pack_weight(f32(w_bits[cols]), FMT_NAME[fmt]))
    return p, wp, cols, ref


@pytest.mark.parametrize("T,K,N,fmt", [(1, 18944, 3584, 0), (16, 3584, 4608, 0), (128, 18944, 3584, 1),
                                       (3, 4096, 1024, 0)])
def test_split_matches_oracle_and_plain_launch(T, K, N, fmt):
    S = require_gpu()
    n_bytes = S.sharq_linear_workspace_size(T, N, K)
    assert n_bytes > 0 and n_bytes % (4 * T * N) == 0
    p, wp, cols, ref = _problem(S, T, K, N, fmt, T + K + N)
    gw, gy = Guarded(n_bytes), Guarded(T * N * 4)
    y = gy.as_type(torch.float32, (T, N))
    S.sharq_linear(p, wp, y=y, workspace=gw.view)
    y_plain = S.sharq_linear(p, wp, out_dtype=torch.float32)
    y_bf16 = S.sharq_linear(p, wp, out_dtype=torch.bfloat16, workspace=gw.view)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    assert gw.intact() and gy.intact()
    got = y.cpu().numpy()
    max_abs, frob = gemm_errors(got[:, cols], ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (max_abs, frob)
    plain = y_plain.cpu().numpy()
    assert np.abs(got - plain).max() <= 1e-5 * np.abs(plain).max()
    assert torch.equal(y_bf16, y.to(torch.bfloat16))  # the float32 sum, rounded once


def test_split_not_called_for_and_small_workspace():
    S = require_gpu()
    assert S.sharq_linear_workspace_size(2048, 6144, 4096) == 0  # enough tiles already
    assert S.sharq_linear_workspace_size(1, 16, 256) == 0        # one K step
    assert S.sharq_linear_workspace_size(256, 3584, 3584) == 0   # partials would cost more than slicing saves
    p, wp, cols, ref = _problem(S, 300, 512, 768, 0, 9)
    ws = torch.full((64,), 0x33, dtype=torch.uint8, device="cuda")
    y = S.sharq_linear(p, wp, out_dtype=torch.float32, workspace=ws)  # plain launch
    torch.cuda.synchronize()
    assert bool((ws == 0x33).all())
    assert torch.equal(y, S.sharq_linear(p, wp, out_dtype=torch.float32))
    p1, wp1, _, _ = _problem(S, 1, 18944, 3584, 0, 10)
    with pytest.raises(S.SharqError) as e:
        S.sharq_linear(p1, wp1, workspace=ws)
    assert e.value.status == S.SHARQ_ERR_INVALID_ARG
