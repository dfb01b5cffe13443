"""Parity of the grouped (mixture-of-experts) SharQ linear with the CPU oracle, expert by expert,
including experts without tokens, ragged token counts and more experts than one launch takes."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests.gpu_common import FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def _experts(S, rng, counts, K, N, fmt):
    preps, wps, refs = [], [], []
    for t in counts:
        w_bits = wl.weight(rng, N, K)
        wp = S.sharq_pack_weight(to_dev_bf16(w_bits), fmt)
        if t == 0:
            p = S.alloc_prep(1, K, 2, 4, 2, fmt)   # buffers unused: tokens = 0 marks an idle expert
            p.tokens = 0
            refs.append(None)
        else:
            x_bits = wl.outlier_activations(rng, t, K, max(2, K // 100), 20.0, 100.0, 0.5)
            p = S.sharq_prepare(to_dev_bf16(x_bits), None, 1e-6, 2, 4, 2, fmt)
            name = O.NVFP4 if fmt == 0 else O.MXFP4
            refs.append(O.linear(O.prepare(f32(x_bits), None, 1e-6, 2, 4, 2, name), O.pack_weight(f32(w_bits), name)))
        preps.append(p)
        wps.append(wp)
    return preps, wps, refs


@pytest.mark.parametrize("fmt", [0, 1])
def test_grouped_matches_oracle_and_single_launches(fmt):
    S = require_gpu()
    rng = np.random.default_rng(40 + fmt)
    counts, K, N = [0, 37, 256, 300, 513], 512, 384
    preps, wps, refs = _experts(S, rng, counts, K, N, fmt)
    ys = [torch.empty(max(t, 1), N, dtype=torch.float32, device="cuda") for t in counts]
    S.sharq_linear_grouped(preps, wps, ys)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    for e, t in enumerate(counts):
        if t == 0:
            continue
        y = ys[e][:t].cpu().numpy()
        max_abs, frob = gemm_errors(y, refs[e])
        assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (e, max_abs, frob)
        single = S.sharq_linear(preps[e], wps[e], out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(single, ys[e][:t]), e  # same tiles, same arithmetic


def test_grouped_more_groups_than_one_launch_bf16():
    S = require_gpu()
    rng = np.random.default_rng(50)
    counts = [int(c) for c in rng.integers(0, 300, size=40)]
    counts[3] = 0
    K, N = 256, 256
    preps, wps, refs = _experts(S, rng, counts, K, N, 0)
    ys = S.sharq_linear_grouped(preps, wps, [torch.empty(max(t, 1), N, dtype=torch.bfloat16, device="cuda")
                                             for t in counts])
    torch.cuda.synchronize()
    for e, t in enumerate(counts):
        if t == 0:
            continue
        y32 = S.sharq_linear(preps[e], wps[e], out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(ys[e][:t], y32.to(torch.bfloat16)), e  # bf16 = RNE of the fp32 output
        max_abs, frob = gemm_errors(y32.cpu().numpy(), refs[e])
        assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (e, max_abs, frob)


def test_grouped_rejects_mismatched_weights():
    S = require_gpu()
    rng = np.random.default_rng(60)
    preps, wps, _ = _experts(S, rng, [64, 64], 256, 256, 0)
    wps[1] = S.sharq_pack_weight(to_dev_bf16(wl.weight(rng, 512, 256)), 0)  # other n_out
    with pytest.raises(S.SharqError):
        S.sharq_linear_grouped(preps, wps, [torch.empty(64, 256, dtype=torch.bfloat16, device="cuda")] * 2)
