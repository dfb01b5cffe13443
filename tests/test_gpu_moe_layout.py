"""The mixture-of-experts layer in the benchmark's own launch configuration: Qwen3-30B-A3B experts
(K=2048, N=2*768), 2048 tokens routed top-8 of 128, the routed rows laid out expert by expert
(each expert padded to 128 rows, 256 rows of slack at the end), ONE sharq_prepare over all of
them, and every expert's view of that buffer in grouped launches (64 experts each, single-CTA
tiles). Sampled experts (the smallest, the largest, some in between) are checked against the
oracle on their own rows; every expert's output is checked to be finite."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests.gpu_common import FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_moe_bench_layout_against_oracle():
    S = require_gpu()
    moe = wl.QWEN3_MOE
    K, N, E, T = moe["hidden"], 2 * moe["moe_intermediate"], moe["n_experts"], 2048
    route = wl.moe_routing(11, T, E, moe["top_k"])
    counts = np.bincount(route.reshape(-1), minlength=E)
    starts = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)])[:-1]
    rows_pad = int(starts[-1] + (counts[-1] + 127) // 128 * 128)
    order = np.argsort(route.reshape(-1), kind="stable")
    src_tok = order // moe["top_k"]
    x_tok = wl.outlier_activations(np.random.default_rng(12), T, K, K // 100, 20.0, 100.0, 0.5)
    x_rows = np.zeros((rows_pad, K), np.uint16)
    dst = np.concatenate([starts[e] + np.arange(counts[e]) for e in range(E)])
    x_rows[dst] = x_tok[src_tok]
    p_all = S.alloc_prep(rows_pad + 256, K)
    p_all.tokens, p_all.row_scale = rows_pad, p_all.row_scale[:rows_pad]
    S.sharq_prepare(to_dev_bf16(x_rows), None, 1e-6, out=p_all)
    chunk = S.sharq_prep_buffer_sizes(256, K, 2, 4, 2, "nvfp4")[0] // 2
    views = [S.Prep(p_all.tiles[int(starts[e]) // 128 * chunk:], p_all.row_scale[int(starts[e]):], int(counts[e]), K,
                    2, 4, 2, S.SHARQ_NVFP4) for e in range(E)]
    nz = np.flatnonzero(counts)
    picks = sorted({int(nz[np.argmin(counts[nz])]), int(np.argmax(counts)), int(nz[len(nz) // 3]),
                    int(nz[2 * len(nz) // 3])})
    rng = np.random.default_rng(13)
    w_bits = {e: wl.weight(rng, N, K) for e in picks}
    gen = torch.Generator(device="cuda").manual_seed(14)
    wps = [S.sharq_pack_weight(to_dev_bf16(w_bits[e]) if e in w_bits else
                               (torch.randn(N, K, device="cuda", generator=gen) * 0.02).to(torch.bfloat16))
           for e in range(E)]
    ys = [torch.empty(max(int(c), 1), N, dtype=torch.float32, device="cuda") for c in counts]
    S.sharq_linear_grouped(views, wps, ys)
    torch.cuda.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    for e in range(E):
        if counts[e]:
            assert bool(torch.isfinite(ys[e][:counts[e]]).all()), e
    for e in picks:
        rows = x_rows[starts[e]:starts[e] + counts[e]]
        ref = O.linear(O.prepare(f32(rows), None, 1e-6, 2, 4, 2, O.NVFP4), O.pack_weight(f32(w_bits[e]), O.NVFP4))
        max_abs, frob = gemm_errors(ys[e][:counts[e]].cpu().numpy(), ref)
        assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL, (e, int(counts[e]), max_abs, frob)
