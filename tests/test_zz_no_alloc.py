"""The per-tensor preparation entry point that allocates nothing (sharq_prepare_tensor_scale_noalloc),
for callers that may not allocate device memory and so cannot pass a workspace: its scratch is
the library's static device array. Through the C ABI, two calls in a row (different sizes, with
and without RMSNorm, so the second starts from the first call's leftovers in the shared array),
each compared with sharq_prepare_tensor_scale given a workspace: the same kernel runs on the same
inputs, so the tiled operand and the row scales must match byte for byte. This file sorts last so
that a run stopping at its first failure has run every other test first; it also passes alone in
a fresh process (the first call performs the per-device set-up)."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests.gpu_common import require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    S = require_gpu()
    rng = np.random.default_rng(2024)
    cases = [(300, 768, False), (2048, 4096, True)]
    for T, K, norm in cases:
        x = to_dev_bf16(wl.outlier_activations(rng, T, K, max(2, K // 100), 20.0, 100.0, 0.5))
        g = to_dev_bf16(wl.rms_gamma(rng, K)) if norm else None
        ref = S.alloc_prep(T, K)
        got = S.alloc_prep(T, K)
        ref.tiles.fill_(0x5A)  # bytes no call writes (chunk padding) compare equal
        got.tiles.fill_(0x5A)
        got.row_scale.fill_(-1.0)
        ws = torch.zeros(S.sharq_tensor_scale_workspace_size(T, K), dtype=torch.uint8, device="cuda")
        S.sharq_prepare_tensor_scale(x, g, 1e-6, out=ref, workspace=ws)
        S.sharq_prepare_tensor_scale_noalloc(x, g, 1e-6, out=got)
        torch.cuda.synchronize()
        assert S.sharq_device_status() == S.SHARQ_OK
        assert torch.equal(got.tiles, ref.tiles), (T, K, norm)
        assert torch.equal(got.row_scale, ref.row_scale), (T, K, norm)
        assert bool((got.row_scale == got.row_scale[0]).all())
