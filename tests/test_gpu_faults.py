"""Failure detection without a GPU fault: the GEMM's bounded waits give up, report a
status the host reads, and leave the context usable.

The wait limit is lowered to 1 ns through the library's test hook, so the waits give
up while data is still arriving; the kernel then drains its own copies and MMAs
(with the full bound), frees its tensor memory and returns. Nothing traps or hangs.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw
from tests.gpu_common import FROB_TOL, MAX_ABS_TOL, f32, gemm_errors, require_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_context_survives():
    S = require_gpu()
    lin = wl.llama_qkv(T=256)
    lin = wl.Linear("qkv_256x4096x512", lin.x, None, lin.w[:512])
    x, w = to_dev_bf16(lin.x), to_dev_bf16(lin.w)
    wp = S.sharq_pack_weight(w, 0)
    p = S.sharq_prepare(x, None, 1e-6, 2, 4, 2, 0)
    assert S.sharq_device_status() == S.SHARQ_OK
    try:
        S.sharq_set_wait_limit(1)
        S.sharq_linear(p, wp, out_dtype=torch.float32)
        assert S.sharq_device_status() == S.SHARQ_ERR_TIMEOUT
    finally:
        S.sharq_set_wait_limit(0)
    # the status word was cleared and the context still works
    y = S.sharq_linear(p, wp, out_dtype=torch.float32)
    assert S.sharq_device_status() == S.SHARQ_OK
    ref = O.linear(O.prepare(f32(lin.x), None, 1e-6, 2, 4, 2, O.NVFP4), O.pack_weight(f32(lin.w), O.NVFP4))
    max_abs, frob = gemm_errors(hw.to_np(y), ref)
    assert max_abs <= MAX_ABS_TOL and frob <= FROB_TOL


def test_invalid_arguments_raise_without_launch():
    S = require_gpu()
    x = torch.zeros(16, 300, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SharqError) as e:
        S.sharq_prepare(x)
    assert e.value.status == S.SHARQ_ERR_INVALID_ARG
    x = torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda")
    p = S.sharq_prepare(x, unit=1)
    wp = S.sharq_pack_weight(torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(S.SharqError) as e:
        S.sharq_linear(p, wp)
    assert e.value.status == S.SHARQ_ERR_UNSUPPORTED
    wp_mx = S.sharq_pack_weight(torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda"), "mxfp4")
    with pytest.raises(S.SharqError) as e:
        S.sharq_linear(S.sharq_prepare(x), wp_mx)
    assert e.value.status == S.SHARQ_ERR_INVALID_ARG
    assert S.sharq_device_status() == S.SHARQ_OK
