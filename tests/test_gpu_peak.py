"""The tensor-core peak loop (the GEMM's roofline denominator): every mode and format runs to
completion with a clean device status, and the timings hang together -- the SharQ K step
(sparse + dense MMAs) takes about as long as its two parts issued separately, and no rate
exceeds the part's nominal dense FP4 figure by more than the sparse factor of two."""
import pytest
import torch

from tests.gpu_common import require_gpu

pytestmark = pytest.mark.gpu

NOMINAL_DENSE_FP4_TFLOPS = 9000.0


def _time(S, mode, fmt, iters):
    S.sharq_mma_peak(mode, fmt, 256)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    S.sharq_mma_peak(mode, fmt, iters)
    b.record()
    b.synchronize()
    assert S.sharq_device_status() == S.SHARQ_OK
    return a.elapsed_time(b) / 1e3


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_peak_loop_modes(fmt):
    S = require_gpu()
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    iters = 8192
    t = {m: _time(S, m, fmt, iters) for m in (0, 1, 2)}
    rates = {m: S.MMA_PEAK_STEP_FLOPS[m] * iters * pairs / t[m] / 1e12 for m in t}
    print(fmt, {m: round(r) for m, r in rates.items()}, {m: round(v * 1e6) for m, v in t.items()})
    assert 0.7 * (t[0] + t[1]) < t[2] < 1.3 * (t[0] + t[1])
    assert rates[0] < 1.2 * NOMINAL_DENSE_FP4_TFLOPS
    assert rates[1] < 2.4 * NOMINAL_DENSE_FP4_TFLOPS
    assert min(rates.values()) > 500.0


def test_peak_loop_argument_checks():
    S = require_gpu()
    for bad in [(3, "nvfp4", 16), (0, "nvfp4", 0), (0, "nvfp4", (1 << 20) + 1)]:
        with pytest.raises(S.SharqError):
            S.sharq_mma_peak(*bad)
    S.sharq_mma_peak(2, "nvfp4", 64, clusters=3)
    assert S.sharq_device_status() == S.SHARQ_OK
