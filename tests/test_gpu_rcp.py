"""The preparation kernel's fast reciprocal (hardware approximation + one Markstein FMA step,
sharq_common.cuh rcp_rn) is checked bit for bit against CUDA's correctly rounded reciprocal over
every normal float32 with a normal reciprocal: the block-scale divisions the oracle performs
exactly (inv = fp32(1/d)) then hold in the kernel by construction, not only on test data."""
import os
import shutil
import subprocess
import tempfile

import pytest

from tests.gpu_common import require_gpu

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_rcp_rn_matches_correctly_rounded_reciprocal_exhaustively():
    require_gpu()
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "rcp_check")
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-o", exe,
                        os.path.join(HERE, "cuda", "rcp_check.cu")], check=True, capture_output=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    assert "status=no error" in out, out
    assert "mismatches=0 " in out, out
