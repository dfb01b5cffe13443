"""Helpers shared by the GPU parity tests: device upload, oracle on the same inputs, tolerances."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import sharq as O
from tests import hwlayout as hw

FMT_NAME = {0: O.NVFP4, 1: O.MXFP4}


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    import fp4_activation_sparse_b200 as S  # raises if libsharq.so is missing
    return S


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32(bits):
    return None if bits is None else wl.bf16_bits_to_f32(bits)


# E2M1 codes in value order: index in this list = position on the signed grid
_ORDER = {c: i for i, c in enumerate([15, 14, 13, 12, 11, 10, 9, 0, 1, 2, 3, 4, 5, 6, 7])}
_ORDER[8] = _ORDER[0]  # -0 sits with +0


def code_steps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in grid steps between two arrays of E2M1 codes."""
    lut = np.array([_ORDER[c] for c in range(16)])
    return np.abs(lut[a] - lut[b])


def gemm_errors(y: np.ndarray, ref: np.ndarray):
    y = y.astype(np.float64)
    max_abs = np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30)
    frob = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-30)
    return max_abs, frob


# GEMM tolerances (same bound for every GEMM test): max |Y - Y64| <= 1e-4 max|Y64| and
# relative Frobenius error <= 1e-5, against the oracle's float64 GEMM.
MAX_ABS_TOL = 1e-4
FROB_TOL = 1e-5
