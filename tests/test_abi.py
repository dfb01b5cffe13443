"""The C-ABI library loads, exports every symbol include/sharq.h declares, sizes its buffers
and rejects bad arguments on the host (no kernel launch; runs without a GPU)."""
import ctypes
import os
import re

import pytest

from fp4_activation_sparse_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def S():
    if not B.up_to_date():
        B.build()
    import fp4_activation_sparse_b200 as S
    return S


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sharq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sharq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(S):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(S.lib, n), n
        assert ctypes.cast(getattr(S.lib, n), ctypes.c_void_p).value


def test_version(S):
    assert S.lib.sharq_version() == 200


def test_prep_buffer_sizes(S):
    """Chunks of 128 rows x 256 K over tokens padded to 256, sizes from the header's table."""
    T, K = 300, 4096
    chunks = (512 // 128) * (K // 256)
    assert S.sharq_prep_buffer_sizes(T, K, 2, 4, 2, "nvfp4") == [chunks * 29696, T * 4]
    assert S.sharq_prep_buffer_sizes(T, K, 2, 4, 2, "mxfp4") == [chunks * 28672, T * 4]
    assert S.sharq_prep_buffer_sizes(T, K, 2, 4, 1, "nvfp4") == [chunks * 31744, T * 4]
    assert S.sharq_prep_buffer_sizes(T, K, 2, 4, 1, "mxfp4") == [chunks * 30720, T * 4]
    assert S.sharq_dense_buffer_sizes(T, K, "nvfp4") == [chunks * 18432, T * 4]
    assert S.sharq_dense_buffer_sizes(T, K, "mxfp4") == [chunks * 17408, T * 4]


def test_prep_buffer_sizes_4of8(S):
    # four of eight elements: 48 metadata bytes per row per K step (6144 per chunk)
    assert S.sharq_prep_buffer_sizes(300, 512, 4, 8, 1, "nvfp4") == [(512 // 128) * 2 * 33792, 1200]
    assert S.sharq_prep_buffer_sizes(300, 512, 4, 8, 1, "mxfp4") == [(512 // 128) * 2 * 32768, 1200]


def test_wpack_buffer_sizes(S):
    assert S.sharq_wpack_buffer_sizes(6144, 4096, "nvfp4") == [(6144 // 128) * 16 * 22528, 8]
    assert S.sharq_wpack_buffer_sizes(208, 256, "mxfp4") == [(256 // 128) * 1 * 19456, 8]


@pytest.mark.parametrize("args,status", [
    ((0, 4096, 2, 4, 2, 0), 1),     # no tokens
    ((16, 4000, 2, 4, 2, 0), 1),    # k not a multiple of 256
    ((16, 4096, 3, 2, 2, 0), 1),    # N > M
    ((16, 4096, 2, 4, 3, 0), 1),    # bad unit
    ((16, 4096, 2, 4, 2, 7), 1),    # bad format
    ((16, 4096, 1, 4, 2, 0), 2),    # valid pattern the library does not compute
    ((16, 4096, 4, 8, 2, 0), 2),    # 4:8 over pairs: not computed (4:8 is over elements)
])
def test_prep_sizes_reject(S, args, status):
    sizes = (ctypes.c_size_t * 2)()
    assert S.lib.sharq_prep_buffer_sizes(*args, sizes) == 0
    assert S.last_error()


def test_calls_reject_bad_arguments_before_launch(S):
    P = S._Prep()
    W = S._WPack()
    null = ctypes.c_void_p(0)
    # null input
    assert S.lib.sharq_prepare(None, 16, 4096, None, 1e-6, 2, 4, 2, 0, ctypes.byref(P), null) == S.SHARQ_ERR_INVALID_ARG
    # misaligned input pointer
    assert S.lib.sharq_prepare(ctypes.c_void_p(0x1008), 16, 4096, None, 1e-6, 2, 4, 2, 0, ctypes.byref(P),
                               null) == S.SHARQ_ERR_INVALID_ARG
    # unsupported pattern
    assert S.lib.sharq_prepare(ctypes.c_void_p(0x1000), 16, 4096, None, 1e-6, 1, 4, 2, 0, ctypes.byref(P),
                               null) == S.SHARQ_ERR_UNSUPPORTED
    # null output buffers in the struct
    assert S.lib.sharq_prepare(ctypes.c_void_p(0x1000), 16, 4096, None, 1e-6, 2, 4, 2, 0, ctypes.byref(P),
                               null) == S.SHARQ_ERR_INVALID_ARG
    # weight pack: bad n_out
    assert S.lib.sharq_pack_weight(ctypes.c_void_p(0x1000), 20, 4096, 0, ctypes.byref(W), null) == S.SHARQ_ERR_INVALID_ARG
    # linear: mismatched formats / k / element pattern
    P2 = S._Prep(0x1000, 0x1000, 16, 4096, 2, 4, 2, 0)
    W2 = S._WPack(0x1000, 0x1000, 256, 4096, 1)
    assert S.lib.sharq_linear(ctypes.byref(P2), ctypes.byref(W2), ctypes.c_void_p(0x1000), 0, null) == S.SHARQ_ERR_INVALID_ARG
    assert "format mismatch" in S.last_error()
    W2.fmt, W2.k = 0, 2048
    assert S.lib.sharq_linear(ctypes.byref(P2), ctypes.byref(W2), ctypes.c_void_p(0x1000), 0, null) == S.SHARQ_ERR_INVALID_ARG
    W2.k, P2.unit = 4096, 1
    assert S.lib.sharq_linear(ctypes.byref(P2), ctypes.byref(W2), ctypes.c_void_p(0x1000), 0, null) == S.SHARQ_ERR_UNSUPPORTED
    assert S.lib.sharq_linear(ctypes.byref(P2), None, ctypes.c_void_p(0x1000), 0, null) == S.SHARQ_ERR_INVALID_ARG
    P2.unit = 2
    assert S.lib.sharq_linear(ctypes.byref(P2), ctypes.byref(W2), ctypes.c_void_p(0x1000), 5, null) == S.SHARQ_ERR_INVALID_ARG
    assert S.lib.sharq_linear_dense(None, None, 16, 4096, ctypes.byref(W2), None, 0, null) == S.SHARQ_ERR_INVALID_ARG
