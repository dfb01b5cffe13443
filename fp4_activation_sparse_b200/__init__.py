"""Python binding of libsharq: SharQ's online sparse-dense FP4 linear layer on B200.

Argument marshalling only (ctypes). Every computation runs in the library's CUDA
kernels; torch supplies device memory and streams. There is no CPU fallback: the
library is loaded on first use (so that ``fp4_activation_sparse_b200.build`` can run on
a fresh tree), and every call raises ImportError if ``libsharq.so`` is missing or does
not export what this binding expects.

The three calls of the method ("SharQ: Bridging Activation Sparsity and FP4
Quantization for LLM Inference", Abstract):
  sharq_pack_weight  - one FP4 weight payload with sparse-path and dense-path scale views
  sharq_prepare      - the fused preparation operator (RMSNorm, N:M mask, FP4 backbone,
                       residual against the quantized backbone, dense FP4 residual)
  sharq_prepare_swiglu - the same operator on a down projection's gated input SiLU(g)*u
  sharq_prepare_tensor_scale - the same operator with one NVFP4 second-level scale per tensor
  sharq_linear       - sparse FP4 GEMM + dense FP4 GEMM into one output
  sharq_linear_grouped - the same for many experts (mixture of experts) in one launch
and the library's dense FP4 baseline (the README's "NVFP4" mode):
  sharq_quantize_dense, sharq_linear_dense.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsharq.so")

SHARQ_NVFP4, SHARQ_MXFP4 = 0, 1
SHARQ_OUT_BF16, SHARQ_OUT_F32 = 0, 1
SHARQ_OK, SHARQ_ERR_INVALID_ARG, SHARQ_ERR_UNSUPPORTED, SHARQ_ERR_CUDA, SHARQ_ERR_TIMEOUT = range(5)
FMT = {"nvfp4": SHARQ_NVFP4, "mxfp4": SHARQ_MXFP4}
UNIT_ELEMENT, UNIT_PAIR = 1, 2


class SharqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"sharq status {status}: {message}")
        self.status = status


class _Prep(ctypes.Structure):
    _fields_ = [("tiles", ctypes.c_void_p), ("row_scale", ctypes.c_void_p),
                ("tokens", ctypes.c_int), ("k", ctypes.c_int), ("nm_n", ctypes.c_int),
                ("nm_m", ctypes.c_int), ("unit", ctypes.c_int), ("fmt", ctypes.c_int)]


class _WPack(ctypes.Structure):
    _fields_ = [("tiles", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("n_out", ctypes.c_int), ("k", ctypes.c_int), ("fmt", ctypes.c_int)]


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m fp4_activation_sparse_b200.build`")
    lib = ctypes.CDLL(path)
    if not hasattr(lib, "sharq_dense_buffer_sizes"):
        raise ImportError(f"{path} is stale (ABI older than this binding): rebuild it")
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "sharq_prep_buffer_sizes": (S, [I, I, I, I, I, I, ctypes.POINTER(S)]),
        "sharq_dense_buffer_sizes": (S, [I, I, I, ctypes.POINTER(S)]),
        "sharq_wpack_buffer_sizes": (S, [I, I, I, ctypes.POINTER(S)]),
        "sharq_pack_weight": (I, [P, I, I, I, ctypes.POINTER(_WPack), P]),
        "sharq_prepare": (I, [P, I, I, P, F, I, I, I, I, ctypes.POINTER(_Prep), P]),
        "sharq_prepare_tensor_scale_noalloc": (I, [P, I, I, P, F, I, I, I, I, ctypes.POINTER(_Prep), P]),
        "sharq_prepare_swiglu": (I, [P, I, I, I, I, I, I, ctypes.POINTER(_Prep), P]),
        "sharq_tensor_scale_workspace_size": (S, [I, I]),
        "sharq_prepare_tensor_scale": (I, [P, I, I, P, F, I, I, I, I, ctypes.POINTER(_Prep), P, P]),
        "sharq_linear": (I, [ctypes.POINTER(_Prep), ctypes.POINTER(_WPack), P, I, P]),
        "sharq_linear_workspace_size": (S, [I, I, I]),
        "sharq_linear_split": (I, [ctypes.POINTER(_Prep), ctypes.POINTER(_WPack), P, I, P, S, P]),
        "sharq_linear_grouped": (I, [ctypes.POINTER(_Prep), ctypes.POINTER(_WPack), ctypes.POINTER(P), I, I, P]),
        "sharq_quantize_dense": (I, [P, I, I, P, F, I, P, P, P]),
        "sharq_linear_dense": (I, [P, P, I, I, ctypes.POINTER(_WPack), P, I, P]),
        "sharq_rmsnorm": (I, [P, I, I, P, F, P, P]),
        "sharq_mma_peak": (I, [I, I, I, I, P]),
        "sharq_device_status": (I, [P]),
        "sharq_set_wait_limit": (None, [ctypes.c_longlong]),
        "sharq_last_error": (ctypes.c_char_p, []),
        "sharq_version": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


class _Lib:
    """The loaded libsharq.so, opened on first attribute access."""
    _cdll: ctypes.CDLL | None = None

    def __getattr__(self, name):
        if _Lib._cdll is None:
            _Lib._cdll = _load()
        return getattr(_Lib._cdll, name)


lib = _Lib()


def load() -> ctypes.CDLL:
    """Open libsharq.so now (raises ImportError if it is missing or stale)."""
    lib.sharq_version  # noqa: B018  (attribute access loads the library)
    return _Lib._cdll


def last_error() -> str:
    return lib.sharq_last_error().decode()


def _check(status: int):
    if status != SHARQ_OK:
        raise SharqError(status, last_error())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _fmt(fmt) -> int:
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


# ------------------------------------------------------------------ buffer holders
@dataclass
class Prep:
    """A prepared activation: the tiled operand, the row scales and the C struct."""
    tiles: torch.Tensor
    row_scale: torch.Tensor
    tokens: int
    k: int
    nm_n: int
    nm_m: int
    unit: int
    fmt: int
    c: _Prep = field(default=None, repr=False)

    def struct(self) -> _Prep:
        if self.c is None:
            self.c = _Prep(self.tiles.data_ptr(), self.row_scale.data_ptr(), self.tokens, self.k, self.nm_n,
                           self.nm_m, self.unit, self.fmt)
        return self.c


@dataclass
class WPack:
    """A packed weight: the tiled operand (codes and both scale views) and the tensor scale."""
    tiles: torch.Tensor
    tensor_scale: torch.Tensor
    n_out: int
    k: int
    fmt: int
    c: _WPack = field(default=None, repr=False)

    def struct(self) -> _WPack:
        if self.c is None:
            self.c = _WPack(self.tiles.data_ptr(), self.tensor_scale.data_ptr(), self.n_out, self.k, self.fmt)
        return self.c


def _sizes(fn, *args) -> list[int]:
    sizes = (ctypes.c_size_t * 2)()
    if fn(*args, sizes) == 0:
        raise SharqError(SHARQ_ERR_INVALID_ARG, last_error())
    return list(sizes)


def sharq_prep_buffer_sizes(tokens: int, k: int, nm_n: int, nm_m: int, unit: int, fmt) -> list[int]:
    return _sizes(lib.sharq_prep_buffer_sizes, tokens, k, nm_n, nm_m, unit, _fmt(fmt))


def sharq_dense_buffer_sizes(tokens: int, k: int, fmt) -> list[int]:
    return _sizes(lib.sharq_dense_buffer_sizes, tokens, k, _fmt(fmt))


def sharq_wpack_buffer_sizes(n_out: int, k: int, fmt) -> list[int]:
    return _sizes(lib.sharq_wpack_buffer_sizes, n_out, k, _fmt(fmt))


def _bytes(n: int, device) -> torch.Tensor:
    # 16-byte aligned (torch's caching allocator aligns to 512 bytes)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def alloc_prep(tokens: int, k: int, nm_n: int = 2, nm_m: int = 4, unit: int = UNIT_PAIR, fmt="nvfp4",
               device="cuda") -> Prep:
    s = sharq_prep_buffer_sizes(tokens, k, nm_n, nm_m, unit, fmt)
    return Prep(_bytes(s[0], device), torch.empty(tokens, dtype=torch.float32, device=device),
                tokens, k, nm_n, nm_m, unit, _fmt(fmt))


def alloc_wpack(n_out: int, k: int, fmt="nvfp4", device="cuda") -> WPack:
    s = sharq_wpack_buffer_sizes(n_out, k, fmt)
    return WPack(_bytes(s[0], device), torch.empty(4, dtype=torch.float32, device=device), n_out, k, _fmt(fmt))


# ------------------------------------------------------------------ the calls
def sharq_pack_weight(w: torch.Tensor, fmt="nvfp4", out: WPack | None = None, stream=None) -> WPack:
    """Pack a bf16 weight [n_out, k] (device) into one FP4 payload with two scale views."""
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    n_out, k = w.shape
    out = out or alloc_wpack(n_out, k, fmt, w.device)
    st = out.struct()
    _check(lib.sharq_pack_weight(_ptr(w), n_out, k, _fmt(fmt), ctypes.byref(st), _stream(stream)))
    return out


def sharq_prepare(x: torch.Tensor, gamma: torch.Tensor | None = None, eps: float = 1e-6, nm_n: int = 2,
                  nm_m: int = 4, unit: int = UNIT_PAIR, fmt="nvfp4", out: Prep | None = None, stream=None) -> Prep:
    """The fused preparation operator on bf16 activations [tokens, k] (device)."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    tokens, k = x.shape
    if gamma is not None:
        assert gamma.dtype == torch.bfloat16 and gamma.is_cuda and gamma.numel() == k
    out = out or alloc_prep(tokens, k, nm_n, nm_m, unit, fmt, x.device)
    st = out.struct()
    _check(lib.sharq_prepare(_ptr(x), tokens, k, _ptr(gamma), ctypes.c_float(eps), nm_n, nm_m, unit, _fmt(fmt),
                             ctypes.byref(st), _stream(stream)))
    return out


def sharq_tensor_scale_workspace_size(tokens: int, k: int) -> int:
    n = lib.sharq_tensor_scale_workspace_size(tokens, k)
    if n == 0:
        raise SharqError(SHARQ_ERR_INVALID_ARG, last_error())
    return n


def sharq_prepare_tensor_scale(x: torch.Tensor, gamma: torch.Tensor | None = None, eps: float = 1e-6,
                               nm_n: int = 2, nm_m: int = 4, unit: int = UNIT_PAIR, fmt="nvfp4",
                               out: Prep | None = None, workspace: torch.Tensor | None = None,
                               stream=None) -> Prep:
    """sharq_prepare with one NVFP4 second-level scale for the whole tensor (every row_scale
    entry holds it). One cooperative launch; `workspace` carries its grid barrier: device bytes
    zeroed once before first use (allocated zeroed here if omitted), reusable afterwards."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    tokens, k = x.shape
    if gamma is not None:
        assert gamma.dtype == torch.bfloat16 and gamma.is_cuda and gamma.numel() == k
    out = out or alloc_prep(tokens, k, nm_n, nm_m, unit, fmt, x.device)
    if workspace is None:
        workspace = torch.zeros(sharq_tensor_scale_workspace_size(tokens, k), dtype=torch.uint8, device=x.device)
    st = out.struct()
    _check(lib.sharq_prepare_tensor_scale(_ptr(x), tokens, k, _ptr(gamma), ctypes.c_float(eps), nm_n, nm_m, unit,
                                          _fmt(fmt), ctypes.byref(st), _ptr(workspace), _stream(stream)))
    return out


def sharq_prepare_tensor_scale_noalloc(x: torch.Tensor, gamma: torch.Tensor | None = None, eps: float = 1e-6,
                                       nm_n: int = 2, nm_m: int = 4, unit: int = UNIT_PAIR, fmt="nvfp4",
                                       out: Prep | None = None, stream=None) -> Prep:
    """sharq_prepare_tensor_scale without a workspace: for callers that may not allocate device
    memory, the library's own static scratch carries the grid barrier (calls that overlap on the
    GPU race on it). Only the output holder is allocated here, and only if `out` is omitted."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    tokens, k = x.shape
    if gamma is not None:
        assert gamma.dtype == torch.bfloat16 and gamma.is_cuda and gamma.numel() == k
    out = out or alloc_prep(tokens, k, nm_n, nm_m, unit, fmt, x.device)
    st = out.struct()
    _check(lib.sharq_prepare_tensor_scale_noalloc(_ptr(x), tokens, k, _ptr(gamma), ctypes.c_float(eps), nm_n, nm_m,
                                                  unit, _fmt(fmt), ctypes.byref(st), _stream(stream)))
    return out


def sharq_prepare_swiglu(gate_up: torch.Tensor, nm_n: int = 2, nm_m: int = 4, unit: int = UNIT_PAIR,
                         fmt="nvfp4", out: Prep | None = None, stream=None) -> Prep:
    """The preparation operator on a down projection's gated input x = SiLU(g) * u, formed in
    registers from the gate/up output [tokens, 2k] = [g | u] (bf16, device)."""
    assert gate_up.dtype == torch.bfloat16 and gate_up.is_cuda and gate_up.is_contiguous()
    tokens, k2 = gate_up.shape
    assert k2 % 2 == 0
    k = k2 // 2
    out = out or alloc_prep(tokens, k, nm_n, nm_m, unit, fmt, gate_up.device)
    st = out.struct()
    _check(lib.sharq_prepare_swiglu(_ptr(gate_up), tokens, k, nm_n, nm_m, unit, _fmt(fmt), ctypes.byref(st),
                                    _stream(stream)))
    return out


def sharq_linear(prep: Prep, w: WPack, y: torch.Tensor | None = None, out_dtype=torch.bfloat16,
                 stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Y [tokens, n_out] = sparse FP4 GEMM (backbone) + dense FP4 GEMM (residual), one output.
    With `workspace` (device bytes, sharq_linear_workspace_size) the split-K form runs where the
    shape calls for it (sharq_linear_split)."""
    if y is None:
        y = torch.empty(prep.tokens, w.n_out, dtype=out_dtype, device=prep.tiles.device)
    code = SHARQ_OUT_F32 if y.dtype == torch.float32 else SHARQ_OUT_BF16
    if workspace is not None:
        _check(lib.sharq_linear_split(ctypes.byref(prep.struct()), ctypes.byref(w.struct()), _ptr(y), code,
                                      _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    else:
        _check(lib.sharq_linear(ctypes.byref(prep.struct()), ctypes.byref(w.struct()), _ptr(y), code,
                                _stream(stream)))
    return y


def sharq_linear_workspace_size(tokens: int, n_out: int, k: int) -> int:
    """Bytes of workspace the split-K form of sharq_linear wants for this shape (0: none)."""
    return int(lib.sharq_linear_workspace_size(tokens, n_out, k))


def sharq_linear_grouped(preps: list[Prep], ws: list[WPack], ys: list[torch.Tensor] | None = None,
                         out_dtype=torch.bfloat16, stream=None) -> list[torch.Tensor]:
    """Mixture-of-experts form: Y_e = sharq_linear(preps[e], ws[e]) for every expert in one
    launch (per 64 experts). Every weight shares n_out and k."""
    n = len(preps)
    assert n == len(ws) and n >= 1
    if ys is None:
        ys = [torch.empty(p.tokens, w.n_out, dtype=out_dtype, device=p.tiles.device) for p, w in zip(preps, ws)]
    code = SHARQ_OUT_F32 if ys[0].dtype == torch.float32 else SHARQ_OUT_BF16
    a = (_Prep * n)(*[p.struct() for p in preps])
    w = (_WPack * n)(*[x.struct() for x in ws])
    y = (ctypes.c_void_p * n)(*[t.data_ptr() for t in ys])
    _check(lib.sharq_linear_grouped(a, w, y, n, code, _stream(stream)))
    return ys


@dataclass
class DenseQ:
    """A dense-quantized activation: the tiled operand and the row scales."""
    tiles: torch.Tensor
    row_scale: torch.Tensor
    tokens: int
    k: int
    fmt: int


def sharq_quantize_dense(x: torch.Tensor, gamma: torch.Tensor | None = None, eps: float = 1e-6, fmt="nvfp4",
                         out: DenseQ | None = None, stream=None) -> DenseQ:
    """The dense FP4 baseline quantizer (optional RMSNorm + block quantization of every element)."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
    tokens, k = x.shape
    if out is None:
        s = sharq_dense_buffer_sizes(tokens, k, fmt)
        out = DenseQ(_bytes(s[0], x.device), torch.empty(tokens, dtype=torch.float32, device=x.device), tokens, k,
                     _fmt(fmt))
    _check(lib.sharq_quantize_dense(_ptr(x), tokens, k, _ptr(gamma), ctypes.c_float(eps), _fmt(fmt),
                                    _ptr(out.tiles), _ptr(out.row_scale), _stream(stream)))
    return out


def sharq_linear_dense(q: DenseQ, w: WPack, y: torch.Tensor | None = None, out_dtype=torch.bfloat16,
                       stream=None) -> torch.Tensor:
    """The dense FP4 baseline GEMM against the weight's dense-path scale view."""
    if y is None:
        y = torch.empty(q.tokens, w.n_out, dtype=out_dtype, device=q.tiles.device)
    code = SHARQ_OUT_F32 if y.dtype == torch.float32 else SHARQ_OUT_BF16
    _check(lib.sharq_linear_dense(_ptr(q.tiles), _ptr(q.row_scale), q.tokens, q.k, ctypes.byref(w.struct()),
                                  _ptr(y), code, _stream(stream)))
    return y


def sharq_rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """The dense baseline's separate RMSNorm pass: y = bf16(fp32(fp32(x*rstd)*gamma))."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous() and gamma.dtype == torch.bfloat16
    tokens, k = x.shape
    out = torch.empty_like(x) if out is None else out
    _check(lib.sharq_rmsnorm(_ptr(x), tokens, k, _ptr(gamma), float(eps), _ptr(out), _stream(stream)))
    return out


# flops one K step of one CTA pair performs in sharq_mma_peak, per mode: dense; sparse (logical,
# counting the dropped half as NVIDIA's sparse peaks do); both, in sharq_linear's dense-equivalent
# units (3 * 256^3: the dense path over all of K plus the sparse path over its kept half)
MMA_PEAK_STEP_FLOPS = {0: 2.0 * 256 ** 3, 1: 2.0 * 256 ** 3, 2: 3.0 * 256 ** 3}


def sharq_mma_peak(mode: int, fmt="nvfp4", iters: int = 65536, clusters: int = 0, stream=None) -> None:
    """Launch the tensor-core peak loop (mode 0 dense, 1 sparse, 2 both); the caller times it."""
    _check(lib.sharq_mma_peak(int(mode), _fmt(fmt), int(iters), int(clusters), _stream(stream)))


def sharq_device_status(stream=None) -> int:
    """Synchronize the stream; return (and clear) the status of the bounded device waits."""
    return lib.sharq_device_status(_stream(stream))


def sharq_set_wait_limit(nanoseconds: int) -> None:
    """Test hook: time limit of the library's bounded device waits (0 restores the default of 4 s)."""
    lib.sharq_set_wait_limit(int(nanoseconds))
