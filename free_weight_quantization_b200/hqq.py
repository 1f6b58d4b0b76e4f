"""Python binding of the C ABI in include/hqq_b200.h (argument marshalling only).

Every step of quantize and dequantize runs in the CUDA kernels of libhqq_b200.so; this module
allocates output buffers with torch when the caller does not pass them, hands raw device
pointers and the current CUDA stream to the library, and raises on a non-zero return code.
There is no CPU fallback: loading fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhqq_b200.so")

HQQ_OK = 0
HQQ_MAX_GROUP_SIZE = 256
HQQ_MAX_ITERS = 64


class HqqOpt(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_int32), ("lp_norm", ctypes.c_double),
                ("beta", ctypes.c_double), ("kappa", ctypes.c_double),
                ("eps_tiny", ctypes.c_float), ("scale_max", ctypes.c_float)]


class HqqError(RuntimeError):
    pass


_lib = None

# (name, restype, argtypes) of every symbol the header declares
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "hqq_default_opt": (None, [ctypes.POINTER(HqqOpt)]),
    "hqq_packed_bytes": (_I64, [_I64, _I32]),
    "hqq_quantize_workspace_bytes": (_SZ, [_I64, _I64, _I32, _I64, _I32, _I32]),
    "hqq_quantize": (_I32, [_P, _I64, _I64, _I32, _I64, _I32, ctypes.POINTER(HqqOpt), _P, _P, _P,
                            _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "hqq_dequantize": (_I32, [_P, _P, _P, _I64, _I64, _I32, _I64, _I32, _P, _P]),
    "hqq_quantize_noalloc": (_I32, [_P, _I64, _I64, _I32, _I64, _I32, ctypes.POINTER(HqqOpt), _P,
                                    _P, _P, _P, _P, _P, _P, _P, _P]),
    "hqq_gemv": (_I32, [_P, _P, _P, _I64, _I64, _I32, _I64, _I32, _P, _P, _P]),
    "hqq_gemm": (_I32, [_P, _P, _P, _I64, _I64, _I32, _I64, _I32, _P, _I64, _P, _P]),
    "hqq_shrink_lp": (_I32, [_P, _I64, ctypes.c_double, ctypes.c_double, _P, _P]),
    "hqq_strerror": (ctypes.c_char_p, [_I32]),
}


def lib():
    """The loaded CUDA library; raises if libhqq_b200.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise HqqError(f"{LIB_PATH} is missing: build it with "
                           "`python -m free_weight_quantization_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != HQQ_OK:
        raise HqqError(f"{what}: {lib().hqq_strerror(rc).decode()} (code {rc})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def default_opt() -> HqqOpt:
    o = HqqOpt()
    lib().hqq_default_opt(ctypes.byref(o))
    return o


def hqq_packed_bytes(n: int, nbits: int) -> int:
    return int(lib().hqq_packed_bytes(n, nbits))


def hqq_quantize_workspace_bytes(rows: int, cols: int, nbits: int, group_size: int, axis: int,
                                 iters: int) -> int:
    return int(lib().hqq_quantize_workspace_bytes(rows, cols, nbits, group_size, axis, iters))


@dataclass
class Quantized:
    """Packed codes + fp16 metadata (the page's W_q, scale = Delta = 1/s, zero) and the shape."""
    packed: torch.Tensor
    scale: torch.Tensor
    zero: torch.Tensor
    rows: int
    cols: int
    nbits: int
    group_size: int
    axis: int
    iters_run: torch.Tensor | None = None
    s: torch.Tensor | None = None
    z: torch.Tensor | None = None
    err_trace: torch.Tensor | None = None
    rounds: torch.Tensor | None = None


def hqq_quantize(W: torch.Tensor, nbits: int = 4, group_size: int = 64, axis: int = 1,
                 iters: int = 20, lp_norm: float = 0.7, beta: float = 10.0, kappa: float = 1.01,
                 eps_tiny: float = 1e-4, scale_max: float = 2e4, *, out: Quantized | None = None,
                 workspace: torch.Tensor | None = None, debug: bool = False,
                 stream: torch.cuda.Stream | None = None) -> Quantized:
    """HQQ quantize + pack of an fp16 CUDA matrix [rows, cols] (see hqq_quantize in the header).
    With debug=True also returns iters_run, binary32 s and z, the exact error trace and the
    rounds each group needed."""
    if W.dtype != torch.float16 or not W.is_cuda or W.dim() != 2 or not W.is_contiguous():
        raise HqqError("W must be a contiguous 2-D float16 CUDA tensor")
    rows, cols = W.shape
    N = rows * cols
    if group_size <= 0 or N % group_size:
        raise HqqError("rows*cols must be a positive multiple of group_size")
    G = N // group_size
    dev = W.device
    if out is None:
        pb = hqq_packed_bytes(N, nbits)
        if pb < 0:
            raise HqqError("nbits must be 2, 3 or 4")
        out = Quantized(torch.empty(max(pb, 1), dtype=torch.uint8, device=dev),
                        torch.empty(G, dtype=torch.float16, device=dev),
                        torch.empty(G, dtype=torch.float16, device=dev),
                        rows, cols, nbits, group_size, axis)
        if debug:
            out.iters_run = torch.zeros(1, dtype=torch.int32, device=dev)
            out.s = torch.empty(G, dtype=torch.float32, device=dev)
            out.z = torch.empty(G, dtype=torch.float32, device=dev)
            out.err_trace = torch.zeros(max(2 * iters, 2), dtype=torch.int64, device=dev)
            out.rounds = torch.empty(G, dtype=torch.uint8, device=dev)
    wsb = hqq_quantize_workspace_bytes(rows, cols, nbits, group_size, axis, iters)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    opt = HqqOpt(iters, lp_norm, beta, kappa, eps_tiny, scale_max)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):  # launches go to the current device: W's
        rc = lib().hqq_quantize(_ptr(W), rows, cols, nbits, group_size, axis, ctypes.byref(opt),
                                _ptr(out.packed), _ptr(out.scale), _ptr(out.zero), _ptr(out.iters_run),
                                _ptr(out.s), _ptr(out.z), _ptr(out.err_trace), _ptr(out.rounds),
                                _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                ctypes.c_void_p(st.cuda_stream))
    _check(rc, "hqq_quantize")
    return out


HQQ_NOALLOC_SCRATCH_BYTES = 4 << 20


def hqq_quantize_noalloc(W: torch.Tensor, nbits: int = 4, group_size: int = 64, axis: int = 1,
                         iters: int = 20, lp_norm: float = 0.7, beta: float = 10.0,
                         kappa: float = 1.01, eps_tiny: float = 1e-4, scale_max: float = 2e4, *,
                         out: Quantized, stream: torch.cuda.Stream | None = None) -> Quantized:
    """hqq_quantize for callers that cannot allocate device memory: the caller passes every
    output buffer in `out` and the library uses its own fixed 4 MiB scratch buffer instead of a
    workspace (see hqq_quantize_noalloc in the header).  Nothing is allocated here either."""
    if W.dtype != torch.float16 or not W.is_cuda or W.dim() != 2 or not W.is_contiguous():
        raise HqqError("W must be a contiguous 2-D float16 CUDA tensor")
    rows, cols = W.shape
    bufs = [out.packed, out.scale, out.zero, out.iters_run, out.s, out.z, out.err_trace, out.rounds]
    if any(t is not None and t.device != W.device for t in bufs):
        raise HqqError("hqq_quantize_noalloc: every output must live on W's device")
    opt = HqqOpt(iters, lp_norm, beta, kappa, eps_tiny, scale_max)
    st = stream if stream is not None else torch.cuda.current_stream(W.device)
    if st.device != W.device:
        raise HqqError("hqq_quantize_noalloc: the stream must belong to W's device")
    # the library finds its scratch buffer on the calling thread's current device
    with torch.cuda.device(W.device):
        rc = lib().hqq_quantize_noalloc(_ptr(W), rows, cols, nbits, group_size, axis,
                                        ctypes.byref(opt), _ptr(out.packed), _ptr(out.scale),
                                        _ptr(out.zero), _ptr(out.iters_run), _ptr(out.s), _ptr(out.z),
                                        _ptr(out.err_trace), _ptr(out.rounds),
                                        ctypes.c_void_p(st.cuda_stream))
    if rc == 3:
        raise HqqError("hqq_quantize_noalloc: this problem needs "
                       f"{hqq_quantize_workspace_bytes(rows, cols, nbits, group_size, axis, iters)}"
                       f" bytes of scratch, more than the built-in {HQQ_NOALLOC_SCRATCH_BYTES}")
    _check(rc, "hqq_quantize_noalloc")
    return out


def hqq_dequantize(q: Quantized, out: torch.Tensor | None = None,
                   stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Unpack + (q - zero) * scale -> fp16 [rows, cols] (see hqq_dequantize in the header)."""
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.float16, device=q.packed.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.packed.device)
    with torch.cuda.device(q.packed.device):
        rc = lib().hqq_dequantize(_ptr(q.packed), _ptr(q.scale), _ptr(q.zero), q.rows, q.cols, q.nbits,
                                  q.group_size, q.axis, _ptr(out), ctypes.c_void_p(st.cuda_stream))
    _check(rc, "hqq_dequantize")
    return out


def hqq_gemv(q: Quantized, x: torch.Tensor, out: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """y = W_hat @ x with dequantization fused in (see hqq_gemv in the header): x is a
    contiguous fp16 CUDA vector of q.cols entries, y a binary32 vector of q.rows."""
    if x.dtype != torch.float16 or not x.is_cuda or x.dim() != 1 or x.numel() != q.cols or not x.is_contiguous():
        raise HqqError("x must be a contiguous fp16 CUDA vector with cols entries")
    if out is None:
        out = torch.empty(q.rows, dtype=torch.float32, device=q.packed.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.packed.device)
    with torch.cuda.device(q.packed.device):
        rc = lib().hqq_gemv(_ptr(q.packed), _ptr(q.scale), _ptr(q.zero), q.rows, q.cols, q.nbits,
                            q.group_size, q.axis, _ptr(x), _ptr(out), ctypes.c_void_p(st.cuda_stream))
    _check(rc, "hqq_gemv")
    return out


def hqq_gemm(q: Quantized, X: torch.Tensor, out: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Y = X @ W_hat.T for a batch of inputs with dequantization fused in (see hqq_gemm in the
    header): X is a contiguous fp16 CUDA matrix [batch, cols], Y binary32 [batch, rows]."""
    if X.dtype != torch.float16 or not X.is_cuda or X.dim() != 2 or X.shape[1] != q.cols or not X.is_contiguous():
        raise HqqError("X must be a contiguous fp16 CUDA matrix [batch, cols]")
    batch = X.shape[0]
    if out is None:
        out = torch.empty(batch, q.rows, dtype=torch.float32, device=q.packed.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.packed.device)
    with torch.cuda.device(q.packed.device):
        rc = lib().hqq_gemm(_ptr(q.packed), _ptr(q.scale), _ptr(q.zero), q.rows, q.cols, q.nbits,
                            q.group_size, q.axis, _ptr(X), batch, _ptr(out), ctypes.c_void_p(st.cuda_stream))
    _check(rc, "hqq_gemm")
    return out


def hqq_shrink_lp(r: torch.Tensor, beta: float, p: float = 0.7, out: torch.Tensor | None = None,
                  stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """The proximal step's lp shrink of binary32 residuals, as the quantizer evaluates it (see
    hqq_shrink_lp in the header)."""
    if r.dtype != torch.float32 or not r.is_cuda or not r.is_contiguous():
        raise HqqError("r must be a contiguous float32 CUDA tensor")
    if out is None:
        out = torch.empty_like(r)
    st = stream if stream is not None else torch.cuda.current_stream(r.device)
    with torch.cuda.device(r.device):
        rc = lib().hqq_shrink_lp(_ptr(r), r.numel(), float(beta), float(p), _ptr(out),
                                 ctypes.c_void_p(st.cuda_stream))
    _check(rc, "hqq_shrink_lp")
    return out


def err_trace_ints(t: torch.Tensor, n: int) -> list[int]:
    """Exact per-round error sums (units of 2^-32) from the (low, high) uint64 pairs."""
    v = t.cpu().view(torch.int64).tolist()
    return [(v[2 * i] & (2 ** 64 - 1)) + ((v[2 * i + 1] & (2 ** 64 - 1)) << 64) for i in range(n)]
