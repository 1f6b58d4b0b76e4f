"""Plain CPU oracle for HQQ group-wise quantization (ctypes binding over hqq_oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, the smoke check in __graft_entry__.py and the CPU-baseline
leg of bench.py may import this package.  The CUDA library and its Python binding never
import it, and it never imports them.

Every function here is argument marshalling around the C file, which states the method
(page "HQQ 算法解读", sections "量化公式", "第一拍", "第二拍", "为什么一定要分组", "`axis`")
and the readings taken where the page is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hqq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhqq_oracle.so")
# The all-core timing build: the same source with its round loop spread over OpenMP threads
# (bench.py's CPU baseline only; every test uses the single-threaded build).
_LIB_PAR_PATH = os.path.join(_HERE, "libhqq_oracle_omp.so")
# Test hook: the mutation test points this at a deliberately broken build of the oracle.
_LIB_OVERRIDE = os.environ.get("HQO_LIB_OVERRIDE")
# No contraction of a*b+c into fma, no fast-math: every binary32 operation rounds once.
CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None
_lib_par = None


def build_parallel(force: bool = False) -> str:
    """Compile the all-core timing build of hqq_oracle.c (OpenMP over groups, exact integer
    reduction of each round's error) into oracle/libhqq_oracle_omp.so."""
    if force or not os.path.exists(_LIB_PAR_PATH) or os.path.getmtime(_LIB_PAR_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PAR_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-fopenmp", "-DHQO_PARALLEL", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PAR_PATH)
    return _LIB_PAR_PATH


def build(force: bool = False) -> str:
    """Compile hqq_oracle.c with gcc into oracle/libhqq_oracle.so (in-tree)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load(parallel: bool = False):
    global _lib, _lib_par
    if parallel:
        if _lib_par is None:
            _lib_par = _declare(ctypes.CDLL(build_parallel()))
        return _lib_par
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(lib):
    P = ctypes.c_void_p
    i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
    lib.hqo_half_to_float.argtypes = [ctypes.c_uint16]
    lib.hqo_half_to_float.restype = f32
    lib.hqo_float_to_half.argtypes = [f32]
    lib.hqo_float_to_half.restype = ctypes.c_uint16
    lib.hqo_minmax_init.argtypes = [P, i64, i32, f32, f32, P, P]
    lib.hqo_minmax_init.restype = None
    lib.hqo_shrink.argtypes = [f32, f64, f64]
    lib.hqo_shrink.restype = f32
    lib.hqo_shrink_n.argtypes = [P, i64, f64, f64, P]
    lib.hqo_shrink_n.restype = None
    lib.hqo_pairwise_sum.argtypes = [P, i64]
    lib.hqo_pairwise_sum.restype = f32
    lib.hqo_group_pass.argtypes = [P, i64, i32, f32, f32, f64, f64, P, P, P]
    lib.hqo_group_pass.restype = None
    lib.hqo_quantize.argtypes = [P, i64, i64, i32, i64, i32, i32, f64, f64, f64, f32, f32,
                                 P, P, P, P, P, P]
    lib.hqo_quantize.restype = i32
    lib.hqo_metadata.argtypes = [P, P, i64, P, P]
    lib.hqo_metadata.restype = None
    lib.hqo_packed_bytes.argtypes = [i64, i32]
    lib.hqo_packed_bytes.restype = i64
    lib.hqo_pack.argtypes = [P, i64, i32, P]
    lib.hqo_pack.restype = None
    lib.hqo_unpack.argtypes = [P, i64, i32, P]
    lib.hqo_unpack.restype = None
    lib.hqo_dequant.argtypes = [P, P, P, i64, i64, i32, i64, i32, P]
    lib.hqo_gemv.argtypes = [P, P, P, i64, i64, i32, i64, i32, P, P, P]
    lib.hqo_dequant.restype = i32
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_u16(W) -> np.ndarray:
    W = np.ascontiguousarray(W)
    if W.dtype == np.float16:
        return W.view(np.uint16)
    if W.dtype == np.uint16:
        return W
    raise TypeError("W must be float16 (or its uint16 bit pattern)")


# ---------------------------------------------------------------- scalar helpers
def half_to_float(h: int) -> float:
    return _load().hqo_half_to_float(int(h))


def float_to_half(f: float) -> int:
    return int(_load().hqo_float_to_half(float(f)))


def shrink(r: float, beta: float, p: float) -> float:
    return _load().hqo_shrink(float(r), float(beta), float(p))


def shrink_array(r, beta: float, p: float) -> np.ndarray:
    """shrink() of every element of a float32 array."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    out = np.empty_like(r)
    _load().hqo_shrink_n(_ptr(r), r.size, float(beta), float(p), _ptr(out))
    return out


def pairwise_sum(x) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return float(_load().hqo_pairwise_sum(_ptr(x), x.size))


def minmax_init(w, nbits: int, eps_tiny: float = 1e-4, scale_max: float = 2e4):
    """(s0, z0) of one group of binary32 values."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    _load().hqo_minmax_init(_ptr(w), w.size, nbits, eps_tiny, scale_max, _ptr(s), _ptr(z))
    return float(s[0]), float(z[0])


def group_pass(w, nbits: int, s: float, z: float, beta: float, p: float):
    """One proximal pass over one group: (codes, sum|W - W_hat|, z_new)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    q = np.zeros(w.size, np.uint8)
    err = np.zeros(1, np.float32)
    zn = np.zeros(1, np.float32)
    _load().hqo_group_pass(_ptr(w), w.size, nbits, s, z, beta, p, _ptr(q), _ptr(err), _ptr(zn))
    return q, float(err[0]), float(zn[0])


# ---------------------------------------------------------------- packing
def packed_bytes(n: int, nbits: int) -> int:
    return int(_load().hqo_packed_bytes(n, nbits))


def pack(codes, nbits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
    out = np.zeros(packed_bytes(codes.size, nbits), np.uint8)
    _load().hqo_pack(_ptr(codes), codes.size, nbits, _ptr(out))
    return out


def unpack(packed, n: int, nbits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8).ravel()
    out = np.zeros(n, np.uint8)
    _load().hqo_unpack(_ptr(packed), n, nbits, _ptr(out))
    return out


# ---------------------------------------------------------------- the method
DEFAULTS = dict(iters=20, lp_norm=0.7, beta=10.0, kappa=1.01, eps_tiny=1e-4, scale_max=2e4)


def quantize(W, nbits: int, group_size: int, axis: int = 1, iters: int = 20, lp_norm: float = 0.7,
             beta: float = 10.0, kappa: float = 1.01, eps_tiny: float = 1e-4,
             scale_max: float = 2e4, parallel: bool = False) -> dict:
    """HQQ quantize+pack of a 2-D fp16 matrix.  Returns a dict with codes (flat, one per
    byte), s, z (binary32 per group; z is the kept zero), scale/zero (fp16 Delta = 1/s and z),
    packed bytes, iters_run, err_trace (exact per-iteration error sums, units of 2^-32, as
    Python ints) and mae_trace.  parallel=True runs the all-core timing build (same results;
    for the benchmark's CPU baseline)."""
    Wu = _as_u16(W)
    assert Wu.ndim == 2
    rows, cols = Wu.shape
    N = rows * cols
    if N % group_size:
        raise ValueError("rows*cols must be a multiple of group_size")
    G = N // group_size
    codes = np.zeros(N, np.uint8)
    s = np.zeros(G, np.float32)
    z = np.zeros(G, np.float32)
    run = ctypes.c_int(0)
    trace = np.zeros(max(2 * iters, 2), np.uint64)
    mae = np.zeros(max(iters, 1), np.float64)
    rc = _load(parallel).hqo_quantize(_ptr(Wu), rows, cols, nbits, group_size, axis, iters, lp_norm, beta,
                              kappa, eps_tiny, scale_max, _ptr(codes), _ptr(s), _ptr(z),
                              ctypes.byref(run), _ptr(trace), _ptr(mae))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    n_run = run.value
    scale_h = np.zeros(G, np.uint16)
    zero_h = np.zeros(G, np.uint16)
    _load().hqo_metadata(_ptr(s), _ptr(z), G, _ptr(scale_h), _ptr(zero_h))
    err = [int(trace[2 * i]) + (int(trace[2 * i + 1]) << 64) for i in range(n_run)]
    return dict(codes=codes, s=s, z=z, scale=scale_h.view(np.float16), zero=zero_h.view(np.float16),
                packed=pack(codes, nbits), iters_run=n_run, err_trace=err,
                mae_trace=[float(x) for x in mae[:n_run]], rows=rows, cols=cols, nbits=nbits,
                group_size=group_size, axis=axis)


def gemv(packed, scale, zero, rows: int, cols: int, nbits: int, group_size: int, axis: int,
         x) -> tuple[np.ndarray, np.ndarray]:
    """y = W_hat @ x in binary64 (W_hat the fp16 dequantized weights, x fp16 [cols]) and the
    per-row sum of |W_hat * x|; see hqo_gemv."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    sc = _as_u16(scale)
    ze = _as_u16(zero)
    xh = _as_u16(x)
    assert xh.size == cols
    y = np.zeros(rows, np.float64)
    mag = np.zeros(rows, np.float64)
    rc = _load().hqo_gemv(_ptr(packed), _ptr(sc), _ptr(ze), rows, cols, nbits, group_size, axis,
                          _ptr(xh), _ptr(y), _ptr(mag))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return y, mag


def gemm(packed, scale, zero, rows: int, cols: int, nbits: int, group_size: int, axis: int,
         X) -> tuple[np.ndarray, np.ndarray]:
    """Y = X @ W_hat.T for a batch X [batch, cols] fp16: hqo_gemv for every row of X (the
    product is defined row by row); returns Y and the per-element sum of |W_hat * x|, both
    [batch, rows] binary64."""
    X = np.ascontiguousarray(X, dtype=np.float16)
    out = [gemv(packed, scale, zero, rows, cols, nbits, group_size, axis, x) for x in X]
    return (np.stack([y for y, _ in out]) if out else np.zeros((0, rows))), \
           (np.stack([m for _, m in out]) if out else np.zeros((0, rows)))


def dequant(packed, scale, zero, rows: int, cols: int, nbits: int, group_size: int,
            axis: int = 1) -> np.ndarray:
    """Unpack + (q - z)*Delta -> fp16 [rows, cols]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    sc = _as_u16(scale)
    ze = _as_u16(zero)
    out = np.zeros(rows * cols, np.uint16)
    rc = _load().hqo_dequant(_ptr(packed), _ptr(sc), _ptr(ze), rows, cols, nbits, group_size, axis,
                             _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out.view(np.float16).reshape(rows, cols)
