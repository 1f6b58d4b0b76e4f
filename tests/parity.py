"""Shared checks: the CUDA path (through the C ABI) against the CPU oracle.

Acceptance, per element and per group:
  - iteration count and the exact per-round error sums: equal;
  - codes: equal, except a code may differ where the oracle's W*s + z lies within 1e-5 of a
    rounding boundary k + 0.5;
  - binary32 s and the kept z: within 1e-5 relative; fp16 scale and zero: equal where the
    binary32 values are equal;
  - dequantized weights: the GPU dequant of the GPU codes equals the oracle dequant of the
    same codes to 1e-3 absolute (in practice bit for bit); the GPU result is within 1e-3 of
    the oracle dequant of the oracle codes except at allowed code flips.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from free_weight_quantization_b200 import hqq

TOL_REL = 1e-5
TOL_TIE = 1e-5
TOL_DEQ = 1e-3


def gpu_quantize(W: np.ndarray, nbits, g, axis, iters=20, **kw):
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    q = hqq.hqq_quantize(Wd, nbits, g, axis, iters=iters, debug=True, **kw)
    deq = hqq.hqq_dequantize(q)
    torch.cuda.synchronize()
    n = int(q.iters_run.item())
    return dict(packed=q.packed.cpu().numpy()[:oracle.packed_bytes(W.size, nbits)],
                scale=q.scale.cpu().numpy(), zero=q.zero.cpu().numpy(), s=q.s.cpu().numpy(),
                z=q.z.cpu().numpy(), iters_run=n, err_trace=hqq.err_trace_ints(q.err_trace, n),
                deq=deq.cpu().numpy(), q=q)


def check(W: np.ndarray, ref: dict, got: dict, label: str = ""):
    nbits, g, axis = ref["nbits"], ref["group_size"], ref["axis"]
    rows, cols = W.shape
    N = W.size
    assert got["iters_run"] == ref["iters_run"], (label, got["iters_run"], ref["iters_run"])
    assert got["err_trace"] == ref["err_trace"], label
    s_ok = np.abs(got["s"].astype(np.float64) - ref["s"]) <= TOL_REL * np.abs(ref["s"])
    assert s_ok.all(), (label, "s", np.flatnonzero(~s_ok)[:5])
    z_ok = np.abs(got["z"].astype(np.float64) - ref["z"]) <= TOL_REL * np.maximum(np.abs(ref["z"]), 1e-30)
    assert z_ok.all(), (label, "z", np.flatnonzero(~z_ok)[:5])
    same = (got["s"] == ref["s"]) & (got["z"] == ref["z"])
    assert np.array_equal(got["scale"].view(np.uint16)[same], ref["scale"].view(np.uint16)[same]), label
    assert np.array_equal(got["zero"].view(np.uint16)[same], ref["zero"].view(np.uint16)[same]), label
    # codes
    codes = oracle.unpack(got["packed"], N, nbits)
    bad = np.flatnonzero(codes != ref["codes"])
    if bad.size:
        G = N // g
        k = bad // g if axis == 1 else bad % G
        t = W.ravel()[bad].astype(np.float64) * ref["s"][k] + ref["z"][k]
        dist = np.abs(t - np.floor(t) - 0.5)
        assert (dist < TOL_TIE).all(), (label, "code mismatch off a tie", bad[dist >= TOL_TIE][:5])
    else:
        assert np.array_equal(got["packed"], ref["packed"]), (label, "padding bits")
    # dequant
    deq_same = oracle.dequant(got["packed"], got["scale"], got["zero"], rows, cols, nbits, g, axis)
    d = np.abs(got["deq"].astype(np.float64) - deq_same.astype(np.float64))
    assert d.max(initial=0) <= TOL_DEQ, (label, "dequant vs oracle dequant of the same codes", d.max())
    deq_ref = oracle.dequant(ref["packed"], ref["scale"], ref["zero"], rows, cols, nbits, g, axis)
    d2 = np.abs(got["deq"].astype(np.float64) - deq_ref.astype(np.float64)).ravel()
    off = d2 > TOL_DEQ
    if off.any():
        assert np.isin(np.flatnonzero(off), bad).all(), (label, "dequant differs beyond flips")
    return dict(code_flips=int(bad.size), deq_bit_exact=bool((d == 0).all()))


def oracle_job(case_name: str, iters: int = 20) -> dict:
    """Runs in a spawned worker: rebuild the seeded workload and quantize it on the CPU."""
    from free_weight_quantization_b200 import workloads as wl
    c = next(c for c in wl.CASES if c.name == case_name)
    return oracle.quantize(c.make(), c.nbits, c.group_size, c.axis, iters=iters)


def oracle_on(W: np.ndarray, nbits, g, axis, iters=20) -> dict:
    return oracle.quantize(W, nbits, g, axis, iters=iters)
