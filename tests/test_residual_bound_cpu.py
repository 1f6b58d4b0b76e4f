"""The streaming kernel's residual bound, checked on the CPU.

The kernel skips the exact lp shrink for a whole group when a bound B, computed from the
group's state alone, is at or below the round's dead-zone threshold; that is exact only if
B >= |RN(W - W_hat)| for every element.  The kernel forms B as
    M     = max(1/2, -RN(lo + z), RN(hi + z) - qmax)
    slack = RN(RN(8 * RN(A + |z|) + 4 qmax) * 2^-23),   A = max(|lo|, |hi|)
    B     = RN(RN(RN(M + slack) * y) * (1 + 2^-20)),    y = RN(1/s)
from lo = RN(min(W) s) and hi = RN(max(W) s).  Here every step of the round is carried out in
IEEE binary32 with numpy, including the clamp the kernel applies whenever some element might
leave [0, qmax].  The zero is then shifted away from its min-max start to force clipping,
and B is checked against the largest residual.  This tests the derivation of the bound, not
the device code that evaluates it.
"""
import numpy as np
import pytest

f32 = np.float32


def _round(Wh, s, z, nbits):
    """One round of the kernel in binary32: t = RN(RN(W s) + z), clamped when needed, rounded
    half to even; W_hat = RN(RN(q - z) / s); r = RN(W - W_hat)."""
    qmax = f32((1 << nbits) - 1)
    w = Wh.astype(f32)
    t = (w * s).astype(f32) + z
    t = t.astype(f32)
    lo = f32(w.min() * s)
    hi = f32(w.max() * s)
    lz, hz = f32(lo + z), f32(hi + z)
    if not (lz >= f32(-0.5) and hz < qmax + f32(0.5)):
        t = np.clip(t, f32(0), qmax)
    q = np.rint(t).astype(f32)
    what = ((q - z).astype(f32) / s).astype(f32)
    r = (w - what).astype(f32)
    return np.abs(r).max(), lo, hi, lz, hz


def _bound(lo, hi, lz, hz, s, z, nbits):
    qmax = f32((1 << nbits) - 1)
    A = max(abs(lo), abs(hi))
    y = f32(f32(1) / s)
    M = max(f32(0.5), -lz, f32(hz - qmax))
    slack = f32(f32(f32(8) * f32(A + abs(z)) + f32(4) * qmax) * f32(2.0 ** -23))
    return f32(f32(f32(M + slack) * y) * f32(1 + 2.0 ** -20))


def _init(Wh, nbits, eps=f32(1e-4), smax=f32(2e4)):
    qmax = f32((1 << nbits) - 1)
    w = Wh.astype(f32)
    d = f32(w.max() - w.min())
    s = f32(1) if d < eps else f32(qmax / d)
    s = min(s, smax)
    z = f32(f32(0) - f32(w.min() * s))
    return s, z


@pytest.mark.parametrize("nbits", [2, 4])
@pytest.mark.parametrize("g", [16, 64])
def test_bound_dominates_every_residual(nbits, g):
    r = np.random.default_rng(1000 * nbits + g)
    worst = 0.0
    for trial in range(3000):
        kind = trial % 4
        if kind == 0:
            Wh = (0.02 * r.standard_t(4, g)).clip(-1, 1).astype(np.float16)
        elif kind == 1:
            Wh = (r.standard_normal(g) * 10.0 ** r.uniform(-4, 4)).clip(-6e4, 6e4).astype(np.float16)
        elif kind == 2:
            Wh = (0.5 + r.integers(0, 3, g) * 2.0 ** -11).astype(np.float16)   # tiny range
        else:
            Wh = r.uniform(-65504, 65504, g).astype(np.float16)                  # full fp16 range
        s, z0 = _init(Wh, nbits)
        for shift in (0.0, r.uniform(-0.49, 0.49), r.uniform(-4, 4), r.uniform(-40, 40)):
            z = f32(z0 + f32(shift))
            mr, lo, hi, lz, hz = _round(Wh, s, z, nbits)
            B = _bound(lo, hi, lz, hz, s, z, nbits)
            assert mr <= B, (trial, kind, shift, float(mr), float(B))
            worst = max(worst, float(mr / B) if B > 0 else 0.0)
    # the bound is tight up to its slack: the largest residual comes close to it
    assert worst > 0.5
