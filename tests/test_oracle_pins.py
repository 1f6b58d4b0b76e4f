"""Pins for the CPU oracle: each test checks it against something other than itself.

Sources: the page "HQQ 算法解读" (worked example, bpw bookkeeping, packing densities, the
least-squares property of the zero update, the loop's stop rule), the page "LLM 量化综述"
at k4i.top (asymmetric affine quantization, the rounding-error bound, RTN as the baseline),
IEEE 754 binary16 as implemented by numpy, and brute-force scans on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from free_weight_quantization_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ binary16 conversions
def test_half_to_float_exhaustive():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(x)) for x in h], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_matches_numpy_rne():
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 65504.0, 65519.996, 65520.0, -65520.0, 1e9, np.inf, -np.inf,
            2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14 - 2.0 ** -25]
    # exact midpoints between neighbouring fp16 values: ties must go to the even one
    h = rng.integers(0, 0x7bff, 2000).astype(np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).view(np.float16).astype(np.float64)
    vals += list(((a + b) / 2).astype(np.float32))
    vals += list(rng.standard_normal(3000).astype(np.float32) * 10.0 ** rng.integers(-9, 5, 3000))
    x = np.array(vals, np.float32)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ the page's worked example
def test_worked_example_binary32():
    ex = golden("worked_example.json")
    w = np.linspace(ex["min"], ex["max"], 64).astype(np.float32)
    w[10] = 0.0
    s, z = oracle.minmax_init(w, ex["nbits"])
    assert abs(s - ex["s0"]) <= 1e-6 and abs(z - ex["z0"]) <= 1e-6
    q, _, _ = oracle.group_pass(w, ex["nbits"], s, z, beta=1e-6, p=0.7)
    lookup = {float(np.float32(v)): c for v, c in ex["codes"]}
    for j, v in enumerate(w):
        if float(v) in lookup:
            assert q[j] == lookup[float(v)], (v, q[j])


def test_worked_example_fp16_input():
    # The same group stored as fp16: fp16(-0.8) = -0.7998046875 and fp16(0.7) = 0.7001953125,
    # so the range is still exactly 1.5 and s0 = 10, but z0 = 0.7998046875*10 = 7.998046875.
    ex = golden("worked_example.json")
    w = np.linspace(ex["min"], ex["max"], 64).astype(np.float16)
    w[10] = 0.0
    r = oracle.quantize(w.reshape(1, 64), ex["nbits"], 64, axis=1, iters=0)
    assert r["s"][0] == np.float32(10.0)
    assert r["z"][0] == np.float32(7.998046875)
    # metadata stores Delta = 1/s (section "量化公式"): fp16(0.1)
    assert r["scale"][0] == np.float16(0.1)
    for v, c in ex["codes"]:
        j = int(np.flatnonzero(w == np.float16(v))[0])
        assert r["codes"][j] == c


# ------------------------------------------------------------------ storage bookkeeping
def test_bits_per_weight_bookkeeping():
    bp = golden("bpw.json")
    g = bp["group_size"]
    assert oracle.packed_bytes(g, bp["nbits"]) == bp["code_bytes_per_group"]
    n = 4096 * 4096
    G = n // g
    total = oracle.packed_bytes(n, bp["nbits"]) + 2 * 2 * G
    assert total * 8 / n == bp["bits_per_weight"]
    assert total / G == bp["bytes_per_group"]
    for nbits, (codes, nbytes) in bp["codes_per_container"].items():
        assert oracle.packed_bytes(codes, int(nbits)) == nbytes
        assert oracle.packed_bytes(codes * 7, int(nbits)) == nbytes * 7


def test_pack_hand_computed():
    # 4 bit: low nibble = lower index.  0x1 | 0xA << 4 = 0xA1, 0xF | 0x0 << 4 = 0x0F
    assert list(oracle.pack([0x1, 0xA, 0xF, 0x0], 4)) == [0xA1, 0x0F]
    # odd count: the last high nibble is 0
    assert list(oracle.pack([7, 8, 9], 4)) == [0x87, 0x09]
    # 2 bit: 1 | 2<<2 | 3<<4 | 0<<6 = 1 + 8 + 48 = 57 = 0x39
    assert list(oracle.pack([1, 2, 3, 0, 3, 3], 2)) == [0x39, 0x0F]
    # 3 bit: codes 0..7,1,2 at bit offsets 0,3,..,27:
    # 8 + 128 + 1536 + 16384 + 163840 + 1572864 + 14680064 + 16777216 + 268435456
    # = 301647496 = 0x11FAC688, stored little-endian; bits 30-31 are 0
    assert list(oracle.pack([0, 1, 2, 3, 4, 5, 6, 7, 1, 2], 3)) == [0x88, 0xC6, 0xFA, 0x11]
    # ten 7s fill bits 0-29; a tail word with three codes is 0o777 = 0x1FF, zero padded
    assert list(oracle.pack([7] * 13, 3)) == [0xFF, 0xFF, 0xFF, 0x3F, 0xFF, 0x01, 0x00, 0x00]


def test_pack_hand_computed_other_widths():
    # 1 bit: eight codes per byte, the lowest index in the lowest bit.
    # 1 + 0*2 + 1*4 + 1*8 + 0 + 0 + 0 + 1*128 = 141 = 0x8D; a ninth code starts the next byte
    assert list(oracle.pack([1, 0, 1, 1, 0, 0, 0, 1, 1], 1)) == [0x8D, 0x01]
    assert oracle.packed_bytes(64, 1) == 8 and oracle.packed_bytes(65, 1) == 9
    # 5 and 6 bit [HQQ 算法解读, "为什么一定要分组"]: one code per byte, unpacked; 7 and 8 bit alike
    for nbits in (5, 6, 7, 8):
        top = (1 << nbits) - 1
        assert list(oracle.pack([top, 0, 17], nbits)) == [top, 0, 17]
        assert oracle.packed_bytes(64, nbits) == 64


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("n", [1, 9, 10, 11, 64, 1001])
def test_pack_roundtrip(nbits, n):
    rng = np.random.default_rng(n * 10 + nbits)
    c = rng.integers(0, 1 << nbits, n).astype(np.uint8)
    assert np.array_equal(oracle.unpack(oracle.pack(c, nbits), n, nbits), c)


# ------------------------------------------------------------------ sums and shrink
def test_pairwise_sum_order():
    t = 2.0 ** -24
    # (1 + 0) + (t + t) = 1 + 2^-23 exactly; a left-to-right sum would give 1.
    assert oracle.pairwise_sum([1.0, 0.0, t, t]) == 1.0 + 2.0 ** -23
    # three elements are padded to four: (1 + 0) + (t + 0) rounds back to 1
    assert oracle.pairwise_sum([1.0, 0.0, t]) == 1.0
    rng = np.random.default_rng(3)
    for n in [1, 2, 5, 16, 37, 64]:
        x = rng.standard_normal(n).astype(np.float32)
        exact = math.fsum(float(v) for v in x)
        bound = math.ceil(math.log2(max(n, 2))) * 2.0 ** -24 * float(np.abs(x).sum()) * 1.01
        assert abs(oracle.pairwise_sum(x) - exact) <= bound


def test_shrink_p1_is_l1_prox():
    # p = 1: shrink is soft thresholding, the minimiser of 0.5 (x - r)^2 + |x| / beta.
    grid = np.linspace(-2, 2, 400001)
    for r, beta in [(0.5, 10.0), (-0.31, 4.0), (0.05, 10.0), (1.7, 1.0), (-0.2, 5.0)]:
        obj = 0.5 * (grid - r) ** 2 + np.abs(grid) / beta
        x = grid[np.argmin(obj)]
        assert abs(oracle.shrink(r, beta, 1.0) - x) <= 2e-5


def test_shrink_lp_shape():
    # "small residuals go to 0; large ones are kept but reduced" (section "shrink 不是删除极值")
    p = 0.7
    for beta in [10.0, 10.0 * 1.01 ** 19, 3.0]:
        thr = beta ** (-1.0 / (2.0 - p))   # |r| - |r|^(p-1)/beta <= 0  <=>  |r| <= thr
        for r in [0.0, thr * 0.5, thr * 0.999, -thr * 0.999]:
            assert oracle.shrink(r, beta, p) == 0.0
        for r in [thr * 1.001, thr * 3, -thr * 3, 5.0]:
            e = oracle.shrink(r, beta, p)
            assert e != 0.0 and np.sign(e) == np.sign(r) and abs(e) < abs(r)
            assert oracle.shrink(-r, beta, p) == -e
        es = [oracle.shrink(v, beta, p) for v in np.linspace(0, 4, 50)]
        assert all(b >= a for a, b in zip(es, es[1:]))


def test_shrink_array_is_the_scalar_shrink():
    # the array form used by the GPU agreement check is the scalar operator, element by element
    r = np.random.default_rng(5).standard_normal(2000).astype(np.float32) * 0.5
    for beta in [10.0, 10.0 * 1.01 ** 19]:
        got = oracle.shrink_array(r, beta, 0.7)
        want = np.array([oracle.shrink(float(v), beta, 0.7) for v in r], np.float32)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ------------------------------------------------------------------ one proximal pass
@pytest.mark.parametrize("g,nbits", [(4, 2), (5, 3), (8, 4), (6, 4)])
def test_zero_update_is_least_squares(g, nbits):
    # Section "为什么 zero 是这个均值": for fixed q and s, mean(q - (W - e)*s) minimises the
    # squared reconstruction error over z.  Brute-force scan of z.
    rng = np.random.default_rng(g * 31 + nbits)
    M = 2 ** nbits - 1
    for trial in range(9):
        # trials 6-8 use a wide range (large residuals: the shrink is active) and push z
        # far enough that some codes clip at 0 or 2^b - 1
        w = (rng.standard_normal(g) * (0.05 if trial < 6 else 5.0)).astype(np.float32)
        s, z = oracle.minmax_init(w, nbits)
        z += float(rng.uniform(-0.4, 0.4) if trial < 6 else rng.choice([-1.7, 1.7]))
        beta = [1e-6, 10.0, 0.5][trial % 3]   # 1e-6: e = 0; others may shrink
        q, _, zn = oracle.group_pass(w, nbits, s, z, beta, 0.7)
        # q itself: the nearest integer code in [0, M] to W*s + z
        t = w.astype(np.float64) * s + z
        qref = np.clip(np.floor(t + 0.5), 0, M)
        near_tie = np.abs(t - np.floor(t) - 0.5) < 1e-5
        assert np.array_equal(q[~near_tie], qref[~near_tie].astype(np.uint8))
        e = np.array([oracle.shrink(float(wi - (qi - z) / s), beta, 0.7)
                      for wi, qi in zip(w.astype(np.float64), q.astype(np.float64))])
        target = q - (w.astype(np.float64) - e) * s
        grid = np.linspace(zn - 0.5, zn + 0.5, 100001)
        sse = ((target[None, :] - grid[:, None]) ** 2).sum(1)
        assert abs(grid[np.argmin(sse)] - zn) <= 2e-5


def test_group_error_is_mae_sum():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(64) * 0.02).astype(np.float32)
    s, z = oracle.minmax_init(w, 4)
    q, err, _ = oracle.group_pass(w, 4, s, z, 10.0, 0.7)
    w_hat = (q.astype(np.float64) - z) / s
    assert abs(err - np.abs(w.astype(np.float64) - w_hat).sum()) <= 1e-6 * max(err, 1e-6)


# ------------------------------------------------------------------ the loop-free special case
@pytest.mark.parametrize("nbits,g", [(4, 64), (3, 64), (2, 16), (1, 32), (5, 64), (6, 64), (8, 128)])
def test_iters0_is_minmax_rtn(nbits, g):
    # With no proximal iteration the method is asymmetric min-max RTN (k4i.top, sections
    # "线性量化：scale、zero point 与舍入" and "RTN：round-to-nearest 是基线").
    W = wl.student_t(64, 256, seed=5)
    r = oracle.quantize(W, nbits, g, axis=1, iters=0)
    assert r["iters_run"] == 0
    # one round measures only z0, so the kept zero is still z0: the same RTN result
    r1 = oracle.quantize(W, nbits, g, axis=1, iters=1)
    assert r1["iters_run"] == 1
    assert np.array_equal(r1["codes"], r["codes"]) and np.array_equal(r1["z"], r["z"])
    w = W.astype(np.float64).reshape(-1, g)
    mn = w.min(1, keepdims=True)
    mx = w.max(1, keepdims=True)
    M = 2 ** nbits - 1
    t = (w - mn) / (mx - mn) * M
    qref = np.clip(np.floor(t + 0.5), 0, M).ravel()
    near_tie = (np.abs(t - np.floor(t) - 0.5) < 1e-4).ravel()
    assert np.array_equal(r["codes"][~near_tie], qref[~near_tie].astype(np.uint8))
    np.testing.assert_allclose(1.0 / r["s"], ((mx - mn) / M).ravel(), rtol=1e-6)


def test_degenerate_groups():
    # constant group: denominator 0 -> s = 1, z = -min, all codes 0, exact reconstruction
    W = np.full((1, 64), 0.375, np.float16)
    r = oracle.quantize(W, 4, 64, iters=20)
    assert r["s"][0] == 1.0 and r["z"][0] == -0.375 and not r["codes"].any()
    Wd = oracle.dequant(r["packed"], r["scale"], r["zero"], 1, 64, 4, 64)
    assert np.array_equal(Wd, W)
    # range below eps_tiny -> s = 1; range just above it -> s clamped to 2e4
    w = np.zeros((1, 64), np.float16)
    w[0, 1] = np.float16(5e-5)
    assert oracle.quantize(w, 4, 64, iters=0)["s"][0] == 1.0
    w[0, 1] = np.float16(2e-4)
    assert oracle.quantize(w, 4, 64, iters=0)["s"][0] == np.float32(2e4)


# ------------------------------------------------------------------ loop invariants
@pytest.fixture(scope="module")
def small_result():
    W = wl.SMALL.make()
    return W, oracle.quantize(W, 4, 64, axis=1, iters=20)


def test_loop_stop_rule(small_result):
    _, r = small_result
    err = r["err_trace"]
    n = r["iters_run"]
    assert 1 <= n <= 20 and len(err) == n
    accepted = [err[0]]
    for e in err[1:]:
        if e < min(accepted):
            accepted.append(e)
        else:
            break
    # every iteration but possibly the last was an improvement; the last, if the loop did not
    # run out, was not (section "第二拍": stop when the MAE is no better)
    assert len(accepted) in (n, n - 1)
    assert all(b < a for a, b in zip(accepted, accepted[1:]))
    if n < 20:
        assert len(accepted) == n - 1 and err[-1] >= min(err[:-1])


def test_kept_zero_reproduces_best_mae(small_result):
    W, r = small_result
    g = 64
    w = W.astype(np.float64).reshape(-1, g)
    q = r["codes"].astype(np.float64).reshape(-1, g)
    w_hat = (q - r["z"][:, None].astype(np.float64)) / r["s"][:, None].astype(np.float64)
    mae = np.abs(w - w_hat).mean()
    best = min(r["mae_trace"])
    assert abs(mae - best) <= 1e-6 * best
    rtn = oracle.quantize(W, 4, 64, axis=1, iters=1)["mae_trace"][0]
    assert best <= rtn


def test_unclipped_rounding_error_bound(small_result):
    # k4i.top, section "误差从哪里来": without clipping each error is at most half a step.
    W, r = small_result
    g = 64
    w = W.astype(np.float64).reshape(-1, g)
    s = r["s"][:, None].astype(np.float64)
    z = r["z"][:, None].astype(np.float64)
    t = w * s + z
    inside = (t > 0) & (t < 15)
    w_hat = (r["codes"].astype(np.float64).reshape(-1, g) - z) / s
    assert np.all(np.abs(w - w_hat)[inside] <= (0.5 / s + 1e-6 / s).repeat(g, 1)[inside])


# ------------------------------------------------------------------ axis and dequant
def test_axis0_is_axis1_of_the_transposed_view():
    # Section "`axis` 不是一个无关紧要的开关": axis=0 groups are the columns of W.reshape(g, -1).
    W = wl.student_t(32, 96, seed=9)
    g = 16
    r0 = oracle.quantize(W, 3, g, axis=0, iters=20)
    Wt = np.ascontiguousarray(W.reshape(g, -1).T)          # [G, g]: groups as rows
    r1 = oracle.quantize(Wt, 3, g, axis=1, iters=20)
    assert r0["iters_run"] == r1["iters_run"] and r0["err_trace"] == r1["err_trace"]
    assert np.array_equal(r0["s"], r1["s"]) and np.array_equal(r0["z"], r1["z"])
    assert np.array_equal(r0["codes"].reshape(g, -1), r1["codes"].reshape(-1, g).T)


def test_dequant_closed_form():
    # (q - z) * Delta with fp16 z = 1.5 and Delta = 0.25: codes 3 and 0 -> 0.375 and -0.375
    packed = oracle.pack([3, 0], 4)
    out = oracle.dequant(packed, np.array([0.25], np.float16), np.array([1.5], np.float16),
                         1, 2, 4, 2, axis=1)
    assert out.tolist() == [[0.375, -0.375]]


def test_dequant_of_quantize_matches_kept_parameters(small_result):
    W, r = small_result
    Wd = oracle.dequant(r["packed"], r["scale"], r["zero"], 256, 512, 4, 64, axis=1)
    q = r["codes"].astype(np.float64).reshape(-1, 64)
    z = r["zero"].astype(np.float64)[:, None]
    d = r["scale"].astype(np.float64)[:, None]
    ref = ((q - z) * d).astype(np.float16).reshape(256, 512)
    # binary32 (q - z)*Delta then one rounding to fp16 against the float64 value: equal except
    # where the float64 value sits on an fp16 rounding boundary
    diff = np.abs(Wd.astype(np.float64) - ref.astype(np.float64))
    assert (diff > 0).mean() < 1e-3 and diff.max() <= 2.0 ** -11 * np.abs(ref).max()
    # and the dequantized matrix reconstructs W about as well as the loop measured
    mae = np.abs(Wd.astype(np.float64) - W.astype(np.float64)).mean()
    assert abs(mae - min(r["mae_trace"])) <= 0.02 * mae


def test_stop_one_iteration_after_convergence():
    # A single group converges in a few rounds; the first round whose MAE is not strictly
    # better (here: equal, the zero no longer moves) ends the loop.
    W = wl.student_t(1, 64, seed=21)
    r = oracle.quantize(W, 4, 64, iters=20)
    err = r["err_trace"]
    assert r["iters_run"] < 20
    assert err[-1] >= min(err[:-1])
    assert all(b < a for a, b in zip(err[:-1], err[1:-1]))


def test_beta_schedule_and_zero_chaining():
    # Rounds chain z_{i+1} = mean(q_i - (W - e_i)*s) with beta_i = beta * kappa^i
    # (section "第二拍").  A wide-range group makes the shrink active so beta matters.
    rng = np.random.default_rng(5)
    w16 = (rng.standard_normal(64) * 3.0).astype(np.float16)
    w = w16.astype(np.float32)
    beta, kappa = 10.0, 1.5
    r = oracle.quantize(w16.reshape(1, 64), 4, 64, iters=3, beta=beta, kappa=kappa)
    s, z0 = oracle.minmax_init(w, 4)
    _, e0, z1 = oracle.group_pass(w, 4, s, z0, beta, 0.7)
    _, e1, z2 = oracle.group_pass(w, 4, s, z1, beta * kappa, 0.7)
    _, e2, _ = oracle.group_pass(w, 4, s, z2, beta * kappa * kappa, 0.7)
    fixed = [int(np.float64(e) * 2.0 ** 32) for e in (e0, e1, e2)]
    assert r["err_trace"] == fixed[:r["iters_run"]]
    assert r["iters_run"] == 3
    # the shrink changes the trajectory: a different kappa gives a different z_2
    _, _, z2b = oracle.group_pass(w, 4, s, z1, beta, 0.7)
    assert z2b != z2


def test_dequant_axis0_layout():
    W = wl.student_t(16, 40, seed=2)
    g = 8
    r0 = oracle.quantize(W, 4, g, axis=0, iters=5)
    d0 = oracle.dequant(r0["packed"], r0["scale"], r0["zero"], 16, 40, 4, g, axis=0)
    Wt = np.ascontiguousarray(W.reshape(g, -1).T)
    r1 = oracle.quantize(Wt, 4, g, axis=1, iters=5)
    d1 = oracle.dequant(r1["packed"], r1["scale"], r1["zero"], Wt.shape[0], g, 4, g, axis=1)
    assert np.array_equal(d0.reshape(g, -1), d1.T)


# ---- the forward product y = W_hat @ x [HQQ 算法解读, "从压缩文件到一次前向"] ----

def _random_quantized(rows, cols, nbits, g, axis, seed):
    r = np.random.default_rng(seed)
    N = rows * cols
    codes = r.integers(0, 1 << nbits, N).astype(np.uint8)
    G = N // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * (1 << nbits)).astype(np.float16)
    return oracle.pack(codes, nbits), scale, zero


@pytest.mark.parametrize("nbits,g,axis", [(4, 64, 1), (3, 64, 1), (2, 16, 1), (4, 32, 0)])
def test_gemv_unit_vectors_give_the_dequantized_columns(nbits, g, axis):
    # x = 2^-3 e_j picks column j of W_hat, scaled exactly: no rounding anywhere
    rows, cols = 48, 128
    packed, scale, zero = _random_quantized(rows, cols, nbits, g, axis, 5)
    Wh = oracle.dequant(packed, scale, zero, rows, cols, nbits, g, axis).astype(np.float64)
    for j in (0, 1, 77, cols - 1):
        x = np.zeros(cols, np.float16)
        x[j] = 0.125
        y, mag = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, axis, x)
        assert np.array_equal(y, Wh[:, j] * 0.125)
        assert np.array_equal(mag, np.abs(Wh[:, j]) * 0.125)


def test_gemv_constant_codes_closed_form():
    # every code k, one (Delta, z) for all groups: W_hat is the constant fp16((k - z) Delta), so
    # y[r] = W_hat * sum(x); x on a 1/8 grid keeps every sum exact in binary64
    rows, cols, nbits, g, k = 16, 256, 4, 64, 11
    codes = np.full(rows * cols, k, np.uint8)
    G = rows * cols // g
    scale = np.full(G, 0.0123, np.float16)
    zero = np.full(G, 7.25, np.float16)
    packed = oracle.pack(codes, nbits)
    x = (np.random.default_rng(3).integers(-32, 33, cols) / 8.0).astype(np.float16)
    w0 = float(np.float16((np.float32(k) - np.float32(zero[0])) * np.float32(scale[0])))
    y, _ = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, x)
    assert np.array_equal(y, np.full(rows, w0 * float(x.astype(np.float64).sum())))


def test_gemv_is_linear_in_x():
    # with x on a coarse grid every partial sum is exact, so linearity holds bit for bit
    rows, cols, nbits, g = 32, 192, 4, 64
    packed, scale, zero = _random_quantized(rows, cols, nbits, g, 1, 9)
    r = np.random.default_rng(4)
    x1 = (r.integers(-8, 9, cols) / 4.0).astype(np.float16)
    x2 = (r.integers(-8, 9, cols) / 4.0).astype(np.float16)
    y1, _ = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, x1)
    y2, _ = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, x2)
    y12, _ = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, (x1 + x2).astype(np.float16))
    assert np.array_equal(y12, y1 + y2)


def test_parallel_timing_build_matches_the_oracle():
    # the benchmark's all-core CPU baseline runs the same source with its round loop spread
    # over threads; the round sums are exact integers, so every output must be identical
    from free_weight_quantization_b200 import workloads as wl
    for W, nbits, g, axis in [(wl.student_t(96, 256, 7), 4, 64, 1), (wl.outlier_normal(64, 96, 3), 3, 32, 0)]:
        a = oracle.quantize(W, nbits, g, axis)
        b = oracle.quantize(W, nbits, g, axis, parallel=True)
        assert a["iters_run"] == b["iters_run"] and a["err_trace"] == b["err_trace"]
        assert np.array_equal(a["codes"], b["codes"])
        assert np.array_equal(a["s"].view(np.uint32), b["s"].view(np.uint32))
        assert np.array_equal(a["z"].view(np.uint32), b["z"].view(np.uint32))
