"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200)."""
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np
import pytest

import oracle
import parity
from free_weight_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def pool():
    # spawn: a forked child of a process that has touched CUDA can hang
    ex = cf.ProcessPoolExecutor(max_workers=min(4, os.cpu_count() or 1),
                                mp_context=mp.get_context("spawn"))
    yield ex
    ex.shutdown(cancel_futures=True)


@pytest.fixture(scope="module", autouse=True)
def built():
    from free_weight_quantization_b200 import build
    build.build()
    assert torch.cuda.is_available(), "these tests need a CUDA device"


def _bimodal(rows, cols, seed):
    r = np.random.default_rng(seed)
    return (np.where(r.random((rows, cols)) < 0.5, -1.0, 1.0)
            * (1 + 0.01 * r.standard_normal((rows, cols)))).astype(np.float16)


def _sparse(rows, cols, seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((rows, cols)) * (r.random((rows, cols)) < 0.1)).astype(np.float16)


def _wide(rows, cols, seed):
    return (np.random.default_rng(seed).standard_normal((rows, cols)) * 3.0).astype(np.float16)


def _const(rows, cols, seed):
    W = np.full((rows, cols), 0.375, np.float16)
    W[rows // 2:] = -1.25
    return W


def _tiny_range(rows, cols, seed):
    r = np.random.default_rng(seed)
    W = 0.5 + r.integers(0, 3, (rows, cols)) * 2.0 ** -11     # ranges of 0 .. 1e-3
    return W.astype(np.float16)


def _negative(rows, cols, seed):
    # every group entirely negative and far from 0: z0 = -min*s is large and positive
    r = np.random.default_rng(seed)
    return (-1000.0 - 24.0 * r.random((rows, cols))).astype(np.float16)


def _positive(rows, cols, seed):
    # every group entirely positive, offset per row: z0 is large and negative
    r = np.random.default_rng(seed)
    base = r.uniform(0.5, 600.0, (rows, 1))
    return (base + r.standard_normal((rows, cols)) * 0.01 * base).astype(np.float16)


GENS = {"t": wl.student_t, "n": wl.outlier_normal, "bimodal": _bimodal, "sparse": _sparse,
        "wide": _wide, "const": _const, "tiny": _tiny_range, "neg": _negative, "pos": _positive}

# rows, cols, nbits, group_size, axis, iters, generator
EDGE = [
    (1, 64, 4, 64, 1, 20, "t"),          # one group
    (1, 64, 4, 64, 1, 20, "const"),
    (4, 64, 4, 64, 1, 20, "tiny"),        # ranges around eps_tiny: s = 1 or clamped 2e4
    (3, 160, 3, 16, 1, 20, "t"),
    (7, 33, 4, 3, 1, 20, "t"),            # g = 3, odd N (last nibble), many tiles of 320 groups
    (5, 50, 3, 25, 1, 7, "t"),
    (9, 100, 2, 12, 1, 20, "t"),
    (64, 96, 4, 48, 1, 20, "t"),          # group padded to 64 slots
    (16, 4096, 4, 256, 1, 20, "t"),       # largest group
    (64, 64, 4, 64, 1, 0, "t"),           # no rounds: min-max RTN
    (64, 64, 4, 64, 1, 1, "t"),
    (64, 128, 4, 64, 1, 64, "t"),         # most rounds
    (64, 256, 4, 64, 1, 20, "wide"),      # lp shrink active
    (64, 256, 2, 16, 1, 20, "wide"),
    (64, 256, 3, 64, 1, 20, "wide"),
    (64, 256, 4, 64, 1, 20, "bimodal"),   # early global stop: stale groups are recomputed
    (64, 256, 2, 16, 1, 20, "bimodal"),
    (64, 256, 3, 64, 1, 20, "bimodal"),
    (64, 256, 4, 32, 1, 20, "sparse"),
    (300, 512, 4, 64, 1, 20, "n"),        # 15 tiles
    (333, 64, 3, 64, 1, 20, "t"),         # ragged last tile
    (256, 128, 4, 128, 0, 20, "t"),       # axis 0, aligned
    (128, 80, 3, 16, 0, 20, "t"),         # axis 0, G = 640
    (32, 64, 2, 32, 0, 20, "t"),          # axis 0, G = 64
    (30, 32, 4, 16, 0, 20, "t"),          # axis 0, G = 60: byte staging + pack kernel
    (40, 41, 3, 8, 0, 20, "t"),           # axis 0, G = 205, odd
    (64, 256, 4, 64, 0, 20, "bimodal"),
    (64, 256, 4, 64, 0, 20, "wide"),
    (64, 256, 4, 64, 1, 20, "neg"),       # one-signed groups far from 0: large |z|
    (64, 256, 2, 16, 1, 20, "pos"),
    (64, 256, 3, 64, 1, 20, "neg"),
    (64, 256, 4, 64, 0, 20, "pos"),
    # the other code widths: 1 bit (eight per byte), 5 to 8 bit (one per byte)
    (64, 256, 1, 64, 1, 20, "t"),
    (33, 96, 1, 32, 0, 20, "t"),           # axis 0, G = 99: byte staging + pack kernel
    (64, 256, 5, 64, 1, 20, "t"),
    (40, 160, 6, 32, 1, 20, "n"),
    (64, 256, 7, 128, 0, 20, "t"),
    (64, 256, 8, 64, 1, 20, "t"),
    (48, 100, 8, 25, 1, 20, "wide"),       # odd group, shrink active
    (64, 256, 6, 64, 1, 20, "bimodal"),    # early global stop with 6-bit codes
    (64, 256, 8, 64, 1, 0, "t"),           # no rounds: min-max RTN at 8 bit
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "x".join(map(str, c)))
def test_edge_case(case):
    rows, cols, nbits, g, axis, iters, gen = case
    W = GENS[gen](rows, cols, 17 + rows)
    ref = parity.oracle_on(W, nbits, g, axis, iters)
    got = parity.gpu_quantize(W, nbits, g, axis, iters)
    parity.check(W, ref, got, str(case))


def test_small_config_and_repeat():
    c = wl.SMALL
    W = c.make()
    ref = parity.oracle_on(W, c.nbits, c.group_size, c.axis)
    a = parity.gpu_quantize(W, c.nbits, c.group_size, c.axis)
    parity.check(W, ref, a, c.name)
    b = parity.gpu_quantize(W, c.nbits, c.group_size, c.axis)  # repeat: deterministic
    assert np.array_equal(a["packed"], b["packed"]) and np.array_equal(a["deq"], b["deq"])


@pytest.mark.parametrize("case", wl.CASES[1:], ids=lambda c: c.name)
def test_full_size_config(case, pool):
    fut = pool.submit(parity.oracle_job, case.name)
    W = case.make()
    got = parity.gpu_quantize(W, case.nbits, case.group_size, case.axis)
    ref = fut.result()
    stats = parity.check(W, ref, got, case.name)
    print(case.name, ref["iters_run"], stats)


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("shape,g,axis", [((64, 64), 64, 1), ((37, 129), 3, 1), ((100, 7), 10, 1),
                                          ((256, 64), 128, 0), ((30, 32), 16, 0),
                                          ((41, 40), 8, 0),
                                          # 3-bit, groups of 40 and more: four words per thread,
                                          # groups that straddle them, a ragged last unit
                                          ((33, 200), 40, 1), ((7, 130), 65, 1), ((96, 160), 96, 1),
                                          # axis 0, 4-bit metadata reuse: g = 24 rows (a short
                                          # last run of words per thread), 128 groups
                                          ((24, 128), 24, 0)])
def test_dequant_random_codes(nbits, shape, g, axis):
    from free_weight_quantization_b200 import hqq
    rows, cols = shape
    N = rows * cols
    r = np.random.default_rng(N + nbits)
    codes = r.integers(0, 1 << nbits, N).astype(np.uint8)
    packed = oracle.pack(codes, nbits)
    G = N // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * (1 << nbits)).astype(np.float16)
    ref = oracle.dequant(packed, scale, zero, rows, cols, nbits, g, axis)
    buf = np.zeros((packed.size + 15) // 16 * 16, np.uint8)
    buf[:packed.size] = packed
    q = hqq.Quantized(torch.from_numpy(buf).cuda(), torch.from_numpy(scale).cuda(),
                      torch.from_numpy(zero).cuda(), rows, cols, nbits, g, axis)
    out = hqq.hqq_dequantize(q).cpu().numpy()
    assert np.array_equal(out.view(np.uint16), ref.view(np.uint16))


def test_native_library_is_loaded():
    from free_weight_quantization_b200 import hqq
    hqq.lib()
    maps = open("/proc/self/maps").read()
    assert "libhqq_b200.so" in maps
