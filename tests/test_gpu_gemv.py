"""Fused dequant-GEMV (hqq_gemv) against the oracle's y = W_hat @ x in binary64.

W_hat is the fp16 dequantized weight in both.  Each product of two fp16 values is exact in
binary32, so the GPU result differs from the exact sum only by the rounding of its binary32
summation, whatever its order: |y - y_ref| <= cols * 2^-24 * sum_c |W_hat x| to first order.
The bound is checked at twice that.
"""
import numpy as np
import pytest

import oracle
import parity
from free_weight_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def hqq():
    from free_weight_quantization_b200 import build
    build.build()
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    from free_weight_quantization_b200 import hqq as h
    return h


def _check(y, ref, mag, cols, label):
    err = np.abs(y.astype(np.float64) - ref)
    bound = 2.0 * cols * 2.0 ** -24 * mag + 1e-30
    assert (err <= bound).all(), (label, float((err / bound).max()))


def _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, axis):
    buf = np.zeros((packed.size + 15) // 16 * 16, np.uint8)
    buf[:packed.size] = packed
    return hqq.Quantized(torch.from_numpy(buf).cuda(), torch.from_numpy(scale).cuda(),
                         torch.from_numpy(zero).cuda(), rows, cols, nbits, g, axis)


# fast path: axis 1, 2/4 bit, cols and g multiples of the codes per word; the rest generic
LAYOUTS = [(4, 64, 1, 96, 512), (2, 16, 1, 64, 256), (4, 128, 1, 33, 1024), (2, 64, 1, 17, 320),
           (3, 64, 1, 40, 640), (3, 10, 1, 21, 130), (4, 64, 0, 64, 192), (2, 16, 0, 48, 80),
           (4, 3, 1, 30, 21), (4, 24, 1, 12, 96),
           # one word per row, a ragged last CTA of rows, the largest group, one row
           (4, 8, 1, 7, 8), (2, 16, 1, 1, 16), (4, 256, 1, 9, 4096), (2, 256, 1, 3, 8192),
           # the other code widths (generic path): 1 bit eight per byte, 5 to 8 bit one per byte
           (1, 64, 1, 16, 512), (1, 32, 0, 24, 100), (5, 32, 1, 20, 256), (6, 64, 0, 64, 96),
           (7, 16, 1, 8, 64), (8, 64, 1, 33, 192),
           # axis-1 groups that cross rows (cols % g != 0): the generic path
           (4, 64, 1, 40, 96), (2, 32, 1, 30, 48),
           # 16 MiB of codes and more: the bulk-copy kernel; 8195 rows end in a 3-row stage
           # whose 195 metadata halves are not whole 16-byte units (65 groups per row)
           (4, 64, 1, 8195, 4160), (2, 64, 1, 8192, 8192),
           # axis 0, 4 bit, g dividing rows: per-code metadata by row (stripes of R = rows / g)
           (4, 32, 0, 96, 64), (4, 8, 0, 40, 320),
           # 3 bit, axis 1: rows that start and end inside a 10-code word, groups not a
           # multiple of 10
           (3, 64, 1, 16, 1004), (3, 12, 1, 7, 96)]


@pytest.mark.parametrize("nbits,g,axis,rows,cols", LAYOUTS, ids=lambda v: str(v))
def test_gemv_random_codes(hqq, nbits, g, axis, rows, cols):
    r = np.random.default_rng(rows * cols + nbits)
    N = rows * cols
    codes = r.integers(0, 1 << nbits, N).astype(np.uint8)
    G = N // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * (1 << nbits)).astype(np.float16)
    packed = oracle.pack(codes, nbits)
    x = r.standard_normal(cols).astype(np.float16)
    ref, mag = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, axis, x)
    q = _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, axis)
    y = hqq.hqq_gemv(q, torch.from_numpy(x).cuda()).cpu().numpy()
    _check(y, ref, mag, cols, (nbits, g, axis, rows, cols))


def test_gemv_large_x(hqq):
    # x near the fp16 range: products up to ~1e5, still exact in binary32 before the sum
    rows, cols, nbits, g = 24, 512, 4, 64
    r = np.random.default_rng(13)
    packed = oracle.pack(r.integers(0, 16, rows * cols).astype(np.uint8), nbits)
    G = rows * cols // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * 16).astype(np.float16)
    x = (r.standard_normal(cols) * 2e4).clip(-6e4, 6e4).astype(np.float16)
    ref, mag = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, x)
    q = _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, 1)
    y = hqq.hqq_gemv(q, torch.from_numpy(x).cuda()).cpu().numpy()
    _check(y, ref, mag, cols, "large x")


def test_gemv_unaligned_x_takes_the_generic_path(hqq):
    rows, cols, nbits, g = 40, 256, 4, 64
    r = np.random.default_rng(7)
    packed = oracle.pack(r.integers(0, 16, rows * cols).astype(np.uint8), nbits)
    G = rows * cols // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * 16).astype(np.float16)
    x = r.standard_normal(cols).astype(np.float16)
    ref, mag = oracle.gemv(packed, scale, zero, rows, cols, nbits, g, 1, x)
    q = _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, 1)
    xd = torch.zeros(cols + 1, dtype=torch.float16, device="cuda")
    xd[1:] = torch.from_numpy(x).cuda()
    y = hqq.hqq_gemv(q, xd[1:]).cpu().numpy()             # x 2-byte but not 16-byte aligned
    _check(y, ref, mag, cols, "unaligned x")


@pytest.mark.parametrize("case", [wl.ATTN, wl.MLP_B2, wl.MLP_B3, wl.ATTN_AX0], ids=lambda c: c.name)
def test_gemv_on_quantized_workload(hqq, case):
    # the full-size workload quantized on the GPU, then the fused product against the oracle's
    # product of the same packed codes and metadata
    W = case.make()
    got = parity.gpu_quantize(W, case.nbits, case.group_size, case.axis)
    q = got["q"]
    x = np.random.default_rng(11).standard_normal(case.cols).astype(np.float16)
    y = hqq.hqq_gemv(q, torch.from_numpy(x).cuda()).cpu().numpy()
    ref, mag = oracle.gemv(got["packed"], got["scale"], got["zero"], case.rows, case.cols,
                           case.nbits, case.group_size, case.axis, x)
    _check(y, ref, mag, case.cols, case.name)
