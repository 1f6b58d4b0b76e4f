"""The batched forward product (hqq_gemm) against the oracle's y = W_hat @ x, row by row.

W_hat is the fp16 dequantized weight in both.  Each product of two fp16 values is exact in
binary32, so the GPU result differs from the exact sum only by its binary32 accumulation,
whatever its order or the tensor cores' rounding of partial sums: the check allows
cols * 2^-23 * sum_c |W_hat x| per element.  Axis-1 2- and 4-bit layouts with cols a multiple
of 64 run the tcgen05 tensor-core kernel when the batch has two entries or more; a batch of one
and the other layouts the one-vector product per batch entry.
"""
import numpy as np
import pytest

import oracle
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


def _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, axis):
    buf = np.zeros((packed.size + 15) // 16 * 16, np.uint8)
    buf[:packed.size] = packed
    return hqq.Quantized(torch.from_numpy(buf).cuda(), torch.from_numpy(scale).cuda(),
                         torch.from_numpy(zero).cuda(), rows, cols, nbits, g, axis)


def _check(Y, ref, mag, cols, label):
    err = np.abs(Y.astype(np.float64) - ref)
    bound = cols * 2.0 ** -23 * mag + 1e-30
    assert np.isfinite(Y).all(), label
    assert (err <= bound).all(), (label, float((err / bound).max()))


# (nbits, group_size, axis, rows, cols, batch): tensor-core layouts first (one tile, split
# columns, ragged row block, the largest MMA N, more than one launch of batch entries, 2 bit),
# then layouts on the generic path
CASES = [(4, 64, 1, 128, 64, 2), (4, 64, 1, 128, 64, 1), (4, 64, 1, 256, 512, 2), (4, 64, 1, 200, 1024, 7),
         (4, 128, 1, 384, 2048, 16), (4, 32, 1, 128, 256, 33), (4, 64, 1, 512, 1024, 256),
         (4, 64, 1, 256, 512, 300), (2, 16, 1, 256, 1024, 5), (2, 64, 1, 130, 128, 64),
         (4, 8, 1, 128, 128, 3),
         (3, 64, 1, 64, 640, 4), (4, 64, 0, 64, 192, 3), (4, 64, 1, 40, 96, 2), (5, 32, 1, 32, 128, 2),
         (4, 128, 1, 96, 192, 4)]  # groups cross rows (192 % 128 != 0): generic


@pytest.mark.parametrize("nbits,g,axis,rows,cols,batch", CASES, ids=lambda v: str(v))
def test_gemm_random_codes(hqq, nbits, g, axis, rows, cols, batch):
    r = np.random.default_rng(rows * cols + nbits + batch)
    N = rows * cols
    codes = r.integers(0, 1 << nbits, N).astype(np.uint8)
    G = N // g
    scale = (r.random(G) * 0.05 + 1e-3).astype(np.float16)
    zero = (r.random(G) * (1 << nbits)).astype(np.float16)
    packed = oracle.pack(codes, nbits)
    X = r.standard_normal((batch, cols)).astype(np.float16)
    ref, mag = oracle.gemm(packed, scale, zero, rows, cols, nbits, g, axis, X)
    q = _gpu_q(hqq, packed, scale, zero, rows, cols, nbits, g, axis)
    Y = hqq.hqq_gemm(q, torch.from_numpy(X).cuda()).cpu().numpy()
    assert Y.shape == (batch, rows)
    _check(Y, ref, mag, cols, (nbits, g, axis, rows, cols, batch))


def test_gemm_matches_the_one_vector_product_and_batch_zero(hqq):
    # a batch of one takes the one-vector product (same bits); a batch of two the tensor cores,
    # each row within the bound of the oracle's product; an empty batch launches nothing
    W = torch.from_numpy(wl.student_t(512, 1024, seed=4)).cuda()
    q = hqq.hqq_quantize(W, 4, 64, 1)
    X = torch.randn(2, 1024, device="cuda").to(torch.float16)
    y1 = hqq.hqq_gemm(q, X[:1])[0].cpu().numpy()
    assert np.array_equal(y1.view(np.uint32), hqq.hqq_gemv(q, X[0]).cpu().numpy().view(np.uint32))
    Y2 = hqq.hqq_gemm(q, X).cpu().numpy().astype(np.float64)
    for b in range(2):
        ref, mag = oracle.gemv(q.packed.cpu().numpy()[:oracle.packed_bytes(512 * 1024, 4)],
                               q.scale.cpu().numpy(), q.zero.cpu().numpy(), 512, 1024, 4, 64, 1,
                               X[b].cpu().numpy())
        assert (np.abs(Y2[b] - ref) <= 1024 * 2.0 ** -23 * mag + 1e-30).all()
    out = hqq.hqq_gemm(q, torch.empty(0, 1024, dtype=torch.float16, device="cuda"))
    assert out.shape == (0, 512)


def test_gemm_full_size_workload(hqq):
    # the 4096x4096 4-bit g64 matrix quantized on the GPU, a batch of 8, against the oracle's
    # product of the same codes
    c = wl.ATTN
    W = torch.from_numpy(c.make()).cuda()
    q = hqq.hqq_quantize(W, c.nbits, c.group_size, c.axis)
    X = torch.randn(8, c.cols, device="cuda").to(torch.float16)
    Y = hqq.hqq_gemm(q, X).cpu().numpy()
    ref, mag = oracle.gemm(q.packed.cpu().numpy()[:oracle.packed_bytes(c.n, c.nbits)],
                           q.scale.cpu().numpy(), q.zero.cpu().numpy(), c.rows, c.cols, c.nbits,
                           c.group_size, c.axis, X.cpu().numpy())
    _check(Y, ref, mag, c.cols, "4096x4096 batch 8")
