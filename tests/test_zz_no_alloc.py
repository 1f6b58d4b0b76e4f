"""hqq_quantize_noalloc: the quantize entry point for callers that cannot allocate device
memory (plugins whose host framework owns the GPU's memory pool, loops that must never call
cudaMalloc).  It must give exactly what hqq_quantize gives with a caller-provided workspace,
call after call, although every call reuses the same built-in scratch buffer.

This file is collected last on purpose (pytest takes files in name order), so a failure here
comes after every other test has run.
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


def _outputs(h, rows, cols, nbits, g, iters, axis=1):
    N, G = rows * cols, rows * cols // g
    dev = "cuda"
    return h.Quantized(torch.empty(max(oracle.packed_bytes(N, nbits), 1), dtype=torch.uint8, device=dev),
                       torch.empty(G, dtype=torch.float16, device=dev),
                       torch.empty(G, dtype=torch.float16, device=dev), rows, cols, nbits, g, axis,
                       torch.zeros(1, dtype=torch.int32, device=dev),
                       torch.empty(G, dtype=torch.float32, device=dev),
                       torch.empty(G, dtype=torch.float32, device=dev),
                       torch.zeros(2 * iters, dtype=torch.int64, device=dev),
                       torch.empty(G, dtype=torch.uint8, device=dev))


def _same(a, b):
    for f in ("packed", "scale", "zero", "iters_run", "s", "z", "rounds"):
        x, y = getattr(a, f), getattr(b, f)
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.float16 else x,
                           y.view(torch.uint8) if y.dtype == torch.float16 else y), f
    n = int(a.iters_run.item())
    assert torch.equal(a.err_trace[:2 * n], b.err_trace[:2 * n])


def _matches_oracle(h, q, Wn, nbits, g, axis):
    o = oracle.quantize(Wn, nbits, g, axis)
    n = int(q.iters_run.item())
    assert n == o["iters_run"]
    assert h.err_trace_ints(q.err_trace, n) == o["err_trace"]
    assert np.array_equal(q.packed.cpu().numpy()[:o["packed"].size], o["packed"])
    assert np.array_equal(q.scale.cpu().numpy().view(np.uint16), o["scale"].view(np.uint16))
    assert np.array_equal(q.zero.cpu().numpy().view(np.uint16), o["zero"].view(np.uint16))


@pytest.mark.parametrize("case", [wl.SMALL, wl.MLP_B2], ids=lambda c: c.name)
def test_noalloc_matches_workspace_entry_point_twice(hqq, case):
    # two calls in a row on different matrices: the second must not see the first's scratch
    rows, cols = (case.rows, case.cols) if case.n <= 1 << 20 else (1024, case.cols)
    mats = [case.make()[:rows, :cols], wl.student_t(rows, cols, seed=99)]
    out = _outputs(hqq, rows, cols, case.nbits, case.group_size, 20)
    for i, Wn in enumerate(mats):
        W = torch.from_numpy(np.ascontiguousarray(Wn)).cuda()
        ref = hqq.hqq_quantize(W, case.nbits, case.group_size, 1, iters=20, debug=True)
        free_before = torch.cuda.mem_get_info()[0]
        hqq.hqq_quantize_noalloc(W, case.nbits, case.group_size, 1, iters=20, out=out)
        torch.cuda.synchronize()
        if i > 0:  # after the first call (which may load the library's module) nothing grows
            assert torch.cuda.mem_get_info()[0] == free_before
        _same(ref, out)
        if rows * cols <= 1 << 20:  # and both are the oracle's result
            _matches_oracle(hqq, out, np.ascontiguousarray(Wn), case.nbits, case.group_size, 1)


# the tile engine's paths: 3-bit codes; axis 0 with a group count (300) that is not a multiple
# of the 8 codes of a packed word, so that the codes go through byte staging in the scratch
@pytest.mark.parametrize("rows,cols,nbits,g,axis", [(64, 640, 3, 64, 1), (128, 300, 4, 128, 0)],
                         ids=["3bit-g64", "axis0-g128-G300"])
def test_noalloc_tile_paths_twice(hqq, rows, cols, nbits, g, axis):
    assert hqq.hqq_quantize_workspace_bytes(rows, cols, nbits, g, axis, 20) <= hqq.HQQ_NOALLOC_SCRATCH_BYTES
    out = _outputs(hqq, rows, cols, nbits, g, 20, axis)
    for Wn in [wl.student_t(rows, cols, seed=5), wl.outlier_normal(rows, cols, seed=6)]:
        W = torch.from_numpy(np.ascontiguousarray(Wn)).cuda()
        ref = hqq.hqq_quantize(W, nbits, g, axis, iters=20, debug=True)
        hqq.hqq_quantize_noalloc(W, nbits, g, axis, iters=20, out=out)
        torch.cuda.synchronize()
        _same(ref, out)
        _matches_oracle(hqq, out, np.ascontiguousarray(Wn), nbits, g, axis)


def test_noalloc_rejects_problems_beyond_its_scratch(hqq):
    # axis 0 with 2.1 M groups whose packed rows do not line up with tiles needs byte staging
    # of all 4.2 M codes: more than the 4 MiB buffer.  Rejected on the host, nothing launched.
    rows, cols, g = 4100, 1030, 2
    need = hqq.hqq_quantize_workspace_bytes(rows, cols, 4, g, 0, 20)
    assert need > hqq.HQQ_NOALLOC_SCRATCH_BYTES
    import ctypes
    rc = hqq.lib().hqq_quantize_noalloc(ctypes.c_void_p(0x10000), rows, cols, 4, g, 0, None,
                                        ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000),
                                        ctypes.c_void_p(0x10000), None, None, None, None, None,
                                        None)
    assert rc == 3
