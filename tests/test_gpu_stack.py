"""The 7B-like stack: 32 layers of 4 fp16 4096x4096 and 3 fp16 4096x11008 matrices, entries
0.02*StudentT(4) clipped to +-1, drawn on the GPU from per-matrix seeds.  Every matrix is
quantized (4-bit, group 64, axis 1, its own early stop) and dequantized through the C ABI.

Three matrices, copied back to the host, are compared with the oracle: the first, a middle
and the last layer, both shapes.  Each of the others is checked for properties that hold at
any size:
  - the iteration count lies in 1..20;
  - the reconstruction is no worse than the round-to-nearest start (iters = 0), since the
    loop keeps the best measured zero;
  - the dequantized weights are finite.
"""
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np
import pytest

import parity
from free_weight_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SAMPLED = [(0, 0), (15, 4), (31, 6)]


@pytest.fixture(scope="module")
def hqq():
    from free_weight_quantization_b200 import build
    build.build()
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    from free_weight_quantization_b200 import hqq as h
    return h


def test_stack_every_matrix_and_sampled_oracle_parity(hqq):
    ex = cf.ProcessPoolExecutor(max_workers=min(3, os.cpu_count() or 1),
                                mp_context=mp.get_context("spawn"))
    try:
        jobs = {}
        n_mat = 0
        for layer in range(wl.STACK_LAYERS):
            for index in range(len(wl.STACK_SHAPES)):
                W = wl.stack_matrix_torch(layer, index, "cuda")
                q = hqq.hqq_quantize(W, 4, 64, 1, debug=True)
                deq = hqq.hqq_dequantize(q)
                q0 = hqq.hqq_quantize(W, 4, 64, 1, iters=0)
                deq0 = hqq.hqq_dequantize(q0)
                Wf = W.float()
                mae = (deq.float() - Wf).abs().mean().item()
                mae0 = (deq0.float() - Wf).abs().mean().item()
                n = int(q.iters_run.item())
                assert 1 <= n <= 20, (layer, index, n)
                assert np.isfinite(mae) and mae <= mae0 * 1.001, (layer, index, mae, mae0)
                if (layer, index) in SAMPLED:
                    Wh = W.cpu().numpy()
                    jobs[(layer, index)] = (Wh, ex.submit(parity.oracle_on, Wh, 4, 64, 1))
                n_mat += 1
        assert n_mat == wl.STACK_LAYERS * len(wl.STACK_SHAPES) == 224
        for key, (Wh, fut) in jobs.items():
            got = parity.gpu_quantize(Wh, 4, 64, 1)
            stats = parity.check(Wh, fut.result(), got, f"stack layer {key[0]} matrix {key[1]}")
            print("stack", key, got["iters_run"], stats)
    finally:
        ex.shutdown(cancel_futures=True)
