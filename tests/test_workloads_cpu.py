"""The seeded synthetic inputs follow their stated recipes (no GPU).

Every parity test and the bench feed these bytes to both the oracle and the CUDA path, so the
recipes are pinned here: shapes, seeds, distribution parameters and determinism.
"""
import numpy as np

from free_weight_quantization_b200 import workloads as wl


def test_cases_have_the_stated_shapes_and_settings():
    got = [(c.rows, c.cols, c.nbits, c.group_size, c.axis, c.seed) for c in wl.CASES]
    assert got == [(256, 512, 4, 64, 1, 0), (4096, 4096, 4, 64, 1, 1), (4096, 11008, 2, 16, 1, 2),
                   (4096, 11008, 3, 64, 1, 2), (4096, 4096, 4, 128, 0, 3)]
    for c in wl.CASES:
        assert c.n % c.group_size == 0


def test_generation_is_deterministic_fp16():
    for c in (wl.SMALL, wl.ATTN):
        a, b = c.make(), c.make()
        assert a.dtype == np.float16 and a.shape == (c.rows, c.cols)
        assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_outlier_normal_recipe():
    W = wl.SMALL.make().astype(np.float64)
    k = int(np.floor(0.001 * W.size))            # 131 outliers of magnitude U(0.2, 1.0)
    big = np.abs(W) >= 0.2 - 1e-3
    assert big.sum() == k
    assert np.abs(W[big]).max() <= 1.0 + 1e-3
    assert abs(W[~big].std() - 0.02) < 0.001    # the N(0, 0.02^2) bulk


def test_student_t_recipe():
    W = wl.ATTN.make().astype(np.float64)
    assert np.abs(W).max() <= 1.0                # clipped to +-1
    # 0.02 * StudentT(4): variance 0.02^2 * 4/(4-2), so std 0.0283 (the clip barely moves it)
    assert abs(W.std() - 0.02 * np.sqrt(2.0)) < 0.001
    assert abs(np.median(W)) < 1e-3


def test_row_lognormal_recipe():
    W = wl.MLP_B2.make().astype(np.float64)
    row_std = W.std(axis=1)
    # per-row scale LogNormal(0, 0.3) times N(0, 0.015^2): log of the row std has spread 0.3
    assert abs(np.log(row_std).std() - 0.3) < 0.02
    assert abs(np.exp(np.log(row_std).mean()) - 0.015) < 0.001


def test_stack_seeds_are_distinct_and_follow_the_formula():
    seeds = {wl.stack_seed(l, i) for l in range(wl.STACK_LAYERS) for i in range(len(wl.STACK_SHAPES))}
    assert len(seeds) == 224
    assert wl.stack_seed(0, 0) == 16000 and wl.stack_seed(31, 6) == (1000 + 31) * 16 + 6
