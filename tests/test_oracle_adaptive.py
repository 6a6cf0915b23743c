"""Pins of the oracle's adaptive per-chunk settings and centroid reuse on the
streaming path (the m.163.com article on Quant VideoGen, section 九: adapt
the compression parameters to the content; section 五: the streaming
centroid cache)."""
import numpy as np
import pytest


def _bits(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_range_stat_hand_examples(ora):
    """Each group contributes the E4M3 code of its range: a range of exactly
    1.0 is code 0x38, 2.0 is 0x40, 0.5 is 0x30, 0 is 0; 448 and more saturate
    at 0x7E."""
    d, G = 16, 8
    X = np.zeros((1, 3, d), np.float32)
    X[0, 0, :8] = np.linspace(-0.5, 0.5, 8)       # range 1.0
    X[0, 0, 8:] = 3.0                              # range 0
    X[0, 1, :8] = [0, 2, 1, 1, 1, 1, 1, 1]          # range 2.0
    X[0, 1, 8:] = [0.25, -0.25] * 4                # range 0.5
    X[0, 2, :8] = [1000, -1000, 0, 0, 0, 0, 0, 0]  # range 2000: saturates
    X[0, 2, 8:] = [7, 7, 7, 7, 7, 7, 7, 7.0]
    assert ora.range_stat(X, G) == 0x38 + 0 + 0x40 + 0x30 + 0x7E + 0
    assert ora.range_stat(_bits(X), G) == 0x38 + 0x40 + 0x30 + 0x7E   # the same values in bf16
    # one group of the whole row: ranges 3.5 (1.75 x 2: code 0x46), 2.25
    # (1.125 x 2: 0x41) and 2000 (saturated)
    assert ora.range_stat(X, 16) == 0x46 + 0x41 + 0x7E


def test_range_stat_grows_with_scale(ora):
    """Doubling every value adds one binade to every range: eight codes per
    group in the normal range."""
    rng = np.random.default_rng(3)
    X = (rng.uniform(0.5, 1.0, (2, 50, 64)) * 4).astype(np.float32)
    n = 2 * 50 * 64 // 16
    assert ora.range_stat(2 * X, 16) - ora.range_stat(X, 16) == 8 * n


def test_adaptive_level_thresholds(ora):
    """Level = the number of ascending thresholds (sixteenths of a code) that
    16 S exceeds relative to the group count; equality does not exceed."""
    th = [16 * 40, 16 * 50, 16 * 60]                # mean codes 40, 50, 60
    n = 1000
    assert ora.adaptive_level(39 * n, n, th, 4) == 0
    assert ora.adaptive_level(40 * n, n, th, 4) == 0
    assert ora.adaptive_level(40 * n + 1, n, th, 4) == 1
    assert ora.adaptive_level(55 * n, n, th, 4) == 2
    assert ora.adaptive_level(61 * n, n, th, 4) == 3
    assert ora.adaptive_level(61 * n, n, th, 2) == 1    # only the first threshold counts with two levels
    assert ora.adaptive_level(10 ** 9, n, th, 1) == 0


@pytest.mark.parametrize("chunk,T_prev,T_cur,refresh,expect", [
    (0, 0, 2, 0, 0),     # the first chunk is cold
    (1, 2, 2, 0, 2),     # same setting: every stage warm
    (1, 1, 4, 0, 1),     # more stages now: only the first is warm
    (3, 4, 1, 0, 1),     # fewer stages now: the first stage warm
    (4, 2, 2, 4, 0),     # a refresh chunk
    (5, 2, 2, 4, 2),
])
def test_warm_stage_rule(ora, chunk, T_prev, T_cur, refresh, expect):
    assert ora.adaptive_warm_stages(chunk, T_prev, T_cur, refresh) == expect


def test_partial_warm_start_composes_warm_and_cold_stages(ora):
    """quantize_ex with the first stage warm and the second cold equals a warm
    one-stage quantisation followed, on its residual, by a cold stage; with
    every stage warm or none it is the plain warm or cold quantisation."""
    rng = np.random.default_rng(9)
    X = rng.standard_normal((1, 300, 32)).astype(np.float32)
    init = rng.standard_normal((2, 1, 8, 32)).astype(np.float32)
    full_warm = ora.quantize_ex(X, K=8, T=2, G=16, iters=4, warm_iters=2, warm_stages=2, init=init)
    ref = ora.quantize(X, K=8, T=2, G=16, iters=2, init=init)
    for k in ref:
        np.testing.assert_array_equal(full_warm[k], ref[k])
    cold = ora.quantize_ex(X, K=8, T=2, G=16, iters=4, warm_iters=2, warm_stages=0)
    ref = ora.quantize(X, K=8, T=2, G=16, iters=4)
    for k in ref:
        np.testing.assert_array_equal(cold[k], ref[k])
    mixed = ora.quantize_ex(X, K=8, T=2, G=16, iters=4, warm_iters=2, warm_stages=1, init=init)
    C1, pi1 = ora.kmeans(X[0], init[0, 0], 2, dtype=1)
    R1 = ora.residual(X[0], C1, pi1, dtype=1)
    C2, pi2 = ora.kmeans(R1, R1[:8], 4, dtype=1)
    np.testing.assert_array_equal(mixed["centroids"][0, 0], C1)
    np.testing.assert_array_equal(mixed["centroids"][1, 0], C2)
    np.testing.assert_array_equal(mixed["assign"][:, 0], np.stack([pi1, pi2]))
