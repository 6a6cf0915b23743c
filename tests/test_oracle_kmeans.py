"""Pins of the oracle's k-means (semantic-aware smoothing: m.163.com article on
Quant VideoGen, section 三; gist.science/de, Technische Zusammenfassung 2A):
a hand-worked example, exact-rational brute force, the K = N special case,
the monotone objective, tie and empty-cluster readings."""
from fractions import Fraction

import numpy as np
import pytest

BF16, FP32 = 0, 1


def _bf16(x):
    """Round float64 values to bf16-representable float32 (test helper, via
    the torch library cast from fp32; inputs here are exact in fp32)."""
    import torch
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def test_worked_example_2d(ora):
    """Hand-worked Lloyd run.  Points a=(0,0) b=(0,1) c=(5,10) e=(5,11), K=2,
    initial centroids = first two points.
    it 1: a->0, b->1 (D(b,c0)=1, D(b,c1)=0), c->1 (125 vs 106),
          e->1 (146 vs 125); means c0=(0,0), c1=(10/3, 22/3).
    it 2: b->0 (1 vs 51.2), c->1 (125 vs 9.89), e->1; means c0=(0,.5), c1=(5,10.5).
    it 3: unchanged.  Final objective 4 * 0.25 = 1."""
    X = np.array([[0, 0], [0, 1], [5, 10], [5, 11]], np.float32)
    for dtype in (FP32, BF16):
        C, pi, tr = ora.kmeans(X, X[:2], 3, dtype=dtype, trace=True)
        np.testing.assert_array_equal(pi, [0, 0, 1, 1])
        np.testing.assert_array_equal(C, [[0, 0.5], [5, 10.5]])
        assert tr[0] == 0 + 0 + 106 + 125          # after first assignment
        assert tr[-1] == 1.0
    # one iteration only: the intermediate means
    C, pi = ora.kmeans(X, X[:2], 1, dtype=FP32)
    np.testing.assert_array_equal(pi, [0, 1, 1, 1])
    np.testing.assert_array_equal(C, np.array([[0, 0], [10 / 3, 22 / 3]], np.float32))


def _exact_argmin(r, C):
    best, bk = None, None
    for k, c in enumerate(C):
        D = sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(r, c))
        if best is None or D < best:
            best, bk = D, k
    return bk


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_assign_matches_exact_rational_brute_force(ora, seed):
    rng = np.random.default_rng(seed)
    N, K, d = 60, 7, 6
    X = _bf16(rng.standard_normal((N, d)) * np.exp(rng.standard_normal(d)))
    C = _bf16(rng.standard_normal((K, d)))
    C[3] = C[5]                                   # exact duplicate -> ties
    X[10] = C[5]                                  # token on a duplicated centroid
    pi = ora.assign(X, C)
    expect = [_exact_argmin(X[i], C) for i in range(N)]
    np.testing.assert_array_equal(pi, expect)
    assert pi[10] == 3                            # lowest index wins the tie


def _bf16_nearest(fr):
    """Nearest bf16 to an exact rational, ties to even (test-side definition)."""
    f = float(fr)
    t = int(np.float32(abs(f)).view(np.uint32) >> 16)
    best = min((c for c in (t - 1, t, t + 1) if c >= 0),
               key=lambda c: (abs(Fraction(float((np.uint32(c) << 16).view(np.float32))) - abs(fr)), c & 1))
    v = float((np.uint32(best) << 16).view(np.float32))
    return -v if fr < 0 else v


def test_update_is_rounded_exact_mean(ora):
    rng = np.random.default_rng(5)
    N, K, d = 200, 9, 4
    X = _bf16(rng.standard_normal((N, d)) * 10.0 ** rng.uniform(-3, 3, (N, d)))
    pi = rng.integers(0, K - 1, N).astype(np.uint8)   # cluster K-1 stays empty
    C0 = _bf16(rng.standard_normal((K, d)))
    C = ora.update(X, pi, C0, dtype=BF16)
    for k in range(K):
        members = X[pi == k]
        if len(members) == 0:
            np.testing.assert_array_equal(C[k], C0[k])   # empty keeps previous
            continue
        for j in range(d):
            mean = sum(Fraction(float(v)) for v in members[:, j]) / len(members)
            assert C[k, j] == np.float32(_bf16_nearest(mean)), (k, j)
    Cf = ora.update(X, pi, C0, dtype=FP32)
    for k in range(K - 1):
        members = X[pi == k]
        mean = sum(Fraction(float(v)) for v in members[:, 0]) / len(members)
        got = Cf[k, 0]
        err = abs(Fraction(float(got)) - mean)
        for nb in (np.nextafter(got, np.float32(np.inf)), np.nextafter(got, np.float32(-np.inf))):
            assert err <= abs(Fraction(float(nb)) - mean)   # nearest fp32


@pytest.mark.parametrize("dtype", [BF16, FP32])
def test_k_equals_n_gives_zero_residual(ora, dtype):
    rng = np.random.default_rng(7)
    N = d = 16
    X = rng.standard_normal((N, d)).astype(np.float32)
    if dtype == BF16:
        X = _bf16(X)
    C, pi = ora.kmeans(X, X, 4, dtype=dtype)
    np.testing.assert_array_equal(pi, np.arange(N))
    np.testing.assert_array_equal(C, X)
    R = ora.residual(X, C, pi, dtype=dtype)
    assert np.all(R == 0)


@pytest.mark.parametrize("dtype", [BF16, FP32])
def test_objective_never_increases(ora, dtype):
    """Each assignment and each update can only lower J; for bf16 centroids
    the componentwise-nearest rounding of the mean keeps this exact."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(1, synth.KVShape(2, 12, 16), seed=11, kinds=[1]).float().numpy()[0]
    if dtype == FP32:
        X = X + np.float32(1e-3) * np.random.default_rng(0).standard_normal(X.shape).astype(np.float32)
    K = 32
    _, _, tr = ora.kmeans(X, X[:K], 8, dtype=dtype, trace=True)
    assert np.all(np.diff(tr) <= 1e-12 * tr[0]), tr
    assert tr[-1] < tr[0]


def test_empty_cluster_keeps_centroid(ora):
    X = np.array([[0, 0], [0, 1], [1, 0], [1, 1]], np.float32)
    C0 = np.array([[0.5, 0.5], [100, 100]], np.float32)
    C, pi = ora.kmeans(X, C0, 3, dtype=FP32)
    np.testing.assert_array_equal(pi, [0, 0, 0, 0])
    np.testing.assert_array_equal(C, C0)


def test_sqdist_is_fp64_sum_in_channel_order(ora):
    r = np.array([1e8, 1, -1e8, 1], np.float32)
    c = np.zeros(4, np.float32)
    # fp64: 1e16 + 1 -> 1e16 (1 lost), + 1e16, + 1 -> 2e16 exactly as ordered
    assert ora.sqdist(r, c) == ((1e16 + 1.0) + 1e16) + 1.0


@pytest.mark.parametrize("family", ["normal", "wide", "cancel", "subnormal"])
def test_update_sum_is_the_correctly_rounded_exact_sum(ora, family):
    """The update's per-channel sum is the exact sum of the members rounded
    once to fp64 -- pinned against Python's correctly rounded math.fsum."""
    import math
    rng = np.random.default_rng({"normal": 1, "wide": 2, "cancel": 3, "subnormal": 4}[family])
    for _ in range(300):
        n = int(rng.integers(1, 300))
        if family == "normal":
            x = rng.standard_normal(n).astype(np.float32)
        elif family == "wide":
            x = (rng.standard_normal(n) * np.exp2(rng.integers(-140, 120, n))).astype(np.float32)
        elif family == "cancel":
            b = (rng.standard_normal(n) * np.float32(1e30)).astype(np.float32)
            x = rng.permutation(np.concatenate([b, -b, rng.standard_normal(3).astype(np.float32)]))
        else:
            x = (rng.integers(-5, 6, n) * np.float32(2.0 ** -149)).astype(np.float32)
        assert ora.exact_sum(x) == math.fsum(float(v) for v in x)


def test_update_mean_survives_cancellation(ora):
    """Members 2^100, 1, -2^100 in one channel: an fp64 running sum would lose
    the 1; the mean is 1/3, rounded to bf16 (and to fp32)."""
    import torch
    X = np.zeros((3, 4), np.float32)
    X[:, 0] = [2.0 ** 100, 1.0, -(2.0 ** 100)]
    X[:, 1] = [1.0, 2.0, 4.0]
    pi = np.zeros(3, np.uint8)
    C0 = np.full((1, 4), 7.0, np.float32)
    third_bf16 = float(torch.tensor(1.0 / 3.0, dtype=torch.float64).to(torch.bfloat16).float())
    Cb = ora.update(X, pi, C0, dtype=BF16)
    assert Cb[0, 0] == np.float32(third_bf16)
    assert Cb[0, 1] == np.float32(float(torch.tensor(7.0 / 3.0, dtype=torch.float64).to(torch.bfloat16).float()))
    Cf = ora.update(X, pi, C0, dtype=FP32)
    assert Cf[0, 0] == np.float32(1.0 / 3.0)
