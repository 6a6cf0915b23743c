"""Pins of the oracle's attention over the reconstructed cache (the consumer
that the m.163.com article on Quant VideoGen, section 五, describes: pre-RoPE
key cache, rotary embedding after dequantisation, fused into attention)."""
import math

import numpy as np
import pytest


def test_rope_hand_example(ora):
    """d = 2: one pair, angle = position (base^0 = 1): (1, 0) at position 1
    becomes (cos 1, sin 1); (0, 2) at position 3 becomes (-2 sin 3, 2 cos 3);
    position 0 is the identity."""
    x = np.array([[1.0, 0.0], [0.0, 2.0], [0.7, -0.3]], np.float32)
    out = ora.rope(x, [1, 3, 0])
    np.testing.assert_allclose(out[0], [math.cos(1), math.sin(1)], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out[1], [-2 * math.sin(3), 2 * math.cos(3)], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(out[2], x[2].astype(np.float64))


def test_rope_frequencies_and_relative_position(ora):
    """Pair i turns by base^(-2i/d) per position (d = 8: 1, 0.1, 0.01, 0.001
    at base 10^4), each pair keeps its length, and the dot product of two
    rotated vectors depends only on the difference of their positions."""
    rng = np.random.default_rng(2)
    d = 8
    e = np.zeros((4, d), np.float32)
    for i in range(4):
        e[i, 2 * i] = 1.0
    out = ora.rope(e, [5] * 4)
    for i in range(4):
        a = 5 * 10.0 ** (-i)
        np.testing.assert_allclose(out[i, 2 * i:2 * i + 2], [math.cos(a), math.sin(a)], atol=1e-14)
    q, k = rng.standard_normal((2, d)).astype(np.float32)
    for p1, p2 in [(7, 3), (1004, 1000), (123456, 123452)]:
        dot = ora.rope(q[None], [p1])[0] @ ora.rope(k[None], [p2])[0]
        ref = ora.rope(q[None], [p1 - p2])[0] @ k.astype(np.float64)
        assert dot == pytest.approx(ref, rel=1e-9, abs=1e-12)
    r = ora.rope(q[None], [98765])[0]
    q64 = q.astype(np.float64)
    np.testing.assert_allclose(np.hypot(r[0::2], r[1::2]), np.hypot(q64[0::2], q64[1::2]), rtol=1e-12)


def test_attention_hand_example(ora):
    """One query (1, 0) at position 0 over two keys (1, 0) at positions 0 and
    1 (the second turns by 1 radian): scores 1/sqrt(2) and cos(1)/sqrt(2),
    weights their softmax, output the weighted mean of the two values."""
    Q = np.array([[1.0, 0.0]], np.float32)
    K = np.array([[1.0, 0.0], [1.0, 0.0]], np.float32)
    V = np.array([[2.0, -1.0], [-4.0, 3.0]], np.float32)
    s0, s1 = 1 / math.sqrt(2), math.cos(1) / math.sqrt(2)
    p0 = 1 / (1 + math.exp(s1 - s0))
    out = ora.attention(Q, [0], K, V)
    V64 = V.astype(np.float64)
    np.testing.assert_allclose(out[0], p0 * V64[0] + (1 - p0) * V64[1], rtol=1e-14)


def test_attention_invariants(ora):
    """Every output row is a convex combination of the value rows; equal keys
    give the plain mean of the values; a key far ahead of the rest takes all
    the weight."""
    rng = np.random.default_rng(4)
    d, nk = 16, 40
    Q = rng.standard_normal((5, d)).astype(np.float32)
    K = rng.standard_normal((nk, d)).astype(np.float32)
    V = rng.standard_normal((nk, d)).astype(np.float32)
    out = ora.attention(Q, np.arange(100, 105), K, V)
    assert np.all(out <= V.max(0) + 1e-12) and np.all(out >= V.min(0) - 1e-12)
    Kz = np.zeros((nk, d), np.float32)                        # zero keys: all scores 0
    np.testing.assert_allclose(ora.attention(Q, np.arange(5), Kz, V), np.tile(V.astype(np.float64).mean(0), (5, 1)),
                               rtol=1e-12, atol=1e-14)
    Kb = np.zeros((nk, d), np.float32)
    Kb[7] = 400.0 * Q[0] / np.linalg.norm(Q[0])               # aligned with query 0 at position 7
    out = ora.attention(Q[:1], [7], Kb, V)
    np.testing.assert_allclose(out[0], V[7], atol=1e-9)
