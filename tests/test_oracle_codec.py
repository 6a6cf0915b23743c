"""Pins of the oracle's group quantisation, packing, progressive residual
stages and reverse-order reconstruction (m.163.com article on Quant VideoGen,
sections 四, 五, 六; gist.science/de, Technische Zusammenfassung 2B/2C):
hand-worked examples, exact special cases and error bounds."""
import numpy as np
import pytest

BF16, FP32 = 0, 1


def _bf16_bits(x):
    import torch
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_pack_layout_worked_example(ora):
    """Group [0, 1, 2, 3] (G = 4): min 0 -> zero point 0, (3 - 0)/3 = 1 -> scale 1,
    codes 0,1,2,3 -> one byte 0b11_10_01_00 = 0xE4 (channel j at bits 2j)."""
    codes, scale, zero = ora.group_quant(np.array([[0, 1, 2, 3]], np.float32), 4)
    assert codes[0, 0] == 0xE4
    assert scale[0, 0] == 0x38 and zero[0, 0] == 0x00        # E4M3 1.0 and 0.0


def test_group_quant_worked_example_with_rounding(ora):
    """[0.3, 0.1, 0.9, 0.0]: lo = 0 -> m = 0; (0.9 - 0)/3 = 0.3 -> E4M3 0.3125
    (exponent -2, mantissa 0.3/0.25 = 1.2 -> 1 + 2/8; code 0b0_0101_010 = 0x2A);
    q = rint(0.96, 0.32, 2.88, 0) = 1, 0, 3, 0 -> byte 1 | 3<<4 = 0x31."""
    codes, scale, zero = ora.group_quant(np.array([[0.3, 0.1, 0.9, 0.0]], np.float32), 4)
    assert scale[0, 0] == 0x2A and zero[0, 0] == 0x00
    assert codes[0, 0] == 0x31


def test_group_quant_grid_values_are_exact(ora):
    """Values m + q*s with E4M3-exact m, s and every q present: lo = m, hi = m+3s,
    (hi - m)/3 = s, so codes and reconstruction are exact."""
    m, s = -1.5, 0.25
    row = np.array([[m + 2 * s, m, m + 3 * s, m + s, m + s, m + 3 * s, m, m + 2 * s]], np.float32)
    codes, scale, zero = ora.group_quant(row, 8)
    assert ora.e4m3_decode(scale)[0, 0] == s and ora.e4m3_decode(zero)[0, 0] == m
    q = [(codes[0, j // 4] >> (2 * (j % 4))) & 3 for j in range(8)]
    assert q == [2, 0, 3, 1, 1, 3, 0, 2]


def test_signed_zero_extremes_are_canonical(ora):
    """A group whose minimum or maximum is -0 stores the same bytes as +0."""
    a = ora.group_quant(np.array([[-0.0, 0.0, 0.0, -0.0]], np.float32), 4)
    b = ora.group_quant(np.array([[0.0, 0.0, 0.0, 0.0]], np.float32), 4)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    assert a[1][0, 0] == 0 and a[2][0, 0] == 0


def test_constant_group_has_zero_scale(ora):
    codes, scale, zero = ora.group_quant(np.full((1, 8), 1.5, np.float32), 8)
    assert scale[0, 0] == 0 and ora.e4m3_decode(zero)[0, 0] == 1.5 and np.all(codes == 0)


def test_saturated_group(ora):
    """lo = -1000 saturates to -448; (1000 + 448)/3 = 482.7 saturates to 448;
    q = rint((r + 448)/448) clamped: -1.23 -> 0, 1 -> 1, 2.12 -> 2, 3.23 -> 3."""
    codes, scale, zero = ora.group_quant(np.array([[-1000, 0, 500, 1000]], np.float32), 4)
    assert zero[0, 0] == 0xFE and scale[0, 0] == 0x7E
    assert codes[0, 0] == (0 | 1 << 2 | 2 << 4 | 3 << 6)


def _unpack(codes, d):
    j = np.arange(d)
    return (codes[..., j // 4] >> (2 * (j % 4))) & 3


def test_quant_error_within_half_step(ora):
    rng = np.random.default_rng(0)
    N, d, G = 500, 128, 32
    R = (rng.standard_normal((N, d)) * 10.0 ** rng.uniform(-2, 1.5, (N, 1))).astype(np.float32)
    R = R.astype(np.float32)
    codes, scale, zero = ora.group_quant(R, G)
    q = _unpack(codes, d).astype(np.float64)
    s = np.repeat(ora.e4m3_decode(scale).astype(np.float64), G, axis=1)
    m = np.repeat(ora.e4m3_decode(zero).astype(np.float64), G, axis=1)
    rec = s * q + m
    r = R.astype(np.float64)
    unclamped = (r >= m - s / 2) & (r <= m + 3.5 * s)
    assert unclamped.mean() > 0.95
    err = np.abs(r - rec)
    assert np.all(err[unclamped] <= s[unclamped] / 2 * (1 + 2.0 ** -20) + 1e-30)
    # clamped values only at the ends of the code range
    assert np.all((q == 0) | (q == 3) | unclamped)


def test_dequant_worked_example(ora):
    """T=2, K=2, d=4, G=4, N=2; tables and codes chosen by hand.
    token 0: q=[0,1,2,3], s=0.25, m=-0.5 -> [-.5,-.25,0,.25];
             + C2[1]=[.25,0,-.25,0] -> [-.25,-.25,-.25,.25];
             + C1[0]=[1,2,3,4] -> [.75, 1.75, 2.75, 4.25]
    token 1: q=[3,3,0,1], s=1, m=2 -> [5,5,2,3]; + C2[0]=[.5]*4 -> [5.5,5.5,2.5,3.5];
             + C1[1]=[-1,-2,-3,-4] -> [4.5, 3.5, -.5, -.5]"""
    C1 = np.array([[1, 2, 3, 4], [-1, -2, -3, -4]], np.float32)
    C2 = np.array([[0.5] * 4, [0.25, 0, -0.25, 0]], np.float32)
    packed = dict(
        codes=np.array([[[0xE4], [0x4F]]], np.uint8),
        scale=np.array([[[0x28], [0x38]]], np.uint8),       # 0.25, 1.0
        zero=np.array([[[0xB0], [0x40]]], np.uint8),        # -0.5, 2.0
        assign=np.array([[[0, 1]], [[1, 0]]], np.uint8),    # [T][H][N]
        centroids=_bf16_bits(np.stack([C1, C2])[:, None]),  # [T][H][K][d]
    )
    Y = ora.dequantize(packed, K=2, T=2, G=4, N=2, H=1, d=4, dtype=BF16)
    got = ora.bf16_to_f32(Y)[0]
    np.testing.assert_array_equal(got, [[0.75, 1.75, 2.75, 4.25], [4.5, 3.5, -0.5, -0.5]])
    packed32 = dict(packed, centroids=np.stack([C1, C2])[:, None].astype(np.float32))
    Y32 = ora.dequantize(packed32, K=2, T=2, G=4, N=2, H=1, d=4, dtype=FP32)
    np.testing.assert_array_equal(Y32[0], got)


def test_dequant_adds_stages_in_reverse_order(ora):
    """fp32 addition is not associative: with y0 = 1, C(2) = 2^24, C(1) = -2^24
    the order ((y0 + C2) + C1) gives 0 while (y0 + C1) + C2 would give 1."""
    packed = dict(
        codes=np.zeros((1, 1, 1), np.uint8), scale=np.zeros((1, 1, 1), np.uint8),
        zero=np.array([[[0x38]]], np.uint8),                 # m = 1
        assign=np.zeros((2, 1, 1), np.uint8),
        centroids=np.array([[[[-2.0 ** 24] * 4]], [[[2.0 ** 24] * 4]]], np.float32),
    )
    Y = ora.dequantize(packed, K=1, T=2, G=4, N=1, H=1, d=4, dtype=FP32)
    np.testing.assert_array_equal(Y[0, 0], [0, 0, 0, 0])


@pytest.mark.parametrize("dtype", [BF16, FP32])
def test_k_equals_n_roundtrip_is_exact(ora, dtype):
    rng = np.random.default_rng(3)
    N, d = 16, 32
    X = rng.standard_normal((1, N, d)).astype(np.float32)
    if dtype == BF16:
        X = _bf16_bits(X)
    p = ora.quantize(X, K=N, T=1, G=16, iters=3)
    assert np.all(p["scale"] == 0) and np.all(p["zero"] == 0) and np.all(p["codes"] == 0)
    np.testing.assert_array_equal(p["assign"][0, 0], np.arange(N))
    Y = ora.dequantize(p, K=N, T=1, G=16, N=N, H=1, d=d, dtype=dtype)
    np.testing.assert_array_equal(Y, X)


def test_progressive_stages_definition(ora):
    """quantize() equals the stage-by-stage composition: kmeans on R(0)=X from
    its first K rows, residual, kmeans on R(1), residual, group quant."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(1, synth.KVShape(2, 8, 16), seed=4, kinds=[0])
    Xb = synth.bf16_bits(X)
    K, G, I = 16, 32, 4
    p = ora.quantize(Xb, K=K, T=2, G=G, iters=I)
    R = ora.bf16_to_f32(Xb[0])
    for t in range(2):
        C, pi = ora.kmeans(R, R[:K], I, dtype=BF16)
        np.testing.assert_array_equal(p["assign"][t, 0], pi)
        np.testing.assert_array_equal(ora.bf16_to_f32(p["centroids"][t, 0]), C)
        R = ora.residual(R, C, pi, dtype=BF16)
    codes, scale, zero = ora.group_quant(R, G)
    np.testing.assert_array_equal(p["codes"][0], codes)
    np.testing.assert_array_equal(p["scale"][0], scale)
    np.testing.assert_array_equal(p["zero"][0], zero)


def test_smoothing_lowers_error_vs_rtn(ora):
    """T >= 1 (centroid subtraction before the 2-bit step) gives a lower MSE than
    T = 0 (plain per-group round-to-nearest) on outlier-heavy prototype data.
    The pages' 6.9x (K) / 2.6x (V) reductions (m.163.com article, section 三)
    are model data; here only the direction is pinned."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(2, synth.KVShape(2, 12, 16), seed=9, kinds=[0, 1])
    Xb = synth.bf16_bits(X)
    x = X.float().numpy()
    H, N, d = x.shape
    mse = {}
    for T in (0, 1, 2):
        p = ora.quantize(Xb, K=32, T=T, G=32, iters=6)
        Y = ora.bf16_to_f32(ora.dequantize(p, K=32, T=T, G=32, N=N, H=H, d=d))
        mse[T] = ((Y - x) ** 2).mean(axis=(1, 2))
    assert np.all(mse[1] < mse[0]) and np.all(mse[2] <= mse[1] * 1.05)


def test_invalid_arguments_rejected(ora):
    X = np.zeros((1, 8, 16), np.float32)
    for kw in (dict(K=0), dict(K=257), dict(G=6), dict(G=32), dict(K=9, T=1), dict(iters=0)):
        args = dict(K=4, T=1, G=8, iters=2)
        args.update(kw)
        with pytest.raises(ValueError):
            ora.quantize(X, **args)


def _e4m3_byte(x):
    import torch
    return int(torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def test_symmetric_group_worked_examples(ora):
    """One E4M3 scale per group: s = E4M3(max |r|), q = clamp(rint(r/s), -2, 1),
    stored u = q + 2 at bits 2*(j mod 4).  Hand-worked groups of four:
      [0.3, -0.9, 1.2, 0.05]: s = E4M3(1.2) = 1.25 (0x3A); r/s = 0.24, -0.72,
        0.96, 0.04 -> q = 0, -1, 1, 0 -> u = 2, 1, 3, 2 -> byte 0xB6;
      [-1, 0.5, -0.5, 1]: s = 1; r/s = -1, 0.5, -0.5, 1 -> ties to even give
        q = -1, 0, 0, 1 -> u = 1, 2, 2, 3 -> byte 0xE9;
      zeros: s = 0, every u = 2 -> byte 0xAA;
      [1000, -3, 0, 2]: s saturates at 448 (0x7E); 1000/448 -> 2 -> clamp 1."""
    R = np.array([[0.3, -0.9, 1.2, 0.05], [-1.0, 0.5, -0.5, 1.0], [0, 0, 0, 0], [1000, -3, 0, 2]], np.float32)
    codes, scale = ora.group_quant_sym(R, 4)
    assert scale[:, 0].tolist() == [0x3A, _e4m3_byte(1.0), 0x00, 0x7E]
    assert scale[0, 0] == _e4m3_byte(1.25)
    assert codes[:, 0].tolist() == [0xB6, 0xE9, 0xAA, 3 | (2 << 2) | (2 << 4) | (2 << 6)]


def test_symmetric_error_bound_and_round_trip(ora):
    """|r - s (u - 2)| <= s/2 for every value (|r| <= 1.0625 s after E4M3
    rounding of the group maximum, inside the [-1.5 s, 1.5 s] the levels
    cover), and the oracle's dequantisation of a T = 0 stream is s (u - 2)."""
    rng = np.random.default_rng(7)
    X = (rng.standard_normal((1, 300, 128)) * np.exp(rng.standard_normal((1, 300, 1)))).astype(np.float32)
    p = ora.quantize(X, K=1, T=0, G=32, iters=0, scale_mode=1)
    Y = ora.dequantize(p, K=1, T=0, G=32, N=300, H=1, d=128, dtype=1, scale_mode=1)
    s = np.repeat(ora.e4m3_decode(p["scale"][0]), 32, axis=-1).astype(np.float64)
    j = np.arange(128)
    u = (p["codes"][0][:, j // 4] >> (2 * (j % 4))) & 3
    np.testing.assert_array_equal(Y[0], (s * (u - 2)).astype(np.float32))
    assert np.all(np.abs(X[0] - Y[0]) <= s / 2 * (1 + 2 ** -22))
    assert (u != 0).all()                      # q = -2 needs r/s < -1.5: never reached


def test_symmetric_dequant_hand_tables(ora):
    """T = 1, K = 2, G = 4, d = 4: y = s (u - 2) + C[pi], one fp32 add."""
    packed = dict(codes=np.array([[[0xB6]], [[0xAA]]], np.uint8).reshape(1, 2, 1),
                  scale=np.array([[[0x3A], [0x38]]], np.uint8),
                  zero=np.zeros((0,), np.uint8),
                  assign=np.array([[[1, 0]]], np.uint8),
                  centroids=np.array([[[[1, 2, 3, 4], [10, 20, 30, 40]]]], np.float32))
    Y = ora.dequantize(packed, K=2, T=1, G=4, N=2, H=1, d=4, dtype=1, scale_mode=1)
    # token 0: u = 2, 1, 3, 2 with s = 1.25, plus centroid 1; token 1: zeros plus centroid 0
    np.testing.assert_array_equal(Y[0, 0], np.array([10, 20 - 1.25, 30 + 1.25, 40], np.float32))
    np.testing.assert_array_equal(Y[0, 1], np.array([1, 2, 3, 4], np.float32))
