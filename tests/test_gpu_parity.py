"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same
seeded inputs.  Sizes span several tiles with ragged tails; the full-size
case runs in the launch configuration the benchmark times and checks sampled
blocks against the oracle one by one."""
import numpy as np
import pytest
import torch

from gpu_util import (BF16, FP32, compare_quantize, compare_reconstruction, np_bits, packed_np,
                      to_dev, values)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


def _rand_packed(rng, K, T, G, N, H, dtype, scale_mode=0):
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    small = finite[(finite & 0x7F) <= 0x50]                     # |v| <= 4
    p = dict(
        codes=rng.integers(0, 256, (H, N, 32), dtype=np.uint8),
        scale=rng.choice(small if scale_mode == 0 else finite, (H, N, 128 // G)),
        zero=rng.choice(finite, (H, N, 128 // G)) if scale_mode == 0 else np.zeros((0,), np.uint8),
        assign=rng.integers(0, K, (T, H, N), dtype=np.uint8),
    )
    tab = (rng.standard_normal((T, H, K, 128)) * 10.0 ** rng.uniform(-2, 3, (T, H, K, 1))).astype(np.float32)
    if dtype == BF16:
        tab = torch.from_numpy(tab).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    p["centroids"] = tab
    return p


@pytest.mark.parametrize("dtype,T,G,K,N,H,mode", [
    (BF16, 2, 64, 256, 4680, 3, 0),
    (BF16, 2, 64, 256, 38000, 8, 0),      # the full-size batch, in the benchmark's launch configuration
    (BF16, 0, 16, 1, 777, 2, 0),
    (BF16, 1, 8, 7, 130, 3, 0),
    (BF16, 3, 32, 256, 1000, 2, 0),       # third table read from L2
    (BF16, 4, 128, 64, 513, 2, 0),
    (FP32, 1, 16, 16, 512, 1, 0),
    (FP32, 2, 64, 256, 300, 2, 0),
    (BF16, 1, 64, 256, 4680, 2, 1),       # one scale per group: the QVG point
    (BF16, 4, 16, 256, 1000, 2, 1),       # the QVG-Pro point
    (BF16, 0, 16, 1, 777, 2, 1),
    (FP32, 2, 32, 100, 300, 2, 1),
])
def test_dequant_of_oracle_layout_is_bit_exact(q, ora, dtype, T, G, K, N, H, mode):
    rng = np.random.default_rng(K * 1000 + N)
    p = _rand_packed(rng, K, T, G, N, H, dtype, mode)
    Yr = ora.dequantize(p, K=K, T=T, G=G, N=N, H=H, d=128, dtype=dtype, scale_mode=mode)
    cfg = q.config(K=K, T=T, group_size=G, scale_mode=mode)
    dp = q.Packed(codes=to_dev(p["codes"]), scale=to_dev(p["scale"]), zero=to_dev(p["zero"]),
                  assign=to_dev(p["assign"]), centroids=to_dev(p["centroids"]),
                  cfg=cfg, N=N, H=H, d=128, dtype=dtype)
    Yg = np_bits(q.dequantize(dp))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Yg, Yr)


def _run(q, ora, X, K, T, G, iters, init=None, warm_iters=None, mode=0):
    """GPU and oracle quantisation + reconstruction of the same input."""
    X_np = np_bits(X)
    dtype = BF16 if X.dtype == torch.bfloat16 else FP32
    cfg = q.config(K=K, T=T, group_size=G, iters=iters, warm_iters=warm_iters or iters, scale_mode=mode)
    init_t = to_dev(init) if init is not None else None
    pg = q.quantize(X.cuda().contiguous(), cfg, init=init_t)
    Yg = np_bits(q.dequantize(pg))
    torch.cuda.synchronize()
    gpu = packed_np(pg)
    ref = ora.quantize(X_np, K=K, T=T, G=G, iters=(warm_iters or iters) if init is not None else iters,
                       init=init, scale_mode=mode)
    H, N, d = X_np.shape
    Yr = ora.dequantize(ref, K=K, T=T, G=G, N=N, H=H, d=d, dtype=dtype, scale_mode=mode)
    compare_quantize(ora, X_np, gpu, ref, K, T, G, iters, dtype)   # the packed streams first
    np.testing.assert_array_equal(Yg, Yr)     # then the GPU's reconstruction of its own stream
    return X_np, gpu, ref, Yg, Yr, dtype


def test_quantize_tiny_fp32_case(q, ora):
    """One head, 2 frames of 16x16 tokens, fp32, K=16, T=1, G=16, 10 iterations
    from the first 16 tokens."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.tiny_block(seed=0)[None]
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, X, K=16, T=1, G=16, iters=10)
    rep = compare_quantize(ora, X_np, gpu, ref, 16, 1, 16, 10, dt)
    compare_reconstruction(ora, X_np, Yg, Yr, gpu, ref, 16)
    assert rep["bit_exact"], rep


@pytest.mark.parametrize("K,T,G,iters,frames,gh,gw,H", [
    (256, 2, 64, 8, 3, 30, 52, 2),     # one Self-Forcing-scale chunk, K and V heads
    (64, 3, 32, 5, 2, 20, 25, 2),      # ragged N = 1000
    (1, 1, 16, 2, 1, 7, 9, 1),         # K = 1
    (200, 1, 128, 4, 1, 17, 17, 1),    # N = 289, K not a multiple of 32
    (256, 4, 16, 3, 1, 25, 41, 2),     # T = 4 (third and fourth tables read from L2), G = 16, N = 1025
    (64, 2, 8, 4, 1, 21, 37, 2),       # G = 8, N = 777
    (256, 2, 16, 3, 1, 30, 52, 2),     # G = 16 at K = 256
])
def test_quantize_bf16_parity(q, ora, K, T, G, iters, frames, gh, gw, H):
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(H, synth.KVShape(frames, gh, gw), seed=17 + K, kinds=[h % 2 for h in range(H)])
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, X, K=K, T=T, G=G, iters=iters)
    rep = compare_quantize(ora, X_np, gpu, ref, K, T, G, iters, dt)
    compare_reconstruction(ora, X_np, Yg, Yr, gpu, ref, G)
    print(rep)


def test_rtn_covers_e4m3_rounding(q, ora):
    """T = 0: the group minimum and maximum sweep the E4M3 range (subnormals,
    exact codes, midpoints, saturation) -- scale and zero bytes bit-exact."""
    rng = np.random.default_rng(5)
    codes = np.array([c for c in range(256) if (c & 0x7F) < 0x7F], np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    mids = (vals[:-1] + vals[1:]) / 2
    lows = np.concatenate([vals, mids, rng.uniform(-500, 500, 2000), rng.uniform(-0.02, 0.02, 500)])
    N = len(lows) // 2 + 1
    X = rng.uniform(0, 1, (1, N, 128)).astype(np.float32)
    for g in range(2):
        lo = lows[g * N:(g + 1) * N]
        X[0, :len(lo), g * 64] = lo
        X[0, :len(lo), g * 64 + 1] = lo + np.abs(rng.standard_normal(len(lo))) * 3 * np.abs(lo + 1e-3)
    Xt = torch.from_numpy(X).to(torch.bfloat16)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xt, K=1, T=0, G=64, iters=1)
    for k in ("codes", "scale", "zero"):
        np.testing.assert_array_equal(gpu[k], ref[k])
    Xf = torch.from_numpy(X)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xf, K=1, T=0, G=16, iters=1)
    for k in ("codes", "scale", "zero"):
        np.testing.assert_array_equal(gpu[k], ref[k])


def test_warm_start_parity(q, ora):
    """Given initial tables, every stage starts from them and runs warm_iters."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(2, synth.KVShape(1, 30, 52), seed=3, kinds=[0, 1])
    X_np = np_bits(X)
    ref0 = ora.quantize(X_np, K=128, T=2, G=64, iters=6)
    init = ref0["centroids"]
    X2 = synth.block_batch(2, synth.KVShape(1, 30, 52), seed=4, kinds=[0, 1])
    X_np2, gpu, ref, Yg, Yr, dt = _run(q, ora, X2, K=128, T=2, G=64, iters=9, init=init, warm_iters=3)
    compare_quantize(ora, X_np2, gpu, ref, 128, 2, 64, 3, dt, init=init)
    compare_reconstruction(ora, X_np2, Yg, Yr, gpu, ref, 64)


@pytest.mark.parametrize("K,H,frames", [
    (64, 2, [3, 3, 3, 1]),
    # 22 chunks at K = 256, four blocks: one of 3 frames, twenty of 1, one of 2
    (256, 4, [3] + [1] * 20 + [2]),
])
def test_streaming_cache_parity(q, ora, K, H, frames):
    """qvg_append_chunk: chunk 0 cold, later chunks warm-started from the
    previous chunk's centroids; every chunk's packed form equals the oracle's,
    and the fused dequantisation of the whole cache equals the oracle's
    chunk-by-chunk reconstruction."""
    from bit_kv_cache_qvg_b200 import synth
    T, G, I, Iw = 2, 64, 6, 3
    stream = synth.PrototypeStream(H, 30, 52, kinds=[h % 2 for h in range(H)], seed=21 + K)
    cfg = q.config(K=K, T=T, group_size=G, iters=I, warm_iters=Iw)
    cache = q.Cache(cfg, H=H, max_tokens=sum(frames) * 1560, max_chunks=len(frames) + 2,
                    max_chunk_tokens=max(frames) * 1560)
    prev = None
    Ys = []
    for c, f in enumerate(frames):
        X = stream.next(f)
        cache.append(X.cuda())
        X_np = np_bits(X)
        ref = ora.quantize(X_np, K=K, T=T, G=G, iters=I if prev is None else Iw, init=prev)
        gpu = packed_np(cache.chunk(c))
        torch.cuda.synchronize()
        compare_quantize(ora, X_np, gpu, ref, K, T, G, I if prev is None else Iw, BF16, init=prev)
        assert cache.chunk_info(c) == dict(level=0, T=T, G=G, stat=0)
        prev = ref["centroids"]                        # the oracle chains its own chunks
        Ys.append(ora.dequantize(ref, K=K, T=T, G=G, N=X_np.shape[1], H=H, d=128))
    assert cache.tokens == sum(frames) * 1560 and cache.chunks == len(frames)
    assert cache.status() == 0
    Y = np_bits(cache.dequantize())
    np.testing.assert_array_equal(Y, np.concatenate(Ys, axis=1))
    with pytest.raises(q.QvgError) as e:               # larger than the cache's largest chunk
        cache.append(stream.next(max(frames) + 1).cuda())
    assert e.value.status == 7 and cache.chunks == len(frames)
    cache.close()


def test_full_size_every_block(q, ora):
    """LongCat-scale blocks (38,000 tokens = 25 frames of 38x40, K=256, T=2,
    G=64, 10 iterations) quantised in the benchmark's batch configuration;
    every block (K and V kinds alternating) checked against the oracle in
    full: packed streams bit-exact, reconstructions identical."""
    from bit_kv_cache_qvg_b200 import synth
    H = 8
    X = synth.block_batch(H, synth.KVShape(25, 38, 40), seed=1234, kinds=[h % 2 for h in range(H)],
                          device="cuda")
    cfg = q.config(K=256, T=2, group_size=64, iters=10)
    pg = q.quantize(X, cfg)
    Yg = np_bits(q.dequantize(pg))
    torch.cuda.synchronize()
    gpu = packed_np(pg)
    X_np = np_bits(X)
    for h in range(H):
        sub = {k: (v[:, h:h + 1] if k in ("assign", "centroids") else v[h:h + 1]) for k, v in gpu.items()}
        ref = ora.quantize(X_np[h:h + 1], K=256, T=2, G=64, iters=10)
        compare_quantize(ora, X_np[h:h + 1], sub, ref, 256, 2, 64, 10, BF16)
        Yr = ora.dequantize(ref, K=256, T=2, G=64, N=38000, H=1, d=128)
        np.testing.assert_array_equal(Yg[h:h + 1], Yr)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


@pytest.mark.parametrize("K", [256, 200])
def test_k_equals_n_gives_exact_reconstruction(q, ora, K):
    """K = N: the first-K start makes every token its own centroid, the
    residual is exactly zero, every later stage and the quantiser see zeros
    (all ties, so every token takes centroid 0), and the reconstruction is X
    itself, bit for bit."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(2, synth.KVShape(1, 1, K), seed=K, kinds=[0, 1])
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, X, K=K, T=2, G=64, iters=3)
    compare_quantize(ora, X_np, gpu, ref, K, 2, 64, 3, dt)
    np.testing.assert_array_equal(gpu["assign"][0], np.tile(np.arange(K, dtype=np.uint8), (2, 1)))
    assert not gpu["assign"][1].any() and not gpu["codes"].any()
    np.testing.assert_array_equal(Yg, X_np)


@pytest.mark.parametrize("T,iters", [(1, 1), (2, 4)])
def test_duplicate_tokens_and_centroids_take_the_lowest_index(q, ora, T, iters):
    """Exact duplicates: the first 256 tokens hold 128 vectors twice each, so
    the cold start has 128 pairs of equal centroids, and later tokens repeat
    earlier ones exactly or with a little noise.  In the first assignment
    every distance tie goes to the lower index and the higher twin is left
    empty (forced empty clusters at K = 256; an empty centroid keeps its
    value).  Later iterations move the lower twin to its members' mean, after
    which tokens equal to the upper twin's kept value go to it: the oracle
    decides the same."""
    rng = np.random.default_rng(11)
    base = rng.standard_normal((128, 128)).astype(np.float32) * np.exp(rng.standard_normal(128)).astype(np.float32)
    head = np.repeat(base, 2, axis=0)                         # rows 2m and 2m+1 equal
    pick = rng.integers(0, 128, 744)
    tail = base[pick] + (rng.random((744, 1)) < 0.5) * 0.05 * rng.standard_normal((744, 128)).astype(np.float32)
    X = np.stack([_bf16_bits(np.concatenate([head, tail])), _bf16_bits(np.concatenate([head, tail[::-1]]))])
    Xt = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xt, K=256, T=T, G=32, iters=iters)
    compare_quantize(ora, X_np, gpu, ref, 256, T, 32, iters, dt)
    if iters == 1:
        for h in range(2):
            pi = gpu["assign"][0, h]
            assert len(np.unique(pi)) <= 128                  # every upper twin is empty
            assert not (pi % 2).any()                         # ties went to the lower index
            np.testing.assert_array_equal(pi[:256], np.repeat(np.arange(0, 256, 2), 2))
        # an empty centroid keeps its value: the upper twins are still the tokens
        np.testing.assert_array_equal(gpu["centroids"][0, 0, 1::2], X_np[0, 1:256:2])


def _near_tie_table_and_tokens(seed):
    """Centroids in 128 pairs that differ only in one channel j_m (by 8, at
    mid_m -+ 4); every centroid shares a common vector B of +-1000 in four
    outlier channels.  Tokens of pair m: the pair's other channels, B plus an
    offset O of +-1000 in the outlier channels (the same for every centroid,
    so it cancels between centroids but makes |r| about 4,000 and the exact
    distances about 4e6), and channel j_m at mid_m + t.  The exact gap between
    the twins is 8 |t| in h and 16 |t| in squared distance: t = 0 is an exact
    tie, t = 0.25 about 1e-6 relative, and |t| up to 500 crosses the
    screening margin, so the screen decides some tokens and the exact pass
    the rest."""
    rng = np.random.default_rng(seed)
    d, K = 128, 256
    big = np.array([5, 37, 70, 111])
    B = np.where(rng.random(4) < 0.5, -1000.0, 1000.0)
    C = np.zeros((K, d), np.float64)
    tokens = []
    ts = np.array([0, 0.25, -0.25, 0.5, -0.5, 1, -1, 2, -3, 8, -16, 30, 60, -120, 250, -500])
    for m in range(128):
        v = np.round(rng.standard_normal(d) * 4.0)         # integers: exact in bf16
        v[big] = B
        j = int(rng.choice(np.setdiff1d(np.arange(d), big)))
        mid = float(rng.integers(-40, 41))
        C[2 * m], C[2 * m + 1] = v, v
        C[2 * m, j], C[2 * m + 1, j] = mid - 4.0, mid + 4.0
        O = np.where(rng.random(4) < 0.5, -1000.0, 1000.0)
        for t in ts:
            r = v.copy()
            r[big] = B + O
            r[j] = mid + t
            tokens.append(r)
    return C.astype(np.float32), np.array(tokens, np.float32)


@pytest.mark.parametrize("T,iters", [(1, 1), (2, 3)])
def test_adversarial_near_ties_at_outlier_scale(q, ora, T, iters):
    """Near-equidistant tokens at x1000 outlier magnitudes decide exactly as
    the oracle: exact ties to the lower index, gaps of about 1e-6 relative by
    the exact pass, and gaps beyond the screening margin by the tensor-core
    screen.  Warm-started from the constructed table, so the first assignment
    is against it."""
    C, R = _near_tie_table_and_tokens(3)
    Xb = _bf16_bits(R)[None]
    Cb = _bf16_bits(C)
    assert np.array_equal(Xb[0].view(np.uint16), _bf16_bits(R)) and np.array_equal(
        (Cb.astype(np.uint32) << 16).view(np.float32), C)   # every value exact in bf16
    init = np.repeat(Cb[None, None], T, axis=0)              # [T][1][K][d]
    if T > 1:
        init[1:] = 0
    Xt = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xt, K=256, T=T, G=64, iters=iters, init=init, warm_iters=iters)
    compare_quantize(ora, X_np, gpu, ref, 256, T, 64, iters, dt, init=init)
    pi = gpu["assign"][0, 0].reshape(128, 16)
    if iters == 1:
        # the first assignment is the table's.  For |t| <= 3 the token's own
        # pair is by far the nearest: t = 0 ties to the lower twin, t > 0 is
        # nearer the upper twin (mid + 4), t < 0 the lower one
        pairs = np.arange(128)[:, None]
        tsign = np.array([0, 1, -1, 1, -1, 1, -1, 1, -1])
        expect = np.where(tsign > 0, 2 * pairs + 1, 2 * pairs)
        np.testing.assert_array_equal(pi[:, :9], expect)


def test_tensor_core_and_exact_assignment_agree(q, monkeypatch):
    """The tcgen05 screening path (with its exact pass for listed near-ties)
    and the all-exact CUDA-core path produce identical packed streams."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(4, synth.KVShape(4, 30, 52), seed=77, kinds=[0, 1, 0, 1], device="cuda")
    cfg = q.config(K=256, T=2, group_size=64, iters=6)
    ws = q.alloc_workspace(cfg, X.shape[1], X.shape[0])
    a = packed_np(q.quantize(X, cfg, workspace=ws))
    flagged = q.workspace_flagged(ws)
    monkeypatch.setenv("QVG_ASSIGN_PATH", "exact")
    b = packed_np(q.quantize(X, cfg))
    torch.cuda.synchronize()
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    total = X.shape[0] * X.shape[1] * 2 * 6
    print(f"near-tie tokens decided exactly: {flagged} of {total} ({flagged / total:.4%})")
    assert 0 <= flagged < 0.2 * total
    assert q.workspace_status(ws) == 0


@pytest.mark.gpu
def test_waves_on_two_streams_match_one_wave(q, monkeypatch):
    """Blocks in several waves -- alternating between the caller's stream and
    the library's second stream, or all on one stream -- give the same packed
    stream as one wave holding every block (waves are independent)."""
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(6, synth.KVShape(3, 30, 52), seed=91, kinds=[0, 1] * 3, device="cuda")
    H, N = X.shape[0], X.shape[1]
    cfg = q.config(K=256, T=2, group_size=64, iters=4)
    one_wave = packed_np(q.quantize(X, cfg, workspace=q.alloc_workspace(cfg, N, H)))
    # room for two one-block waves: six waves, alternating lanes
    ws = torch.zeros(2 * q.workspace_bytes(cfg, N, 1), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        two_lanes = packed_np(q.quantize(X, cfg, workspace=ws, stream=stream))
    assert q.workspace_status(ws, stream=stream) == 0
    monkeypatch.setenv("QVG_WAVE_LANES", "1")
    one_lane = packed_np(q.quantize(X, cfg, workspace=ws))
    torch.cuda.synchronize()
    for k in one_wave:
        np.testing.assert_array_equal(two_lanes[k], one_wave[k])
        np.testing.assert_array_equal(one_lane[k], one_wave[k])


def _wide_channel_block(rng, N, big, tiny, dtype):
    """16 well-separated prototypes; channel 0 holds values near `big` for
    prototypes 0-7 and near `tiny` (nonzero) for 8-15, so a cluster of small
    values shares its channel with magnitudes far above it."""
    proto = rng.standard_normal((16, 128)) * 20.0
    k = rng.integers(0, 16, N)
    X = proto[k] + 0.3 * rng.standard_normal((N, 128))
    scale = np.where(k < 8, big, tiny)
    X[:, 0] = scale * (1.0 + 0.25 * rng.standard_normal(N))
    X = X.astype(np.float32)
    if dtype == BF16:
        return _bf16_bits(X)
    return X


@pytest.mark.parametrize("dtype,big,tiny,T", [
    (BF16, 1.0e4, 1.0e-11, 1),
    (BF16, 1.0e4, 1.0e-11, 2),
    (FP32, 1.0e3, 1.0e-7, 2),
])
def test_centroid_sums_beyond_the_fixed_point_window(q, ora, dtype, big, tiny, T):
    """A channel with values more than the fixed-point window (39 binades for
    bf16 at this N, 23 for fp32) below its largest magnitude: its centroid
    sums are formed exactly by the wide path, and the result is bit-exact."""
    rng = np.random.default_rng(41 + T)
    N = 1024
    X = np.stack([_wide_channel_block(rng, N, big, tiny, dtype) for _ in range(2)])
    vals = values(X[0, :, 0])
    log2n = int(np.floor(np.log2(N))) + 1                    # smallest k with 2^k > N
    L = int(np.floor(np.log2(np.abs(vals).max()))) + log2n - 62
    e_min = int(np.floor(np.log2(np.abs(vals[vals != 0]).min())))
    assert e_min - (7 if dtype == BF16 else 23) < L           # the data is outside the window
    Xt = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16) if dtype == BF16 else torch.from_numpy(X)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xt, K=16, T=T, G=32, iters=4)
    compare_quantize(ora, X_np, gpu, ref, 16, T, 32, 4, dt)
    tiny_means = values(gpu["centroids"][0, :, :, 0])
    assert (np.abs(tiny_means) < 1e-6).any()                  # some centroid is a mean of tiny values


@pytest.mark.parametrize("name,N,H,dtype", [
    ("qvg", 4680, 2, BF16),            # T = 1, G = 64, one scale per group
    ("qvg-pro", 1560, 2, BF16),        # T = 4, G = 16
    ("qvg", 700, 1, FP32),
])
def test_operating_points_with_one_scale_per_group(q, ora, name, N, H, dtype):
    """The named QVG and QVG-Pro settings (one E4M3 scale per group): packed
    streams bit-exact against the oracle, packed size equal to the closed
    form, and a reconstruction error below plain rounding at the same group
    size (the smoothing stages at work)."""
    from bit_kv_cache_qvg_b200 import synth
    P = q.PRESETS[name]
    X = synth.block_batch(H, synth.KVShape(1, 1, N), seed=N + H, kinds=[h % 2 for h in range(H)],
                          dtype=torch.bfloat16 if dtype == BF16 else torch.float32)
    X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, X, K=P["K"], T=P["T"], G=P["group_size"], iters=4,
                                      mode=P["scale_mode"])
    compare_quantize(ora, X_np, gpu, ref, P["K"], P["T"], P["group_size"], 4, dt)
    cfg = q.preset(name)
    assert sum(a.nbytes for a in gpu.values()) == q.packed_bytes(cfg, N, H, 128, dtype) == ora.packed_bytes(
        P["K"], P["T"], P["group_size"], N, H, 128, dtype=dtype, scale_mode=1)
    rtn = ora.quantize(X_np, K=1, T=0, G=P["group_size"], iters=0, scale_mode=1)
    Y0 = ora.dequantize(rtn, K=1, T=0, G=P["group_size"], N=N, H=H, d=128, dtype=dt, scale_mode=1)
    x = values(X_np)
    assert ((values(Yg) - x) ** 2).mean() < ((values(Y0) - x) ** 2).mean()


def test_symmetric_rtn_covers_e4m3_rounding(q, ora):
    """T = 0 with one scale per group: the group's largest magnitude sweeps
    the E4M3 range (subnormals, exact codes, midpoints, saturation) -- scale
    bytes and codes bit-exact, bf16 and fp32."""
    rng = np.random.default_rng(6)
    codes = np.array([c for c in range(128) if c < 0x7F], np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    mids = (vals[:-1] + vals[1:]) / 2
    amax = np.concatenate([vals, mids, rng.uniform(0, 600, 1000), rng.uniform(0, 0.02, 300)])
    N = len(amax)
    X = (rng.uniform(-1, 1, (1, N, 128)) * amax[None, :, None]).astype(np.float32)
    sign = np.where(rng.random(N) < 0.5, -1.0, 1.0)
    for g in range(2):
        X[0, :, g * 64 + 5] = sign * amax
    for Xt, G in ((torch.from_numpy(X).to(torch.bfloat16), 64), (torch.from_numpy(X), 32)):
        X_np, gpu, ref, Yg, Yr, dt = _run(q, ora, Xt, K=1, T=0, G=G, iters=1, mode=1)
        for k in ("codes", "scale"):
            np.testing.assert_array_equal(gpu[k], ref[k])
        np.testing.assert_array_equal(Yg, Yr)


def test_symmetric_streaming_cache(q, ora):
    """The streaming cache at the QVG point: chunk 0 cold, later chunks warm,
    every chunk bit-exact and the whole-cache dequantisation equal to the
    oracle's chunk-by-chunk reconstruction."""
    from bit_kv_cache_qvg_b200 import synth
    H, frames = 2, [3, 1, 1, 2, 1]
    stream = synth.PrototypeStream(H, 30, 52, kinds=[0, 1], seed=77)
    cfg = q.preset("qvg", iters=5, warm_iters=2)
    cache = q.Cache(cfg, H=H, max_tokens=sum(frames) * 1560, max_chunks=len(frames),
                    max_chunk_tokens=3 * 1560)
    prev, Ys = None, []
    for c, f in enumerate(frames):
        X = stream.next(f)
        cache.append(X.cuda())
        X_np = np_bits(X)
        it = 5 if prev is None else 2
        ref = ora.quantize(X_np, K=256, T=1, G=64, iters=it, init=prev, scale_mode=1)
        gpu = packed_np(cache.chunk(c))
        torch.cuda.synchronize()
        compare_quantize(ora, X_np, gpu, ref, 256, 1, 64, it, BF16, init=prev)
        prev = ref["centroids"]
        Ys.append(ora.dequantize(ref, K=256, T=1, G=64, N=X_np.shape[1], H=H, d=128, scale_mode=1))
    np.testing.assert_array_equal(np_bits(cache.dequantize()), np.concatenate(Ys, axis=1))
    cache.close()
