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


def _rand_packed(rng, K, T, G, N, H, dtype):
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    small = finite[(finite & 0x7F) <= 0x50]                     # |v| <= 4
    p = dict(
        codes=rng.integers(0, 256, (H, N, 32), dtype=np.uint8),
        scale=rng.choice(small, (H, N, 128 // G)),
        zero=rng.choice(finite, (H, N, 128 // G)),
        assign=rng.integers(0, K, (T, H, N), dtype=np.uint8),
    )
    tab = (rng.standard_normal((T, H, K, 128)) * 10.0 ** rng.uniform(-2, 3, (T, H, K, 1))).astype(np.float32)
    if dtype == BF16:
        tab = torch.from_numpy(tab).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    p["centroids"] = tab
    return p


@pytest.mark.parametrize("dtype,T,G,K,N,H", [
    (BF16, 2, 64, 256, 4680, 3),
    (BF16, 0, 16, 1, 777, 2),
    (BF16, 1, 8, 7, 130, 3),
    (BF16, 3, 32, 256, 1000, 2),       # third table read from L2
    (BF16, 4, 128, 64, 513, 2),
    (FP32, 1, 16, 16, 512, 1),
    (FP32, 2, 64, 256, 300, 2),
])
def test_dequant_of_oracle_layout_is_bit_exact(q, ora, dtype, T, G, K, N, H):
    rng = np.random.default_rng(K * 1000 + N)
    p = _rand_packed(rng, K, T, G, N, H, dtype)
    Yr = ora.dequantize(p, K=K, T=T, G=G, N=N, H=H, d=128, dtype=dtype)
    cfg = q.config(K=K, T=T, group_size=G)
    dp = q.Packed(codes=to_dev(p["codes"]), scale=to_dev(p["scale"]), zero=to_dev(p["zero"]),
                  assign=to_dev(p["assign"]), centroids=to_dev(p["centroids"]),
                  cfg=cfg, N=N, H=H, d=128, dtype=dtype)
    Yg = np_bits(q.dequantize(dp))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Yg, Yr)


def _run(q, ora, X, K, T, G, iters, init=None, warm_iters=None):
    """GPU and oracle quantisation + reconstruction of the same input."""
    X_np = np_bits(X)
    dtype = BF16 if X.dtype == torch.bfloat16 else FP32
    cfg = q.config(K=K, T=T, group_size=G, iters=iters, warm_iters=warm_iters or iters)
    init_t = to_dev(init) if init is not None else None
    pg = q.quantize(X.cuda().contiguous(), cfg, init=init_t)
    Yg = np_bits(q.dequantize(pg))
    torch.cuda.synchronize()
    gpu = packed_np(pg)
    ref = ora.quantize(X_np, K=K, T=T, G=G, iters=(warm_iters or iters) if init is not None else iters,
                       init=init)
    H, N, d = X_np.shape
    Yr = ora.dequantize(ref, K=K, T=T, G=G, N=N, H=H, d=d, dtype=dtype)
    Yo = ora.dequantize(gpu, K=K, T=T, G=G, N=N, H=H, d=d, dtype=dtype)
    np.testing.assert_array_equal(Yg, Yo)     # GPU dequant of its own stream == oracle dequant
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


def test_streaming_cache_parity(q, ora):
    """qvg_append_chunk: chunk 0 cold, later chunks warm-started from the
    previous chunk's centroids; the fused dequantisation of the whole cache
    equals the oracle's chunk-by-chunk reconstruction."""
    from bit_kv_cache_qvg_b200 import synth
    K, T, G, I, Iw = 64, 2, 64, 6, 3
    H = 2
    stream = synth.PrototypeStream(H, 30, 52, kinds=[0, 1], seed=21)
    frames = [3, 3, 3, 1]
    cfg = q.config(K=K, T=T, group_size=G, iters=I, warm_iters=Iw)
    cache = q.Cache(cfg, H=H, max_tokens=sum(frames) * 1560, max_chunks=8)
    prev = None
    Ys = []
    xs = []
    for c, f in enumerate(frames):
        X = stream.next(f)
        cache.append(X.cuda())
        X_np = np_bits(X)
        xs.append(X_np)
        ref = ora.quantize(X_np, K=K, T=T, G=G, iters=I if prev is None else Iw, init=prev)
        gpu = packed_np(cache.chunk(c))
        torch.cuda.synchronize()
        compare_quantize(ora, X_np, gpu, ref, K, T, G, I if prev is None else Iw, BF16, init=prev)
        prev = gpu["centroids"]
        Ys.append(ora.dequantize(gpu, K=K, T=T, G=G, N=X_np.shape[1], H=H, d=128))
    assert cache.tokens == sum(frames) * 1560 and cache.chunks == len(frames)
    Y = np_bits(cache.dequantize())
    np.testing.assert_array_equal(Y, np.concatenate(Ys, axis=1))
    cache.close()


def test_full_size_sampled(q, ora):
    """LongCat-scale blocks (38,000 tokens = 25 frames of 38x40, K=256, T=2,
    G=64, 10 iterations) quantised in the benchmark's batch configuration;
    one block checked against the oracle in full, the reconstruction of every
    block checked against the oracle's reconstruction of the GPU stream."""
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
    Yo = ora.dequantize(gpu, K=256, T=2, G=64, N=38000, H=H, d=128)
    np.testing.assert_array_equal(Yg, Yo)
    h = 5                                            # a V block (outliers x1000)
    sub = {k: (v[:, h:h + 1] if k in ("assign", "centroids") else v[h:h + 1]) for k, v in gpu.items()}
    ref = ora.quantize(X_np[h:h + 1], K=256, T=2, G=64, iters=10)
    rep = compare_quantize(ora, X_np[h:h + 1], sub, ref, 256, 2, 64, 10, BF16)
    Yr = ora.dequantize(ref, K=256, T=2, G=64, N=38000, H=1, d=128)
    compare_reconstruction(ora, X_np[h:h + 1], Yg[h:h + 1], Yr, sub, ref, 64)
    print(rep)


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
