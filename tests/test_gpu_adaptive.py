"""The streaming cache with per-chunk settings (qvg_cache_create_adaptive)
against the oracle: for every chunk the range statistic, the level the
policy picks, the number of stages started from the previous chunk's
centroids, and the packed streams are identical to the oracle's
(range_stat, adaptive_level, adaptive_warm_stages and quantize_ex chained
over the oracle's own chunks); the whole-cache reconstruction equals the
concatenation of the oracle's chunk reconstructions.  The pages (the
m.163.com article on Quant VideoGen, section 九) name adapting the
compression parameters to the content as future work; the rule is this
library's and the oracle states it in plain code."""
import numpy as np
import pytest
import torch

from gpu_util import BF16, compare_quantize, np_bits, packed_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


def _chunks(H, frames, scales, seed):
    """Chunks of a synthetic stream, each scaled by a power of two (exact in
    bf16), which moves every group's range code by eight per doubling."""
    from bit_kv_cache_qvg_b200 import synth
    stream = synth.PrototypeStream(H, 30, 52, kinds=[h % 2 for h in range(H)], seed=seed)
    return [(stream.next(f).float() * s).to(torch.bfloat16).contiguous() for f, s in zip(frames, scales)]


def _mean_code16(ora, X_np, pg):
    H, N, d = X_np.shape
    return 16 * ora.range_stat(X_np, pg) // (H * N * d // pg)


@pytest.mark.parametrize("mode,Ts,Gs,offsets,refresh,scales,frames", [
    # four levels in the asymmetric mode; chunk 3 is a refresh chunk
    (0, [1, 2, 1, 3], [64, 32, 16, 64], [-128, 128, 384], 3,
     [1.0, 4.0, 0.25, 4.0, 1.0, 16.0, 1.0], [1, 1, 2, 1, 1, 1, 1]),
    # the QVG / QVG-Pro ladder with one scale per group
    (1, [1, 4], [64, 16], [128], 0, [1.0, 4.0, 4.0, 1.0, 0.5], [2, 1, 1, 1, 1]),
])
def test_adaptive_cache_matches_oracle(q, ora, mode, Ts, Gs, offsets, refresh, scales, frames):
    H, K, I, Iw, PG = 2, 32, 4, 2, 16
    chunks = _chunks(H, frames, scales, seed=31 + mode)
    Xs = [np_bits(x) for x in chunks]
    base = _mean_code16(ora, Xs[0], PG)
    th = [base + o for o in offsets]
    pol = q.policy(T=Ts, group_size=Gs, thresholds=th, probe_group=PG, refresh_every=refresh)
    cfg = q.config(K=K, T=0, group_size=64, iters=I, warm_iters=Iw, scale_mode=mode)
    N = sum(x.shape[1] for x in Xs)
    cache = q.Cache(cfg, H=H, max_tokens=N, max_chunks=len(Xs), max_chunk_tokens=max(x.shape[1] for x in Xs),
                    policy=pol)
    prev, prev_T, levels, Ys = None, 0, [], []
    for c, (X, X_np) in enumerate(zip(chunks, Xs)):
        cache.append(X.cuda())
        n = X_np.shape[1]
        S = ora.range_stat(X_np, PG)
        lvl = ora.adaptive_level(S, H * n * 128 // PG, th, len(Ts))
        T, G = Ts[lvl], Gs[lvl]
        warm = ora.adaptive_warm_stages(c, prev_T, T, refresh)
        ref = ora.quantize_ex(X_np, K=K, T=T, G=G, iters=I, warm_iters=Iw, warm_stages=warm,
                              init=prev["centroids"] if warm else None, scale_mode=mode)
        assert cache.chunk_info(c) == dict(level=lvl, T=T, G=G, stat=S)
        gpu = packed_np(cache.chunk(c))
        torch.cuda.synchronize()
        compare_quantize(ora, X_np, gpu, ref, K, T, G, I, BF16)
        Ys.append(ora.dequantize(ref, K=K, T=T, G=G, N=n, H=H, d=128, scale_mode=mode))
        prev, prev_T = ref, T
        levels.append(lvl)
    assert len(set(levels)) == len(Ts), levels          # the stream visits every level
    assert cache.tokens == N and cache.chunks == len(Xs) and cache.status() == 0
    np.testing.assert_array_equal(np_bits(cache.dequantize()), np.concatenate(Ys, axis=1))
    cache.close()


def test_adaptive_cache_rejects_a_short_cold_chunk_and_stays_usable(q, ora):
    """A chunk with fewer than K tokens is rejected when a stage of its level
    has to start cold (the first chunk always does); nothing is committed and
    the next chunk goes in as the first."""
    H, K = 1, 64
    pol = q.policy(T=[1, 2], group_size=[64, 32], thresholds=[0], probe_group=32)   # every chunk at level 1
    cfg = q.config(K=K, T=0, iters=3, warm_iters=2)
    cache = q.Cache(cfg, H=H, max_tokens=4000, max_chunks=4, max_chunk_tokens=1560, policy=pol)
    chunks = _chunks(H, [1, 1], [1.0, 1.0], seed=5)
    with pytest.raises(q.QvgError) as e:
        cache.append(chunks[0][:, :K - 1].contiguous().cuda())
    assert e.value.status == 1 and cache.chunks == 0 and cache.tokens == 0
    cache.append(chunks[0].cuda())
    cache.append(chunks[1][:, :K - 1].contiguous().cuda())   # warm in both stages: short is fine
    torch.cuda.synchronize()
    X0, X1 = np_bits(chunks[0]), np_bits(chunks[1][:, :K - 1])
    r0 = ora.quantize_ex(X0, K=K, T=2, G=32, iters=3, warm_iters=2, warm_stages=0)
    r1 = ora.quantize_ex(X1, K=K, T=2, G=32, iters=3, warm_iters=2, warm_stages=2, init=r0["centroids"])
    for c, (X_np, ref) in enumerate(((X0, r0), (X1, r1))):
        assert cache.chunk_info(c)["level"] == 1
        compare_quantize(ora, X_np, packed_np(cache.chunk(c)), ref, K, 2, 32, 3, BF16)
    cache.close()


def test_fixed_cache_reports_its_own_settings(q):
    cfg = q.config(K=16, T=2, group_size=32, iters=3, warm_iters=2)
    cache = q.Cache(cfg, H=1, max_tokens=2000, max_chunks=2)
    cache.append(_chunks(1, [1], [1.0], seed=2)[0].cuda())
    assert cache.chunk_info(0) == dict(level=0, T=2, G=32, stat=0)
    with pytest.raises(q.QvgError):
        cache.chunk_info(1)
    cache.close()
