"""qvg_attention (the consumer of the compressed cache, with dequantisation
and the rotary embedding fused into the K/V load) against the oracle's fp64
attention over the oracle's reconstruction of the same packed caches (the
oracle's own compression of seeded K and V blocks).

Tolerance, from the arithmetic of the kernel: the rotated queries and keys
enter the tensor cores rounded to bf16 (relative error 2^-9 each), so a score
s_j = q'.k'_j / sqrt(d) is off by at most eps_j = 2^-8 sum_c |q'_c k'_jc| /
sqrt(d) (plus fp32 sums, far smaller); a perturbation of at most eps in every
score changes the softmax weights by at most 2(e^(2 eps) - 1) in total, and
rounding the weights to bf16 adds 2^-8 more.  So output element (i, c) is
within max_j |v_jc| (2(e^(2 eps_i) - 1) + 2^-7) of the exact value, eps_i
the row's largest eps_j.  The tests also check that the typical error is far
below that bound."""
import numpy as np
import pytest
import torch

from gpu_util import np_bits, to_dev, values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


def _run_case(q, ora, cfg, H, Nk, Nq, q_scale, seed, base=10000.0):
    from bit_kv_cache_qvg_b200 import synth
    frames = -(-Nk // 1560)
    Xk = synth.block_batch(H, synth.KVShape(frames, 30, 52), seed=seed, kinds=[0] * H)[:, :Nk].contiguous()
    Xv = synth.block_batch(H, synth.KVShape(frames, 30, 52), seed=seed + 1, kinds=[1] * H)[:, :Nk].contiguous()
    # the caches are the oracle's own packed streams of the seeded blocks
    mode = cfg.scale_mode
    kn = ora.quantize(np_bits(Xk), K=cfg.K, T=cfg.T, G=cfg.group_size, iters=cfg.iters, scale_mode=mode)
    vn = ora.quantize(np_bits(Xv), K=cfg.K, T=cfg.T, G=cfg.group_size, iters=cfg.iters, scale_mode=mode)
    kp, vp = (q.Packed(codes=to_dev(p["codes"]), scale=to_dev(p["scale"]), zero=to_dev(p["zero"]),
                       assign=to_dev(p["assign"]), centroids=to_dev(p["centroids"]),
                       cfg=cfg, N=Nk, H=H, d=128, dtype=0) for p in (kn, vn))
    rng = np.random.default_rng(seed)
    Qf = (rng.standard_normal((H, Nq, 128)) * q_scale).astype(np.float32)
    Q = torch.from_numpy(Qf).to(torch.bfloat16)
    qpos = np.arange(Nk, Nk + Nq, dtype=np.int64)
    tables = q.rope_tables(Nk + Nq, base=base)
    O = q.attention(kp, vp, Q.cuda(), torch.from_numpy(qpos).cuda(), tables)
    torch.cuda.synchronize()
    assert q.workspace_status(tables) == 0
    O = O.cpu().numpy()
    Kh = values(ora.dequantize(kn, K=cfg.K, T=cfg.T, G=cfg.group_size, N=Nk, H=H, d=128, scale_mode=mode))
    Vh = values(ora.dequantize(vn, K=cfg.K, T=cfg.T, G=cfg.group_size, N=Nk, H=H, d=128, scale_mode=mode))
    Qv = values(np_bits(Q))
    worst = 0.0
    for h in range(H):
        ref = ora.attention(Qv[h].astype(np.float32), qpos, Kh[h].astype(np.float32), Vh[h].astype(np.float32),
                            base=base)
        qr = ora.rope(Qv[h].astype(np.float32), qpos, base)
        kr = ora.rope(Kh[h].astype(np.float32), np.arange(Nk), base)
        eps = 2.0 ** -8 * (np.abs(qr) @ np.abs(kr).T).max(axis=1) / np.sqrt(128)
        # element (i, c): the weights' total change times channel c's largest |v|
        bound = np.outer(2 * np.expm1(2 * eps) + 2.0 ** -7, np.abs(Vh[h]).max(axis=0)) + 1e-30
        err = np.abs(O[h] - ref)
        assert np.all(err <= bound), (h, float((err / bound).max()))
        worst = max(worst, float(np.median(err / bound)))
    return worst


@pytest.mark.parametrize("H,Nk,Nq,T,G,K,mode,q_scale", [
    (2, 1000, 200, 2, 64, 64, 0, 0.05),      # ragged cache and query tiles, two stages
    (2, 256, 128, 1, 64, 256, 1, 0.05),      # the QVG point (one scale per group), whole tiles
    (1, 77, 33, 0, 32, 1, 0, 0.2),           # plain rounding, one partial tile each
    (2, 4680, 130, 4, 16, 256, 1, 0.02),     # the QVG-Pro point, a Self-Forcing-scale chunk
    (2, 2900, 600, 2, 64, 128, 0, 0.05),     # three query blocks: two CTAs share each tile, one CTA has no queries
    (1, 1300, 512, 1, 32, 64, 1, 0.05),      # two whole query blocks, one pair
    (2, 3000, 600, 4, 16, 256, 1, 0.02),     # the QVG-Pro point, paired (four stages: no prefetch of the next step)
    (1, 2000, 300, 3, 32, 128, 0, 0.05),     # three stages, paired
    (1, 700, 260, 5, 64, 32, 0, 0.05),       # five stages: the instance with the stage count at run time
])
def test_attention_matches_oracle(q, ora, H, Nk, Nq, T, G, K, mode, q_scale):
    cfg = q.config(K=K, T=T, group_size=G, iters=3, scale_mode=mode)
    typical = _run_case(q, ora, cfg, H, Nk, Nq, q_scale, seed=Nk + T)
    assert typical < 0.25          # the usual error is well inside the worst-case bound


@pytest.mark.parametrize("split", [2, 3, 4, 8])
@pytest.mark.parametrize("Nq", [200, 300])
def test_attention_split_over_a_cluster_matches_oracle(q, ora, split, Nq):
    """The cache of each query block split over a cluster of `split` CTAs
    (ragged ranges: 8 tiles over 3 CTAs; 8 CTAs of one tile each) stays
    within the bound.  With one block of 256 queries (Nq = 200) the CTAs
    are alone; with two (Nq = 300) they come in pairs that share the
    reconstruction, and a cluster holds at most 4 ranges."""
    cfg = q.config(K=64, T=2, group_size=64, iters=3, scale_mode=0)
    prev = q.attention_set_split(split)
    try:
        assert q.attention_split(cfg, 1000, 2, Nq) == min(split, 8 if Nq <= 256 else 4)
        typical = _run_case(q, ora, cfg, 2, 1000, Nq, 0.05, seed=1002)
    finally:
        q.attention_set_split(prev)
    assert typical < 0.25


def test_attention_split_over_clusters_matches_oracle(q, ora):
    """With a workspace the cache of a query block is cut into up to 16
    ranges over clusters, merged by a second kernel: here 32 tiles into 16
    ranges for each of four pairs of query blocks."""
    cfg = q.config(K=64, T=2, group_size=64, iters=3, scale_mode=0)
    ws = q.attention_workspace_bytes(cfg, 4000, 2, 600)
    assert ws == 16 * 2 * 600 * (128 * 4 + 8)
    assert q.attention_split(cfg, 4000, 2, 600, ws) == 16
    assert q.attention_split(cfg, 4000, 2, 600, ws - 1) < 16
    typical = _run_case(q, ora, cfg, 2, 4000, 600, 0.05, seed=4004)
    assert typical < 0.25


def test_attention_splits_agree(q):
    """Each CTA of a split rounds its weights to bf16 against its own running
    maximum (as the unsplit kernel does against the maximum so far), so the
    splits differ by weight roundings of 2^-9 relative, far inside the
    bound, and never by more than 2^-7 of the largest output."""
    from bit_kv_cache_qvg_b200 import synth
    cfg = q.config(K=32, T=1, group_size=64, iters=2)
    H, Nk, Nq = 2, 3000, 520
    X = synth.block_batch(H, synth.KVShape(2, 30, 52), seed=9, kinds=[0, 1])[:, :Nk].contiguous().cuda()
    kp = q.quantize(X, cfg)
    Q = (torch.randn((H, Nq, 128), generator=torch.Generator().manual_seed(4)) * 0.1).to(torch.bfloat16).cuda()
    pos = torch.arange(Nk, Nk + Nq, dtype=torch.int64, device="cuda")
    tables = q.rope_tables(Nk + Nq)
    outs = {}
    for split in (1, 2, 3, 5, 8):
        prev = q.attention_set_split(split)
        try:
            outs[split] = q.attention(kp, kp, Q, pos, tables).cpu()
        finally:
            q.attention_set_split(prev)
    outs["clusters"] = q.attention(kp, kp, Q, pos, tables, workspace=None).cpu()
    outs["global"] = q.attention(kp, kp, Q, pos, tables).cpu()
    torch.cuda.synchronize()
    assert q.workspace_status(tables) == 0
    scale = outs[1].abs().max().item()
    for split, O in outs.items():
        assert torch.isfinite(O).all()
        assert (O - outs[1]).abs().max().item() <= 2.0 ** -7 * scale, split


def test_attention_split_setting_is_checked(q):
    cfg = q.config(K=256, T=2, group_size=64)
    with pytest.raises(q.QvgError):
        q.attention_set_split(9)
    with pytest.raises(q.QvgError):
        q.attention_set_split(-1)
    auto = q.attention_split(cfg, 38000, 32, 1520)
    assert 1 <= auto <= 4
    ws = q.attention_workspace_bytes(cfg, 38000, 32, 1520)
    assert 1 <= q.attention_split(cfg, 38000, 32, 1520, ws) <= 16
    assert q.attention_split(cfg, 100, 32, 1520) == 1      # one tile: nothing to split
    prev = q.attention_set_split(3)
    try:
        assert q.attention_split(cfg, 38000, 32, 1520) == 3
        assert q.attention_split(cfg, 200, 32, 1520) == 2   # capped at the two tiles
    finally:
        assert q.attention_set_split(prev) == 3


def test_attention_reports_a_stale_timeout_and_rejects_uncovered_positions(q):
    from bit_kv_cache_qvg_b200 import synth
    cfg = q.config(K=16, T=1, group_size=64, iters=2)
    X = synth.block_batch(1, synth.KVShape(1, 10, 30), seed=3, kinds=[0]).cuda()
    kp = q.quantize(X, cfg)
    Q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    pos = torch.arange(8, dtype=torch.int64, device="cuda")
    small = q.rope_tables(400)                       # positions 0 .. 400 are covered
    big = q.rope_tables(5000)
    q.attention(kp, kp, Q, pos, big)
    torch.cuda.synchronize()
    X2 = synth.block_batch(1, synth.KVShape(1, 30, 52), seed=3, kinds=[0]).cuda()  # 1560 tokens
    kp2 = q.quantize(X2, cfg)
    with pytest.raises(q.QvgError) as e:
        q.attention(kp2, kp2, Q, pos, small)         # token 1559 is beyond the small tables
    assert e.value.status == 1
    small[:4] = torch.tensor([1, 0, 0, 0], dtype=torch.uint8)   # a timeout recorded earlier
    torch.cuda.synchronize()
    with pytest.raises(q.QvgError) as e:
        q.attention(kp, kp, Q, pos, small)
    assert e.value.status == 5
    assert q.workspace_status(small) == 5 and q.workspace_status(small) == 0
