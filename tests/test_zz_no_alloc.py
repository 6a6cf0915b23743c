"""qvg_quantize_static (the allocation-free variant of qvg_quantize, whose
scratch is the library's static per-device reserve) against qvg_quantize with
a caller workspace: same inputs, two static calls in a row, every output
compared.  The file is named to be collected last, so that it also runs after
every other test has used the library in the same process."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


def _host(p):
    return {k: getattr(p, k).cpu().numpy() for k in ("codes", "scale", "zero", "assign")} | {
        "centroids": p.centroids.view(torch.int16).cpu().numpy() if p.centroids.dtype == torch.bfloat16
        else p.centroids.cpu().numpy()}


def _assert_same(a, b, what):
    # Same kernels on the same inputs: the test tolerance is equality.
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=f"{what}: {k}")


@pytest.mark.parametrize("K,T,G,iters,frames,H", [
    (256, 2, 64, 3, 3, 3),      # Self-Forcing-scale chunk shape, 3 heads: 4,680 tokens per block
    (64, 1, 16, 4, 1, 5),       # one frame, smaller K: five blocks in one wave
    (256, 2, 64, 2, 25, 3),     # 39,000 tokens per block: two blocks per wave, so two waves
])
def test_static_reserve_matches_workspace_call(q, K, T, G, iters, frames, H):
    from bit_kv_cache_qvg_b200 import synth
    X = synth.block_batch(H, synth.KVShape(frames, 30, 52), seed=K + H,
                          kinds=[h % 2 for h in range(H)]).cuda()
    cfg = q.config(K=K, T=T, group_size=G, iters=iters)
    ref = _host(q.quantize(X, cfg))
    torch.cuda.synchronize()
    # two calls in a row on the same stream and the same reserve
    first = q.quantize_static(X, cfg)
    second = q.quantize_static(X, cfg)
    torch.cuda.synchronize()
    _assert_same(ref, _host(first), "first static call")
    _assert_same(ref, _host(second), "second static call")


def test_static_reserve_warm_start_matches(q):
    from bit_kv_cache_qvg_b200 import synth
    s = synth.PrototypeStream(2, 30, 52, kinds=[0, 1], seed=5)
    a, b = s.next(3).cuda(), s.next(3).cuda()
    cfg = q.config(K=256, T=2, group_size=64, iters=4, warm_iters=2)
    cold = q.quantize(a, cfg)
    ref = _host(q.quantize(b, cfg, init=cold.centroids))
    got = _host(q.quantize_static(b, cfg, init=cold.centroids))
    torch.cuda.synchronize()
    _assert_same(ref, got, "warm static call")


def test_static_reserve_rejects_block_too_large(q):
    cfg = q.config(K=256, T=2, group_size=64, iters=1)
    N = 200_000                           # one block's working set exceeds the 32 MiB reserve
    assert q.workspace_bytes(cfg, N, 1) > 32 << 20
    X = torch.zeros((1, N, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.QvgError) as e:
        q.quantize_static(X, cfg)
    assert e.value.status == 6             # QVG_ERR_WORKSPACE_TOO_SMALL, before any work is queued
