"""Failure handling on the GPU, without any GPU fault.

QVG_FAULT_INJECT=timeout makes the first CTA of the tensor-core assignment
withhold one tile load and give its waits a 1 ms limit, so that those bounded
waits run out.  The kernel records the timeout in the sticky status word of
the workspace (or cache, or static reserve), its other roles drain, it frees
its tensor memory and returns; the context stays usable.  The next call on the
same object returns QVG_ERR_DEVICE_TIMEOUT without queueing anything, the
status query reads and clears the word, and work after that matches the
oracle again.

QVG_FAULT_INJECT=alloc and =stream make the host report a failed device
allocation or a stream error; the cache stays consistent (no handle, or no
chunk appended) and the next call without injection succeeds."""
import numpy as np
import pytest
import torch

from gpu_util import BF16, compare_quantize, np_bits, packed_np

pytestmark = pytest.mark.gpu

TIMEOUT, NO_MEMORY, CUDA, OK = 5, 3, 4, 0


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


def _blocks(seed, H=2, frames=1):
    from bit_kv_cache_qvg_b200 import synth
    return synth.block_batch(H, synth.KVShape(frames, 30, 52), seed=seed, kinds=[h % 2 for h in range(H)])


def _check_against_oracle(ora, X, p, K, T, G, iters):
    gpu = packed_np(p)
    ref = ora.quantize(np_bits(X), K=K, T=T, G=G, iters=iters)
    compare_quantize(ora, np_bits(X), gpu, ref, K, T, G, iters, BF16)


def test_workspace_timeout_is_reported_then_cleared(q, ora, monkeypatch):
    X = _blocks(5)
    Xd = X.cuda()
    H, N = X.shape[0], X.shape[1]
    cfg = q.config(K=256, T=2, group_size=64, iters=2)
    ws = q.alloc_workspace(cfg, N, H)
    monkeypatch.setenv("QVG_FAULT_INJECT", "timeout")
    q.quantize(Xd, cfg, workspace=ws)          # queued; the timeout happens on the device
    torch.cuda.synchronize()
    monkeypatch.delenv("QVG_FAULT_INJECT")
    with pytest.raises(q.QvgError) as e:       # the next call on this workspace reports it
        q.quantize(Xd, cfg, workspace=ws)
    assert e.value.status == TIMEOUT
    assert q.workspace_status(ws) == TIMEOUT   # read and cleared
    assert q.workspace_status(ws) == OK
    p = q.quantize(Xd, cfg, workspace=ws)      # the same workspace works again
    torch.cuda.synchronize()
    assert q.workspace_status(ws) == OK
    _check_against_oracle(ora, X, p, 256, 2, 64, 2)
    p2 = q.quantize(Xd, cfg)                   # and so does a fresh one
    torch.cuda.synchronize()
    _check_against_oracle(ora, X, p2, 256, 2, 64, 2)


def test_static_reserve_timeout_is_reported_then_cleared(q, ora, monkeypatch):
    X = _blocks(6)
    Xd = X.cuda()
    cfg = q.config(K=256, T=1, group_size=64, iters=2)
    assert q.static_status() == OK
    monkeypatch.setenv("QVG_FAULT_INJECT", "timeout")
    q.quantize_static(Xd, cfg)
    torch.cuda.synchronize()
    monkeypatch.delenv("QVG_FAULT_INJECT")
    with pytest.raises(q.QvgError) as e:
        q.quantize_static(Xd, cfg)
    assert e.value.status == TIMEOUT
    assert q.static_status() == TIMEOUT
    assert q.static_status() == OK
    p = q.quantize_static(Xd, cfg)
    torch.cuda.synchronize()
    assert q.static_status() == OK
    _check_against_oracle(ora, X, p, 256, 1, 64, 2)


@pytest.mark.parametrize("adaptive", [False, True])
def test_cache_timeout_leaves_the_cache_usable(q, ora, monkeypatch, adaptive):
    """A timeout in chunk 0 is reported by the next append (nothing
    committed), read and cleared by the cache's status query; appends then go
    on.  The adaptive cache is given a policy that starts every chunk cold,
    so chunk 1 does not depend on chunk 0's invalid tables and is checked
    against the oracle; the fixed cache warm-starts from them, so only its
    bookkeeping is checked."""
    from bit_kv_cache_qvg_b200 import synth
    H = 2
    s = synth.PrototypeStream(H, 30, 52, kinds=[0, 1], seed=9)
    cfg = q.config(K=256, T=2, group_size=64, iters=3, warm_iters=2)
    pol = q.policy(T=[2], group_size=[64], refresh_every=1) if adaptive else None
    cache = q.Cache(cfg, H=H, max_tokens=6 * 1560, max_chunks=6, max_chunk_tokens=1560, policy=pol)
    monkeypatch.setenv("QVG_FAULT_INJECT", "timeout")
    cache.append(s.next(1).cuda())             # chunk 0: its packed data is invalid
    torch.cuda.synchronize()
    monkeypatch.delenv("QVG_FAULT_INJECT")
    X1 = s.next(1)
    with pytest.raises(q.QvgError) as e:
        cache.append(X1.cuda())
    assert e.value.status == TIMEOUT and cache.chunks == 1
    assert cache.status() == TIMEOUT and cache.status() == OK
    cache.append(X1.cuda())                    # appends go on after the status is read
    torch.cuda.synchronize()
    assert cache.chunks == 2 and cache.tokens == 2 * 1560 and cache.status() == OK
    if adaptive:
        ref = ora.quantize(np_bits(X1), K=256, T=2, G=64, iters=3)
        compare_quantize(ora, np_bits(X1), packed_np(cache.chunk(1)), ref, 256, 2, 64, 3, BF16)
    cache.close()


def test_injected_allocation_and_stream_errors(q, monkeypatch):
    cfg = q.config(K=64, T=2, group_size=64, iters=2, warm_iters=1)
    monkeypatch.setenv("QVG_FAULT_INJECT", "alloc")
    with pytest.raises(q.QvgError) as e:
        q.Cache(cfg, H=2, max_tokens=4 * 1560, max_chunks=4, max_chunk_tokens=1560)
    assert e.value.status == NO_MEMORY
    monkeypatch.delenv("QVG_FAULT_INJECT")
    cache = q.Cache(cfg, H=2, max_tokens=4 * 1560, max_chunks=4, max_chunk_tokens=1560)
    X = _blocks(8).cuda()
    cache.append(X)
    monkeypatch.setenv("QVG_FAULT_INJECT", "stream")
    with pytest.raises(q.QvgError) as e:
        cache.append(X)
    assert e.value.status == CUDA and cache.chunks == 1     # the failed append is not counted
    with pytest.raises(q.QvgError) as e:
        cache.dequantize()
    assert e.value.status == CUDA
    with pytest.raises(q.QvgError) as e:
        q.quantize(X, cfg)
    assert e.value.status == CUDA
    monkeypatch.delenv("QVG_FAULT_INJECT")
    cache.append(X)
    Y = cache.dequantize()
    torch.cuda.synchronize()
    assert cache.chunks == 2 and Y.shape == (2, 2 * 1560, 128)
    x = X.float()
    for c in range(2):                         # both chunks reconstruct the input closely
        err = ((Y[:, c * 1560:(c + 1) * 1560].float() - x) ** 2).mean() / (x ** 2).mean()
        assert float(err) < 1e-2
    cache.close()
    # attention over a compressed cache: the injected stream error, then a clean call
    kp = q.quantize(X, cfg)
    Q = torch.zeros((X.shape[0], 8, 128), dtype=torch.bfloat16, device="cuda")
    pos = torch.arange(8, dtype=torch.int64, device="cuda")
    tables = q.rope_tables(X.shape[1])
    monkeypatch.setenv("QVG_FAULT_INJECT", "stream")
    with pytest.raises(q.QvgError) as e:
        q.attention(kp, kp, Q, pos, tables)
    assert e.value.status == CUDA
    monkeypatch.delenv("QVG_FAULT_INJECT")
    O = q.attention(kp, kp, Q, pos, tables)
    torch.cuda.synchronize()
    assert torch.isfinite(O).all() and q.workspace_status(tables) == 0
