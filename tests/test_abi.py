"""CPU checks of the C ABI: the library loads, exports every function that
include/qvg.h declares, and its host-only functions (sizes, argument checks)
behave as declared.  No kernel is launched here."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    qvg.lib()
    return qvg


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"QVG_API[^;(]*?\b(qvg_\w+)\s*\(", src, re.S))
    return names


def test_library_exports_every_declared_symbol(q):
    declared = _declared()
    assert len(declared) >= 15
    L = C.CDLL(q.LIB_PATH)
    for name in declared:
        assert hasattr(L, name), name
    assert declared == set(q.exported_symbols())


def test_version_and_status_strings(q):
    assert q.lib().qvg_version().decode().startswith("qvg-b200")
    assert q.status_string(0) == "ok"
    assert q.status_string(6) == "workspace too small"


@pytest.mark.parametrize("K,T,G,N,H,dtype", [
    (16, 1, 16, 512, 1, 1), (256, 2, 64, 4680, 12, 0), (256, 2, 64, 38000, 32, 0),
    (64, 4, 32, 38000, 32, 0), (256, 0, 64, 100, 3, 0), (7, 3, 8, 1000, 5, 1),
])
@pytest.mark.parametrize("mode", [0, 1])
def test_packed_bytes_matches_oracle_closed_form(q, ora, K, T, G, N, H, dtype, mode):
    cfg = q.config(K=K, T=T, group_size=G, scale_mode=mode)
    assert q.packed_bytes(cfg, N, H, 128, dtype) == ora.packed_bytes(K, T, G, N, H, 128, dtype=dtype,
                                                                     scale_mode=mode)


def test_presets_are_the_closed_form_operating_points(q, ora):
    """The named points land in the pages' ranges by the library's own size."""
    for name, lo, hi in (("qvg", 6.94, 7.05), ("qvg-pro", 4.97, 5.20)):
        cfg = q.preset(name)
        ratio = 38000 * 128 * 2 / q.packed_bytes(cfg, 38000, 1)
        assert lo <= ratio <= hi, (name, ratio)
    assert q.packed_bytes(q.config(scale_mode=2), 100, 1) == 0


def test_workspace_bytes_positive_and_monotone(q):
    cfg = q.config(K=256, T=2, group_size=64)
    one = q.workspace_bytes(cfg, 38000, 1)
    many = q.workspace_bytes(cfg, 38000, 64)
    assert 0 < one <= many
    assert q.workspace_bytes(q.config(K=0), 100, 1) == 0


def _quantize_status(q, cfg, N=512, H=1, d=128, dtype=0, init=None, X=0x1000, ws=0x10000,
                     ws_bytes=1 << 30, packed=None):
    p = packed or q._Packed(0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    return q.lib().qvg_quantize(C.byref(cfg), X, dtype, N, H, d, init, C.byref(p), ws, ws_bytes, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(K=0), 1), (dict(K=257), 1), (dict(T=-1), 1), (dict(bits=3), 1),
    (dict(group_size=6), 1), (dict(group_size=48), 1), (dict(iters=0), 1),
    (dict(group_size=4), 2), (dict(T=9), 2), (dict(scale_mode=2), 1), (dict(scale_mode=-1), 1),
])
def test_quantize_rejects_bad_config_without_touching_the_gpu(q, kw, expect):
    args = dict(K=16, T=1, group_size=16, iters=4)
    args.update(kw)
    assert _quantize_status(q, q.config(**args)) == expect


def test_quantize_rejects_bad_shapes_and_pointers(q):
    cfg = q.config(K=16, T=1, group_size=16, iters=4)
    assert _quantize_status(q, cfg, d=64) == 2                  # kernels are d = 128
    assert _quantize_status(q, cfg, N=8) == 1                   # N < K on a cold start
    assert _quantize_status(q, cfg, H=0) == 1
    assert _quantize_status(q, cfg, X=None) == 1
    assert _quantize_status(q, cfg, X=0x1001) == 1              # misaligned X
    assert _quantize_status(q, cfg, ws=None) == 1
    assert _quantize_status(q, cfg, dtype=7) == 1
    assert _quantize_status(q, cfg, ws_bytes=16) == 6           # workspace too small
    assert _quantize_status(q, cfg, packed=q._Packed(0x2000, 0x3000, 0x4000, None, None)) == 1


def test_dequantize_and_cache_reject_bad_arguments(q):
    cfg = q.config(K=16, T=1, group_size=16, iters=4)
    p = q._Packed(0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    L = q.lib()
    assert L.qvg_dequantize(C.byref(cfg), C.byref(p), 0, 10, 1, 128, None, None) == 1
    assert L.qvg_dequantize(C.byref(cfg), None, 0, 10, 1, 128, 0x1000, None) == 1
    assert L.qvg_dequantize(C.byref(q.config(K=300)), C.byref(p), 0, 10, 1, 128, 0x1000, None) == 1
    h = C.c_void_p()
    assert L.qvg_cache_create(C.byref(cfg), 0, 1, 128, 0, 4, 0, C.byref(h)) == 1
    assert L.qvg_cache_create(C.byref(cfg), 0, 1, 96, 100, 4, 0, C.byref(h)) == 2
    assert L.qvg_cache_create(C.byref(cfg), 0, 1, 128, 100, 4, -1, C.byref(h)) == 1
    assert L.qvg_cache_create(C.byref(cfg), 0, 1, 128, 100, 4, 8, C.byref(h)) == 1    # a chunk below K
    assert not h.value
    assert L.qvg_append_chunk(None, 0x1000, 10, None) == 1
    assert L.qvg_cache_tokens(None) == 0 and L.qvg_cache_chunks(None) == 0


def test_workspace_covers_two_waves_when_blocks_exceed_one(q, monkeypatch):
    """Host logic of the wave lanes: a wave holds up to one block per SM (the
    SM count the library reads; 148 on this part, the fallback without a
    device); when the blocks need more than one wave the workspace holds two
    waves, one per lane; QVG_WAVE_LANES=1 asks for one wave."""
    cfg = q.config(K=256, T=2, group_size=64)
    N = 38000
    sizes = {H: q.workspace_bytes(cfg, N, H) for H in range(1, 400)}
    # past one wave the size no longer grows with H: W is the largest one-wave batch
    W = min(H for H in sizes if sizes[H] == sizes[399]) - 1
    assert all(sizes[H] < sizes[H + 1] for H in range(1, W))
    assert sizes[W + 1] == 2 * sizes[W]
    assert all(sizes[H] == 2 * sizes[W] for H in range(W + 1, 400))
    monkeypatch.setenv("QVG_WAVE_LANES", "1")
    assert q.workspace_bytes(cfg, N, W + 1) == sizes[W]


def test_fault_injection_follows_argument_checks(q, monkeypatch):
    """QVG_FAULT_INJECT=alloc makes qvg_cache_create report NO_MEMORY before
    any device allocation and leave no handle; arguments are checked first, so
    an invalid call still reports INVALID_ARG.  The binding raises QvgError
    with the status."""
    cfg = q.config(K=16, T=1, group_size=16, iters=4, warm_iters=2)
    L = q.lib()
    h = C.c_void_p()
    monkeypatch.setenv("QVG_FAULT_INJECT", "stream,alloc")
    assert L.qvg_cache_create(C.byref(cfg), 0, 2, 128, 1000, 4, 0, C.byref(h)) == 3
    assert not h.value
    assert L.qvg_cache_create(C.byref(cfg), 0, 2, 128, 0, 4, 0, C.byref(h)) == 1
    with pytest.raises(q.QvgError) as e:
        q.Cache(cfg, H=2, max_tokens=1000, max_chunks=4)
    assert e.value.status == 3 and "NO_MEMORY" in str(e.value)
    # a name that is not in the list injects nothing: arguments are still checked
    monkeypatch.setenv("QVG_FAULT_INJECT", "allocate")
    assert L.qvg_cache_create(C.byref(cfg), 0, 2, 128, 1000, 0, 0, C.byref(h)) == 1
    assert q.status_string(5) == "device-side wait timed out"


def test_adaptive_cache_rejects_bad_policies_without_touching_the_gpu(q, monkeypatch):
    """qvg_cache_create_adaptive checks the policy and every level's setting
    before any device work: 1-4 levels, ascending thresholds, a supported
    probe group, a non-negative refresh period, a valid (T, G) per level.
    With QVG_FAULT_INJECT=alloc a valid policy reaches the allocation and
    reports NO_MEMORY, leaving no handle."""
    cfg = q.config(K=16, T=9, group_size=7, iters=4, warm_iters=2)   # T and G come from the policy
    L = q.lib()
    h = C.c_void_p()

    def create(pol, **kw):
        a = dict(dtype=0, H=2, d=128, max_tokens=1000, max_chunks=4, max_chunk_tokens=0)
        a.update(kw)
        return L.qvg_cache_create_adaptive(C.byref(cfg), C.byref(pol), a["dtype"], a["H"], a["d"],
                                           a["max_tokens"], a["max_chunks"], a["max_chunk_tokens"], C.byref(h))

    good = q.policy(T=[1, 2], group_size=[64, 16], thresholds=[16 * 50])
    bad = [q.policy(T=[1, 2, 4], group_size=[64, 32, 16], thresholds=[900, 800]),   # descending
           q.policy(T=[1, 2], group_size=[64, 16], thresholds=[800], probe_group=12),
           q.policy(T=[1, 2], group_size=[64, 16], thresholds=[800], refresh_every=-1),
           q.policy(T=[1, 2], group_size=[64, 24], thresholds=[800]),            # G does not divide d
           q.policy(T=[1, 9], group_size=[64, 16], thresholds=[800])]            # T above 8
    zero = q.policy(T=[1], group_size=[64])
    zero.levels = 0
    five = q.policy(T=[1], group_size=[64])
    five.levels = 5
    for pol in bad + [zero, five]:
        assert create(pol) in (1, 2), pol
    assert create(good, d=96) == 1                 # 64 does not divide 96
    assert create(good, max_tokens=0) == 1
    assert L.qvg_cache_create_adaptive(C.byref(cfg), None, 0, 2, 128, 1000, 4, 0, C.byref(h)) == 1
    assert not h.value
    monkeypatch.setenv("QVG_FAULT_INJECT", "alloc")
    assert create(good) == 3 and not h.value
    with pytest.raises(q.QvgError):
        q.policy(T=[1, 2], group_size=[64], thresholds=[1])
    assert L.qvg_cache_chunk_info(None, 0, None, None, None, None) == 1


def test_status_queries_reject_missing_objects(q):
    L = q.lib()
    assert L.qvg_cache_status(None, None) == 1
    assert L.qvg_workspace_status(None, 0, None) == 1


def test_attention_host_calls_without_a_gpu(q):
    """qvg_rope_tables_bytes is the closed form 256 + (max_pos + 1) * 512 bytes
    (d = 128, positions below 2^24); qvg_attention rejects missing or
    misaligned arguments, and caches whose positions the tables do not cover,
    before it touches the GPU; qvg_attention_set_split takes 0 .. 8 only; the
    planner queries answer -1 and 0 without a device."""
    import torch
    L = q.lib()
    assert L.qvg_rope_tables_bytes(128, 0) == 256 + 512
    assert L.qvg_rope_tables_bytes(128, 39519) == 256 + 39520 * 512
    assert L.qvg_rope_tables_bytes(128, (1 << 24) - 1) == 256 + (1 << 24) * 512
    assert L.qvg_rope_tables_bytes(128, 1 << 24) == 0
    assert L.qvg_rope_tables_bytes(128, -1) == 0
    assert L.qvg_rope_tables_bytes(96, 100) == 0
    cfg = q.config(K=16, T=1, group_size=64, iters=2)
    p = q._Packed(0x2000, 0x3000, 0x4000, 0x5000, 0x6000)
    tb = L.qvg_rope_tables_bytes(128, 999)                    # positions 0 .. 999

    def att(Nk=1000, d=128, Q=0x10000, Nq=8, tbytes=tb, O=0x40000, ws=None, wsn=0, kp=p):
        return L.qvg_attention(C.byref(cfg), C.byref(kp) if kp is not None else None, C.byref(p), Nk, 1, d, Q,
                               0x20000, Nq, 0x30000, tbytes, O, ws, wsn, None)

    assert att(Q=None) == 1
    assert att(O=None) == 1
    assert att(Q=0x10008) == 1                 # Q must be 16-byte aligned
    assert att(ws=0x50008, wsn=4096) == 1      # and so must a workspace
    assert att(Nq=0) == 1
    assert att(Nk=1001) == 1                   # token 1000 lies beyond the tables
    assert att(tbytes=256) == 1                # tables with no position
    assert att(kp=None) == 1
    assert att(d=96) != 0
    assert L.qvg_attention_set_split(9) == -1 and L.qvg_attention_set_split(-1) == -1
    prev = L.qvg_attention_set_split(3)
    assert L.qvg_attention_set_split(prev) == 3
    if not torch.cuda.is_available():
        assert L.qvg_attention_split(C.byref(cfg), 1000, 1, 8, 0) == -1
        assert L.qvg_attention_workspace_bytes(C.byref(cfg), 1000, 1, 8) == 0
    assert L.qvg_attention_split(C.byref(q.config(K=300)), 1000, 1, 8, 0) == -1
    assert L.qvg_attention_workspace_bytes(C.byref(cfg), 0, 1, 8) == 0
