"""Thin ctypes binding of libqvg.so (the C ABI in include/qvg.h).

Argument marshalling only: every step of the codec runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  If the library is
missing, every call raises ``QvgError`` -- there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqvg.so")

BF16, FP32 = 0, 1
_DTYPES = {torch.bfloat16: BF16, torch.float32: FP32}
_TORCH = {BF16: torch.bfloat16, FP32: torch.float32}

STATUS = {
    0: "QVG_OK", 1: "QVG_ERR_INVALID_ARG", 2: "QVG_ERR_UNSUPPORTED", 3: "QVG_ERR_NO_MEMORY",
    4: "QVG_ERR_CUDA", 5: "QVG_ERR_DEVICE_TIMEOUT", 6: "QVG_ERR_WORKSPACE_TOO_SMALL",
    7: "QVG_ERR_CAPACITY",
}


class QvgError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" if what else STATUS.get(status, str(status)))


ASYM, SYM = 0, 1     # qvg_scale_mode: scale and zero point per group, or one scale per group


class Config(C.Structure):
    _fields_ = [("K", C.c_int32), ("T", C.c_int32), ("group_size", C.c_int32),
                ("bits", C.c_int32), ("iters", C.c_int32), ("warm_iters", C.c_int32),
                ("scale_mode", C.c_int32)]

    def __repr__(self):
        return (f"Config(K={self.K}, T={self.T}, group_size={self.group_size}, bits={self.bits}, "
                f"iters={self.iters}, warm_iters={self.warm_iters}, scale_mode={self.scale_mode})")


class Policy(C.Structure):
    """qvg_adaptive_policy: a ladder of (T, group_size) settings chosen per
    chunk from the mean E4M3 code of the chunk's group ranges."""
    _fields_ = [("levels", C.c_int32), ("T", C.c_int32 * 4), ("group_size", C.c_int32 * 4),
                ("thresholds", C.c_int32 * 3), ("probe_group", C.c_int32), ("refresh_every", C.c_int32)]


def policy(T, group_size, thresholds=(), probe_group=16, refresh_every=0) -> Policy:
    """A policy of len(T) levels; thresholds in sixteenths of an E4M3 code."""
    p = Policy()
    p.levels = len(T)
    if not 1 <= p.levels <= 4 or len(group_size) != p.levels or len(thresholds) != p.levels - 1:
        raise QvgError(1, "policy: 1-4 levels, one group size per level, levels - 1 thresholds")
    for i in range(p.levels):
        p.T[i], p.group_size[i] = T[i], group_size[i]
    for i, t in enumerate(thresholds):
        p.thresholds[i] = t
    p.probe_group, p.refresh_every = probe_group, refresh_every
    return p


class _Packed(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scale", C.c_void_p), ("zero", C.c_void_p),
                ("assign", C.c_void_p), ("centroids", C.c_void_p)]


_lib = None

# Every exported symbol of include/qvg.h with its ctypes signature.
_SIGS = {
    "qvg_status_string": (C.c_char_p, [C.c_int]),
    "qvg_version": (C.c_char_p, []),
    "qvg_packed_bytes": (C.c_size_t, [C.POINTER(Config), C.c_int64, C.c_int32, C.c_int32, C.c_int]),
    "qvg_workspace_bytes": (C.c_size_t, [C.POINTER(Config), C.c_int64, C.c_int32, C.c_int32, C.c_int]),
    "qvg_quantize": (C.c_int, [C.POINTER(Config), C.c_void_p, C.c_int, C.c_int64, C.c_int32, C.c_int32,
                               C.c_void_p, C.POINTER(_Packed), C.c_void_p, C.c_size_t, C.c_void_p]),
    "qvg_quantize_static": (C.c_int, [C.POINTER(Config), C.c_void_p, C.c_int, C.c_int64, C.c_int32,
                                      C.c_int32, C.c_void_p, C.POINTER(_Packed), C.c_void_p]),
    "qvg_dequantize": (C.c_int, [C.POINTER(Config), C.POINTER(_Packed), C.c_int, C.c_int64, C.c_int32,
                                 C.c_int32, C.c_void_p, C.c_void_p]),
    "qvg_workspace_status": (C.c_int, [C.c_void_p, C.c_size_t, C.c_void_p]),
    "qvg_workspace_flagged": (C.c_int64, [C.c_void_p, C.c_size_t, C.c_void_p]),
    "qvg_cache_create": (C.c_int, [C.POINTER(Config), C.c_int, C.c_int32, C.c_int32, C.c_int64, C.c_int32,
                                   C.c_int64, C.POINTER(C.c_void_p)]),
    "qvg_cache_create_adaptive": (C.c_int, [C.POINTER(Config), C.POINTER(Policy), C.c_int, C.c_int32, C.c_int32,
                                            C.c_int64, C.c_int32, C.c_int64, C.POINTER(C.c_void_p)]),
    "qvg_cache_chunk_info": (C.c_int, [C.c_void_p, C.c_int32, C.POINTER(C.c_int32), C.POINTER(C.c_int32),
                                       C.POINTER(C.c_int32), C.POINTER(C.c_uint64)]),
    "qvg_cache_status": (C.c_int, [C.c_void_p, C.c_void_p]),
    "qvg_static_status": (C.c_int, [C.c_void_p]),
    "qvg_append_chunk": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p]),
    "qvg_cache_dequantize": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "qvg_cache_tokens": (C.c_int64, [C.c_void_p]),
    "qvg_cache_chunks": (C.c_int32, [C.c_void_p]),
    "qvg_cache_chunk_view": (C.c_int, [C.c_void_p, C.c_int32, C.POINTER(_Packed), C.POINTER(C.c_int64),
                                       C.POINTER(C.c_int64)]),
    "qvg_cache_device_bytes": (C.c_size_t, [C.c_void_p]),
    "qvg_cache_destroy": (None, [C.c_void_p]),
    "qvg_rope_tables_bytes": (C.c_size_t, [C.c_int32, C.c_int64]),
    "qvg_rope_tables": (C.c_int, [C.c_double, C.c_int32, C.c_int64, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qvg_attention": (C.c_int, [C.POINTER(Config), C.POINTER(_Packed), C.POINTER(_Packed), C.c_int64, C.c_int32,
                                C.c_int32, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_size_t, C.c_void_p,
                                C.c_void_p, C.c_size_t, C.c_void_p]),
    "qvg_attention_set_split": (C.c_int32, [C.c_int32]),
    "qvg_attention_split": (C.c_int32, [C.POINTER(Config), C.c_int64, C.c_int32, C.c_int64, C.c_size_t]),
    "qvg_attention_workspace_bytes": (C.c_size_t, [C.POINTER(Config), C.c_int64, C.c_int32, C.c_int64]),
    "qvg_profile_enable": (None, [C.c_int]),
    "qvg_profile_reset": (None, []),
    "qvg_profile_launches": (C.c_int64, []),
    "qvg_profile_report": (C.c_int, [C.c_char_p, C.c_size_t]),
}


def lib():
    """Load libqvg.so (raises QvgError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise QvgError(4, f"libqvg.so not found at {LIB_PATH}; run "
                              "python -m bit_kv_cache_qvg_b200.build")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return sorted(_SIGS)


def status_string(st: int) -> str:
    return lib().qvg_status_string(st).decode()


def _check(st: int, what: str):
    if st != 0:
        raise QvgError(st, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def config(K=256, T=2, group_size=64, iters=10, warm_iters=3, bits=2, scale_mode=ASYM) -> Config:
    return Config(K, T, group_size, bits, iters, warm_iters, scale_mode)


# Named operating points.  With one E4M3 scale per group the closed-form
# compression at K = 256 on a 38,000-token block is 6.97x for "qvg" and
# 5.03x for "qvg-pro" (the m.163.com article on Quant VideoGen, section 六,
# reports 6.94-7.05x and 4.97-5.20x; section 七 names G = 64 the best
# trade-off and G = 16 the high-quality setting).  The pages do not print the
# settings themselves: these are the ones the closed form admits.
PRESETS = {
    "qvg": dict(K=256, T=1, group_size=64, scale_mode=SYM),
    "qvg-pro": dict(K=256, T=4, group_size=16, scale_mode=SYM),
}


def preset(name: str, iters=10, warm_iters=3) -> Config:
    return config(iters=iters, warm_iters=warm_iters, **PRESETS[name])


@dataclass
class Packed:
    """Packed tensors of H blocks of N tokens (layouts of qvg_packed)."""
    codes: torch.Tensor       # [H][N][d/4] uint8
    scale: torch.Tensor       # [H][N][d/G] uint8 (E4M3)
    zero: torch.Tensor        # [H][N][d/G] uint8 (E4M3)
    assign: torch.Tensor      # [T][H][N] uint8
    centroids: torch.Tensor   # [T][H][K][d] storage dtype
    cfg: Config
    N: int
    H: int
    d: int
    dtype: int

    def struct(self) -> _Packed:
        return _Packed(_ptr(self.codes), _ptr(self.scale), _ptr(self.zero) if self.zero.numel() else None,
                       _ptr(self.assign) if self.assign.numel() else None,
                       _ptr(self.centroids) if self.centroids.numel() else None)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.scale, self.zero, self.assign, self.centroids))


def packed_bytes(cfg: Config, N: int, H: int, d: int = 128, dtype: int = BF16) -> int:
    return int(lib().qvg_packed_bytes(C.byref(cfg), N, H, d, dtype))


def workspace_bytes(cfg: Config, N: int, H: int, d: int = 128, dtype: int = BF16) -> int:
    return int(lib().qvg_workspace_bytes(C.byref(cfg), N, H, d, dtype))


def alloc_packed(cfg: Config, N: int, H: int, d: int = 128, dtype: int = BF16, device="cuda") -> Packed:
    G, T, K = cfg.group_size, cfg.T, cfg.K
    u8 = dict(dtype=torch.uint8, device=device)
    return Packed(
        codes=torch.empty((H, N, d // 4), **u8),
        scale=torch.empty((H, N, d // G), **u8),
        zero=torch.empty((H, N, d // G) if cfg.scale_mode == ASYM else (0,), **u8),
        assign=torch.empty((T, H, N), **u8),
        centroids=torch.empty((T, H, K, d), dtype=_TORCH[dtype], device=device),
        cfg=cfg, N=N, H=H, d=d, dtype=dtype)


def alloc_workspace(cfg: Config, N: int, H: int, d: int = 128, dtype: int = BF16, device="cuda"):
    n = workspace_bytes(cfg, N, H, d, dtype)
    if n == 0:
        raise QvgError(1, "workspace size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:16].zero_()     # status word and near-tie counter
    return ws


def quantize(X: torch.Tensor, cfg: Config, init: Optional[torch.Tensor] = None,
             out: Optional[Packed] = None, workspace: Optional[torch.Tensor] = None,
             stream=None) -> Packed:
    """qvg_quantize on X [H][N][d] (bf16 or fp32, CUDA, contiguous)."""
    if X.dim() != 3 or not X.is_contiguous():
        raise QvgError(1, "X must be a contiguous [H][N][d] tensor")
    H, N, d = X.shape
    dt = _DTYPES[X.dtype]
    if out is None:
        out = alloc_packed(cfg, N, H, d, dt, X.device)
    if workspace is None:
        workspace = alloc_workspace(cfg, N, H, d, dt, X.device)
    ps = out.struct()
    st = lib().qvg_quantize(C.byref(cfg), _ptr(X), dt, N, H, d, _ptr(init), C.byref(ps),
                            _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "qvg_quantize")
    return out


def quantize_static(X: torch.Tensor, cfg: Config, init: Optional[torch.Tensor] = None,
                    out: Optional[Packed] = None, stream=None) -> Packed:
    """qvg_quantize_static on X [H][N][d]: no workspace argument; the library's
    per-device static reserve is the scratch (calls must not overlap)."""
    if X.dim() != 3 or not X.is_contiguous():
        raise QvgError(1, "X must be a contiguous [H][N][d] tensor")
    H, N, d = X.shape
    dt = _DTYPES[X.dtype]
    if out is None:
        out = alloc_packed(cfg, N, H, d, dt, X.device)
    ps = out.struct()
    st = lib().qvg_quantize_static(C.byref(cfg), _ptr(X), dt, N, H, d, _ptr(init), C.byref(ps), _stream(stream))
    _check(st, "qvg_quantize_static")
    return out


def dequantize(p: Packed, Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if Y is None:
        Y = torch.empty((p.H, p.N, p.d), dtype=_TORCH[p.dtype], device=p.codes.device)
    ps = p.struct()
    st = lib().qvg_dequantize(C.byref(p.cfg), C.byref(ps), p.dtype, p.N, p.H, p.d, _ptr(Y), _stream(stream))
    _check(st, "qvg_dequantize")
    return Y


def rope_tables(max_pos: int, base: float = 10000.0, d: int = 128, device="cuda", stream=None) -> torch.Tensor:
    """qvg_rope_tables: the rotary (cos, sin) tables for positions 0 .. max_pos
    (a uint8 device tensor; its first 4 bytes are the attention status word)."""
    n = int(lib().qvg_rope_tables_bytes(d, max_pos))
    if n == 0:
        raise QvgError(1, "qvg_rope_tables_bytes")
    t = torch.empty(n, dtype=torch.uint8, device=device)
    _check(lib().qvg_rope_tables(float(base), d, max_pos, _ptr(t), n, _stream(stream)), "qvg_rope_tables")
    return t


def attention(kp: Packed, vp: Packed, Q: torch.Tensor, q_pos: torch.Tensor, tables: torch.Tensor,
              O: Optional[torch.Tensor] = None, stream=None, workspace=True) -> torch.Tensor:
    """qvg_attention: softmax(rope(Q) rope(K^)^T / sqrt(d)) V^ per head over the
    compressed caches kp (keys, before the rotary embedding) and vp (values);
    Q [H][Nq][d] bf16, q_pos [Nq] int64 (device); returns O [H][Nq][d] fp32.
    `workspace`: a uint8 device tensor, True (one of
    qvg_attention_workspace_bytes is allocated) or None (no workspace)."""
    if Q.dim() != 3 or not Q.is_contiguous() or Q.dtype != torch.bfloat16:
        raise QvgError(1, "Q must be a contiguous bf16 [H][Nq][d] tensor")
    H, Nq, d = Q.shape
    if O is None:
        O = torch.empty((H, Nq, d), dtype=torch.float32, device=Q.device)
    if workspace is True:
        n = attention_workspace_bytes(kp.cfg, kp.N, H, Nq)
        workspace = torch.empty(n, dtype=torch.uint8, device=Q.device) if n > 0 else None
    ws_ptr, ws_n = (_ptr(workspace), workspace.numel()) if workspace is not None else (None, 0)
    ks, vs = kp.struct(), vp.struct()
    _check(lib().qvg_attention(C.byref(kp.cfg), C.byref(ks), C.byref(vs), kp.N, H, d, _ptr(Q),
                               _ptr(q_pos), Nq, _ptr(tables), tables.numel(), _ptr(O), ws_ptr, ws_n,
                               _stream(stream)),
           "qvg_attention")
    return O


def attention_set_split(split: int) -> int:
    """qvg_attention_set_split: fix the cluster split of qvg_attention for the
    process (1 .. 8; 0 = the library's choice); returns the previous setting."""
    prev = int(lib().qvg_attention_set_split(int(split)))
    if prev < 0:
        raise QvgError(1, "qvg_attention_set_split")
    return prev


def attention_split(cfg: Config, Nk: int, H: int, Nq: int, ws_bytes: int = 0) -> int:
    """qvg_attention_split: the ranges the cache of a query block is cut into
    by a qvg_attention call with these sizes and a workspace of ws_bytes."""
    n = int(lib().qvg_attention_split(C.byref(cfg), Nk, H, Nq, ws_bytes))
    if n < 0:
        raise QvgError(1, "qvg_attention_split")
    return n


def attention_workspace_bytes(cfg: Config, Nk: int, H: int, Nq: int) -> int:
    """qvg_attention_workspace_bytes: the workspace the preferred cut needs."""
    return int(lib().qvg_attention_workspace_bytes(C.byref(cfg), Nk, H, Nq))


def profile_enable(on: bool = True):
    lib().qvg_profile_enable(1 if on else 0)


def profile_reset():
    lib().qvg_profile_reset()


def profile_launches() -> int:
    return int(lib().qvg_profile_launches())


def profile_report() -> dict:
    import json
    n = lib().qvg_profile_report(None, 0)
    buf = C.create_string_buffer(max(n, 2))
    st = lib().qvg_profile_report(buf, len(buf))
    if st != 0:
        raise QvgError(4, "qvg_profile_report")
    return json.loads(buf.value.decode())


def workspace_flagged(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().qvg_workspace_flagged(_ptr(workspace), workspace.numel(), _stream(stream)))


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().qvg_workspace_status(_ptr(workspace), workspace.numel(), _stream(stream)))


def static_status(stream=None) -> int:
    """qvg_static_status: read and clear the static reserve's status word."""
    return int(lib().qvg_static_status(_stream(stream)))


class _DevView:
    """__cuda_array_interface__ wrapper of a raw device pointer (for views)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = dict(shape=tuple(shape), typestr=typestr, data=(ptr, False),
                                             version=3, strides=None)


def _view(ptr, shape, torch_dtype):
    if ptr is None or 0 in shape:
        return torch.empty(shape, dtype=torch_dtype, device="cuda")
    typestr = {torch.uint8: "|u1", torch.float32: "<f4", torch.bfloat16: "<u2"}[torch_dtype]
    t = torch.as_tensor(_DevView(ptr, shape, typestr), device="cuda")
    return t.view(torch.bfloat16) if torch_dtype == torch.bfloat16 else t


class Cache:
    """Streaming compressed KV cache (qvg_cache_*): append chunks, each
    warm-started from the previous chunk's centroids; dequantise all.  With a
    Policy (qvg_cache_create_adaptive) every chunk takes its own T and G."""

    def __init__(self, cfg: Config, H: int, max_tokens: int, max_chunks: int, d: int = 128,
                 dtype: int = BF16, max_chunk_tokens: int = 0, policy: Optional[Policy] = None):
        self.cfg, self.H, self.d, self.dtype, self.policy = cfg, H, d, dtype, policy
        self._h = C.c_void_p()
        h = C.c_void_p()
        if policy is None:
            _check(lib().qvg_cache_create(C.byref(cfg), dtype, H, d, max_tokens, max_chunks, max_chunk_tokens,
                                          C.byref(h)), "qvg_cache_create")
        else:
            _check(lib().qvg_cache_create_adaptive(C.byref(cfg), C.byref(policy), dtype, H, d, max_tokens,
                                                   max_chunks, max_chunk_tokens, C.byref(h)),
                   "qvg_cache_create_adaptive")
        self._h = h

    def chunk_info(self, c: int) -> dict:
        """qvg_cache_chunk_info: level, T, G and statistic of chunk c."""
        lvl, T, G, S = C.c_int32(), C.c_int32(), C.c_int32(), C.c_uint64()
        _check(lib().qvg_cache_chunk_info(self._h, c, C.byref(lvl), C.byref(T), C.byref(G), C.byref(S)),
               "qvg_cache_chunk_info")
        return dict(level=lvl.value, T=T.value, G=G.value, stat=S.value)

    def append(self, X: torch.Tensor, stream=None):
        if X.dim() != 3 or X.shape[0] != self.H or X.shape[2] != self.d or not X.is_contiguous():
            raise QvgError(1, "chunk must be a contiguous [H][N][d] tensor")
        _check(lib().qvg_append_chunk(self._h, _ptr(X), X.shape[1], _stream(stream)), "qvg_append_chunk")

    @property
    def tokens(self) -> int:
        return int(lib().qvg_cache_tokens(self._h))

    @property
    def chunks(self) -> int:
        return int(lib().qvg_cache_chunks(self._h))

    def device_bytes(self) -> int:
        return int(lib().qvg_cache_device_bytes(self._h))

    def status(self, stream=None) -> int:
        """qvg_cache_status: read and clear the cache's device status word."""
        return int(lib().qvg_cache_status(self._h, _stream(stream)))

    def dequantize(self, Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if Y is None:
            Y = torch.empty((self.H, self.tokens, self.d), dtype=_TORCH[self.dtype], device="cuda")
        _check(lib().qvg_cache_dequantize(self._h, _ptr(Y), _stream(stream)), "qvg_cache_dequantize")
        return Y

    def chunk(self, c: int) -> Packed:
        """Device views of chunk c's packed arrays (valid while the cache lives)."""
        v = _Packed()
        first, n = C.c_int64(), C.c_int64()
        _check(lib().qvg_cache_chunk_view(self._h, c, C.byref(v), C.byref(first), C.byref(n)),
               "qvg_cache_chunk_view")
        H, d, N, cfg = self.H, self.d, n.value, self.cfg
        if self.policy is not None:             # the chunk's own settings
            info = self.chunk_info(c)
            cfg = config(K=cfg.K, T=info["T"], group_size=info["G"], bits=cfg.bits, iters=cfg.iters,
                         warm_iters=cfg.warm_iters, scale_mode=cfg.scale_mode)
        G, T, K = cfg.group_size, cfg.T, cfg.K
        return Packed(codes=_view(v.codes, (H, N, d // 4), torch.uint8),
                      scale=_view(v.scale, (H, N, d // G), torch.uint8),
                      zero=_view(v.zero, (H, N, d // G) if cfg.scale_mode == ASYM else (0,), torch.uint8),
                      assign=_view(v.assign, (T, H, N), torch.uint8),
                      centroids=_view(v.centroids, (T, H, K, d), _TORCH[self.dtype]),
                      cfg=cfg, N=N, H=H, d=d, dtype=self.dtype)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().qvg_cache_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
