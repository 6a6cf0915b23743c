"""ctypes wrapper of the plain C oracle (``qvg_oracle.c``).

Test infrastructure only: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path never
imports this module, and this module imports nothing from the product package.

Every function takes and returns numpy arrays.  bf16 data travels as
``np.uint16`` bit patterns, fp32 data as ``np.float32``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qvg_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

BF16, FP32 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: -O2, no fast-math, no FMA contraction."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
               "-fopenmp", "-fPIC", "-shared", SRC, "-o", LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        i64, i32, vp, f64 = C.c_int64, C.c_int, C.c_void_p, C.c_double
        L.ref_e4m3_encode.restype = C.c_uint8
        L.ref_e4m3_encode.argtypes = [C.c_float]
        L.ref_e4m3_decode.restype = C.c_float
        L.ref_e4m3_decode.argtypes = [C.c_uint8]
        L.ref_bf16_round.restype = C.c_uint16
        L.ref_bf16_round.argtypes = [f64]
        for n in ("ref_e4m3_encode_array", "ref_e4m3_decode_array", "ref_bf16_round_array"):
            getattr(L, n).argtypes = [vp, vp, i64]
            getattr(L, n).restype = None
        L.ref_set_threads.argtypes = [i32]
        L.ref_get_threads.restype = i32
        L.ref_sqdist.restype = f64
        L.ref_sqdist.argtypes = [vp, vp, i32]
        L.ref_assign.argtypes = [vp, i64, i32, vp, i32, vp]
        L.ref_objective.restype = f64
        L.ref_objective.argtypes = [vp, i64, i32, vp, vp]
        L.ref_update.argtypes = [vp, i64, i32, vp, i32, i32, vp]
        L.ref_exact_sum.restype = f64
        L.ref_exact_sum.argtypes = [vp, i64]
        L.ref_kmeans.argtypes = [vp, i64, i32, i32, i32, i32, vp, vp, vp]
        L.ref_residual.argtypes = [vp, i64, i32, vp, vp, i32, vp]
        L.ref_group_quant.argtypes = [vp, i64, i32, i32, vp, vp, vp]
        L.ref_group_quant_sym.argtypes = [vp, i64, i32, i32, vp, vp]
        L.ref_quantize.restype = i32
        L.ref_quantize.argtypes = [i32, i32, i32, i32, i32, i32, vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]
        L.ref_quantize_ex.restype = i32
        L.ref_quantize_ex.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, vp, i64, i32, i32, vp,
                                      vp, vp, vp, vp, vp]
        L.ref_range_stat.restype = C.c_uint64
        L.ref_range_stat.argtypes = [vp, i32, i64, i32, i32, i32]
        L.ref_adaptive_level.restype = i32
        L.ref_adaptive_level.argtypes = [C.c_uint64, i64, vp, i32]
        L.ref_adaptive_warm_stages.restype = i32
        L.ref_adaptive_warm_stages.argtypes = [i32, i32, i32, i32]
        L.ref_dequantize.restype = i32
        L.ref_dequantize.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i64, i32, i32, vp]
        L.ref_rope.argtypes = [vp, i64, i32, vp, f64, vp]
        L.ref_rope.restype = None
        L.ref_attention.restype = i32
        L.ref_attention.argtypes = [vp, vp, i64, vp, vp, i64, i32, f64, vp]
        L.ref_kv_cache_bytes.restype = f64
        L.ref_kv_cache_bytes.argtypes = [i64, i64, i64, i64]
        L.ref_bits_per_element.restype = f64
        L.ref_bits_per_element.argtypes = [i32, i32, i32, i32, i64, i32, i32, i32]
        L.ref_packed_bytes.restype = i64
        L.ref_packed_bytes.argtypes = [i32, i32, i32, i32, i64, i32, i32, i32, i32]
        _lib = L
    return _lib


# ---------------------------------------------------------------- formats
def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ref_e4m3_encode_array(_p(x), _p(out), x.size)
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().ref_e4m3_decode_array(_p(c), _p(out), c.size)
    return out


def bf16_round(x) -> np.ndarray:
    """bf16 bits (uint16) nearest to each double, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().ref_bf16_round_array(_p(x), _p(out), x.size)
    return out


def bf16_to_f32(b) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def set_threads(n: int) -> None:
    lib().ref_set_threads(int(n))


def get_threads() -> int:
    return int(lib().ref_get_threads())


# ---------------------------------------------------------------- k-means
def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def sqdist(r, c) -> float:
    r, c = _f32(r), _f32(c)
    return float(lib().ref_sqdist(_p(r), _p(c), r.size))


def assign(R, Cc) -> np.ndarray:
    R, Cc = _f32(R), _f32(Cc)
    N, d = R.shape
    pi = np.empty(N, np.uint8)
    lib().ref_assign(_p(R), N, d, _p(Cc), Cc.shape[0], _p(pi))
    return pi


def objective(R, Cc, pi) -> float:
    R, Cc = _f32(R), _f32(Cc)
    pi = np.ascontiguousarray(pi, dtype=np.uint8)
    return float(lib().ref_objective(_p(R), R.shape[0], R.shape[1], _p(Cc), _p(pi)))


def exact_sum(x) -> float:
    """The exact sum of fp32 values, rounded once to fp64 (the update's sum)."""
    x = _f32(x).ravel()
    return float(lib().ref_exact_sum(_p(x), x.size))


def update(R, pi, Cc, dtype=BF16) -> np.ndarray:
    R = _f32(R)
    out = _f32(Cc).copy()
    pi = np.ascontiguousarray(pi, dtype=np.uint8)
    lib().ref_update(_p(R), R.shape[0], R.shape[1], _p(pi), out.shape[0], dtype, _p(out))
    return out


def kmeans(R, C0, iters, dtype=BF16, trace=False):
    """Returns (C, pi[, trace]) for one block; values carried as float32."""
    R = _f32(R)
    N, d = R.shape
    Cc = _f32(C0).copy()
    pi = np.empty(N, np.uint8)
    tr = np.empty(2 * iters, np.float64) if trace else None
    lib().ref_kmeans(_p(R), N, d, Cc.shape[0], iters, dtype, _p(Cc), _p(pi),
                     _p(tr) if trace else None)
    return (Cc, pi, tr) if trace else (Cc, pi)


def residual(R, Cc, pi, dtype=BF16) -> np.ndarray:
    R, Cc = _f32(R), _f32(Cc)
    pi = np.ascontiguousarray(pi, dtype=np.uint8)
    out = np.empty_like(R)
    lib().ref_residual(_p(R), R.shape[0], R.shape[1], _p(Cc), _p(pi), dtype, _p(out))
    return out


def group_quant(R, G):
    R = _f32(R)
    N, d = R.shape
    codes = np.empty((N, d // 4), np.uint8)
    scale = np.empty((N, d // G), np.uint8)
    zero = np.empty((N, d // G), np.uint8)
    lib().ref_group_quant(_p(R), N, d, G, _p(codes), _p(scale), _p(zero))
    return codes, scale, zero


def group_quant_sym(R, G):
    """Symmetric mode: one E4M3 scale per group; returns (codes, scale)."""
    R = _f32(R)
    N, d = R.shape
    codes = np.empty((N, d // 4), np.uint8)
    scale = np.empty((N, d // G), np.uint8)
    lib().ref_group_quant_sym(_p(R), N, d, G, _p(codes), _p(scale))
    return codes, scale


# ---------------------------------------------------------------- codec
def _dt(X):
    return FP32 if X.dtype == np.float32 else BF16


def quantize(X, K, T, G, iters, init=None, scale_mode=0):
    """X: [H][N][d] uint16 (bf16 bits) or float32.  Returns a dict of the
    packed arrays in the codec's layouts (scale_mode 1: one E4M3 scale per
    group; ``zero`` is then an empty array)."""
    X = np.ascontiguousarray(X)
    dtype = _dt(X)
    H, N, d = X.shape
    out = dict(
        codes=np.zeros((H, N, d // 4), np.uint8),
        scale=np.zeros((H, N, d // G), np.uint8),
        zero=np.zeros((H, N, d // G) if scale_mode == 0 else (0,), np.uint8),
        assign=np.zeros((T, H, N), np.uint8),
        centroids=np.zeros((T, H, K, d), X.dtype),
    )
    if init is not None:
        init = np.ascontiguousarray(init, dtype=X.dtype)
        assert init.shape == (T, H, K, d)
    rc = lib().ref_quantize(K, T, G, iters, dtype, scale_mode, _p(X), N, H, d,
                            _p(init) if init is not None else None,
                            _p(out["codes"]), _p(out["scale"]), _p(out["zero"]) if scale_mode == 0 else None,
                            _p(out["assign"]), _p(out["centroids"]))
    if rc != 0:
        raise ValueError("oracle quantize rejected its arguments")
    return out


def quantize_ex(X, K, T, G, iters, warm_iters, warm_stages, init=None, scale_mode=0):
    """quantize with the first warm_stages stages started from init (and
    warm_iters iterations), the rest cold (iters)."""
    X = np.ascontiguousarray(X)
    dtype = _dt(X)
    H, N, d = X.shape
    out = dict(
        codes=np.zeros((H, N, d // 4), np.uint8),
        scale=np.zeros((H, N, d // G), np.uint8),
        zero=np.zeros((H, N, d // G) if scale_mode == 0 else (0,), np.uint8),
        assign=np.zeros((T, H, N), np.uint8),
        centroids=np.zeros((T, H, K, d), X.dtype),
    )
    if init is not None:
        init = np.ascontiguousarray(init, dtype=X.dtype)
    rc = lib().ref_quantize_ex(K, T, G, iters, warm_iters, warm_stages, dtype, scale_mode, _p(X), N, H, d,
                               _p(init) if init is not None else None,
                               _p(out["codes"]), _p(out["scale"]), _p(out["zero"]) if scale_mode == 0 else None,
                               _p(out["assign"]), _p(out["centroids"]))
    if rc != 0:
        raise ValueError("oracle quantize_ex rejected its arguments")
    return out


def range_stat(X, G) -> int:
    """Sum of the E4M3 codes of the fp32 ranges (max - min) of every group of
    G channels of every token of X [H][N][d]."""
    X = np.ascontiguousarray(X)
    H, N, d = X.shape
    return int(lib().ref_range_stat(_p(X), _dt(X), N, H, d, G))


def adaptive_level(S, n_groups, thresholds, levels) -> int:
    th = np.ascontiguousarray(list(thresholds) + [0] * (3 - len(thresholds)), dtype=np.int32)
    return int(lib().ref_adaptive_level(int(S), int(n_groups), _p(th), int(levels)))


def adaptive_warm_stages(chunk, T_prev, T_cur, refresh_every) -> int:
    return int(lib().ref_adaptive_warm_stages(chunk, T_prev, T_cur, refresh_every))


def dequantize(packed, K, T, G, N, H, d, dtype=BF16, scale_mode=0) -> np.ndarray:
    Y = np.empty((H, N, d), np.float32 if dtype == FP32 else np.uint16)
    cen = np.ascontiguousarray(packed["centroids"])
    zero = np.ascontiguousarray(packed["zero"]) if scale_mode == 0 else None
    rc = lib().ref_dequantize(K, T, G, dtype, scale_mode,
                              _p(np.ascontiguousarray(packed["codes"])),
                              _p(np.ascontiguousarray(packed["scale"])),
                              _p(zero) if zero is not None else None,
                              _p(np.ascontiguousarray(packed["assign"])),
                              _p(cen), N, H, d, _p(Y))
    if rc != 0:
        raise ValueError("oracle dequantize rejected its arguments")
    return Y


# ---------------------------------------------------------------- closed forms
def kv_cache_bytes(L, tokens, hidden, nbytes) -> float:
    return float(lib().ref_kv_cache_bytes(L, tokens, hidden, nbytes))


def bits_per_element(K, T, G, N, d, bits=2, dtype=BF16, scale_mode=0) -> float:
    return float(lib().ref_bits_per_element(K, T, G, bits, N, d, dtype, scale_mode))


def packed_bytes(K, T, G, N, H, d, bits=2, dtype=BF16, scale_mode=0) -> int:
    return int(lib().ref_packed_bytes(K, T, G, bits, N, H, d, dtype, scale_mode))


# ---------------------------------------------------------------- attention
def rope(x, pos, base=10000.0) -> np.ndarray:
    """Rotary embedding (fp64) of x [n][d] at positions pos [n]."""
    x = _f32(x)
    n, d = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty((n, d), np.float64)
    lib().ref_rope(_p(x), n, d, _p(pos), float(base), _p(out))
    return out


def attention(Q, qpos, K, V, base=10000.0) -> np.ndarray:
    """softmax(rope(Q) rope(K)^T / sqrt(d)) V for one head (fp64); keys at
    positions 0 .. len(K)-1."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    nq, d = Q.shape
    nk = K.shape[0]
    qpos = np.ascontiguousarray(qpos, dtype=np.int64)
    O = np.empty((nq, d), np.float64)
    if lib().ref_attention(_p(Q), _p(qpos), nq, _p(K), _p(V), nk, d, float(base), _p(O)) != 0:
        raise ValueError("oracle attention rejected its arguments")
    return O
