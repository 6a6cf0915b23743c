"""Shared helpers of the GPU parity tests: move packed outputs between the
CUDA path and the oracle, and assess agreement with the tolerances of the
codec's contract (bit-exact dequantisation; >= 99.9 % agreement of
assignments and codes, disagreements only at near-ties; reconstruction MSE
within 1 % and max error <= 1e-2 x group scale where codes agree)."""
import numpy as np
import torch

BF16, FP32 = 0, 1


def np_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


def packed_np(p) -> dict:
    return dict(codes=np_bits(p.codes), scale=np_bits(p.scale), zero=np_bits(p.zero),
                assign=np_bits(p.assign), centroids=np_bits(p.centroids))


def values(a: np.ndarray) -> np.ndarray:
    """float64 values of bf16 bits or fp32."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def unpack_codes(codes: np.ndarray, d: int = 128) -> np.ndarray:
    j = np.arange(d)
    return (codes[..., j // 4] >> (2 * (j % 4))) & 3


def e4m3_values(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).float().numpy()


def compare_quantize(ora, X_np, gpu: dict, ref: dict, K, T, G, iters, dtype, init=None):
    """Compare GPU quantisation with the oracle's: the agreement of every
    packed array, then the contract of this implementation, which takes every
    decision the oracle's way (assignments in fp64, exact centroid sums,
    bit-exact E4M3 and rounding): the packed streams are identical.  The
    spec tolerance (>= 99.9 % agreement, disagreements only at
    near-ties) is looser than this, so a pass here implies it."""
    d = X_np.shape[-1]
    rep = {}
    rep["bit_exact"] = all(np.array_equal(gpu[k], ref[k]) for k in ("codes", "scale", "zero", "assign", "centroids"))
    rep["codes_agree"] = float((unpack_codes(gpu["codes"], d) == unpack_codes(ref["codes"], d)).mean())
    rep["scale_agree"] = float((gpu["scale"] == ref["scale"]).mean())
    rep["zero_agree"] = float((gpu["zero"] == ref["zero"]).mean())
    rep["assign_agree"] = [float((gpu["assign"][t] == ref["assign"][t]).mean()) for t in range(T)]
    rep["centroids_agree"] = [float((gpu["centroids"][t] == ref["centroids"][t]).mean()) for t in range(T)]
    assert rep["bit_exact"], rep
    return rep


def compare_reconstruction(ora, X_np, Yg: np.ndarray, Yr: np.ndarray, gpu, ref, G):
    x = values(X_np)
    yg, yr = values(Yg), values(Yr)
    mse_g = float(((yg - x) ** 2).mean())
    mse_r = float(((yr - x) ** 2).mean())
    assert abs(mse_g - mse_r) <= 0.01 * mse_r + 1e-30, (mse_g, mse_r)
    d = x.shape[-1]
    agree = unpack_codes(gpu["codes"], d) == unpack_codes(ref["codes"], d)
    T = gpu["assign"].shape[0]
    for t in range(T):
        agree &= (gpu["assign"][t] == ref["assign"][t])[..., None]
    s = np.repeat(np.abs(e4m3_values(ref["scale"])), G, axis=-1)
    err = np.abs(yg - yr)
    assert np.all(err[agree] <= 1e-2 * s[agree] + 0.0), float(err[agree].max())
    return mse_g, mse_r
