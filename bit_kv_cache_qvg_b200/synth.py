"""Seeded synthetic KV-cache generator.

This module holds input synthesis only: none of the codec's arithmetic lives
here.  The oracle and the CUDA path both receive the exact bytes it returns.

The pages describe the data the codec is built for (m.163.com article on
Quant VideoGen, sections 二 and 三; gist.science/de, "Technische
Zusammenfassung" 1 and 2A): latent video tokens whose neighbours in space and
time are nearly equal, and whose K and V caches carry token-varying outlier
channels about 100x (K) and 1000x (V) larger than the rest.  The trained
models and datasets are not available, so tokens are drawn from a prototype
model with those properties:

* each block has ``n_proto`` Gaussian prototypes p ~ N(0, I_d);
* a per-channel log-normal scale sigma_c = exp(z_c), z_c ~ N(0, 1);
* the latent grid is cut into 4x4 spatial patches, each mapped to one
  prototype by a seeded uniform draw (or, in the tiny case, patch (py, px)
  takes prototype 4*py + px);
* prototypes evolve from frame to frame as an AR(1) process with correlation
  ``frame_corr`` (cosine about 0.95 between consecutive frames), or, in the
  tiny case, drift linearly by ``drift * f * delta_k``;
* token (f, y, x) = sigma * (p_f[k(y, x)] + noise * eps), eps ~ N(0, I_d);
* K blocks get ``n_outlier`` seeded channels multiplied by 100, V blocks by
  1000, each on a Bernoulli(0.2) subset of tokens;
* tokens are ordered frame-major, then row, then column.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass
class KVShape:
    frames: int
    grid_h: int
    grid_w: int
    d: int = 128

    @property
    def tokens(self) -> int:
        return self.frames * self.grid_h * self.grid_w


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def unit_seed(base: int, layer: int, head: int, kv: int) -> int:
    """Counter-style seed of one (layer, head, K|V) block."""
    return (base * 1_000_003 + layer * 7919 + head * 131 + kv * 17 + 1) % (2**62)


def tiny_block(seed: int = 0, frames: int = 2, grid: int = 16, d: int = 128,
               n_proto: int = 16, drift: float = 0.05, noise: float = 0.1,
               device="cpu") -> torch.Tensor:
    """The one-head fp32 case: 2 frames of 16x16 tokens, 16 prototypes tiled
    over 4x4 patches, linear temporal drift.  Returns [N, d] float32."""
    g = _gen(seed, device)
    sigma = torch.exp(torch.randn(d, generator=g, device=device))
    proto = torch.randn(n_proto, d, generator=g, device=device)
    delta = torch.randn(n_proto, d, generator=g, device=device)
    ys = torch.arange(grid, device=device)
    k = (4 * (ys[:, None] // 4) + (ys[None, :] // 4)).reshape(-1) % n_proto
    out = []
    for f in range(frames):
        eps = torch.randn(grid * grid, d, generator=g, device=device)
        out.append(sigma * (proto[k] + drift * f * delta[k] + noise * eps))
    return torch.cat(out, 0).float().contiguous()


class PrototypeStream:
    """Frame-by-frame generator for U independent blocks (e.g. heads x K/V).

    ``kinds`` gives, per block, 0 for a K block (outliers x100) or 1 for a V
    block (outliers x1000).  ``next(frames)`` returns [U, frames*H*W, d] in
    ``dtype``; successive calls continue the same AR(1) prototype process, so
    a long stream can be cut into chunks."""

    def __init__(self, U: int, grid_h: int, grid_w: int, d: int = 128, *, kinds=None,
                 seed: int = 0, n_proto: int = 64, frame_corr: float = 0.95,
                 noise: float = 0.1, n_outlier: int = 4, outlier_prob: float = 0.2,
                 outlier_scale=(100.0, 1000.0), patch: int = 4, device="cpu",
                 dtype=torch.bfloat16):
        self.U, self.gh, self.gw, self.d = U, grid_h, grid_w, d
        self.device, self.dtype = device, dtype
        self.rho, self.noise, self.prob = frame_corr, noise, outlier_prob
        self.g = _gen(seed, device)
        g = self.g
        kinds = torch.zeros(U, dtype=torch.long) if kinds is None else torch.as_tensor(kinds).long()
        self.sigma = torch.exp(torch.randn(U, d, generator=g, device=device))
        self.proto = torch.randn(U, n_proto, d, generator=g, device=device)
        nph, npw = math.ceil(grid_h / patch), math.ceil(grid_w / patch)
        pmap = torch.randint(0, n_proto, (U, nph, npw), generator=g, device=device)
        ys = torch.arange(grid_h, device=device) // patch
        xs = torch.arange(grid_w, device=device) // patch
        self.tok_proto = pmap[:, ys][:, :, xs].reshape(U, grid_h * grid_w)  # [U, HW]
        # n_outlier distinct channels per block
        ch = torch.rand(U, d, generator=g, device=device).argsort(dim=1)[:, :n_outlier]
        scale = torch.tensor(outlier_scale, device=device)[kinds.to(device)]  # [U]
        self.out_ch = ch
        self.out_scale = scale
        self.frame = 0

    def next(self, frames: int) -> torch.Tensor:
        U, d, HW = self.U, self.d, self.gh * self.gw
        g = self.g
        out = []
        for _ in range(frames):
            if self.frame > 0:
                eta = torch.randn(self.proto.shape, generator=g, device=self.device)
                self.proto = self.rho * self.proto + math.sqrt(1.0 - self.rho ** 2) * eta
            self.frame += 1
            base = torch.gather(self.proto, 1, self.tok_proto[:, :, None].expand(U, HW, d))
            eps = torch.randn(U, HW, d, generator=g, device=self.device)
            x = self.sigma[:, None, :] * (base + self.noise * eps)
            mask = torch.rand(U, HW, self.out_ch.shape[1], generator=g, device=self.device) < self.prob
            mult = torch.where(mask, self.out_scale[:, None, None], torch.ones((), device=self.device))
            cols = self.out_ch[:, None, :].expand(U, HW, self.out_ch.shape[1])
            x.scatter_(2, cols, torch.gather(x, 2, cols) * mult)
            out.append(x.to(self.dtype))
        return torch.cat(out, 1).contiguous()


def block_batch(U: int, shape: KVShape, *, seed: int, kinds=None, device="cpu",
                dtype=torch.bfloat16, n_proto: int = 64) -> torch.Tensor:
    """U independent blocks of ``shape`` in one tensor [U, N, d]."""
    s = PrototypeStream(U, shape.grid_h, shape.grid_w, shape.d, kinds=kinds, seed=seed,
                        n_proto=n_proto, device=device, dtype=dtype)
    return s.next(shape.frames)


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bits (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
