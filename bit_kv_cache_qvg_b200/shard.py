"""Head sharding of one compressed KV cache across GPUs.

The codec's blocks -- one (layer, head, K or V) unit each -- are independent:
k-means runs per block (m.163.com article on Quant VideoGen, section 五), so a
cache splits across ranks by heads with no exchange on the data path.  Each
rank takes a contiguous share of every layer's heads, K and V together, holds
its blocks in its own HBM, and compresses and reconstructs them alone.

Block order of a whole cache (and of a rank's share): layer-major, then the K
heads, then the V heads of that layer.  Host logic only; the codec's work
runs in the library's kernels.
"""
from __future__ import annotations


def shard_units(n: int, world: int, rank: int):
    """Contiguous share [first, last) of n units (heads) for `rank` of
    `world`; the shares partition [0, n) and differ in size by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    base, extra = divmod(n, world)
    first = rank * base + min(rank, extra)
    return first, first + base + (1 if rank < extra else 0)


def share_blocks(layers: int, heads: int, world: int, rank: int):
    """Indices, in the whole cache's block order, of the blocks that `rank`
    holds: for every layer its K heads h0..h1-1, then its V heads h0..h1-1.
    The rank's own blocks are laid out in this order."""
    h0, h1 = shard_units(heads, world, rank)
    out = []
    for l in range(layers):
        base = l * 2 * heads
        out += [base + h for h in range(h0, h1)]
        out += [base + heads + h for h in range(h0, h1)]
    return out
