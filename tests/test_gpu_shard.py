"""Head sharding of one cache (each rank a contiguous share of every layer's
heads, K and V together): every share compressed on its own -- here the
ranks' shares one after another on one GPU -- and reassembled is bit-identical
to compressing the whole cache at once, and so is its reconstruction."""
import numpy as np
import pytest
import torch

from gpu_util import np_bits, packed_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_kv_cache_qvg_b200 import build
    build.build()
    from bit_kv_cache_qvg_b200 import qvg
    return qvg


@pytest.mark.parametrize("world,mode", [(2, 0), (3, 0), (4, 1)])
def test_head_shards_reassemble_to_the_one_rank_cache(q, world, mode):
    from bit_kv_cache_qvg_b200 import synth
    from bit_kv_cache_qvg_b200.shard import share_blocks
    L, H = 2, 6
    shape = synth.KVShape(1, 30, 52)
    X = torch.cat([synth.block_batch(2 * H, shape, seed=synth.unit_seed(5, l, 0, 0), kinds=[0] * H + [1] * H)
                   for l in range(L)]).cuda()
    cfg = q.config(K=128, T=2, group_size=64, iters=3, scale_mode=mode)
    whole = q.quantize(X, cfg)
    Y_whole = np_bits(q.dequantize(whole))
    ref = packed_np(whole)
    got = {k: np.zeros_like(v) for k, v in ref.items()}
    Y = np.zeros_like(Y_whole)
    for r in range(world):
        idx = share_blocks(L, H, world, r)
        part = q.quantize(X[idx].contiguous(), cfg)
        Yp = np_bits(q.dequantize(part))
        pp = packed_np(part)
        for k in ("codes", "scale", "zero"):
            if ref[k].size:
                got[k][idx] = pp[k]
        for k in ("assign", "centroids"):
            got[k][:, idx] = pp[k]
        Y[idx] = Yp
    torch.cuda.synchronize()
    for k in ref:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    np.testing.assert_array_equal(Y, Y_whole)
