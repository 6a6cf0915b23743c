"""Host logic of the streaming bench line: the chunk schedule of a long
generation (700 frames in chunks of 3, the last chunk of 1 frame) and the
algorithmic bytes of one fused dequant of the growing cache."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_chunk_schedule():
    wl = bench.WORKLOADS["stream"]
    sizes = bench.stream_chunks(wl)
    assert len(sizes) == 234
    assert sizes[:-1] == [4680] * 233 and sizes[-1] == 1560
    assert sum(sizes) == 1_092_000


def test_chunk_schedule_exact_multiple():
    wl = dict(bench.WORKLOADS["stream"], frames=9)
    assert bench.stream_chunks(wl) == [4680] * 3


def test_dequant_bytes():
    # one block, one chunk, K=1, T=1, G=64: per token 32 code bytes + 2 scale/zero
    # bytes + 1 assignment byte read, 256 bytes written; one 256-byte table
    assert bench.dequant_alg_bytes(1, 1, 1, 1, 1, 64) == 32 + 4 + 1 + 256 + 256
    # tables scale with the chunk count, the rest with the tokens
    b1 = bench.dequant_alg_bytes(64, 4680, 1, 256, 2, 64)
    b2 = bench.dequant_alg_bytes(64, 4680, 2, 256, 2, 64)
    assert b2 - b1 == 2 * 64 * 256 * 128 * 2
