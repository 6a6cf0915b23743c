"""Host logic of the bench's extra workloads: the streaming line's chunk
schedule (700 frames in chunks of 3, the last chunk of 1 frame) and the
algorithmic bytes of one fused dequant of the growing cache; the design
sweep's closed-form compression ratio; and the oracle reference arm of both
lines (run on the host cores)."""
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import pytest  # noqa: E402


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


def test_sweep_closed_form_matches_library_packed_size():
    """The sweep's closed-form compression ratio is the library's packed size
    (codes, E4M3 scale and zero, uint8 assignments, bf16 centroid tables)."""
    from bit_kv_cache_qvg_b200 import qvg
    for T, G, K, N in [(0, 16, 1, 38000), (1, 64, 256, 38000), (2, 64, 256, 38000), (4, 16, 64, 4680),
                       (3, 32, 256, 1000)]:
        cfg = qvg.config(K=K, T=T, group_size=G)
        packed = qvg.packed_bytes(cfg, N, 1)
        ratio = N * 128 * 2 / packed
        assert abs(ratio - bench.compression_ratio(K, T, G, N)) < 1e-9 * ratio
        packed1 = qvg.packed_bytes(qvg.config(K=K, T=T, group_size=G, scale_mode=1), N, 1)
        ratio1 = N * 128 * 2 / packed1
        assert abs(ratio1 - bench.compression_ratio(K, T, G, N, scale_bytes=1)) < 1e-9 * ratio1


def test_named_points_land_in_the_pages_ranges():
    """The sweep labels the QVG and QVG-Pro settings and plain rounding at
    G = 16 (one scale per group) with the pages' compression figures."""
    from bit_kv_cache_qvg_b200 import qvg
    for name in ("qvg", "qvg-pro"):
        P = qvg.PRESETS[name]
        r = bench.compression_ratio(P["K"], P["T"], P["group_size"], 38000, scale_bytes=1)
        lo, hi = bench.PAGE_RATIOS[name]
        assert lo <= r <= hi
    assert bench.compression_ratio(1, 0, 16, 38000, scale_bytes=1) == bench.PAGE_RATIOS["rtn"][0]


def test_sweep_grid_covers_the_design_space():
    wl = bench.WORKLOADS["sweep"]
    assert wl["frames"] * wl["gh"] * wl["gw"] == 38000 and wl["heads"] == 32
    # the headline operating point: 2 bits + 0.25 (two E4M3 bytes per 64) +
    # 0.125 (two uint8 assignments per 128 channels) + 0.2156 (two bf16 tables)
    assert abs(bench.bits_per_element(256, 2, 64, 38000) - (2 + 0.25 + 0.125 + 16 * 2 * 256 / 38000)) < 1e-12


def test_adaptive_stream_scenes_cycle_through_the_gains():
    """Scenes of 26 chunks scaled by 1, 8 and 1/4 in turn (powers of two, so
    the bf16 inputs are scaled exactly); the ladder is the two named points."""
    wl = bench.WORKLOADS["adaptive"]
    gains = [bench.scene_gain(wl, c) for c in range(len(bench.stream_chunks(wl)))]
    assert gains[:26] == [1.0] * 26 and gains[26:52] == [8.0] * 26 and gains[52:78] == [0.25] * 26
    assert gains[78] == 1.0 and len(gains) == 234
    assert all(math.frexp(g)[0] == 0.5 for g in set(gains))
    assert tuple(wl["ladder"]) == ("qvg", "qvg-pro")


@pytest.mark.parametrize("workload", ["stream", "sweep", "adaptive"])
def test_reference_arm_prints_one_line(workload):
    """--impl reference runs the oracle on the host cores and prints the
    workload's own metric with the reference keys (no GPU involved)."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          workload, "--steps", "1", "--warmup", "0", "--ref-tokens", "1600"],
                         capture_output=True, text=True, timeout=600, check=True).stdout.strip().splitlines()
    line = json.loads(out[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["metric"] == {"stream": bench.STREAM_METRIC, "sweep": bench.SWEEP_METRIC,
                              "adaptive": bench.ADAPTIVE_METRIC}[workload]
    for key in ("unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "cpu_baseline", "e2e"):
        assert key in line
    assert line["cpu_baseline"]["kind"] == "oracle"
