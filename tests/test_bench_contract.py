"""The reference arm's JSON line (bench.py --impl reference), built on CPU
with a small sample: every key of the contract, the oracle as the timed
baseline, and an end-to-end block with no host-device copies."""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


class _Args:
    steps, warmup, workload, reference_seconds = 2, 1, "decode70b", 0.5


def test_reference_line_keys():
    line = bench.run_reference(_Args(), 1, 0)
    assert line is not None
    json.dumps(line)  # serialisable as one JSON line
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert "workload" in line["config"] and "model" not in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == len(os.sched_getaffinity(0)) and cb["sample"]
    assert cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_line_only_on_rank_0():
    assert bench.run_reference(_Args(), 2, 1) is None


def test_weight_copies_exceed_l2():
    """Back-to-back timings cycle over enough distinct weight copies that
    their bytes exceed three L2s, within the caps (64 copies, ~6 GB)."""
    for nbytes in (15_000, 9_437_184, 47_185_920, 132_120_576, 358_000_000, 2_000_000_000):
        n = bench.copies_for(nbytes)
        assert 1 <= n <= 64 and n * nbytes <= (6 << 30) + nbytes
        if n < 64 and n * nbytes < (6 << 30) - nbytes:
            assert n * nbytes >= 3 * bench.L2_BYTES or n == 2 and nbytes > 3 * bench.L2_BYTES / 2
    assert bench.copies_for(132_120_576) == 3 and bench.copies_for(15_000) == 64


def test_crossover_from_points():
    """The crossover is the first measured M whose fused time exceeds the
    split path's HBM-peak estimate, else a line through the last two points."""
    from bit_weight_dequant_b200 import inputs
    peak = 6448.1
    c = lambda M: inputs.Case(M, 5120, 5120)
    split = {M: bench.split_time_est_us(c(M), peak) for M in (1, 8, 16)}
    got = bench.crossover_from_points([(c(1), 5.0), (c(8), split[8] + 1.0), (c(16), 99.0)], peak)
    assert got[0]["M"] == 8 and got[0]["how"] == "measured point"
    got = bench.crossover_from_points([(c(1), 5.0), (c(16), 5.0)], peak)
    assert got[0]["M"] is None  # fused time flat: no crossover
    assert bench.crossover_from_points([(c(1), 5.0)], peak) == []  # one M only
