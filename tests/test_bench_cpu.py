"""bench.py on the CPU: the reference arm's JSON line and the host helpers.

The reference arm times the fp64 oracle on the host cores; on the tiny
workload it finishes in seconds.  Nothing here touches a GPU.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS, make_qkv  # noqa: E402


def _reference_line(*extra):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "3", *extra], capture_output=True, text=True, env=env,
                         timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("extra", [(), ("--kv-heads", "2"), ("--seed", "9")])
def test_reference_arm_line(extra):
    d = _reference_line(*extra)
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert cb["split"]["select_ms_per_head"] > 0 and cb["split"]["attention_us_per_row"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["H_kv"] == (2 if "--kv-heads" in extra else 4)
    assert d["config"]["workload"].startswith("tiny: B1 H4")


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600,
                         check=True)
    assert out.stdout.strip() == ""


def test_bad_kv_heads_rejected():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "3", "--kv-heads", "3"], capture_output=True, text=True, env=env,
                         timeout=600)
    assert out.returncode != 0 and "kv-heads" in out.stderr


def test_grouped_kv_takes_each_groups_first_head():
    w = WORKLOADS["tiny"]
    _, K, V = make_qkv(w)
    Kg, Vg = bench.grouped_kv(K, V, 2)
    assert Kg.shape == (1, 2, w.N, w.d) and Kg.flags.c_contiguous
    np.testing.assert_array_equal(Kg[:, 1], K[:, 2])
    np.testing.assert_array_equal(Vg[:, 0], V[:, 0])


def test_describe_names_grouped_heads():
    w = WORKLOADS["joint"]
    assert "(K/V heads 6)" in bench.describe(w, 0.3, 6)
    assert "K/V heads" not in bench.describe(w, 0.3, 24)
    assert "K/V heads" not in bench.describe(w, 0.3)


def test_traffic_is_null_when_the_kernel_source_differs(tmp_path):
    src = tmp_path / "attention.cu"
    src.write_text("// not the profiled kernel\n")
    assert bench.traffic_from_profile(str(src)) is None


def test_time_stats():
    assert bench.time_stats([3.0]) == {"mean": 3.0, "median": 3.0, "p90": 3.0}
    xs = [float(i) for i in range(1, 11)]             # 1 .. 10: nearest-rank p90 is the 9th value
    assert bench.time_stats(xs[::-1]) == {"mean": 5.5, "median": 5.5, "p90": 9.0}
    assert bench.time_stats(list(range(1, 21)))["p90"] == 18.0
    assert bench.time_stats([1, 2, 3])["p90"] == 3.0
    with pytest.raises(ValueError):
        bench.time_stats([])


def test_crossover_interpolates_in_log_n():
    # speedups 0.5 at 4096 and 2.0 at 16384: 1.0 lies a third of the way in log N, at 4096 * 4^(1/3)
    n, kind = bench.crossover([(4096, 2.0, 1.0), (16384, 1.0, 2.0)])
    assert kind == "interpolated" and abs(n - 4096 * 4 ** (1 / 3)) < 1e-6
    # the last loss counts: a win below a later loss is ignored
    n, kind = bench.crossover([(2048, 1.0, 1.5), (4096, 1.0, 0.9), (8192, 1.0, 1.1)])
    assert kind == "interpolated" and 4096 < n < 8192
    assert bench.crossover([(2048, 1.0, 1.2), (4096, 1.0, 3.0)]) == (2048.0, "at or below")
    assert bench.crossover([(2048, 2.0, 1.0), (4096, 2.0, 1.5)]) == (None, "above")
    assert bench.crossover([(8192, 1.0, 1.0)]) == (8192.0, "at or below")  # equal times count as a win


def test_paired_tiles_matches_brute_force():
    """bench.paired_tiles restates the planner's pairing (strides 1, 2, 4; smallest summed union, the smaller
    stride on ties; two 64 x 64 tiles per union entry): checked against sets on random lists."""
    import numpy as np
    import bench
    rng = np.random.default_rng(0)
    for trial in range(20):
        B, H = 2, 3
        nB = int(rng.integers(1, 40))
        cnt = rng.integers(0, nB + 1, size=(B, H, nB)).astype(np.int32)
        idx = np.full((B, H, nB, nB), -1, np.int32)
        for b in range(B):
            for h in range(H):
                for i in range(nB):
                    idx[b, h, i, :cnt[b, h, i]] = np.sort(rng.choice(nB, cnt[b, h, i], replace=False))
        mask = rng.integers(0, 2, H).astype(bool) if trial % 2 else None
        want = 0
        for b in range(B):
            for h in range(H):
                if mask is not None and not mask[h]:
                    continue
                sets = [set(idx[b, h, i, :cnt[b, h, i]].tolist()) for i in range(nB)]
                per_stride = []
                for s in (1, 2, 4):
                    per_stride.append(sum(len(sets[a] | (sets[a + s] if a + s < nB else set()))
                                          for a in range(nB) if (a // s) % 2 == 0))
                want += 2 * min(per_stride)
        assert bench.paired_tiles(idx, cnt, mask, H, nB) == want
