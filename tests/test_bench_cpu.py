"""bench.py's host side on CPU: the reference arm (the oracle timed on host
cores) prints one JSON line with the contract's keys, other ranks stay
silent, warm-up below 3 is refused, and the FLOP count behind the metric
counts visible pairs as the mask definition does (brute force on small N)."""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    res = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["steps"] == 2 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    res = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    res = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2"])
    assert res.returncode != 0 and "warmup" in res.stderr


def _brute_pairs(N, mask, window):
    count = 0
    for i in range(N):
        for j in range(N):
            if mask == "full":
                count += 1
            elif mask == "causal":
                count += j <= i
            else:
                count += i - window < j <= i
    return count


@pytest.mark.parametrize("N", [1, 2, 7, 64, 129])
@pytest.mark.parametrize("mask,window", [("full", None), ("causal", None), ("sliding_window", 1),
                                         ("sliding_window", 5), ("sliding_window", 64), ("sliding_window", 200)])
def test_visible_pairs_counts_the_mask(N, mask, window):
    assert bench.visible_pairs(N, mask, window) == _brute_pairs(N, mask, window)


def test_workload_flops_are_four_d_per_visible_pair():
    from harness.inputs import WORKLOADS
    w = WORKLOADS["swa"]
    assert bench.workload_flops(w, w.B) == 4 * w.B * w.Hq * w.d * bench.visible_pairs(w.N, w.mask, w.window)
    # the long workload: N = 131072, d = 128, 32 heads, causal
    w = WORKLOADS["long"]
    assert bench.workload_flops(w, 1) == 4 * 32 * 128 * (131072 * 131073 // 2)


def _brute_decode_keys(L, Nq, mask, window):
    """Positions j < L that at least one of the step's queries (positions L-Nq .. L-1) sees."""
    seen = set()
    for i in range(L - Nq, L):
        for j in range(L):
            if mask == "full" or (mask == "causal" and j <= i) or \
                    (mask == "sliding_window" and i - window < j <= i):
                seen.add(j)
    return len(seen)


@pytest.mark.parametrize("mask,window,Nq", [("causal", None, 1), ("causal", None, 4), ("full", None, 2),
                                            ("sliding_window", 1, 1), ("sliding_window", 7, 3),
                                            ("sliding_window", 50, 4), ("sliding_window", 500, 2)])
def test_decode_bytes_count_the_visible_cached_positions(mask, window, Nq):
    from dataclasses import replace
    from harness.inputs import DECODE_WORKLOADS
    lens = [Nq, Nq + 1, 37, 64, 129, 300]
    w = replace(DECODE_WORKLOADS["decode_gqa"], B=len(lens), Nq=Nq, mask=mask, window=window)
    keys = sum(_brute_decode_keys(L, Nq, mask, window) for L in lens)
    expect = 2 * 2 * w.d * w.Hkv * keys + w.B * w.Hq * Nq * (2 * 2 * w.d + 4)
    assert bench.decode_bytes(w, lens) == expect
