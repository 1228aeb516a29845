"""The JSON line of bench.py's reference arm (the fp64 oracle on the host cores) keeps the keys
the benchmark contract fixes, on a small workload (CPU only)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
            "cpu_baseline", "e2e"}


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["impl"] == "reference" and d["higher_is_better"] is False
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["unit"] == d["e2e"]["unit"] and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "workload" in d["config"] and d["config"]["workload"].startswith("tiny")


def test_spread_reports_median_and_deciles():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.spread([5.0, 1.0, 3.0, 2.0, 4.0])
    assert d == {"p10": 1.4, "p50": 3.0, "p90": 4.6}
    assert bench.spread([]) == {"p10": None, "p50": None, "p90": None}


def test_head_density_and_attention_flops():
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from long_context_prefill_rr_b200 import workloads as wl
    idx, cnt = wl.random_kept_lists(1, 2, 4, 0.0, seed=0)       # diagonal only
    d = bench.head_density(cnt)
    assert d == {"min": 0.4, "median": 0.4, "max": 0.4}          # 4 of 10 causal blocks
    useful, executed, n = bench.attention_flops(idx, cnt, 128, 64)
    assert n == 8 and executed == 4.0 * 64 * 128 * 128 * 8
    assert useful == 4.0 * 64 * (128 * 129 / 2) * 8              # every kept block is diagonal
    idx, cnt = wl.random_kept_lists(1, 1, 4, 1.0, seed=0)       # dense causal
    assert bench.head_density(cnt)["max"] == 1.0
    useful, _, n = bench.attention_flops(idx, cnt, 128, 64)
    assert n == 10 and useful == 4.0 * 64 * (128 * 128 * 6 + 128 * 129 / 2 * 4)


def test_workload_overrides_reach_the_config():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--stride", "16", "--tau", "0.95", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["stride"] == 16 and d["config"]["tau"] == 0.95
    assert "S16" in d["config"]["workload"] and "tau0.95" in d["config"]["workload"]


def test_l2_flush_applies_where_inputs_fit_twice_the_l2(monkeypatch):
    """Layers whose Q, K and V fit within twice the L2 are flushed before each timed step, and
    the config says which case applies with the real input size."""
    sys.path.insert(0, ROOT)
    import bench
    from long_context_prefill_rr_b200 import workloads as wl
    monkeypatch.setattr(bench, "_l2_bytes", lambda: 126 << 20)
    w8, w32, w128 = (wl.WORKLOADS[n] for n in ("llama8k", "llama32k", "llama128k"))
    assert bench._input_bytes(w128) == 2 * 131072 * 128 * (32 + 16)
    assert bench._needs_flush(w8) and not bench._needs_flush(w32)
    assert not bench._needs_flush(w128) and not bench._needs_flush(wl.WORKLOADS["video64k"])
    assert "flushed" in bench._workload_desc(w8)["l2"] and "0.10 GB" in bench._l2_note(w8)
    assert "no flush" in bench._workload_desc(w128)["l2"] and "1.61 GB" in bench._l2_note(w128)
