"""Benchmark of the RRAttention prefill hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama128k] [--impl reference]

One step = one attention layer's prefill: pooled-key estimate, Top-tau select and block-sparse
attention (rra_estimate, rra_select, rra_sparse_attn through the C ABI) on the seeded
Llama-3.1-8B-like layer at 128K tokens (b1, 32 Q / 8 KV heads, d 128, B 128, S 8, tau 0.9).
Inputs (2.7 GB) are larger than L2, so no flush is needed between steps. With N > 1 (torchrun)
every rank runs an independent replica of the layer (default), or with --shard heads its share
of the KV-head groups of one layer (no exchange between ranks); the time is the max over ranks.

Prints one JSON line (rank 0). `value` is milliseconds per layer for the whole job
(max-over-ranks step time / layers processed per step). The reference arm times the fp64 CPU
oracle on a bounded sample of block rows of the same workload and extrapolates to a layer.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from long_context_prefill_rr_b200 import sharding  # noqa: E402
from long_context_prefill_rr_b200 import workloads as wl  # noqa: E402

METRIC = "prefill attn ms/layer @128K (estimate+select+sparse) & TFLOP/s vs roofline"
UNIT = "ms/layer"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1590.0,
            "source": "fallback"}


def _workload_desc(w: wl.Workload, parallelism: str = "replicas") -> dict:
    return {"workload": f"{w.name}: b{w.batch} Hq{w.heads_q} Hkv{w.heads_kv} d{w.head_dim} "
                        f"L{w.seqlen} B{w.block} S{w.stride} tau{w.tau}",
            "model": "Llama-3.1-8B-like attention layer (random synthetic Q/K/V)"
            if w.kind == "llama" else w.kind,
            "global_batch": w.batch, "seq_len": w.seqlen, "heads_q": w.heads_q,
            "heads_kv": w.heads_kv, "head_dim": w.head_dim, "block": w.block, "stride": w.stride,
            "tau": w.tau, "parallelism": parallelism, "l2": "inputs (2.7 GB) larger than L2"
            if w.seqlen >= 32768 else "L2 flushed between steps"}


def attention_flops(kept_idx: np.ndarray, kept_cnt: np.ndarray, block: int, d: int):
    """(useful, executed) flops of the block-sparse attention: 2 GEMMs x 2 flops per MAC;
    useful counts only the causal half (B(B+1)/2 pairs) of diagonal blocks."""
    b, h, nb = kept_cnt.shape
    n_kept = int(kept_cnt.sum(dtype=np.int64))
    n_diag = 0
    for I in range(nb):
        off = I * (I + 1) // 2
        cnt = kept_cnt[:, :, I]
        last = kept_idx[:, :, off:off + I + 1]
        # the diagonal, if kept, is the last entry of the ascending row
        pos = np.clip(cnt - 1, 0, None)
        lastv = np.take_along_axis(last, pos[..., None], axis=2)[..., 0]
        n_diag += int(((cnt > 0) & (lastv == I)).sum())
    useful = 4.0 * d * (block * block * (n_kept - n_diag) + block * (block + 1) / 2 * n_diag)
    executed = 4.0 * d * block * block * n_kept
    return useful, executed, n_kept


def head_density(kept_cnt: np.ndarray) -> dict:
    """Kept-block density per (batch row, head) of kept_cnt [b, H, NB]: min, median, max."""
    b, h, nb = kept_cnt.shape
    per = kept_cnt.sum(axis=2, dtype=np.int64) / (nb * (nb + 1) / 2)
    return {"min": float(per.min()), "median": float(np.median(per)), "max": float(per.max())}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 20 ms while active."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # raw samples go to a scratch file; the JSON line carries their summary
        self.path = os.path.join(tempfile.gettempdir(), f"rra_clocks_gpu{index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def cpu_oracle_sample(w: wl.Workload, q_bits, k_bits, v_bits, n_rows: int, seed: int = 0,
                      total_kept: int | None = None) -> dict:
    """Time the fp64 oracle (estimate -> select -> attention, each on the oracle's own outputs)
    on a seeded sample of block rows and extrapolate to one layer.

    Estimate and select cost scale with the row length (I + 1 blocks), attention with the
    row's kept blocks; each phase's per-unit time from the sample is multiplied by the layer's
    total units (total kept blocks: ``total_kept`` when known, else the sample's kept fraction
    times every causal block).
    """
    import oracle as orc
    scale = w.softmax_scale if w.softmax_scale > 0 else 1.0 / np.sqrt(w.head_dim)
    nb = w.seqlen // w.block
    rng = np.random.default_rng(seed)
    rows = [(0, int(rng.integers(w.heads_q)), int(rng.integers(nb))) for _ in range(n_rows)]
    t_est = t_att = 0.0
    u_est = u_att = 0
    kbars = {}
    t0 = time.perf_counter()
    for b, h, I in rows:
        kv = orc.kv_head(h, w.heads_q, w.heads_kv)
        q = wl.bf16_bits_to_f64(q_bits[b, h])
        k = wl.bf16_bits_to_f64(k_bits[b, kv])
        v = wl.bf16_bits_to_f64(v_bits[b, kv])
        a = time.perf_counter()
        if (b, kv) not in kbars:
            kbars[(b, kv)] = orc.pooled_keys(k, w.stride)
        mass = orc.estimate_block_row(q, kbars[(b, kv)], h, I, w.block, w.stride, w.shift, scale)
        kept = orc.select_row(mass, I, w.tau)
        c = time.perf_counter()
        orc.attention_block(q, k, v, I, kept, w.block, scale)
        e = time.perf_counter()
        t_est += c - a
        t_att += e - c
        u_est += I + 1
        u_att += len(kept)
    wall = time.perf_counter() - t0
    total_causal = w.batch * w.heads_q * nb * (nb + 1) // 2
    if total_kept is None:
        total_kept = u_att / u_est * total_causal
        how = "the sample's kept fraction"
    else:
        how = "the GPU run's kept-block count"
    ms = 1e3 * (t_est / u_est * total_causal + t_att / max(u_att, 1) * total_kept)
    return {"value": ms, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{n_rows} seeded (head, block-row) pairs of {w.name}, fp64 numpy "
                      f"({wall:.1f} s), extrapolated to the layer by row length (estimate + "
                      f"select) and kept blocks (attention; total from {how})",
            "sample_seconds": wall}


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the process group (identity when there is
    none); every rank takes this collective at the same point."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def spread(values) -> dict:
    """Median and 10th / 90th percentiles (linear interpolation) of per-step timings."""
    v = np.asarray(list(values), dtype=np.float64)
    if v.size == 0:
        return {"p10": None, "p50": None, "p90": None}
    p10, p50, p90 = np.percentile(v, [10, 50, 90])
    return {"p10": float(p10), "p50": float(p50), "p90": float(p90)}


def sum_over_ranks(values, device=None):
    """Element-wise sum over the process group (identity when there is none)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()]


def run_reference(args, w):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    q_bits, k_bits, v_bits = wl.make_workload(w)
    step_ms = []
    cb = None
    for s in range(args.warmup + args.steps):
        cb = cpu_oracle_sample(w, q_bits, k_bits, v_bits, n_rows=args.ref_rows, seed=s)
        if s >= args.warmup:
            step_ms.append(cb["value"])
    value = float(np.mean(step_ms))
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": value, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": _workload_desc(w), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from long_context_prefill_rr_b200 import native

    ws_n, rank, local = _dist_env()
    if ws_n > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    native.load()
    p = native.params(w.batch, w.heads_q, w.heads_kv, w.seqlen, w.head_dim, w.stride, w.tau,
                      shift=w.shift, softmax_scale=w.softmax_scale, block=w.block)
    q_bits, k_bits, v_bits = wl.make_workload(w)
    sharded = args.shard == "heads"
    if sharded:
        # this rank's KV-head groups; no data moves between ranks on the path
        p, shard = sharding.shard_params(p, rank, ws_n)
        q_bits = sharding.take_heads(q_bits, shard.q0, shard.q1)
        k_bits = sharding.take_heads(k_bits, shard.kv0, shard.kv1)
        v_bits = sharding.take_heads(v_bits, shard.kv0, shard.kv1)
    sh = native.shapes(p)

    def host_pinned(bits):
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv = host_pinned(q_bits), host_pinned(k_bits), host_pinned(v_bits)
    q = hq.to(dev)
    k = hk.to(dev)
    v = hv.to(dev)
    out = torch.empty(sh["q"], dtype=torch.bfloat16, device=dev)
    mass = torch.empty(sh["mass"], dtype=torch.float32, device=dev)
    idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device=dev)
    cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device=dev)
    wsp = native.new_workspace(p, dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        native.estimate(p, q, k, mass, wsp)
        if ev is not None:
            ev[1].record(stream)
        native.select(p, mass, idx, cnt)
        if ev is not None:
            ev[2].record(stream)
        native.sparse_attn(p, q, k, v, idx, cnt, out, wsp)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, raw = native.check_device_status(wsp)
    if st != 0:
        raise RuntimeError(f"device status {raw:#x} after warm-up")
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws_n > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for s in range(args.steps):
            step(events[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if ws_n > 1:
        dist.barrier()
    total_ms = start.elapsed_time(stop)
    est_ms = [e[0].elapsed_time(e[1]) for e in events]
    sel_ms = [e[1].elapsed_time(e[2]) for e in events]
    att_ms = [e[2].elapsed_time(e[3]) for e in events]
    st, raw = native.check_device_status(wsp)
    if st != 0:
        raise RuntimeError(f"device status {raw:#x} after the timed steps")

    # ---- end to end through the C-ABI host-buffer call (rra_prefill_host): pinned host
    # inputs in, host output back, the copies overlapped with the compute chunk by chunk
    hout = torch.empty(sh["q"], dtype=torch.bfloat16).pin_memory()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, min(args.steps, 5))
    native.prefill_host(p, hq, hk, hv, hout, q, k, v, out, idx, cnt, wsp)   # warm-up
    torch.cuda.synchronize(dev)
    e_start.record(stream)
    for _ in range(e_steps):
        native.prefill_host(p, hq, hk, hv, hout, q, k, v, out, idx, cnt, wsp)
    e_stop.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_stop) / e_steps

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    cnt_host = cnt.cpu().numpy()
    useful, executed, n_kept = attention_flops(idx.cpu().numpy(), cnt_host, w.block, w.head_dim)
    h2d_bytes = int(hq.numel() + hk.numel() + hv.numel()) * 2
    d2h_bytes = int(hout.numel()) * 2
    # whole-job figures: kept blocks over every rank's heads, bytes every rank moved
    n_kept_all, h2d_all, d2h_all = sum_over_ranks([n_kept, h2d_bytes, d2h_bytes], dev)

    if rank == 0:
        peaks = _peaks()
        nb = w.seqlen // w.block
        heads_all = w.heads_q * (1 if sharded else ws_n)
        density = n_kept_all / (w.batch * heads_all * nb * (nb + 1) / 2)
        att_avg = float(np.mean(att_ms))
        est_avg = float(np.mean(est_ms))
        sel_avg = float(np.mean(sel_ms))
        achieved = useful / (att_avg * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        ns = w.seqlen // w.stride
        # per-rank algorithmic bytes (this rank's heads)
        est_bytes = (p.batch * p.heads_kv * w.seqlen * w.head_dim * 2          # K read once
                     + p.batch * p.heads_q * ns * w.head_dim * 2               # sampled Q rows
                     + p.batch * p.heads_q * nb * (nb + 1) // 2 * 4)           # masses out
        sel_bytes = (p.batch * p.heads_q * nb * (nb + 1) // 2 * 4 + n_kept * 4 +
                     p.batch * p.heads_q * nb * 4)
        ms_per_step = total_ms / args.steps
        # ms per layer of the whole job: replicas finish ws_n layers per step, head shards one
        value = ms_per_step if sharded else ms_per_step / ws_n
        cpu = None
        if ws_n == 1 and not args.no_cpu_baseline:
            cpu = cpu_oracle_sample(w, q_bits, k_bits, v_bits, n_rows=args.ref_rows,
                                    total_kept=n_kept)
        traffic = None
        tpath = os.path.join(ROOT, "profiles", "bs_attn_fwd_llama128k_traffic.json")
        if os.path.exists(tpath):
            td = json.load(open(tpath))
            if td.get("workload") == w.name and td.get("kernel_rev") == KERNEL_REV:
                traffic = td.get("bytes_per_launch")
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": False, "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, shaped like the pages' Llama-3.1-8B 128K workload)",
            "config": _workload_desc(w, f"heads{ws_n}" if sharded else "replicas"),
            "phases_ms": {"estimate": est_avg, "select": sel_avg, "sparse_attn": att_avg},
            "phases_ms_spread": {"estimate": spread(est_ms), "select": spread(sel_ms),
                                 "sparse_attn": spread(att_ms),
                                 "step": spread([a + b + c for a, b, c in
                                                 zip(est_ms, sel_ms, att_ms)])},
            "density": density,
            "density_per_head": head_density(cnt_host),
            "attn_tflops": achieved, "attn_tflops_executed": executed / (att_avg * 1e-3) / 1e12,
            "estimate_gbs": est_bytes / (est_avg * 1e-3) / 1e9,
            "estimate_frac_hbm": est_bytes / (est_avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "select_gbs": sel_bytes / (sel_avg * 1e-3) / 1e9,
            "estimate_select_frac_hbm": (est_bytes + sel_bytes) / ((est_avg + sel_avg) * 1e-3)
            / 1e9 / peaks["hbm_gbs"],
            "roofline": {"bound": "tensor", "kernel": "bs_attn_fwd_kernel", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peaks['source']} bf16 sustained",
                         "traffic": traffic,
                         "per_launch_flops": useful},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_ms if sharded else e2e_ms / ws_n, "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d_all), "d2h_bytes_per_step": int(d2h_all)},
            "gpu_launches": 4 * args.steps,
            "e2e_api": "rra_prefill_host (pinned host buffers; copies overlapped with the "
                       "compute, chunk by chunk)",
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_speedup_study(args):
    """Dense-vs-sparse study: per length, the full RR path (estimate + select + sparse
    attention), the same attention kernel on every causal block (tau = 1: dense causal), and
    torch's fused scaled_dot_product_attention (causal, GQA) on the same bf16 inputs, as a
    library reference point. Prints one JSON line per length."""
    import torch

    from long_context_prefill_rr_b200 import native

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    native.load()
    out_lines = []
    for L in [int(x) for x in args.lengths.split(",")]:
        w = wl.WORKLOADS["llama128k"].with_(seqlen=L, name=f"llama{L // 1024}k")
        q_bits, k_bits, v_bits = wl.make_workload(w)
        to = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
        q, k, v = to(q_bits), to(k_bits), to(v_bits)
        res = {"seq_len": L}
        for tau, name in ((w.tau, "rr"), (1.0, "dense_tau1")):
            p = native.params(w.batch, w.heads_q, w.heads_kv, L, w.head_dim, w.stride, tau,
                              shift=w.shift, softmax_scale=w.softmax_scale)
            run = native.RRAttentionPrefill(p, dev)
            out = torch.empty_like(q)
            for _ in range(3):
                run(q, k, v, out)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = max(3, min(20, int(2e9 / L / L * 4096)))
            e0.record()
            for _ in range(n):
                run(q, k, v, out)
            e1.record()
            torch.cuda.synchronize()
            run.check()
            res[f"{name}_ms"] = e0.elapsed_time(e1) / n
            if name == "rr":
                cnt = run.kept_cnt.cpu().numpy()
                nb = L // 128
                res["density"] = float(cnt.sum() / (w.heads_q * nb * (nb + 1) / 2))
            del run, out
        g = w.heads_q // w.heads_kv
        def sdpa():
            return torch.nn.functional.scaled_dot_product_attention(
                q, k, v, is_causal=True, scale=w.softmax_scale, enable_gqa=True)
        try:
            for _ in range(3):
                sdpa()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = max(3, min(20, int(2e9 / L / L * 4096)))
            e0.record()
            for _ in range(n):
                sdpa()
            e1.record()
            torch.cuda.synchronize()
            res["torch_sdpa_causal_ms"] = e0.elapsed_time(e1) / n
        except (RuntimeError, torch.cuda.OutOfMemoryError) as err:   # no fused backend: report
            res["torch_sdpa_causal_ms"] = None
            res["torch_sdpa_error"] = str(err).splitlines()[0][:200]
            torch.cuda.empty_cache()
        res["speedup_rr_vs_dense_tau1"] = res["dense_tau1_ms"] / res["rr_ms"]
        if res["torch_sdpa_causal_ms"]:
            res["speedup_rr_vs_torch_sdpa"] = res["torch_sdpa_causal_ms"] / res["rr_ms"]
        dense_flops = 4.0 * w.head_dim * w.heads_q * (128 * 128 * (L // 128) * (L // 128 - 1) / 2
                                                      + 128 * 129 / 2 * (L // 128))
        res["dense_tau1_tflops"] = dense_flops / (res["dense_tau1_ms"] * 1e-3) / 1e12
        if res["torch_sdpa_causal_ms"]:
            res["torch_sdpa_tflops"] = dense_flops / (res["torch_sdpa_causal_ms"] * 1e-3) / 1e12
        del g
        print(json.dumps({"study": "speedup", "workload": w.name, **res}), flush=True)
        out_lines.append(res)
        del q, k, v
        torch.cuda.empty_cache()
    return 0


def run_search_study(args):
    """Pattern-search time: the round-robin estimate (stride pooling + estimate) against the
    XAttention antidiagonal estimate, both followed by the same select; per length."""
    import torch

    from long_context_prefill_rr_b200 import native

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    native.load()
    for L in [int(x) for x in args.lengths.split(",")]:
        w = wl.WORKLOADS["llama128k"].with_(seqlen=L, name=f"llama{L // 1024}k")
        q_bits, k_bits, _ = wl.make_workload(w)
        to = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
        q, k = to(q_bits), to(k_bits)
        res = {"seq_len": L, "stride": w.stride}
        p = native.params(w.batch, w.heads_q, w.heads_kv, L, w.head_dim, w.stride, w.tau,
                          shift=w.shift, softmax_scale=w.softmax_scale)
        sh = native.shapes(p)
        mass = torch.empty(sh["mass"], dtype=torch.float32, device=dev)
        idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device=dev)
        cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device=dev)
        ws = native.new_workspace(p, dev)
        for name, fn in (("rr", lambda: native.estimate(p, q, k, mass, ws)),
                         ("xattn", lambda: native.estimate_xattn(p, q, k, mass, ws))):
            for _ in range(3):
                fn()
                native.select(p, mass, idx, cnt)
            torch.cuda.synchronize()
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            n = 10
            t_est = t_sel = 0.0
            for _ in range(n):
                e0.record()
                fn()
                e1.record()
                native.select(p, mass, idx, cnt)
                e2.record()
                torch.cuda.synchronize()
                t_est += e0.elapsed_time(e1)
                t_sel += e1.elapsed_time(e2)
            st, raw = native.check_device_status(ws)
            if st != 0:
                raise RuntimeError(f"device status {raw:#x}")
            nb = L // 128
            res[f"{name}_estimate_ms"] = t_est / n
            res[f"{name}_select_ms"] = t_sel / n
            res[f"{name}_density"] = float(cnt.sum().item() / (w.heads_q * nb * (nb + 1) / 2))
        res["xattn_over_rr_search_time"] = ((res["xattn_estimate_ms"] + res["xattn_select_ms"]) /
                                            (res["rr_estimate_ms"] + res["rr_select_ms"]))
        print(json.dumps({"study": "search", "workload": w.name, **res}), flush=True)
        del q, k, mass, idx, cnt, ws
        torch.cuda.empty_cache()
    return 0


# bump when the attention kernel changes, so stale ncu traffic is not reported
KERNEL_REV = "attn-v3"


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama128k", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--study", choices=["speedup", "search"], default=None,
                    help="instead of the bench line: dense-vs-sparse speedup over --lengths")
    ap.add_argument("--lengths", default="8192,16384,32768,65536,131072")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: every rank runs the whole layer (replicas, weak scaling) or "
                         "its share of the KV-head groups (heads, strong scaling)")
    args = ap.parse_args(argv)
    if args.study == "speedup":
        return run_speedup_study(args)
    if args.study == "search":
        return run_search_study(args)
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
