"""Benchmark of the RRAttention prefill hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama128k] [--impl reference]

One step = one attention layer's prefill: pooled-key estimate, Top-tau select and block-sparse
attention (rra_estimate, rra_select, rra_sparse_attn through the C ABI) on the seeded
Llama-3.1-8B-like layer at 128K tokens (b1, 32 Q / 8 KV heads, d 128, B 128, S 8, tau 0.9).
Inputs (1.61 GB at 128K) are larger than L2, so no flush is needed between steps; workloads whose
inputs fit within twice the L2 size get an L2 flush before every timed step. With N > 1 (torchrun)
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
            "tau": w.tau, "parallelism": parallelism, "l2": _l2_note(w)}


def _input_bytes(w: wl.Workload) -> int:
    """Q, K and V of the layer in bytes (bf16)."""
    return 2 * w.batch * w.seqlen * w.head_dim * (w.heads_q + 2 * w.heads_kv)


def _l2_bytes() -> int:
    import torch
    if torch.cuda.is_available():
        return int(torch.cuda.get_device_properties(0).L2_cache_size)
    return 126 << 20


def _needs_flush(w: wl.Workload) -> bool:
    """Inputs under twice the L2 size could be served from L2 across steps: flush between them."""
    return _input_bytes(w) < 2 * _l2_bytes()


def _l2_note(w: wl.Workload) -> str:
    if _needs_flush(w):
        return (f"inputs ({_input_bytes(w) / 1e9:.2f} GB) within 2x L2: L2 flushed between steps "
                f"by writing {2 * _l2_bytes() >> 20} MiB (outside the per-step events)")
    return f"inputs ({_input_bytes(w) / 1e9:.2f} GB) larger than 2x L2: no flush between steps"


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
    """SM clock, power and clock-event (throttle) reasons sampled every 5 ms while active, by
    NVML in a thread of this process (reading only; nothing is set), with nvidia-smi as the
    fallback. The device is matched to the CUDA device by UUID."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               # a clock set by an application or a user (a leftover lock) shows up here
               ("applications_clocks_setting", "nvmlClocksEventReasonApplicationsClocksSetting"),
               ("user_defined_clocks", "nvmlClocksEventReasonUserDefinedClocks"),
               ("sync_boost", "nvmlClocksEventReasonSyncBoost"),
               ("display_clock_setting", "nvmlClocksEventReasonDisplayClockSetting"))
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (sm_mhz, max_mhz, power_w, reasons)
        self.how = None
        self._stop = None
        self._thread = None
        self._proc = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
            uuid if uuid.startswith("GPU-") else "GPU-" + uuid)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS if hasattr(nv, attr)]
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(mx), pw,
                                             [n for n, b in bits if rs & b]))
                    except Exception:
                        pass
                    self._stop.wait(self.period)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            self.how = "nvml, 5 ms"
        except Exception:
            self._start_smi()
        return self

    def _start_smi(self):
        self.path = os.path.join(tempfile.gettempdir(),
                                 f"rra_clocks_{self.cuda_index}_{os.getpid()}.csv")
        try:
            self._f = open(self.path, "w")
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self._f,
                stderr=subprocess.DEVNULL)
            self.how = "nvidia-smi, 20 ms"
        except Exception:
            self._proc = None

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
            self._f.close()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            with open(self.path) as f:
                for line in f:
                    r = [x.strip() for x in line.split(",")]
                    if len(r) >= 9 and r[1].replace(".", "").isdigit():
                        self.samples.append((float(r[1]), float(r[2]) if r[2].replace(
                            ".", "").isdigit() else None, None,
                            [n for n, v in zip(names, r[5:9]) if v == "Active"]))
            try:
                os.remove(self.path)
            except OSError:
                pass

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "samples": 0, "how": self.how}
        sm = [x[0] for x in self.samples]
        mx = [x[1] for x in self.samples if x[1]]
        pw = [x[2] for x in self.samples if x[2] is not None]
        reasons = sorted({r for x in self.samples for r in x[3]})
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
               "sm_mhz_min": min(sm), "reasons": reasons, "samples": len(sm), "how": self.how}
        if pw:
            out["power_w_max"] = max(pw)
        return out


def _est_seconds_per_head(w: wl.Workload) -> float:
    """Rough fp64-oracle cost of one head's estimate + select on one host core (measured:
    about 0.16 s for 4096 sampled queries at d 128; it grows with (L/S)^2 d)."""
    return 0.16 * (w.seqlen / w.stride / 4096.0) ** 2 * (w.head_dim / 128.0)


def cpu_oracle_baseline(w: wl.Workload, q_bits, k_bits, v_bits, est_heads, attn_rows: int,
                        seed: int = 0, total_kept: int | None = None, gpu=None) -> dict:
    """Time the fp64 oracle (oracle/, as it stands) on a bounded sample of one layer and scale
    the time to the layer.

    * estimate + select: every block row of each (batch row, head) in ``est_heads``;
    * attention: ``attn_rows`` seeded (head, block row) pairs on the oracle's own kept lists.

    Scaling: the estimate + select time by (b * Hq) / len(est_heads) (every head costs the
    same), the attention time by the layer's kept blocks over the sample's (the layer's count is
    ``total_kept`` when the GPU run gave it, else the sampled heads' kept fraction times every
    causal block). With ``gpu`` (numpy mass / idx / cnt / out of the GPU run on the same
    inputs) the oracle's results on the sample are also compared with the GPU's.
    """
    import oracle as orc
    scale = w.softmax_scale if w.softmax_scale > 0 else 1.0 / np.sqrt(w.head_dim)
    nb = w.seqlen // w.block
    tau32 = float(np.float32(w.tau))
    t_est = t_sel = t_att = 0.0
    rows_est = 0
    mass_err = 0.0
    list_diff = 0
    kept = {}
    masses = {}
    t0 = time.perf_counter()
    for b, h in est_heads:
        kv = orc.kv_head(h, w.heads_q, w.heads_kv)
        q = wl.bf16_bits_to_f64(q_bits[b, h])      # input conversion, not timed
        k = wl.bf16_bits_to_f64(k_bits[b, kv])
        a = time.perf_counter()
        kbar = orc.pooled_keys(k, w.stride)
        rows = [orc.estimate_block_row(q, kbar, h, I, w.block, w.stride, w.shift, scale)
                for I in range(nb)]
        c = time.perf_counter()
        lists = [orc.select_row(r, I, tau32) for I, r in enumerate(rows)]
        e = time.perf_counter()
        t_est += c - a
        t_sel += e - c
        rows_est += nb
        for I in range(nb):
            kept[(b, h, I)] = lists[I]
            masses[(b, h, I)] = rows[I]
        if gpu is not None:
            for I in range(nb):
                off = orc.tri_offset(I)
                mass_err = max(mass_err, float(np.abs(gpu["mass"][b, h, off:off + I + 1]
                                                      - rows[I]).max()))
                got = gpu["idx"][b, h, off:off + gpu["cnt"][b, h, I]]
                list_diff += int(not np.array_equal(got, lists[I]))
    rng = np.random.default_rng(seed)
    pairs = set()
    while len(pairs) < min(attn_rows, w.batch * w.heads_q * nb):
        pairs.add((int(rng.integers(w.batch)), int(rng.integers(w.heads_q)),
                   int(rng.integers(nb))))
    u_att = 0
    attn_err = 0.0
    attn_checked = 0
    conv = {}

    def f64(bits, key):   # input conversion (cached per head, not timed)
        if key not in conv:
            if len(conv) > 6:
                conv.clear()
            conv[key] = wl.bf16_bits_to_f64(bits[key[1], key[2]])
        return conv[key]

    for b, h, I in sorted(pairs):
        kv = orc.kv_head(h, w.heads_q, w.heads_kv)
        q, k, v = f64(q_bits, ("q", b, h)), f64(k_bits, ("k", b, kv)), f64(v_bits, ("v", b, kv))
        lst = kept.get((b, h, I))
        if lst is None:   # the row's own estimate + select, untimed (timed per head above)
            lst = orc.select_row(orc.estimate_block_row(q, orc.pooled_keys(k, w.stride), h, I,
                                                        w.block, w.stride, w.shift, scale),
                                 I, tau32)
        a = time.perf_counter()
        o = orc.attention_block(q, k, v, I, lst, w.block, scale)
        t_att += time.perf_counter() - a
        u_att += len(lst)
        if gpu is not None:
            off = orc.tri_offset(I)
            if np.array_equal(gpu["idx"][b, h, off:off + gpu["cnt"][b, h, I]], lst):
                g = gpu["out_rows"](b, h, I * w.block, (I + 1) * w.block)
                attn_err = max(attn_err, float(np.abs(g - o).max()))
                attn_checked += 1
    wall = time.perf_counter() - t0
    units = w.batch * w.heads_q
    est_sel_layer = (t_est + t_sel) * units / max(len(est_heads), 1)
    if total_kept is None:
        n_samp = sum(len(x) for x in kept.values())
        total_kept = n_samp / max(rows_est, 1) * nb * units   # kept per row x rows
        how = "the sampled heads' kept blocks"
    else:
        how = "the GPU run's kept-block count"
    att_layer = t_att / max(u_att, 1) * total_kept
    ms = 1e3 * (est_sel_layer + att_layer)
    full = len(est_heads) == units
    out = {"value": ms, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
           "sample": (f"estimate + select of every block row of {len(est_heads)} of {units} "
                      f"heads ({'the whole layer' if full else 'scaled by heads'}; "
                      f"{t_est + t_sel:.1f} s), attention of {len(pairs)} seeded query blocks "
                      f"({t_att:.1f} s, scaled by kept blocks, layer total from {how}); fp64 "
                      f"numpy of {w.name}, {wall:.1f} s in all"),
           "phases_s_measured": {"estimate": t_est, "select": t_sel, "attention": t_att},
           "sample_seconds": wall, "estimate_select_whole_layer": full,
           "attention_extrapolated": True}
    if gpu is not None:
        bd = sum(1 for (b, h, I), a in masses.items() if I > 0 and _boundary_row(a, tau32))
        out["parity_on_sample"] = {
            "mass_rows": rows_est, "mass_max_err": mass_err, "list_rows": rows_est,
            "list_rows_differing": list_diff, "boundary_rows": bd,
            "attn_query_blocks": attn_checked, "attn_max_abs": attn_err,
            "tolerances": "mass 1e-3 abs; lists exact outside 1e-4 of the tau boundary; "
                          "attention max-abs 2e-2"}
    return out


def _boundary_row(a, tau: float, eps: float = 1e-4) -> bool:
    """The oracle row's descending running sum comes within eps of tau * total, or the masses
    on both sides of its cut are within eps (where float rounding may decide the list)."""
    a = np.asarray(a, dtype=np.float64)
    srt = -np.sort(-a, kind="stable")
    cs = np.cumsum(srt)
    target = tau * a.sum()
    if np.min(np.abs(cs - target)) <= eps:
        return True
    hit = np.nonzero(cs >= target)[0]
    k = int(hit[0]) if hit.size else len(a) - 1
    return k + 1 < len(a) and abs(srt[k] - srt[k + 1]) <= eps


def est_heads_for(w: wl.Workload, budget_s: float) -> list:
    """(batch, head) pairs whose estimate + select fit the budget: every head when they all
    do, else an evenly spread subset."""
    units = [(b, h) for b in range(w.batch) for h in range(w.heads_q)]
    n = max(1, min(len(units), int(budget_s / max(_est_seconds_per_head(w), 1e-9))))
    if n >= len(units):
        return units
    pick = np.linspace(0, len(units) - 1, n).round().astype(int)
    return [units[i] for i in sorted(set(pick.tolist()))]


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
    """The oracle on the host cores, one bounded sample of the layer per step: estimate +
    select of every block row of one head (a different head each step) and attention of a few
    seeded query blocks. ms_per_step is the time each step took; value is that sample scaled to
    the layer (mean over the timed steps)."""
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    q_bits, k_bits, v_bits = wl.make_workload(w)
    units = [(b, h) for b in range(w.batch) for h in range(w.heads_q)]
    step_ms, layer_ms = [], []
    cb = None
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_oracle_baseline(w, q_bits, k_bits, v_bits, [units[s % len(units)]],
                                 attn_rows=args.ref_rows or (4 if w.seqlen >= 65536 else 16),
                                 seed=s)
        if s >= args.warmup:
            step_ms.append(1e3 * (time.perf_counter() - t0))
            layer_ms.append(cb["value"])
    value = float(np.mean(layer_ms))
    cb["value"] = value
    cb["sample"] = ("per step: " + cb["sample"] + f"; value = mean over {args.steps} steps "
                    "of the sample scaled to one layer")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": float(np.mean(step_ms)),
            "ms_per_step_is": "host time of one step's sample (value scales it to a layer)",
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": _workload_desc(w),
            "cpu_baseline": cb,
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
        # steps 1 + 2 in one launch (the estimate kernel also selects), then step 3
        if ev is not None:
            ev[0].record(stream)
        native.estimate_select(p, q, k, idx, cnt, wsp, mass=mass)
        if ev is not None:
            ev[1].record(stream)
        native.sparse_attn(p, q, k, v, idx, cnt, out, wsp)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, raw = native.check_device_status(wsp)
    if st != 0:
        raise RuntimeError(f"device status {raw:#x} after warm-up")
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush = _needs_flush(w)
    scrub = torch.empty(2 * _l2_bytes(), dtype=torch.uint8, device=dev) if flush else None
    if ws_n > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for s in range(args.steps):
            if flush:
                scrub.fill_(s & 0xFF)   # evicts the inputs from L2 before every timed step
            step(events[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if ws_n > 1:
        dist.barrier()
    total_ms = start.elapsed_time(stop)
    es_ms = [e[0].elapsed_time(e[1]) for e in events]
    att_ms = [e[1].elapsed_time(e[2]) for e in events]
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

    ev_step_ms = float(np.mean(es_ms)) + float(np.mean(att_ms))
    total_ms, e2e_ms, ev_step_ms = max_over_ranks([total_ms, e2e_ms, ev_step_ms], dev)
    cnt_host = cnt.cpu().numpy()
    idx_host = idx.cpu().numpy()
    useful, executed, n_kept = attention_flops(idx_host, cnt_host, w.block, w.head_dim)
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
        es_avg = float(np.mean(es_ms))
        achieved = useful / (att_avg * 1e-3) / 1e12
        # a timed region under 2 s is a burst: the burst GEMM peak applies; a longer one runs
        # into the power cap, where the sustained peak applies
        long_region = total_ms >= 2000.0
        peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
        ns = w.seqlen // w.stride
        # per-rank algorithmic bytes (this rank's heads)
        est_bytes = (p.batch * p.heads_kv * w.seqlen * w.head_dim * 2          # K read once
                     + p.batch * p.heads_q * ns * w.head_dim * 2               # sampled Q rows
                     + p.batch * p.heads_q * nb * (nb + 1) // 2 * 4)           # masses out
        sel_bytes = (p.batch * p.heads_q * nb * (nb + 1) // 2 * 4 + n_kept * 4 +
                     p.batch * p.heads_q * nb * 4)
        # with L2 flushes between the steps, a step's time is its own events' span (the flush
        # sits outside it); otherwise the whole region over the steps
        if flush:
            ms_per_step = ev_step_ms
        else:
            ms_per_step = total_ms / args.steps
        # ms per layer of the whole job: replicas finish ws_n layers per step, head shards one
        value = ms_per_step if sharded else ms_per_step / ws_n
        cpu = None
        if ws_n == 1 and not args.no_cpu_baseline and not sharded:
            def out_rows(b, h, r0, r1):
                return out[b, h, r0:r1].float().cpu().numpy().astype(np.float64)
            gpu_np = {"mass": mass.cpu().numpy(), "idx": idx_host, "cnt": cnt_host,
                      "out_rows": out_rows}
            cpu = cpu_oracle_baseline(w, q_bits, k_bits, v_bits,
                                      est_heads_for(w, args.cpu_budget),
                                      attn_rows=args.ref_rows or 32, total_kept=n_kept,
                                      gpu=gpu_np)
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
            "data": f"synthetic (seeded, shaped like the pages' workloads: {w.name})",
            "config": _workload_desc(w, f"heads{ws_n}" if sharded else "replicas"),
            "phases_ms": {"estimate_select": es_avg, "sparse_attn": att_avg},
            "phases_ms_spread": {"estimate_select": spread(es_ms), "sparse_attn": spread(att_ms),
                                 "step": spread([a + b for a, b in zip(es_ms, att_ms)])},
            "phases_note": "estimate and select are one call (rra_estimate_select: the pooled-key, "
                           "estimate and select kernels)",
            "density": density,
            "density_per_head": head_density(cnt_host),
            "attn_tflops": achieved, "attn_tflops_executed": executed / (att_avg * 1e-3) / 1e12,
            "estimate_select_gbs": (est_bytes + sel_bytes) / (es_avg * 1e-3) / 1e9,
            "estimate_select_frac_hbm": (est_bytes + sel_bytes) / (es_avg * 1e-3) / 1e9
            / peaks["hbm_gbs"],
            "roofline": {"bound": "tensor", "kernel": "bs_attn_fwd_kernel", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peaks['source']} bf16 "
                                        f"{'sustained' if long_region else 'burst'} "
                                        f"(timed region {total_ms / 1e3:.2f} s)",
                         "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                         "traffic": traffic,
                         "per_launch_flops": useful},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_ms if sharded else e2e_ms / ws_n, "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d_all), "d2h_bytes_per_step": int(d2h_all)},
            "gpu_launches": 3 * args.steps,
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
KERNEL_REV = "attn-v9-pq4"


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama128k", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--stride", type=int, default=None, help="override the workload's S")
    ap.add_argument("--tau", type=float, default=None, help="override the workload's tau")
    ap.add_argument("--seqlen", type=int, default=None, help="override the workload's L")
    ap.add_argument("--shift", type=int, default=None, help="override the round-robin shift")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="seeded query blocks of oracle attention in the CPU baseline "
                         "(default 32) or per step of the reference arm (default 4)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle estimate + select in the CPU baseline: every "
                         "head if they fit, else an evenly spread subset")
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
    over = {k: getattr(args, k) for k in ("stride", "tau", "seqlen", "shift")
            if getattr(args, k) is not None}
    if over:   # the same recipe and seed at other settings (e.g. the 32K sweep points)
        w = w.with_(**over)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
