"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI, run the fp64
oracle on the same bf16 inputs, and compare with the tolerances the benchmark spec fixes:

* block masses within 1e-3 absolute;
* kept lists bit-exact, except rows whose oracle running sum comes within 1e-4 of the tau
  boundary or whose cut falls between masses closer than 1e-4 (counted and reported);
* attention output (given the GPU's own kept lists) within max-abs 2e-2 and relative RMS 1e-2
  of the fp64 result.
"""
from __future__ import annotations

import json
import os
import time

import numpy as np
import torch

import oracle as orc
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

MASS_ATOL = 1e-3
BOUNDARY = 1e-4
ATTN_MAX_ABS = 2e-2
ATTN_REL_RMS = 1e-2


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_dev_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def resolved_scale(p) -> float:
    return float(p.softmax_scale) if p.softmax_scale > 0 else 1.0 / np.sqrt(p.head_dim)


def run_prefill(p, qd, kd, vd):
    """Full path on the GPU; returns numpy mass, kept_idx, kept_cnt, out (fp32 copy of the bf16
    output) and the device status."""
    sh = native.shapes(p)
    mass = torch.empty(sh["mass"], dtype=torch.float32, device="cuda")
    idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda")
    cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda")
    out = torch.empty(sh["q"], dtype=torch.bfloat16, device="cuda")
    ws = native.new_workspace(p)
    native.prefill(p, qd, kd, vd, out, idx, cnt, ws, mass=mass)
    st, raw = native.check_device_status(ws)
    return dict(mass=mass.cpu().numpy(), idx=idx.cpu().numpy(), cnt=cnt.cpu().numpy(),
                out=bf16_dev_to_f32(out), status=st, raw=raw)


def boundary_row(a_oracle: np.ndarray, tau: float) -> bool:
    """True if the oracle's descending running sum comes within BOUNDARY of tau * total, or the
    masses on both sides of the cut are within BOUNDARY of each other."""
    a = np.asarray(a_oracle, dtype=np.float64)
    order = np.argsort(-a, kind="stable")
    srt = a[order]
    cs = np.cumsum(srt)
    target = tau * a.sum()
    if np.min(np.abs(cs - target)) <= BOUNDARY:
        return True
    hit = np.nonzero(cs >= target)[0]
    k = int(hit[0]) if hit.size else len(a) - 1
    if k + 1 < len(a) and abs(srt[k] - srt[k + 1]) <= BOUNDARY:
        return True
    return False


def kept_row(idx, cnt, bh, I):
    b, h = bh
    off = orc.tri_offset(I)
    return idx[b, h, off:off + cnt[b, h, I]]


def compare_select_rows(gpu, oracle_mass_rows: dict, tau: float):
    """oracle_mass_rows: {(b, h, I): fp64 masses}. Returns (mismatches, excused, n)."""
    tau32 = float(np.float32(tau))
    mism, excused = [], []
    for (b, h, I), a in oracle_mass_rows.items():
        want = orc.select_row(a, I, tau32)
        got = kept_row(gpu["idx"], gpu["cnt"], (b, h), I)
        if not np.array_equal(want, got):
            (excused if boundary_row(a, tau32) else mism).append((b, h, I))
    return mism, excused, len(oracle_mass_rows)


def select_on_gpu_masses_exact(gpu, tau: float, nb: int):
    """The GPU's lists must equal the oracle's select run on the GPU's own fp32 masses
    (the decision taken on identical inputs, both in fp64 accumulation)."""
    idx, cnt = orc.select(gpu["mass"].astype(np.float64), nb, float(np.float32(tau)))
    return np.array_equal(idx, gpu["idx"]) and np.array_equal(cnt, gpu["cnt"])


def attention_errors(gpu_out: np.ndarray, ref: np.ndarray, rows=None, block=128):
    """(max_abs, rel_rms) over all rows, or over the (b, h, I) query blocks in ``rows``."""
    if rows is not None:
        g = np.concatenate([gpu_out[b, h, I * block:(I + 1) * block] for b, h, I in rows])
        r = np.concatenate([ref[b, h, I * block:(I + 1) * block] for b, h, I in rows])
    else:
        g, r = gpu_out, ref
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    diff = g - r
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.sqrt(np.mean(r * r))) if r.size else 1.0
    rel_rms = float(np.sqrt(np.mean(diff * diff)) / max(denom, 1e-30)) if diff.size else 0.0
    return max_abs, rel_rms


class HeadCache:
    """fp64 copies of single (batch, head) slices of a bf16-bit array, made on demand (the full
    fp64 tensors of the long workloads would not fit comfortably in host memory)."""

    def __init__(self, bits: np.ndarray):
        self.bits = bits
        self._c = {}

    def __call__(self, b: int, h: int) -> np.ndarray:
        if (b, h) not in self._c:
            self._c[(b, h)] = wl.bf16_bits_to_f64(self.bits[b, h])
        return self._c[(b, h)]


def oracle_mass_rows(qc: HeadCache, kc: HeadCache, p, rows):
    """fp64 oracle masses for the sampled block rows (b, h, I)."""
    scale = resolved_scale(p)
    kbars = {}
    out = {}
    for b, h, I in rows:
        kv = orc.kv_head(h, p.heads_q, p.heads_kv)
        if (b, kv) not in kbars:
            kbars[(b, kv)] = orc.pooled_keys(kc(b, kv), p.stride)
        out[(b, h, I)] = orc.estimate_block_row(qc(b, h), kbars[(b, kv)], h, I, p.block,
                                                p.stride, p.shift, scale)
    return out


def oracle_attention_rows(qc: HeadCache, kc: HeadCache, vc: HeadCache, p, idx, cnt, rows):
    """{(b, h, I): fp64 O block} for the given rows, using the kept lists idx / cnt."""
    scale = resolved_scale(p)
    out = {}
    for b, h, I in rows:
        kv = orc.kv_head(h, p.heads_q, p.heads_kv)
        kept = kept_row(idx, cnt, (b, h), I)
        out[(b, h, I)] = orc.attention_block(qc(b, h), kc(b, kv), vc(b, kv), I, kept, p.block,
                                             scale)
    return out


def attention_rows_errors(gpu_out: np.ndarray, ref_rows: dict, block=128):
    g = np.concatenate([gpu_out[b, h, I * block:(I + 1) * block] for b, h, I in ref_rows])
    r = np.concatenate([ref_rows[k] for k in ref_rows])
    return attention_errors(g, r)


def sample_rows(p, n, seed):
    """Seeded (b, h, I) sample that always includes the first and last block rows."""
    rng = np.random.default_rng(seed)
    nb = p.seqlen // p.block
    rows = {(0, 0, 0), (p.batch - 1, p.heads_q - 1, nb - 1), (0, p.heads_q // 2, nb // 2)}
    while len(rows) < n:
        rows.add((int(rng.integers(p.batch)), int(rng.integers(p.heads_q)),
                  int(rng.integers(nb))))
    return sorted(rows)


def workload_params(w: wl.Workload, **over):
    w = w.with_(**over) if over else w
    return w, native.params(w.batch, w.heads_q, w.heads_kv, w.seqlen, w.head_dim, w.stride,
                            w.tau, shift=w.shift, softmax_scale=w.softmax_scale, block=w.block)


# ------------------------------------------------------------------ full-coverage oracle passes
def oracle_masses_full(q_bits, k_bits, p, heads=None, workers=None) -> dict:
    """{(b, h): fp64 oracle masses of every block row} for every (b, h) (or the listed ones)."""
    import oracle_pool
    return oracle_pool.masses_full(q_bits, k_bits, p.batch, p.heads_q, p.heads_kv, p.seqlen,
                                   p.block, p.stride, p.shift, resolved_scale(p), heads, workers)


def mass_rows(full: dict, nb: int) -> dict:
    """{(b, h, I): masses of row I} views of oracle_masses_full's per-head arrays."""
    return {(b, h, I): a[orc.tri_offset(I):orc.tri_offset(I + 1)]
            for (b, h), a in full.items() for I in range(nb)}


# ------------------------------------------------------------------ parity report
# Every parity check appends one record here; tests/conftest.py prints them at the end of the
# session (so the boundary-excused counts appear in `pytest -q` output). If RRA_PARITY_REPORT
# names an existing directory, each record is also appended to parity_report.jsonl there.
RECORDS: list = []


def record(label: str, **fields) -> dict:
    rec = {"label": label, **fields, "when": time.strftime("%Y-%m-%dT%H:%M:%S")}
    RECORDS.append(rec)
    out_dir = os.environ.get("RRA_PARITY_REPORT")
    if out_dir and os.path.isdir(out_dir):
        with open(os.path.join(out_dir, "parity_report.jsonl"), "a") as f:
            f.write(json.dumps(rec) + "\n")
    return rec


def boundary_count(rows: dict, tau: float) -> int:
    """Oracle rows (of {(b, h, I): masses}) that fall under the boundary rule."""
    tau32 = float(np.float32(tau))
    return sum(1 for (b, h, I), a in rows.items() if I > 0 and boundary_row(a, tau32))


# ------------------------------------------------------------------ the comparisons
def full_check(w, p, bits, gpu, label):
    """Every mass, kept list and output row of a small problem against the oracle."""
    q64, k64, v64 = (wl.bf16_bits_to_f64(x) for x in bits)
    scale = resolved_scale(p)
    nb = w.seqlen // w.block
    assert gpu["status"] == 0, f"{label}: device status {gpu['raw']:#x}"
    om = orc.estimate(q64, k64, w.block, w.stride, w.shift, scale)
    merr = float(np.abs(gpu["mass"] - om).max())
    assert merr <= MASS_ATOL, f"{label}: mass err {merr}"
    assert select_on_gpu_masses_exact(gpu, w.tau, nb), f"{label}: select on GPU masses"
    rows = {(b, h, I): om[b, h, orc.tri_offset(I):orc.tri_offset(I + 1)]
            for b in range(w.batch) for h in range(w.heads_q) for I in range(nb)}
    mism, exc, n = compare_select_rows(gpu, rows, w.tau)
    assert not mism, f"{label}: kept-list mismatches outside the boundary rule: {mism[:5]}"
    ref = orc.sparse_attention(q64, k64, v64, gpu["idx"], gpu["cnt"], w.block, scale)
    ma, rr = attention_errors(gpu["out"], ref)
    assert ma <= ATTN_MAX_ABS and rr <= ATTN_REL_RMS, f"{label}: attn {ma} {rr}"
    dens = gpu["cnt"].sum() / (w.batch * w.heads_q * orc.tri_offset(nb))
    record(label, mass_rows=n, mass_max_err=merr, list_rows=n,
           list_mismatch_excused=len(exc), boundary_rows=boundary_count(rows, w.tau),
           attn_rows=f"all {w.batch * w.heads_q * nb}", attn_max_abs=ma, attn_rel_rms=rr,
           density=float(dens))


def long_check(w, p, bits, gpu, label, attn_rows, seed, mass_heads=None):
    """Every mass and kept list (of every head, or of ``mass_heads``) against the oracle, the
    select on the GPU's own masses over every row, and the attention output on every query
    block (attn_rows = "all") or on ``attn_rows`` seeded ones."""
    qb, kb, vb = bits
    assert gpu["status"] == 0, f"{label}: device status {gpu['raw']:#x}"
    nb = w.seqlen // w.block
    assert select_on_gpu_masses_exact(gpu, w.tau, nb), f"{label}: select on GPU masses"
    full = oracle_masses_full(qb, kb, p, heads=mass_heads)
    merr = max(float(np.abs(gpu["mass"][b, h] - a).max()) for (b, h), a in full.items())
    assert merr <= MASS_ATOL, f"{label}: mass err {merr}"
    rows = mass_rows(full, nb)
    mism, exc, n = compare_select_rows(gpu, rows, w.tau)
    assert not mism, f"{label}: kept-list mismatches outside the boundary rule: {mism[:5]}"
    if attn_rows == "all":
        import oracle_pool
        ma, rr, n_attn = oracle_pool.attention_errors_full(
            qb, kb, vb, gpu["out"], gpu["idx"], gpu["cnt"], p.heads_q, p.heads_kv, p.block,
            resolved_scale(p))
        arows = range(n_attn)
    else:
        qc, kc, vc = HeadCache(qb), HeadCache(kb), HeadCache(vb)
        arows = sample_rows(p, attn_rows, seed)
        ref = oracle_attention_rows(qc, kc, vc, p, gpu["idx"], gpu["cnt"], arows)
        ma, rr = attention_rows_errors(gpu["out"], ref)
    assert ma <= ATTN_MAX_ABS and rr <= ATTN_REL_RMS, f"{label}: attn {ma} {rr}"
    dens = gpu["cnt"].sum(dtype=np.int64) / (w.batch * w.heads_q * orc.tri_offset(nb))
    record(label, mass_rows=n, mass_max_err=merr, list_rows=n,
           list_mismatch_excused=len(exc), boundary_rows=boundary_count(rows, w.tau),
           attn_rows=("all " if attn_rows == "all" else "sampled ") + str(len(arows)),
           attn_max_abs=ma, attn_rel_rms=rr, density=float(dens))
