"""The fp64 oracle over many heads at once, on a pool of spawned processes (test helper).

Spawned, not forked: the test process holds a CUDA context, and a child forked from it hangs.
This module imports only numpy, the oracle and the input generator, so the workers start
quickly; each worker uses a single BLAS thread and computes every block row of one head.
"""
from __future__ import annotations

import concurrent.futures
import multiprocessing
import os

import numpy as np

import oracle as orc
from long_context_prefill_rr_b200 import workloads as wl


def head_masses(args):
    """fp64 oracle masses of every block row of one (batch, head): [NB(NB+1)/2]."""
    q_bits, k_bits, h, nb, block, stride, shift, scale = args
    q = wl.bf16_bits_to_f64(q_bits)
    kbar = orc.pooled_keys(wl.bf16_bits_to_f64(k_bits), stride)
    out = np.empty(orc.tri_offset(nb), dtype=np.float64)
    for I in range(nb):
        out[orc.tri_offset(I):orc.tri_offset(I + 1)] = orc.estimate_block_row(
            q, kbar, h, I, block, stride, shift, scale)
    return out


def masses_full(q_bits, k_bits, batch, heads_q, heads_kv, seqlen, block, stride, shift, scale,
                heads=None, workers=None) -> dict:
    """{(b, h): masses of every block row} for every (b, h), or the listed ones."""
    nb = seqlen // block
    keys = heads if heads is not None else [(b, h) for b in range(batch) for h in range(heads_q)]
    tasks = [(np.ascontiguousarray(q_bits[b, h]),
              np.ascontiguousarray(k_bits[b, orc.kv_head(h, heads_q, heads_kv)]),
              h, nb, block, stride, shift, scale) for b, h in keys]
    if workers is None:
        # below 64K tokens a head takes well under a second: starting workers costs more
        workers = 1 if seqlen < 65536 else max(1, min(len(tasks), len(os.sched_getaffinity(0))))
    if workers == 1 or len(tasks) == 1:
        return {key: head_masses(t) for key, t in zip(keys, tasks)}
    names = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    saved = {v: os.environ.get(v) for v in names}
    for v in names:
        os.environ[v] = "1"
    try:
        ctx = multiprocessing.get_context("spawn")
        with concurrent.futures.ProcessPoolExecutor(workers, mp_context=ctx) as ex:
            res = list(ex.map(head_masses, tasks))
    finally:
        for v, old in saved.items():
            if old is None:
                os.environ.pop(v, None)
            else:
                os.environ[v] = old
    return dict(zip(keys, res))


def head_xattn_masses(args):
    """fp64 XAttention (antidiagonal) masses of every block row of one (batch, head)."""
    q_bits, k_bits, nb, block, stride, scale = args
    q = wl.bf16_bits_to_f64(q_bits)
    k = wl.bf16_bits_to_f64(k_bits)
    out = np.empty(orc.tri_offset(nb), dtype=np.float64)
    for I in range(nb):
        out[orc.tri_offset(I):orc.tri_offset(I + 1)] = orc.xattn_estimate_block_row(
            q, k, I, block, stride, scale)
    return out


def _pool_map(fn, tasks, workers):
    """fn over tasks, serially or on spawned processes with one BLAS thread each."""
    if workers is None:
        workers = max(1, min(len(tasks), len(os.sched_getaffinity(0))))
    if workers == 1 or len(tasks) <= 1:
        return [fn(t) for t in tasks]
    names = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    saved = {v: os.environ.get(v) for v in names}
    for v in names:
        os.environ[v] = "1"
    try:
        ctx = multiprocessing.get_context("spawn")
        with concurrent.futures.ProcessPoolExecutor(workers, mp_context=ctx) as ex:
            return list(ex.map(fn, tasks))
    finally:
        for v, old in saved.items():
            if old is None:
                os.environ.pop(v, None)
            else:
                os.environ[v] = old


def xattn_masses_full(q_bits, k_bits, batch, heads_q, heads_kv, seqlen, block, stride, scale,
                      workers=None) -> dict:
    """{(b, h): XAttention masses of every block row} for every (b, h)."""
    nb = seqlen // block
    keys = [(b, h) for b in range(batch) for h in range(heads_q)]
    tasks = [(np.ascontiguousarray(q_bits[b, h]),
              np.ascontiguousarray(k_bits[b, orc.kv_head(h, heads_q, heads_kv)]),
              nb, block, stride, scale) for b, h in keys]
    return dict(zip(keys, _pool_map(head_xattn_masses, tasks, workers)))


def head_attention_errors(args):
    """Oracle attention of every query block of one (batch, head) on the GPU's kept lists,
    compared with the GPU's output rows: (max |gpu - ref|, sum (gpu - ref)^2, sum ref^2)."""
    q_bits, k_bits, v_bits, gpu_out, idx, cnt, block, scale = args
    q = wl.bf16_bits_to_f64(q_bits)
    k = wl.bf16_bits_to_f64(k_bits)
    v = wl.bf16_bits_to_f64(v_bits)
    nb = q.shape[0] // block
    max_abs, sq_diff, sq_ref = 0.0, 0.0, 0.0
    for I in range(nb):
        off = orc.tri_offset(I)
        ref = orc.attention_block(q, k, v, I, idx[off:off + int(cnt[I])], block, scale)
        diff = gpu_out[I * block:(I + 1) * block].astype(np.float64) - ref
        max_abs = max(max_abs, float(np.abs(diff).max()))
        sq_diff += float(np.sum(diff * diff))
        sq_ref += float(np.sum(ref * ref))
    return max_abs, sq_diff, sq_ref


def attention_errors_full(q_bits, k_bits, v_bits, gpu_out, idx, cnt, heads_q, heads_kv, block,
                          scale, workers=None):
    """Every output row of every (batch, head) against the oracle, one head per task on a pool
    of spawned processes: (max-abs error, relative RMS error, rows compared). gpu_out is the GPU
    output as a float32 array [b, Hq, L, d]; idx / cnt are the GPU's kept lists."""
    b = gpu_out.shape[0]
    keys = [(bi, h) for bi in range(b) for h in range(heads_q)]

    def task(bi, h):
        kv = orc.kv_head(h, heads_q, heads_kv)
        return (np.ascontiguousarray(q_bits[bi, h]), np.ascontiguousarray(k_bits[bi, kv]),
                np.ascontiguousarray(v_bits[bi, kv]), np.ascontiguousarray(gpu_out[bi, h]),
                np.ascontiguousarray(idx[bi, h]), np.ascontiguousarray(cnt[bi, h]), block, scale)

    if workers is None:
        workers = max(1, min(len(keys), len(os.sched_getaffinity(0))))
    if workers == 1:
        res = [head_attention_errors(task(bi, h)) for bi, h in keys]
    else:
        names = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        saved = {v: os.environ.get(v) for v in names}
        for v in names:
            os.environ[v] = "1"
        try:
            ctx = multiprocessing.get_context("spawn")
            with concurrent.futures.ProcessPoolExecutor(workers, mp_context=ctx) as ex:
                res = list(ex.map(head_attention_errors, (task(bi, h) for bi, h in keys)))
        finally:
            for v, old in saved.items():
                if old is None:
                    os.environ.pop(v, None)
                else:
                    os.environ[v] = old
    max_abs = max(r[0] for r in res)
    rel_rms = float(np.sqrt(sum(r[1] for r in res) / max(sum(r[2] for r in res), 1e-300)))
    return max_abs, rel_rms, len(keys) * (gpu_out.shape[2] // block)
