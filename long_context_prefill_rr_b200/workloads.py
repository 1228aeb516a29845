"""Seeded synthetic prefill-attention inputs (Q, K, V) shaped like the RRAttention workloads.

This module only draws random numbers and plants structure in them; it holds none of the
method's arithmetic. Both the CUDA path (through the binding) and the fp64 oracle consume
exactly the arrays produced here, so a parity test compares the two on identical bf16 values.

Workloads (RRAttention, "Experiments": LLaMA-3.1-8B-Instruct and Qwen on HELMET 8K-128K and
Video-MME; the datasets and weights are not available, so these seeded stand-ins keep the
shapes, the GQA ratio and plausible attention structure):

* ``tiny``     b1, 8 Q / 8 KV heads, d 64, L 1024, S 8, tau 0.9, softmax scale 1.
* ``llama8k``  b1, 32 Q / 8 KV heads, d 128, L 8192, S 8, tau 0.9, scale 1.
* ``llama32k`` same layer at L 32768 (S in {8, 16}, tau in {0.9, 0.95}).
* ``llama128k`` same layer at L 131072, S 8, tau 0.9.
* ``video64k`` b1, 28 Q / 4 KV heads, d 128, L 65536 = 256 frames x 256 tokens, S 16, tau 0.9,
  scale 1/sqrt(d).

Value recipe (fp32 draws, rounded once to bf16 with round-to-nearest-even):

* tiny: Q, K, V ~ N(0,1)/d^(1/4). Sink K[0] += 3 qbar. Vertical lines K[j] += 2 qbar for
  j % 97 == 0, j > 0.
* llama*: Q, K ~ N(0,1)/d^(1/4), V ~ N(0,1). Sink K[0] += 3 qbar; 16 distinct random key
  columns per KV head in [1, L) get K += 2.5 qbar; local band K[j] += 1.5 w_j.
* video: Q and K tokens = N(0,1) + F[frame] (sigma 1.0) + P[pos] (sigma 0.7); F and P are drawn
  per KV head and shared by its Q heads and its keys; V ~ N(0,1).

``qbar`` (per KV head) = d^(1/4) * unit(mean of Q over the group's heads and all positions):
the mean query direction at a typical query norm. ``w_j`` = d^(1/4) * unit(sum of the group's
queries at positions j+1 .. min(j+256, L-1)), so key j leans towards the next 256 queries.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "make_workload", "bf16_round_bits", "bf16_bits_to_f32",
    "bf16_bits_to_f64", "random_kept_lists",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seqlen: int
    head_dim: int
    stride: int
    tau: float
    softmax_scale: float   # <= 0 means 1/sqrt(head_dim)
    seed: int
    kind: str              # "tiny" | "llama" | "video"
    block: int = 128
    shift: int = 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 8, 8, 1024, 64, 8, 0.9, 1.0, 0, "tiny"),
    "llama8k": Workload("llama8k", 1, 32, 8, 8192, 128, 8, 0.9, 1.0, 1, "llama"),
    "llama32k": Workload("llama32k", 1, 32, 8, 32768, 128, 8, 0.9, 1.0, 2, "llama"),
    "llama128k": Workload("llama128k", 1, 32, 8, 131072, 128, 8, 0.9, 1.0, 3, "llama"),
    "video64k": Workload("video64k", 1, 28, 4, 65536, 128, 16, 0.9, -1.0, 4, "video"),
}


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> uint16 bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def _unit(v: np.ndarray, axis: int = -1) -> np.ndarray:
    n = np.linalg.norm(v, axis=axis, keepdims=True)
    return np.where(n > 0, v / np.where(n > 0, n, 1.0), 0.0)


def _normal(seq: np.random.SeedSequence, shape, scale: float = 1.0) -> np.ndarray:
    """fp32 N(0, scale^2) draws of ``shape``; each leading-two-axes slice has its own PCG64
    stream spawned from ``seq``, so the values do not depend on the thread count."""
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1, *shape[2:]) if len(shape) > 2 else out.reshape(1, -1)
    children = seq.spawn(flat.shape[0])

    def fill(i):
        np.random.Generator(np.random.PCG64(children[i])).standard_normal(
            dtype=np.float32, out=flat[i])
        if scale != 1.0:
            flat[i] *= np.float32(scale)

    workers = max(1, min(len(children), len(os.sched_getaffinity(0))))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        list(ex.map(fill, range(len(children))))
    return out


def make_workload(w: Workload | str, seqlen: int | None = None):
    """Draw the seeded inputs of workload ``w``.

    Returns ``(q, k, v)`` as uint16 bf16 bit patterns, shapes [b, Hq, L, d], [b, Hkv, L, d],
    [b, Hkv, L, d], C-contiguous. ``seqlen`` overrides the workload length (same recipe).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if seqlen is not None:
        w = w.with_(seqlen=seqlen)
    b, hq, hkv, L, d = w.batch, w.heads_q, w.heads_kv, w.seqlen, w.head_dim
    g = hq // hkv
    ss = np.random.SeedSequence(w.seed)
    sq, sk, sv, sxs = ss.spawn(4)
    sx = np.random.Generator(np.random.PCG64(sxs))
    d4 = float(d) ** 0.25
    if w.kind in ("tiny", "llama"):
        q = _normal(sq, (b, hq, L, d), 1.0 / d4)
        k = _normal(sk, (b, hkv, L, d), 1.0 / d4)
        v = _normal(sv, (b, hkv, L, d), 1.0 / d4 if w.kind == "tiny" else 1.0)
        qg = q.reshape(b, hkv, g, L, d)
        # mean query direction of each KV group, rescaled to a typical query norm
        qbar = (d4 * _unit(qg.mean(axis=(2, 3), dtype=np.float64))).astype(np.float32)  # [b,hkv,d]
        k[:, :, 0, :] += 3.0 * qbar
        if w.kind == "tiny":
            cols = np.arange(97, L, 97)
            k[:, :, cols, :] += 2.0 * qbar[:, :, None, :]
        else:
            for bi in range(b):
                for kv in range(hkv):
                    cols = sx.choice(np.arange(1, L), size=min(16, L - 1), replace=False)
                    k[bi, kv, cols, :] += 2.5 * qbar[bi, kv][None, :]
            # local band: key j leans towards the group's queries at j+1 .. min(j+256, L-1)
            qs = qg.sum(axis=2, dtype=np.float64)                      # [b,hkv,L,d]
            cs = np.zeros((b, hkv, L + 1, d), dtype=np.float64)
            np.cumsum(qs, axis=2, out=cs[:, :, 1:, :])
            j = np.arange(L)
            hi = np.minimum(j + 256, L - 1) + 1                          # exclusive end
            lo = np.minimum(j + 1, hi)
            win = cs[:, :, hi, :] - cs[:, :, lo, :]
            del cs, qs
            k += (1.5 * d4 * _unit(win)).astype(np.float32)
            del win
    elif w.kind == "video":
        tok = 256
        if L % tok:
            raise ValueError("video workload needs L to be a multiple of 256 tokens per frame")
        nf = L // tok
        fr = _normal(sxs.spawn(1)[0], (b, hkv, nf, d), 1.0)
        po = _normal(sxs.spawn(1)[0], (b, hkv, tok, d), 0.7)
        struct = (fr[:, :, :, None, :] + po[:, :, None, :, :]).reshape(b, hkv, L, d)
        q = _normal(sq, (b, hq, L, d)).reshape(b, hkv, g, L, d)
        q += struct[:, :, None, :, :]
        q = q.reshape(b, hq, L, d)
        k = _normal(sk, (b, hkv, L, d)) + struct
        v = _normal(sv, (b, hkv, L, d))
    else:
        raise ValueError(f"unknown workload kind {w.kind}")
    return bf16_round_bits(q), bf16_round_bits(k), bf16_round_bits(v)


def random_kept_lists(batch: int, heads: int, nb: int, density: float, seed: int):
    """Seeded random causal block masks in the packed kept-list layout.

    Each row I keeps its diagonal block plus each J < I independently with probability
    ``density``. Returns (kept_idx int32 [b, H, nb(nb+1)/2] ascending, -1 padded,
    kept_cnt int32 [b, H, nb]).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    T = nb * (nb + 1) // 2
    idx = np.full((batch, heads, T), -1, dtype=np.int32)
    cnt = np.zeros((batch, heads, nb), dtype=np.int32)
    for bi in range(batch):
        for h in range(heads):
            for I in range(nb):
                keep = np.nonzero(rng.random(I) < density)[0].astype(np.int32)
                row = np.concatenate([keep, np.array([I], np.int32)])
                off = I * (I + 1) // 2
                idx[bi, h, off:off + row.size] = row
                cnt[bi, h, I] = row.size
    return idx, cnt
