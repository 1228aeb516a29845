"""fp64 CPU oracle of the RRAttention prefill hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or executes this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` use it. It shares no code with the CUDA library; both sides only consume the
same seeded inputs.

Sources (titles of the pages that describe the method):

* [RR]  "RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
        Long-Context Inference" (arXiv 2602.05853), abstract: in every stride the query
        sampling position rotates across heads; stride-level aggregation cuts estimation
        from O(L^2) to O(L^2/S^2); adaptive Top-tau selection.
* [RRs] research summary page of the same paper, "Summary" and "Key points": one query per
        stride of S tokens per head, offset rotating from head to head; scores pooled per
        stride; softmax at stride granularity ("Table 1"); B = 128, S = 8 default; coverage
        of all positions fails when S exceeds the number of heads.
* [XA]  "XAttention: Block Sparse Attention with Antidiagonal Scoring" review, section 3
        ("threshold block selection"): softmax the stride scores, then ``find_blocks``:
        the smallest set of blocks whose summed probability reaches tau.

Every step below follows those passages; where they leave a detail open, the reading taken is
written at the step (and collected in the design notes of the repository):

1. offset        o_h = (h + shift) mod S                      (rotation across heads [RR])
2. sampled query q_{h,i} = Q[h, i*S + o_h]                     (one query per stride [RRs])
3. pooled key    Kbar_{kv,j} = sum_{t<S} K[kv, j*S + t]        (stride aggregation; a SUM)
4. logits        z_{h,i,j} = scale * q_{h,i} . Kbar_{kv(h),j}, j <= i   (no extra 1/S)
5. stride softmax P_{h,i,j} = softmax over j <= i of z_{h,i,.}  (stride-level causality,
                 the diagonal stride j = i included in full)
6. block mass    A_{h,I,J} = (1/m) sum_{i in I} sum_{j in J, j<=i} P_{h,i,j}, m = B/S,
                 so each block row sums to 1 and tau is a fraction of the row mass.
7. select        per block row: sort J descending by A (ties: J ascending), keep the smallest
                 prefix whose running sum reaches tau * sum_J A (inclusive >=), then add the
                 diagonal block I; tau >= 1 keeps every causal block ([XA] find_blocks).
8. attention     O[h,t] = softmax over the keys u of the kept blocks with u <= t of
                 scale * Q[h,t].K[kv(h),u], applied to V; a query with no key gets 0.
                 GQA: kv(h) = floor(h / (Hq/Hkv)).

The XAttention antidiagonal estimator (the predecessor method, [XA] sections 2-3) replaces
steps 1-4: within every S x S sub-block of the attention logits the S elements of the
antidiagonal (bottom-left to top-right: query offset t with key offset S-1-t) are summed,

   z^xa_{h,i,j} = scale * sum_{t<S} Q[h, i*S + t] . K[kv(h), j*S + S-1-t],  j <= i,

followed by the same stride-level causal softmax, block masses (step 6) and selection (step 7).
There is no per-head rotation: every head scores all of its queries.

Parity pins for every step live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rr_offset", "pooled_keys", "block_row_logits", "stride_softmax_rows", "block_masses_row",
    "estimate", "estimate_block_row", "select_row", "select", "attention_block",
    "sparse_attention", "tri_offset", "kv_head", "xattn_block_row_logits",
    "xattn_estimate_block_row", "xattn_estimate",
]


def tri_offset(I: int) -> int:
    """Offset of block row I in the packed lower-triangular per-head layout."""
    return I * (I + 1) // 2


def kv_head(h: int, heads_q: int, heads_kv: int) -> int:
    """GQA: contiguous groups of Hq/Hkv query heads share one KV head."""
    return h // (heads_q // heads_kv)


def rr_offset(h: int, stride: int, shift: int) -> int:
    """Step 1: in-stride position sampled by head h; rotates by one position per head [RR]."""
    return (h + shift) % stride


def pooled_keys(k: np.ndarray, stride: int) -> np.ndarray:
    """Step 3: stride sums of the keys of one KV head. k [L, d] -> [L/S, d] (fp64)."""
    L, d = k.shape
    return k.astype(np.float64).reshape(L // stride, stride, d).sum(axis=1)


def block_row_logits(q: np.ndarray, kbar: np.ndarray, h: int, I: int, block: int,
                     stride: int, shift: int, scale: float) -> np.ndarray:
    """Steps 2 and 4 for block row I of head h.

    q [L, d] (this head's queries), kbar [L/S, d] (this head's KV group, pooled).
    Returns z [m, (I+1)*m]: rows are the m sampled queries i = I*m .. I*m+m-1, columns are
    the stride indices j = 0 .. (I+1)*m - 1 (entries with j > i are later masked out).
    """
    m = block // stride
    o = rr_offset(h, stride, shift)
    rows = (np.arange(I * m, (I + 1) * m) * stride + o)
    qhat = q[rows].astype(np.float64)                       # step 2
    return scale * (qhat @ kbar[: (I + 1) * m].T)           # step 4


def stride_softmax_rows(z: np.ndarray, first_row: int) -> np.ndarray:
    """Step 5: causal softmax of each row over strides j <= i, i = first_row + row."""
    nrows, ncols = z.shape
    i = first_row + np.arange(nrows)[:, None]
    j = np.arange(ncols)[None, :]
    valid = j <= i
    zmax = np.where(valid, z, -np.inf).max(axis=1, keepdims=True)
    e = np.where(valid, np.exp(np.where(valid, z, 0.0) - zmax), 0.0)
    return e / e.sum(axis=1, keepdims=True)


def block_masses_row(p: np.ndarray, m: int) -> np.ndarray:
    """Step 6: A_{I,J} for J = 0..I from the probabilities of block row I, p [m, (I+1)*m]."""
    nrows, ncols = p.shape
    return p.reshape(nrows, ncols // m, m).sum(axis=(0, 2)) / m


def estimate_block_row(q: np.ndarray, kbar: np.ndarray, h: int, I: int, block: int,
                       stride: int, shift: int, scale: float) -> np.ndarray:
    """Masses A_{h,I,0..I} (fp64) of one block row: steps 2, 4, 5, 6."""
    m = block // stride
    z = block_row_logits(q, kbar, h, I, block, stride, shift, scale)
    p = stride_softmax_rows(z, I * m)
    return block_masses_row(p, m)


def _check_shapes(q, k, block, stride):
    b, hq, L, d = q.shape
    bk, hkv, Lk, dk = k.shape
    assert (b, L, d) == (bk, Lk, dk) and hq % hkv == 0
    assert L % block == 0 and block % stride == 0
    return b, hq, hkv, L, d


def estimate(q: np.ndarray, k: np.ndarray, block: int, stride: int, shift: int,
             scale: float) -> np.ndarray:
    """All block masses. q [b,Hq,L,d], k [b,Hkv,L,d] (any float dtype; promoted to fp64).

    Returns A [b, Hq, NB(NB+1)/2] fp64, block row I of each head at offset I(I+1)/2.
    """
    b, hq, hkv, L, d = _check_shapes(q, k, block, stride)
    nb = L // block
    out = np.zeros((b, hq, tri_offset(nb)), dtype=np.float64)
    for bi in range(b):
        kbars = [pooled_keys(k[bi, kv], stride) for kv in range(hkv)]
        for h in range(hq):
            qh = q[bi, h]
            kb = kbars[kv_head(h, hq, hkv)]
            for I in range(nb):
                out[bi, h, tri_offset(I):tri_offset(I + 1)] = estimate_block_row(
                    qh, kb, h, I, block, stride, shift, scale)
    return out


def xattn_block_row_logits(q: np.ndarray, k: np.ndarray, I: int, block: int, stride: int,
                           scale: float) -> np.ndarray:
    """Antidiagonal stride scores of block row I for one head ([XA] sections 2-3).

    q [L, d] (this head's queries), k [L, d] (its KV head's keys). Returns z [m, (I+1)*m]:
    rows i = I*m .. I*m+m-1, columns j = 0 .. (I+1)*m - 1 (j > i is masked later).
    """
    m = block // stride
    L, d = q.shape
    qs = q.astype(np.float64).reshape(L // stride, stride, d)[I * m:(I + 1) * m]   # [m, S, d]
    ks = k.astype(np.float64).reshape(L // stride, stride, d)[:(I + 1) * m]       # [n, S, d]
    z = np.zeros((m, (I + 1) * m))
    for t in range(stride):
        z += qs[:, t, :] @ ks[:, stride - 1 - t, :].T     # query offset t with key offset S-1-t
    return scale * z


def xattn_estimate_block_row(q: np.ndarray, k: np.ndarray, I: int, block: int, stride: int,
                             scale: float) -> np.ndarray:
    """XAttention masses A^xa_{h,I,0..I}: antidiagonal scores, stride softmax, block sums."""
    m = block // stride
    z = xattn_block_row_logits(q, k, I, block, stride, scale)
    p = stride_softmax_rows(z, I * m)
    return block_masses_row(p, m)


def xattn_estimate(q: np.ndarray, k: np.ndarray, block: int, stride: int,
                   scale: float) -> np.ndarray:
    """All XAttention block masses, in the packed layout of ``estimate``."""
    b, hq, hkv, L, d = _check_shapes(q, k, block, stride)
    nb = L // block
    out = np.zeros((b, hq, tri_offset(nb)), dtype=np.float64)
    for bi in range(b):
        for h in range(hq):
            kh = k[bi, kv_head(h, hq, hkv)]
            for I in range(nb):
                out[bi, h, tri_offset(I):tri_offset(I + 1)] = xattn_estimate_block_row(
                    q[bi, h], kh, I, block, stride, scale)
    return out


def select_row(a: np.ndarray, I: int, tau: float) -> np.ndarray:
    """Step 7 for one block row: masses a[0..I] -> ascending kept block indices (int32)."""
    n = I + 1
    if tau >= 1.0:
        return np.arange(n, dtype=np.int32)
    a = np.asarray(a, dtype=np.float64)[:n]
    order = np.argsort(-a, kind="stable")          # descending mass, ties by J ascending
    total = float(np.sum(a))
    csum = np.cumsum(a[order])
    hit = np.nonzero(csum >= tau * total)[0]
    k = int(hit[0]) + 1 if hit.size else n          # no prefix reaches tau: keep all
    kept = set(order[:k].tolist())
    kept.add(I)                                     # diagonal always kept
    return np.array(sorted(kept), dtype=np.int32)


def select(mass: np.ndarray, nb: int, tau: float):
    """Step 7 for every row. mass [b, H, NB(NB+1)/2] -> (kept_idx, kept_cnt).

    kept_idx int32 [b, H, NB(NB+1)/2]: row I at offset I(I+1)/2, ascending, -1 padded.
    kept_cnt int32 [b, H, NB].
    """
    b, h, t = mass.shape
    assert t == tri_offset(nb)
    idx = np.full((b, h, t), -1, dtype=np.int32)
    cnt = np.zeros((b, h, nb), dtype=np.int32)
    for bi in range(b):
        for hh in range(h):
            for I in range(nb):
                off = tri_offset(I)
                row = select_row(mass[bi, hh, off:off + I + 1], I, tau)
                idx[bi, hh, off:off + row.size] = row
                cnt[bi, hh, I] = row.size
    return idx, cnt


def attention_block(q: np.ndarray, k: np.ndarray, v: np.ndarray, I: int, kept: np.ndarray,
                    block: int, scale: float) -> np.ndarray:
    """Step 8 for query block I of one head: q [L,d], k/v [L,d] of its KV head.

    Two-pass masked softmax over the keys of the kept blocks (materialise, max, sum).
    Returns O [block, d] fp64.
    """
    kept = np.asarray(kept, dtype=np.int64)
    t = I * block + np.arange(block)
    d = q.shape[1]
    if kept.size == 0:
        return np.zeros((block, d))
    keys = (kept[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    s = scale * (q[t].astype(np.float64) @ k[keys].astype(np.float64).T)   # [block, nkeys]
    allowed = keys[None, :] <= t[:, None]
    smax = np.where(allowed, s, -np.inf).max(axis=1, keepdims=True)
    has = np.isfinite(smax)
    e = np.where(allowed, np.exp(np.where(allowed, s, 0.0) - np.where(has, smax, 0.0)), 0.0)
    den = e.sum(axis=1, keepdims=True)
    o = (e @ v[keys].astype(np.float64)) / np.where(den > 0, den, 1.0)
    return np.where(has, o, 0.0)


def sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, kept_idx: np.ndarray,
                     kept_cnt: np.ndarray, block: int, scale: float,
                     rows=None) -> np.ndarray:
    """Step 8 for every (b, h, I) (or only ``rows``, a list of (b, h, I)).

    Returns O [b, Hq, L, d] fp64 (rows not requested stay 0).
    """
    b, hq, L, d = q.shape
    hkv = k.shape[1]
    nb = L // block
    out = np.zeros((b, hq, L, d), dtype=np.float64)
    if rows is None:
        rows = [(bi, h, I) for bi in range(b) for h in range(hq) for I in range(nb)]
    for bi, h, I in rows:
        kv = kv_head(h, hq, hkv)
        off = tri_offset(I)
        kept = kept_idx[bi, h, off:off + int(kept_cnt[bi, h, I])]
        out[bi, h, I * block:(I + 1) * block] = attention_block(
            q[bi, h], k[bi, kv], v[bi, kv], I, kept, block, scale)
    return out
