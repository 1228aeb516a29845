"""The pooled oracle helpers used by the GPU parity tests give what the oracle gives: the per-head
work on spawned processes reassembles the oracle's own results, and the attention comparison
reports a planted error at its size (CPU only)."""
import numpy as np

import oracle as orc
import oracle_pool
from long_context_prefill_rr_b200 import workloads as wl

W = wl.WORKLOADS["tiny"].with_(heads_q=4, heads_kv=2, shift=3)
SCALE = 1.0 / np.sqrt(W.head_dim)


def _bits():
    return wl.make_workload(W)


def test_masses_full_equals_oracle_estimate():
    qb, kb, _ = _bits()
    full = oracle_pool.masses_full(qb, kb, W.batch, W.heads_q, W.heads_kv, W.seqlen, W.block,
                                   W.stride, W.shift, SCALE, workers=2)
    ref = orc.estimate(wl.bf16_bits_to_f64(qb), wl.bf16_bits_to_f64(kb), W.block, W.stride,
                       W.shift, SCALE)
    assert sorted(full) == [(0, h) for h in range(W.heads_q)]
    for (b, h), a in full.items():
        np.testing.assert_array_equal(a, ref[b, h])


def test_xattn_masses_full_equals_oracle_xattn():
    qb, kb, _ = _bits()
    full = oracle_pool.xattn_masses_full(qb, kb, W.batch, W.heads_q, W.heads_kv, W.seqlen,
                                         W.block, W.stride, SCALE, workers=2)
    ref = orc.xattn_estimate(wl.bf16_bits_to_f64(qb), wl.bf16_bits_to_f64(kb), W.block,
                             W.stride, SCALE)
    for (b, h), a in full.items():
        np.testing.assert_array_equal(a, ref[b, h])


def test_attention_errors_full_reports_a_planted_error():
    qb, kb, vb = _bits()
    q, k, v = (wl.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    nb = W.seqlen // W.block
    idx, cnt = orc.select(orc.estimate(q, k, W.block, W.stride, W.shift, SCALE), nb, W.tau)
    ref = orc.sparse_attention(q, k, v, idx, cnt, W.block, SCALE)
    out = ref.astype(np.float32)
    ma, rr, n = oracle_pool.attention_errors_full(qb, kb, vb, out, idx, cnt, W.heads_q,
                                                  W.heads_kv, W.block, SCALE, workers=2)
    assert n == W.heads_q * nb and ma < 1e-6 and rr < 1e-7
    out[0, 2, 300, 5] += 0.25
    ma, rr, _ = oracle_pool.attention_errors_full(qb, kb, vb, out, idx, cnt, W.heads_q,
                                                  W.heads_kv, W.block, SCALE, workers=1)
    assert abs(ma - 0.25) < 1e-6 and rr > 0
