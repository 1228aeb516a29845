"""Block-selection quality of the round-robin estimate against exact Top-tau (CPU, oracle).

The RRAttention summary page reports "higher precision and F1 for selecting important blocks".
Here the reference set is Top-tau on the EXACT block masses (the oracle's estimate at S = 1, which
the pins tie to the dense causal softmax), and the candidate set is Top-tau on the round-robin
masses at S in {4, 8, 16}. Per (head, block row): precision = |RR & exact| / |RR|, recall =
|RR & exact| / |exact|, F1 their harmonic mean, averaged over rows. The page also notes that
coverage of the in-stride positions fails when S exceeds the number of heads; the H < S case is
included (4 heads, S 8 and 16).

`python tests/test_selection_quality.py` prints the table recorded in the design notes.
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle as orc  # noqa: E402
from long_context_prefill_rr_b200 import workloads as wl  # noqa: E402


def selection_quality(q, k, block, stride, shift, scale, tau):
    """Mean (precision, recall, f1, rr_density, exact_density) over all (head, block row)."""
    b, hq, L, d = q.shape
    nb = L // block
    exact = orc.estimate(q, k, block, 1, 0, scale)
    rr = orc.estimate(q, k, block, stride, shift, scale)
    prec, rec, f1, n_rr, n_ex = [], [], [], 0, 0
    for bi in range(b):
        for h in range(hq):
            for I in range(nb):
                off = orc.tri_offset(I)
                se = set(orc.select_row(exact[bi, h, off:off + I + 1], I, tau).tolist())
                sr = set(orc.select_row(rr[bi, h, off:off + I + 1], I, tau).tolist())
                inter = len(se & sr)
                p_ = inter / len(sr)
                r_ = inter / len(se)
                prec.append(p_)
                rec.append(r_)
                f1.append(0.0 if p_ + r_ == 0 else 2 * p_ * r_ / (p_ + r_))
                n_rr += len(sr)
                n_ex += len(se)
    tot = b * hq * orc.tri_offset(nb)
    return (float(np.mean(prec)), float(np.mean(rec)), float(np.mean(f1)), n_rr / tot,
            n_ex / tot)


def _inputs(heads_q, heads_kv, seqlen):
    w = wl.WORKLOADS["llama8k"].with_(heads_q=heads_q, heads_kv=heads_kv, seqlen=seqlen)
    q, k, _ = wl.make_workload(w)
    return wl.bf16_bits_to_f64(q), wl.bf16_bits_to_f64(k)


def test_stride_one_is_exact():
    q, k = _inputs(4, 2, 1024)
    p_, r_, f_, dr, de = selection_quality(q, k, 128, 1, 0, 1.0, 0.9)
    assert p_ == r_ == f_ == 1.0 and dr == de


def test_quality_metrics_are_sane_on_the_llama_recipe():
    """RR at S = 8 on the Llama-like recipe: every kept set reaches tau of its own masses and
    contains the diagonal, so recall and precision are well above chance (a coarse floor, not
    a claim about the pages' numbers)."""
    q, k = _inputs(8, 2, 2048)
    p_, r_, f_, dr, de = selection_quality(q, k, 128, 8, 0, 1.0, 0.9)
    for v in (p_, r_, f_):
        assert 0.0 <= v <= 1.0
    assert f_ > 0.5 and 0.0 < dr <= 1.0 and 0.0 < de <= 1.0


def table(seqlen=4096):
    rows = []
    for heads_q, heads_kv in ((32, 8), (4, 1)):
        q, k = _inputs(heads_q, heads_kv, seqlen)
        for S in (4, 8, 16):
            for tau in (0.9, 0.95):
                p_, r_, f_, dr, de = selection_quality(q, k, 128, S, 0, 1.0, tau)
                rows.append((heads_q, S, tau, p_, r_, f_, dr, de))
    return rows


if __name__ == "__main__":
    print("| heads | S | tau | precision | recall | F1 | RR density | exact density |")
    print("|---|---|---|---|---|---|---|---|")
    for hq, S, tau, p_, r_, f_, dr, de in table():
        print(f"| {hq} | {S} | {tau} | {p_:.3f} | {r_:.3f} | {f_:.3f} | {dr:.3f} | {de:.3f} |")
