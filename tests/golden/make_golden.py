"""Write tests/golden/tiny_oracle.json from the fp64 oracle alone.

The fixture freezes the oracle's masses, kept lists, a few attention outputs and the XAttention
estimator's masses on the seeded tiny workload (8 heads, d 64, L 1024, B 128, S 8, shift 0, tau 0.9, scale 1), so that a later
change to the oracle's arithmetic shows up as a diff of this file. Inputs come from the seeded
generator; every stored value comes from ``oracle``.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))


import oracle as orc  # noqa: E402
from long_context_prefill_rr_b200 import workloads as wl  # noqa: E402

SAMPLE_ROWS = [(0, 0, 0), (0, 3, 5), (0, 7, 7)]   # (b, h, query block I)
SAMPLE_T = [0, 1, 63, 127]                          # query offsets inside the block


def main():
    w = wl.WORKLOADS["tiny"]
    q, k, v = (wl.bf16_bits_to_f64(x) for x in wl.make_workload(w))
    nb = w.seqlen // w.block
    mass = orc.estimate(q, k, w.block, w.stride, w.shift, w.softmax_scale)
    idx, cnt = orc.select(mass, nb, w.tau)
    o = orc.sparse_attention(q, k, v, idx, cnt, w.block, w.softmax_scale, rows=SAMPLE_ROWS)
    xa = orc.xattn_estimate(q, k, w.block, w.stride, w.softmax_scale)
    out = {
        "source": "oracle (fp64) on the seeded tiny workload; written by make_golden.py",
        "workload": w.name, "block": w.block, "stride": w.stride, "shift": w.shift,
        "tau": w.tau, "softmax_scale": w.softmax_scale,
        "mass": [[float(x) for x in mass[0, h]] for h in range(w.heads_q)],
        "kept_cnt": cnt[0].tolist(),
        "kept_idx": idx[0].tolist(),
        "xattn_mass": [[float(x) for x in xa[0, h]] for h in range(w.heads_q)],
        "attn_samples": [
            {"b": b, "h": h, "I": I, "t": t, "o_first8": [float(x) for x in o[b, h, I * w.block + t, :8]]}
            for (b, h, I) in SAMPLE_ROWS for t in SAMPLE_T],
    }
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(out, f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main()
