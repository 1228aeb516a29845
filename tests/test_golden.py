"""The oracle still reproduces the frozen tiny fixture (tests/golden/tiny_oracle.json, written
by tests/golden/make_golden.py from the oracle alone); a change to the oracle's arithmetic
must regenerate it and say why."""
import json
import os

import numpy as np

import oracle as orc
from long_context_prefill_rr_b200 import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_oracle_matches_frozen_tiny_fixture():
    g = json.load(open(GOLD))
    w = wl.WORKLOADS[g["workload"]]
    q, k, v = (wl.bf16_bits_to_f64(x) for x in wl.make_workload(w))
    nb = w.seqlen // w.block
    mass = orc.estimate(q, k, g["block"], g["stride"], g["shift"], g["softmax_scale"])
    assert np.abs(mass[0] - np.array(g["mass"])).max() < 1e-12
    idx, cnt = orc.select(mass, nb, g["tau"])
    assert cnt[0].tolist() == g["kept_cnt"] and idx[0].tolist() == g["kept_idx"]
    rows = sorted({(s["b"], s["h"], s["I"]) for s in g["attn_samples"]})
    o = orc.sparse_attention(q, k, v, idx, cnt, g["block"], g["softmax_scale"], rows=rows)
    for s in g["attn_samples"]:
        got = o[s["b"], s["h"], s["I"] * g["block"] + s["t"], :8]
        assert np.abs(got - np.array(s["o_first8"])).max() < 1e-12
    xa = orc.xattn_estimate(q, k, g["block"], g["stride"], g["softmax_scale"])
    assert np.abs(xa[0] - np.array(g["xattn_mass"])).max() < 1e-12
