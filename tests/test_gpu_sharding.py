"""Head-sharded layers on the GPU. Each shard of a layer runs through the C ABI with its own head
counts and the round-robin shift advanced by its first query head (the offset rotates across
heads: RRAttention abstract, "rotating query sampling positions across attention heads within
each stride"). The shards run one after another on one device, as W ranks would each run
theirs. Their outputs, put back at their global head positions, are compared with the fp64
oracle run on the GLOBAL heads and shift (every mass, kept list and output row), and must equal
the whole-layer run bit for bit."""
import numpy as np
import pytest

import parity as par
from long_context_prefill_rr_b200 import sharding
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_gqa": wl.WORKLOADS["tiny"].with_(heads_kv=4, shift=5),
    "llama8k": wl.WORKLOADS["llama8k"].with_(shift=3),
    "video_short": wl.WORKLOADS["video64k"].with_(seqlen=8192),
}


@pytest.mark.parametrize("name,world", [("tiny_gqa", 2), ("tiny_gqa", 4), ("llama8k", 2),
                                        ("llama8k", 8), ("video_short", 4)])
def test_shards_match_the_oracle_and_the_whole_layer(cuda_device, name, world):
    w, p = par.workload_params(CASES[name])
    qb, kb, vb = wl.make_workload(w)
    full = par.run_prefill(p, par.to_dev(qb), par.to_dev(kb), par.to_dev(vb))
    assert full["status"] == 0, full["raw"]
    joined = {key: np.zeros_like(full[key]) for key in ("mass", "idx", "cnt", "out")}
    for r in range(world):
        ps, s = sharding.shard_params(p, r, world)
        part = par.run_prefill(ps, par.to_dev(sharding.take_heads(qb, s.q0, s.q1)),
                               par.to_dev(sharding.take_heads(kb, s.kv0, s.kv1)),
                               par.to_dev(sharding.take_heads(vb, s.kv0, s.kv1)))
        assert part["status"] == 0, part["raw"]
        for key in joined:
            joined[key][:, s.q0:s.q1] = part[key]
    joined["status"], joined["raw"] = 0, 0
    label = f"shards_{name}_w{world}"
    if name == "tiny_gqa":
        par.full_check(w, p, (qb, kb, vb), joined, label)
    else:
        par.long_check(w, p, (qb, kb, vb), joined, label, attn_rows="all", seed=world)
    for key in ("mass", "idx", "cnt", "out"):
        assert np.array_equal(joined[key], full[key]), (name, world, key)
