"""Head-sharded layers on the GPU: each shard of a layer, run through the C ABI with its own
head counts and shifted round-robin shift, gives exactly (bit for bit) the masses, kept lists
and attention output the whole-layer run gives for those heads. The shards run one after another
on one device, as W ranks would each run theirs."""
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
def test_shards_reproduce_the_whole_layer(cuda_device, name, world):
    w, p = par.workload_params(CASES[name])
    qb, kb, vb = wl.make_workload(w)
    full = par.run_prefill(p, par.to_dev(qb), par.to_dev(kb), par.to_dev(vb))
    assert full["status"] == 0, full["raw"]
    for r in range(world):
        ps, s = sharding.shard_params(p, r, world)
        part = par.run_prefill(ps, par.to_dev(sharding.take_heads(qb, s.q0, s.q1)),
                               par.to_dev(sharding.take_heads(kb, s.kv0, s.kv1)),
                               par.to_dev(sharding.take_heads(vb, s.kv0, s.kv1)))
        assert part["status"] == 0, part["raw"]
        for key in ("mass", "idx", "cnt", "out"):
            assert np.array_equal(part[key], full[key][:, s.q0:s.q1]), (name, world, r, key)
