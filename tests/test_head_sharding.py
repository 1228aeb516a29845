"""Head-sharded layers (CPU): the partition, the shard's round-robin shift, and that the oracle
run shard by shard reproduces the whole layer exactly; one gloo world of two ranks runs the
shards as separate processes and gathers them."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as orc
from long_context_prefill_rr_b200 import sharding
from long_context_prefill_rr_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GQA_TINY = wl.WORKLOADS["tiny"].with_(heads_kv=4, seqlen=512, shift=5)


@pytest.mark.parametrize("hq,hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8),
                                          (28, 4, 2), (28, 4, 4), (8, 8, 8), (8, 4, 2)])
def test_partition_covers_each_head_once_with_whole_groups(hq, hkv, world):
    g = hq // hkv
    shards = [sharding.head_shard(hq, hkv, 8, 0, r, world) for r in range(world)]
    assert shards[0].q0 == 0 and shards[-1].q1 == hq and shards[-1].kv1 == hkv
    for a, b in zip(shards, shards[1:]):
        assert a.q1 == b.q0 and a.kv1 == b.kv0
    for s in shards:
        assert s.heads_q == g * s.heads_kv and s.heads_kv == hkv // world
        for h in range(s.q0, s.q1):
            assert s.kv0 <= orc.kv_head(h, hq, hkv) < s.kv1
            # the local GQA mapping of the shard lands on the same KV head
            assert orc.kv_head(h - s.q0, s.heads_q, s.heads_kv) + s.kv0 == orc.kv_head(h, hq, hkv)


@pytest.mark.parametrize("stride,shift", [(8, 0), (8, 5), (16, -3), (4, 1001)])
def test_shard_shift_keeps_global_round_robin_offsets(stride, shift):
    hq, hkv = 32, 8
    for world in (2, 4, 8):
        for r in range(world):
            s = sharding.head_shard(hq, hkv, stride, shift, r, world)
            assert 0 <= s.shift < stride
            for i in range(s.heads_q):
                assert orc.rr_offset(i, stride, s.shift) == orc.rr_offset(s.q0 + i, stride, shift)


def test_invalid_partitions_are_refused():
    with pytest.raises(ValueError):
        sharding.head_shard(32, 8, 8, 0, 0, 3)          # 8 KV heads over 3 ranks
    with pytest.raises(ValueError):
        sharding.head_shard(32, 8, 8, 0, 2, 2)          # rank outside the world
    with pytest.raises(ValueError):
        sharding.head_shard(30, 8, 8, 0, 0, 2)          # Hq not a multiple of Hkv
    with pytest.raises(ValueError):
        sharding.head_shard(32, 8, 0, 0, 0, 2)          # stride < 1


def _oracle_layer(w, q, k, v, shift):
    scale = w.softmax_scale if w.softmax_scale > 0 else 1.0 / np.sqrt(w.head_dim)
    nb = w.seqlen // w.block
    mass = orc.estimate(q, k, w.block, w.stride, shift, scale)
    idx, cnt = orc.select(mass, nb, w.tau)
    out = orc.sparse_attention(q, k, v, idx, cnt, w.block, scale)
    return mass, idx, cnt, out


def _inputs(w):
    qb, kb, vb = wl.make_workload(w)
    return wl.bf16_bits_to_f64(qb), wl.bf16_bits_to_f64(kb), wl.bf16_bits_to_f64(vb)


def _shard_layer(w, q, k, v, rank, world):
    s = sharding.head_shard(w.heads_q, w.heads_kv, w.stride, w.shift, rank, world)
    return _oracle_layer(w, sharding.take_heads(q, s.q0, s.q1), sharding.take_heads(k, s.kv0, s.kv1),
                         sharding.take_heads(v, s.kv0, s.kv1), s.shift)


@pytest.mark.parametrize("world", [2, 4])
def test_oracle_shards_reassemble_the_layer(world):
    w = GQA_TINY
    q, k, v = _inputs(w)
    full = _oracle_layer(w, q, k, v, w.shift)
    parts = [_shard_layer(w, q, k, v, r, world) for r in range(world)]
    for i in range(4):
        got = np.concatenate([p[i] for p in parts], axis=1)
        assert np.array_equal(got, full[i])
    # a shard run with the unshifted shift samples other queries: the masses move
    s1 = sharding.head_shard(w.heads_q, w.heads_kv, w.stride, w.shift, 1, world)
    wrong = orc.estimate(q[:, s1.q0:s1.q1], k[:, s1.kv0:s1.kv1], w.block, w.stride, w.shift,
                         w.softmax_scale)
    assert not np.array_equal(wrong, full[0][:, s1.q0:s1.q1])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", init_method="env://", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    w = GQA_TINY
    q, k, v = _inputs(w)
    mine = _shard_layer(w, q, k, v, rank, world)
    gathered = [None] * world
    dist.all_gather_object(gathered, mine)
    ok = None
    if rank == 0:
        full = _oracle_layer(w, q, k, v, w.shift)
        ok = all(np.array_equal(np.concatenate([g[i] for g in gathered], axis=1), full[i])
                 for i in range(4))
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, ok))


def test_two_gloo_ranks_each_run_their_heads():
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, qu)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(qu.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] is True
