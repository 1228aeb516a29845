"""The seeded input generators (CPU): bf16 rounding equals torch's round-to-nearest-even
conversion, the draws do not depend on the thread count, the shapes follow the workload table,
and the planted structure is where the recipe puts it."""
import numpy as np
import torch

from long_context_prefill_rr_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
                                  3.3895314e38], dtype=np.float32)]).astype(np.float32)
    ours = wl.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = wl.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_draws_do_not_depend_on_the_thread_count(monkeypatch):
    w = wl.WORKLOADS["tiny"].with_(seqlen=512)
    a = wl.make_workload(w)
    monkeypatch.setattr(wl.os, "sched_getaffinity", lambda pid: {0})
    b = wl.make_workload(w)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_shapes_and_seeds():
    for name, w in wl.WORKLOADS.items():
        if w.seqlen > 8192:
            w = w.with_(seqlen=2048)
        q, k, v = wl.make_workload(w)
        assert q.shape == (w.batch, w.heads_q, w.seqlen, w.head_dim) and q.dtype == np.uint16
        assert k.shape == v.shape == (w.batch, w.heads_kv, w.seqlen, w.head_dim)
        assert q.flags.c_contiguous and k.flags.c_contiguous and v.flags.c_contiguous
    q1, _, _ = wl.make_workload(wl.WORKLOADS["llama8k"].with_(seqlen=1024))
    q2, _, _ = wl.make_workload(wl.WORKLOADS["llama8k"].with_(seqlen=1024, seed=7))
    assert not np.array_equal(q1, q2)


def test_planted_sink_is_aligned_with_the_mean_query():
    """Key 0 of every KV head carries +3 qbar, qbar the group's mean query direction at norm
    d^(1/4): its logit against the mean query is far above the other keys'."""
    w = wl.WORKLOADS["tiny"]
    q, k, _ = (wl.bf16_bits_to_f64(x) for x in wl.make_workload(w))
    g = w.heads_q // w.heads_kv
    for kv in range(w.heads_kv):
        qbar = q[0, kv * g:(kv + 1) * g].mean(axis=(0, 1))
        s = k[0, kv] @ qbar
        assert s[0] > s[1:].max()


def test_random_kept_lists_are_valid():
    idx, cnt = wl.random_kept_lists(2, 3, 9, 0.4, seed=1)
    nb = 9
    for b in range(2):
        for h in range(3):
            for I in range(nb):
                off = I * (I + 1) // 2
                row = idx[b, h, off:off + I + 1]
                n = int(cnt[b, h, I])
                assert 1 <= n <= I + 1
                kept = row[:n]
                assert np.all(np.diff(kept) > 0) and kept[0] >= 0 and kept[-1] <= I
                assert np.all(row[n:] == -1)
