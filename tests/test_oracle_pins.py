"""Pins of the fp64 oracle against facts fixed outside it.

Each test ties one oracle step to something it does not compute itself: a library routine
(torch scaled-dot-product attention and softmax in fp64) on a special case the method reduces
to, a closed form, an invariant the RRAttention pages state (query independence, coverage when
heads >= stride), or brute force over every subset on tiny rows. Together they are chosen so
that a dropped term, a wrong sign, index, offset or GQA mapping, a transposed operand, a mean
taken for a sum, or a wrong causal edge fails at least one of them.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle as orc
from long_context_prefill_rr_b200 import workloads as wl


def _rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def _sdpa(q, k, v, scale, mask=None, causal=False):
    t = [torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)) for x in (q, k, v)]
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(
        *t, attn_mask=m, is_causal=causal, scale=scale, enable_gqa=True).numpy()


def _unpack_rows(packed, nb):
    """packed [T] -> dense lower-triangular [nb, nb]."""
    out = np.zeros((nb, nb))
    for I in range(nb):
        out[I, :I + 1] = packed[orc.tri_offset(I):orc.tri_offset(I + 1)]
    return out


# ---------------------------------------------------------------- step 8 (attention)

@pytest.mark.parametrize("b,hq,hkv,L,d,B", [(2, 4, 2, 256, 16, 32), (1, 8, 8, 1024, 64, 128)])
def test_tau1_keeps_all_and_equals_dense_causal(b, hq, hkv, L, d, B):
    """tau = 1 keeps every causal block, and the block-sparse output then equals dense causal
    attention computed by torch's fp64 scaled_dot_product_attention (GQA by repeat)."""
    q, k, v = _rand((b, hq, L, d), 1, 0.5), _rand((b, hkv, L, d), 2, 0.5), _rand((b, hkv, L, d), 3)
    nb = L // B
    mass = orc.estimate(q, k, B, 4, 1, 0.7)
    idx, cnt = orc.select(mass, nb, 1.0)
    assert (cnt == np.arange(1, nb + 1)[None, None, :]).all()
    o = orc.sparse_attention(q, k, v, idx, cnt, B, 0.7)
    ref = _sdpa(q, k, v, 0.7, causal=True)
    assert np.abs(o - ref).max() < 1e-12


def test_attention_arbitrary_mask_equals_masked_dense():
    """On a random block mask the output equals dense attention whose dropped blocks (and the
    causal upper triangle) are masked out, via torch's fp64 attention with a boolean mask.
    Queries whose row has no key at all (diagonal dropped from a caller's list) give 0."""
    b, hq, hkv, L, d, B = 1, 4, 2, 256, 16, 32
    nb = L // B
    q, k, v = _rand((b, hq, L, d), 4), _rand((b, hkv, L, d), 5), _rand((b, hkv, L, d), 6)
    idx, cnt = wl.random_kept_lists(b, hq, nb, 0.4, seed=7)
    # head 1, row 3: replace the list by {0} without the diagonal, so queries 96..127 keep
    # keys 0..31 and nothing else; and row 2 gets an empty list (every query keyless)
    off = orc.tri_offset(3)
    idx[0, 1, off:off + 4] = [0, -1, -1, -1]
    cnt[0, 1, 3] = 1
    off = orc.tri_offset(2)
    idx[0, 1, off:off + 3] = -1
    cnt[0, 1, 2] = 0
    o = orc.sparse_attention(q, k, v, idx, cnt, B, 0.25)
    for h in range(hq):
        allowed = np.zeros((L, L), dtype=bool)
        for I in range(nb):
            for J in idx[0, h, orc.tri_offset(I):orc.tri_offset(I) + cnt[0, h, I]]:
                allowed[I * B:(I + 1) * B, J * B:(J + 1) * B] = True
        allowed &= np.tril(np.ones((L, L), dtype=bool))
        ref = _sdpa(q[:, h:h + 1], k[:, h // 2:h // 2 + 1], v[:, h // 2:h // 2 + 1], 0.25,
                    mask=allowed)[0, 0]
        has = allowed.any(axis=1)
        assert np.abs(o[0, h][has] - ref[has]).max() < 1e-12
        assert (o[0, h][~has] == 0).all()


# ---------------------------------------------------------------- steps 3-6 (estimate)

@pytest.mark.parametrize("shift", [0, 3, -5])
def test_stride1_equals_exact_block_softmax_mass(shift):
    """With S = 1 every query is sampled, pooling is the identity and stride causality is
    token causality, so A_{I,J} must equal (1/B) x the exact block sums of the dense causal
    softmax probabilities (torch fp64 softmax), for any shift. GQA 4:2 checks the head map."""
    b, hq, hkv, L, d, B = 1, 4, 2, 256, 16, 32
    q, k = _rand((b, hq, L, d), 10, 0.4), _rand((b, hkv, L, d), 11, 0.4)
    scale = 0.9
    A = orc.estimate(q, k, B, 1, shift, scale)
    nb = L // B
    kt = torch.from_numpy(k).repeat_interleave(hq // hkv, dim=1)
    s = scale * torch.from_numpy(q) @ kt.transpose(-1, -2)
    s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
    p = torch.softmax(s, dim=-1).numpy()
    exact = p.reshape(b, hq, nb, B, nb, B).sum(axis=(3, 5)) / B
    for h in range(hq):
        assert np.abs(_unpack_rows(A[0, h], nb) - exact[0, h]).max() < 1e-12


@pytest.mark.parametrize("S", [2, 4, 8])
def test_zero_keys_closed_form(S):
    """K = 0 makes every stride logit equal, so P_{i,j} = 1/(i+1) on j <= i and
    A_{I,J} = (1/m) sum_{i in I} #{j in J : j <= i} / (i + 1) with m = B/S."""
    b, hq, hkv, L, d, B = 1, 2, 1, 128, 8, 16
    q = _rand((b, hq, L, d), 12)
    k = np.zeros((b, hkv, L, d))
    A = orc.estimate(q, k, B, S, 0, 1.0)
    m, nb = B // S, L // B
    for h in range(hq):
        got = _unpack_rows(A[0, h], nb)
        for I in range(nb):
            for J in range(I + 1):
                want = sum(sum(1 for j in range(J * m, J * m + m) if j <= i) / (i + 1)
                           for i in range(I * m, I * m + m)) / m
                assert abs(got[I, J] - want) < 1e-14


@pytest.mark.parametrize("S", [2, 4])
def test_stride_constant_keys_give_summed_logits(S):
    """Keys constant inside every stride (K[jS+t] = c_j) make the pooled key S*c_j, so the
    stride logits are scale*S*q_hat.c_j (a sum, not a mean, and no extra 1/S); the masses are
    then the block sums of torch's causal softmax of exactly those logits."""
    b, hq, hkv, L, d, B, shift, scale = 1, 3, 1, 64, 8, 16, 1, 0.3
    q = _rand((b, hq, L, d), 13)
    c = _rand((b, hkv, L // S, d), 14)
    k = np.repeat(c, S, axis=2)
    A = orc.estimate(q, k, B, S, shift, scale)
    m, nb, ns = B // S, L // B, L // S
    for h in range(hq):
        o = (h + shift) % S
        z = torch.from_numpy(scale * S * q[0, h, o::S] @ c[0, 0].T)
        z = z.masked_fill(~torch.ones(ns, ns, dtype=torch.bool).tril(), float("-inf"))
        p = torch.softmax(z, dim=-1).numpy()
        want = p.reshape(nb, m, nb, m).sum(axis=(1, 3)) / m
        assert np.abs(_unpack_rows(A[0, h], nb) - want).max() < 1e-12


def test_rows_sum_to_one_and_dominant_key():
    """Every block row of A sums to 1; a key far more aligned with every query than the rest
    (placed at position 0) drives A_{I,0} to 1 for every row."""
    b, hq, hkv, L, d, B, S = 1, 4, 2, 512, 16, 64, 8
    q, k = _rand((b, hq, L, d), 15, 0.3), _rand((b, hkv, L, d), 16, 0.3)
    A = orc.estimate(q, k, B, S, 2, 1.0)
    nb = L // B
    for h in range(hq):
        rows = _unpack_rows(A[0, h], nb)
        assert np.abs(rows.sum(axis=1) - 1).max() < 1e-12
    u = np.zeros(d)
    u[3] = 1.0                       # a shared query direction; key 0 points along it
    k2 = k.copy()
    k2[:, :, 0, :] += 50.0 * u
    q2 = q + 3.0 * u
    A2 = orc.estimate(q2, k2, B, S, 2, 1.0)
    for h in range(hq):
        rows = _unpack_rows(A2[0, h], nb)
        assert rows[:, 0].min() > 0.999


def test_query_independence_and_offsets():
    """Head h's masses depend on Q only through positions i*S + (h+shift) mod S: perturbing
    any other query row leaves them bit-identical, perturbing a sampled row changes them."""
    b, hq, hkv, L, d, B, S, shift = 1, 4, 2, 256, 8, 32, 8, 5
    q, k = _rand((b, hq, L, d), 17), _rand((b, hkv, L, d), 18)
    A = orc.estimate(q, k, B, S, shift, 0.5)
    for h in range(hq):
        o = (h + shift) % S
        unsampled = [t for t in range(L) if t % S != o]
        q2 = q.copy()
        q2[0, h, unsampled] += _rand((len(unsampled), d), 19 + h)
        A2 = orc.estimate(q2, k, B, S, shift, 0.5)
        assert np.array_equal(A2[0, h], A[0, h])
        q3 = q.copy()
        q3[0, h, 5 * S + o] += 1.0
        A3 = orc.estimate(q3, k, B, S, shift, 0.5)
        assert not np.array_equal(A3[0, h], A[0, h])


@pytest.mark.parametrize("H,S,shift", [(8, 8, 0), (28, 16, 3), (32, 8, -1), (4, 8, 2), (6, 16, 0)])
def test_coverage_iff_heads_at_least_stride(H, S, shift):
    """The heads together cover every in-stride position exactly when H >= S; with H < S
    exactly H distinct positions are covered (the limitation the pages report)."""
    offs = {orc.rr_offset(h, S, shift) for h in range(H)}
    if H >= S:
        assert offs == set(range(S))
    else:
        assert len(offs) == H and offs <= set(range(S))


# ---------------------------------------------------------------- step 7 (select)

def test_select_hand_examples():
    """find_blocks by hand on one row I = 3 with masses [0.1, 0.5, 0.15, 0.25]:
    tau 0.7: descending 0.5 (J1), 0.25 (J3) -> 0.75 >= 0.7, prefix {1,3}, diagonal 3 present.
    tau 0.8: add 0.15 (J2) -> 0.9, kept {1,2,3}.   tau 0.4: {1} then diagonal -> {1,3}.
    tau 1.0: every causal block. Ties: [0.3, 0.3, 0.4] at tau 0.6 keeps J2 then J0 (lower J
    first among equals) -> {0, 2}. Equality counts as reaching tau: [0.25, 0.25, 0.5] at
    tau 0.75 -> {0, 2}."""
    a = np.array([0.1, 0.5, 0.15, 0.25])
    assert orc.select_row(a, 3, 0.7).tolist() == [1, 3]
    assert orc.select_row(a, 3, 0.8).tolist() == [1, 2, 3]
    assert orc.select_row(a, 3, 0.4).tolist() == [1, 3]
    assert orc.select_row(a, 3, 1.0).tolist() == [0, 1, 2, 3]
    assert orc.select_row(np.array([0.3, 0.3, 0.4]), 2, 0.6).tolist() == [0, 2]
    # inclusive comparison: 0.5 + 0.25 reaches 0.75 exactly (all binary fractions)
    assert orc.select_row(np.array([0.25, 0.25, 0.5]), 2, 0.75).tolist() == [0, 2]


def test_select_is_minimum_cardinality_by_brute_force():
    """On the tiny workload (8 block rows) the greedy prefix has the minimum size of ANY block
    set whose mass reaches tau * row total (checked over every subset), it reaches that mass,
    and dropping its smallest member falls below it; the kept set is the prefix plus the
    diagonal."""
    q, k, _ = wl.make_workload("tiny")
    q, k = wl.bf16_bits_to_f64(q), wl.bf16_bits_to_f64(k)
    w = wl.WORKLOADS["tiny"]
    nb = w.seqlen // w.block
    A = orc.estimate(q[:, :4], k[:, :4], w.block, w.stride, w.shift, 1.0)
    for tau in (0.5, 0.9, 0.97):
        for h in range(4):
            for I in range(nb):
                a = A[0, h, orc.tri_offset(I):orc.tri_offset(I + 1)]
                total = a.sum()
                best = min(len(c) for r in range(1, I + 2)
                           for c in itertools.combinations(range(I + 1), r)
                           if sum(a[list(c)]) >= tau * total)
                kept = orc.select_row(a, I, tau)
                order = np.argsort(-a, kind="stable")
                prefix = order[:best]
                assert set(kept.tolist()) == set(prefix.tolist()) | {I}
                assert a[prefix].sum() >= tau * total
                assert a[prefix[:-1]].sum() < tau * total


def test_select_tau_one_and_layout():
    idx, cnt = orc.select(np.random.default_rng(0).random((1, 2, orc.tri_offset(5))), 5, 1.0)
    assert (cnt == np.arange(1, 6)).all()
    for I in range(5):
        assert idx[0, 0, orc.tri_offset(I):orc.tri_offset(I + 1)].tolist() == list(range(I + 1))
    idx, cnt = orc.select(np.random.default_rng(1).random((1, 2, orc.tri_offset(6))), 6, 0.5)
    for h in range(2):
        for I in range(6):
            row = idx[0, h, orc.tri_offset(I):orc.tri_offset(I + 1)]
            n = cnt[0, h, I]
            assert (np.diff(row[:n]) > 0).all() and row[n - 1] == I and (row[n:] == -1).all()


# ---------------------------------------------------------------- XAttention antidiagonal estimator

def test_xattn_stride1_equals_exact_block_softmax_mass():
    """At S = 1 the antidiagonal of a 1x1 sub-block is the logit itself: the XAttention masses
    equal the exact block sums of the dense causal softmax (torch fp64), GQA 4:2."""
    b, hq, hkv, L, d, B = 1, 4, 2, 256, 16, 32
    q, k = _rand((b, hq, L, d), 30, 0.4), _rand((b, hkv, L, d), 31, 0.4)
    A = orc.xattn_estimate(q, k, B, 1, 0.8)
    nb = L // B
    kt = torch.from_numpy(k).repeat_interleave(hq // hkv, dim=1)
    s = 0.8 * torch.from_numpy(q) @ kt.transpose(-1, -2)
    s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
    exact = torch.softmax(s, dim=-1).numpy().reshape(b, hq, nb, B, nb, B).sum(axis=(3, 5)) / B
    for h in range(hq):
        assert np.abs(_unpack_rows(A[0, h], nb) - exact[0, h]).max() < 1e-12


def test_xattn_stride_constant_queries_reduce_to_pooled_keys():
    """Queries constant inside every stride (Q[iS+t] = c_i) turn the antidiagonal sum into
    c_i . sum_t K[jS+t]: the masses are the block sums of torch's causal softmax of
    scale * c_i . Kbar_j."""
    b, hq, hkv, L, d, B, S, scale = 1, 2, 1, 64, 8, 16, 4, 0.3
    c = _rand((b, hq, L // S, d), 32)
    q = np.repeat(c, S, axis=2)
    k = _rand((b, hkv, L, d), 33)
    A = orc.xattn_estimate(q, k, B, S, scale)
    m, nb, ns = B // S, L // B, L // S
    kbar = k[0, 0].reshape(ns, S, d).sum(axis=1)
    for h in range(hq):
        z = torch.from_numpy(scale * c[0, h] @ kbar.T)
        z = z.masked_fill(~torch.ones(ns, ns, dtype=torch.bool).tril(), float("-inf"))
        want = torch.softmax(z, dim=-1).numpy().reshape(nb, m, nb, m).sum(axis=(1, 3)) / m
        assert np.abs(_unpack_rows(A[0, h], nb) - want).max() < 1e-12


def test_xattn_direction_is_the_antidiagonal():
    """Only in-stride query offset 0 carries a query vector and only in-stride key offset S-1
    carries a key vector, so only the antidiagonal pairing (t, S-1-t) = (0, S-1) sees them:
    the masses equal the block sums of torch's softmax of scale * Q[iS] . K[jS+S-1]; the main
    diagonal pairing (t, t) would see zeros everywhere (uniform masses)."""
    b, hq, hkv, L, d, B, S, scale = 1, 1, 1, 64, 8, 16, 4, 1.0
    q = np.zeros((b, hq, L, d))
    k = np.zeros((b, hkv, L, d))
    q[0, 0, 0::S] = _rand((L // S, d), 34)
    k[0, 0, S - 1::S] = _rand((L // S, d), 35)
    A = orc.xattn_estimate(q, k, B, S, scale)
    m, nb, ns = B // S, L // B, L // S
    z = torch.from_numpy(scale * q[0, 0, 0::S] @ k[0, 0, S - 1::S].T)
    z = z.masked_fill(~torch.ones(ns, ns, dtype=torch.bool).tril(), float("-inf"))
    want = torch.softmax(z, dim=-1).numpy().reshape(nb, m, nb, m).sum(axis=(1, 3)) / m
    assert np.abs(_unpack_rows(A[0, 0], nb) - want).max() < 1e-12
