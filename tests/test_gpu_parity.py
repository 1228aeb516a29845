"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on seeded inputs.

Every workload is compared at its full size on every block mass, every kept list and every
attention output row: the Tiny variants, the Llama-like layer at 8K, at 32K over the whole sweep
S in {8, 16} x tau in {0.9, 0.95}, and at 128K, and the video-like layer at 64K. The oracle runs
one head per task on a pool of spawned processes for the long workloads. The GPU's select must
also equal the oracle's select run on the GPU's own masses, over every row. Each check appends
a record (rows checked, errors, boundary-excused rows) to the session's parity report.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import parity as par
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _prepare(w):
    qb, kb, vb = wl.make_workload(w)
    return (qb, kb, vb), (par.to_dev(qb), par.to_dev(kb), par.to_dev(vb))


def test_tiny_full_parity(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["tiny"])
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    par.full_check(w, p, bits, gpu, "tiny")


@pytest.mark.parametrize("label,over", [
    ("s4_shift3_tau0.8", dict(stride=4, shift=3, tau=0.8)),
    ("s16_shiftm1_scale", dict(stride=16, shift=-1, tau=0.95, softmax_scale=0.125)),
    ("s32_default_scale", dict(stride=32, shift=5, tau=0.5, softmax_scale=-1.0)),
    ("gqa4_d128_ragged", dict(heads_q=8, heads_kv=2, head_dim=128, seqlen=1152, stride=8)),
    ("batch2_short", dict(batch=2, seqlen=768, stride=16, heads_q=4, heads_kv=4)),
    ("one_block", dict(seqlen=128, stride=8)),
])
def test_tiny_variants_full_parity(cuda_device, label, over):
    w, p = par.workload_params(wl.WORKLOADS["tiny"], **over)
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    par.full_check(w, p, bits, gpu, label)


def test_tau_one_is_dense_causal(cuda_device):
    """tau = 1 keeps every causal block and the output is dense causal attention."""
    w, p = par.workload_params(wl.WORKLOADS["tiny"], tau=1.0, heads_q=8, heads_kv=2,
                               head_dim=128)
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    nb = w.seqlen // w.block
    assert (gpu["cnt"] == np.arange(1, nb + 1)[None, None, :]).all()
    q64, k64, v64 = (wl.bf16_bits_to_f64(x) for x in bits)
    qt = torch.from_numpy(q64)
    kt = torch.from_numpy(k64).repeat_interleave(4, dim=1)
    vt = torch.from_numpy(v64).repeat_interleave(4, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                           scale=1.0).numpy()
    ma, rr = par.attention_errors(gpu["out"], ref)
    assert ma <= par.ATTN_MAX_ABS and rr <= par.ATTN_REL_RMS, (ma, rr)


def test_attention_rescale_divergent_rows(cuda_device):
    """Rows whose running max jumps by far more than the lazy-rescale threshold in a later
    block (only every other query row, so the rescale decision differs across a warp) still
    match the oracle."""
    w, p = par.workload_params(wl.WORKLOADS["tiny"], heads_q=4, heads_kv=2, head_dim=128,
                               seqlen=1024)
    qb, kb, vb = wl.make_workload(w)
    q = wl.bf16_bits_to_f32(qb)
    k = wl.bf16_bits_to_f32(kb)
    u = np.zeros(w.head_dim, np.float32)
    u[7] = 1.0
    q[:, :, ::2, :] += 4.0 * u                  # even query rows lean along u
    k[:, :, 3 * 128:4 * 128, :] += 5.0 * u      # keys of block 3 point along u: +20 logit jump
    qb, kb = wl.bf16_round_bits(q), wl.bf16_round_bits(k)
    nb = w.seqlen // w.block
    idx, cnt = wl.random_kept_lists(1, 4, nb, 1.0, seed=0)
    dev = [par.to_dev(x) for x in (qb, kb, vb)]
    out = torch.empty_like(dev[0])
    ws = native.new_workspace(p)
    native.sparse_attn(p, *dev, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), out,
                       ws)
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    q64, k64, v64 = (wl.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref = orc.sparse_attention(q64, k64, v64, idx, cnt, w.block, 1.0)
    ma, rr = par.attention_errors(par.bf16_dev_to_f32(out), ref)
    assert ma <= par.ATTN_MAX_ABS and rr <= par.ATTN_REL_RMS, (ma, rr)


@pytest.mark.parametrize("density,d", [(0.5, 128), (0.15, 128), (0.3, 64)])
def test_sparse_attn_random_masks(cuda_device, density, d):
    """rra_sparse_attn on caller-supplied random masks, including a row without its diagonal
    and an empty row, against the oracle."""
    w, p = par.workload_params(wl.WORKLOADS["tiny"], heads_q=8, heads_kv=2, head_dim=d,
                               seqlen=2048)
    bits, dev = _prepare(w)
    nb = w.seqlen // w.block
    idx, cnt = wl.random_kept_lists(1, 8, nb, density, seed=11)
    off = orc.tri_offset(5)
    idx[0, 3, off:off + 6] = [0, 2, -1, -1, -1, -1]   # no diagonal
    cnt[0, 3, 5] = 2
    off = orc.tri_offset(9)
    idx[0, 6, off:off + 10] = -1                      # empty row
    cnt[0, 6, 9] = 0
    out = torch.empty_like(dev[0])
    ws = native.new_workspace(p)
    native.sparse_attn(p, *dev, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), out,
                       ws)
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    q64, k64, v64 = (wl.bf16_bits_to_f64(x) for x in bits)
    ref = orc.sparse_attention(q64, k64, v64, idx, cnt, w.block, 1.0)
    ma, rr = par.attention_errors(par.bf16_dev_to_f32(out), ref)
    assert ma <= par.ATTN_MAX_ABS and rr <= par.ATTN_REL_RMS, (ma, rr)
    o = par.bf16_dev_to_f32(out)
    assert (o[0, 6, 9 * 128:10 * 128] == 0).all()


def test_invalid_list_entries_are_skipped_and_flagged(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["tiny"], heads_q=2, heads_kv=2)
    bits, dev = _prepare(w)
    nb = w.seqlen // w.block
    idx, cnt = wl.random_kept_lists(1, 2, nb, 1.0, seed=3)
    off = orc.tri_offset(4)
    idx[0, 1, off:off + 5] = [1, 0, 3, 9, 4]   # 0 not ascending, 9 > I: both skipped
    cnt[0, 1, 4] = 5
    out = torch.empty_like(dev[0])
    ws = native.new_workspace(p)
    native.sparse_attn(p, *dev, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), out,
                       ws)
    st, raw = native.check_device_status(ws)
    assert st == 1 and raw == 2
    st2, raw2 = native.check_device_status(ws)
    assert st2 == 0 and raw2 == 0                   # cleared by the first read
    idx[0, 1, off:off + 5] = [1, 3, 4, -1, -1]      # the valid subsequence
    cnt[0, 1, 4] = 3
    q64, k64, v64 = (wl.bf16_bits_to_f64(x) for x in bits)
    ref = orc.sparse_attention(q64, k64, v64, idx, cnt, w.block, 1.0)
    ma, rr = par.attention_errors(par.bf16_dev_to_f32(out), ref)
    assert ma <= par.ATTN_MAX_ABS and rr <= par.ATTN_REL_RMS, (ma, rr)


def test_select_edge_cases(cuda_device):
    """All-zero rows, exact ties, a single dominant block and tau = 1, on rra_select alone,
    against the oracle's select on the same fp32 masses."""
    p = native.params(1, 4, 4, 1024, 64, 8, 0.9)
    nb = 8
    T = orc.tri_offset(nb)
    rng = np.random.default_rng(5)
    m = rng.random((1, 4, T)).astype(np.float32)
    m[0, 0] = 0.0                                            # head 0: all zero
    m[0, 1] = 0.25                                           # head 1: all tied
    m[0, 2] = 1e-6
    for I in range(nb):
        m[0, 2, orc.tri_offset(I)] = 1.0                     # head 2: dominant J = 0
    for tau in (0.9, 0.5, 1.0):
        p.tau = tau
        md = torch.from_numpy(m).cuda()
        idx = torch.empty((1, 4, T), dtype=torch.int32, device="cuda")
        cnt = torch.empty((1, 4, nb), dtype=torch.int32, device="cuda")
        native.select(p, md, idx, cnt)
        ri, rc = orc.select(m.astype(np.float64), nb, float(np.float32(tau)))
        assert np.array_equal(idx.cpu().numpy(), ri) and np.array_equal(cnt.cpu().numpy(), rc)


def test_empty_problem(cuda_device):
    p = native.params(0, 8, 8, 1024, 64, 8, 0.9)
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    assert native.load().rra_prefill(native._p(p), *([native._ptr(z)] * 8), 16,
                                     native._stream(None)) == 0


def test_llama8k_parity(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["llama8k"])
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    par.long_check(w, p, bits, gpu, "llama8k", attn_rows="all", seed=1)


@pytest.mark.parametrize("S,tau", [(8, 0.9), (8, 0.95), (16, 0.9), (16, 0.95)])
def test_llama32k_parity(cuda_device, S, tau):
    w, p = par.workload_params(wl.WORKLOADS["llama32k"], stride=S, tau=tau)
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    del dev
    par.long_check(w, p, bits, gpu, f"llama32k_S{S}_tau{tau}", attn_rows="all", seed=2)


@pytest.mark.parametrize("label,base,over", [
    # d = 64: the attention's 10-stage ring and the estimate's 64-wide tiles at length
    ("llama8k_d64", "llama8k", dict(head_dim=64)),
    # the widest and the narrowest stride: m = 4 and m = 32 sampled rows per block row
    ("llama16k_s32", "llama32k", dict(seqlen=16384, stride=32)),
    ("llama16k_s4_shift7", "llama32k", dict(seqlen=16384, stride=4, shift=7)),
    # two batch rows at length
    ("llama8k_b2", "llama8k", dict(batch=2)),
])
def test_long_variants_parity(cuda_device, label, base, over):
    w, p = par.workload_params(wl.WORKLOADS[base], **over)
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    par.long_check(w, p, bits, gpu, label, attn_rows="all", seed=5)


def test_video64k_parity(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["video64k"])
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    del dev
    par.long_check(w, p, bits, gpu, "video64k", attn_rows="all", seed=4)


def test_llama128k_parity(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["llama128k"])
    bits, dev = _prepare(w)
    gpu = par.run_prefill(p, *dev)
    del dev
    torch.cuda.empty_cache()
    par.long_check(w, p, bits, gpu, "llama128k", attn_rows="all", seed=3)


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("tiny", dict(stride=4, tau=0.5, heads_q=8, heads_kv=2, head_dim=128, seqlen=1152)),
    ("tiny", dict(stride=32, tau=1.0)),
    ("llama8k", {}),
    ("llama32k", dict(stride=16, tau=0.95)),
])
def test_estimate_select_equals_estimate_then_select(cuda_device, name, over):
    """rra_estimate_select (steps 1 and 2 in one call) gives the masses and kept lists of
    rra_estimate followed by rra_select, bit for bit, with the masses in a caller buffer or kept
    in the workspace."""
    w, p = par.workload_params(wl.WORKLOADS[name], **over)
    bits, (q, k, _) = _prepare(w)
    sh = native.shapes(p)
    m1 = torch.empty(sh["mass"], dtype=torch.float32, device="cuda")
    i1 = torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda")
    c1 = torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda")
    ws = native.new_workspace(p)
    native.estimate(p, q, k, m1, ws)
    native.select(p, m1, i1, c1)
    m2, i2, c2 = torch.empty_like(m1), torch.full_like(i1, 7), torch.full_like(c1, 7)
    native.estimate_select(p, q, k, i2, c2, ws, mass=m2)
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    assert torch.equal(m1, m2) and torch.equal(i1, i2) and torch.equal(c1, c2)
    i3, c3 = torch.full_like(i1, 7), torch.full_like(c1, 7)
    native.estimate_select(p, q, k, i3, c3, ws)          # masses kept in the workspace
    assert torch.equal(i1, i3) and torch.equal(c1, c3)
