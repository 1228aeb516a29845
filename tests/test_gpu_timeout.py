"""Failure detection on the GPU without a GPU fault: a barrier wait that really expires.

Every barrier wait in the kernels is bounded in time. rra_set_wait_limit_ns cuts the bound to
1 microsecond, far below how long the estimate kernel's reduction warps wait for the first
(longest) work item of the 32K layer, so waits give up mid-kernel. The kernel must then drain the
copies and MMAs it has in flight, set the timeout bit in the workspace status word and return;
the attention kernel enqueued after it must see the bit and exit at once. The host reads
RRA_ERR_DEVICE_TIMEOUT, the read clears the word, and the next call on the same workspace, with
the default limit, gives exactly the results of a run on a fresh workspace (and the oracle's on
sampled rows): the context stays usable.
"""
import numpy as np
import pytest
import torch

import parity as par
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu

RRA_ERR_DEVICE_TIMEOUT = 5
SHORT_LIMIT_NS = 1000


def _buffers(p):
    sh = native.shapes(p)
    return dict(mass=torch.empty(sh["mass"], dtype=torch.float32, device="cuda"),
                idx=torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda"),
                cnt=torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda"),
                out=torch.zeros(sh["q"], dtype=torch.bfloat16, device="cuda"))


def test_expired_wait_is_reported_and_the_workspace_recovers(cuda_device):
    w, p = par.workload_params(wl.WORKLOADS["llama32k"])
    qb, kb, vb = wl.make_workload(w)
    q, k, v = par.to_dev(qb), par.to_dev(kb), par.to_dev(vb)
    ws = native.new_workspace(p)
    b = _buffers(p)
    native.set_wait_limit_ns(SHORT_LIMIT_NS)
    try:
        native.prefill(p, q, k, v, b["out"], b["idx"], b["cnt"], ws, mass=b["mass"])
        st, raw = native.check_device_status(ws)
    finally:
        native.set_wait_limit_ns(0)
    assert st == RRA_ERR_DEVICE_TIMEOUT and raw & 1, (st, raw)
    # the attention kernel saw the sticky bit and wrote nothing
    assert not b["out"].any().item()
    st, raw = native.check_device_status(ws)
    assert st == 0 and raw == 0, "the first read clears the word"

    # the same workspace, default limit: identical to a fresh workspace's run
    native.prefill(p, q, k, v, b["out"], b["idx"], b["cnt"], ws, mass=b["mass"])
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    ref = par.run_prefill(p, q, k, v)
    assert ref["status"] == 0, ref["raw"]
    assert np.array_equal(b["mass"].cpu().numpy(), ref["mass"])
    assert np.array_equal(b["idx"].cpu().numpy(), ref["idx"])
    assert np.array_equal(b["cnt"].cpu().numpy(), ref["cnt"])
    assert np.array_equal(b["out"].float().cpu().numpy(), ref["out"])
    # and the oracle agrees on sampled rows
    qc, kc, vc = par.HeadCache(qb), par.HeadCache(kb), par.HeadCache(vb)
    rows = par.sample_rows(p, 6, seed=9)
    om = par.oracle_mass_rows(qc, kc, p, rows)
    merr = max(float(np.abs(ref["mass"][bb, h, par.orc.tri_offset(I):par.orc.tri_offset(I + 1)]
                            - om[(bb, h, I)]).max()) for bb, h, I in rows)
    assert merr <= par.MASS_ATOL, merr


def test_timeout_bit_makes_later_kernels_exit(cuda_device):
    """A word left set (its read not yet taken) makes every later kernel on that workspace return
    without work, including a call made with the default limit."""
    w, p = par.workload_params(wl.WORKLOADS["llama32k"], stride=16)
    qb, kb, vb = wl.make_workload(w)
    q, k, v = par.to_dev(qb), par.to_dev(kb), par.to_dev(vb)
    ws = native.new_workspace(p)
    b = _buffers(p)
    native.set_wait_limit_ns(SHORT_LIMIT_NS)
    try:
        native.estimate(p, q, k, b["mass"], ws)
        torch.cuda.synchronize()
    finally:
        native.set_wait_limit_ns(0)
    b["mass"].fill_(-7.0)
    native.sparse_attn(p, q, k, v, b["idx"].fill_(0), b["cnt"].fill_(1), b["out"], ws)
    native.estimate(p, q, k, b["mass"], ws)
    st, raw = native.check_device_status(ws)
    assert st == RRA_ERR_DEVICE_TIMEOUT, (st, raw)
    assert not b["out"].any().item()
    assert (b["mass"] == -7.0).all().item()
