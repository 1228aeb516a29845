"""rra_prefill_host: host buffers in and out, chunked so that the copies overlap the compute.
The chunks are independent sub-problems: query-head groups within a KV head, whole KV heads when
there are more than 32 (the mha48 case), or batch rows. A chunk of heads runs with the
round-robin shift advanced by its first head (the sampled offset rotates across heads:
RRAttention abstract). Its kept lists and output are compared with the fp64 oracle run on the
global heads and shift (kept lists of every row under the boundary rule, every output row),
and must equal rra_prefill's on the same inputs bit for bit. The cases cover each kind of
chunk."""
import numpy as np
import pytest
import torch

import parity as par
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_gqa_shift": (wl.WORKLOADS["tiny"].with_(heads_kv=4, shift=5), 1),
    "llama8k": (wl.WORKLOADS["llama8k"], 1),
    "tiny_batch3": (wl.WORKLOADS["tiny"].with_(heads_kv=2, shift=3), 3),
    "video_short": (wl.WORKLOADS["video64k"].with_(seqlen=4096), 1),
    "tiny_mha48": (wl.WORKLOADS["tiny"].with_(heads_q=48, heads_kv=48, shift=1), 1),
}


def _host(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefill_host_equals_prefill(cuda_device, name):
    w, batch = CASES[name]
    w = w.with_(batch=batch)
    w, p = par.workload_params(w)
    qb, kb, vb = wl.make_workload(w)
    ref = par.run_prefill(p, par.to_dev(qb), par.to_dev(kb), par.to_dev(vb))
    assert ref["status"] == 0, ref["raw"]
    sh = native.shapes(p)
    qh, kh, vh = (_host(x).pin_memory() for x in (qb, kb, vb))
    oh = torch.empty(sh["q"], dtype=torch.bfloat16).pin_memory()
    qd = torch.empty(sh["q"], dtype=torch.bfloat16, device="cuda")
    kd = torch.empty(sh["kv"], dtype=torch.bfloat16, device="cuda")
    vd = torch.empty(sh["kv"], dtype=torch.bfloat16, device="cuda")
    od = torch.empty(sh["q"], dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda")
    cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda")
    ws = native.new_workspace(p)
    for _ in range(2):   # twice in a row: the staging buffers and the internal events are reused
        oh.zero_()
        native.prefill_host(p, qh, kh, vh, oh, qd, kd, vd, od, idx, cnt, ws)
        torch.cuda.current_stream().synchronize()
        st, raw = native.check_device_status(ws)
        assert st == 0, raw
        got = dict(idx=idx.cpu().numpy(), cnt=cnt.cpu().numpy(), out=oh.float().numpy())
        assert np.array_equal(got["idx"], ref["idx"])
        assert np.array_equal(got["cnt"], ref["cnt"])
        assert np.array_equal(got["out"], ref["out"])
    # against the oracle on the global heads (the masses stay in the workspace: the lists are
    # checked against the oracle's select on the oracle's masses)
    nb = w.seqlen // w.block
    full = par.oracle_masses_full(qb, kb, p)
    mism, exc, n = par.compare_select_rows(got, par.mass_rows(full, nb), w.tau)
    assert not mism, f"{name}: kept-list mismatches outside the boundary rule: {mism[:5]}"
    import oracle_pool
    ma, rr, n_attn = oracle_pool.attention_errors_full(
        qb, kb, vb, got["out"], got["idx"], got["cnt"], p.heads_q, p.heads_kv, p.block,
        par.resolved_scale(p))
    assert ma <= par.ATTN_MAX_ABS and rr <= par.ATTN_REL_RMS, (name, ma, rr)
    par.record(f"prefill_host_{name}", list_rows=n, list_mismatch_excused=len(exc),
               attn_rows=f"all {n_attn}", attn_max_abs=ma, attn_rel_rms=rr)
