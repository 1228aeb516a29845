"""rra_prefill_host: host buffers in and out, chunked so that the copies overlap the compute.
Its kept lists and output equal rra_prefill's on the same inputs, bit for bit. The chunks are
independent sub-problems: query-head groups within a KV head, whole KV heads when there are more
than 16, or batch rows. A chunk of heads runs with the round-robin shift advanced by its first
head. The cases cover each kind of chunk."""
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
    "tiny_mha32": (wl.WORKLOADS["tiny"].with_(heads_q=32, heads_kv=32, shift=1), 1),
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
        assert np.array_equal(idx.cpu().numpy(), ref["idx"])
        assert np.array_equal(cnt.cpu().numpy(), ref["cnt"])
        assert np.array_equal(oh.float().numpy(), ref["out"])
