"""rra_estimate_static_scratch: the estimate for callers that cannot allocate device memory.

Such callers (a server whose pool allocator already owns the device and forbids further
cudaMalloc, or code that must not call cudaMalloc / cudaFree because they can synchronise the
device) get their scratch from a fixed array inside the library instead of a workspace. This
file checks, through the C ABI, that it returns exactly the masses of the workspace-based
rra_estimate on the same inputs (both run the same kernels on the same geometry), on two calls
in a row (the array keeps the previous call's contents, so the second call must not depend on
them), also after a call of another shape; that a problem larger than the array is refused; and
that a barrier wait that expires inside it is reported by rra_static_scratch_status, after
which the array serves the next call normally. It is collected last on purpose.
"""
import pytest
import torch

import parity as par
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(name, **over):
    w, p = par.workload_params(wl.WORKLOADS[name], **over)
    qb, kb, _ = wl.make_workload(w)
    return p, par.to_dev(qb), par.to_dev(kb)


def _workspace_estimate(p, q, k):
    mass = torch.empty(native.shapes(p)["mass"], dtype=torch.float32, device="cuda")
    ws = native.new_workspace(p)
    native.estimate(p, q, k, mass, ws)
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    return mass


def _static_estimate(p, q, k):
    mass = torch.full(native.shapes(p)["mass"], float("nan"), dtype=torch.float32,
                      device="cuda")
    native.estimate_static_scratch(p, q, k, mass)
    st, raw = native.static_scratch_status()
    assert st == 0, raw
    return mass


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("llama8k", {}),
    ("tiny", dict(stride=16, shift=3, heads_q=8, heads_kv=2, head_dim=128, seqlen=1152)),
])
def test_static_scratch_matches_workspace_estimate_twice(cuda_device, name, over):
    p, q, k = _inputs(name, **over)
    ref = _workspace_estimate(p, q, k)
    for _ in range(2):
        got = _static_estimate(p, q, k)
        assert torch.equal(got, ref)


def test_static_scratch_after_a_call_of_another_shape(cuda_device):
    pa, qa, ka = _inputs("llama8k")
    pb, qb, kb = _inputs("tiny")
    ref_b = _workspace_estimate(pb, qb, kb)
    _static_estimate(pa, qa, ka)
    got = _static_estimate(pb, qb, kb)
    assert torch.equal(got, ref_b)


def test_static_scratch_refuses_problems_above_its_limit(cuda_device):
    p = native.params(1, 32, 8, 131072, 128, 8, 0.9)
    assert native.workspace_bytes(p) > 48 << 20
    z = torch.zeros(64, dtype=torch.uint8, device="cuda")
    st = native.load().rra_estimate_static_scratch(native._p(p), native._ptr(z), native._ptr(z),
                                                   native._ptr(z), native._stream(None))
    assert st == 3       # RRA_ERR_WORKSPACE, nothing enqueued


def test_static_scratch_reports_an_expired_wait(cuda_device):
    """With the wait limit cut to 1 us the kernel gives up mid-way; the array's status word says
    so (and is cleared by the read), and the next call with the default limit is exact."""
    p, q, k = _inputs("llama8k", seqlen=16384, stride=16)
    ref = _workspace_estimate(p, q, k)
    mass = torch.empty_like(ref)
    native.set_wait_limit_ns(1000)
    try:
        native.estimate_static_scratch(p, q, k, mass)
        st, raw = native.static_scratch_status()
    finally:
        native.set_wait_limit_ns(0)
    assert st == 5 and raw & 1, (st, raw)
    assert native.static_scratch_status() == (0, 0)
    assert torch.equal(_static_estimate(p, q, k), ref)
