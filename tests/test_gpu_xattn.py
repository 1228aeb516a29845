"""GPU parity of the XAttention antidiagonal estimator (rra_estimate_xattn) against the fp64
oracle, and of the selection that follows it: in full on Tiny variants and on every block row
of the Llama-like layer at 8K and 32K."""
import numpy as np
import pytest
import torch

import oracle as orc
import parity as par
from long_context_prefill_rr_b200 import native
from long_context_prefill_rr_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _run(p, qb, kb):
    mass = torch.empty(native.shapes(p)["mass"], dtype=torch.float32, device="cuda")
    ws = native.new_workspace(p)
    native.estimate_xattn(p, par.to_dev(qb), par.to_dev(kb), mass, ws)
    st, raw = native.check_device_status(ws)
    assert st == 0, raw
    return mass.cpu().numpy()


@pytest.mark.parametrize("label,over", [
    ("tiny_s8", {}),
    ("s4_gqa_d128_ragged", dict(stride=4, heads_q=8, heads_kv=2, head_dim=128, seqlen=1152)),
    ("s16_scale", dict(stride=16, softmax_scale=0.125)),
    ("s32_d128", dict(stride=32, head_dim=128, seqlen=2048, heads_q=4, heads_kv=4)),
])
def test_xattn_full_parity(cuda_device, label, over):
    w, p = par.workload_params(wl.WORKLOADS["tiny"], **over)
    qb, kb, _ = wl.make_workload(w)
    gpu = _run(p, qb, kb)
    q64, k64 = wl.bf16_bits_to_f64(qb), wl.bf16_bits_to_f64(kb)
    om = orc.xattn_estimate(q64, k64, w.block, w.stride, par.resolved_scale(p))
    err = float(np.abs(gpu - om).max())
    assert err <= par.MASS_ATOL, (label, err)
    nb = w.seqlen // w.block
    # select on these masses: GPU select equals the oracle's select on the same fp32 masses
    sh = native.shapes(p)
    idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda")
    cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda")
    native.select(p, torch.from_numpy(gpu).cuda(), idx, cnt)
    ri, rc = orc.select(gpu.astype(np.float64), nb, float(np.float32(w.tau)))
    assert np.array_equal(idx.cpu().numpy(), ri) and np.array_equal(cnt.cpu().numpy(), rc)
    print(f"[xattn {label}] mass_err={err:.3g}")


@pytest.mark.parametrize("name", ["llama8k", "llama32k"])
def test_xattn_parity_at_length(cuda_device, name):
    """Every mass of every head against the fp64 oracle (one head per spawned process), the
    select on those masses bit-exact against the oracle's select on the same fp32 masses, and
    the kept lists against the oracle's own lists outside the boundary rule."""
    import oracle_pool
    w, p = par.workload_params(wl.WORKLOADS[name])
    qb, kb, _ = wl.make_workload(w)
    gpu = _run(p, qb, kb)
    full = oracle_pool.xattn_masses_full(qb, kb, p.batch, p.heads_q, p.heads_kv, p.seqlen,
                                         p.block, p.stride, par.resolved_scale(p))
    err = max(float(np.abs(gpu[b, h] - a).max()) for (b, h), a in full.items())
    assert err <= par.MASS_ATOL, err
    nb = w.seqlen // w.block
    sh = native.shapes(p)
    idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device="cuda")
    cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device="cuda")
    native.select(p, torch.from_numpy(gpu).cuda(), idx, cnt)
    res = dict(mass=gpu, idx=idx.cpu().numpy(), cnt=cnt.cpu().numpy())
    assert par.select_on_gpu_masses_exact(res, w.tau, nb), "select on GPU masses"
    rows = par.mass_rows(full, nb)
    mism, exc, n = par.compare_select_rows(res, rows, w.tau)
    assert not mism, mism[:5]
    par.record(f"xattn_{name}", mass_rows=len(rows), mass_max_err=err, list_rows=n,
               list_mismatch_excused=len(exc), boundary_rows=par.boundary_count(rows, w.tau))
