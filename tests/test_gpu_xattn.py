"""GPU parity of the XAttention antidiagonal estimator (rra_estimate_xattn) against the fp64
oracle, and of the selection that follows it."""
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


@pytest.mark.parametrize("name,n_rows", [("llama8k", 96), ("llama32k", 32)])
def test_xattn_sampled_parity(cuda_device, name, n_rows):
    w, p = par.workload_params(wl.WORKLOADS[name])
    qb, kb, _ = wl.make_workload(w)
    gpu = _run(p, qb, kb)
    qc, kc = par.HeadCache(qb), par.HeadCache(kb)
    scale = par.resolved_scale(p)
    err = 0.0
    for b, h, I in par.sample_rows(p, n_rows, seed=7):
        kv = orc.kv_head(h, w.heads_q, w.heads_kv)
        want = orc.xattn_estimate_block_row(qc(b, h), kc(b, kv), I, w.block, w.stride, scale)
        got = gpu[b, h, orc.tri_offset(I):orc.tri_offset(I + 1)]
        err = max(err, float(np.abs(got - want).max()))
    assert err <= par.MASS_ATOL, err
    print(f"[xattn {name}] mass_err={err:.3g}")
