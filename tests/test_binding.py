"""The Python binding's own checks (CPU): shapes, dtypes, devices and contiguity are refused with
a ValueError before the library is called, and parameters and shapes follow rra_params."""
import pytest
import torch

from long_context_prefill_rr_b200 import native


def _p():
    return native.params(1, 4, 2, 256, 64, 8, 0.9, shift=3)


def test_params_and_shapes():
    p = _p()
    assert (p.batch, p.heads_q, p.heads_kv, p.seqlen, p.head_dim, p.block, p.stride, p.shift) == \
        (1, 4, 2, 256, 64, 128, 8, 3)
    assert abs(p.tau - 0.9) < 1e-7 and p.softmax_scale == -1.0
    sh = native.shapes(p)
    assert sh["q"] == (1, 4, 256, 64) and sh["kv"] == (1, 2, 256, 64)
    assert sh["mass"] == sh["kept_idx"] == (1, 4, 3) and sh["kept_cnt"] == (1, 4, 2)


def test_device_tensors_are_required():
    p = _p()
    sh = native.shapes(p)
    q = torch.zeros(sh["q"], dtype=torch.bfloat16)            # on the CPU
    k = torch.zeros(sh["kv"], dtype=torch.bfloat16)
    mass = torch.zeros(sh["mass"], dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        native.estimate(p, q, k, mass, torch.zeros(16, dtype=torch.uint8))


def test_host_entry_checks_its_host_buffers():
    p = _p()
    sh = native.shapes(p)
    good = torch.zeros(sh["q"], dtype=torch.bfloat16)
    kv = torch.zeros(sh["kv"], dtype=torch.bfloat16)
    bad_dtype = torch.zeros(sh["q"], dtype=torch.float16)
    bad_shape = torch.zeros((1, 4, 128, 64), dtype=torch.bfloat16)
    strided = torch.zeros((1, 4, 256, 128), dtype=torch.bfloat16)[..., :64]
    for q_host in (bad_dtype, bad_shape, strided):
        with pytest.raises(ValueError, match="q_host"):
            native.prefill_host(p, q_host, kv, kv, good, None, None, None, None, None, None, None)
