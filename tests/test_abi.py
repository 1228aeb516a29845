"""The C ABI library loads, exports every entry point include/rra.h declares, and rejects bad
arguments before touching a GPU (these run on the CPU-only build host)."""
import ctypes
import os
import re

import pytest

from long_context_prefill_rr_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rra.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(rra_[a-z_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(native.LIB_PATH):
        from long_context_prefill_rr_b200 import build
        build.build()
    return native.load()


def test_header_declares_the_boundary():
    assert _declared() == sorted([
        "rra_workspace_bytes", "rra_estimate", "rra_estimate_select", "rra_select", "rra_sparse_attn", "rra_prefill",
        "rra_estimate_static_scratch", "rra_estimate_xattn", "rra_prefill_host",
        "rra_check_device_status", "rra_static_scratch_status", "rra_set_wait_limit_ns",
        "rra_status_string", "rra_version"])


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(native._SIGS)


def test_params_struct_layout():
    assert ctypes.sizeof(native.RraParams) == 40
    assert native.RraParams.tau.offset == 32 and native.RraParams.softmax_scale.offset == 36


def test_status_strings(lib):
    assert native.status_string(0) == "ok"
    assert native.status_string(3) == "workspace too small"
    assert native.version().startswith("rra")


def _call_estimate(p, q=16, k=16, mass=16, ws=16, nws=1 << 20):
    return native.load().rra_estimate(ctypes.byref(p), ctypes.c_void_p(q), ctypes.c_void_p(k),
                                      ctypes.c_void_p(mass), ctypes.c_void_p(ws), nws, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(heads_q=6, heads_kv=4), 1),      # Hq % Hkv != 0
    (dict(seqlen=1000), 1),                # L % B != 0
    (dict(stride=3), 1),                   # B % S != 0
    (dict(tau=0.0), 1),                    # tau <= 0
    (dict(tau=float("nan")), 1),
    (dict(batch=-1), 1),
    (dict(block=64, seqlen=1024), 2),      # only B = 128
    (dict(head_dim=96), 2),
    (dict(stride=2), 2),                   # S outside {4, 8, 16, 32} for the estimate
])
def test_estimate_rejects_bad_params_before_any_launch(lib, kw, expect):
    base = dict(batch=1, heads_q=8, heads_kv=8, seqlen=1024, head_dim=64, stride=8, tau=0.9)
    base.update(kw)
    p = native.params(**base)
    assert _call_estimate(p) == expect


def test_pointer_checks(lib):
    p = native.params(1, 8, 8, 1024, 64, 8, 0.9)
    assert _call_estimate(p, q=0) == 1           # null
    assert _call_estimate(p, k=8) == 1           # not 16-byte aligned
    assert lib.rra_select(ctypes.byref(p), None, ctypes.c_void_p(16), ctypes.c_void_p(16),
                          None) == 1
    assert lib.rra_check_device_status(None, None, None) == 1
    # host entry: a missing host buffer or a misaligned staging buffer is refused up front
    ok, bad = ctypes.c_void_p(16), ctypes.c_void_p(8)
    assert lib.rra_prefill_host(ctypes.byref(p), None, ok, ok, ok, ok, ok, ok, ok, ok, ok, ok,
                                1 << 30, None) == 1
    assert lib.rra_prefill_host(ctypes.byref(p), ok, ok, ok, ok, bad, ok, ok, ok, ok, ok, ok,
                                1 << 30, None) == 1


def test_empty_problem_is_a_noop(lib):
    p = native.params(0, 8, 8, 1024, 64, 8, 0.9)
    assert _call_estimate(p, q=0, k=0, mass=0, ws=0, nws=0) == 0
    p = native.params(1, 8, 8, 0, 64, 8, 0.9)
    assert lib.rra_prefill(ctypes.byref(p), *([None] * 8), 0, None) == 0


def test_workspace_query_rejects_invalid_params(lib):
    assert lib.rra_workspace_bytes(ctypes.byref(native.params(1, 8, 8, 1000, 64, 8, 0.9))) == 0
