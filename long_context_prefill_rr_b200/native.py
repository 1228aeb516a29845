"""ctypes binding of ``librra.so`` (the C ABI declared in ``include/rra.h``).

Argument marshalling only: every step of the path runs in the library's sm_100a kernels. The
functions take torch CUDA tensors (PyTorch supplies device memory and streams) and pass raw
device pointers. If the library is not built the import of a compute entry point raises; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librra.so")

RRA_OK = 0
STATUS_NAMES = {
    0: "RRA_OK", 1: "RRA_ERR_INVALID_ARG", 2: "RRA_ERR_UNSUPPORTED", 3: "RRA_ERR_WORKSPACE",
    4: "RRA_ERR_CUDA", 5: "RRA_ERR_DEVICE_TIMEOUT",
}

# every entry point declared in include/rra.h, with its ctypes signature
_c = ctypes
_SIGS = {
    "rra_workspace_bytes": (_c.c_size_t, [_c.c_void_p]),
    "rra_estimate": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                _c.c_size_t, _c.c_void_p]),
    "rra_select": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "rra_sparse_attn": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                   _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                   _c.c_size_t, _c.c_void_p]),
    "rra_prefill": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                               _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                               _c.c_void_p]),
    "rra_prefill_host": (_c.c_int, [_c.c_void_p] + [_c.c_void_p] * 11 + [_c.c_size_t,
                                                                          _c.c_void_p]),
    "rra_estimate_select": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                       _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                       _c.c_void_p]),
    "rra_estimate_xattn": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                      _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "rra_estimate_static_scratch": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p,
                                               _c.c_void_p, _c.c_void_p]),
    "rra_check_device_status": (_c.c_int, [_c.c_void_p, _c.c_void_p,
                                           _c.POINTER(_c.c_uint32)]),
    "rra_static_scratch_status": (_c.c_int, [_c.c_void_p, _c.POINTER(_c.c_uint32)]),
    "rra_set_wait_limit_ns": (None, [_c.c_uint64]),
    "rra_status_string": (_c.c_char_p, [_c.c_int]),
    "rra_version": (_c.c_char_p, []),
}


class RraParams(ctypes.Structure):
    """Mirror of ``rra_params``."""
    _fields_ = [
        ("batch", ctypes.c_int), ("heads_q", ctypes.c_int), ("heads_kv", ctypes.c_int),
        ("seqlen", ctypes.c_int), ("head_dim", ctypes.c_int), ("block", ctypes.c_int),
        ("stride", ctypes.c_int), ("shift", ctypes.c_int), ("tau", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
    ]


class RraError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load() -> ctypes.CDLL:
    """Load librra.so (raises if it has not been built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m long_context_prefill_rr_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def params(batch: int, heads_q: int, heads_kv: int, seqlen: int, head_dim: int, stride: int,
           tau: float, shift: int = 0, softmax_scale: float = -1.0, block: int = 128) -> RraParams:
    return RraParams(batch, heads_q, heads_kv, seqlen, head_dim, block, stride, shift, tau,
                     softmax_scale)


def _p(p: RraParams):
    return ctypes.byref(p)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != RRA_OK:
        raise RraError(status, what)


def _expect(t, dtype, shape, name):
    import torch
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    del torch


def shapes(p: RraParams) -> dict:
    nb = p.seqlen // p.block if p.block else 0
    tri = nb * (nb + 1) // 2
    return {
        "q": (p.batch, p.heads_q, p.seqlen, p.head_dim),
        "kv": (p.batch, p.heads_kv, p.seqlen, p.head_dim),
        "mass": (p.batch, p.heads_q, tri),
        "kept_idx": (p.batch, p.heads_q, tri),
        "kept_cnt": (p.batch, p.heads_q, nb),
    }


def status_string(status: int) -> str:
    return load().rra_status_string(status).decode()


def version() -> str:
    return load().rra_version().decode()


def workspace_bytes(p: RraParams) -> int:
    return int(load().rra_workspace_bytes(_p(p)))


def estimate(p: RraParams, q, k, mass, ws, stream=None):
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(mass, torch.float32, sh["mass"], "mass")
    _check(load().rra_estimate(_p(p), _ptr(q), _ptr(k), _ptr(mass), _ptr(ws), ws.numel(),
                               _stream(stream)), "rra_estimate")


def estimate_select(p: RraParams, q, k, kept_idx, kept_cnt, ws, mass=None, stream=None):
    """Steps 1 and 2 in one launch (rra_estimate_select): masses (into ``mass``, or the
    workspace when None) and the kept lists of rra_select."""
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(kept_idx, torch.int32, sh["kept_idx"], "kept_idx")
    _expect(kept_cnt, torch.int32, sh["kept_cnt"], "kept_cnt")
    if mass is not None:
        _expect(mass, torch.float32, sh["mass"], "mass")
    _check(load().rra_estimate_select(_p(p), _ptr(q), _ptr(k), _ptr(mass), _ptr(kept_idx),
                                      _ptr(kept_cnt), _ptr(ws), ws.numel(), _stream(stream)),
           "rra_estimate_select")


def estimate_xattn(p: RraParams, q, k, mass, ws, stream=None):
    """XAttention antidiagonal estimate (same mass layout as ``estimate``)."""
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(mass, torch.float32, sh["mass"], "mass")
    _check(load().rra_estimate_xattn(_p(p), _ptr(q), _ptr(k), _ptr(mass), _ptr(ws), ws.numel(),
                                     _stream(stream)), "rra_estimate_xattn")


def estimate_static_scratch(p: RraParams, q, k, mass, stream=None):
    """rra_estimate without a workspace, for callers that cannot allocate device memory: the
    library's fixed 48 MiB device array serves as scratch (problems that need more are
    refused; calls that overlap on the GPU race on the shared array)."""
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(mass, torch.float32, sh["mass"], "mass")
    _check(load().rra_estimate_static_scratch(_p(p), _ptr(q), _ptr(k), _ptr(mass),
                                              _stream(stream)), "rra_estimate_static_scratch")


def select(p: RraParams, mass, kept_idx, kept_cnt, stream=None):
    import torch
    sh = shapes(p)
    _expect(mass, torch.float32, sh["mass"], "mass")
    _expect(kept_idx, torch.int32, sh["kept_idx"], "kept_idx")
    _expect(kept_cnt, torch.int32, sh["kept_cnt"], "kept_cnt")
    _check(load().rra_select(_p(p), _ptr(mass), _ptr(kept_idx), _ptr(kept_cnt), _stream(stream)),
           "rra_select")


def sparse_attn(p: RraParams, q, k, v, kept_idx, kept_cnt, out, ws, stream=None):
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(v, torch.bfloat16, sh["kv"], "v")
    _expect(kept_idx, torch.int32, sh["kept_idx"], "kept_idx")
    _expect(kept_cnt, torch.int32, sh["kept_cnt"], "kept_cnt")
    _expect(out, torch.bfloat16, sh["q"], "out")
    _check(load().rra_sparse_attn(_p(p), _ptr(q), _ptr(k), _ptr(v), _ptr(kept_idx),
                                  _ptr(kept_cnt), _ptr(out), _ptr(ws), ws.numel(),
                                  _stream(stream)), "rra_sparse_attn")


def prefill(p: RraParams, q, k, v, out, kept_idx, kept_cnt, ws, mass=None, stream=None):
    import torch
    sh = shapes(p)
    _expect(q, torch.bfloat16, sh["q"], "q")
    _expect(k, torch.bfloat16, sh["kv"], "k")
    _expect(v, torch.bfloat16, sh["kv"], "v")
    _expect(out, torch.bfloat16, sh["q"], "out")
    _expect(kept_idx, torch.int32, sh["kept_idx"], "kept_idx")
    _expect(kept_cnt, torch.int32, sh["kept_cnt"], "kept_cnt")
    if mass is not None:
        _expect(mass, torch.float32, sh["mass"], "mass")
    _check(load().rra_prefill(_p(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(mass),
                              _ptr(kept_idx), _ptr(kept_cnt), _ptr(ws), ws.numel(),
                              _stream(stream)), "rra_prefill")


def check_device_status(ws, stream=None) -> tuple[int, int]:
    """(status, raw status word); synchronises the stream and clears the word."""
    raw = ctypes.c_uint32(0)
    st = load().rra_check_device_status(_ptr(ws), _stream(stream), ctypes.byref(raw))
    return int(st), int(raw.value)


def static_scratch_status(stream=None) -> tuple[int, int]:
    """(status, raw status word) of the fixed scratch array behind estimate_static_scratch;
    synchronises the stream and clears the word."""
    raw = ctypes.c_uint32(0)
    st = load().rra_static_scratch_status(_stream(stream), ctypes.byref(raw))
    return int(st), int(raw.value)


def set_wait_limit_ns(ns: int) -> None:
    """Time limit of the kernels' barrier waits for later calls (0 restores the 4 s default);
    a test hook for the timeout path."""
    load().rra_set_wait_limit_ns(int(ns))


def prefill_host(p: RraParams, q_host, k_host, v_host, out_host, q_dev, k_dev, v_dev, out_dev,
                 kept_idx, kept_cnt, ws, stream=None):
    """rra_prefill_host: host (preferably pinned) bf16 q/k/v in, host bf16 out, with device
    staging buffers of the same shapes; chunked so that copies overlap the compute."""
    import torch
    sh = shapes(p)
    for t, name, shp in ((q_host, "q_host", sh["q"]), (k_host, "k_host", sh["kv"]),
                         (v_host, "v_host", sh["kv"]), (out_host, "out_host", sh["q"])):
        if t.device.type != "cpu" or t.dtype != torch.bfloat16 or tuple(t.shape) != shp \
                or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous CPU bf16 tensor of shape {shp}")
    _expect(q_dev, torch.bfloat16, sh["q"], "q_dev")
    _expect(k_dev, torch.bfloat16, sh["kv"], "k_dev")
    _expect(v_dev, torch.bfloat16, sh["kv"], "v_dev")
    _expect(out_dev, torch.bfloat16, sh["q"], "out_dev")
    _expect(kept_idx, torch.int32, sh["kept_idx"], "kept_idx")
    _expect(kept_cnt, torch.int32, sh["kept_cnt"], "kept_cnt")
    _check(load().rra_prefill_host(_p(p), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                   _ptr(out_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                   _ptr(out_dev), _ptr(kept_idx), _ptr(kept_cnt), _ptr(ws),
                                   ws.numel(), _stream(stream)), "rra_prefill_host")


def new_workspace(p: RraParams, device=None):
    """Zero-filled uint8 workspace of rra_workspace_bytes(p) on the current CUDA device."""
    import torch
    n = workspace_bytes(p)
    if n == 0:
        raise RraError(1, "rra_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


class RRAttentionPrefill:
    """Owns the workspace for one parameter set and runs estimate -> select -> attention."""

    def __init__(self, p: RraParams, device=None):
        import torch
        self.p = p
        sh = shapes(p)
        dev = device or torch.device("cuda")
        self.ws = new_workspace(p, dev)
        self.mass = torch.empty(sh["mass"], dtype=torch.float32, device=dev)
        self.kept_idx = torch.empty(sh["kept_idx"], dtype=torch.int32, device=dev)
        self.kept_cnt = torch.empty(sh["kept_cnt"], dtype=torch.int32, device=dev)

    def __call__(self, q, k, v, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        prefill(self.p, q, k, v, out, self.kept_idx, self.kept_cnt, self.ws, mass=self.mass,
                stream=stream)
        return out

    def check(self):
        st, raw = check_device_status(self.ws)
        _check(st, f"device status word {raw:#x}")
