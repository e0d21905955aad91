"""ctypes binding of liblinattn.so: the C ABI of include/linattn.h, same names.

Only argument marshalling lives here. Every step of the computation runs in
the CUDA kernels of the shared library; if the library is missing this module
raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblinattn.so")

LA_OK = 0
LA_ERR_INVALID_ARG = 1
LA_ERR_UNSUPPORTED = 2
LA_ERR_WORKSPACE = 3
LA_ERR_CUDA = 4
LA_ERR_DEVICE_TIMEOUT = 5

LA_WORKSPACE_CONTROL_BYTES = 65536   # control block at the start of a workspace

LA_F32 = 0
LA_BF16 = 1
LA_LAYOUT_BHND = 0
LA_LAYOUT_BNHD = 1
LA_BIDIRECTIONAL = 0
LA_BLOCK_CAUSAL = 1
LA_TOKEN_CAUSAL = 2


class la_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("D", ctypes.c_int),
        ("dtype", ctypes.c_int), ("mode", ctypes.c_int), ("block_tokens", ctypes.c_int),
        ("rope", ctypes.c_int),
        ("grid_t", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("rope_dt", ctypes.c_int), ("rope_dh", ctypes.c_int), ("rope_dw", ctypes.c_int),
        ("rope_theta", ctypes.c_double), ("eps", ctypes.c_float), ("layout", ctypes.c_int),
    ]


class la_state(ctypes.Structure):
    _fields_ = [("S", ctypes.c_void_p), ("z", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int)]


# Every exported symbol of include/linattn.h with its signature.
_P = ctypes.POINTER(la_params)
_ST = ctypes.POINTER(la_state)
_V = ctypes.c_void_p
SIGNATURES = {
    "lin_attn_workspace_size": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "lin_attn_block_step_workspace_size": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "lin_attn_forward": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, ctypes.c_size_t, _V]),
    "lin_attn_forward_timed": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, ctypes.c_size_t, _V,
                                              ctypes.POINTER(ctypes.c_void_p)]),
    "lin_attn_forward_noalloc": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V]),
    "lin_attn_cross_forward": (ctypes.c_int, [_P, ctypes.c_int, _V, _V, _V, _V, _V, _V,
                                              ctypes.c_size_t, _V]),
    "lin_attn_cross_workspace_size": (ctypes.c_int, [_P, ctypes.c_int,
                                                     ctypes.POINTER(ctypes.c_size_t)]),
    "lin_attn_state_init": (ctypes.c_int, [_ST, ctypes.c_int, ctypes.c_int, ctypes.c_int, _V, _V]),
    "lin_attn_state_reset": (ctypes.c_int, [_ST, _V]),
    "lin_attn_block_step": (ctypes.c_int, [_P, _ST, ctypes.c_int, _V, _V, _V, _V, _V, ctypes.c_int,
                                           _V, ctypes.c_size_t, _V]),
    "lin_attn_state_update": (ctypes.c_int, [_P, _ST, ctypes.c_int, _V, _V, _V, ctypes.c_size_t,
                                             _V]),
    "lin_attn_device_status": (ctypes.c_int, [_V, _V]),
    "lin_attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lin_attn_uses_tensor_cores": (ctypes.c_int, [_P]),
    "lin_attn_temporal_conv": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, _V, _V, _V, _V, _V,
                                              _V, _V]),
}

_lib = None


class LinAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


def load():
    """Load liblinattn.so (built in-tree by __graft_entry__.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("liblinattn.so is not built at %s; run __graft_entry__.build() "
                              "(or python linear_attention_video_relu_b200/build.py)" % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def status_string(s: int) -> str:
    return load().lin_attn_status_string(s).decode()


def check(status: int, what: str) -> None:
    if status != LA_OK:
        raise LinAttnError(status, what)


def lin_attn_workspace_size(p: la_params) -> int:
    n = ctypes.c_size_t(0)
    check(load().lin_attn_workspace_size(ctypes.byref(p), ctypes.byref(n)), "lin_attn_workspace_size")
    return n.value


def lin_attn_block_step_workspace_size(p: la_params) -> int:
    n = ctypes.c_size_t(0)
    check(load().lin_attn_block_step_workspace_size(ctypes.byref(p), ctypes.byref(n)),
          "lin_attn_block_step_workspace_size")
    return n.value


def lin_attn_forward(p, q, k, v, gate, out, workspace, workspace_bytes, stream) -> int:
    return load().lin_attn_forward(ctypes.byref(p), q, k, v, gate, out, workspace,
                                   workspace_bytes, stream)


def lin_attn_forward_timed(p, q, k, v, gate, out, workspace, workspace_bytes, stream,
                           events) -> int:
    ev = None
    if events is not None:
        ev = (ctypes.c_void_p * 4)(*events)
    return load().lin_attn_forward_timed(ctypes.byref(p), q, k, v, gate, out, workspace,
                                         workspace_bytes, stream, ev)


def lin_attn_forward_noalloc(p, q, k, v, gate, out, stream) -> int:
    return load().lin_attn_forward_noalloc(ctypes.byref(p), q, k, v, gate, out, stream)


def lin_attn_cross_forward(p, n_kv, q, k, v, gate, out, workspace, workspace_bytes,
                           stream) -> int:
    return load().lin_attn_cross_forward(ctypes.byref(p), n_kv, q, k, v, gate, out, workspace,
                                         workspace_bytes, stream)


def lin_attn_cross_workspace_size(p: la_params, n_kv: int) -> int:
    n = ctypes.c_size_t(0)
    check(load().lin_attn_cross_workspace_size(ctypes.byref(p), n_kv, ctypes.byref(n)),
          "lin_attn_cross_workspace_size")
    return n.value


def lin_attn_state_init(st: la_state, B, H, D, S, z) -> int:
    return load().lin_attn_state_init(ctypes.byref(st), B, H, D, S, z)


def lin_attn_state_reset(st: la_state, stream) -> int:
    return load().lin_attn_state_reset(ctypes.byref(st), stream)


def lin_attn_block_step(p, st, t_offset, q, k, v, gate, out, commit, workspace,
                        workspace_bytes, stream) -> int:
    return load().lin_attn_block_step(ctypes.byref(p), ctypes.byref(st), t_offset, q, k, v, gate,
                                      out, commit, workspace, workspace_bytes, stream)


def lin_attn_state_update(p, st, t_offset, k, v, workspace, workspace_bytes, stream) -> int:
    return load().lin_attn_state_update(ctypes.byref(p), ctypes.byref(st), t_offset, k, v,
                                        workspace, workspace_bytes, stream)


def lin_attn_device_status(workspace, stream) -> int:
    return load().lin_attn_device_status(workspace, stream)


def lin_attn_uses_tensor_cores(p: la_params) -> int:
    return load().lin_attn_uses_tensor_cores(ctypes.byref(p))


def lin_attn_temporal_conv(B, T, S, C, dtype, x, weight, bias, cache_in, y, cache_out,
                           stream) -> int:
    return load().lin_attn_temporal_conv(B, T, S, C, dtype, x, weight, bias, cache_in, y,
                                         cache_out, stream)
