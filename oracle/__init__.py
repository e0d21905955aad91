"""fp64 CPU oracle for ReLU linear attention with 3D RoPE (ctypes loader).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` use it; the CUDA library and its binding never do.
The arithmetic lives in ``oracle.c`` (plain C, fp64, index-order sums); this
file compiles it with gcc and marshals numpy arrays, and holds the plain fp64
numpy form of linear cross-attention at its end. ``oracle.tconv`` holds the
fp64 Mix-FFN temporal convolution with its last-frame cache.

Every function here is pinned by ``tests/test_oracle.py`` against the brute
force O(N^2) form, closed forms, invariants of the SANA-Video equations and
hand-worked examples under ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# ORACLE_SRC / ORACLE_LIB let the mutation test build a deliberately broken
# copy of the oracle elsewhere and check that the pins reject it.
_SRC = os.environ.get("ORACLE_SRC", os.path.join(_HERE, "oracle.c"))
_LIB = os.environ.get("ORACLE_LIB", os.path.join(_HERE, "liborc.so"))

BIDIRECTIONAL = 0
BLOCK_CAUSAL = 1
TOKEN_CAUSAL = 2

_MODES = {"bidirectional": BIDIRECTIONAL, "block_causal": BLOCK_CAUSAL,
          "token_causal": TOKEN_CAUSAL}


class Params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("D", ctypes.c_int),
        ("mode", ctypes.c_int), ("block_tokens", ctypes.c_int), ("rope", ctypes.c_int),
        ("grid_t", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("rope_dt", ctypes.c_int), ("rope_dh", ctypes.c_int), ("rope_dw", ctypes.c_int),
        ("t_offset", ctypes.c_int), ("theta", ctypes.c_double), ("eps", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile oracle.c into liborc.so next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-shared",
                               "-fPIC", "-pthread", _SRC, "-lm", "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        pp = ctypes.POINTER(Params)
        _lib.orc_check.argtypes = [pp]
        _lib.orc_rope.argtypes = [pp, ctypes.c_long, dp, dp]
        _lib.orc_forward.argtypes = [pp, fp, fp, fp, fp, dp, dp, dp, dp, dp, ctypes.c_int]
        _lib.orc_forward_rows.argtypes = [pp, fp, fp, fp, fp, dp, dp,
                                          ctypes.POINTER(ctypes.c_longlong), ctypes.c_long,
                                          dp, ctypes.c_int]
        _lib.orc_state.argtypes = [pp, fp, fp, ctypes.c_long, ctypes.c_long, dp, dp, ctypes.c_int]
        _lib.orc_bruteforce.argtypes = [pp, fp, fp, fp, fp, dp, ctypes.c_int]
        _lib.orc_resolve_threads.argtypes = [ctypes.c_int]
        for f in ("orc_check", "orc_rope", "orc_forward", "orc_forward_rows", "orc_state",
                  "orc_bruteforce", "orc_resolve_threads"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def make_params(B, H, N, D, mode="bidirectional", block_tokens=0, grid=None,
                rope_split=None, theta=10000.0, eps=1e-6, t_offset=0) -> Params:
    p = Params()
    p.B, p.H, p.N, p.D = B, H, N, D
    p.mode = _MODES[mode] if isinstance(mode, str) else int(mode)
    p.block_tokens = block_tokens
    p.rope = 1 if grid is not None else 0
    if grid is not None:
        p.grid_t, p.grid_h, p.grid_w = grid
        p.rope_dt, p.rope_dh, p.rope_dw = rope_split
    p.t_offset = t_offset
    p.theta = theta
    p.eps = eps
    return p


def params_for(w, mode=None) -> Params:
    """Params for a ``workloads.Workload``."""
    mode = mode or w.modes[0]
    return make_params(w.B, w.H, w.N, w.D, mode=mode,
                       block_tokens=w.block_tokens if mode == "block_causal" else 0,
                       grid=w.grid, rope_split=w.rope_split, theta=w.rope_theta, eps=w.eps)


def _f32(a):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _f64(a):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def threads(nthreads: int = 0) -> int:
    return lib().orc_resolve_threads(nthreads)


def rope(p: Params, n: int, x: np.ndarray) -> np.ndarray:
    x, xp = _f64(x)
    y = np.empty_like(x)
    _check(lib().orc_rope(ctypes.byref(p), n, xp, y.ctypes.data_as(ctypes.POINTER(ctypes.c_double))), "rope")
    return y


def forward(p: Params, q, k, v, g=None, S0=None, z0=None, nthreads: int = 0,
            want_state: bool = False, want_out: bool = True):
    """Full fp64 output [B,H,N,D] (and the final carried state if asked)."""
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    g, gp = _f32(g)
    S0, S0p = _f64(S0)
    z0, z0p = _f64(z0)
    out = np.empty((p.B, p.H, p.N, p.D), dtype=np.float64) if want_out else None
    outp = out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if want_out else None
    Sf = zf = Sfp = zfp = None
    if want_state:
        Sf = np.empty((p.B, p.H, p.D, p.D), dtype=np.float64)
        zf = np.empty((p.B, p.H, p.D), dtype=np.float64)
        Sfp = Sf.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
        zfp = zf.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    _check(lib().orc_forward(ctypes.byref(p), qp, kp, vp, gp, S0p, z0p, outp, Sfp, zfp,
                             nthreads), "forward")
    if want_state:
        return out, Sf, zf
    return out


def forward_rows(p: Params, q, k, v, rows, g=None, S0=None, z0=None, nthreads: int = 0):
    """Rows ``rows`` (flattened (b*H+h)*N+n) of the fp64 output, [len(rows), D]."""
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    g, gp = _f32(g)
    S0, S0p = _f64(S0)
    z0, z0p = _f64(z0)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, p.D), dtype=np.float64)
    _check(lib().orc_forward_rows(ctypes.byref(p), qp, kp, vp, gp, S0p, z0p,
                                  rows.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
                                  rows.size, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                  nthreads), "forward_rows")
    return out


def state(p: Params, k, v, n0: int = 0, n1: Optional[int] = None,
          nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """(S [B,H,D,D], z [B,H,D]) over tokens [n0, n1) of every head."""
    n1 = p.N if n1 is None else n1
    k, kp = _f32(k)
    v, vp = _f32(v)
    S = np.empty((p.B, p.H, p.D, p.D), dtype=np.float64)
    z = np.empty((p.B, p.H, p.D), dtype=np.float64)
    _check(lib().orc_state(ctypes.byref(p), kp, vp, n0, n1,
                           S.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                           z.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), nthreads), "state")
    return S, z


def bruteforce(p: Params, q, k, v, g=None, nthreads: int = 0) -> np.ndarray:
    """Literal O(N^2) attention-weight form; tiny inputs only."""
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    g, gp = _f32(g)
    out = np.empty((p.B, p.H, p.N, p.D), dtype=np.float64)
    _check(lib().orc_bruteforce(ctypes.byref(p), qp, kp, vp, gp,
                                out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                nthreads), "bruteforce")
    return out


# ---- linear cross-attention -------------------------------------------------
#
# Queries of one sequence read the keys and values of another (N_q != N_kv,
# e.g. video tokens attending to text tokens), with the same ReLU kernel and
# no rotation (the two sequences share no positions): the linear
# cross-attention the SANA-Video paper-graph page names beside its
# self-attention. Plain fp64 numpy, written from the definition.

def cross_forward(q, k, v, g=None, eps: float = 1e-6) -> np.ndarray:
    """out[b,h,i] = phi(q_i) S / (phi(q_i) . z + eps) (* sigmoid(g_i)), with
    S = sum_j phi(k_j)^T v_j and z = sum_j phi(k_j) over the N_kv keys of the
    same (b, h). q, g: [B,H,Nq,D]; k, v: [B,H,Nkv,D]."""
    q = np.maximum(np.asarray(q, dtype=np.float64), 0.0)
    k = np.maximum(np.asarray(k, dtype=np.float64), 0.0)
    v = np.asarray(v, dtype=np.float64)
    S = np.einsum("bhja,bhjc->bhac", k, v)
    z = k.sum(axis=2)
    num = np.einsum("bhia,bhac->bhic", q, S)
    den = np.einsum("bhia,bha->bhi", q, z) + eps
    out = num / den[..., None]
    if g is not None:
        out = out / (1.0 + np.exp(-np.asarray(g, dtype=np.float64)))
    return out


def cross_bruteforce(q, k, v, g=None, eps: float = 1e-6) -> np.ndarray:
    """The attention-weight form: out_i = sum_j w_ij v_j / (sum_j w_ij + eps)
    with w_ij = phi(q_i) . phi(k_j); tiny inputs only."""
    q = np.maximum(np.asarray(q, dtype=np.float64), 0.0)
    k = np.maximum(np.asarray(k, dtype=np.float64), 0.0)
    v = np.asarray(v, dtype=np.float64)
    B, H, Nq, D = q.shape
    out = np.zeros((B, H, Nq, D))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                w = [float(np.dot(q[b, h, i], k[b, h, j])) for j in range(k.shape[2])]
                acc = np.zeros(D)
                for j, wj in enumerate(w):
                    acc += wj * v[b, h, j]
                out[b, h, i] = acc / (sum(w) + eps)
    if g is not None:
        out = out / (1.0 + np.exp(-np.asarray(g, dtype=np.float64)))
    return out
