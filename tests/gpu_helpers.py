"""Helpers for the GPU parity tests: upload seeded inputs, run the CUDA path
through the C ABI, compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la

# Tolerances of the parity gate (max-abs and relative L2 over the output).
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_REL_L2 = 1e-4

# Per-row gate, on top of the whole-tensor one: for every output row i (one
# token of one head, D values), ||got_i - ref_i|| / max(||ref_i||, floor) with
# floor = ROW_FLOOR x the RMS row norm of the reference. Over the whole tensor
# one fully wrong row among 1e5 moves the rel-L2 by only ~3e-3; this bound
# catches it. bf16 budget: the rotated phi(q) and phi(k) are rounded to bf16
# for the MMAs and the output is rounded to bf16, three roundings of at most
# 2^-9 relative each, which give a typical row error of 2-3e-3; the bound
# leaves about 8x that for rows whose dot products cancel, while a row with a
# dropped term, the wrong block's state or no rotation is off by 5e-2 to 1.
# fp32 I/O: FFMA kernels with fp32 state, typical row error ~1e-6.
BF16_ROW_REL = 2.5e-2
F32_ROW_REL = 1e-3
ROW_FLOOR = 0.125


def upload(w: workloads.Workload, x: dict, dev="cuda"):
    t = {}
    for n in ("q", "k", "v", "g"):
        if w.dtype == "bf16" and n + "_bits" in x:
            t[n] = torch.from_numpy(x[n + "_bits"]).view(torch.bfloat16).to(dev)
        elif n in x:
            t[n] = torch.from_numpy(x[n]).to(dev)
    return t


def run_forward(w: workloads.Workload, t: dict, mode: str, **kw) -> torch.Tensor:
    bt = w.block_tokens if mode == "block_causal" else 0
    p = la.make_params(w.B, w.H, w.N, w.D, t["q"].dtype, mode, bt, w.grid, w.rope_split,
                       w.rope_theta, w.eps)
    ws = la.workspace_for(p, t["q"].device)
    out = la.forward(t["q"], t["k"], t["v"], t.get("g"), mode=mode, block_tokens=bt,
                     grid=w.grid, rope_split=w.rope_split, theta=w.rope_theta, eps=w.eps,
                     workspace=ws, **kw)
    torch.cuda.synchronize()
    # the arrival counters and the flag are back at zero, and no kernel gave
    # up a bounded wait
    assert ws.control_block_is_zero()
    assert ws.status() == la._native.LA_OK
    return out


def to64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    diff = got - ref
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return rel, float(np.abs(diff).max())


def row_errors(got: np.ndarray, ref: np.ndarray, floor: float = ROW_FLOOR) -> np.ndarray:
    """Per-row relative L2 error over the last axis (rows of D values), the
    denominator floored at `floor` x the RMS row norm of ref."""
    d = ref.shape[-1]
    g = np.asarray(got, dtype=np.float64).reshape(-1, d)
    r = np.asarray(ref, dtype=np.float64).reshape(-1, d)
    if r.shape[0] == 0:
        return np.zeros(0)
    rn = np.linalg.norm(r, axis=1)
    rms = float(np.sqrt(np.mean(rn * rn)))
    den = np.maximum(rn, max(floor * rms, 1e-300))
    return np.linalg.norm(g - r, axis=1) / den


def assert_parity(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert np.all(np.isfinite(got)), what
    rel, mx = errors(got, ref)
    rows = row_errors(got, ref)
    worst = float(rows.max()) if rows.size else 0.0
    at = int(rows.argmax()) if rows.size else -1
    if dtype == "bf16":
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, \
            "%s: rel-L2 %.3e (<= %.0e), max-abs %.3e (<= %.0e)" % (what, rel, BF16_REL_L2, mx,
                                                                BF16_MAX_ABS)
        assert worst <= BF16_ROW_REL, "%s: row %d rel error %.3e (<= %.1e)" % (
            what, at, worst, BF16_ROW_REL)
    else:
        assert rel <= F32_REL_L2, "%s: rel-L2 %.3e (<= %.0e)" % (what, rel, F32_REL_L2)
        assert worst <= F32_ROW_REL, "%s: row %d rel error %.3e (<= %.0e)" % (
            what, at, worst, F32_ROW_REL)
    return rel, mx


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values (8 significant bits) at the magnitude of x:
    2^(e - 7) for 2^e <= |x| < 2^(e + 1); 0 at x = 0."""
    m, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))
    return np.where(m == 0, 0.0, np.ldexp(1.0, e - 8))


def assert_elementwise(got: np.ndarray, ref: np.ndarray, absum: np.ndarray, dtype: str,
                       what: str = ""):
    """Element-by-element bound for an op with fp32 arithmetic and one
    rounding to the output dtype per element: |got - ref| <= 1 bf16 ulp of ref
    (bf16) plus 2^-21 x absum, where absum is the sum of the magnitudes of the
    terms the element adds up (it bounds a handful of fp32 roundings, 2^-24
    relative each, and is what remains where the terms cancel to ~0)."""
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - ref)
    bound = 2.0 ** -21 * np.abs(absum)
    if dtype == "bf16":
        bound = bound + bf16_ulp(ref)
    bad = err > bound
    if bad.any():
        i = int(np.flatnonzero(bad.reshape(-1))[0])
        raise AssertionError("%s: %d elements out of bound; first at %d: got %r ref %r "
                             "bound %.3e" % (what, int(bad.sum()), i, got.reshape(-1)[i],
                                             ref.reshape(-1)[i], bound.reshape(-1)[i]))


def sample_rows(w: workloads.Workload, count: int, seed: int, mode: str) -> np.ndarray:
    """Flattened (b*H + h)*N + n rows: random ones plus the edges that matter
    (first/last token of a head, both sides of every few block edges)."""
    rng = np.random.default_rng(seed)
    heads = w.B * w.H
    rows = set(int(r) for r in rng.integers(0, heads * w.N, size=count))
    for hh in (0, heads - 1):
        base = hh * w.N
        rows.update((base, base + 1, base + w.N - 1))
        if mode == "block_causal":
            for b in range(1, w.N // w.block_tokens, max(1, (w.N // w.block_tokens) // 4)):
                rows.update((base + b * w.block_tokens - 1, base + b * w.block_tokens))
        if mode == "token_causal":
            # both sides of 128-token chunk edges
            for c in range(1, (w.N + 127) // 128, max(1, (w.N // 128) // 6)):
                rows.update((base + 128 * c - 1, base + 128 * c))
    return np.array(sorted(rows), dtype=np.int64)
