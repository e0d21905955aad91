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


def assert_parity(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    rel, mx = errors(got, ref)
    if dtype == "bf16":
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, \
            "%s: rel-L2 %.3e (<= %.0e), max-abs %.3e (<= %.0e)" % (what, rel, BF16_REL_L2, mx,
                                                                BF16_MAX_ABS)
    else:
        assert rel <= F32_REL_L2, "%s: rel-L2 %.3e (<= %.0e)" % (what, rel, F32_REL_L2)
    assert np.all(np.isfinite(got)), what
    return rel, mx


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
    return np.array(sorted(rows), dtype=np.int64)
