"""GPU parity of the linear cross-attention entry point (queries of one
sequence reading the state of another, no RoPE) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_parity, to64, upload

pytestmark = pytest.mark.gpu

# name, B, H, query tokens, key/value tokens, D, dtype, gate
CASES = [
    ("d64_300q_77kv", 2, 3, 300, 77, 64, "bf16", False),
    ("d64_ragged_long_kv", 1, 4, 257, 1000, 64, "bf16", True),
    ("d64_one_key", 1, 2, 129, 1, 64, "bf16", False),
    ("d128_gate_ragged", 1, 2, 333, 130, 128, "bf16", True),
    ("d128_one_query", 2, 2, 1, 300, 128, "bf16", False),
    ("f32_d32_gate", 2, 2, 100, 45, 32, "f32", True),
    ("f32_d64", 1, 3, 70, 200, 64, "f32", False),
]


def _inputs(name, B, H, Nq, Nkv, D, dtype, gate, seed=41):
    mk = workloads.Workload
    wq = mk(name + "_q", B=B, H=H, N=Nq, D=D, dtype=dtype, seed=seed, gate=gate)
    wk = mk(name + "_kv", B=B, H=H, N=Nkv, D=D, dtype=dtype, seed=seed + 1)
    xq, xk = workloads.make_inputs(wq), workloads.make_inputs(wk)
    return wq, xq, xk, upload(wq, xq), upload(wk, xk)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_cross_attention_matches_oracle(case):
    name, B, H, Nq, Nkv, D, dtype, gate = case
    wq, xq, xk, tq, tk = _inputs(*case)
    out = la.cross_forward(tq["q"], tk["k"], tk["v"], tq.get("g"), eps=wq.eps)
    torch.cuda.synchronize()
    ref = oracle.cross_forward(xq["q"], xk["k"], xk["v"], g=xq.get("g"), eps=wq.eps)
    assert_parity(to64(out), ref, dtype, name)


def test_cross_attention_video_to_text_shape():
    # 480p latent tokens of a head group reading a 300-token prompt, the
    # tensor-core path at D = 64
    case = ("video_text", 1, 8, 2 * 30 * 52, 300, 64, "bf16", False)
    wq, xq, xk, tq, tk = _inputs(*case, seed=51)
    assert la.uses_tensor_cores(1, 8, 300, 64, torch.bfloat16)
    ws = la.Workspace(la._native.lin_attn_cross_workspace_size(
        la.make_params(1, 8, 2 * 30 * 52, 64, torch.bfloat16), 300), tq["q"].device)
    a = la.cross_forward(tq["q"], tk["k"], tk["v"], workspace=ws)
    b = la.cross_forward(tq["q"], tk["k"], tk["v"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert ws.control_block_is_zero() and ws.status() == 0
    ref = oracle.cross_forward(xq["q"], xk["k"], xk["v"], eps=wq.eps)
    assert_parity(to64(a), ref, "bf16", "video_text")


def test_cross_attention_equal_lengths_is_self_attention():
    # with the same sequence on both sides and no RoPE the cross entry point
    # is the bidirectional forward: same kernels, same bits
    case = ("self", 1, 3, 500, 500, 64, "bf16", True)
    wq, xq, xk, tq, tk = _inputs(*case, seed=61)
    a = la.cross_forward(tq["q"], tq["q"], tq["q"], tq["g"])
    b = la.forward(tq["q"], tq["q"], tq["q"], tq["g"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)
