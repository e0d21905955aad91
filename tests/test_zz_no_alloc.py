"""lin_attn_forward_noalloc: the forward for callers that cannot allocate a
device workspace (a plugin inside an engine that pre-plans all device memory,
a real-time loop that must not call cudaMalloc). It runs on a fixed scratch
array inside the library instead of a caller workspace.

Checked through the C ABI against lin_attn_forward (which takes a caller
workspace) on two calls in a row with different inputs, so stale contents of
the shared scratch from the first call would show up in the second. Both run
the same deterministic kernels in the same fixed reduction order, so the two
outputs must be equal bit for bit; each call is also checked against the
fp64 oracle. This file is collected last on purpose; it must also pass when
run alone.
"""
import dataclasses

import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_parity, to64, upload

pytestmark = pytest.mark.gpu

C = la._native


def _params(w, dtype):
    return la.make_params(w.B, w.H, w.N, w.D, dtype, "bidirectional", 0, w.grid, w.rope_split,
                          w.rope_theta, w.eps)


def _with_workspace(p, t, stream):
    ws = la.workspace_for(p, t["q"].device)
    out = torch.empty_like(t["q"])
    C.check(C.lin_attn_forward(p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                               t["g"].data_ptr() if "g" in t else None, out.data_ptr(), ws.ptr,
                               ws.nbytes, stream), "lin_attn_forward")
    return out


def _without_workspace(p, t, stream):
    out = torch.empty_like(t["q"])
    C.check(C.lin_attn_forward_noalloc(p, t["q"].data_ptr(), t["k"].data_ptr(),
                                       t["v"].data_ptr(), t["g"].data_ptr() if "g" in t else None,
                                       out.data_ptr(), stream), "lin_attn_forward_noalloc")
    return out


@pytest.mark.parametrize("base", ["480p_bidir", "gated_d128"])
def test_noalloc_matches_workspace_forward_on_two_calls(base):
    w0 = workloads.WORKLOADS[base]
    w = w0.scaled(3) if base == "480p_bidir" else dataclasses.replace(w0, B=1).scaled(4)
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((w.seed, w.seed + 100)):
        x = workloads.make_inputs(w, seed=seed)
        t = upload(w, x)
        p = _params(w, t["q"].dtype)
        ref = _with_workspace(p, t, stream)
        got = _without_workspace(p, t, stream)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), "noalloc call %d differs from lin_attn_forward" % call
        want = oracle.forward(oracle.params_for(w, "bidirectional"), x["q"], x["k"], x["v"],
                              g=x.get("g"))
        assert_parity(to64(got), want, w.dtype, "noalloc call %d vs oracle" % call)


def test_noalloc_rejects_problems_beyond_the_scratch_limit():
    # 720p block-causal needs a workspace larger than the fixed 32 MiB scratch
    w = workloads.WORKLOADS["720p_long"]
    p = la.make_params(w.B, w.H, w.N, w.D, torch.bfloat16, "block_causal", w.block_tokens,
                       w.grid, w.rope_split, w.rope_theta, w.eps)
    need = C.lin_attn_workspace_size(p)
    assert need > (32 << 20)
    # The size check comes before any launch, so these addresses (aligned,
    # non-overlapping, never dereferenced) only have to pass the host checks.
    base = 1 << 40
    q, k, v, out = (base + i * (1 << 30) for i in range(4))
    rc = C.lin_attn_forward_noalloc(p, q, k, v, None, out,
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == C.LA_ERR_WORKSPACE
