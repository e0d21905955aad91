"""GPU parity at head dim 112 (the SANA-Video 2B model's head dim: 56 rotary
pairs split over t, h, w) on the CUDA-core kernels, against the fp64 oracle,
in every mode and for cross-attention."""
import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_parity, run_forward, to64, upload

pytestmark = pytest.mark.gpu

mk = workloads.Workload
CASES = [
    (mk("d112_bidir", B=1, H=3, N=3 * 6 * 10, D=112, dtype="bf16", seed=901, grid=(3, 6, 10),
        rope_split=(16, 48, 48)), "bidirectional"),
    (mk("d112_blocks", B=2, H=2, N=4 * 5 * 6, D=112, dtype="bf16", seed=902, grid=(4, 5, 6),
        rope_split=(32, 40, 40), modes=("block_causal",), block_tokens=2 * 5 * 6), "block_causal"),
    (mk("d112_f32_gate", B=1, H=2, N=100, D=112, dtype="f32", seed=903, gate=True),
     "bidirectional"),
    (mk("d112_token_causal", B=1, H=2, N=2 * 5 * 7, D=112, dtype="bf16", seed=904,
        grid=(2, 5, 7), rope_split=(16, 48, 48), modes=("token_causal",)), "token_causal"),
    (mk("d112_480p_two_frames", B=1, H=4, N=2 * 30 * 52, D=112, dtype="bf16", seed=905,
        grid=(2, 30, 52), rope_split=(16, 48, 48), gate=True), "bidirectional"),
]


@pytest.mark.parametrize("w,mode", CASES, ids=[c[0].name for c in CASES])
def test_head_dim_112_matches_oracle(w, mode):
    assert not la.uses_tensor_cores(w.B, w.H, w.N, w.D, torch.bfloat16, grid=w.grid,
                                    rope_split=w.rope_split)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    got = to64(run_forward(w, t, mode))
    ref = oracle.forward(oracle.params_for(w, mode), x["q"], x["k"], x["v"], g=x.get("g"))
    assert_parity(got, ref, w.dtype, w.name)


def test_head_dim_112_cross_attention():
    wq = mk("d112_q", B=2, H=2, N=90, D=112, dtype="bf16", seed=906, gate=True)
    wk = mk("d112_kv", B=2, H=2, N=33, D=112, dtype="bf16", seed=907)
    xq, xk = workloads.make_inputs(wq), workloads.make_inputs(wk)
    tq, tk = upload(wq, xq), upload(wk, xk)
    out = la.cross_forward(tq["q"], tk["k"], tk["v"], tq["g"])
    torch.cuda.synchronize()
    ref = oracle.cross_forward(xq["q"], xk["k"], xk["v"], g=xq["g"])
    assert_parity(to64(out), ref, "bf16", "d112 cross")
