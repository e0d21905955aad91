"""GPU parity at head dim 112 (the SANA-Video 2B model's head dim: 56 rotary
pairs split over t, h, w) against the fp64 oracle, in every mode and for
cross-attention: bf16 forwards on the tensor-core kernels (112-wide rows on
the 128 kernels), fp32, token-causal and block steps on the CUDA-core ones."""
import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_parity, run_forward, sample_rows, to64, upload

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
    tc = la.uses_tensor_cores(w.B, w.H, w.N, w.D, torch.bfloat16 if w.dtype == "bf16" else
                              torch.float32, mode=mode,
                              block_tokens=w.block_tokens if mode == "block_causal" else 0,
                              grid=w.grid, rope_split=w.rope_split)
    assert tc == (w.dtype == "bf16" and mode != "token_causal")
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


def test_head_dim_112_block_steps():
    # block steps carry a 112 x 112 state: CUDA-core kernels, against the
    # oracle's block-causal forward
    w = mk("d112_steps", B=1, H=2, N=3 * 4 * 6, D=112, dtype="bf16", seed=908, grid=(3, 4, 6),
           rope_split=(16, 48, 48), modes=("block_causal",), block_tokens=4 * 6)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    st = la.BlockState(w.B, w.H, w.D)
    bt = w.block_tokens
    outs = [st.step(*(t[n][:, :, b * bt:(b + 1) * bt].contiguous() for n in ("q", "k", "v")),
                    t_offset=b, grid=(1, 4, 6), rope_split=w.rope_split, eps=w.eps)
            for b in range(3)]
    torch.cuda.synchronize()
    ref = oracle.forward(oracle.params_for(w, "block_causal"), x["q"], x["k"], x["v"])
    assert_parity(to64(torch.cat(outs, dim=2)), ref, "bf16", "d112 block steps")
    # a read-only step (commit off) leaves the state byte for byte as it was
    # and gives the output the committing step gives
    S0, z0 = st.S.clone(), st.z.clone()
    blk = [t[n][:, :, :bt].contiguous() for n in ("q", "k", "v")]
    kw = dict(t_offset=3, grid=(1, 4, 6), rope_split=w.rope_split, eps=w.eps)
    a = st.step(*blk, commit=False, **kw)
    torch.cuda.synchronize()
    assert torch.equal(st.S, S0) and torch.equal(st.z, z0)
    b = st.step(*blk, commit=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert not torch.equal(st.S, S0)


def test_head_dim_112_480p_full_size_sampled_rows():
    # the 2B model's attention at 480p (20 heads of 112, 21 x 30 x 52 tokens)
    # on the tensor-core kernels, checked on sampled rows
    w = mk("d112_480p", B=1, H=20, N=21 * 30 * 52, D=112, dtype="bf16", seed=909,
           grid=(21, 30, 52), rope_split=(16, 48, 48))
    x = workloads.make_inputs(w)
    t = upload(w, x)
    out = run_forward(w, t, "bidirectional")
    rows = sample_rows(w, 192, seed=w.seed, mode="bidirectional")
    got = to64(out.view(-1, w.D)[torch.from_numpy(rows).cuda()])
    ref = oracle.forward_rows(oracle.params_for(w, "bidirectional"), x["q"], x["k"], x["v"], rows)
    assert_parity(got, ref, "bf16", "d112 480p sampled")
