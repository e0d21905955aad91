"""GPU: [B, N, H, D] inputs (the order a fused QKV projection writes) give the
same outputs, bit for bit, as the same tensors in [B, H, N, D] order, on
every kernel family and mode; one case is also checked against the oracle."""
import dataclasses

import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_parity, to64, upload

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
mk = workloads.Workload


def _bnhd(t):
    return None if t is None else t.transpose(1, 2).contiguous()


CASES = [
    (W["480p_bidir"].scaled(2), "bidirectional"),                          # tensor cores, D 64
    (W["480p_block_causal"].scaled(6), "block_causal"),                     # + block scan
    (dataclasses.replace(W["gated_d128"], B=2).scaled(2), "bidirectional"),  # D 128, gate
    (mk("bnhd_d112", B=2, H=3, N=3 * 6 * 10, D=112, dtype="bf16", seed=1101, grid=(3, 6, 10),
        rope_split=(16, 48, 48), gate=True), "bidirectional"),              # 112 on the 128 kernels
    (mk("bnhd_f32", B=2, H=3, N=100, D=32, dtype="f32", seed=1102, gate=True), "bidirectional"),
    (mk("bnhd_token_causal", B=2, H=2, N=2 * 5 * 7, D=64, dtype="bf16", seed=1103,
        grid=(2, 5, 7), rope_split=(16, 24, 24)), "token_causal"),
]


@pytest.mark.parametrize("w,mode", CASES, ids=[c[0].name + "-" + c[1] for c in CASES])
def test_bnhd_equals_bhnd_bitwise(w, mode):
    t = upload(w, workloads.make_inputs(w))
    kw = dict(mode=mode, block_tokens=w.block_tokens if mode == "block_causal" else 0,
              grid=w.grid, rope_split=w.rope_split, theta=w.rope_theta, eps=w.eps)
    a = la.forward(t["q"], t["k"], t["v"], t.get("g"), **kw)
    b = la.forward(_bnhd(t["q"]), _bnhd(t["k"]), _bnhd(t["v"]), _bnhd(t.get("g")),
                   layout="bnhd", **kw)
    torch.cuda.synchronize()
    assert torch.equal(_bnhd(a), b)


def test_bnhd_matches_oracle():
    w = mk("bnhd_oracle", B=2, H=3, N=2 * 7 * 9, D=64, dtype="bf16", seed=1104, grid=(2, 7, 9),
           rope_split=(16, 24, 24), gate=True)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    out = la.forward(_bnhd(t["q"]), _bnhd(t["k"]), _bnhd(t["v"]), _bnhd(t["g"]),
                     grid=w.grid, rope_split=w.rope_split, layout="bnhd")
    torch.cuda.synchronize()
    ref = oracle.forward(oracle.params_for(w, "bidirectional"), x["q"], x["k"], x["v"], g=x["g"])
    assert_parity(to64(out.transpose(1, 2)), ref, "bf16", "bnhd")


def test_bnhd_cross_attention_and_block_steps():
    wq = mk("bnhd_q", B=2, H=2, N=150, D=64, dtype="bf16", seed=1105, gate=True)
    wk = mk("bnhd_kv", B=2, H=2, N=40, D=64, dtype="bf16", seed=1106)
    tq, tk = upload(wq, workloads.make_inputs(wq)), upload(wk, workloads.make_inputs(wk))
    a = la.cross_forward(tq["q"], tk["k"], tk["v"], tq["g"])
    b = la.cross_forward(_bnhd(tq["q"]), _bnhd(tk["k"]), _bnhd(tk["v"]), _bnhd(tq["g"]),
                         layout="bnhd")
    torch.cuda.synchronize()
    assert torch.equal(_bnhd(a), b)
    # two block steps, each block's tensors in [B, N, H, D]
    w = mk("bnhd_steps", B=1, H=2, N=2 * 4 * 6, D=64, dtype="bf16", seed=1107, grid=(2, 4, 6),
           rope_split=(16, 24, 24))
    t = upload(w, workloads.make_inputs(w))
    s1, s2 = la.BlockState(1, 2, 64), la.BlockState(1, 2, 64)
    for blk in range(2):
        sl = [t[n][:, :, blk * 24:(blk + 1) * 24].contiguous() for n in ("q", "k", "v")]
        o1 = s1.step(*sl, t_offset=blk, grid=(1, 4, 6), rope_split=w.rope_split)
        o2 = s2.step(*(_bnhd(x) for x in sl), t_offset=blk, grid=(1, 4, 6),
                     rope_split=w.rope_split, layout="bnhd")
        torch.cuda.synchronize()
        assert torch.equal(_bnhd(o1), o2)
    assert torch.equal(s1.S, s2.S) and torch.equal(s1.z, s2.z)
