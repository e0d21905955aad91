"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, plus the invariants the equations fix, re-run on the GPU.

Tolerances: bf16 I/O max-abs <= 2e-2 and rel-L2 <= 5e-3; fp32 I/O rel-L2 <= 1e-4.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import (assert_parity, errors, run_forward, sample_rows, to64, upload)

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def small_cases():
    """Reduced copies of the five workloads: same structure, fewer frames."""
    return [
        (W["tiny_f32"], "bidirectional"),
        (W["480p_bidir"].scaled(2), "bidirectional"),
        (W["480p_block_causal"].scaled(6), "block_causal"),
        (W["720p_long"].scaled(8), "bidirectional"),
        (W["720p_long"].scaled(8), "block_causal"),
        (dataclasses.replace(W["gated_d128"], B=2).scaled(4), "bidirectional"),
    ]


def edge_cases():
    mk = workloads.Workload
    return [
        # one token, RoPE on a 1x1x1 grid
        (mk("one_token", B=1, H=3, N=1, D=64, dtype="bf16", seed=11, grid=(1, 1, 1),
            rope_split=(16, 24, 24)), "bidirectional"),
        # ragged: 105 tokens is not a multiple of any tile size
        (mk("ragged_105", B=2, H=3, N=105, D=64, dtype="bf16", seed=12, grid=(3, 5, 7),
            rope_split=(16, 24, 24)), "bidirectional"),
        (mk("ragged_d128", B=1, H=2, N=3 * 5 * 7, D=128, dtype="bf16", seed=13, grid=(3, 5, 7),
            rope_split=(32, 48, 48), gate=True), "bidirectional"),
        # one token per block
        (mk("block_of_one", B=1, H=2, N=24, D=64, dtype="bf16", seed=14, grid=(2, 3, 4),
            rope_split=(16, 24, 24), modes=("block_causal",), block_tokens=1), "block_causal"),
        # blocks that do not align with frames or tiles
        (mk("block_ragged", B=1, H=2, N=4 * 9 * 11, D=64, dtype="bf16", seed=15, grid=(4, 9, 11),
            rope_split=(16, 24, 24), modes=("block_causal",), block_tokens=99), "block_causal"),
        # CUDA-core path: D = 32 in bf16, and fp32 with RoPE, block-causal and gate
        (mk("d32_bf16", B=1, H=4, N=3 * 4 * 5, D=32, dtype="bf16", seed=16, grid=(3, 4, 5),
            rope_split=(8, 12, 12)), "bidirectional"),
        (mk("f32_rope_block", B=2, H=2, N=4 * 4 * 5, D=64, dtype="f32", seed=17, grid=(4, 4, 5),
            rope_split=(16, 24, 24), gate=True, modes=("block_causal",), block_tokens=40),
         "block_causal"),
        (mk("f32_d128", B=1, H=2, N=2 * 4 * 4, D=128, dtype="f32", seed=18, grid=(2, 4, 4),
            rope_split=(32, 48, 48)), "bidirectional"),
        # rope widths that are not multiples of 8 take the CUDA-core kernels
        (mk("odd_split", B=1, H=2, N=2 * 3 * 4, D=64, dtype="bf16", seed=19, grid=(2, 3, 4),
            rope_split=(20, 22, 22)), "bidirectional"),
        # no RoPE in bf16
        (mk("no_rope_bf16", B=1, H=2, N=300, D=64, dtype="bf16", seed=20), "bidirectional"),
        # D = 128 without a gate (output stored from registers), several tiles and a
        # ragged tail, bidirectional and in blocks that split tiles
        (mk("d128_ragged_tiles", B=1, H=3, N=3 * 7 * 13, D=128, dtype="bf16", seed=21,
            grid=(3, 7, 13), rope_split=(32, 48, 48)), "bidirectional"),
        (mk("d128_blocks", B=1, H=3, N=3 * 7 * 13, D=128, dtype="bf16", seed=22,
            grid=(3, 7, 13), rope_split=(32, 48, 48), gate=True, modes=("block_causal",),
            block_tokens=91), "block_causal"),
        # D = 128 with a gate and a RoPE table too large for a two-tile gate
        # ring (2 x 3 x 134: 3598 entries): the apply kernel's one-tile ring
        (mk("d128_wide_table", B=1, H=2, N=2 * 3 * 134, D=128, dtype="bf16", seed=25,
            grid=(2, 3, 134), rope_split=(32, 48, 48), gate=True), "bidirectional"),
        (mk("d128_wide_table_blocks", B=1, H=2, N=2 * 3 * 134, D=128, dtype="bf16", seed=26,
            grid=(2, 3, 134), rope_split=(32, 48, 48), gate=True, modes=("block_causal",),
            block_tokens=402), "block_causal"),
        # thousands of one-tile heads: a CTA completes more heads than it can
        # leave to its tail and reduces the rest on the spot
        (mk("many_small_heads", B=64, H=128, N=16, D=64, dtype="bf16", seed=23,
            grid=(1, 4, 4), rope_split=(16, 24, 24)), "bidirectional"),
        # more heads than the workspace has arrival counters: the separate
        # reduction kernel takes over
        (mk("counter_overflow", B=136, H=128, N=8, D=64, dtype="bf16", seed=24,
            grid=(1, 2, 4), rope_split=(16, 24, 24)), "bidirectional"),
    ]


def token_causal_cases():
    """Per-token causal attention (Eq. 3): chunks of 32 tokens, ragged tails."""
    mk = workloads.Workload
    return [
        mk("tc_one_token", B=1, H=2, N=1, D=64, dtype="bf16", seed=31, grid=(1, 1, 1),
           rope_split=(16, 24, 24), modes=("token_causal",)),
        mk("tc_ragged_105", B=2, H=2, N=3 * 5 * 7, D=64, dtype="bf16", seed=32, grid=(3, 5, 7),
           rope_split=(16, 24, 24), modes=("token_causal",)),
        mk("tc_f32_gate", B=1, H=3, N=100, D=32, dtype="f32", seed=33, gate=True,
           modes=("token_causal",)),
        mk("tc_d128_gate", B=1, H=2, N=2 * 4 * 6, D=128, dtype="bf16", seed=34, grid=(2, 4, 6),
           rope_split=(32, 48, 48), gate=True, modes=("token_causal",)),
        dataclasses.replace(W["480p_bidir"].scaled(1), name="tc_480p_1frame",
                            modes=("token_causal",)),
        # tensor-core path: one 128-token tile per CTA (each CTA starts from
        # the sum of up to 39 earlier partials of its head)
        mk("tc_multi_cta", B=1, H=3, N=5 * 32 * 32, D=64, dtype="bf16", seed=35,
           grid=(5, 32, 32), rope_split=(16, 24, 24), modes=("token_causal",)),
        # ranges of one or two tiles that cross head boundaries, with the gate
        mk("tc_span_heads_gate", B=1, H=5, N=4 * 37 * 32, D=64, dtype="bf16", seed=36,
           grid=(4, 37, 32), rope_split=(16, 24, 24), gate=True, modes=("token_causal",)),
        # no RoPE, a ragged last tile
        mk("tc_no_rope", B=2, H=2, N=300, D=64, dtype="bf16", seed=37,
           modes=("token_causal",)),
    ]


def _check_against_oracle(w, mode):
    x = workloads.make_inputs(w)
    t = upload(w, x)
    got = to64(run_forward(w, t, mode))
    ref = oracle.forward(oracle.params_for(w, mode), x["q"], x["k"], x["v"], g=x.get("g"))
    return assert_parity(got, ref, w.dtype, "%s/%s" % (w.name, mode))


@pytest.mark.parametrize("w,mode", small_cases(), ids=lambda c: getattr(c, "name", c))
def test_small_workloads_match_oracle(w, mode):
    _check_against_oracle(w, mode)


@pytest.mark.parametrize("w,mode", edge_cases(), ids=lambda c: getattr(c, "name", c))
def test_edge_cases_match_oracle(w, mode):
    _check_against_oracle(w, mode)


@pytest.mark.parametrize("w", token_causal_cases(), ids=lambda c: c.name)
def test_token_causal_matches_oracle(w):
    _check_against_oracle(w, "token_causal")


FULL = [("480p_bidir", "bidirectional"), ("480p_block_causal", "block_causal"),
        ("720p_long", "bidirectional"), ("720p_long", "block_causal"),
        ("gated_d128", "bidirectional"), ("480p_bidir", "token_causal")]


@pytest.mark.parametrize("name,mode", FULL)
def test_full_size_sampled_rows(name, mode):
    """Full-size workloads in the benchmark's launch configuration, checked on
    sampled rows (random, plus head and block edges) the oracle computes one
    by one, and on properties of the whole output."""
    w = W[name]
    x = workloads.make_inputs(w)
    t = upload(w, x)
    out = run_forward(w, t, mode)
    assert bool(torch.isfinite(out).all())
    rows = sample_rows(w, 192, seed=w.seed, mode=mode)
    got = to64(out.view(-1, w.D)[torch.from_numpy(rows).cuda()])
    ref = oracle.forward_rows(oracle.params_for(w, mode), x["q"], x["k"], x["v"], rows,
                              g=x.get("g"))
    assert_parity(got, ref, w.dtype, "%s/%s sampled" % (name, mode))


def test_deterministic_bitwise():
    w = W["480p_bidir"].scaled(3)
    t = upload(w, workloads.make_inputs(w))
    a = run_forward(w, t, "bidirectional")
    b = run_forward(w, t, "bidirectional")
    assert torch.equal(a, b)
    wc = W["480p_block_causal"].scaled(6)
    tc = upload(wc, workloads.make_inputs(wc))
    assert torch.equal(run_forward(wc, tc, "block_causal"), run_forward(wc, tc, "block_causal"))
    assert torch.equal(run_forward(w, t, "token_causal"), run_forward(w, t, "token_causal"))


def test_one_block_equals_bidirectional():
    w = dataclasses.replace(W["480p_bidir"].scaled(2), block_tokens=2 * 30 * 52)
    t = upload(w, workloads.make_inputs(w))
    a = run_forward(w, t, "bidirectional")
    b = run_forward(w, t, "block_causal")
    assert torch.equal(a, b)


def _block_view(x, b, bt):
    return x[:, :, b * bt:(b + 1) * bt].contiguous()


@pytest.mark.parametrize("grid,fpb", [((4, 6, 8), 2), ((8, 6, 8), 4), ((4, 3, 134), 1)],
                         ids=["4x6x8", "8x6x8", "wide_table_4x3x134"])
def test_block_steps_d128_gated_match_oracle(grid, fpb):
    # the carried state at D = 128 with the gate, blocks committed in turn.
    # The state build's tail takes each of its paths: 2 partials per head
    # (the carried state transposed in shared memory), 3 (the partial slots
    # fill the room: carried values read per item), 7 (partials read from
    # L2). A 1 x 3 x 134 block has 3580 RoPE table entries, too many for a
    # two-tile gate ring beside the table (the apply kernel's one-tile ring).
    T, Hg, Wg = grid
    w = workloads.Workload("d128_steps", B=1, H=2, N=T * Hg * Wg, D=128, dtype="bf16",
                           seed=25, grid=grid, rope_split=(32, 48, 48), gate=True,
                           modes=("block_causal",), block_tokens=fpb * Hg * Wg)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    bt = w.block_tokens
    st = la.BlockState(w.B, w.H, w.D)
    outs = [st.step(_block_view(t["q"], b, bt), _block_view(t["k"], b, bt),
                    _block_view(t["v"], b, bt), _block_view(t["g"], b, bt), t_offset=fpb * b,
                    commit=True, grid=(fpb, Hg, Wg), rope_split=w.rope_split, eps=w.eps)
            for b in range(T // fpb)]
    seq = torch.cat(outs, dim=2)
    torch.cuda.synchronize()
    ref = oracle.forward(oracle.params_for(w, "block_causal"), x["q"], x["k"], x["v"],
                         g=x["g"])
    assert_parity(to64(seq), ref, w.dtype, "d128 block steps")


def test_block_steps_match_forward_and_oracle():
    w = W["720p_long"].scaled(12)              # 3 blocks of 4 frames
    x = workloads.make_inputs(w)
    t = upload(w, x)
    fwd = run_forward(w, t, "block_causal")
    bt = w.block_tokens
    T, Hg, Wg = w.grid
    fpb = bt // (Hg * Wg)
    st = la.BlockState(w.B, w.H, w.D)
    outs = []
    for b in range(w.N // bt):
        o = st.step(_block_view(t["q"], b, bt), _block_view(t["k"], b, bt),
                    _block_view(t["v"], b, bt), t_offset=b * fpb, commit=True,
                    grid=(fpb, Hg, Wg), rope_split=w.rope_split, eps=w.eps)
        outs.append(o)
    seq = torch.cat(outs, dim=2)
    torch.cuda.synchronize()
    assert all(ws.control_block_is_zero() for ws in st._ws.values())
    ref = oracle.forward(oracle.params_for(w, "block_causal"), x["q"], x["k"], x["v"])
    assert_parity(to64(seq), ref, w.dtype, "block steps")
    rel, _ = errors(to64(seq), to64(fwd))
    assert rel <= 1e-3
    # the carried state equals the sums over the whole sequence
    S_ref, z_ref = oracle.state(oracle.params_for(w, "bidirectional"), x["k"], x["v"])
    rel_S, _ = errors(st.S.double().cpu().numpy(), S_ref)
    rel_z, _ = errors(st.z.double().cpu().numpy(), z_ref)
    assert rel_S <= 5e-3 and rel_z <= 1e-5, (rel_S, rel_z)


def test_commit_zero_leaves_state_and_matches_commit_output():
    w = W["480p_block_causal"].scaled(6)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    bt = w.block_tokens
    T, Hg, Wg = w.grid
    fpb = bt // (Hg * Wg)
    st = la.BlockState(w.B, w.H, w.D)
    args = dict(grid=(fpb, Hg, Wg), rope_split=w.rope_split, eps=w.eps)
    st.step(_block_view(t["q"], 0, bt), _block_view(t["k"], 0, bt), _block_view(t["v"], 0, bt),
            t_offset=0, commit=True, **args)
    S0, z0 = st.S.clone(), st.z.clone()
    blk = [_block_view(t[n], 1, bt) for n in ("q", "k", "v")]
    o_peek = st.step(*blk, t_offset=fpb, commit=False, **args)
    torch.cuda.synchronize()
    assert torch.equal(st.S, S0) and torch.equal(st.z, z0)
    o_commit = st.step(*blk, t_offset=fpb, commit=True, **args)
    torch.cuda.synchronize()
    assert torch.equal(o_peek, o_commit)
    assert not torch.equal(st.S, S0)
    # resume: restoring the saved state and repeating the block gives the same bits
    S1, z1 = st.S.clone(), st.z.clone()
    st.S.copy_(S0)
    st.z.copy_(z0)
    o_again = st.step(*blk, t_offset=fpb, commit=True, **args)
    torch.cuda.synchronize()
    assert torch.equal(o_again, o_commit) and torch.equal(st.S, S1) and torch.equal(st.z, z1)
    # the cache update alone folds the same sums into the state
    st.S.copy_(S0)
    st.z.copy_(z0)
    st.update(blk[1], blk[2], t_offset=fpb, grid=args["grid"], rope_split=w.rope_split)
    torch.cuda.synchronize()
    assert torch.equal(st.S, S1) and torch.equal(st.z, z1)
    st.reset()
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(st.S)) == 0 and int(torch.count_nonzero(st.z)) == 0


def test_gate_zero_halves_exactly():
    w = dataclasses.replace(W["gated_d128"], B=1).scaled(2)
    x = workloads.make_inputs(w)
    t = upload(w, x)
    plain = run_forward(w, {**t, "g": None}, "bidirectional")
    half = run_forward(w, {**t, "g": torch.zeros_like(t["q"])}, "bidirectional")
    assert torch.equal(half, plain * 0.5)


def test_zero_features_give_zero_output():
    w = W["480p_bidir"].scaled(1)
    t = upload(w, workloads.make_inputs(w))
    o = run_forward(w, {**t, "q": -t["q"].abs()}, "bidirectional")
    assert int(torch.count_nonzero(o)) == 0
    o = run_forward(w, {**t, "k": -t["k"].abs()}, "bidirectional")
    assert int(torch.count_nonzero(o)) == 0


def test_future_blocks_do_not_change_past_outputs():
    w = W["480p_block_causal"].scaled(9)       # 3 blocks
    x = workloads.make_inputs(w)
    t = upload(w, x)
    base = run_forward(w, t, "block_causal")
    cut = 2 * w.block_tokens
    t2 = {n: v.clone() for n, v in t.items()}
    t2["k"][:, :, cut:] = torch.randn_like(t2["k"][:, :, cut:])
    t2["v"][:, :, cut:] = torch.randn_like(t2["v"][:, :, cut:])
    out = run_forward(w, t2, "block_causal")
    assert torch.equal(out[:, :, :cut], base[:, :, :cut])
    assert not torch.equal(out[:, :, cut:], base[:, :, cut:])


def test_workspace_too_small_is_rejected():
    w = W["480p_bidir"].scaled(1)
    t = upload(w, workloads.make_inputs(w))
    p = la.make_params(w.B, w.H, w.N, w.D, torch.bfloat16, grid=w.grid, rope_split=w.rope_split)
    need = la._native.lin_attn_workspace_size(p)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(t["q"])
    s = torch.cuda.current_stream().cuda_stream
    rc = la._native.lin_attn_forward(p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                                     None, out.data_ptr(), ws.data_ptr(), need - 256, s)
    assert rc == la._native.LA_ERR_WORKSPACE
    rc = la._native.lin_attn_forward(p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                                     None, out.data_ptr(), ws.data_ptr() + 16, need, s)
    assert rc == la._native.LA_ERR_WORKSPACE
    rc = la._native.lin_attn_forward(p, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                                     None, out.data_ptr(), ws.data_ptr(), need, s)
    assert rc == la._native.LA_OK
    assert la._native.lin_attn_device_status(ws.data_ptr(), s) == la._native.LA_OK


def test_tensor_core_path_is_selected_for_the_bf16_workloads():
    for name in ("480p_bidir", "480p_block_causal", "720p_long", "gated_d128"):
        w = W[name]
        assert la.uses_tensor_cores(w.B, w.H, w.N, w.D, torch.bfloat16, grid=w.grid,
                                    rope_split=w.rope_split)
    w = W["480p_bidir"]
    assert la.uses_tensor_cores(w.B, w.H, w.N, w.D, torch.bfloat16, mode="token_causal",
                                grid=w.grid, rope_split=w.rope_split)
    # D = 128 on the 720p grid (3628 table entries) and the wide-table case
    for grid in ((21, 45, 80), (2, 3, 134)):
        n = grid[0] * grid[1] * grid[2]
        assert la.uses_tensor_cores(1, 2, n, 128, torch.bfloat16, grid=grid,
                                    rope_split=(32, 48, 48))
    # fp32 I/O, D = 32 and RoPE widths that are not multiples of 8 use CUDA cores
    assert not la.uses_tensor_cores(1, 2, 256, 32, torch.float32)
    assert not la.uses_tensor_cores(1, 4, 60, 32, torch.bfloat16, grid=(3, 4, 5),
                                    rope_split=(8, 12, 12))
    assert not la.uses_tensor_cores(1, 2, 24, 64, torch.bfloat16, grid=(2, 3, 4),
                                    rope_split=(20, 22, 22))


def _chain(call, x0, n=3):
    """n calls enqueued back to back on one stream, each reading the previous
    one's output (as q, and as k where the call takes one), then the same
    calls one at a time after a synchronize: bitwise equal."""
    outs = [x0]
    for _ in range(n):
        outs.append(call(outs[-1]))
    torch.cuda.synchronize()
    for i in range(1, n):
        ref = call(outs[i].clone())
        torch.cuda.synchronize()
        assert torch.equal(outs[i + 1], ref), "call %d of the chain" % (i + 1)


def test_chained_calls_read_the_previous_output():
    # The apply kernel loads its first q (and gate) tiles before its
    # dependency wait, relying on the state build letting it launch only
    # after the state build's own wait: everything before the state build in
    # the stream -- here the previous call's apply kernel, which wrote this
    # call's q and k -- has completed by then.
    w = workloads.Workload("chain_d128", B=2, H=3, N=6 * 8 * 10, D=128, dtype="bf16", seed=31,
                           grid=(6, 8, 10), rope_split=(32, 48, 48), gate=True)
    t = upload(w, workloads.make_inputs(w))
    p = la.make_params(w.B, w.H, w.N, w.D, t["q"].dtype, "bidirectional", 0, w.grid,
                       w.rope_split, w.rope_theta, w.eps)
    ws = la.workspace_for(p, t["q"].device)
    _chain(lambda x: la.forward(x, x, t["v"], t["g"], grid=w.grid, rope_split=w.rope_split,
                                theta=w.rope_theta, eps=w.eps, workspace=ws), t["q"])
    # D = 64 with RoPE (loads after the wait) and cross-attention (no RoPE,
    # loads before it)
    w64 = W["480p_bidir"].scaled(2)
    t64 = upload(w64, workloads.make_inputs(w64))
    p64 = la.make_params(w64.B, w64.H, w64.N, w64.D, t64["q"].dtype, "bidirectional", 0,
                         w64.grid, w64.rope_split, w64.rope_theta, w64.eps)
    ws64 = la.workspace_for(p64, t64["q"].device)
    _chain(lambda x: la.forward(x, x, t64["v"], grid=w64.grid, rope_split=w64.rope_split,
                                theta=w64.rope_theta, eps=w64.eps, workspace=ws64), t64["q"])
    kv = t64["k"][:, :, :300].contiguous(), t64["v"][:, :, :300].contiguous()
    pc = la.make_params(w64.B, w64.H, w64.N, w64.D, t64["q"].dtype, eps=w64.eps)
    wsc = la.Workspace(la._native.lin_attn_cross_workspace_size(pc, 300), t64["q"].device)
    _chain(lambda x: la.cross_forward(x, kv[0], kv[1], eps=w64.eps, workspace=wsc), t64["q"])


@pytest.mark.parametrize("H,D,fgrid,split,gate", [
    (2, 128, (1, 6, 8), (32, 48, 48), True),
    # a 720p block: 32 heads x 3680 tokens, whose apply loads q early and
    # gives its last CTAs half the tiles
    (32, 64, (4, 23, 40), (16, 24, 24), False)], ids=["d128_gated", "720p_block"])
def test_chained_block_steps_read_the_previous_output(H, D, fgrid, split, gate):
    # Algorithm 1's per-block call where the apply kernel loads its first q
    # stages before its dependency wait: each step's q is the previous step's
    # output, enqueued back to back; the same steps made one at a time after a
    # synchronize, from the same starting state, give the same outputs and
    # the same committed state, bit for bit.
    fpb, Hg, Wg = fgrid
    w = workloads.Workload("chain_steps", B=1, H=H, N=3 * fpb * Hg * Wg, D=D, dtype="bf16",
                           seed=32, grid=(3 * fpb, Hg, Wg), rope_split=split, gate=gate)
    t = upload(w, workloads.make_inputs(w))
    bt = fpb * Hg * Wg
    names = ("q", "k", "v", "g") if gate else ("q", "k", "v")
    blk = [{n: t[n][:, :, b * bt:(b + 1) * bt].contiguous() for n in names} for b in range(3)]
    kw = dict(grid=fgrid, rope_split=w.rope_split, eps=w.eps)

    def run(sync):
        st = la.BlockState(w.B, w.H, w.D)
        x = blk[0]["q"]
        outs = []
        for b in range(3):
            x = st.step(x, blk[b]["k"], blk[b]["v"], blk[b].get("g"), t_offset=b * fpb,
                        commit=True, **kw)
            if sync:
                torch.cuda.synchronize()
                x = x.clone()
            outs.append(x)
        torch.cuda.synchronize()
        return outs, st

    a, sa = run(False)
    b, sb = run(True)
    for i in range(3):
        assert torch.equal(a[i], b[i]), "step %d" % i
    assert torch.equal(sa.S, sb.S) and torch.equal(sa.z, sb.z)
