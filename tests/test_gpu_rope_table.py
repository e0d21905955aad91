"""GPU: the 3D RoPE cos/sin table that a call builds on the device (the
rotation of Eq. 2, SANA-Video paper-graph page, section 3.4) against fp64
cos/sin of pos * theta^(-2m/d), entry by entry, at the large angles of the
720p/60 s latent grid (t up to 239, so angles up to 239 rad on the first
t pair).

The table sits right after the workspace's control block: per axis (t, h, w)
and position a row of ceil(half/4) groups of 8 floats (cos of 4 pairs, then
their sin) and 4 padding floats; pairs past `half` in the last group hold
cos 1, sin 0. The t positions of a call are t_offset + local frame.

Bound: 4 fp32 ulps of 1.0 (2^-22) absolute. The angle is formed as a float
sum hi + lo carrying ~2^-48 relative, reduced exactly by multiples of 2 pi,
so the only error left is the final fp32 sin/cos (a couple of ulps).
"""
import numpy as np
import pytest
import torch

import workloads
import linear_attention_video_relu_b200 as la
from linear_attention_video_relu_b200 import _native as C

pytestmark = pytest.mark.gpu

TOL = 2.0 ** -22


def _stride(half):
    return 0 if half == 0 else 4 * ((half + 3) // 4) + 2


def check_table(buf: torch.Tensor, grid, split, theta, t_offset, what):
    T, Hg, Wg = grid
    halves = [d // 2 for d in split]
    strides = [_stride(h) for h in halves]
    offs = [0, T * strides[0], T * strides[0] + Hg * strides[1]]
    entries = offs[2] + Wg * strides[2]
    start = C.LA_WORKSPACE_CONTROL_BYTES
    tab = buf[start:start + 8 * entries].cpu().numpy().view(np.float32).astype(np.float64)
    worst = 0.0
    for a, (npos, half) in enumerate(zip((T, Hg, Wg), halves)):
        if half == 0:
            continue
        G = (half + 3) // 4
        rows = tab[2 * offs[a]:2 * (offs[a] + npos * strides[a])].reshape(npos, 2 * strides[a])
        pos = np.arange(npos, dtype=np.float64) + (t_offset if a == 0 else 0)
        m = np.arange(4 * G)
        freq = np.where(m < half, float(theta) ** (-m / half), 0.0)   # theta^(-2m/d), d = 2 half
        ang = pos[:, None] * freq[None, :]
        want_c = np.where(m < half, np.cos(ang), 1.0)
        want_s = np.where(m < half, np.sin(ang), 0.0)
        got_c = rows[:, :8 * G].reshape(npos, G, 2, 4)[:, :, 0, :].reshape(npos, 4 * G)
        got_s = rows[:, :8 * G].reshape(npos, G, 2, 4)[:, :, 1, :].reshape(npos, 4 * G)
        err = max(np.abs(got_c - want_c).max(), np.abs(got_s - want_s).max())
        assert err <= TOL, "%s axis %d: max |error| %.3e > %.3e" % (what, a, err, TOL)
        assert np.all(rows[:, 8 * G:8 * G + 4] == 0.0), "%s axis %d: padding" % (what, a)
        worst = max(worst, err)
    return worst


def test_720p_grid_table_forward_d64():
    # one head over the whole 720p/60 s grid (240 x 23 x 40), split 16/24/24
    w = workloads.Workload("rope_720p", B=1, H=1, N=240 * 23 * 40, D=64, dtype="bf16",
                           seed=1201, grid=(240, 23, 40), rope_split=(16, 24, 24))
    t = {n: torch.randn((1, 1, w.N, 64), device="cuda").to(torch.bfloat16) for n in "qkv"}
    p = la.make_params(1, 1, w.N, 64, torch.bfloat16, "bidirectional", 0, w.grid, w.rope_split,
                       w.rope_theta, w.eps)
    ws = la.workspace_for(p, "cuda")
    la.forward(t["q"], t["k"], t["v"], grid=w.grid, rope_split=w.rope_split, workspace=ws)
    torch.cuda.synchronize()
    assert la.uses_tensor_cores(1, 1, w.N, 64, torch.bfloat16, grid=w.grid,
                                rope_split=w.rope_split)
    check_table(ws.buf, w.grid, w.rope_split, w.rope_theta, 0, "720p d64")


@pytest.mark.parametrize("dtype,D,split", [(torch.bfloat16, 128, (32, 48, 48)),
                                           (torch.float32, 64, (16, 24, 24))],
                         ids=["tc_d128", "simt_f32"])
def test_block_step_table_at_a_late_frame_offset(dtype, D, split):
    # the last 4 frames of the 720p grid as one block step: t = 236 .. 239
    grid = (4, 23, 40)
    N = 4 * 23 * 40
    st = la.BlockState(1, 2, D)
    q, k, v = (torch.randn((1, 2, N, D), device="cuda").to(dtype) for _ in range(3))
    st.step(q, k, v, t_offset=236, commit=False, grid=grid, rope_split=split)
    torch.cuda.synchronize()
    (ws,) = st._ws.values()
    check_table(ws.buf, grid, split, 10000.0, 236, "block step %s D=%d" % (dtype, D))
