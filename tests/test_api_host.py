"""Host-side argument checks of the torch wrapper, on CPU tensors: shape,
dtype, contiguity and one device for every tensor of a call."""
import pytest
import torch

from linear_attention_video_relu_b200 import api


def _p(dtype=torch.bfloat16):
    return api.make_params(1, 2, 6, 32, dtype)


def test_io_shape_dtype_and_layout():
    q = torch.zeros((1, 2, 6, 32), dtype=torch.bfloat16)
    api._check_io(_p(), q, q.clone(), None, require_cuda=False)
    with pytest.raises(ValueError):
        api._check_io(_p(), torch.zeros((1, 2, 5, 32), dtype=torch.bfloat16), require_cuda=False)
    with pytest.raises(TypeError):      # an fp32 gate beside bf16 q, k, v
        api._check_io(_p(), q, torch.zeros((1, 2, 6, 32)), require_cuda=False)
    with pytest.raises(ValueError):     # a strided view
        api._check_io(_p(), torch.zeros((1, 2, 32, 6), dtype=torch.bfloat16).transpose(2, 3),
                      require_cuda=False)
    with pytest.raises(ValueError):     # host memory is refused on the product path
        api._check_io(_p(), q)


def test_one_device_per_call():
    a = torch.zeros(4)
    api._same_device(a, a.clone(), None)
    with pytest.raises(ValueError):
        api._same_device(a, torch.zeros(4, device="meta"))


def test_fp32_params_want_fp32_tensors():
    x = torch.zeros((1, 2, 6, 32))
    api._check_io(_p(torch.float32), x, require_cuda=False)
    with pytest.raises(TypeError):
        api._check_io(_p(torch.float32), x.to(torch.bfloat16), require_cuda=False)


def test_bnhd_shapes():
    p = api.make_params(1, 2, 6, 32, torch.bfloat16, layout="bnhd")
    api._check_io(p, torch.zeros((1, 6, 2, 32), dtype=torch.bfloat16), require_cuda=False)
    with pytest.raises(ValueError):
        api._check_io(p, torch.zeros((1, 2, 6, 32), dtype=torch.bfloat16), require_cuda=False)
    assert api._dims(torch.zeros((1, 6, 2, 32)), "bnhd") == (1, 2, 6, 32)
    assert api._dims(torch.zeros((1, 2, 6, 32)), "bhnd") == (1, 2, 6, 32)
    with pytest.raises(ValueError):
        api.make_params(1, 2, 6, 32, torch.bfloat16, layout="nbhd")


def test_block_state_plan_cache(monkeypatch):
    """BlockState keeps one (params, workspace) per distinct call: the same
    call reuses it, and any change of shape, dtype, grid, split, theta, eps or
    layout gets params of its own with that setting (a key that missed one
    would run a later call with an earlier call's eps or grid)."""
    made = []

    def fake_workspace(p, device, block_step=False):
        assert block_step
        made.append((p.N, p.D))
        return object()

    monkeypatch.setattr(api, "workspace_for", fake_workspace)
    st = object.__new__(api.BlockState)
    st.S = torch.zeros(1)
    st._ws, st._plans = {}, {}
    q = torch.zeros((1, 2, 24, 64), dtype=torch.bfloat16)
    grid, split = (2, 3, 4), (16, 24, 24)
    p1, w1 = st._plan(q, grid, split, 10000.0, 1e-6, "bhnd")
    p2, w2 = st._plan(q, list(grid), list(split), 10000.0, 1e-6, "bhnd")
    assert p2 is p1 and w2 is w1 and len(made) == 1
    assert (p1.N, p1.D, p1.grid_t, p1.rope_dh) == (24, 64, 2, 24)
    p3, w3 = st._plan(q, grid, split, 10000.0, 1e-5, "bhnd")
    assert p3 is not p1 and abs(p3.eps - 1e-5) < 1e-12
    p4, w4 = st._plan(q, grid, split, 500.0, 1e-6, "bhnd")
    assert p4 is not p1 and p4.rope_theta == 500.0
    # eps and theta do not size the workspace: it is shared
    assert w3 is w1 and w4 is w1 and len(made) == 1
    p5, _ = st._plan(q, (2, 4, 3), split, 10000.0, 1e-6, "bhnd")
    assert p5 is not p1 and (p5.grid_h, p5.grid_w) == (4, 3)
    p6, _ = st._plan(q, grid, (16, 16, 32), 10000.0, 1e-6, "bhnd")
    assert p6 is not p1 and p6.rope_dw == 32
    p7, _ = st._plan(q, None, None, 10000.0, 1e-6, "bhnd")
    assert p7 is not p1 and p7.rope == 0
    p8, _ = st._plan(torch.zeros((1, 24, 2, 64), dtype=torch.bfloat16), grid, split, 10000.0,
                     1e-6, "bnhd")
    assert p8 is not p1 and (p8.H, p8.N, p8.layout) == (2, 24, api.C.LA_LAYOUT_BNHD)
    p9, _ = st._plan(q.float(), grid, split, 10000.0, 1e-6, "bhnd")
    assert p9 is not p1 and p9.dtype == api.C.LA_F32
    p10, _ = st._plan(torch.zeros((1, 2, 12, 64), dtype=torch.bfloat16), (1, 3, 4), split,
                      10000.0, 1e-6, "bhnd")
    assert p10.N == 12 and made[-1] == (12, 64)
    # a workspace per grid, split, RoPE on/off, layout, dtype and N
    assert len(made) == 7
