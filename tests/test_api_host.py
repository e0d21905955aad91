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
