"""smoke()'s logic on the CPU: the same passes run through stand-ins for the
CUDA calls (the oracle, rounded to bf16 like the GPU output), so a slip in the
smoke code itself shows here rather than on the GPU. It checks the harness,
not the kernels."""
import types

import numpy as np
import torch

import __graft_entry__
import oracle
from oracle import tconv


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def _f64(t):
    return None if t is None else t.float().numpy().astype(np.float64)


def _stand_in():
    calls = []

    def forward(q, k, v, g=None, *, mode, block_tokens, grid, rope_split, theta, eps):
        calls.append("forward/" + mode)
        B, H, N, D = q.shape
        p = oracle.make_params(B, H, N, D, mode=mode, block_tokens=block_tokens, grid=grid,
                               rope_split=rope_split, theta=theta, eps=eps)
        return _bf16(oracle.forward(p, _f64(q), _f64(k), _f64(v), g=_f64(g)))

    def cross_forward(q, k, v, g=None):
        calls.append("cross")
        return _bf16(oracle.cross_forward(_f64(q), _f64(k), _f64(v), g=_f64(g)))

    def temporal_conv(x, weight, bias, cache_in, *, cache_out):
        calls.append("temporal_conv")
        y, last = tconv.temporal_conv(_f64(x), weight.numpy(), bias.numpy(), _f64(cache_in))
        cache_out.copy_(_bf16(last))
        return _bf16(y)

    def uses_tensor_cores(*a, **k):
        return True

    la = types.SimpleNamespace(forward=forward, cross_forward=cross_forward,
                               temporal_conv=temporal_conv, uses_tensor_cores=uses_tensor_cores)
    return la, calls


def test_smoke_logic_with_stand_ins(capsys):
    oracle.build()
    la, calls = _stand_in()
    __graft_entry__._smoke_checks(torch.device("cpu"), la, lambda: None)
    assert calls == ["forward/bidirectional", "forward/block_causal", "cross", "temporal_conv"]
    out = capsys.readouterr().out
    for name in ("smoke_gated ok", "smoke_block ok", "cross ok", "temporal_conv ok"):
        assert "smoke " + name in out
