"""GPU parity of the Mix-FFN temporal convolution with its last-frame cache
(lin_attn_temporal_conv) against the fp64 oracle, and the cache's behaviour
over a chain of blocks.

The op is fp32 arithmetic with one rounding per output, so beside the
attention's whole-tensor gate (bf16 max-abs <= 2e-2 and rel-L2 <= 5e-3, fp32
rel-L2 <= 1e-4) every element is checked on its own: within one bf16 ulp of
the fp64 value (bf16 I/O) plus 2^-21 times the sum of the magnitudes of its
terms (the fp32 roundings; all there is of the bound for fp32 I/O).
"""
import numpy as np
import pytest
import torch

import workloads
import linear_attention_video_relu_b200 as la
from gpu_helpers import assert_elementwise, assert_parity, to64
from oracle import tconv

pytestmark = pytest.mark.gpu


def _up(x, name, dtype):
    if name not in x:
        return None
    if dtype == "bf16":
        return torch.from_numpy(x[name + "_bits"]).view(torch.bfloat16).cuda()
    return torch.from_numpy(x[name]).cuda()


def _abs(a):
    return None if a is None else np.abs(np.asarray(a, dtype=np.float64))


def _absum(x, sel=None):
    """Per output element, the sum of the magnitudes of the terms it adds up:
    the convolution of |x| with |w|, |bias| and the |cache| frame."""
    pick = (lambda a: a) if sel is None else (lambda a: a[..., sel])
    return tconv.temporal_conv(_abs(pick(x["x"])), _abs(x["weight"][:, sel] if sel is not None
                                                        else x["weight"]),
                               _abs(pick(x["bias"])) if "bias" in x else None,
                               _abs(pick(x["cache"])) if "cache" in x else None)[0]


def _upload(x, dtype):
    t = {n: _up(x, n, dtype) for n in ("x", "cache")}
    t["weight"] = torch.from_numpy(x["weight"]).cuda()
    t["bias"] = torch.from_numpy(x["bias"]).cuda() if "bias" in x else None
    return t


# name, B, T, S, C, dtype, cache, bias
CASES = [
    ("bf16_small", 2, 5, 7, 40, "bf16", True, True),
    ("bf16_one_frame", 1, 1, 9, 64, "bf16", True, True),
    ("bf16_two_frames_no_cache", 3, 2, 11, 24, "bf16", False, False),
    ("bf16_ragged_columns", 1, 6, 37, 136, "bf16", True, False),
    ("bf16_23_frames", 1, 23, 4, 8, "bf16", False, True),
    ("f32_small", 2, 4, 5, 12, "f32", True, True),
    ("f32_9_frames", 1, 9, 13, 20, "f32", False, True),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_matches_oracle(case):
    name, B, T, S, nc, dtype, with_cache, with_bias = case
    x = workloads.make_tconv_inputs(B, T, S, nc, dtype, seed=700 + len(name),
                                    cache=with_cache, bias=with_bias)
    t = _upload(x, dtype)
    cache_out = torch.empty((B, S, nc), dtype=t["x"].dtype, device="cuda")
    cache_before = None if t["cache"] is None else t["cache"].clone()
    y = la.temporal_conv(t["x"], t["weight"], t["bias"], t["cache"], cache_out=cache_out)
    torch.cuda.synchronize()
    ref, last = tconv.temporal_conv(x["x"], x["weight"], x.get("bias"), x.get("cache"))
    assert_parity(to64(y), ref, dtype, name)
    assert_elementwise(to64(y), ref, _absum(x), dtype, name)
    assert torch.equal(cache_out, t["x"][:, T - 1])
    if cache_before is not None:
        assert torch.equal(t["cache"], cache_before)


def test_blocks_with_an_in_place_cache():
    # Algorithm 1's chain: the first block without a cache, then each block
    # reads and replaces one cache frame in place
    B, T, S, nc, fpb = 2, 9, 30, 64, 3
    x = workloads.make_tconv_inputs(B, T, S, nc, "bf16", seed=801, cache=False)
    t = _upload(x, "bf16")
    cache = torch.empty((B, S, nc), dtype=torch.bfloat16, device="cuda")
    outs = []
    for t0 in range(0, T, fpb):
        xb = t["x"][:, t0:t0 + fpb].contiguous()
        outs.append(la.temporal_conv(xb, t["weight"], t["bias"], None if t0 == 0 else cache,
                                     cache_out=cache))
    torch.cuda.synchronize()
    ref, last = tconv.temporal_conv_blocks(x["x"], x["weight"], fpb, x["bias"])
    assert_parity(to64(torch.cat(outs, dim=1)), ref, "bf16", "blocks")
    absum, _ = tconv.temporal_conv_blocks(_abs(x["x"]), _abs(x["weight"]), fpb, _abs(x["bias"]))
    assert_elementwise(to64(torch.cat(outs, dim=1)), ref, absum, "bf16", "blocks")
    assert torch.equal(cache, t["x"][:, T - 1])


def test_zero_weights_give_the_input_back():
    # the zero-initialised temporal conv leaves the hidden states as they are
    x = workloads.make_tconv_inputs(1, 4, 10, 32, "bf16", seed=802)
    t = _upload(x, "bf16")
    y = la.temporal_conv(t["x"], torch.zeros_like(t["weight"]), None, t["cache"])
    torch.cuda.synchronize()
    assert torch.equal(y, t["x"])


def test_grid_shaped_input():
    # [B, T, Hg, Wg, C] is the same memory as [B, T, Hg*Wg, C]
    x = workloads.make_tconv_inputs(1, 3, 6 * 5, 16, "bf16", seed=803)
    t = _upload(x, "bf16")
    a = la.temporal_conv(t["x"], t["weight"], t["bias"], t["cache"])
    b = la.temporal_conv(t["x"].view(1, 3, 6, 5, 16), t["weight"], t["bias"],
                         t["cache"].view(1, 6, 5, 16))
    torch.cuda.synchronize()
    assert torch.equal(a, b.view(a.shape))


def test_480p_hidden_states_sampled_channels():
    # the measured shape (21 frames x 1560 positions x 2240 channels, bf16),
    # checked on channel groups at both ends and in the middle: channels are
    # independent, so the oracle runs on the selected channels alone
    sh = workloads.TCONV_480P
    x = workloads.make_tconv_inputs(sh["B"], sh["T"], sh["S"], sh["C"], "bf16", seed=804)
    t = _upload(x, "bf16")
    cache_out = torch.empty_like(t["cache"])
    y = la.temporal_conv(t["x"], t["weight"], t["bias"], t["cache"], cache_out=cache_out)
    torch.cuda.synchronize()
    sel = np.r_[0:8, 1112:1128, 2232:2240]
    ref, _ = tconv.temporal_conv(x["x"][..., sel], x["weight"][:, sel], x["bias"][sel],
                                 x["cache"][..., sel])
    got = to64(y[..., torch.from_numpy(sel).cuda()])
    assert_parity(got, ref, "bf16", "480p hidden states")
    assert_elementwise(got, ref, _absum(x, sel), "bf16", "480p hidden states")
    assert torch.equal(cache_out, t["x"][:, -1])
    assert bool(torch.isfinite(y).all())
