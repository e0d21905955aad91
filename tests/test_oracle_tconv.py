"""Pins of the temporal-convolution oracle (Mix-FFN, last-frame cache) against
things other than itself: per-element loops, scipy's correlate1d, the
zero-initialised identity the pages state, a hand-worked case, the relation
between block-wise and whole-sequence calls, and causality."""
import numpy as np
import pytest
from scipy.ndimage import correlate1d

from oracle import tconv


def _draw(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _case(B, T, S, C, seed):
    x = _draw((B, T, S, C), seed)
    w = 0.5 * _draw((3, C), seed + 1)
    bias = 0.1 * _draw((C,), seed + 2)
    cache = _draw((B, S, C), seed + 3)
    return x, w, bias, cache


def test_hand_worked_case():
    # one channel, three frames: x = 1, 2, 3; taps 0.5, -1, 2; cached frame 4
    x = np.array([1.0, 2.0, 3.0]).reshape(1, 3, 1, 1)
    w = np.array([[0.5], [-1.0], [2.0]])
    y, new = tconv.temporal_conv(x, w, cache=np.array([[[4.0]]]))
    # y0 = 1 + 0.5*4 - 1*1 + 2*2;  y1 = 2 + 0.5*1 - 1*2 + 2*3;  y2 = 3 + 0.5*2 - 1*3 + 0
    assert y.ravel().tolist() == [6.0, 6.5, 1.0]
    assert new.ravel().tolist() == [3.0]
    y, _ = tconv.temporal_conv(x, w, bias=np.array([0.25]))
    assert y.ravel().tolist() == [4.25, 6.75, 1.25]


@pytest.mark.parametrize("T", [1, 2, 5])
@pytest.mark.parametrize("with_cache,with_bias", [(False, False), (True, False), (True, True)])
def test_matches_loops(T, with_cache, with_bias):
    x, w, bias, cache = _case(2, T, 3, 4, 10 + T)
    got, new = tconv.temporal_conv(x, w, bias if with_bias else None,
                                   cache if with_cache else None)
    ref = tconv.temporal_conv_loops(x, w, bias if with_bias else None,
                                    cache if with_cache else None)
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-14)
    assert np.array_equal(new, x[:, T - 1])


def test_matches_scipy_correlation():
    # scipy.ndimage.correlate1d with a 3-tap kernel and zero padding computes
    # w0 x[t-1] + w1 x[t] + w2 x[t+1] along the chosen axis
    x, w, bias, cache = _case(2, 6, 5, 3, 20)
    y, _ = tconv.temporal_conv(x, w)
    for c in range(3):
        conv = correlate1d(x[..., c], w[:, c], axis=1, mode="constant", cval=0.0)
        np.testing.assert_allclose(y[..., c], x[..., c] + conv, rtol=1e-13, atol=1e-13)
    # with a cache: the cached frame prepended, then the first output dropped
    y, _ = tconv.temporal_conv(x, w, bias, cache)
    ext = np.concatenate([cache[:, None], x], axis=1)
    for c in range(3):
        conv = correlate1d(ext[..., c], w[:, c], axis=1, mode="constant", cval=0.0)[:, 1:]
        np.testing.assert_allclose(y[..., c], x[..., c] + conv + bias[c], rtol=1e-13,
                                   atol=1e-13)


def test_zero_initialised_conv_is_the_identity():
    # the pages' zero-initialised temporal conv leaves the block's output as is
    x, _, _, cache = _case(1, 4, 3, 8, 30)
    y, _ = tconv.temporal_conv(x, np.zeros((3, 8)), np.zeros(8), cache)
    assert np.array_equal(y, x)


def test_blocks_versus_whole_sequence():
    # block-wise with the last-frame cache equals the whole-sequence call
    # except on each block's last frame, which sees the zero frame instead of
    # the next block's first frame: there the difference is w2 * x[next first]
    x, w, bias, _ = _case(2, 9, 4, 5, 40)
    whole, _ = tconv.temporal_conv(x, w, bias)
    blocks, last = tconv.temporal_conv_blocks(x, w, 3, bias)
    assert np.array_equal(last, x[:, 8])
    diff = whole - blocks
    for t in range(9):
        if t % 3 == 2 and t + 1 < 9:
            np.testing.assert_allclose(diff[:, t], w[2] * x[:, t + 1], rtol=1e-13, atol=1e-13)
        else:
            np.testing.assert_allclose(diff[:, t], 0.0, atol=1e-13)
    # one block spanning the sequence is the whole-sequence call
    one, _ = tconv.temporal_conv_blocks(x, w, 9, bias)
    assert np.array_equal(one, whole)


def test_causality_across_blocks():
    # a later block never changes an earlier block's outputs or the cache it hands on
    x, w, bias, _ = _case(1, 8, 3, 4, 50)
    a, _ = tconv.temporal_conv_blocks(x, w, 2, bias)
    x2 = x.copy()
    x2[:, 4:] = _draw(x2[:, 4:].shape, 51)
    b, _ = tconv.temporal_conv_blocks(x2, w, 2, bias)
    assert np.array_equal(a[:, :4], b[:, :4])
    assert not np.allclose(a[:, 4:], b[:, 4:])


def test_channels_and_positions_are_independent():
    # depthwise along T only: a channel subset or a position subset of the
    # input gives the same subset of the output
    x, w, bias, cache = _case(2, 5, 6, 7, 60)
    y, _ = tconv.temporal_conv(x, w, bias, cache)
    sel = [0, 3, 6]
    ys, _ = tconv.temporal_conv(x[..., sel], w[:, sel], bias[sel], cache[..., sel])
    assert np.array_equal(ys, y[..., sel])
    ys, _ = tconv.temporal_conv(x[:, :, 2:4], w, bias, cache[:, 2:4])
    assert np.array_equal(ys, y[:, :, 2:4])


def test_golden_two_block_chain():
    # tests/golden/temporal_conv_worked.txt: a hand-worked chain of two blocks
    import os
    rows = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "temporal_conv_worked.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                rows[key] = np.array([float(x) for x in vals])
    w = np.stack([rows["w0"], rows["w1"], rows["w2"]])
    cache = rows["cache"].reshape(1, 1, 2)
    for blk in ("block1", "block2"):
        x = rows[blk + ".x"].reshape(1, -1, 1, 2)
        y, cache = tconv.temporal_conv(x, w, rows["bias"], cache)
        assert y.ravel().tolist() == rows[blk + ".y"].tolist()
        assert cache.ravel().tolist() == rows[blk + ".cache"].tolist()
