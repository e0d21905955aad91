"""fp64 oracle of the Mix-FFN temporal convolution with its last-frame cache.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``: the tests, ``smoke()``
and the CPU baseline of ``bench.py`` may use it; the CUDA library never does.

What it computes (SANA-Video paper-graph page, "Spatial-Temporal Mix-FFN" and
"Block Causal Mix-FFN"; Algorithm 1's third cache entry):

  * the block's hidden states x_spatial, shape [B, T, S, C] with S = Hg * Wg
    spatial positions per latent frame, go through a temporal convolution of
    kernel size 3 along T (a 3x1x1 kernel on the [T, H, W, C] tensor), added
    back through the shortcut: y[t] = x[t] + conv(x)[t];
  * the convolution is per channel (depthwise), tap 0 on frame t-1, tap 1 on
    frame t, tap 2 on frame t+1, with an optional per-channel bias;
  * frame t+1 past the block's end is the all-zero frame the pages append to
    each block; frame -1 is the cached last frame of the previous block (the
    prepended conv cache), or zero when there is none (the first block, or a
    whole-sequence call);
  * the new cache is the block's own last input frame.

Pinned by ``tests/test_oracle_tconv.py`` against per-element loops, scipy's
correlate1d, the zero-initialised identity, the block/whole-sequence relation
and causality.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np


def temporal_conv(x, w, bias=None, cache=None) -> Tuple[np.ndarray, np.ndarray]:
    """y = x + w[0] * x[t-1] + w[1] * x[t] + w[2] * x[t+1] (+ bias), fp64.

    x: [B, T, S, C]; w: [3, C]; bias: [C] or None; cache: [B, S, C] or None
    (then frame -1 is zero). Returns (y [B, T, S, C], new cache = x[:, T-1]).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, T, S, C = x.shape
    zero = np.zeros((B, 1, S, C))
    prev = zero if cache is None else np.asarray(cache, dtype=np.float64).reshape(B, 1, S, C)
    framed = np.concatenate([prev, x, zero], axis=1)          # frames -1 .. T
    y = x + w[0] * framed[:, 0:T] + w[1] * framed[:, 1:T + 1] + w[2] * framed[:, 2:T + 2]
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y, x[:, T - 1].copy()


def temporal_conv_loops(x, w, bias=None, cache=None) -> np.ndarray:
    """The same output element by element, with the boundary frames spelled
    out as conditions; tiny inputs only."""
    x = np.asarray(x, dtype=np.float64)
    B, T, S, C = x.shape
    y = np.zeros((B, T, S, C))
    for b in range(B):
        for t in range(T):
            for s in range(S):
                for c in range(C):
                    if t > 0:
                        before = x[b, t - 1, s, c]
                    elif cache is not None:
                        before = float(cache[b, s, c])
                    else:
                        before = 0.0
                    after = x[b, t + 1, s, c] if t + 1 < T else 0.0
                    acc = x[b, t, s, c]
                    acc += float(w[0][c]) * before
                    acc += float(w[1][c]) * x[b, t, s, c]
                    acc += float(w[2][c]) * after
                    if bias is not None:
                        acc += float(bias[c])
                    y[b, t, s, c] = acc
    return y


def temporal_conv_blocks(x, w, frames_per_block: int, bias=None,
                         cache: Optional[np.ndarray] = None):
    """Algorithm 1's chain: the frames in blocks of ``frames_per_block``, each
    block convolved with the previous block's last frame as its cache."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[1]
    outs = []
    for t0 in range(0, T, frames_per_block):
        y, cache = temporal_conv(x[:, t0:t0 + frames_per_block], w, bias, cache)
        outs.append(y)
    return np.concatenate(outs, axis=1), cache
