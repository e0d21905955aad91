"""Property-based pins of the oracles: on random tiny shapes, latent grids,
rotary splits and modes, the factorised forms equal their brute-force
definitions (the attention-weight sums of the paper-graph page's section 3.4
and Eq. 3; the temporal convolution element by element)."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from oracle import tconv


@st.composite
def attention_case(draw):
    T = draw(st.integers(1, 3))
    Hg = draw(st.integers(1, 3))
    Wg = draw(st.integers(1, 4))
    N = T * Hg * Wg
    # even rotary widths (t, h, w) summing to D
    wt, wh, ww = (2 * draw(st.integers(0, 3)) for _ in range(3))
    D = wt + wh + ww
    if D == 0:
        wt, D = 2, 2 + wh + ww
    rope = draw(st.booleans())
    mode = draw(st.sampled_from(["bidirectional", "block_causal", "token_causal"]))
    fpb = draw(st.sampled_from([f for f in range(1, T + 1) if T % f == 0]))
    return dict(B=draw(st.integers(1, 2)), H=draw(st.integers(1, 2)), N=N, D=D,
                grid=(T, Hg, Wg) if rope else None, split=(wt, wh, ww) if rope else None,
                mode=mode, bt=fpb * Hg * Wg if mode == "block_causal" else 0,
                gate=draw(st.booleans()), seed=draw(st.integers(0, 2 ** 31 - 1)))


@settings(max_examples=60, deadline=None)
@given(attention_case())
def test_factorised_equals_bruteforce(c):
    oracle.build()
    rng = np.random.default_rng(c["seed"])
    shape = (c["B"], c["H"], c["N"], c["D"])
    q, k, v = (rng.standard_normal(shape) for _ in range(3))
    g = rng.standard_normal(shape) if c["gate"] else None
    p = oracle.make_params(c["B"], c["H"], c["N"], c["D"], mode=c["mode"], block_tokens=c["bt"],
                           grid=c["grid"], rope_split=c["split"])
    fac = oracle.forward(p, q, k, v, g=g)
    bru = oracle.bruteforce(p, q, k, v, g=g)
    assert np.abs(fac - bru).max() <= 1e-11 * max(np.abs(bru).max(), 1.0)


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 2), st.integers(1, 2), st.integers(1, 9), st.integers(1, 9),
       st.integers(1, 6), st.booleans(), st.integers(0, 2 ** 31 - 1))
def test_cross_factorised_equals_bruteforce(B, H, Nq, Nkv, D, gate, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Nq, D))
    k = rng.standard_normal((B, H, Nkv, D))
    v = rng.standard_normal((B, H, Nkv, D))
    g = rng.standard_normal((B, H, Nq, D)) if gate else None
    fac = oracle.cross_forward(q, k, v, g)
    bru = oracle.cross_bruteforce(q, k, v, g)
    assert np.abs(fac - bru).max() <= 1e-11 * max(np.abs(bru).max(), 1.0)


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 2), st.integers(1, 6), st.integers(1, 3), st.integers(1, 4),
       st.booleans(), st.booleans(), st.integers(0, 2 ** 31 - 1))
def test_temporal_conv_equals_loops(B, T, S, C, with_cache, with_bias, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, T, S, C))
    w = rng.standard_normal((3, C))
    bias = rng.standard_normal(C) if with_bias else None
    cache = rng.standard_normal((B, S, C)) if with_cache else None
    y, last = tconv.temporal_conv(x, w, bias, cache)
    ref = tconv.temporal_conv_loops(x, w, bias, cache)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(last, x[:, T - 1])
