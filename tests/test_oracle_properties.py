"""Property-based pins of the oracles: on random tiny shapes, latent grids,
rotary splits and modes, the factorised forms equal their brute-force
definitions (the attention-weight sums of the paper-graph page's section 3.4
and Eq. 3; the temporal convolution element by element)."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from oracle import tconv

U = 2.0 ** -53   # fp64 unit roundoff


def rounding_bound(q, k, v, mask, eps, out):
    """Per-element bound on |factorised - brute force| for out_i =
    sum_j (RoPE(phi q_i) . RoPE(phi k_j)) v_j / (sum_j phi q_i . phi k_j + eps)
    over the keys j that mask[i, j] admits. The two forms add the same
    products in different orders, so each is within (N + D) u of the exact
    value times the sum of the magnitudes it adds. RoPE keeps each pair's
    norm, so |RoPE(phi q) . RoPE(phi k)| <= |phi q| |phi k|, and that sum is
    at most M_ic = sum_j |phi q_i| |phi k_j| |v_jc|. The denominator adds
    non-negative terms, so it is accurate to (N + D) u relative. For both
    forms together: 4 (N + D) u (M / den + |out|)."""
    pq, pk = np.maximum(q, 0.0), np.maximum(k, 0.0)
    den = np.einsum("bhid,bhjd,ij->bhi", pq, pk, mask) + eps
    M = np.einsum("bhi,bhj,bhjc,ij->bhic", np.linalg.norm(pq, axis=-1),
                  np.linalg.norm(pk, axis=-1), np.abs(v), mask)
    n_terms = k.shape[2] + q.shape[3]
    return 4.0 * n_terms * U * (M / den[..., None] + np.abs(out))


def attended(N, mode, bt):
    """mask[i, j]: key j is summed for query i (bidirectional: all; block
    causal: blocks up to i's; token causal: j <= i)."""
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    if mode == "block_causal":
        return (j // bt <= i // bt).astype(float)
    if mode == "token_causal":
        return (j <= i).astype(float)
    return np.ones((N, N))


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
    bound = rounding_bound(q, k, v, attended(c["N"], c["mode"], c["bt"]), 1e-6, bru)
    assert (np.abs(fac - bru) <= bound).all(), np.max(np.abs(fac - bru) / bound)


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
    bound = rounding_bound(q, k, v, np.ones((Nq, Nkv)), 1e-6, bru)
    assert (np.abs(fac - bru) <= bound).all(), np.max(np.abs(fac - bru) / bound)


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
