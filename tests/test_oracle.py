"""Pins for the fp64 oracle, on the CPU.

Each test ties the oracle to something other than itself: hand-worked
examples (tests/golden/), the literal O(N^2) attention-weight form, closed
forms and invariants that the SANA-Video equations fix. A plausible mistake in
the oracle (a dropped term, a transposed state, a wrong RoPE pairing or
frequency, rotated denominators, an off-by-one block scope) fails at least one.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows[key] = vals
    return rows


def _rand(shape, seed, dist="normal"):
    rng = np.random.default_rng(seed)
    if dist == "t3":
        return (rng.standard_t(3, size=shape) / math.sqrt(3)).astype(np.float32)
    return rng.standard_normal(shape).astype(np.float32)


def _qkv(B, H, N, D, seed, gate=False):
    x = [_rand((B, H, N, D), seed + i) for i in range(4 if gate else 3)]
    return x


# ---------------------------------------------------------------- golden ----

EPS = 1e-6


def _worked():
    g = _read_golden("relu_linear_attention_worked.txt")
    arr = lambda k: np.array([float(x) for x in g[k]], dtype=np.float32)
    q = arr("q").reshape(1, 1, 4, 2)
    k = arr("k").reshape(1, 1, 4, 2)
    v = arr("v").reshape(1, 1, 4, 2)
    return g, q, k, v


@pytest.mark.parametrize("mode,key,bt", [
    ("bidirectional", "bidirectional", 0),
    ("block_causal", "block_causal_2", 2),
    ("token_causal", "token_causal", 0),
])
def test_worked_example_all_modes(mode, key, bt):
    g, q, k, v = _worked()
    num = np.array([float(x) for x in g[key + ".num"]]).reshape(4, 2)
    den = np.array([float(x) for x in g[key + ".den"]])
    want = num / (den[:, None] + EPS)
    p = oracle.make_params(1, 1, 4, 2, mode=mode, block_tokens=bt, eps=EPS)
    got = oracle.forward(p, q, k, v)[0, 0]
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=0)
    assert np.all(got[2] == 0.0)           # phi(q_2) = 0 -> exactly 0, no NaN
    brute = oracle.bruteforce(p, q, k, v)[0, 0]
    np.testing.assert_allclose(brute, want, rtol=1e-15, atol=0)


def test_worked_example_state():
    g, q, k, v = _worked()
    p = oracle.make_params(1, 1, 4, 2)
    S, z = oracle.state(p, k, v)
    np.testing.assert_array_equal(S[0, 0].ravel(), [float(x) for x in g["state.S"]])
    np.testing.assert_array_equal(z[0, 0], [float(x) for x in g["state.z"]])


def test_worked_example_gate_closed_form():
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4, sigmoid(0) = 1/2 exactly.
    gdat, q, k, v = _worked()
    num = np.array([float(x) for x in gdat["bidirectional.num"]]).reshape(4, 2)
    den = np.array([float(x) for x in gdat["bidirectional.den"]])
    base = num / (den[:, None] + EPS)
    gl = np.zeros((1, 1, 4, 2), dtype=np.float32)
    gl[0, 0, 0] = [math.log(3.0), -math.log(3.0)]
    p = oracle.make_params(1, 1, 4, 2, eps=EPS)
    got = oracle.forward(p, q, k, v, g=gl)[0, 0]
    lg3 = float(np.float32(math.log(3.0)))
    want = base * 0.5
    want[0] = base[0] * [1 / (1 + math.exp(-lg3)), 1 / (1 + math.exp(lg3))]
    np.testing.assert_allclose(got, want, rtol=1e-15)
    np.testing.assert_allclose(got[0], base[0] * [0.75, 0.25], rtol=1e-7)


def test_rope_worked_example():
    g = _read_golden("rope_3d_worked.txt")
    D = int(g["D"][0])
    split = tuple(int(x) for x in g["split"])
    grid = tuple(int(x) for x in g["grid"])
    p = oracle.make_params(1, 1, int(np.prod(grid)), D, grid=grid, rope_split=split,
                           theta=float(g["theta"][0]))
    x = np.array([float(t) for t in g["x"]])
    env = {"cos": math.cos, "sin": math.sin}
    want = np.array([eval(e, {"__builtins__": {}}, env) for e in g["y"]])
    got = oracle.rope(p, int(g["token"][0]), x)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(oracle.rope(p, 0, x), [float(t) for t in g["y_token0"]])


# ------------------------------------------------------------- RoPE pins ----

def _p64(N=60, mode="bidirectional", t_offset=0):
    return oracle.make_params(1, 1, N, 32, mode=mode, grid=(N // 20, 4, 5),
                              rope_split=(8, 12, 12), t_offset=t_offset)


def test_rope_unit_vectors_each_axis_and_frequency():
    # A unit vector on dim 2m of an axis segment of width d rotates by
    # pos * theta^(-2m/d) inside its own pair only (theta = 10000 here).
    p = oracle.make_params(1, 1, 21 * 30 * 52, 64, grid=(21, 30, 52), rope_split=(16, 24, 24))
    t, h, w = 13, 7, 41
    n = (t * 30 + h) * 52 + w
    for base, d, pos in ((0, 16, t), (16, 24, h), (40, 24, w)):
        for m in range(d // 2):
            x = np.zeros(64)
            x[base + 2 * m] = 1.0
            y = oracle.rope(p, n, x)
            ang = pos * 10000.0 ** (-2.0 * m / d)
            want = np.zeros(64)
            want[base + 2 * m] = math.cos(ang)
            want[base + 2 * m + 1] = math.sin(ang)
            np.testing.assert_allclose(y, want, atol=1e-12)


def test_rope_preserves_norm():
    p = _p64()
    rng = np.random.default_rng(5)
    for n in (0, 7, 33, 59):
        x = rng.standard_normal(32)
        assert abs(np.linalg.norm(oracle.rope(p, n, x)) - np.linalg.norm(x)) < 1e-12


def test_rope_relative_position():
    # RoPE(a at p1) . RoPE(b at p2) depends only on p2 - p1: shifting every
    # frame index (t_offset) leaves it unchanged; so does moving both tokens
    # one row down in h.
    rng = np.random.default_rng(6)
    a, b = rng.standard_normal(32), rng.standard_normal(32)
    p0, p5 = _p64(t_offset=0), _p64(t_offset=5)
    for n1, n2 in ((0, 59), (13, 21), (40, 2)):
        d0 = oracle.rope(p0, n1, a) @ oracle.rope(p0, n2, b)
        d5 = oracle.rope(p5, n1, a) @ oracle.rope(p5, n2, b)
        assert abs(d0 - d5) < 1e-12
    # (t,h,w) = (1,0,2),(2,1,4) vs (1,2,2),(2,3,4): same offsets, shifted h
    nA1, nA2 = (1 * 4 + 0) * 5 + 2, (2 * 4 + 1) * 5 + 4
    nB1, nB2 = (1 * 4 + 2) * 5 + 2, (2 * 4 + 3) * 5 + 4
    dA = oracle.rope(p0, nA1, a) @ oracle.rope(p0, nA2, b)
    dB = oracle.rope(p0, nB1, a) @ oracle.rope(p0, nB2, b)
    assert abs(dA - dB) < 1e-12


def test_output_invariant_to_global_frame_shift():
    q, k, v = _qkv(2, 2, 60, 32, 10)
    o0 = oracle.forward(_p64(), q, k, v)
    o9 = oracle.forward(_p64(t_offset=9), q, k, v)
    np.testing.assert_allclose(o9, o0, rtol=1e-11, atol=1e-14)


# ------------------------------------------------- brute force vs factorised ----

CASES = [
    # (B, H, N, D, grid, split, gate)
    (1, 2, 256, 32, None, None, False),            # the tiny fp32 workload's shape
    (2, 2, 60, 32, (3, 4, 5), (8, 12, 12), False),  # RoPE on a 3x4x5 grid
    (1, 3, 64, 16, (4, 4, 4), (4, 6, 6), True),     # gate + odd head count
    (1, 2, 48, 112, (3, 4, 4), (16, 48, 48), True),  # the 2B model's head dim, 56 pairs
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("mode", ["bidirectional", "block_causal", "token_causal"])
def test_factorised_matches_bruteforce(case, mode):
    B, H, N, D, grid, split, gate = case
    bt = 0
    if mode == "block_causal":
        bt = (grid[1] * grid[2]) if grid else 64
    p = oracle.make_params(B, H, N, D, mode=mode, block_tokens=bt, grid=grid, rope_split=split)
    xs = _qkv(B, H, N, D, 100 + N, gate)
    g = xs[3] if gate else None
    fac = oracle.forward(p, xs[0], xs[1], xs[2], g=g)
    bru = oracle.bruteforce(p, xs[0], xs[1], xs[2], g=g)
    scale = np.abs(bru).max()
    assert np.abs(fac - bru).max() <= 1e-12 * max(scale, 1.0)


def test_bruteforce_of_outlier_inputs():
    B, H, N, D = 1, 2, 48, 16
    p = oracle.make_params(B, H, N, D, grid=(3, 4, 4), rope_split=(4, 6, 6))
    q = _rand((B, H, N, D), 1, "t3")
    k = _rand((B, H, N, D), 2, "t3")
    v = _rand((B, H, N, D), 3)
    fac = oracle.forward(p, q, k, v)
    bru = oracle.bruteforce(p, q, k, v)
    assert np.abs(fac - bru).max() <= 1e-12 * np.abs(bru).max()


# ------------------------------------------------------------- invariants ----

def test_constant_v_returns_the_constant_without_rope():
    # v_j = c for all j: num = c (phi(q) . z), so out = c * den/(den + eps).
    B, H, N, D = 1, 2, 256, 32
    q, k, _ = _qkv(B, H, N, D, 20)
    c = _rand((D,), 21)
    v = np.broadcast_to(c, (B, H, N, D)).copy()
    p = oracle.make_params(B, H, N, D)
    out = oracle.forward(p, q, k, v)
    rows = np.any(q > 0, axis=-1)          # rows with phi(q) = 0 give 0
    np.testing.assert_allclose(out[rows], np.broadcast_to(c, out[rows].shape), rtol=1e-8)
    assert np.all(out[~rows] == 0)


def test_one_block_equals_bidirectional_bitwise():
    B, H, N, D = 2, 2, 60, 32
    q, k, v = _qkv(B, H, N, D, 30)
    pb = oracle.make_params(B, H, N, D, grid=(3, 4, 5), rope_split=(8, 12, 12))
    pc = oracle.make_params(B, H, N, D, mode="block_causal", block_tokens=N,
                            grid=(3, 4, 5), rope_split=(8, 12, 12))
    np.testing.assert_array_equal(oracle.forward(pc, q, k, v), oracle.forward(pb, q, k, v))


def test_sequential_block_steps_equal_bruteforce_causal_by_block():
    # Algorithm 1: run blocks one call at a time with the carried state; the
    # concatenation equals both the one-call block-causal forward (bitwise)
    # and the literal causal-by-block O(N^2) form.
    B, H, D = 1, 2, 32
    grid = (6, 4, 5)
    N = 120
    bt = 40  # two frames per block
    q, k, v = _qkv(B, H, N, D, 40)
    full_p = oracle.make_params(B, H, N, D, mode="block_causal", block_tokens=bt,
                                grid=grid, rope_split=(8, 12, 12))
    one_call = oracle.forward(full_p, q, k, v)
    brute = oracle.bruteforce(full_p, q, k, v)
    S = np.zeros((B, H, D, D))
    z = np.zeros((B, H, D))
    pieces = []
    for b in range(N // bt):
        sl = slice(b * bt, (b + 1) * bt)
        p = oracle.make_params(B, H, bt, D, mode="block_causal", block_tokens=bt,
                               grid=(2, 4, 5), rope_split=(8, 12, 12), t_offset=2 * b)
        o, S, z = oracle.forward(p, q[:, :, sl], k[:, :, sl], v[:, :, sl], S0=S, z0=z,
                                 want_state=True)
        pieces.append(o)
    seq = np.concatenate(pieces, axis=2)
    np.testing.assert_array_equal(seq, one_call)
    assert np.abs(seq - brute).max() <= 1e-12 * np.abs(brute).max()
    # the carried state after the last block is the state of the whole sequence
    S_all, z_all = oracle.state(full_p, k, v)
    np.testing.assert_allclose(S, S_all, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, z_all, rtol=1e-12)


def test_zero_phi_gives_zero_output():
    B, H, N, D = 1, 1, 40, 16
    q, k, v = _qkv(B, H, N, D, 50)
    p = oracle.make_params(B, H, N, D, grid=(2, 4, 5), rope_split=(4, 6, 6))
    out = oracle.forward(p, -np.abs(q), k, v)                # phi(q) = 0 everywhere
    assert np.all(out == 0) and np.all(np.isfinite(out))
    out = oracle.forward(p, q, -np.abs(k), v)                # S = 0, z = 0
    assert np.all(out == 0)
    S, z = oracle.state(p, -np.abs(k), v)
    assert np.all(S == 0) and np.all(z == 0)


def test_linear_in_v_and_gate_zero_halves():
    B, H, N, D = 1, 2, 60, 32
    q, k, v1 = _qkv(B, H, N, D, 60)
    v2 = _rand((B, H, N, D), 64)
    p = _p64()
    p.B, p.H = B, H
    o1 = oracle.forward(p, q, k, v1)
    o2 = oracle.forward(p, q, k, v2)
    o12 = oracle.forward(p, q, k, (v1.astype(np.float64) + 2 * v2).astype(np.float32))
    # v1 + 2 v2 is rounded to fp32 before the oracle reads it
    v12 = (v1.astype(np.float64) + 2 * v2).astype(np.float32).astype(np.float64)
    assert np.allclose(v12, v1 + 2.0 * v2, rtol=1e-7)
    np.testing.assert_allclose(o12, o1 + 2 * o2, rtol=1e-6, atol=1e-6 * np.abs(o1).max())
    half = oracle.forward(p, q, k, v1, g=np.zeros_like(v1))
    np.testing.assert_array_equal(half, o1 * 0.5)


def test_permutation_invariance_without_rope():
    B, H, N, D = 1, 2, 64, 16
    q, k, v = _qkv(B, H, N, D, 70)
    p = oracle.make_params(B, H, N, D)
    out = oracle.forward(p, q, k, v)
    perm = np.random.default_rng(71).permutation(N)
    outp = oracle.forward(p, q[:, :, perm], k[:, :, perm], v[:, :, perm])
    np.testing.assert_allclose(outp, out[:, :, perm], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("mode", ["block_causal", "token_causal"])
def test_causality_future_tokens_do_not_change_the_past(mode):
    B, H, N, D = 1, 2, 60, 32
    q, k, v = _qkv(B, H, N, D, 80)
    p = oracle.make_params(B, H, N, D, mode=mode, block_tokens=20 if mode == "block_causal" else 0,
                           grid=(3, 4, 5), rope_split=(8, 12, 12))
    base = oracle.forward(p, q, k, v)
    cut = 40 if mode == "block_causal" else 33
    k2, v2 = k.copy(), v.copy()
    k2[:, :, cut:] = _rand(k2[:, :, cut:].shape, 81)
    v2[:, :, cut:] = _rand(v2[:, :, cut:].shape, 82)
    out = oracle.forward(p, q, k2, v2)
    np.testing.assert_array_equal(out[:, :, :cut], base[:, :, :cut])
    assert not np.array_equal(out[:, :, cut:], base[:, :, cut:])


def test_token_causal_equals_blocks_of_one_token():
    # blocks of one token see exactly the tokens 0..i: the block-causal form
    # with block_tokens = 1 and the per-token causal form are the same sums
    B, H, N, D = 1, 2, 60, 32
    q, k, v = _qkv(B, H, N, D, 85)
    g = _rand(q.shape, 86)
    kw = dict(grid=(3, 4, 5), rope_split=(8, 12, 12))
    a = oracle.forward(oracle.make_params(B, H, N, D, mode="token_causal", **kw), q, k, v, g=g)
    b = oracle.forward(oracle.make_params(B, H, N, D, mode="block_causal", block_tokens=1, **kw),
                       q, k, v, g=g)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    # and the last token sees the whole head: the bidirectional output there
    c = oracle.forward(oracle.make_params(B, H, N, D, **kw), q, k, v, g=g)
    np.testing.assert_allclose(a[:, :, -1], c[:, :, -1], rtol=1e-12, atol=1e-14)


def test_rows_match_full_output():
    B, H, N, D = 2, 2, 60, 32
    q, k, v = _qkv(B, H, N, D, 90)
    for mode in ("bidirectional", "block_causal", "token_causal"):
        p = oracle.make_params(B, H, N, D, mode=mode, block_tokens=20 if mode == "block_causal" else 0,
                               grid=(3, 4, 5), rope_split=(8, 12, 12))
        full = oracle.forward(p, q, k, v).reshape(-1, D)
        rows = np.array([0, 5, 59, 60, 119, 200, 239, 5, 131])
        got = oracle.forward_rows(p, q, k, v, rows)
        np.testing.assert_array_equal(got, full[rows])


def test_bad_arguments_are_rejected():
    p = oracle.make_params(1, 1, 10, 8, mode="block_causal", block_tokens=3)
    with pytest.raises(ValueError):
        oracle.forward(p, *_qkv(1, 1, 10, 8, 1))
    p = oracle.make_params(1, 1, 12, 8, grid=(1, 3, 4), rope_split=(2, 2, 2))
    with pytest.raises(ValueError):
        oracle.forward(p, *_qkv(1, 1, 12, 8, 1))


# ---- linear cross-attention (numpy fp64 form) --------------------------------

def test_cross_matches_bruteforce_with_gate():
    rng = np.random.default_rng(301)
    q = rng.standard_normal((2, 2, 9, 8))
    k = rng.standard_normal((2, 2, 5, 8))
    v = rng.standard_normal((2, 2, 5, 8))
    g = rng.standard_normal((2, 2, 9, 8))
    np.testing.assert_allclose(oracle.cross_forward(q, k, v, g), oracle.cross_bruteforce(q, k, v, g),
                               rtol=1e-12, atol=1e-14)


def test_cross_with_equal_lengths_is_the_self_attention_oracle():
    # the C oracle's bidirectional form without RoPE is an independent
    # implementation of the same sums when queries and keys share a length
    B, H, N, D = 1, 3, 40, 32
    q, k, v = _qkv(B, H, N, D, 302)
    g = _rand(q.shape, 303)
    ref = oracle.forward(oracle.make_params(B, H, N, D), q, k, v, g=g)
    got = oracle.cross_forward(q, k, v, g)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_cross_closed_forms():
    # a hand-worked case: phi(q) = (1, 0) meets k_0 = (2, 1) with weight 2 and
    # k_1 = (0, 3) with weight 0, so out = 2 v_0 / (2 + eps)
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[2.0, 1.0], [0.0, 3.0]]]])
    v = np.array([[[[1.0, 2.0], [3.0, 4.0]]]])
    out = oracle.cross_forward(q, k, v, eps=1e-6)
    np.testing.assert_allclose(out[0, 0, 0], np.array([1.0, 2.0]) * 2.0 / (2.0 + 1e-6), rtol=1e-15)
    # constant values come back (up to eps) whatever the queries and keys
    rng = np.random.default_rng(304)
    q = rng.standard_normal((1, 2, 7, 4))
    k = np.abs(rng.standard_normal((1, 2, 3, 4))) + 0.5
    v = np.broadcast_to(np.array([0.5, -1.0, 2.0, 3.0]), (1, 2, 3, 4))
    out = oracle.cross_forward(q, k, v, eps=0.0)
    rows = (np.maximum(q, 0).sum(-1) > 0)
    np.testing.assert_allclose(out[rows], np.broadcast_to(v[0, 0, 0], out[rows].shape), rtol=1e-12)
    # queries with no positive entry give exactly zero
    assert np.array_equal(oracle.cross_forward(-np.abs(q), k, v), np.zeros_like(q))


def test_cross_golden_worked_example():
    # tests/golden/cross_attention_worked.txt: 2 queries, 3 keys, D = 2
    g = _read_golden("cross_attention_worked.txt")
    arr = lambda key, *shape: np.array([float(x) for x in g[key]]).reshape(shape)
    q, k, v = arr("q", 1, 1, 2, 2), arr("k", 1, 1, 3, 2), arr("v", 1, 1, 3, 2)
    num, den = arr("num", 2, 2), arr("den", 2)
    out = oracle.cross_forward(q, k, v, eps=1e-6)
    np.testing.assert_allclose(out[0, 0], num / (den[:, None] + 1e-6), rtol=1e-15, atol=0)
    # a zero gate halves it exactly
    half = oracle.cross_forward(q, k, v, g=np.zeros_like(q), eps=1e-6)
    assert np.array_equal(half, out / 2)
