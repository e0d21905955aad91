"""The C-ABI library on the CPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

import __graft_entry__
from linear_attention_video_relu_b200 import _native as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "linattn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    __graft_entry__.build()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^LA_API\s+[\w\s\*]+?\b(lin_attn_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("lin_attn_forward", "lin_attn_block_step", "lin_attn_state_init",
              "lin_attn_state_reset", "lin_attn_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(C.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_mirrors_the_header():
    assert set(C.SIGNATURES) == set(declared_functions())
    for name in declared_functions():
        assert callable(getattr(C, name, None)) or name == "lin_attn_status_string"


def test_status_strings():
    for s in range(6):
        assert C.status_string(s)
    assert C.status_string(99) == "unknown status"


def _params(**kw):
    p = C.la_params()
    p.B, p.H, p.N, p.D = 1, 2, 60, 32
    p.dtype = C.LA_BF16
    p.mode = C.LA_BIDIRECTIONAL
    p.rope = 1
    p.grid_t, p.grid_h, p.grid_w = 3, 4, 5
    p.rope_dt, p.rope_dh, p.rope_dw = 8, 12, 12
    p.rope_theta = 10000.0
    p.eps = 1e-6
    for k, v in kw.items():
        setattr(p, k, v)
    return p


# Pointers below are fake device addresses: every case must be rejected by the
# host checks, before any CUDA call (there is no GPU here).
Q, K, V, O, WS = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000

BAD = [
    ("D not supported", dict(D=48), C.LA_ERR_INVALID_ARG),
    ("negative N", dict(N=-1), C.LA_ERR_INVALID_ARG),
    ("bad dtype", dict(dtype=7), C.LA_ERR_INVALID_ARG),
    ("bad mode", dict(mode=5), C.LA_ERR_INVALID_ARG),
    ("block does not divide N", dict(mode=C.LA_BLOCK_CAUSAL, block_tokens=7), C.LA_ERR_INVALID_ARG),
    ("block of zero tokens", dict(mode=C.LA_BLOCK_CAUSAL, block_tokens=0), C.LA_ERR_INVALID_ARG),
    ("split does not sum to D", dict(rope_dw=10), C.LA_ERR_INVALID_ARG),
    ("odd split", dict(rope_dt=7, rope_dh=13), C.LA_ERR_INVALID_ARG),
    ("grid does not match N", dict(grid_t=4), C.LA_ERR_INVALID_ARG),
    ("theta not positive", dict(rope_theta=0.0), C.LA_ERR_INVALID_ARG),
    ("negative eps", dict(eps=-1.0), C.LA_ERR_INVALID_ARG),
    ("rope table too large", dict(N=8000 * 1 * 1, grid_t=8000, grid_h=1, grid_w=1),
     C.LA_ERR_UNSUPPORTED),
]


@pytest.mark.parametrize("name,kw,want", BAD, ids=[b[0] for b in BAD])
def test_forward_rejects_bad_params(name, kw, want):
    assert C.lin_attn_forward(_params(**kw), Q, K, V, None, O, WS, 1 << 20, None) == want


def test_forward_rejects_bad_pointers():
    p = _params()
    assert C.lin_attn_forward(p, None, K, V, None, O, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_forward(p, Q, K, V, None, None, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_forward(p, Q + 8, K, V, None, O, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_forward(p, Q, K, V, V + 2, O, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    # out overlapping an input
    assert C.lin_attn_forward(p, Q, K, V, None, Q + 64, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_forward(p, Q, K, V, None, K, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG


def test_empty_problem_is_a_no_op():
    # N = 0 (and B*H = 0) is valid and launches nothing, even with null pointers
    p = _params(N=0, rope=0)
    assert C.lin_attn_forward(p, None, None, None, None, None, None, 0, None) == C.LA_OK
    p = _params(B=0)
    assert C.lin_attn_forward(p, None, None, None, None, None, None, 0, None) == C.LA_OK


def test_state_init_and_block_step_argument_checks():
    st = C.la_state()
    assert C.lin_attn_state_init(st, 1, 2, 32, 0x1000, 0x2000) == C.LA_OK
    assert (st.B, st.H, st.D) == (1, 2, 32)
    assert C.lin_attn_state_init(st, 1, 2, 33, 0x1000, 0x2000) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_state_init(st, 1, 2, 32, None, 0x2000) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_state_init(st, 1, 2, 32, 0x1004, 0x2000) == C.LA_ERR_INVALID_ARG
    p = _params()
    # state shape must match the params
    bad = C.la_state()
    assert C.lin_attn_state_init(bad, 1, 3, 32, 0x1000, 0x2000) == C.LA_OK
    assert C.lin_attn_block_step(p, bad, 0, Q, K, V, None, O, 1, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_block_step(p, st, -1, Q, K, V, None, O, 1, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_block_step(p, st, 0, None, K, V, None, O, 1, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_state_update(p, st, 0, None, V, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG


def test_tensor_core_path_selection_is_host_logic():
    # bf16 with D in {64, 128} and rope widths that are multiples of 8 take the
    # tensor-core kernels; fp32, D = 32 and other widths never do.
    assert C.lin_attn_uses_tensor_cores(_params(dtype=C.LA_F32)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=32)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=16, rope_dh=24, rope_dw=24)) == 1
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=20, rope_dh=22, rope_dw=22)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=128, rope_dt=32, rope_dh=48, rope_dw=48)) == 1
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope=0)) == 1
    # token-causal runs on the tensor cores at bf16 and D = 64 only
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=16, rope_dh=24, rope_dw=24,
                                                mode=C.LA_TOKEN_CAUSAL)) == 1
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=16, rope_dh=24, rope_dw=24,
                                                mode=C.LA_TOKEN_CAUSAL, dtype=C.LA_F32)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=128, rope_dt=32, rope_dh=48, rope_dw=48,
                                                mode=C.LA_TOKEN_CAUSAL)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=20, rope_dh=22, rope_dw=22,
                                                mode=C.LA_TOKEN_CAUSAL)) == 0


def test_token_causal_mode_is_accepted_and_ignores_block_tokens():
    # passes the host checks (the fake pointers then fail only at the device
    # query, never as an argument error), for any block_tokens
    for bt in (0, 7):
        rc = C.lin_attn_forward(_params(mode=C.LA_TOKEN_CAUSAL, block_tokens=bt), Q, K, V, None,
                                O, WS, 1 << 20, None)
        assert rc != C.LA_ERR_INVALID_ARG


def test_control_block_size_matches_the_header():
    text = open(HEADER).read()
    m = re.search(r"#define\s+LA_WORKSPACE_CONTROL_BYTES\s+(\d+)u?", text)
    assert m and int(m.group(1)) == C.LA_WORKSPACE_CONTROL_BYTES


def _cross(**kw):
    return _params(rope=0, **kw)


def test_cross_forward_rejects_what_it_does_not_define():
    ok = _cross()
    for p, n_kv in ((_params(), 40), (_cross(mode=C.LA_BLOCK_CAUSAL, block_tokens=20), 40),
                    (_cross(mode=C.LA_TOKEN_CAUSAL), 40), (ok, 0), (ok, -3), (_cross(D=48), 40)):
        assert C.lin_attn_cross_forward(p, n_kv, Q, K, V, None, O, WS, 1 << 20, None) == \
            C.LA_ERR_INVALID_ARG
        with pytest.raises(C.LinAttnError):
            C.lin_attn_cross_workspace_size(p, n_kv)


def test_cross_forward_pointer_checks_use_each_sequence_length():
    p = _cross()                       # q, out: 2 heads x 60 x 32 bf16 = 7680 bytes
    assert C.lin_attn_cross_forward(p, 40, None, K, V, None, O, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_cross_forward(p, 40, Q, K, None, None, O, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_cross_forward(p, 40, Q, K, V, O + 2, O, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    # out 32 KB past k: clear of k when k holds 40 tokens, inside it at 500
    out = K + 0x8000
    assert C.lin_attn_cross_forward(p, 500, Q, K, V, None, out, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_cross_forward(p, 40, Q, K, V, None, out, WS, 1 << 20, None) != \
        C.LA_ERR_INVALID_ARG
    # no queries: no work, whatever the pointers
    assert C.lin_attn_cross_forward(_cross(N=0), 7, None, None, None, None, None, None, 0,
                                    None) == C.LA_OK


def _tconv(B=1, T=3, S=5, nc=16, dtype=C.LA_BF16, x=0x100000, w=0x200000, b=None,
           cin=None, y=0x300000, cout=None):
    return C.lin_attn_temporal_conv(B, T, S, nc, dtype, x, w, b, cin, y, cout, None)


def test_temporal_conv_rejects_bad_arguments_on_the_host():
    bad = C.LA_ERR_INVALID_ARG
    assert _tconv(T=-1) == bad and _tconv(S=-2) == bad and _tconv(nc=-8) == bad
    assert _tconv(dtype=9) == bad
    assert _tconv(nc=12) == bad                          # bf16: 8 channels per 16 bytes
    assert _tconv(nc=12, dtype=C.LA_F32) != bad          # fp32: 4 channels per 16 bytes
    assert _tconv(x=None) == bad and _tconv(y=None) == bad and _tconv(w=None) == bad
    assert _tconv(x=0x100008) == bad and _tconv(b=0x400004) == bad
    assert _tconv(cin=0x500002) == bad and _tconv(cout=0x600001) == bad
    # x: 1 x 3 x 5 x 16 bf16 = 480 bytes; one cache frame: 160 bytes
    assert _tconv(y=0x100000 + 256) == bad               # y overlapping x
    assert _tconv(cin=0x300000 + 64) == bad              # y overlapping cache_in
    assert _tconv(cout=0x100000 + 320) == bad            # cache_out overlapping x
    assert _tconv(cin=0x500000, cout=0x500000 + 16) == bad   # partial overlap of the caches
    assert _tconv(cin=0x500000, cout=0x500000) != bad    # the in-place cache update
    assert _tconv(b=0x400000, cin=0x500000, cout=0x600000) != bad


def test_temporal_conv_without_work_is_a_no_op():
    for kw in (dict(B=0), dict(T=0), dict(S=0), dict(nc=0)):
        assert _tconv(x=None, w=None, y=None, **kw) == C.LA_OK


def test_head_dim_112_is_accepted():
    # 56 rotary pairs split over (t, h, w); passes the host checks (the fake
    # pointers then fail only at the device query); bf16 with widths that are
    # multiples of 8 takes the (padded) tensor-core kernels, fp32 does not
    p = _params(D=112, rope_dt=16, rope_dh=48, rope_dw=48)
    assert C.lin_attn_forward(p, Q, K, V, None, O, WS, 1 << 20, None) != C.LA_ERR_INVALID_ARG
    assert C.lin_attn_uses_tensor_cores(p) == 1
    assert C.lin_attn_uses_tensor_cores(_params(D=112, rope_dt=16, rope_dh=48, rope_dw=48,
                                                dtype=C.LA_F32)) == 0
    assert C.lin_attn_uses_tensor_cores(_params(D=112, rope_dt=20, rope_dh=46, rope_dw=46)) == 0
    assert C.lin_attn_forward(_params(D=96, rope_dt=32, rope_dh=32, rope_dw=32), Q, K, V, None,
                              O, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG


def test_segment_count_limit():
    # B * H times the segments of a head must fit an int: 2^24 heads of
    # 256-token blocks of one token each would need 2^32 segments
    p = _params(B=1 << 12, H=1 << 12, N=256, rope=0, mode=C.LA_BLOCK_CAUSAL, block_tokens=1)
    assert C.lin_attn_forward(p, Q, K, V, None, O, WS, 1 << 20, None) == C.LA_ERR_UNSUPPORTED
    p = _params(B=1 << 12, H=1 << 12, N=256 * 32, rope=0, mode=C.LA_TOKEN_CAUSAL)
    assert C.lin_attn_forward(p, Q, K, V, None, O, WS, 1 << 20, None) == C.LA_ERR_UNSUPPORTED
    # 2^24 heads with 64 segments each fit (2^30): past the host checks
    # (fake pointers 2^40 bytes apart, clear of one another at this size)
    p = _params(B=1 << 12, H=1 << 12, N=64, rope=0, mode=C.LA_BLOCK_CAUSAL, block_tokens=1)
    far = [i << 40 for i in range(1, 6)]
    assert C.lin_attn_forward(p, far[0], far[1], far[2], None, far[3], far[4], 1 << 20,
                              None) not in (C.LA_ERR_UNSUPPORTED, C.LA_ERR_INVALID_ARG)


def test_layout_field():
    # [B,N,H,D] passes the host checks; anything else but the two orders is refused
    p = _params(layout=C.LA_LAYOUT_BNHD)
    assert C.lin_attn_forward(p, Q, K, V, None, O, WS, 1 << 20, None) != C.LA_ERR_INVALID_ARG
    assert C.lin_attn_forward(_params(layout=2), Q, K, V, None, O, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    assert C.lin_attn_uses_tensor_cores(_params(D=64, rope_dt=16, rope_dh=24, rope_dw=24,
                                                layout=C.LA_LAYOUT_BNHD)) == 1


def test_block_step_rejects_tensors_sharing_bytes_with_the_state():
    # A block step reads the state and (commit) updates it in place while q,
    # k, v and gate are still being read and out written, so none of them may
    # overlap S or z, and S and z may not overlap each other.
    p = _params()                       # B=1, H=2, N=60, D=32, bf16: 7680-byte tensors
    S, Z = 0x100000, 0x110000           # S: 8192 bytes, z: 256 bytes
    st = C.la_state()
    assert C.lin_attn_state_init(st, 1, 2, 32, S, Z) == C.LA_OK
    # clear of the state: past the host checks (fails only at the device query)
    assert C.lin_attn_block_step(p, st, 0, Q, K, V, None, O, 1, WS, 1 << 20, None) != \
        C.LA_ERR_INVALID_ARG
    bad = [
        (Q, K, V, None, S + 64),        # out inside S
        (Q, K, V, None, Z - 128),       # out running into z
        (S + 4096, K, V, None, O),      # q inside S
        (Q, Z, V, None, O),             # k on z
        (Q, K, S, None, O),             # v on S
        (Q, K, V, Z - 16, O),           # gate running into z
    ]
    for q, k, v, g, o in bad:
        assert C.lin_attn_block_step(p, st, 0, q, k, v, g, o, 1, WS, 1 << 20, None) == \
            C.LA_ERR_INVALID_ARG, (q, k, v, g, o)
    assert C.lin_attn_state_update(p, st, 0, Z, V, WS, 1 << 20, None) == C.LA_ERR_INVALID_ARG
    assert C.lin_attn_state_update(p, st, 0, K, S + 8176, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG
    # S and z sharing bytes
    st2 = C.la_state()
    assert C.lin_attn_state_init(st2, 1, 2, 32, S, S + 4096) == C.LA_OK
    assert C.lin_attn_block_step(p, st2, 0, Q, K, V, None, O, 1, WS, 1 << 20, None) == \
        C.LA_ERR_INVALID_ARG


def test_state_init_accepts_every_head_dim_of_the_forward():
    st = C.la_state()
    for d in (32, 64, 112, 128):
        assert C.lin_attn_state_init(st, 1, 2, d, 0x100000, 0x200000) == C.LA_OK
        assert st.D == d
    assert C.lin_attn_state_init(st, 1, 2, 96, 0x100000, 0x200000) == C.LA_ERR_INVALID_ARG
