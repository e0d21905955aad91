"""Torch-facing wrapper of the C ABI: tensors in, tensors out.

PyTorch provides device memory and streams only; the computation is the
CUDA library's. Shapes follow include/linattn.h: q, k, v, gate, out are
contiguous [B, H, N, D] (layout="bhnd") or [B, N, H, D] (layout="bnhd") in
bf16 or fp32; the carried state is fp32 S [B, H, D, D] and z [B, H, D].
"""
from __future__ import annotations

import contextlib
from typing import Optional, Sequence

import torch

from . import _native as C

_DTYPES = {torch.bfloat16: C.LA_BF16, torch.float32: C.LA_F32}
_MODES = {"bidirectional": C.LA_BIDIRECTIONAL, "block_causal": C.LA_BLOCK_CAUSAL,
          "token_causal": C.LA_TOKEN_CAUSAL}
_LAYOUTS = {"bhnd": C.LA_LAYOUT_BHND, "bnhd": C.LA_LAYOUT_BNHD}


def _dims(t: torch.Tensor, layout: str):
    """(B, H, N, D) of a [B, H, N, D] or [B, N, H, D] tensor."""
    if layout not in _LAYOUTS:
        raise ValueError("layout must be 'bhnd' or 'bnhd'")
    if t.dim() != 4:
        raise ValueError("expected a 4D tensor, got shape %s" % (tuple(t.shape),))
    a, b, c, d = (int(x) for x in t.shape)
    return (a, b, c, d) if layout == "bhnd" else (a, c, b, d)


def make_params(B: int, H: int, N: int, D: int, dtype: torch.dtype, mode: str = "bidirectional",
                block_tokens: int = 0, grid: Optional[Sequence[int]] = None,
                rope_split: Optional[Sequence[int]] = None, theta: float = 10000.0,
                eps: float = 1e-6, layout: str = "bhnd") -> C.la_params:
    p = C.la_params()
    p.B, p.H, p.N, p.D = B, H, N, D
    if dtype not in _DTYPES:
        raise TypeError("dtype must be torch.bfloat16 or torch.float32")
    p.dtype = _DTYPES[dtype]
    p.mode = _MODES[mode]
    p.block_tokens = block_tokens
    p.rope = 1 if grid is not None else 0
    if grid is not None:
        p.grid_t, p.grid_h, p.grid_w = (int(x) for x in grid)
        p.rope_dt, p.rope_dh, p.rope_dw = (int(x) for x in rope_split)
    p.rope_theta = float(theta)
    p.eps = float(eps)
    if layout not in _LAYOUTS:
        raise ValueError("layout must be 'bhnd' or 'bnhd'")
    p.layout = _LAYOUTS[layout]
    return p


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


# torch's raw current-stream query, when this torch has it: the handle without
# building a Stream object (a per-call cost on the host)
_current_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream: Optional[torch.cuda.Stream], device: Optional[int] = None):
    """The handle of `stream`, else of the current stream of `device` (an
    index; None: the current device)."""
    if stream is not None:
        return stream.cuda_stream
    if device is None:
        device = torch.cuda.current_device()
    if _current_raw_stream is not None:
        return _current_raw_stream(device)
    return torch.cuda.current_stream(device).cuda_stream


def _on_device(t: torch.Tensor):
    """t's device made current for the call; no switch when it already is."""
    idx = t.get_device()
    if idx == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(idx)


_DTYPE_OF = {v: k for k, v in _DTYPES.items()}


def _same_device(ref: torch.Tensor, *ts):
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError("all tensors must be on %s, got one on %s" % (ref.device, t.device))


def _check_io(p: C.la_params, *ts, require_cuda: bool = True):
    """Contiguous CUDA tensors of shape [B, H, N, D] (or [B, N, H, D]) in the
    params' dtype (require_cuda=False checks the rest on host tensors)."""
    shape = ((p.B, p.H, p.N, p.D) if p.layout == C.LA_LAYOUT_BHND else (p.B, p.N, p.H, p.D))
    dt = _DTYPE_OF[p.dtype]
    for t in ts:
        if t is None:
            continue
        if t.dtype is dt and t.is_contiguous() and t.shape == shape and (t.is_cuda or
                                                                         not require_cuda):
            continue
        if (require_cuda and not t.is_cuda) or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if tuple(t.shape) != shape:
            raise ValueError("expected shape %s, got %s" % (shape, tuple(t.shape)))
        if t.dtype != _DTYPE_OF[p.dtype]:
            raise TypeError("expected dtype %s, got %s" % (_DTYPE_OF[p.dtype], t.dtype))


class Workspace:
    """A device scratch buffer sized by the library, zeroed once: its leading
    control block must be zero before the first call, and every call leaves it
    zero."""

    def __init__(self, nbytes: int, device):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self):
        return self.buf.data_ptr()

    def control_block_is_zero(self) -> bool:
        n = min(self.nbytes, C.LA_WORKSPACE_CONTROL_BYTES)
        return int(torch.count_nonzero(self.buf[:n])) == 0

    def status(self, stream=None) -> int:
        """Synchronise and read the bounded-wait flag (see lin_attn_device_status)."""
        return C.lin_attn_device_status(self.ptr, _stream(stream))


def workspace_for(p: C.la_params, device, block_step: bool = False) -> Workspace:
    with torch.cuda.device(device):
        n = C.lin_attn_block_step_workspace_size(p) if block_step else C.lin_attn_workspace_size(p)
    return Workspace(n, device)


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor] = None,
            *, mode: str = "bidirectional", block_tokens: int = 0,
            grid: Optional[Sequence[int]] = None, rope_split: Optional[Sequence[int]] = None,
            theta: float = 10000.0, eps: float = 1e-6, out: Optional[torch.Tensor] = None,
            workspace: Optional[Workspace] = None, stream=None,
            layout: str = "bhnd") -> torch.Tensor:
    """out = RoPE(phi q) S / (phi q . z + eps) [* sigmoid(gate)] over [B, H, N, D]
    tensors (or [B, N, H, D] ones with layout="bnhd")."""
    B, H, N, D = _dims(q, layout)
    p = make_params(B, H, N, D, q.dtype, mode, block_tokens, grid, rope_split, theta, eps,
                    layout)
    _check_io(p, q, k, v, gate)
    if out is None:
        out = torch.empty_like(q)
    _check_io(p, out)
    _same_device(q, k, v, gate, out, None if workspace is None else workspace.buf)
    if workspace is None:
        workspace = workspace_for(p, q.device)
    with _on_device(q):
        C.check(C.lin_attn_forward(p, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(out),
                                   workspace.ptr, workspace.nbytes,
                                   _stream(stream, q.get_device())), "lin_attn_forward")
    return out


def cross_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  gate: Optional[torch.Tensor] = None, *, eps: float = 1e-6,
                  out: Optional[torch.Tensor] = None, workspace: Optional[Workspace] = None,
                  stream=None, layout: str = "bhnd") -> torch.Tensor:
    """Linear cross-attention: q, gate, out [B, H, N, D] read the state of
    k, v [B, H, M, D] (no RoPE; every query sees every key); [B, N, H, D] and
    [B, M, H, D] with layout="bnhd"."""
    B, H, N, D = _dims(q, layout)
    kB, kH, M, kD = _dims(k, layout)
    if (kB, kH, kD) != (B, H, D):
        raise ValueError("k must have q's B, H and D; got shape %s" % (tuple(k.shape),))
    p = make_params(B, H, N, D, q.dtype, eps=eps, layout=layout)
    pk = make_params(B, H, M, D, q.dtype, eps=eps, layout=layout)
    _check_io(p, q, gate)
    _check_io(pk, k, v)
    if out is None:
        out = torch.empty_like(q)
    _check_io(p, out)
    _same_device(q, k, v, gate, out, None if workspace is None else workspace.buf)
    if workspace is None:
        with torch.cuda.device(q.device):
            workspace = Workspace(C.lin_attn_cross_workspace_size(p, M), q.device)
    with _on_device(q):
        C.check(C.lin_attn_cross_forward(p, M, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(out),
                                         workspace.ptr, workspace.nbytes,
                                         _stream(stream, q.get_device())),
                "lin_attn_cross_forward")
    return out


class BlockState:
    """The constant-memory cache (S, z) of block-causal generation."""

    def __init__(self, B: int, H: int, D: int, device="cuda"):
        self.S = torch.zeros((B, H, D, D), dtype=torch.float32, device=device)
        self.z = torch.zeros((B, H, D), dtype=torch.float32, device=device)
        self.B, self.H, self.D = B, H, D
        self._st = C.la_state()
        C.check(C.lin_attn_state_init(self._st, B, H, D, self.S.data_ptr(), self.z.data_ptr()),
                "lin_attn_state_init")
        self._ws = {}
        self._plans = {}

    def reset(self, stream=None) -> None:
        with torch.cuda.device(self.S.device):
            C.check(C.lin_attn_state_reset(self._st, _stream(stream)), "lin_attn_state_reset")

    def _workspace(self, p):
        key = (p.N, p.D, p.dtype, p.rope, p.grid_t, p.grid_h, p.grid_w, p.rope_dt, p.rope_dh,
               p.rope_dw, p.layout)
        ws = self._ws.get(key)
        if ws is None:
            ws = workspace_for(p, self.S.device, block_step=True)
            self._ws[key] = ws
        return ws

    def _plan(self, x, grid, rope_split, theta, eps, layout):
        """(params, workspace) of a block of x's shape and dtype with these
        settings, made once per distinct call and kept (params are only read
        by the library)."""
        key = (x.shape, x.dtype, None if grid is None else tuple(grid),
               None if rope_split is None else tuple(rope_split), theta, eps, layout)
        ent = self._plans.get(key)
        if ent is None:
            B, H, N, D = _dims(x, layout)
            p = make_params(B, H, N, D, x.dtype, "bidirectional", 0, grid, rope_split, theta,
                            eps, layout)
            ent = (p, self._workspace(p))
            self._plans[key] = ent
        return ent

    def step(self, q, k, v, gate=None, *, t_offset: int = 0, commit: bool = True,
             grid=None, rope_split=None, theta: float = 10000.0, eps: float = 1e-6,
             out=None, stream=None, layout: str = "bhnd") -> torch.Tensor:
        """One block of block-causal attention against the carried state."""
        p, ws = self._plan(q, grid, rope_split, theta, eps, layout)
        _check_io(p, q, k, v, gate)
        if out is None:
            out = torch.empty_like(q)
        else:
            _check_io(p, out)
        _same_device(self.S, q, k, v, gate, out)
        dev = q.get_device()
        with _on_device(q):
            C.check(C.lin_attn_block_step(p, self._st, t_offset, q.data_ptr(), k.data_ptr(),
                                          v.data_ptr(), _ptr(gate), out.data_ptr(),
                                          1 if commit else 0, ws.ptr, ws.nbytes,
                                          _stream(stream, dev)), "lin_attn_block_step")
        return out

    def update(self, k, v, *, t_offset: int = 0, grid=None, rope_split=None,
               theta: float = 10000.0, stream=None, layout: str = "bhnd") -> None:
        """Fold a block's k, v into the state without producing output."""
        p, ws = self._plan(k, grid, rope_split, theta, 1e-6, layout)
        _check_io(p, k, v)
        _same_device(self.S, k, v)
        with _on_device(k):
            C.check(C.lin_attn_state_update(p, self._st, t_offset, k.data_ptr(), v.data_ptr(),
                                            ws.ptr, ws.nbytes, _stream(stream, k.get_device())),
                    "lin_attn_state_update")


def uses_tensor_cores(B, H, N, D, dtype, **kw) -> bool:
    return bool(C.lin_attn_uses_tensor_cores(make_params(B, H, N, D, dtype, **kw)))


def temporal_conv(x: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                  cache_in: Optional[torch.Tensor] = None, *,
                  cache_out: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """Mix-FFN temporal convolution with the last-frame cache:
    y[t] = x[t] + w0 * x[t-1] + w1 * x[t] + w2 * x[t+1] (+ bias), per channel,
    with a zero frame after the block and cache_in (or zero) before it.

    x, out: [B, T, S, C] or [B, T, Hg, Wg, C] (bf16 or fp32); weight fp32
    [3, C]; bias fp32 [C]; cache_in, cache_out: one frame, [B, S, C] or
    [B, Hg, Wg, C], in x's dtype. cache_out receives x's last frame (it may be
    cache_in itself)."""
    if x.dim() not in (4, 5):
        raise ValueError("x must be [B, T, S, C] or [B, T, Hg, Wg, C]")
    if x.dtype not in _DTYPES:
        raise TypeError("x must be bf16 or fp32")
    B, T, nc = int(x.shape[0]), int(x.shape[1]), int(x.shape[-1])
    S = 1
    for d in x.shape[2:-1]:
        S *= int(d)
    frame_shape = (B,) + tuple(x.shape[2:])
    if out is None:
        out = torch.empty_like(x)
    for t, shape, dt, what in ((x, tuple(x.shape), x.dtype, "x"),
                               (out, tuple(x.shape), x.dtype, "out"),
                               (weight, (3, nc), torch.float32, "weight"),
                               (bias, (nc,), torch.float32, "bias"),
                               (cache_in, frame_shape, x.dtype, "cache_in"),
                               (cache_out, frame_shape, x.dtype, "cache_out")):
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous CUDA tensor" % what)
        if tuple(t.shape) != shape or t.dtype != dt:
            raise ValueError("%s must be %s %s, got %s %s" % (what, shape, dt, tuple(t.shape),
                                                            t.dtype))
    _same_device(x, out, weight, bias, cache_in, cache_out)
    with torch.cuda.device(x.device):
        C.check(C.lin_attn_temporal_conv(B, T, S, nc, _DTYPES[x.dtype], _ptr(x), _ptr(weight),
                                         _ptr(bias), _ptr(cache_in), _ptr(out), _ptr(cache_out),
                                         _stream(stream)),
                "lin_attn_temporal_conv")
    return out
