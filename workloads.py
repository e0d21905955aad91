"""Seeded synthetic workloads for ReLU linear attention with 3D RoPE.

This module only draws random numbers and rounds them to the I/O precision.
It holds none of the attention arithmetic, so both the fp64 oracle (under
``oracle/``) and the CUDA path (``linear_attention_video_relu_b200``) can take
their inputs from it without sharing any of the method.

Shapes follow the latent token grids of the SANA-Video pages: a 480p, 81-frame
clip is 21 latent frames of 30 x 52 tokens (N = 32760); a 720p, 60-second clip
is 240 latent frames of 23 x 40 tokens (N = 220800). Tensors are laid out
``[B, H, N, D]`` with D innermost and the token index n = (t*Hg + h)*Wg + w.

Recipe (also stated in the design notes): one numpy PCG64 generator per
workload, seeded with the workload's seed; q, k, v are drawn in that order,
then the gate logits g. Normal draws are ``standard_normal`` in fp32; the
outlier-heavy workload draws q, k from a Student-t with 3 degrees of freedom
divided by sqrt(3) (unit variance). bf16 workloads round each fp32 sample to
bf16 with round-to-nearest-even; the rounded values are exact in fp32 and are
what both the oracle and the GPU see.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np

BIDIRECTIONAL = "bidirectional"
BLOCK_CAUSAL = "block_causal"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: str                      # "f32" or "bf16" (I/O precision)
    seed: int
    grid: Optional[Tuple[int, int, int]] = None     # (T, Hg, Wg); None = no RoPE
    rope_split: Optional[Tuple[int, int, int]] = None
    rope_theta: float = 10000.0
    gate: bool = False
    modes: Tuple[str, ...] = (BIDIRECTIONAL,)
    block_tokens: int = 0           # block-causal block size in tokens
    qk_dist: str = "normal"         # "normal" or "student_t3"
    eps: float = 1e-6

    @property
    def rope(self) -> bool:
        return self.grid is not None

    def algorithmic_bytes(self) -> int:
        """Bytes the op must move once: read q, k, v (+ g), write out."""
        elt = 2 if self.dtype == "bf16" else 4
        ntensors = 5 if self.gate else 4
        return ntensors * self.B * self.H * self.N * self.D * elt

    def scaled(self, frames: int, name_suffix: str = "_small") -> "Workload":
        """Same structure with fewer latent frames (for fast parity runs)."""
        if self.grid is None:
            raise ValueError("only grid workloads can be scaled by frames")
        T, Hg, Wg = self.grid
        n = frames * Hg * Wg
        bt = self.block_tokens
        if bt:
            fpb = bt // (Hg * Wg)
            if frames % fpb:
                raise ValueError("frames must be a multiple of frames per block")
        return dataclasses.replace(self, name=self.name + name_suffix, N=n,
                                   grid=(frames, Hg, Wg))


# The five workloads: shapes, distributions, RoPE splits, modes and seeds.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        name="tiny_f32", B=1, H=2, N=256, D=32, dtype="f32", seed=1001),
    "480p_bidir": Workload(
        name="480p_bidir", B=1, H=32, N=32760, D=64, dtype="bf16", seed=1002,
        grid=(21, 30, 52), rope_split=(16, 24, 24)),
    "480p_block_causal": Workload(
        name="480p_block_causal", B=1, H=32, N=32760, D=64, dtype="bf16",
        seed=1003, grid=(21, 30, 52), rope_split=(16, 24, 24),
        modes=(BLOCK_CAUSAL,), block_tokens=3 * 30 * 52),
    "720p_long": Workload(
        name="720p_long", B=1, H=32, N=220800, D=64, dtype="bf16", seed=1004,
        grid=(240, 23, 40), rope_split=(16, 24, 24),
        modes=(BIDIRECTIONAL, BLOCK_CAUSAL), block_tokens=4 * 23 * 40),
    "gated_d128": Workload(
        name="gated_d128", B=8, H=16, N=4096, D=128, dtype="bf16", seed=1005,
        grid=(16, 16, 16), rope_split=(32, 48, 48), gate=True,
        qk_dist="student_t3"),
}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.

    The inputs here are finite, so no NaN handling is needed.
    """
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((bits >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((bits + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw(rng: np.random.Generator, dist: str, shape) -> np.ndarray:
    if dist == "normal":
        out = np.empty(shape, dtype=np.float32)
        flat = out.reshape(-1)
        step = 1 << 24
        for i in range(0, flat.size, step):
            flat[i:i + step] = rng.standard_normal(min(step, flat.size - i),
                                                   dtype=np.float32)
        return out
    if dist == "student_t3":
        return (rng.standard_t(3, size=shape) / math.sqrt(3.0)).astype(np.float32)
    raise ValueError(dist)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw q, k, v (and g) for workload ``w``.

    Returns fp32 arrays holding the values in I/O precision (bf16-rounded for
    bf16 workloads) and, for bf16 workloads, the raw bf16 bit patterns under
    ``"<name>_bits"`` for upload to the device.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    shape = (w.B, w.H, w.N, w.D)
    names = ["q", "k", "v"] + (["g"] if w.gate else [])
    out: Dict[str, np.ndarray] = {}
    for name in names:
        dist = w.qk_dist if name in ("q", "k") else "normal"
        x = _draw(rng, dist, shape)
        if w.dtype == "bf16":
            bits = round_to_bf16_bits(x)
            del x
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
        else:
            out[name] = x
    return out


# Hidden states of a DiT block at 480p (21 x 30 x 52 latent grid, width 2240):
# the temporal convolution's measured shape.
TCONV_480P = dict(B=1, T=21, S=30 * 52, C=2240)


def make_tconv_inputs(B: int, T: int, S: int, C: int, dtype: str, seed: int,
                      cache: bool = True, bias: bool = True) -> Dict[str, np.ndarray]:
    """Draw x [B, T, S, C], weight [3, C], bias [C] and a cache frame [B, S, C]
    for the Mix-FFN temporal convolution, in that order: x and the cache
    ~ N(0, 1) in I/O precision (plus ``*_bits`` for bf16), weight ~ 0.5 N(0, 1)
    and bias ~ 0.1 N(0, 1) in fp32 (the op's weight precision)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out: Dict[str, np.ndarray] = {}

    def io(name, shape):
        x = _draw(rng, "normal", shape)
        if dtype == "bf16":
            bits = round_to_bf16_bits(x)
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
        else:
            out[name] = x

    io("x", (B, T, S, C))
    out["weight"] = (0.5 * _draw(rng, "normal", (3, C))).astype(np.float32)
    if bias:
        out["bias"] = (0.1 * _draw(rng, "normal", (C,))).astype(np.float32)
    if cache:
        io("cache", (B, S, C))
    return out
