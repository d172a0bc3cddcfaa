"""Seeded synthetic inputs for the DiG token mixer.

This module holds only the input recipe: shapes, random draws and bf16
rounding.  It contains none of the method's arithmetic and is the one module
shared by the CUDA path's tests and the oracle's tests.

Workloads (DiG-S/2 and DiG-XL/2 token mixers; L = (resolution / 8 / patch)^2,
the VAE downsamples by 8 and the patch size is 2; the DiG paper's Fig. 1 caption
pairs 1792x1792 with 12544 tokens, Table 1 gives D and the head count):

  0 tiny-fp32     B=1 H=1  16x16 grid (L=256)   dk=64 dv=64  fp32, gate logits ~ N(0,1)
  1 dig-s2-256    B=8 H=6  16x16 grid (L=256)   dk=32 dv=64  bf16, low-rank gate 384->16->32
  2 dig-s2-1024   B=4 H=6  64x64 grid (L=4096)  dk=32 dv=64  bf16
  3 dig-s2-1792   B=2 H=6  112x112 (L=12544)    dk=32 dv=64  bf16, + SREM conv (C=384) + epilogue
  4 dig-xl2-2048  B=1 H=16 128x128 (L=16384)    dk=36 dv=72  bf16, low-rank gate 1152->16->36

Draws: q, k ~ N(0,1)/sqrt(dk); v ~ N(0,1)/sqrt(dv); dO, r ~ N(0,1); the gate
logits z are either N(0,1) (workload 0) or x W1 W2 with x ~ N(0,1) [B,L,D] and
W1 [D,16], W2 [16,dk] ~ N(0, 0.02^2), bias 0; inv_tau = 1/16.  SREM conv input
~ N(0,1) [B,Hg,Wg,C], weights ~ N(0, 0.1^2) [C,3,3].  Tensors of a bf16 workload
are rounded to bf16 (round-to-nearest-even) and handed out as float32 arrays
holding bf16-exact values; z, the conv weights and gamma stay fp32.
Seed of workload i: 20240528 + i.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

SEED_BASE = 20240528


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid_h: int
    grid_w: int
    dk: int
    dv: int
    dtype: str            # "f32" or "bf16" (input storage type)
    gate: str             # "direct" (z ~ N(0,1)) or "lowrank" (z = x W1 W2)
    D: int = 0            # model width feeding the low-rank gate
    rank: int = 16
    inv_tau: float = 1.0 / 16.0
    conv_C: int = 0       # channels of the SREM conv (0: not part of the workload)
    epilogue: bool = False
    resolution: int = 0   # image side in pixels (context)

    @property
    def L(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def tokens(self) -> int:
        return self.B * self.L


WORKLOADS = [
    Workload("tiny-fp32", 1, 1, 16, 16, 64, 64, "f32", "direct", conv_C=64, resolution=256),
    Workload("dig-s2-256", 8, 6, 16, 16, 32, 64, "bf16", "lowrank", D=384, resolution=256),
    Workload("dig-s2-1024", 4, 6, 64, 64, 32, 64, "bf16", "lowrank", D=384, resolution=1024),
    Workload("dig-s2-1792", 2, 6, 112, 112, 32, 64, "bf16", "lowrank", D=384, conv_C=384,
             epilogue=True, resolution=1792),
    Workload("dig-xl2-2048", 1, 16, 128, 128, 36, 72, "bf16", "lowrank", D=1152, resolution=2048),
]


def tokens_for_resolution(resolution: int, vae_down: int = 8, patch: int = 2) -> int:
    side = resolution // vae_down // patch
    return side * side


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bf16 (ties to even); returns float32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    nan = np.isnan(f)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out.reshape(f.shape)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a)


def make_inputs(w: Workload, seed: int | None = None, with_conv: bool | None = None,
                with_epilogue: bool | None = None) -> dict:
    """All inputs of one workload as float32 numpy arrays (bf16-exact for bf16).

    Keys: q, k [B,L,H,dk]; v, dO [B,L,H,dv]; z [B,L,1,dk]; and, when asked for,
    r [B,L,H,dv] (epilogue), x_conv [B,Hg,Wg,C], w_conv [C,3,3] (SREM conv).
    Tokens are in grid row-major order.
    """
    if seed is None:
        seed = SEED_BASE + (WORKLOADS.index(w) if w in WORKLOADS else 0)
    rng = np.random.default_rng(seed)
    B, L, H, dk, dv = w.B, w.L, w.H, w.dk, w.dv
    out = {}
    out["q"] = _store(rng.standard_normal((B, L, H, dk)) / math.sqrt(dk), w.dtype)
    out["k"] = _store(rng.standard_normal((B, L, H, dk)) / math.sqrt(dk), w.dtype)
    out["v"] = _store(rng.standard_normal((B, L, H, dv)) / math.sqrt(dv), w.dtype)
    out["dO"] = _store(rng.standard_normal((B, L, H, dv)), w.dtype)
    if w.gate == "direct":
        z = rng.standard_normal((B, L, 1, dk))
    else:
        x = rng.standard_normal((B, L, w.D))
        w1 = 0.02 * rng.standard_normal((w.D, w.rank))
        w2 = 0.02 * rng.standard_normal((w.rank, dk))
        z = ((x @ w1) @ w2).reshape(B, L, 1, dk)
    out["z"] = np.ascontiguousarray(z, dtype=np.float32)
    if with_epilogue if with_epilogue is not None else w.epilogue:
        out["r"] = _store(rng.standard_normal((B, L, H, dv)), w.dtype)
    conv = with_conv if with_conv is not None else (w.conv_C > 0)
    if conv:
        C = w.conv_C or H * dv
        out["x_conv"] = _store(rng.standard_normal((B, w.grid_h, w.grid_w, C)), w.dtype)
        out["w_conv"] = np.ascontiguousarray(0.1 * rng.standard_normal((C, 3, 3)), dtype=np.float32)
    return out


def gate_proj_inputs(w: Workload, seed: int, dtype: str | None = None, with_bias: bool = False) -> dict:
    """Inputs of the gate projection for workload w: x [B, L, D] ~ N(0,1) (stored in
    the workload's dtype), W1 [D, rank] and W2 [rank, dk] ~ N(0, 0.02^2) and, when
    asked for, b [dk] ~ N(0, 1), all float32 numpy arrays (bf16-exact x for bf16)."""
    rng = np.random.default_rng(seed)
    D = w.D or 384
    out = {"x": _store(rng.standard_normal((w.B, w.L, D)), dtype or w.dtype),
           "W1": np.ascontiguousarray(0.02 * rng.standard_normal((D, w.rank)), dtype=np.float32),
           "W2": np.ascontiguousarray(0.02 * rng.standard_normal((w.rank, w.dk)), dtype=np.float32)}
    if with_bias:
        out["b"] = np.ascontiguousarray(rng.standard_normal(w.dk), dtype=np.float32)
    return out


def custom(B, H, grid_h, grid_w, dk, dv, dtype="bf16", gate="direct", inv_tau=1.0 / 16.0,
           D=384, conv_C=0) -> Workload:
    """A workload of arbitrary shape with the same generators (parity edge cases)."""
    return Workload("custom", B, H, grid_h, grid_w, dk, dv, dtype, gate, D=D, inv_tau=inv_tau,
                    conv_C=conv_C)


def strong_gate(w: Workload, kind: str, seed: int, gate_heads: int = 1) -> np.ndarray:
    """Gate logits z [B, L, gate_heads, dk] (float32) whose decay within a chunk
    leaves the range of the chunk factorisation (more than 115 halvings over half
    a chunk in some key channel), for the strong-gate parity cases:
      "alpha0": z = -1e4 everywhere, so alpha = 0 to fp32 precision and the state
                keeps only the current token (o_t = (q_t . k_t) v_t);
      "tau1":   z ~ N(-3, 1), meant with inv_tau = 1 (alpha ~ 0.05, ~4.4 halvings per token);
      "mixed":  z ~ N(0, 1), except z = -1e4 on the grid tokens of the top-left
                quadrant (rows < grid_h / 2, columns < grid_w / 2), so that every scan
                order has both flagged and ordinary chunks, and flagged chunks hold
                ordinary tokens too."""
    rng = np.random.default_rng(seed)
    B, L, dk = w.B, w.L, w.dk
    if kind == "alpha0":
        z = np.full((B, L, gate_heads, dk), -1e4)
    elif kind == "tau1":
        z = rng.standard_normal((B, L, gate_heads, dk)) - 3.0
    elif kind == "mixed":
        z = rng.standard_normal((B, L, gate_heads, dk))
        gy, gx = np.divmod(np.arange(L), w.grid_w)
        quad = (gy < w.grid_h // 2) & (gx < w.grid_w // 2)
        z[:, quad] = -1e4
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(z, dtype=np.float32)
