"""Seeded synthetic workloads for Pyramid Sparse Attention (PSA).

This module holds the workload shapes and the input generator only. It contains
none of PSA's arithmetic (no pooling, scoring, thresholding or attention), so the
CPU oracle (``oracle/``) and the CUDA path (``level_sparse_attention_b200``) can
both draw their inputs from it without sharing any method code.

The pages behind PSA measure on video generation (Wan2.1-1.3B, Wan2.1-14B,
CogVideoX-5B) and video understanding (Qwen2.5-VL on Video-MME); trained weights
and datasets are not available here, so Q/K/V are synthetic: a smooth 3-D field
on the latent (t, h, w) grid, upsampled trilinearly from a coarse grid, plus
i.i.d. noise.  The smooth field stands in for the similarity of neighbouring
frames that the top168.com article on PSA (arXiv:2512.04025) gives as the
motivation for pooling.

Recipe, per tensor X in (Q, K, V) and per head h (KV heads for K and V):
  * rng = numpy.random.default_rng([seed, tensor_index, h]) (tensor_index 0/1/2);
  * text tokens first (CogVideoX shape only): iid N(0,1), shape [n_text, d];
  * coarse field iid N(0,1) of shape [ct, ch, cw, d], then trilinear,
    align-corners upsampling to [T, H, W, d] (raster t, h, w order);
  * noise iid N(0,1) of shape [T*H*W, d];
  * value = 0.8 * field + 0.2 * noise, in float32, then rounded to the config's
    storage dtype (bf16 by round-to-nearest-even; fp32 unchanged).
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field, asdict
from typing import List, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
THRESHOLDS_FILE = os.path.join(_HERE, "thresholds.json")

# The cumulative-mass thresholds of the tiny case; the larger workloads scale
# this shape by alpha / 0.97 so that tau_3 = alpha.
TAU_SHAPE = (0.6, 0.8, 0.9, 0.97)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    dtype: str                      # "f32" or "bf16"
    grid: Tuple[int, int, int]      # latent (T, H, W) of the video tokens
    coarse: Tuple[int, int, int]    # coarse field grid
    n_text: int                     # text tokens before the video tokens
    q_blk: int
    kv_blk: int
    causal: bool
    forced_prefix_tokens: int       # KV blocks holding any of these tokens get level 0
    seed: int
    target: str                     # how tau is chosen: "fixed", "alpha:0.15", "binary:0.2",
                                    # "skip:0.91", "keep:0.35"
    pool: Tuple[int, int, int, int] = (1, 2, 4, 8)
    assign: str = "threshold"       # level assignment rule: "threshold" or "quantile"

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return self.n_text + t * h * w

    @property
    def Nq(self) -> int:
        return -(-self.N // self.q_blk)

    @property
    def Nk(self) -> int:
        return -(-self.N // self.kv_blk)

    def dense_flops(self) -> float:
        """4*B*Hq*d*(N^2, or N(N+1)/2 when causal): QK^T plus PV, 2 FLOPs per MAC."""
        N = self.N
        pairs = N * (N + 1) / 2 if self.causal else float(N) * N
        return 4.0 * self.B * self.Hq * self.d * pairs


def _coarse(n: int) -> int:
    return max(1, -(-n // 4))


WORKLOADS: List[Workload] = [
    Workload("tiny_f32", B=1, Hq=2, Hkv=2, d=64, dtype="f32", grid=(4, 16, 16),
             coarse=(1, 4, 4), n_text=0, q_blk=64, kv_blk=64, causal=False,
             forced_prefix_tokens=0, seed=0, target="fixed"),
    Workload("wan2.1_1.3b", B=1, Hq=12, Hkv=12, d=128, dtype="bf16", grid=(21, 30, 52),
             coarse=(_coarse(21), _coarse(30), _coarse(52)), n_text=0, q_blk=128,
             kv_blk=64, causal=False, forced_prefix_tokens=0, seed=1, target="skip:0.91"),
    Workload("cogvideox_5b", B=1, Hq=48, Hkv=48, d=64, dtype="bf16", grid=(13, 30, 45),
             coarse=(_coarse(13), _coarse(30), _coarse(45)), n_text=226, q_blk=128,
             kv_blk=64, causal=False, forced_prefix_tokens=226, seed=2, target="skip:0.85"),
    Workload("wan2.1_14b_720p", B=1, Hq=40, Hkv=40, d=128, dtype="bf16", grid=(21, 45, 80),
             coarse=(_coarse(21), _coarse(45), _coarse(80)), n_text=0, q_blk=128,
             kv_blk=64, causal=False, forced_prefix_tokens=0, seed=3, target="skip:0.90"),
    Workload("qwen2.5_vl_7b", B=1, Hq=28, Hkv=4, d=128, dtype="bf16", grid=(16, 32, 32),
             coarse=(_coarse(16), _coarse(32), _coarse(32)), n_text=0, q_blk=128,
             kv_blk=64, causal=True, forced_prefix_tokens=0, seed=4, target="keep:0.35"),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def thresholds(w: Workload) -> Tuple[float, float, float, float]:
    """The cumulative-mass thresholds tau_0..tau_3 of a workload.

    The tiny case fixes them; "alpha:X" scales the shape to tau_3 = X;
    "binary:X" sets all four to X (keep/drop: every kept block at level 0);
    the others read the alpha frozen in ``thresholds.json`` (written by
    ``oracle/tune_thresholds.py``)."""
    if w.target == "fixed":
        return TAU_SHAPE
    if w.target.startswith("binary:"):
        x = float(w.target.split(":", 1)[1])
        return (x, x, x, x)
    if w.target.startswith("alpha:"):
        alpha = float(w.target.split(":", 1)[1])
        return tuple(float(alpha * t / TAU_SHAPE[-1]) for t in TAU_SHAPE)
    with open(THRESHOLDS_FILE) as f:
        alpha = json.load(f)[w.name]["alpha"]
    return tuple(float(alpha * t / TAU_SHAPE[-1]) for t in TAU_SHAPE)


def with_overrides(w: Workload, **kw) -> Workload:
    d = asdict(w)
    d.update(kw)
    return Workload(**d)


# ---------------------------------------------------------------- generator

def _upsample_axis(x: np.ndarray, axis: int, n: int) -> np.ndarray:
    c = x.shape[axis]
    if c == n:
        return x
    if c == 1:
        return np.repeat(x, n, axis=axis)
    pos = np.arange(n, dtype=np.float64) * (c - 1) / max(n - 1, 1)
    i0 = np.floor(pos).astype(np.int64)
    i1 = np.minimum(i0 + 1, c - 1)
    wgt = (pos - i0).astype(np.float32)
    shape = [1] * x.ndim
    shape[axis] = n
    wgt = wgt.reshape(shape)
    return np.take(x, i0, axis=axis) * (1.0 - wgt) + np.take(x, i1, axis=axis) * wgt


def smooth_field(rng: np.random.Generator, grid, coarse, d: int) -> np.ndarray:
    """[T*H*W, d] float32 smooth field: coarse iid N(0,1), trilinear align-corners."""
    x = rng.standard_normal((*coarse, d), dtype=np.float32)
    for ax, n in enumerate(grid):
        x = _upsample_axis(x, ax, n)
    return np.ascontiguousarray(x.reshape(-1, d), dtype=np.float32)


def head_values(w: Workload, tensor_index: int, head: int, batch: int = 0) -> np.ndarray:
    """float32 [N, d] values of one head of Q (0), K (1) or V (2), before rounding."""
    rng = np.random.default_rng([w.seed, tensor_index, head, batch])
    parts = []
    if w.n_text:
        parts.append(rng.standard_normal((w.n_text, w.d), dtype=np.float32))
    fld = smooth_field(rng, w.grid, w.coarse, w.d)
    noise = rng.standard_normal(fld.shape, dtype=np.float32)
    parts.append(0.8 * fld + 0.2 * noise)
    return np.concatenate(parts, axis=0) if len(parts) > 1 else parts[0]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Inputs:
    """Q/K/V of one workload in storage form.

    ``q``, ``k``, ``v`` are numpy arrays [B, H, N, d]: float32 for "f32",
    uint16 bfloat16 bit patterns for "bf16".  ``as_f64`` gives the exact values
    the GPU receives, widened to float64."""
    w: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray

    def as_f64(self, name: str, b: Optional[int] = None, h: Optional[int] = None) -> np.ndarray:
        x = getattr(self, name)
        if b is not None:
            x = x[b]
            if h is not None:
                x = x[h]
        if self.w.dtype == "bf16":
            return bf16_bits_to_f32(x).astype(np.float64)
        return x.astype(np.float64)


def make_inputs(w: Workload, heads_q: Optional[List[int]] = None,
                heads_kv: Optional[List[int]] = None, batch0: int = 0) -> Inputs:
    """Generate the workload's inputs.  ``heads_q``/``heads_kv`` restrict the
    heads generated (others are left zero) so that samples stay cheap.
    ``batch0`` is the global index of the first batch element: local element b
    holds global batch element batch0 + b, so that ranks that each run their
    own share of a larger batch see different data."""
    N, d = w.N, w.d
    store = np.uint16 if w.dtype == "bf16" else np.float32
    out = []
    for ti, (H, sel) in enumerate(((w.Hq, heads_q), (w.Hkv, heads_kv), (w.Hkv, heads_kv))):
        arr = np.zeros((w.B, H, N, d), dtype=store)
        for b in range(w.B):
            for h in (range(H) if sel is None else sel):
                vals = head_values(w, ti, h, batch0 + b)
                arr[b, h] = f32_to_bf16_bits(vals) if w.dtype == "bf16" else vals
        out.append(arr)
    return Inputs(w, *out)
