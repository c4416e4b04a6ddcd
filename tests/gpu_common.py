"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library's stages through the C ABI, read intermediate results out of the
workspace, and compare with the CPU oracle under the stated criteria."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

import level_sparse_attention_b200 as P
import oracle as O
import workloads as W

# Tolerances: bf16 outputs against the fp64 oracle fed the same map; fp32 path.
BF16_MAX_ABS, BF16_MEAN_REL = 2e-2, 5e-3
F32_MAX_ABS = 1e-4
# Map parity: a level may differ only when the oracle's cumulative mass is this
# close to a threshold separating the two levels (absolute), or the block's
# mass is this close, relative to the larger of the two, to that of a block
# holding the GPU's level (a near-tie in the ranking).  The GPU's block masses
# carry a relative error of about 1e-5 (split-precision fp32 logits, fp32
# softmax), so two masses closer than that may rank either way.
MAP_EPS_C, MAP_EPS_P_REL = 1e-5, 1e-4


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(x).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def params_for(w: W.Workload, tau=None) -> P.Params:
    return P.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.q_blk, w.kv_blk,
                         W.thresholds(w) if tau is None else tau, w.causal,
                         w.forced_prefix_tokens, 0.0,
                         torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                         P.ASSIGN_QUANTILE if w.assign == "quantile" else P.ASSIGN_THRESHOLD)


@dataclass
class GpuRun:
    p: P.Params
    ws: torch.Tensor
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    level_map: torch.Tensor
    mass: torch.Tensor
    O: torch.Tensor
    lse: torch.Tensor

    def view(self, key, shape, dtype, level=None):
        L = P.workspace_layout(self.p)
        off = L[key] if level is None else L[key][level]
        return P.workspace_view(self.ws, off, shape, dtype)


def run_stages(w: W.Workload, inp: W.Inputs, tau=None, external_map: Optional[np.ndarray] = None,
               fused: bool = False) -> GpuRun:
    p = params_for(w, tau)
    ws = P.new_workspace(p)
    q, k, v = (to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    lm = torch.full(P.map_shape(p), -7, dtype=torch.int8, device="cuda")
    mass = torch.zeros(P.map_shape(p), dtype=torch.float32, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    if fused:
        P.forward(p, q, k, v, out, ws, lse, lm)
    else:
        P.build_pyramid(p, k, v, ws)
        P.score_and_mask(p, q, ws, lm, mass)
        ext = None
        if external_map is not None:
            ext = torch.from_numpy(np.ascontiguousarray(external_map, dtype=np.int8)).cuda()
        P.attention_fwd(p, q, k, v, ws, out, lse, ext)
    torch.cuda.synchronize()
    # a caller's map that breaks the contract (out-of-range values; causally,
    # future or pooled diagonal blocks) is corrected on the device and
    # reported as PSA_ERR_LEVEL_MAP; the oracle corrects it the same way
    changed = 0
    if external_map is not None and not fused:
        changed = sum(O.correct_map(external_map[b, h], w.N, w.q_blk, w.kv_blk, w.causal)[1]
                      for b in range(w.B) for h in range(w.Hq))
    if changed:
        try:
            P.check_device(p, ws)
            raise AssertionError("a corrected map was not reported")
        except P.PSAError as e:
            assert e.status == 7, e
    P.check_device(p, ws)
    return GpuRun(p, ws, q, k, v, lm, mass, out, lse)


def oracle_heads(w: W.Workload, inp: W.Inputs, heads, tau=None, level_map=None):
    """Oracle results for the listed (b, hq) heads: dict -> HeadResult."""
    tau = W.thresholds(w) if tau is None else tau
    grp = w.Hq // w.Hkv
    res = {}
    for b, h in heads:
        Q = inp.as_f64("q", b, h)
        K = inp.as_f64("k", b, h // grp)
        V = inp.as_f64("v", b, h // grp)
        res[(b, h)] = O.psa_head(Q, K, V, w.q_blk, w.kv_blk, tau, w.causal,
                                 w.forced_prefix_tokens, None,
                                 None if level_map is None else level_map[b, h], rule=w.assign)
    return res


def map_mismatch_report(gpu_map: np.ndarray, mask: O.MaskResult, tau: Sequence[float],
                        rule: str = "threshold"):
    """Counts (unexplained, near_threshold, near_tie) mismatches of one head's map.
    Under the quantile rule levels follow ranks only, so no mismatch is
    excused by a running mass near a threshold; near-ties still are."""
    om = mask.level_map
    unexplained = near_thr = near_tie = 0
    bad = np.argwhere(gpu_map != om)
    for a, j in bad:
        g, o = int(gpu_map[a, j]), int(om[a, j])
        lo, hi = sorted((4 if g < 0 else g, 4 if o < 0 else o))
        c = mask.cum_before[a, j]
        if rule == "threshold" and any(abs(c - tau[l]) < MAP_EPS_C for l in range(lo, min(hi, 4))):
            near_thr += 1
            continue
        pj = mask.mass[a, j]
        close = np.abs(mask.mass[a] - pj) <= MAP_EPS_P_REL * np.maximum(mask.mass[a], pj)
        close[j] = False
        if np.any(close & (om[a] == g)):
            near_tie += 1
            continue
        unexplained += 1
    return unexplained, near_thr, near_tie


def compare_out(gpu_O: np.ndarray, ref_O: np.ndarray, dtype: str, rows: Optional[np.ndarray] = None):
    """Returns (max_abs, mean_rel) and asserts the dtype's tolerance."""
    if rows is not None:
        gpu_O, ref_O = gpu_O[rows], ref_O[rows]
    diff = np.abs(gpu_O - ref_O)
    max_abs = float(diff.max()) if diff.size else 0.0
    mean_rel = float(diff.mean() / max(np.abs(ref_O).mean(), 1e-30)) if diff.size else 0.0
    if dtype == "bf16":
        assert max_abs <= BF16_MAX_ABS and mean_rel <= BF16_MEAN_REL, (max_abs, mean_rel)
    else:
        assert max_abs <= F32_MAX_ABS, max_abs
    return max_abs, mean_rel


def compare_lse(gpu_lse: np.ndarray, ref_lse: np.ndarray, dtype: str):
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(gpu_lse))
    if fin.any():
        err = np.abs(gpu_lse[fin] - ref_lse[fin]).max()
        assert err <= (2e-2 if dtype == "bf16" else 1e-4), err
    assert np.all(np.isneginf(gpu_lse[~fin]))


def rand_map(rng, Nq, Nk, lo=-1, hi=4) -> np.ndarray:
    return rng.integers(lo, hi, size=(Nq, Nk)).astype(np.int8)


def sequence_map(rng, Nq, Nk) -> np.ndarray:
    """A row keeps no block (a quarter of the rows), or 1 to 16 random blocks
    at random levels: 0 to 8 packed tiles per query block, mixed along every
    persistent CTA's sequence of blocks when there are many query blocks."""
    m = np.full((Nq, Nk), -1, dtype=np.int8)
    for a in range(Nq):
        if rng.random() < 0.25:
            continue
        n = int(rng.choice([1, 2, 3, 4, 6, 10, 16]))
        js = rng.permutation(Nk)[:n]
        m[a, js] = rng.integers(0, 4, size=len(js))
    return m
