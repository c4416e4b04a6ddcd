"""CPU oracle for the backward pass of Pyramid Sparse Attention, in float64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference legs of ``bench.py`` use it.  It shares no code with the CUDA
path.

Sources (the web pages describing PSA, arXiv:2512.04025):
  [news] top168.com article on arXiv:2512.04025: the pyramid levels are
         average-pooled copies of the original KV; adaptive pyramid attention
         keeps the probability distribution consistent; PSA is combined with
         the TDM distillation framework on CogVideoX-5B, which trains through
         the attention and so needs its gradients.
The pages print no backward pass.  Reading used here: the gradient of the
forward pass of ``psa_oracle.pyramid_attention`` with respect to Q, K and V,
with the level map held fixed (it is a discrete function of Q and K and passes
no gradient) and the ln c_g bias a constant.  The forward is the composition
  K_l = A_l K, V_l = A_l V           (A_l: the mean-pooling matrix of level l)
  x_ig = s q_i . K_l[g] + ln c_g     (keys g kept by row i's query block)
  P_ig = exp(x_ig - lse_i),  O_i = sum_g P_ig V_l[g]
so by the chain rule, with D_i = dO_i . O_i:
  dV_l[g] += sum_i P_ig dO_i
  dX_ig    = P_ig (dO_i . V_l[g] - D_i)
  dQ_i     = s sum_g dX_ig K_l[g]
  dK_l[g] += s sum_i dX_ig q_i
  dK = sum_l A_l^T dK_l,  dV = sum_l A_l^T dV_l
where A_l^T hands each pooled row's gradient, divided by its count c_g, to
each of the c_g tokens it averages.  Grouped queries: a KV head's gradients
sum over the query heads that read it.

Every function works on one (batch, head) slice; ``psa_backward`` loops.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional, Sequence

import numpy as np

from .psa_oracle import POOL, block_rows, build_pyramid, correct_map


def unpool(g: np.ndarray, counts: np.ndarray, f: int, N: int) -> np.ndarray:
    """Adjoint of ``psa_oracle.pool_tokens``: pooled row r averaged tokens
    [r*f, min((r+1)*f, N)), so each of them receives g[r] / c_r.
    g: [ceil(N/f), d].  Returns [N, d]."""
    out = np.empty((N, g.shape[1]), dtype=np.float64)
    for r in range(g.shape[0]):
        lo, hi = r * f, min((r + 1) * f, N)
        out[lo:hi] = g[r] / counts[r]
    return out


@dataclass
class HeadGrads:
    dQ: np.ndarray                 # [N, d]
    dK: np.ndarray                 # [N, d]   (this query head's share)
    dV: np.ndarray                 # [N, d]
    dK_levels: Dict[int, np.ndarray]   # gradients of the pooled levels, before unpooling
    dV_levels: Dict[int, np.ndarray]
    D: np.ndarray                  # [N]  dO_i . O_i


def pyramid_attention_backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray,
                               level_map: np.ndarray, dO: np.ndarray, bq: int, bk: int,
                               scale: Optional[float] = None, causal: bool = False,
                               pool: Sequence[int] = POOL) -> HeadGrads:
    """Gradients of one head's pyramid attention (see the module docstring).

    Q, K, V, dO: [N, d]; level_map [Nq, Nk] held fixed.  Query block a gathers
    the same kept keys as the forward pass (each kept block j's rows of level
    map[a, j], a token mask on causal diagonal blocks), recomputes P, and
    spreads the gradients back to the level rows they came from.  Rows that
    keep no key have O = 0 and pass no gradient.  The map is corrected as
    the forward pass corrects it (``psa_oracle.correct_map``)."""
    N, d = Q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    level_map, _ = correct_map(level_map, N, bq, bk, causal)
    pyr = build_pyramid(K, V, pool)
    Nq, Nk = level_map.shape
    dQ = np.zeros((N, d), dtype=np.float64)
    dKl = {l: np.zeros_like(pyr.keys[l]) for l in range(len(pool))}
    dVl = {l: np.zeros_like(pyr.values[l]) for l in range(len(pool))}
    D = np.zeros(N, dtype=np.float64)
    for a in range(Nq):
        segs, ks, vs, bias, kpos = [], [], [], [], []
        for j in range(Nk):
            l = int(level_map[a, j])
            if l < 0:
                continue
            rows = block_rows(j, l, bk, pyr, pool)
            segs.append((l, rows.start, rows.stop))
            ks.append(pyr.keys[l][rows.start:rows.stop])
            vs.append(pyr.values[l][rows.start:rows.stop])
            bias.append(np.log(pyr.counts[l][rows.start:rows.stop]))
            kpos.append(np.arange(rows.start, rows.stop) * pool[l] if l == 0
                        else np.full(len(rows), -1))
        if not segs:
            continue
        Kk, Vk = np.concatenate(ks), np.concatenate(vs)
        bias_a, kpos_a = np.concatenate(bias), np.concatenate(kpos)
        rows_i = np.arange(a * bq, min((a + 1) * bq, N))
        logit = s * (Q[rows_i] @ Kk.T) + bias_a[None, :]
        if causal:
            logit = np.where(kpos_a[None, :] > rows_i[:, None], -np.inf, logit)
        m = logit.max(axis=1)
        ok = np.isfinite(m)
        if not ok.any():
            continue
        ri = rows_i[ok]
        lg = logit[ok]
        lse = m[ok] + np.log(np.exp(lg - m[ok, None]).sum(axis=1))
        P = np.exp(lg - lse[:, None])                       # [rows, keys]
        O = P @ Vk
        g = dO[ri]
        Di = (g * O).sum(axis=1)
        D[ri] = Di
        dP = g @ Vk.T
        dX = P * (dP - Di[:, None])
        dQ[ri] = s * (dX @ Kk)
        dKk = s * (dX.T @ Q[ri])
        dVk = P.T @ g
        off = 0
        for l, r0, r1 in segs:
            n = r1 - r0
            dKl[l][r0:r1] += dKk[off:off + n]
            dVl[l][r0:r1] += dVk[off:off + n]
            off += n
    dK = np.zeros((N, d), dtype=np.float64)
    dV = np.zeros((N, d), dtype=np.float64)
    for l, f in enumerate(pool):
        dK += unpool(dKl[l], pyr.counts[l], f, N)
        dV += unpool(dVl[l], pyr.counts[l], f, N)
    return HeadGrads(dQ, dK, dV, dKl, dVl, D)


@dataclass
class BackwardResult:
    dQ: np.ndarray     # [B, Hq, N, d]
    dK: np.ndarray     # [B, Hkv, N, d]
    dV: np.ndarray     # [B, Hkv, N, d]
    D: np.ndarray      # [B, Hq, N]


def psa_backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray,
                 level_map: np.ndarray, bq: int, bk: int, causal: bool = False,
                 scale: Optional[float] = None) -> BackwardResult:
    """Backward over [B, Hq, N, d] queries and [B, Hkv, N, d] keys/values with
    a fixed int8 map [B, Hq, Nq, Nk].  Query head h reads KV head h // (Hq/Hkv);
    a KV head's gradients sum over its query heads."""
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    grp = Hq // Hkv
    dQ = np.zeros((B, Hq, N, d))
    dK = np.zeros((B, Hkv, N, d))
    dV = np.zeros((B, Hkv, N, d))
    D = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = pyramid_attention_backward(Q[b, h], K[b, h // grp], V[b, h // grp],
                                           level_map[b, h], dO[b, h], bq, bk, scale, causal)
            dQ[b, h] = g.dQ
            dK[b, h // grp] += g.dK
            dV[b, h // grp] += g.dV
            D[b, h] = g.D
    return BackwardResult(dQ, dK, dV, D)

