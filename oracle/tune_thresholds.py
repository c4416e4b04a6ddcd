"""Freeze the cumulative-mass thresholds of the larger workloads.

TEST INFRASTRUCTURE: calls only ``oracle/`` (and the seeded input generator).

The pages report sparsity levels (91% on Wan2.1-1.3B, about 35% of compute kept
on Qwen2.5-VL; top168.com article on arXiv:2512.04025, results paragraph) but
not the thresholds behind them.  Each workload's thresholds are
tau(alpha) = alpha * (0.6, 0.8, 0.9, 0.97) / 0.97, with alpha bisected on the
oracle's mask stage so that the executed fraction of dense FLOPs hits the
workload's target.  The ranking does not depend on alpha, so it is computed
once per head and only the level cut moves.

Usage: python -m oracle.tune_thresholds [workload ...]   (writes workloads/thresholds.json)
"""
from __future__ import annotations

import json
import math
import sys
import time

import numpy as np

import workloads as W
from oracle import psa_oracle as O


def _head_ranking(w: W.Workload, inp: W.Inputs, b: int, h: int):
    grp = w.Hq // w.Hkv
    Q = inp.as_f64("q", b, h)
    K = inp.as_f64("k", b, h // grp)
    K3, c3 = O.pool_tokens(K, O.POOL[-1])
    pyr = O.Pyramid({len(O.POOL) - 1: K3}, {}, {len(O.POOL) - 1: c3}, w.N)
    z = O.block_logits(O.query_block_means(Q, w.q_blk), pyr, w.kv_blk, 1.0 / math.sqrt(w.d))
    rows = []
    for a in range(w.Nq):
        vis = np.array([j for j in range(w.Nk)
                        if O.visible(a, j, w.N, w.q_blk, w.kv_blk, w.causal)])
        order, _, c = O.rank_blocks(z[a], vis)
        rows.append((order, c))
    return rows


def executed_fraction(w: W.Workload, rankings, alpha: float) -> float:
    tau = [alpha * t / W.TAU_SHAPE[-1] for t in W.TAU_SHAPE]
    total = 0.0
    for rows in rankings:
        lm = np.full((w.Nq, w.Nk), O.PRUNED, dtype=np.int8)
        for a, (order, c) in enumerate(rows):
            lm[a, order] = O.level_of(c, tau)
            O.apply_overrides(lm[a], a, w.N, w.q_blk, w.kv_blk, w.causal,
                              w.forced_prefix_tokens)
        total += O.executed_flops(lm, w.N, w.d, w.q_blk, w.kv_blk, w.causal)
    return total / w.dense_flops()


def tune(w: W.Workload, iters: int = 40):
    kind, val = w.target.split(":")
    goal = 1.0 - float(val) if kind == "skip" else float(val)
    t0 = time.time()
    inp = W.make_inputs(w, heads_kv=None)
    rankings = [_head_ranking(w, inp, b, h) for b in range(w.B) for h in range(w.Hq)]
    lo, hi = 0.0, 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if executed_fraction(w, rankings, mid) < goal:
            lo = mid
        else:
            hi = mid
    alpha = lo
    frac = executed_fraction(w, rankings, alpha)
    return {"alpha": alpha, "executed_fraction": frac, "target": w.target,
            "tau": [alpha * t / W.TAU_SHAPE[-1] for t in W.TAU_SHAPE],
            "seconds": round(time.time() - t0, 1)}


def main(names):
    try:
        with open(W.THRESHOLDS_FILE) as f:
            table = json.load(f)
    except FileNotFoundError:
        table = {}
    for w in W.WORKLOADS:
        if w.target == "fixed" or (names and w.name not in names):
            continue
        table[w.name] = tune(w)
        print(w.name, table[w.name], flush=True)
        with open(W.THRESHOLDS_FILE, "w") as f:
            json.dump(table, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:])
