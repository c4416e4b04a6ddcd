"""Scalar brute force of the whole PSA forward for tiny inputs: plain Python
loops and the math module only, written separately from the oracle (no numpy
vectorisation, no shared helpers), so that the two can be compared.

Steps: pool each level group by group; mean of each query block; block logit =
log of sum over the block's level-3 keys of c_g * exp(s * qbar . k_g); softmax
over visible blocks; rank by (-P, j); exclusive running mass; threshold cut;
causal / forced overrides; per-row softmax over the kept keys with ln c_g."""
import math
import struct
from fractions import Fraction


def _mean(rows):
    n = len(rows)
    return [sum(r[c] for r in rows) / n for c in range(len(rows[0]))]


def _dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def psa_bruteforce(Q, K, V, bq, bk, tau, causal=False, forced=0, scale=None, rule="threshold"):
    N, d = len(Q), len(Q[0])
    s = 1.0 / math.sqrt(d) if scale is None else scale
    pools = (1, 2, 4, 8)
    lev = []
    for f in pools:
        ks, vs, cs = [], [], []
        g = 0
        while g * f < N:
            lo, hi = g * f, min(g * f + f, N)
            ks.append(_mean(K[lo:hi]))
            vs.append(_mean(V[lo:hi]))
            cs.append(hi - lo)
            g += 1
        lev.append((ks, vs, cs))
    Nq = (N + bq - 1) // bq
    Nk = (N + bk - 1) // bk
    levels = [[-1] * Nk for _ in range(Nq)]
    for a in range(Nq):
        q_lo, q_hi = a * bq, min(a * bq + bq, N)
        qbar = _mean(Q[q_lo:q_hi])
        vis = [j for j in range(Nk) if (not causal) or j * bk <= q_hi - 1]
        z = {}
        k3, _, c3 = lev[3]
        for j in vis:
            tot = 0.0
            for g in range(j * bk // 8, min((j + 1) * bk // 8, len(k3))):
                tot += c3[g] * math.exp(s * _dot(qbar, k3[g]))
            z[j] = math.log(tot)
        zmax = max(z.values())
        w = {j: math.exp(z[j] - zmax) for j in vis}
        tw = sum(w.values())
        P = {j: w[j] / tw for j in vis}
        ranked = sorted(vis, key=lambda j: (-P[j], j))
        c = 0.0
        # quantile rule: quota of the l-th level = ceil(tau_l * visible blocks),
        # with tau_l at the float32 value the C interface carries, in exact
        # rational arithmetic
        quota = [math.ceil(Fraction(struct.unpack("f", struct.pack("f", t))[0]) * len(vis))
                 for t in tau]
        for r, j in enumerate(ranked):
            lv = -1
            for l in range(4):
                if (r < quota[l]) if rule == "quantile" else (c < tau[l]):
                    lv = l
                    break
            levels[a][j] = lv
            c += P[j]
        for j in range(Nk):
            if j not in vis:
                levels[a][j] = -1
            elif causal and min(j * bk + bk, N) - 1 >= q_lo:
                levels[a][j] = 0
            elif j * bk < forced:
                levels[a][j] = 0
    O = [[0.0] * d for _ in range(N)]
    lse = [-math.inf] * N
    for a in range(Nq):
        for i in range(a * bq, min(a * bq + bq, N)):
            logits, vals = [], []
            for j in range(Nk):
                l = levels[a][j]
                if l < 0:
                    continue
                ks, vs, cs = lev[l]
                f = pools[l]
                for g in range(j * bk // f, min((j + 1) * bk // f, len(ks))):
                    if l == 0 and causal and g > i:
                        continue
                    logits.append(s * _dot(Q[i], ks[g]) + math.log(cs[g]))
                    vals.append(vs[g])
            if not logits:
                continue
            m = max(logits)
            ws = [math.exp(x - m) for x in logits]
            tot = sum(ws)
            O[i] = [sum(w * v[c] for w, v in zip(ws, vals)) / tot for c in range(d)]
            lse[i] = m + math.log(tot)
    return O, lse, levels
