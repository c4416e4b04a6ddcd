"""Pins for the CPU oracle: facts the method and the mathematics fix, checked
without re-typing the oracle's own formulas.

Each ``pin_*`` takes the oracle module as its argument so that the mutation
tests can run the same pins against deliberately broken copies of the oracle
and check that some pin fails.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
from scipy.special import logsumexp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    """Dense softmax attention from torch (float64, CPU): a library routine."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    am = None if mask is None else t(mask)
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=am, is_causal=causal, scale=scale)
    return out[0, 0].numpy()


# ------------------------------------------------------------------ pyramid

def pin_pool_closed_form(O):
    """K[t, c] = t + 1000 c: a full group of level l averages an arithmetic run,
    mean g*f + (f-1)/2; the ragged tail group averages [g*f, N): (g*f + N - 1)/2."""
    N, d = 1003, 3
    K = np.arange(N, dtype=np.float64)[:, None] + 1000.0 * np.arange(d)[None, :]
    pyr = O.build_pyramid(K, -K)
    for l, f in enumerate((1, 2, 4, 8)):
        G = -(-N // f)
        assert pyr.keys[l].shape == (G, d), (l, pyr.keys[l].shape)
        for g in range(G):
            lo, hi = g * f, min((g + 1) * f, N)
            want = (lo + hi - 1) / 2.0 + 1000.0 * np.arange(d)
            assert np.array_equal(pyr.keys[l][g], want), (l, g)
            assert np.array_equal(pyr.values[l][g], -want), (l, g)
            assert pyr.counts[l][g] == hi - lo, (l, g)


def pin_progressive_equals_direct(O):
    """The article builds the pyramid by progressive pooling; pooling level l-1
    in pairs, weighted by counts, must give level l."""
    rng = np.random.default_rng(11)
    N, d = 203, 5
    K, V = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    pyr = O.build_pyramid(K, V)
    for l in range(1, 4):
        prev, cprev = pyr.keys[l - 1], pyr.counts[l - 1]
        G = pyr.keys[l].shape[0]
        for g in range(G):
            idx = [i for i in (2 * g, 2 * g + 1) if i < prev.shape[0]]
            w = cprev[idx].astype(np.float64)
            prog = (prev[idx] * w[:, None]).sum(0) / w.sum()
            assert np.allclose(prog, pyr.keys[l][g], rtol=0, atol=1e-13), (l, g)
            assert pyr.counts[l][g] == w.sum()


def pin_query_means_closed_form(O):
    """Q[t] = t: the mean of query block a is the midpoint of its valid rows."""
    N, bq = 300, 128
    Q = np.repeat(np.arange(N, dtype=np.float64)[:, None], 2, axis=1)
    qb = O.query_block_means(Q, bq)
    assert qb.shape == (3, 2)
    for a in range(3):
        lo, hi = a * bq, min((a + 1) * bq, N)
        assert np.all(qb[a] == (lo + hi - 1) / 2.0)


# ------------------------------------------------------------ block scoring

def pin_block_logits_uniform_blocks(O):
    """A KV block whose tokens are all equal to k_j: the block logit is the
    logsumexp of the block's own token logits, s*qbar.k_j + ln(#tokens), which
    scipy computes from the explicit per-token list (ragged tail included)."""
    rng = np.random.default_rng(3)
    N, d, bq, bk = 64 * 5 + 40, 16, 64, 64
    Nk = -(-N // bk)
    kj = rng.standard_normal((Nk, d))
    K = np.concatenate([np.repeat(kj[j:j + 1], min(bk, N - j * bk), 0) for j in range(Nk)])
    Q = rng.standard_normal((N, d))
    s = 0.37
    pyr = O.build_pyramid(K, K)
    qb = np.stack([Q[a * bq:min((a + 1) * bq, N)].mean(0) for a in range(-(-N // bq))])
    z = O.block_logits(qb, pyr, bk, s)
    for a in range(qb.shape[0]):
        for j in range(Nk):
            toks = [s * qb[a] @ K[t] for t in range(j * bk, min((j + 1) * bk, N))]
            assert abs(z[a, j] - logsumexp(toks)) < 1e-12, (a, j)


def pin_block_logits_mass_of_pooled_keys(O):
    """General block: exp(z) is the total weight the block's level-3 keys carry,
    sum_g c_g exp(s*qbar.K3_g), each pooled key standing for c_g tokens."""
    rng = np.random.default_rng(4)
    N, d, bk = 64 * 3 + 24, 8, 64
    K = rng.standard_normal((N, d))
    qb = rng.standard_normal((2, d))
    s = 0.5
    z = O.block_logits(qb, O.build_pyramid(K, K), bk, s)
    for j in range(-(-N // bk)):
        for a in range(2):
            tot = 0.0
            for g in range(j * 8, min((j + 1) * 8, -(-N // 8))):
                lo, hi = g * 8, min(g * 8 + 8, N)
                k3 = K[lo:hi].sum(0) / (hi - lo)
                tot += (hi - lo) * math.exp(s * float(qb[a] @ k3))
            assert abs(z[a, j] - math.log(tot)) < 1e-12


# ------------------------------------------------------------- assignment

def pin_assign_handmade(O):
    """Hand-worked level assignments (tests/golden/assign_levels_handmade.json)."""
    with open(os.path.join(GOLDEN, "assign_levels_handmade.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        P = np.array(c["P"], dtype=np.float64)
        z = np.log(P)[None, :]
        r = O.assign_levels(z, c["tau"], N=64 * len(P), bq=64, bk=64)
        assert r.level_map[0].tolist() == c["levels"], (c["name"], r.level_map[0].tolist())
        assert np.allclose(r.mass[0], P / P.sum(), atol=1e-15)


def pin_assign_permutation(O):
    """Shuffling the KV blocks shuffles the map the same way (no position bias
    beyond the tie rule)."""
    rng = np.random.default_rng(5)
    z = rng.standard_normal((3, 40)) * 2.0
    tau = (0.5, 0.7, 0.85, 0.95)
    base = O.assign_levels(z, tau, N=64 * 40, bq=64, bk=64).level_map
    perm = rng.permutation(40)
    shuf = O.assign_levels(z[:, perm], tau, N=64 * 40, bq=64, bk=64).level_map
    assert np.array_equal(shuf, base[:, perm])


def pin_assign_coverage(O):
    """Blocks at level <= l hold at least tau_l of the row's mass, and dropping
    the smallest of them would fall below tau_l (the cut is the shortest one)."""
    rng = np.random.default_rng(6)
    z = rng.standard_normal((4, 50)) * 1.5
    tau = (0.5, 0.7, 0.85, 0.95)
    r = O.assign_levels(z, tau, N=64 * 50, bq=64, bk=64)
    for a in range(4):
        for l, t in enumerate(tau):
            sel = (r.level_map[a] >= 0) & (r.level_map[a] <= l)
            m = r.mass[a][sel].sum()
            assert m >= t - 1e-12
            assert m - r.mass[a][sel].min() < t + 1e-12


def pin_causal_overrides(O):
    """Causal, N=512, 128-row query blocks, 64-token KV blocks: query block 1
    (rows 128..255) sees KV blocks 0..3, blocks 2 and 3 straddle its diagonal
    (level 0), blocks 4..7 are in its future (pruned).  Forced prefix: blocks
    holding any of the first 70 tokens (0 and 1) get level 0."""
    z = np.zeros((4, 8))
    z[:, 0] = 5.0
    r = O.assign_levels(z, (0.1, 0.2, 0.3, 0.4), N=512, bq=128, bk=64, causal=True)
    row = r.level_map[1].tolist()
    assert row[2] == 0 and row[3] == 0 and row[4:] == [-1] * 4, row
    assert row[0] == 0
    assert r.level_map[0].tolist()[2:] == [-1] * 6
    r2 = O.assign_levels(np.zeros((2, 8)) + np.arange(8)[None, :], (0.1, 0.2, 0.3, 0.4),
                         N=512, bq=256, bk=64, forced_prefix_tokens=70)
    assert r2.level_map[:, 0].tolist() == [0, 0] and r2.level_map[:, 1].tolist() == [0, 0]


def pin_assign_quantile_handmade(O):
    """Hand-worked quantile-rule assignments
    (tests/golden/assign_levels_quantile_handmade.json)."""
    with open(os.path.join(GOLDEN, "assign_levels_quantile_handmade.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        P = np.array(c["P"], dtype=np.float64)
        z = np.log(P)[None, :]
        r = O.assign_levels(z, c["tau"], N=64 * len(P), bq=64, bk=64, rule="quantile")
        assert r.level_map[0].tolist() == c["levels"], (c["name"], r.level_map[0].tolist())


def pin_assign_quantile_counts(O):
    """Quantile rule, non-causal rows with no overrides: level l holds exactly
    ceil(t_l n) - ceil(t_(l-1) n) blocks (t = the float32 tau, worked here in
    exact rational arithmetic), and they are the next-heaviest blocks."""
    from fractions import Fraction
    rng = np.random.default_rng(7)
    n = 37
    z = rng.standard_normal((5, n)) * 2.0
    tau = (0.1, 0.3, 0.55, 0.8)
    r = O.assign_levels(z, tau, N=64 * n, bq=64, bk=64, rule="quantile")
    K = [math.ceil(Fraction(float(np.float32(t))) * n) for t in tau]
    for a in range(5):
        row = r.level_map[a]
        prev = 0
        for l in range(4):
            assert int((row == l).sum()) == K[l] - prev
            prev = K[l]
        assert int((row == -1).sum()) == n - K[3]
        # heavier blocks never get a higher level than lighter ones
        order = np.argsort(-z[a], kind="stable")
        lv = np.where(row[order] < 0, 4, row[order])
        assert np.all(np.diff(lv) >= 0)


def pin_assign_quantile_permutation_and_causal(O):
    """Quantile rule: shuffling the KV blocks shuffles the map the same way;
    causal rows take their quotas of their own visible blocks."""
    rng = np.random.default_rng(8)
    z = rng.standard_normal((3, 40)) * 2.0
    tau = (0.25, 0.5, 0.75, 0.875)
    base = O.assign_levels(z, tau, N=64 * 40, bq=64, bk=64, rule="quantile").level_map
    perm = rng.permutation(40)
    shuf = O.assign_levels(z[:, perm], tau, N=64 * 40, bq=64, bk=64, rule="quantile").level_map
    assert np.array_equal(shuf, base[:, perm])
    # causal, N = 1024, 128-row query blocks: query block 3 sees KV blocks 0..7
    zc = rng.standard_normal((8, 16))
    rc = O.assign_levels(zc, tau, N=1024, bq=128, bk=64, causal=True, rule="quantile")
    row = rc.level_map[3]
    assert np.all(row[8:] == -1)
    # blocks 6, 7 straddle the diagonal (level 0); the rest follow quotas of 8
    assert row[6] == 0 and row[7] == 0
    vis_rank = np.argsort(-zc[3, :8], kind="stable")
    K = [2, 4, 6, 7]                                   # ceil(8 * tau)
    for rnk, j in enumerate(vis_rank):
        if j in (6, 7):
            continue
        want = next((l for l in range(4) if rnk < K[l]), -1)
        assert row[j] == want, (j, rnk, row[j], want)


def pin_assign_quantile_listing(O):
    """The level-assignment sketch of "Psa Pyramid Sparse Attention"
    (skillmd.com, Implementation), worked by hand in
    tests/golden/assign_levels_quantile_listing.json: with the stated tau the
    quantile rule gives the sketch's counts (int(n * keep_ratio) blocks at
    level 0, the rest in thirds, nothing pruned) with the remainder cut in rank
    order, not in the sketch's index order; decimal tau whose float32 values
    lie above K_l / n take one block more; and a quota below one block still
    keeps the top block at level 0."""
    with open(os.path.join(GOLDEN, "assign_levels_quantile_listing.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        P = np.array(c["P"], dtype=np.float64)
        z = np.log(P)[None, :]
        r = O.assign_levels(z, c["tau"], N=64 * len(P), bq=64, bk=64, rule="quantile")
        got = r.level_map[0].tolist()
        assert got == c["levels"], (c["name"], got)
        if "index_order_levels" in c:
            n, k0 = c["n"], int(c["n"] * c["keep_ratio"])
            rest = n - k0
            want = [k0, rest // 3, 2 * rest // 3 - rest // 3, rest - 2 * rest // 3, 0]
            have = [got.count(l) for l in (0, 1, 2, 3, -1)]
            assert have == want, (c["name"], have, want)
            assert got != c["index_order_levels"]


# --------------------------------------------------------------- attention

def _rand_head(seed, N, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, d)), rng.standard_normal((N, d)),
            rng.standard_normal((N, d)))


def pin_attention_level0_is_dense(O):
    """An all-level-0 map is dense softmax attention (torch SDPA), ragged N;
    causal with every visible block at level 0 is causal SDPA.  LSE matches the
    logsumexp of the dense logits."""
    N, d, bq, bk = 200, 16, 64, 64
    Q, K, V = _rand_head(1, N, d)
    pyr = O.build_pyramid(K, V)
    s = 1 / math.sqrt(d)
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = np.zeros((Nq, Nk), dtype=np.int8)
    out, lse = O.pyramid_attention(Q, pyr, lm, bq, bk, s)
    assert np.allclose(out, _sdpa(Q, K, V), atol=1e-12)
    assert np.allclose(lse, logsumexp(s * Q @ K.T, axis=1), atol=1e-12)
    lmc = np.array([[0 if j * bk <= min((a + 1) * bq, N) - 1 else -1 for j in range(Nk)]
                    for a in range(Nq)], dtype=np.int8)
    outc, _ = O.pyramid_attention(Q, pyr, lmc, bq, bk, s, causal=True)
    assert np.allclose(outc, _sdpa(Q, K, V, causal=True), atol=1e-12)


def pin_attention_binary_is_block_sparse(O):
    """A {0, -1} map is binary block-sparse attention: SDPA with -inf on the
    dropped blocks."""
    N, d, bq, bk = 256 + 40, 8, 64, 64
    Q, K, V = _rand_head(2, N, d)
    rng = np.random.default_rng(7)
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = np.where(rng.random((Nq, Nk)) < 0.5, 0, -1).astype(np.int8)
    lm[:, 0] = 0
    out, _ = O.pyramid_attention(Q, O.build_pyramid(K, V), lm, bq, bk, 1 / math.sqrt(d))
    mask = np.zeros((N, N))
    for a in range(Nq):
        for j in range(Nk):
            if lm[a, j] < 0:
                mask[a * bq:(a + 1) * bq, j * bk:(j + 1) * bk] = -np.inf
    assert np.allclose(out, _sdpa(Q, K, V, mask=mask), atol=1e-12)


def pin_attention_pooled_is_repeated(O):
    """A block at level l behaves as its pooled keys/values each repeated c_g
    times (the closed form of the ln c_g logit offset): SDPA over the expanded
    key list of each query block, ragged tails included."""
    N, d, bq, bk = 64 * 4 + 24, 8, 64, 64
    Q, K, V = _rand_head(3, N, d)
    pyr = O.build_pyramid(K, V)
    rng = np.random.default_rng(8)
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = rng.integers(-1, 4, size=(Nq, Nk)).astype(np.int8)
    lm[:, 1] = 3
    s = 1 / math.sqrt(d)
    out, lse = O.pyramid_attention(Q, pyr, lm, bq, bk, s)
    for a in range(Nq):
        ks, vs = [], []
        for j in range(Nk):
            l = int(lm[a, j])
            if l < 0:
                continue
            f = 1 << l
            for g in range(j * bk // f, min((j + 1) * bk // f, -(-N // f))):
                lo, hi = g * f, min(g * f + f, N)
                ks += [K[lo:hi].mean(0)] * (hi - lo)
                vs += [V[lo:hi].mean(0)] * (hi - lo)
        rows = slice(a * bq, min((a + 1) * bq, N))
        ref = _sdpa(Q[rows], np.array(ks), np.array(vs), scale=s)
        assert np.allclose(out[rows], ref, atol=1e-12), a
        ref_lse = logsumexp(s * Q[rows] @ np.array(ks).T, axis=1)
        assert np.allclose(lse[rows], ref_lse, atol=1e-12), a


def pin_attention_identical_tokens(O):
    """If the 8 tokens of every level-3 group are identical, pooling loses
    nothing: any map without pruned blocks equals dense attention."""
    N, d, bq, bk = 64 * 3 + 16, 8, 64, 64
    rng = np.random.default_rng(9)
    G = -(-N // 8)
    K = np.repeat(rng.standard_normal((G, d)), 8, 0)[:N]
    V = np.repeat(rng.standard_normal((G, d)), 8, 0)[:N]
    Q = rng.standard_normal((N, d))
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = rng.integers(0, 4, size=(Nq, Nk)).astype(np.int8)
    out, _ = O.pyramid_attention(Q, O.build_pyramid(K, V), lm, bq, bk, 1 / math.sqrt(d))
    assert np.allclose(out, _sdpa(Q, K, V), atol=1e-12)


def pin_attention_constant_v_and_empty_rows(O):
    """V constant: every row with a kept key outputs that constant.  A query
    block with every KV block pruned gets O = 0 and LSE = -inf."""
    N, d, bq, bk = 192, 8, 64, 64
    Q, K, _ = _rand_head(4, N, d)
    V = np.tile(np.linspace(-1, 2, d), (N, 1))
    lm = np.array([[0, 3, -1], [-1, -1, -1], [2, 1, 0]], dtype=np.int8)
    out, lse = O.pyramid_attention(Q, O.build_pyramid(K, V), lm, bq, bk, 0.3)
    assert np.allclose(out[:64], V[:64], atol=1e-13)
    assert np.allclose(out[128:], V[128:], atol=1e-13)
    assert np.all(out[64:128] == 0) and np.all(np.isneginf(lse[64:128]))


def pin_attention_scale_shift(O):
    """Adding a constant to every logit of a row changes nothing: every key (and
    so every pooled key) has last coordinate 1, so raising q's last coordinate
    adds the same amount to all of the row's logits."""
    N, d, bq, bk = 128, 8, 64, 64
    Q, K, V = _rand_head(5, N, d)
    K[:, -1] = 1.0
    lm = np.array([[0, 2], [1, 3]], dtype=np.int8)
    pyr = O.build_pyramid(K, V)
    out, _ = O.pyramid_attention(Q, pyr, lm, bq, bk, 0.4)
    Q2 = Q.copy()
    Q2[:, -1] += 3.0
    out2, _ = O.pyramid_attention(Q2, pyr, lm, bq, bk, 0.4)
    assert np.allclose(out, out2, atol=1e-13)


def pin_attention_causal_never_reads_the_future(O):
    """Causal attention on a caller's map that breaks the contract (future
    blocks and diagonal blocks at pooled levels, values outside -1..3): row i
    must not depend on any token after i.  Changing K and V after token t0
    (inside a diagonal block) leaves rows <= t0 exactly as they were, for
    every t0 tried; and a value outside -1..3 acts as a pruned block (SDPA
    with that block masked, the other blocks at level 0)."""
    N, d, bq, bk = 64 * 6 + 24, 8, 128, 64
    Q, K, V = _rand_head(31, N, d)
    rng = np.random.default_rng(32)
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = rng.integers(-1, 4, size=(Nq, Nk)).astype(np.int8)
    lm[:, -1] = 2                                    # the future of every row but the last
    lm[1, 2:4] = 3                                   # diagonal blocks of query block 1 pooled
    lm[2, 4] = 7                                     # out of range
    pyr = O.build_pyramid(K, V)
    s = 1 / math.sqrt(d)
    out, _ = O.pyramid_attention(Q, pyr, lm, bq, bk, s, causal=True)
    for t0 in (140, 200, 255, 300, 333):
        K2, V2 = K.copy(), V.copy()
        K2[t0 + 1:] = rng.standard_normal((N - t0 - 1, d)) * 5.0
        V2[t0 + 1:] = rng.standard_normal((N - t0 - 1, d)) * 5.0
        out2, _ = O.pyramid_attention(Q, O.build_pyramid(K2, V2), lm, bq, bk, s, causal=True)
        assert np.allclose(out2[:t0 + 1], out[:t0 + 1], atol=1e-12, rtol=0), t0
    # out-of-range values are pruned blocks
    lmb = np.zeros((Nq, Nk), dtype=np.int8)
    lmb[0, 1], lmb[2, 3], lmb[3, 0] = 7, -5, 100
    outb, _ = O.pyramid_attention(Q, pyr, lmb, bq, bk, s)
    mask = np.zeros((N, N))
    for a, j in ((0, 1), (2, 3), (3, 0)):
        mask[a * bq:(a + 1) * bq, j * bk:(j + 1) * bk] = -np.inf
    assert np.allclose(outb, _sdpa(Q, K, V, mask=mask), atol=1e-12)


# --------------------------------------------- cosine-similarity constraint

def _rot(x, ang):
    c, s_ = math.cos(ang), math.sin(ang)
    return np.array([c * x[0] - s_ * x[1], s_ * x[0] + c * x[1]])


def pin_similarity_closed_form_angles(O):
    """Every 8-token group: tokens (u, u, v, v, R u, R u, R v, R v) with
    angle(u, v) = 60 degrees and R a 30-degree rotation.  Level-1 merges join
    equal tokens (cos 1), level-2 merges join u and v (cos 1/2), level-3 merges
    join mean(u, v) and its rotation (cos 30 degrees)."""
    u = np.array([1.0, 0.0])
    v = _rot(u, math.pi / 3)
    grp = [u, u, v, v, _rot(u, math.pi / 6), _rot(u, math.pi / 6), _rot(v, math.pi / 6),
           _rot(v, math.pi / 6)]
    K = np.array(grp * 16)                               # N = 128: two blocks of 64
    ml, mc = O.block_max_levels(K, 64, 0.6)
    assert np.allclose(mc[:, 1], 1.0) and np.allclose(mc[:, 2], 0.5)
    assert np.allclose(mc[:, 3], math.cos(math.pi / 6))
    assert list(ml) == [1, 1]                            # level 2 fails at 0.6, so level 3 is out
    assert list(O.block_max_levels(K, 64, 0.4)[0]) == [3, 3]
    assert list(O.block_max_levels(K, 64, 0.9)[0]) == [1, 1]
    assert list(O.block_max_levels(K, 64, 1.0 + 1e-9)[0]) == [0, 0]


def pin_similarity_orthogonal_opposite_ragged_zero(O):
    """Exact cosines 0 and -1, an absent second half at the ragged end, and a
    zero-mean half (which always passes)."""
    e1, e2 = np.array([1.0, 0.0]), np.array([0.0, 1.0])
    K = np.tile(e1, (64 + 3, 1))
    K[1] = e2                                            # block 0: one orthogonal token pair
    assert O.block_max_levels(K, 64, 0.0)[0][0] >= 1     # cos 0 >= 0 passes
    assert O.block_max_levels(K, 64, 1e-6)[0][0] == 0
    K = np.tile(e1, (64 + 3, 1))
    K[66] = -e1                                          # block 1 = tokens 64, 65, 66
    ml, mc = O.block_max_levels(K, 64, -0.5)
    assert mc[1, 1] == 1.0                               # (64, 65); 66 has no partner
    assert mc[1, 2] == -1.0                              # (64, 65) against (66)
    assert np.isinf(mc[1, 3])                            # tokens 68.. do not exist
    assert ml[1] == 1 and ml[0] == 3
    K = np.tile(e1, (64, 1))
    K[0] = 0.0                                           # zero-mean half: the merge passes
    assert O.block_max_levels(K, 64, 0.99)[0][0] == 3


def pin_similarity_scale_invariance(O):
    """Cosines do not change when every key is scaled by a positive constant,
    and every min cosine lies in [-1, 1]."""
    rng = np.random.default_rng(17)
    K = rng.standard_normal((200, 8)) + 2.0
    a, ca = O.block_max_levels(K, 64, 0.8)
    b, cb = O.block_max_levels(3.7 * K, 64, 0.8)
    assert np.array_equal(a, b) and np.allclose(ca, cb)
    fin = np.isfinite(ca[:, 1:])
    assert np.all(np.abs(ca[:, 1:][fin]) <= 1 + 1e-12)


def pin_similarity_clamps_assignment(O):
    """The constraint only lowers kept levels (to min(level, max level)) and
    never touches pruned blocks; theta = -1 changes nothing, and a theta no
    random merge reaches leaves every kept block at level 0."""
    rng = np.random.default_rng(19)
    N, d, bq, bk = 64 * 9 + 5, 8, 64, 64
    Q, K, V = rng.standard_normal((N, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    tau = (0.3, 0.5, 0.7, 0.9)
    free = O.psa_head(Q, K, V, bq, bk, tau).mask.level_map
    ml = rng.integers(0, 4, size=free.shape[1])
    z = O.block_logits(O.query_block_means(Q, bq), O.build_pyramid(K, V), bk, 1 / math.sqrt(d))
    got = O.assign_levels(z, tau, N, bq, bk, max_level=ml).level_map
    want = np.where(free >= 0, np.minimum(free, ml[None, :]), -1)
    assert np.array_equal(got, want)
    assert np.array_equal(O.psa_head(Q, K, V, bq, bk, tau, sim_threshold=-1.0).mask.level_map, free)
    one = O.psa_head(Q, K, V, bq, bk, tau, sim_threshold=1.0).mask.level_map
    assert np.array_equal(one, np.where(free >= 0, 0, -1))


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
