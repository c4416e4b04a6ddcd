"""CPU oracle for the Pyramid Sparse Attention (PSA) forward pass, in float64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference legs of ``bench.py`` use it.  It shares no code with the CUDA
path.

Sources (the web pages describing PSA, arXiv:2512.04025):
  [abs]  "PSA: Pyramid Sparse Attention for Efficient Video Understanding and
         Generation" (chatpaper.ai), abstract: each query block gives every KV
         block a pooling level, lower levels to critical blocks, higher levels
         to less important ones, or prunes it; the kernel decouples the logical
         block size from the hardware tile.
  [news] top168.com article on arXiv:2512.04025: the pyramid's bottom level is
         the original KV and every level above is average-pooled and coarser;
         three components (pyramid KV blocks built by progressive pooling, a
         multi-level mask generator driven by query-key block importance, and
         adaptive pyramid attention that keeps the probability distribution
         consistent); threshold-based assignment beats quantile-based.
  [skill] "Psa Pyramid Sparse Attention" (skillmd.com), "Core Technique": levels
         0/1/2/3 are the KV pooled 1x/2x/4x/8x; "Implementation": sketches of the
         pooled cache, block scoring, a quantile-style level assignment (top
         keep-ratio blocks at level 0, the rest in thirds) and the attention.

Where the pages leave a step open, the reading used is stated at the function.
Every function below works on one (batch, head) slice; ``psa_forward`` loops.

Notation: N tokens, d head dim, bq / bk query / KV block size, f_l = 2**l the
pool factor of level l, s = softmax scale (1/sqrt(d) unless given).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

PRUNED = -1
POOL = (1, 2, 4, 8)


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


# --------------------------------------------------------------------- pyramid

def pool_tokens(x: np.ndarray, f: int) -> Tuple[np.ndarray, np.ndarray]:
    """Average-pool tokens by factor f ([news] pyramid paragraph; [skill] Core
    Technique, pooled KV cache).

    Pooled token g is the mean of rows [g*f, min((g+1)*f, N)); the returned
    counts c_g are the number of rows averaged (f except in a ragged tail).
    x: [N, d] float64.  Returns ([ceil(N/f), d], [ceil(N/f)] int)."""
    N, d = x.shape
    G = cdiv(N, f)
    full = N // f
    out = np.empty((G, d), dtype=np.float64)
    counts = np.full(G, f, dtype=np.int64)
    out[:full] = x[:full * f].reshape(full, f, d).mean(axis=1)
    if G > full:                                   # ragged tail group
        out[full] = x[full * f:].mean(axis=0)
        counts[full] = N - full * f
    return out, counts


@dataclass
class Pyramid:
    """Levels l = 0..3 of K and V of one head: keys[l], values[l] are
    [ceil(N/f_l), d]; counts[l] the tokens behind each pooled row."""
    keys: Dict[int, np.ndarray]
    values: Dict[int, np.ndarray]
    counts: Dict[int, np.ndarray]
    N: int


def build_pyramid(K: np.ndarray, V: np.ndarray, pool: Sequence[int] = POOL) -> Pyramid:
    """Pyramid KV construction ([news] component one; [skill] levels 0..3).

    Level 0 is K/V itself; level l pools the original tokens directly by f_l.
    The article says the levels are built progressively; in exact arithmetic,
    pooling level l-1 by 2 with count weights equals pooling level 0 by f_l, so
    the oracle takes the direct form (a test checks the two agree)."""
    N = K.shape[0]
    keys, values, counts = {}, {}, {}
    for l, f in enumerate(pool):
        if f == 1:
            keys[l], values[l] = K.astype(np.float64), V.astype(np.float64)
            counts[l] = np.ones(N, dtype=np.int64)
        else:
            keys[l], counts[l] = pool_tokens(K, f)
            values[l], _ = pool_tokens(V, f)
    return Pyramid(keys, values, counts, N)


def block_rows(j: int, l: int, bk: int, pyr: Pyramid, pool: Sequence[int] = POOL) -> range:
    """Rows of level l that summarise KV block j: [j*bk/f_l, min((j+1)*bk/f_l, rows_l))."""
    f = pool[l]
    per = bk // f
    return range(j * per, min((j + 1) * per, pyr.keys[l].shape[0]))


# ------------------------------------------------------------ mask generation

def query_block_means(Q: np.ndarray, bq: int) -> np.ndarray:
    """q_bar[a] = mean of the valid rows of query block a.  The pages score
    query-key block pairs ([news] component two) without saying how a query
    block is summarised; the mean is the reading used.  Returns [Nq, d]."""
    N = Q.shape[0]
    Nq = cdiv(N, bq)
    return np.stack([Q[a * bq:min((a + 1) * bq, N)].mean(axis=0) for a in range(Nq)])


def block_logits(qbar: np.ndarray, pyr: Pyramid, bk: int, scale: float,
                 pool: Sequence[int] = POOL) -> np.ndarray:
    """Block importance z[a, j] ([news] component two; [skill] block scoring).

    Reading: the query-block mean is scored against the coarsest (level-3)
    pooled keys of block j, and the block's logit is the log of the softmax mass
    those pooled keys stand for: z = logsumexp_g(s * q_bar . K3[g] + ln c_g).
    For a block whose tokens are identical this is exactly the logsumexp of the
    block's own token logits.  Returns [Nq, Nk]."""
    L = len(pool) - 1
    K3, c3 = pyr.keys[L], pyr.counts[L]
    Nq, Nk = qbar.shape[0], cdiv(pyr.N, bk)
    z = np.empty((Nq, Nk), dtype=np.float64)
    logits = scale * (qbar @ K3.T) + np.log(c3)[None, :]
    for j in range(Nk):
        rows = block_rows(j, L, bk, pyr, pool)
        part = logits[:, rows.start:rows.stop]
        m = part.max(axis=1, keepdims=True)
        z[:, j] = m[:, 0] + np.log(np.exp(part - m).sum(axis=1))
    return z


def visible(a: int, j: int, N: int, bq: int, bk: int, causal: bool) -> bool:
    """Causal: KV block j is visible to query block a iff its first token is at
    or before the query block's last row."""
    if not causal:
        return True
    return j * bk <= min((a + 1) * bq, N) - 1


def straddles(a: int, j: int, N: int, bq: int, bk: int) -> bool:
    """Causal: KV block j overlaps the row range of query block a, so a token
    mask (key position <= query position) is needed inside it."""
    q_lo, q_hi = a * bq, min((a + 1) * bq, N) - 1
    k_lo, k_hi = j * bk, min((j + 1) * bk, N) - 1
    return k_lo <= q_hi and k_hi >= q_lo


@dataclass
class MaskResult:
    level_map: np.ndarray    # int8 [Nq, Nk]; -1 = pruned
    mass: np.ndarray         # P[a, j], softmax over visible blocks (0 for invisible)
    cum_before: np.ndarray   # C[a, j]: mass of the blocks ranked before j in row a
    rank: np.ndarray         # rank of j in row a (visible blocks only; -1 otherwise)


def rank_blocks(z_row: np.ndarray, vis: np.ndarray):
    """One query block's softmax over its visible KV blocks, ranked.

    P = softmax(z) over the visible blocks ``vis``; the ranking is P descending
    with ties going to the lower block index; C[r] is the mass of the blocks
    ranked before r (exclusive prefix, summed in rank order).
    Returns (order: block indices by rank, P in rank order, C in rank order)."""
    zz = z_row[vis]
    p = np.exp(zz - zz.max())
    p = p / p.sum()
    idx = np.lexsort((vis, -p))            # primary key -P, then block index
    p_sorted = p[idx]
    c = np.concatenate(([0.0], np.cumsum(p_sorted)[:-1]))
    return vis[idx], p_sorted, c


def level_of(c: np.ndarray, tau: Sequence[float]) -> np.ndarray:
    """level = the smallest l with C < tau_l, else pruned (-1)."""
    out = np.full(c.shape, PRUNED, dtype=np.int8)
    for l in reversed(range(len(tau))):
        out[c < tau[l]] = l
    return out


def quotas(n_visible: int, tau: Sequence[float]) -> np.ndarray:
    """Quantile rule: K_l = ceil(tau_l * n_visible), the number of top-ranked
    blocks at level <= l.  tau is taken at the single precision the C
    interface carries it in, and the product is exact in float64 (a 24-bit
    significand times an integer below 2^14).

    Source: [skill] Implementation, the level-assignment sketch: the top
    int(n * keep_ratio) blocks by score get level 0 and the rest are cut into
    thirds for levels 1..3, nothing pruned.  Readings that depart from it:
      * quotas per level (tau_0..tau_3) instead of one keep ratio and fixed
        thirds; the sketch is the case tau = (K_0, K_0 + r//3, K_0 + 2r//3, n)/n
        with K_0 = int(n * keep_ratio), r = n - K_0;
      * rounded up, not down: a positive tau_0 keeps the top block at level 0,
        as the threshold rule's exclusive mass does (the sketch's int() gives 0
        blocks when n * keep_ratio < 1, and its slice of the last 0 sorted
        indices then selects every block);
      * blocks ranked at or past K_3 are pruned, so that the rule can be
        compared with the threshold rule at equal compute (the ablation of
        [news]); tau_3 = 1 prunes nothing, as the sketch."""
    t = np.asarray(tau, dtype=np.float32).astype(np.float64)
    return np.ceil(t * float(n_visible)).astype(np.int64)


def level_of_rank(rank: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Quantile rule: level = the smallest l with rank < K_l, else pruned (-1).
    The rank is the block's place in the ranking by P (descending, ties to the
    lower index), so the blocks past level 0 are cut in order of importance.
    [skill]'s sketch cuts them in block-index order, which would give level 1
    to the lowest indices whatever their score, against its own Core
    Technique (level 1 = medium importance, level 3 = minimal) and [abs]
    (higher levels for less important blocks); the index order is read as a
    slip of the sketch."""
    out = np.full(rank.shape, PRUNED, dtype=np.int8)
    for l in reversed(range(len(K))):
        out[rank < K[l]] = l
    return out


def block_max_levels(K: np.ndarray, bk: int, theta: float,
                     pool: Sequence[int] = POOL) -> Tuple[np.ndarray, np.ndarray]:
    """Cosine-similarity constraint on the pyramid ([news] ablations name a
    cosine-similarity constraint and its gain; the pages do not define it).

    Reading: every pooled row of level l >= 1 merges two rows of level l - 1,
    the token ranges [2g f', (2g+1) f') and [(2g+1) f', (2g+2) f') with
    f' = f_(l-1), cut at N.  The merge is similar when the cosine of the two
    halves' mean keys is >= theta; a merge whose second half is empty, or one
    of whose halves has a zero mean, passes.  KV block j may be represented at
    level l when every merge at levels 1..l inside it is similar.
    Returns (max_level [Nk] int: the largest such l, or 0; min_cos [Nk, L+1]:
    the smallest cosine among block j's merges at each level, +inf where a
    level has no merge, column 0 unused)."""
    N, _ = K.shape
    L = len(pool) - 1
    Nk = cdiv(N, bk)
    min_cos = np.full((Nk, L + 1), np.inf)
    for j in range(Nk):
        for l in range(1, L + 1):
            half = pool[l - 1]
            for start in range(j * bk, min((j + 1) * bk, N), pool[l]):
                a_lo, a_hi = start, min(start + half, N)
                b_lo, b_hi = a_hi, min(start + pool[l], N)
                if b_hi <= b_lo:
                    continue                       # no second half: nothing merged
                a = K[a_lo:a_hi].mean(axis=0)
                b = K[b_lo:b_hi].mean(axis=0)
                na, nb = np.linalg.norm(a), np.linalg.norm(b)
                c = 1.0 if na == 0 or nb == 0 else float(a @ b) / (na * nb)
                min_cos[j, l] = min(min_cos[j, l], c)
    max_level = np.zeros(Nk, dtype=np.int64)
    for j in range(Nk):
        for l in range(1, L + 1):
            if min_cos[j, l] >= theta:
                max_level[j] = l
            else:
                break
    return max_level, min_cos


def apply_overrides(row: np.ndarray, a: int, N: int, bq: int, bk: int, causal: bool,
                    forced_prefix_tokens: int) -> None:
    """In place: causal blocks after the query block are pruned and blocks
    straddling its diagonal get level 0; visible blocks holding any of the first
    ``forced_prefix_tokens`` tokens get level 0."""
    j = np.arange(row.shape[0])
    q_lo, q_hi = a * bq, min((a + 1) * bq, N) - 1
    vis = (j * bk <= q_hi) if causal else np.ones(row.shape[0], dtype=bool)
    strad = vis & (np.minimum((j + 1) * bk, N) - 1 >= q_lo) if causal else ~vis
    forced = vis & (j * bk < forced_prefix_tokens)
    row[~vis] = PRUNED
    row[strad | forced] = 0


def assign_levels(z: np.ndarray, tau: Sequence[float], N: int, bq: int, bk: int,
                  causal: bool = False, forced_prefix_tokens: int = 0,
                  rule: str = "threshold",
                  max_level: Optional[np.ndarray] = None) -> MaskResult:
    """Multi-level mask ([news] ablations: threshold-based assignment, compared
    there with a quantile-based one; [abs] lower levels to critical blocks,
    higher to less important).

    For each query block a: P = softmax over visible j of z[a, j]; rank blocks by
    P descending, ties to the lower j; C_r = mass of the blocks ranked before r.
    Threshold rule: level = the smallest l with C_r < tau_l, else pruned.
    Quantile rule: level = the smallest l with r < K_l = ceil(tau_l * n_visible)
    (``quotas``), else pruned.  Then the overrides of ``apply_overrides``.
    With ``max_level`` (``block_max_levels``), every kept level is then
    lowered to at most its block's max_level (finer, never coarser; pruned
    blocks stay pruned).
    Readings where the pages leave the step open: the exclusive cumulative
    mass (so the top block always gets level 0), the quotas as cumulative
    fractions of the visible blocks rounded up, and the override order."""
    if rule not in ("threshold", "quantile"):
        raise ValueError(rule)
    Nq, Nk = z.shape
    level_map = np.full((Nq, Nk), PRUNED, dtype=np.int8)
    mass = np.zeros((Nq, Nk), dtype=np.float64)
    cum = np.zeros((Nq, Nk), dtype=np.float64)
    rank = np.full((Nq, Nk), -1, dtype=np.int64)
    for a in range(Nq):
        vis = np.array([j for j in range(Nk) if visible(a, j, N, bq, bk, causal)])
        order, p, c = rank_blocks(z[a], vis)
        mass[a, order], cum[a, order] = p, c
        rank[a, order] = np.arange(len(order))
        if rule == "threshold":
            level_map[a, order] = level_of(c, tau)
        else:
            level_map[a, order] = level_of_rank(np.arange(len(order)), quotas(len(order), tau))
        apply_overrides(level_map[a], a, N, bq, bk, causal, forced_prefix_tokens)
        if max_level is not None:
            kept = level_map[a] >= 0
            level_map[a, kept] = np.minimum(level_map[a, kept], max_level[kept])
    return MaskResult(level_map, mass, cum, rank)


# ----------------------------------------------------------------- attention

def correct_map(level_map: np.ndarray, N: int, bq: int, bk: int,
                causal: bool) -> Tuple[np.ndarray, int]:
    """A level map as the attention uses it, and how many entries were changed.

    A map handed in by a caller may break the method's contract; the attention
    never reads future tokens and never reads an undefined level:
      * a value outside -1..3 is treated as pruned;
      * causal: a block after the query block's last row is pruned, and a kept
        block that straddles its diagonal is attended at level 0 with the
        token mask (a pooled key there would average future tokens; reading:
        [news] causal and bidirectional paragraph says PSA serves causal
        generation, and the assignment's own causal overrides do the same).
    Maps made by ``assign_levels`` already satisfy this and pass unchanged."""
    lm = np.array(level_map, dtype=np.int64)
    out = np.where((lm >= -1) & (lm <= 3), lm, PRUNED)
    if causal:
        Nq, Nk = out.shape
        for a in range(Nq):
            for j in range(Nk):
                if not visible(a, j, N, bq, bk, True):
                    out[a, j] = PRUNED
                elif out[a, j] > 0 and straddles(a, j, N, bq, bk):
                    out[a, j] = 0
    return out.astype(np.int8), int((out != lm).sum())


def pyramid_attention(Q: np.ndarray, pyr: Pyramid, level_map: np.ndarray, bq: int, bk: int,
                      scale: float, causal: bool = False,
                      pool: Sequence[int] = POOL) -> Tuple[np.ndarray, np.ndarray]:
    """Adaptive pyramid attention ([news] component three, keeping the
    probability distribution consistent).

    Row i of query block a takes ONE softmax over every key it keeps: for each
    block j with level l = map[a, j] >= 0, the level-l pooled rows of block j,
    each with logit s * q_i . K_l[g] + ln c_g.  The ln c_g term lets a pooled key
    carry the softmax mass of the c_g tokens it averages: it equals attending to
    the pooled key repeated c_g times.  Causal blocks straddling the diagonal
    (always level 0) also mask keys after row i.  A row that keeps no key gets
    O = 0 and LSE = -inf.  The map is first put through ``correct_map`` (values
    outside -1..3 pruned; causally, no future block and no pooled diagonal
    block).  Returns (O [N, d], LSE [N], natural log)."""
    N, d = Q.shape
    level_map, _ = correct_map(level_map, N, bq, bk, causal)
    Nq, Nk = level_map.shape
    O = np.zeros((N, d), dtype=np.float64)
    lse = np.full(N, -np.inf, dtype=np.float64)
    for a in range(Nq):
        ks, vs, bias, kpos = [], [], [], []
        for j in range(Nk):
            l = int(level_map[a, j])
            if l < 0:
                continue
            rows = block_rows(j, l, bk, pyr, pool)
            ks.append(pyr.keys[l][rows.start:rows.stop])
            vs.append(pyr.values[l][rows.start:rows.stop])
            bias.append(np.log(pyr.counts[l][rows.start:rows.stop]))
            # token position of each key; pooled keys (level > 0) never straddle.
            kpos.append(np.arange(rows.start, rows.stop) * pool[l] if l == 0
                        else np.full(len(rows), -1))
        if not ks:
            continue
        Kk, Vk = np.concatenate(ks), np.concatenate(vs)
        bias_a, kpos_a = np.concatenate(bias), np.concatenate(kpos)
        rows_i = np.arange(a * bq, min((a + 1) * bq, N))
        # every row of block a keeps the same keys: one matrix product per block
        logit = scale * (Q[rows_i] @ Kk.T) + bias_a[None, :]
        if causal:
            logit = np.where(kpos_a[None, :] > rows_i[:, None], -np.inf, logit)
        m = logit.max(axis=1)
        ok = np.isfinite(m)
        w = np.exp(logit[ok] - m[ok, None])
        ssum = w.sum(axis=1)
        O[rows_i[ok]] = (w @ Vk) / ssum[:, None]
        lse[rows_i[ok]] = m[ok] + np.log(ssum)
    return O, lse


# ------------------------------------------------------------------- driver

@dataclass
class HeadResult:
    O: np.ndarray
    lse: np.ndarray
    mask: MaskResult
    z: np.ndarray


def psa_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray, bq: int, bk: int,
             tau: Sequence[float], causal: bool = False, forced_prefix_tokens: int = 0,
             scale: Optional[float] = None, level_map: Optional[np.ndarray] = None,
             pool: Sequence[int] = POOL, rule: str = "threshold",
             sim_threshold: Optional[float] = None) -> HeadResult:
    """The whole PSA forward for one (batch, query head): pyramid, query-block
    means, block logits, level assignment (unless ``level_map`` is given; with
    the cosine-similarity constraint when ``sim_threshold`` is given), then
    pyramid attention.  Q [N, d]; K, V [N, d] of the matching KV head."""
    N, d = Q.shape
    s = 1.0 / math.sqrt(d) if scale is None else scale
    pyr = build_pyramid(K, V, pool)
    z = block_logits(query_block_means(Q, bq), pyr, bk, s, pool)
    ml = None if sim_threshold is None else block_max_levels(K, bk, sim_threshold, pool)[0]
    mask = assign_levels(z, tau, N, bq, bk, causal, forced_prefix_tokens, rule, ml)
    lm = mask.level_map if level_map is None else level_map
    O, lse = pyramid_attention(Q, pyr, lm, bq, bk, s, causal, pool)
    return HeadResult(O, lse, mask, z)


def executed_flops(level_map: np.ndarray, N: int, d: int, bq: int, bk: int,
                   causal: bool = False, pool: Sequence[int] = POOL) -> float:
    """FLOPs the method executes for one head's map: 4*d per (query row, kept
    key); a causal block straddling the diagonal counts only unmasked pairs."""
    Nq, Nk = level_map.shape
    qrows = np.array([min((a + 1) * bq, N) - a * bq for a in range(Nq)], dtype=np.float64)
    valid = np.array([min((j + 1) * bk, N) - j * bk for j in range(Nk)], dtype=np.int64)
    keys = np.zeros((Nk, len(pool) + 1), dtype=np.float64)   # column -1 <- pruned = 0
    for l, f in enumerate(pool):
        keys[:, l] = -(-valid // f)
    per = keys[np.arange(Nk)[None, :], level_map.astype(np.int64)]   # [Nq, Nk]
    total = float((qrows[:, None] * per).sum())
    if causal:
        for a in range(Nq):
            i = np.arange(a * bq, min((a + 1) * bq, N))
            for j in range(Nk):
                if level_map[a, j] >= 0 and straddles(a, j, N, bq, bk):
                    k_lo, k_hi = j * bk, min((j + 1) * bk, N)
                    exact = np.maximum(0, np.minimum(k_hi, i + 1) - k_lo).sum()
                    total += float(exact) - qrows[a] * per[a, j]
    return 4.0 * d * total


@dataclass
class ForwardResult:
    O: np.ndarray            # [B, Hq, N, d]
    lse: np.ndarray          # [B, Hq, N]
    level_map: np.ndarray    # int8 [B, Hq, Nq, Nk]
    mass: np.ndarray         # [B, Hq, Nq, Nk]
    cum_before: np.ndarray   # [B, Hq, Nq, Nk]


def psa_forward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, bq: int, bk: int,
                tau: Sequence[float], causal: bool = False, forced_prefix_tokens: int = 0,
                scale: Optional[float] = None, level_map: Optional[np.ndarray] = None,
                heads: Optional[Sequence[Tuple[int, int]]] = None) -> ForwardResult:
    """PSA forward over [B, Hq, N, d] queries and [B, Hkv, N, d] keys/values
    (float64).  Query head h reads KV head h // (Hq / Hkv) (grouped queries);
    maps are per query head.  ``heads`` restricts the work to some (b, h) pairs
    (the others stay zero / pruned)."""
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    grp = Hq // Hkv
    Nq, Nk = cdiv(N, bq), cdiv(N, bk)
    O = np.zeros_like(Q, dtype=np.float64)
    lse = np.full((B, Hq, N), -np.inf)
    lm = np.full((B, Hq, Nq, Nk), PRUNED, dtype=np.int8)
    mass = np.zeros((B, Hq, Nq, Nk))
    cum = np.zeros((B, Hq, Nq, Nk))
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        r = psa_head(Q[b, h], K[b, h // grp], V[b, h // grp], bq, bk, tau, causal,
                     forced_prefix_tokens, scale,
                     None if level_map is None else level_map[b, h])
        O[b, h], lse[b, h] = r.O, r.lse
        lm[b, h] = r.mask.level_map if level_map is None else level_map[b, h]
        mass[b, h], cum[b, h] = r.mask.mass, r.mask.cum_before
    return ForwardResult(O, lse, lm, mass, cum)
