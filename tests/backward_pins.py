"""Pins for the backward-pass oracle (``oracle/psa_backward.py``): facts the
mathematics fixes, checked without re-typing the oracle's own formulas.

- Library autograd: torch differentiates its own float64 formulation of the
  forward pass, written differently from the oracle: one masked softmax over
  ALL rows of the pyramid, with the pooling as explicit averaging matrices.
  Dense and block-sparse maps go through torch's scaled_dot_product_attention.
- Finite differences of the forward oracle itself.
- Exact invariants: shifting every value by u shifts every output by u, so
  sum dV = sum dO; shifting every key by u adds a per-row constant to the
  logits, so sum dK = 0; and sum <Q, dQ> = sum <K, dK> (both are
  sum_ig dX_ig * x_ig without the bias).

Each ``pin_*`` takes the backward module as its argument so that the mutation
tests can run the pins against deliberately broken copies.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _t(x, grad=False):
    return torch.tensor(np.ascontiguousarray(x), dtype=torch.float64, requires_grad=grad)


def _pool_matrix(N, f):
    """A[g, t] = 1 / c_g for the tokens t that pooled row g averages."""
    G = -(-N // f)
    A = np.zeros((G, N))
    for g in range(G):
        lo, hi = g * f, min(g * f + f, N)
        A[g, lo:hi] = 1.0 / (hi - lo)
    return A


def torch_pyramid_forward(Q, K, V, lm, bq, bk, s, causal):
    """The forward pass as one masked softmax per row over every row of every
    level: row i keeps pooled row g of level l iff its query block's map entry
    for g's KV block is l (and, causally, g's token is not after i).  Q, K, V
    torch float64 [N, d]; rows that keep nothing get O = 0."""
    N = Q.shape[0]
    keys, vals, bias, keep = [], [], [], []
    qa = np.arange(N) // bq
    for l, f in enumerate((1, 2, 4, 8)):
        A = torch.from_numpy(_pool_matrix(N, f))
        keys.append(A @ K)
        vals.append(A @ V)
        G = A.shape[0]
        c = np.array([min(g * f + f, N) - g * f for g in range(G)], dtype=np.float64)
        bias.append(np.log(c))
        blk = (np.arange(G) * f) // bk
        k = lm[qa[:, None], blk[None, :]] == l
        if causal and l == 0:
            k &= np.arange(G)[None, :] <= np.arange(N)[:, None]
        keep.append(k)
    Kall, Vall = torch.cat(keys), torch.cat(vals)
    b = torch.from_numpy(np.concatenate(bias))
    keep = torch.from_numpy(np.concatenate(keep, axis=1))
    logit = s * (Q @ Kall.T) + b[None, :]
    logit = torch.where(keep, logit, torch.full_like(logit, -math.inf))
    any_k = keep.any(dim=1, keepdim=True)
    P = torch.softmax(torch.where(any_k, logit, torch.zeros_like(logit)), dim=1)
    return torch.where(any_k, P @ Vall, torch.zeros((), dtype=torch.float64))


def _autograd(Q, K, V, dO, lm, bq, bk, s, causal):
    q, k, v = _t(Q, True), _t(K, True), _t(V, True)
    out = torch_pyramid_forward(q, k, v, lm, bq, bk, s, causal)
    return [x.numpy() for x in torch.autograd.grad(out, (q, k, v), _t(dO))]


def _causal_map(rng, Nq, Nk, N, bq, bk):
    lm = rng.integers(-1, 4, size=(Nq, Nk)).astype(np.int8)
    for a in range(Nq):
        O.apply_overrides(lm[a], a, N, bq, bk, True, 0)
    return lm


def pin_bwd_autograd_of_pooled_formulation(B):
    """Random maps with every level, ragged N, causal and not: the oracle's
    gradients equal torch autograd of the all-levels masked formulation."""
    rng = np.random.default_rng(31)
    for N, d, bq, bk, causal in ((203, 8, 32, 16, False), (171, 4, 64, 32, True),
                                 (96, 8, 16, 16, True)):
        Q, K, V, dO = (_rand(N + i, N, d) for i in range(4))
        Nq, Nk = -(-N // bq), -(-N // bk)
        lm = (_causal_map(rng, Nq, Nk, N, bq, bk) if causal
              else rng.integers(-1, 4, size=(Nq, Nk)).astype(np.int8))
        lm[0, :] = -1                                   # one query block keeps nothing
        s = 0.7 / math.sqrt(d)
        g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk, s, causal)
        dq, dk, dv = _autograd(Q, K, V, dO, lm, bq, bk, s, causal)
        assert np.allclose(g.dQ, dq, atol=1e-11), (N, causal)
        assert np.allclose(g.dK, dk, atol=1e-11), (N, causal)
        assert np.allclose(g.dV, dv, atol=1e-11), (N, causal)


def _sdpa_grads(Q, K, V, dO, mask=None, causal=False):
    q, k, v = _t(Q, True)[None, None], _t(K, True)[None, None], _t(V, True)[None, None]
    am = None if mask is None else _t(mask)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=am,
                                                           is_causal=causal)
    g = torch.autograd.grad(out, (q, k, v), _t(dO)[None, None])
    return [x[0, 0].numpy() for x in g]


def pin_bwd_level0_is_dense_sdpa(B):
    """All-level-0 maps: the gradients of dense softmax attention (torch SDPA
    autograd), bidirectional and causal, ragged N."""
    N, d, bq, bk = 200, 16, 64, 64
    Q, K, V, dO = (_rand(40 + i, N, d) for i in range(4))
    Nq, Nk = -(-N // bq), -(-N // bk)
    g = B.pyramid_attention_backward(Q, K, V, np.zeros((Nq, Nk), np.int8), dO, bq, bk)
    for got, want in zip((g.dQ, g.dK, g.dV), _sdpa_grads(Q, K, V, dO)):
        assert np.allclose(got, want, atol=1e-11)
    lmc = np.array([[0 if j * bk <= min((a + 1) * bq, N) - 1 else -1 for j in range(Nk)]
                    for a in range(Nq)], dtype=np.int8)
    g = B.pyramid_attention_backward(Q, K, V, lmc, dO, bq, bk, causal=True)
    for got, want in zip((g.dQ, g.dK, g.dV), _sdpa_grads(Q, K, V, dO, causal=True)):
        assert np.allclose(got, want, atol=1e-11)


def _block_mask(lm, N, bq, bk):
    mask = np.zeros((N, N))
    for a in range(lm.shape[0]):
        for j in range(lm.shape[1]):
            if lm[a, j] < 0:
                mask[a * bq:(a + 1) * bq, j * bk:(j + 1) * bk] = -np.inf
    return mask


def pin_bwd_binary_is_block_sparse_sdpa(B):
    """{0, -1} maps: the gradients of SDPA with -inf on the dropped blocks."""
    N, d, bq, bk = 256 + 40, 8, 64, 64
    Q, K, V, dO = (_rand(50 + i, N, d) for i in range(4))
    rng = np.random.default_rng(51)
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = np.where(rng.random((Nq, Nk)) < 0.5, 0, -1).astype(np.int8)
    lm[:, 1] = 0
    g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk)
    for got, want in zip((g.dQ, g.dK, g.dV), _sdpa_grads(Q, K, V, dO, _block_mask(lm, N, bq, bk))):
        assert np.allclose(got, want, atol=1e-11)


def pin_bwd_group_constant_tokens_equal_level0(B):
    """K and V constant inside every 8-token group: a pooled row equals each of
    its tokens, so any level's gradient reaching a token equals level 0's, and
    a map with levels 0..3 has the gradients of SDPA over its kept blocks."""
    N, d, bq, bk = 64 * 3 + 16, 8, 64, 64
    rng = np.random.default_rng(61)
    G = -(-N // 8)
    K = np.repeat(rng.standard_normal((G, d)), 8, 0)[:N]
    V = np.repeat(rng.standard_normal((G, d)), 8, 0)[:N]
    Q, dO = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = rng.integers(-1, 4, size=(Nq, Nk)).astype(np.int8)
    lm[:, 0] = 2
    g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk)
    want = _sdpa_grads(Q, K, V, dO, _block_mask(lm, N, bq, bk))
    for got, w in zip((g.dQ, g.dK, g.dV), want):
        assert np.allclose(got, w, atol=1e-11)


def pin_bwd_finite_differences(B):
    """Central differences of L = sum(dO * O) through the forward oracle, for
    every entry of Q, K and V of a small head (ragged, causal, all levels)."""
    N, d, bq, bk = 44, 3, 16, 16
    rng = np.random.default_rng(71)
    Q, K, V, dO = (rng.standard_normal((N, d)) for _ in range(4))
    lm = _causal_map(rng, 3, 3, N, bq, bk)
    lm[2, 0] = 3
    lm[1, 0] = 1
    s = 0.9

    def loss(Q_, K_, V_):
        out, _ = O.pyramid_attention(Q_, O.build_pyramid(K_, V_), lm, bq, bk, s, causal=True)
        return float((dO * out).sum())

    g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk, s, causal=True)
    h = 1e-5
    for name, X, G in (("Q", Q, g.dQ), ("K", K, g.dK), ("V", V, g.dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            args = {"Q": Q, "K": K, "V": V}
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            num[idx] = (loss(**{**{k + "_": v for k, v in args.items()}, name + "_": Xp})
                        - loss(**{**{k + "_": v for k, v in args.items()}, name + "_": Xm})) / (2 * h)
        assert np.allclose(G, num, atol=1e-8), name


def pin_bwd_invariants(B):
    """sum_t dV[t] = sum of dO over rows that keep a key; sum_t dK[t] = 0;
    sum_i <Q_i, dQ_i> = sum_t <K_t, dK_t> (causal, ragged, all levels)."""
    N, d, bq, bk = 331, 8, 64, 64
    rng = np.random.default_rng(81)
    Q, K, V, dO = (rng.standard_normal((N, d)) for _ in range(4))
    Nq, Nk = -(-N // bq), -(-N // bk)
    lm = _causal_map(rng, Nq, Nk, N, bq, bk)
    lm[1, :] = -1
    g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk, 0.5, causal=True)
    live = np.ones(N, bool)
    live[bq:2 * bq] = False
    assert np.allclose(g.dV.sum(0), dO[live].sum(0), atol=1e-11)
    assert np.allclose(g.dK.sum(0), 0.0, atol=1e-11)
    assert math.isclose((Q * g.dQ).sum(), (K * g.dK).sum(), rel_tol=1e-11, abs_tol=1e-11)
    assert np.all(g.dQ[bq:2 * bq] == 0)


def pin_bwd_constant_values(B):
    """V constant: O does not depend on Q or K, so dQ = dK = 0 and dV sums to
    the dO of the live rows."""
    N, d, bq, bk = 192, 8, 64, 64
    rng = np.random.default_rng(91)
    Q, K, dO = (rng.standard_normal((N, d)) for _ in range(3))
    V = np.tile(np.linspace(-1, 2, d), (N, 1))
    lm = np.array([[0, 3, -1], [1, 2, 2], [2, 1, 0]], dtype=np.int8)
    g = B.pyramid_attention_backward(Q, K, V, lm, dO, bq, bk, 0.3)
    assert np.allclose(g.dQ, 0.0, atol=1e-12) and np.allclose(g.dK, 0.0, atol=1e-12)
    assert np.allclose(g.dV.sum(0), dO.sum(0), atol=1e-12)


def pin_bwd_grouped_queries(B):
    """Grouped queries: torch autograd with each query head's forward reading
    the shared KV head sums the KV gradients over the group."""
    rng = np.random.default_rng(101)
    Bn, Hq, Hkv, N, d, bq, bk = 2, 4, 2, 96, 4, 32, 16
    Q, dO = rng.standard_normal((Bn, Hq, N, d)), rng.standard_normal((Bn, Hq, N, d))
    K, V = rng.standard_normal((Bn, Hkv, N, d)), rng.standard_normal((Bn, Hkv, N, d))
    lm = rng.integers(-1, 4, size=(Bn, Hq, 3, 6)).astype(np.int8)
    r = B.psa_backward(Q, K, V, dO, lm, bq, bk)
    s = 1 / math.sqrt(d)
    for b in range(Bn):
        k, v = _t(K[b], True), _t(V[b], True)
        qs = [_t(Q[b, h], True) for h in range(Hq)]
        outs = [torch_pyramid_forward(qs[h], k[h // 2], v[h // 2], lm[b, h], bq, bk, s, False)
                for h in range(Hq)]
        loss = sum((o * _t(dO[b, h])).sum() for h, o in enumerate(outs))
        grads = torch.autograd.grad(loss, qs + [k, v])
        for h in range(Hq):
            assert np.allclose(r.dQ[b, h], grads[h].numpy(), atol=1e-11)
        assert np.allclose(r.dK[b], grads[Hq].numpy(), atol=1e-11)
        assert np.allclose(r.dV[b], grads[Hq + 1].numpy(), atol=1e-11)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
