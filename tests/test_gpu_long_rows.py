"""Work lists longer than the tensor-core kernels' shared-memory copy.

The attention kernels stage the first 1024 entries of a query block's work
list in shared memory and read later entries from global memory.  Rows that
keep more than 1024 KV blocks (N >= 65600 with 64-token blocks) reach that
second path, in the forward kernel and in the gradient kernel.  One head,
N = 66000 (1032 KV blocks per row, 516 query blocks: the persistent grid's
bands of 148 CTAs end at blocks 147, 295, 443 and 515), checked against the
oracle on sampled query blocks, including the first and last blocks of every
band, and on every gradient element of a map that keeps only those blocks."""
import zlib

import numpy as np
import pytest
import torch

import level_sparse_attention_b200 as P
import oracle as O
import workloads as W
from oracle import psa_backward as OB
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

BASE = W.BY_NAME
N_GRID = (4, 110, 150)                       # N = 66000
SAMPLE = [0, 1, 147, 148, 295, 296, 443, 444, 514, 515]


def _workload(d, causal=False, seed=51, target="fixed"):
    base = BASE["qwen2.5_vl_7b"] if causal else BASE["wan2.1_1.3b"]
    return W.with_overrides(base, Hq=1, Hkv=1, d=d, n_text=0, grid=N_GRID, coarse=(1, 28, 38),
                            forced_prefix_tokens=0, seed=seed, target=target)


def _rows(w, blocks):
    return np.concatenate([np.arange(a * w.q_blk, min((a + 1) * w.q_blk, w.N)) for a in blocks])


def _map(w, kind, rng):
    m = np.zeros((w.Nq, w.Nk), dtype=np.int8)
    if kind == "all_level3":
        m[:] = 3
    elif kind == "random":
        m[:] = rng.integers(0, 4, size=m.shape)
        for a in range(w.Nq):                       # 3 pruned blocks: 1029 kept per row
            m[a, rng.choice(w.Nk, 3, replace=False)] = -1
    if w.causal:
        for a in range(w.Nq):
            O.apply_overrides(m[a], a, w.N, w.q_blk, w.kv_blk, True, 0)
    return m


def _entries(m):
    return (m >= 0).sum(-1)


@pytest.mark.parametrize("d,causal,kind", [(128, False, "all_level0"), (128, False, "random"),
                                           (64, False, "all_level3"), (128, True, "all_level0")])
def test_forward_rows_past_the_list_cache(d, causal, kind):
    w = _workload(d, causal)
    assert w.Nk == 1032 and w.Nq == 516
    rng = np.random.default_rng(zlib.crc32(f"long/{d}/{causal}/{kind}".encode()))
    m = _map(w, kind, rng)
    blocks = SAMPLE + sorted(rng.choice(np.arange(2, 514), 6, replace=False).tolist())
    assert _entries(m)[blocks].max() > 1024
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp, external_map=m[None, None])
    sub = np.full_like(m, -1)
    sub[blocks] = m[blocks]
    Q, K, V = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0), inp.as_f64("v", 0, 0)
    ref_O, ref_lse = O.pyramid_attention(Q, O.build_pyramid(K, V), sub, w.q_blk, w.kv_blk,
                                         1.0 / np.sqrt(d), causal)
    rows = _rows(w, blocks)
    G.compare_out(G.to_f64(run.O[0, 0]), ref_O, w.dtype, rows=rows)
    G.compare_lse(run.lse[0, 0].cpu().numpy().astype(np.float64)[rows], ref_lse[rows], w.dtype)


def test_forward_mask_with_tau3_one_keeps_every_block():
    """psa_forward with tau_3 = 1: every block of every row kept at some
    level (1032 entries per row); the map against the oracle's on sampled
    rows, the output on them."""
    w = _workload(128, seed=52, target="alpha:1.0")
    tau = W.thresholds(w)
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp, fused=True)
    gm = run.level_map.cpu().numpy()[0, 0]
    assert np.all(gm >= 0)
    Q, K, V = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0), inp.as_f64("v", 0, 0)
    pyr = O.build_pyramid(K, V)
    s = 1.0 / np.sqrt(w.d)
    z = O.block_logits(O.query_block_means(Q, w.q_blk)[SAMPLE], pyr, w.kv_blk, s)
    mask = O.assign_levels(z, tau, w.N, w.q_blk, w.kv_blk)
    assert G.map_mismatch_report(gm[SAMPLE], mask, tau)[0] == 0
    sub = np.full_like(gm, -1)
    sub[SAMPLE] = gm[SAMPLE]
    ref_O, _ = O.pyramid_attention(Q, pyr, sub, w.q_blk, w.kv_blk, s)
    G.compare_out(G.to_f64(run.O[0, 0]), ref_O, w.dtype, rows=_rows(w, SAMPLE))


def _grad_out(w, seed):
    g = np.random.default_rng(seed).standard_normal((w.B, w.Hq, w.N, w.d)).astype(np.float32)
    bits = W.f32_to_bf16_bits(g)
    return G.to_device(bits, "bf16"), W.bf16_bits_to_f32(bits).astype(np.float64)


def _backward(run, dO, m):
    p = run.p
    dQ, dK, dV = (torch.full_like(t, float("nan")) for t in (run.q, run.k, run.v))
    bws = P.new_backward_workspace(p)
    P.backward(p, run.q, run.k, run.v, run.O, run.lse, dO, run.ws, bws, dQ, dK, dV,
               torch.from_numpy(np.ascontiguousarray(m[None, None])).cuda())
    torch.cuda.synchronize()
    P.check_device(p, run.ws)
    return G.to_f64(dQ[0, 0]), G.to_f64(dK[0, 0]), G.to_f64(dV[0, 0])


def _compare_grad(got, ref, what):
    scale = float(np.abs(ref).max())
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    assert float(err.max()) <= 3e-2 * scale, (what, float(err.max()) / scale)
    assert float(err.mean()) <= 1e-2 * float(np.abs(ref).mean()), what


@pytest.mark.parametrize("kind", ["all_level0", "random"])
def test_backward_rows_past_the_list_cache(kind):
    """dQ of sampled blocks on the full map (each depends only on its own
    kept keys), then every element of dQ, dK and dV on a map that keeps only
    the sampled blocks, each with more than 1024 entries."""
    w = _workload(128, seed=53)
    rng = np.random.default_rng(zlib.crc32(f"long-bwd/{kind}".encode()))
    m = _map(w, kind, rng)
    inp = W.make_inputs(w)
    Q, K, V = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0), inp.as_f64("v", 0, 0)
    dO, dO64 = _grad_out(w, 61)
    s = 1.0 / np.sqrt(w.d)
    sub = np.full_like(m, -1)
    sub[SAMPLE] = m[SAMPLE]
    assert _entries(sub)[SAMPLE].min() > 1024
    run = G.run_stages(w, inp, external_map=m[None, None])
    gq, _, _ = _backward(run, dO, m)
    ref = OB.pyramid_attention_backward(Q, K, V, sub, dO64[0, 0], w.q_blk, w.kv_blk, s)
    rows = _rows(w, SAMPLE)
    _compare_grad(gq[rows], ref.dQ[rows], "dQ (full map)")
    del run
    run = G.run_stages(w, inp, external_map=sub[None, None])
    gq, gk, gv = _backward(run, dO, sub)
    _compare_grad(gq, ref.dQ, "dQ")
    _compare_grad(gk, ref.dK, "dK")
    _compare_grad(gv, ref.dV, "dV")


def _ramp_inputs(w, pairs=False):
    """Q and K whose block logits rise by s * a0 = 0.002 per KV block: every
    query row is a0 * (e_0 + 256 e_1), every key of block j is
    (j mod 256) e_0 + (j div 256) e_1, so q . k = a0 * j exactly in bf16.
    With pairs, blocks 2i and 2i + 1 share the keys of 2i: exactly equal P."""
    inp = W.make_inputs(w)
    a0 = 0.002 * np.sqrt(w.d)
    q = np.zeros((w.B, w.Hq, w.N, w.d), dtype=np.float32)
    q[..., 0], q[..., 1] = a0, 256.0 * a0
    j = np.arange(w.N) // w.kv_blk
    if pairs:
        j = j & ~1
    k = np.zeros((w.B, w.Hkv, w.N, w.d), dtype=np.float32)
    k[..., 0], k[..., 1] = j % 256, j // 256
    inp.q, inp.k = W.f32_to_bf16_bits(q), W.f32_to_bf16_bits(k)
    return inp


@pytest.mark.parametrize("profile", ["peaked", "flat", "quantile", "ties", "causal"])
def test_mask_long_rows_compact_assignment(profile):
    """The assignment of rows of 1032 blocks, which keeps only P and a
    candidate set in shared memory, against the oracle's map on sampled rows.
    peaked: the workload's own inputs and thresholds (the candidate cut holds
    about a tenth of the row).  flat: block logits rising by 0.002 per block,
    so neighbouring P differ by 0.2% and tau_3 = 0.98 keeps about 970 blocks,
    past the candidate set: every block is ranked against every other.
    quantile: the quantile rule with K_3 = ceil(0.2 * 1032) = 207.  ties: the
    flat rise with blocks paired to exactly equal P, through the pairwise
    ranking (ties to the lower index; no mismatch may hide as a near tie).
    causal: the causal VLM shape, where a row sees only the blocks up to its
    diagonal."""
    if profile == "quantile":
        w = W.with_overrides(_workload(128, seed=56), assign="quantile")
        tau = (0.05, 0.1, 0.15, 0.2)
        inp = W.make_inputs(w)
    elif profile in ("flat", "ties"):
        w = _workload(128, seed=55)
        tau = (0.3, 0.6, 0.8, 0.98)
        inp = _ramp_inputs(w, pairs=profile == "ties")
    elif profile == "causal":
        w = _workload(128, causal=True, seed=57)
        tau = W.thresholds(w)
        inp = W.make_inputs(w)
    else:
        w = _workload(128, seed=54)
        tau = W.thresholds(w)
        inp = W.make_inputs(w)
    run = G.run_stages(w, inp, tau=tau)
    gm = run.level_map.cpu().numpy()[0, 0]
    Q, K, V = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0), inp.as_f64("v", 0, 0)
    pyr = O.build_pyramid(K, V)
    # causally a row's visible blocks depend on its index: every row is assigned
    rows = np.arange(w.Nq) if w.causal else np.array(SAMPLE)
    z = O.block_logits(O.query_block_means(Q, w.q_blk)[rows], pyr, w.kv_blk, 1.0 / np.sqrt(w.d))
    mask = O.assign_levels(z, tau, w.N, w.q_blk, w.kv_blk, w.causal, w.forced_prefix_tokens,
                           rule=w.assign)
    kept = (mask.level_map >= 0).sum(-1)
    if profile in ("flat", "ties"):
        assert kept.min() > 900            # well past the 256-block candidate set
    elif profile == "quantile":
        assert kept.max() <= 207
    unexplained, _, near_tie = G.map_mismatch_report(gm[rows], mask, tau, rule=w.assign)
    assert unexplained == 0
    if profile == "ties":
        assert near_tie == 0
