"""Degenerate sizes through the forward and backward passes, against the
oracle: a single token, fewer tokens than one level-3 group, one KV block
minus / plus one token, one query block minus / plus one token.  Both the
tensor-core path (bf16, 128-row query blocks) and the CUDA-core path (fp32),
causal and not."""
import numpy as np
import pytest
import torch

import level_sparse_attention_b200 as P
import oracle as O
import workloads as W
from oracle import psa_backward as OB
from tests import gpu_common as G
from tests.test_gpu_backward import _grad_out, _run_backward, compare_grad

pytestmark = pytest.mark.gpu

SIZES = {1: (1, 1, 1), 5: (1, 1, 5), 63: (1, 7, 9), 65: (1, 5, 13), 127: (1, 1, 127),
         129: (1, 3, 43)}


def _case(N, path, causal):
    base = W.BY_NAME["qwen2.5_vl_7b"] if causal else W.BY_NAME["wan2.1_1.3b"]
    # coarse = grid: every token drawn independently.  (A single coarse point
    # would make K and V nearly constant, dP ~ D, and dQ, dK differences of
    # nearly equal terms: ill-conditioned, a case this test is not about.)
    kw = dict(B=1, Hq=2, Hkv=1 if causal else 2, grid=SIZES[N], coarse=SIZES[N], n_text=0,
              forced_prefix_tokens=0, seed=60 + N, target="fixed")
    if path == "f32":
        kw.update(dtype="f32", d=64, q_blk=64)
    return W.with_overrides(base, **kw)


@pytest.mark.parametrize("N", sorted(SIZES))
@pytest.mark.parametrize("path", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_sequences_forward_and_backward(N, path, causal):
    w = _case(N, path, causal)
    assert w.N == N
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp, fused=True)
    gm = run.level_map.cpu().numpy()
    tau = W.thresholds(w)
    ref = G.oracle_heads(w, inp, [(0, h) for h in range(w.Hq)])
    gO = G.to_f64(run.O)
    glse = run.lse.cpu().numpy().astype(np.float64)
    for (b, h), r in ref.items():
        assert G.map_mismatch_report(gm[b, h], r.mask, tau)[0] == 0
        G.compare_out(gO[b, h], r.O, w.dtype)
        G.compare_lse(glse[b, h], r.lse, w.dtype)
    # backward on a map with every level (the diagonal forced to 0 when causal)
    rng = np.random.default_rng(N)
    m = G.rand_map(rng, w.Nq, w.Nk, 0, 4)[None, None].repeat(w.Hq, axis=1)
    if causal:
        for h in range(w.Hq):
            for a in range(w.Nq):
                O.apply_overrides(m[0, h, a], a, w.N, w.q_blk, w.kv_blk, True, 0)
    run2 = G.run_stages(w, inp, external_map=m)
    dO, dO64 = _grad_out(w, 100 + N)
    gq, gk, gv = _run_backward(w, inp, run2, dO, m)
    Q = np.stack([inp.as_f64("q", 0, h) for h in range(w.Hq)])[None]
    K = np.stack([inp.as_f64("k", 0, h) for h in range(w.Hkv)])[None]
    V = np.stack([inp.as_f64("v", 0, h) for h in range(w.Hkv)])[None]
    r = OB.psa_backward(Q, K, V, dO64, m, w.q_blk, w.kv_blk, w.causal)
    # a single token: dQ = dK = 0 in exact arithmetic (P = 1, O = V), so the
    # errors are measured against a floor of 1e-2 (the gradients' scale here is 1)
    compare_grad(gq, r.dQ, w.dtype, "dQ", floor=1e-2)
    compare_grad(gk, r.dK, w.dtype, "dK", floor=1e-2)
    compare_grad(gv, r.dV, w.dtype, "dV", floor=1e-2)
