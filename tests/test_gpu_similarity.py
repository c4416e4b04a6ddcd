"""GPU parity of the cosine-similarity constraint (sim_threshold) against the
oracle: the largest level each KV block may use, the clamped level maps, and
the attention on them.

A block's largest level is exact unless a cosine that decides it lies within
1e-4 of the threshold: the kernel takes the cosines in fp32 from the same
input values (relative error ~1e-6), the oracle in float64."""
import numpy as np
import pytest
import torch

import level_sparse_attention_b200 as P
import oracle as O
import workloads as W
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

BASE = W.BY_NAME
CASES = {
    "bf16_d128_ragged": W.with_overrides(BASE["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 17, 59),
                                         coarse=(1, 5, 15), seed=51, target="fixed"),
    "bf16_d64_text": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, grid=(1, 20, 38),
                                      coarse=(1, 5, 10), seed=52, target="fixed"),
    "bf16_gqa_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=4, Hkv=2, grid=(1, 25, 40),
                                        coarse=(1, 7, 10), seed=53, target="fixed"),
    "tiny_f32": BASE["tiny_f32"],
}
EPS_COS = 1e-4


def _params(w, theta):
    return P.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.q_blk, w.kv_blk, W.thresholds(w), w.causal,
                         w.forced_prefix_tokens, 0.0,
                         torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                         sim_threshold=theta)


def _maxlev_ok(gpu, ref, min_cos, theta):
    """Unexplained differences between the GPU's and the oracle's largest
    levels (a difference is explained by a deciding cosine within EPS_COS of
    theta)."""
    bad = 0
    for j in np.nonzero(gpu != ref)[0]:
        lo, hi = sorted((int(gpu[j]), int(ref[j])))
        if not any(abs(min_cos[j, l] - theta) < EPS_COS for l in range(lo + 1, hi + 1)):
            bad += 1
    return bad


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("theta", [0.0, 0.3, 0.55])
def test_similarity_constraint(name, theta):
    w = CASES[name]
    inp = W.make_inputs(w)
    p = _params(w, theta)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    ws = P.new_workspace(p)
    lm = torch.full(P.map_shape(p), -7, dtype=torch.int8, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    P.forward(p, q, k, v, out, ws, lse, lm)
    torch.cuda.synchronize()
    P.check_device(p, ws)
    L = P.workspace_layout(p)
    gml = P.workspace_view(ws, L["maxlev"], (w.B, w.Hkv, w.Nk), torch.int8).cpu().numpy()
    gm = lm.cpu().numpy()
    tau = W.thresholds(w)
    grp = w.Hq // w.Hkv
    s = 1.0 / np.sqrt(w.d)
    levels_seen = set()
    for hk in range(w.Hkv):
        K = inp.as_f64("k", 0, hk)
        ml, mc = O.block_max_levels(K, w.kv_blk, theta)
        levels_seen |= set(ml.tolist())
        assert _maxlev_ok(gml[0, hk], ml, mc, theta) == 0, (hk, gml[0, hk], ml)
        near = np.nonzero(gml[0, hk] != ml)[0]           # excused above: a cosine within EPS_COS
        V = inp.as_f64("v", 0, hk)
        pyr = O.build_pyramid(K, V)
        for h in range(hk * grp, (hk + 1) * grp):
            Q = inp.as_f64("q", 0, h)
            z = O.block_logits(O.query_block_means(Q, w.q_blk), pyr, w.kv_blk, s)
            mask = O.assign_levels(z, tau, w.N, w.q_blk, w.kv_blk, w.causal,
                                   w.forced_prefix_tokens, max_level=ml)
            cmp = gm[0, h].copy()
            cmp[:, near] = mask.level_map[:, near]
            assert G.map_mismatch_report(cmp, mask, tau)[0] == 0, h
            # kept levels never exceed the block's largest level
            kept = gm[0, h] >= 0
            assert np.all(gm[0, h][kept] <= gml[0, hk][np.nonzero(kept)[1]])
            # attention on the GPU's (clamped) map
            ref_O, ref_lse = O.pyramid_attention(Q, pyr, gm[0, h], w.q_blk, w.kv_blk, s, w.causal)
            G.compare_out(G.to_f64(out[0, h]), ref_O, w.dtype)
    if theta == 0.3 and name != "tiny_f32":
        assert len(levels_seen) >= 2, levels_seen          # the constraint binds


def test_similarity_off_equals_no_constraint():
    """sim_threshold = -1 (and below) gives the same map and output as the
    constraint never being computed."""
    w = CASES["bf16_d128_ragged"]
    inp = W.make_inputs(w)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    outs = []
    for theta in (-1.0, -3.0):
        p = _params(w, theta)
        ws = P.new_workspace(p)
        lm = torch.full(P.map_shape(p), -7, dtype=torch.int8, device="cuda")
        out = torch.zeros_like(q)
        P.forward(p, q, k, v, out, ws, None, lm)
        torch.cuda.synchronize()
        outs.append((lm.cpu(), out.cpu()))
    run = G.run_stages(w, inp, fused=True)
    for lm_, out_ in outs:
        assert torch.equal(lm_, run.level_map.cpu()) and torch.equal(out_, run.O.cpu())
