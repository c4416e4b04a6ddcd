"""GPU parity of psa_backward (dQ, dK, dV with the level map held fixed)
against the float64 backward oracle, through the C ABI.

Tolerance (bf16 path), per gradient tensor, relative to its largest reference
magnitude: max |err| <= 3e-2 and mean |err| / mean |ref| <= 1e-2.  The kernel
stores P and dS = P (dP - D) in bf16 for the tensor-core products (relative
rounding 2^-9 ~ 2e-3 each), reads the bf16-stored pyramid levels and the
bf16 forward output O (through D = dO . O), and rounds the gradients to bf16
once; the fp32 accumulation over many keys and query rows averages those
roundings.  The fp32 CUDA-core path: max |err| <= 1e-4 of the largest
magnitude."""
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
CASES = {
    # tensor-core path, d = 128, ragged N = 1000
    "bf16_d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 20, 50),
                                  coarse=(1, 5, 13), seed=41, target="fixed"),
    # tensor-core path, d = 64, N = 226 + 760 with a forced text prefix
    "bf16_d64": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, grid=(1, 20, 38),
                                 coarse=(1, 5, 10), seed=42, target="fixed"),
    # grouped queries (2 per KV head), causal
    "bf16_gqa_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=4, Hkv=2, grid=(1, 25, 40),
                                        coarse=(1, 7, 10), seed=43, target="fixed"),
    # ragged pooled groups: N = 1003 (the last level-3 group averages 3 tokens)
    "bf16_ragged_groups": W.with_overrides(BASE["wan2.1_1.3b"], Hq=1, Hkv=1, grid=(1, 17, 59),
                                           coarse=(1, 5, 15), seed=44, target="fixed"),
    # two batch elements
    "bf16_batch2": W.with_overrides(BASE["wan2.1_1.3b"], B=2, Hq=1, Hkv=1, grid=(1, 16, 40),
                                    coarse=(1, 4, 10), seed=45, target="fixed"),
    # CUDA-core path: bf16 with 64-row query blocks, causal, grouped queries
    "bf16_q64_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=2, Hkv=1, grid=(1, 20, 33),
                                        coarse=(1, 5, 9), seed=46, q_blk=64, target="fixed"),
    # CUDA-core path: fp32, d = 128 and the tiny fp32 workload (d = 64)
    "f32_d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=2, Hkv=2, dtype="f32",
                                 grid=(1, 18, 40), coarse=(1, 5, 10), seed=47, target="fixed"),
    "tiny_f32": BASE["tiny_f32"],
}


def _map(w, kind, rng):
    m = np.empty((w.B, w.Hq, w.Nq, w.Nk), dtype=np.int8)
    for b in range(w.B):
        for h in range(w.Hq):
            if kind == "random":
                m[b, h] = G.rand_map(rng, w.Nq, w.Nk)
            elif kind == "all_level0":
                m[b, h] = 0
            elif kind == "all_level3":
                m[b, h] = 3
            else:                                   # "pruned_rows"
                m[b, h] = G.rand_map(rng, w.Nq, w.Nk, 0, 4)
                m[b, h, 1::3] = -1
            if w.causal:
                for a in range(w.Nq):
                    O.apply_overrides(m[b, h, a], a, w.N, w.q_blk, w.kv_blk, True, 0)
                if kind == "pruned_rows":
                    m[b, h, 1::3] = -1
    return m


def _grad_out(w, seed, wide=True):
    """dO: seeded N(0, 1) in the workload's dtype, on the device, and the same
    values on the host (float64 if ``wide``, else float32)."""
    g = np.random.default_rng(seed).standard_normal((w.B, w.Hq, w.N, w.d)).astype(np.float32)
    if w.dtype == "bf16":
        bits = W.f32_to_bf16_bits(g)
        g = W.bf16_bits_to_f32(bits)
        dev = G.to_device(bits, "bf16")
    else:
        dev = G.to_device(g, "f32")
    return dev, (g.astype(np.float64) if wide else g)


def _run_backward(w, inp, run, dO, m=None, host=True):
    p = run.p
    dQ = torch.full_like(run.q, float("nan"))
    dK = torch.full_like(run.k, float("nan"))
    dV = torch.full_like(run.v, float("nan"))
    bws = P.new_backward_workspace(p)
    lm = None if m is None else torch.from_numpy(np.ascontiguousarray(m)).cuda()
    P.backward(p, run.q, run.k, run.v, run.O, run.lse, dO, run.ws, bws, dQ, dK, dV, lm)
    torch.cuda.synchronize()
    P.check_device(p, run.ws)
    del bws
    if not host:
        return dQ, dK, dV
    return G.to_f64(dQ), G.to_f64(dK), G.to_f64(dV)


def _oracle(w, inp, m, dO64):
    Q, K, V = (np.stack([np.stack([inp.as_f64(n, b, h) for h in range(H)]) for b in range(w.B)])
               for n, H in (("q", w.Hq), ("k", w.Hkv), ("v", w.Hkv)))
    return OB.psa_backward(Q, K, V, dO64, m, w.q_blk, w.kv_blk, w.causal)


def compare_grad(got, ref, dtype, what, floor=1e-30):
    """Errors relative to the reference's largest and mean magnitudes (each at
    least ``floor``, for gradients that vanish in exact arithmetic)."""
    scale = max(float(np.abs(ref).max()), floor)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    max_rel = float(err.max()) / scale
    mean_rel = float(err.mean() / max(np.abs(ref).mean(), floor))
    if dtype == "bf16":
        assert max_rel <= 3e-2 and mean_rel <= 1e-2, (what, max_rel, mean_rel)
    else:
        assert max_rel <= 1e-4, (what, max_rel, mean_rel)
    return max_rel, mean_rel


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("kind", ["random", "all_level0", "all_level3", "pruned_rows"])
def test_backward_on_external_maps(name, kind):
    w = CASES[name]
    inp = W.make_inputs(w)
    rng = np.random.default_rng(zlib.crc32(f"bwd/{name}/{kind}".encode()))
    m = _map(w, kind, rng)
    run = G.run_stages(w, inp, external_map=m)
    dO, dO64 = _grad_out(w, zlib.crc32(f"dO/{name}".encode()))
    gq, gk, gv = _run_backward(w, inp, run, dO, m)
    ref = _oracle(w, inp, m, dO64)
    compare_grad(gq, ref.dQ, w.dtype, "dQ")
    compare_grad(gk, ref.dK, w.dtype, "dK")
    compare_grad(gv, ref.dV, w.dtype, "dV")
    if kind == "pruned_rows":
        # query blocks that keep nothing pass no gradient: dQ rows exactly 0
        for a in range(1, w.Nq, 3):
            rows = slice(a * w.q_blk, min((a + 1) * w.q_blk, w.N))
            assert np.all(gq[:, :, rows] == 0)


SEQUENCE_CASES = {
    # d = 128 and d = 64, 128-row query blocks (the tensor-core kernel); N = 1000 and 986
    "d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=192, Hkv=192, grid=(1, 20, 50),
                             coarse=(1, 5, 13), seed=51, target="fixed"),
    "d64": W.with_overrides(BASE["cogvideox_5b"], Hq=192, Hkv=192, n_text=0, grid=(1, 29, 34),
                            coarse=(1, 8, 9), forced_prefix_tokens=0, seed=52, target="fixed"),
}


@pytest.mark.parametrize("name", sorted(SEQUENCE_CASES))
def test_backward_block_sequences(name):
    """About ten query blocks per persistent CTA, of 0 to 8 tiles in random
    order (a quarter keep no block): dQ accumulates in TMEM over each block's
    tiles and is stored at its end, and dK, dV are added row by row into the
    level accumulators across blocks.  Every head's gradients against the
    oracle (the criterion of the other cases, over the whole tensors), and
    exact zeros where nothing is kept."""
    w = SEQUENCE_CASES[name]
    inp = W.make_inputs(w)
    rng = np.random.default_rng(zlib.crc32(f"bwd-sequences/{name}".encode()))
    m = np.stack([G.sequence_map(rng, w.Nq, w.Nk) for _ in range(w.B * w.Hq)])
    m = m.reshape(w.B, w.Hq, w.Nq, w.Nk)
    assert w.B * w.Hq * w.Nq >= 8 * 148
    run = G.run_stages(w, inp, external_map=m)
    dO, dO64 = _grad_out(w, zlib.crc32(f"dO-sequences/{name}".encode()))
    gq, gk, gv = _run_backward(w, inp, run, dO, m)
    ref = _oracle(w, inp, m, dO64)
    compare_grad(gq, ref.dQ, w.dtype, "dQ")
    compare_grad(gk, ref.dK, w.dtype, "dK")
    compare_grad(gv, ref.dV, w.dtype, "dV")
    # query blocks that keep nothing pass no gradient: their dQ rows are 0
    for h in range(w.Hq):
        for a in np.nonzero((m[0, h] < 0).all(axis=1))[0]:
            rows = slice(a * w.q_blk, min((a + 1) * w.q_blk, w.N))
            assert np.all(gq[0, h, rows] == 0)


@pytest.mark.parametrize("name", ["bf16_d128", "bf16_gqa_causal", "tiny_f32"])
def test_backward_after_fused_forward_uses_its_work_list(name):
    """level_map = NULL: the backward walks the list psa_forward left in the
    workspace; the oracle is given the map the GPU chose."""
    w = CASES[name]
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp, fused=True)
    gm = run.level_map.cpu().numpy()
    dO, dO64 = _grad_out(w, 99)
    gq, gk, gv = _run_backward(w, inp, run, dO, None)
    ref = _oracle(w, inp, gm, dO64)
    compare_grad(gq, ref.dQ, w.dtype, "dQ")
    compare_grad(gk, ref.dK, w.dtype, "dK")
    compare_grad(gv, ref.dV, w.dtype, "dV")


def test_backward_invariants_on_gpu():
    """Properties that hold at any size, on the tensor-core path: the dV sum
    equals the dO sum over rows that keep a key, and dK sums to 0."""
    w = CASES["bf16_d128"]
    inp = W.make_inputs(w)
    m = _map(w, "random", np.random.default_rng(5))
    run = G.run_stages(w, inp, external_map=m)
    dO, dO64 = _grad_out(w, 7)
    gq, gk, gv = _run_backward(w, inp, run, dO, m)
    live = np.isfinite(run.lse.cpu().numpy())
    for b in range(w.B):
        for h in range(w.Hkv):
            want = (dO64[b, h] * live[b, h][:, None]).sum(0)
            scale = np.abs(dO64[b, h]).sum(0).max()
            assert np.abs(gv[b, h].sum(0) - want).max() <= 1e-2 * scale
            assert np.abs(gk[b, h].sum(0)).max() <= 1e-2 * np.abs(gk[b, h]).sum(0).max()


FULL = ["wan2.1_1.3b", "cogvideox_5b", "wan2.1_14b_720p", "qwen2.5_vl_7b"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_backward_full_size_sampled(name):
    """Full-size workloads in the benchmark's launch configuration.
    1. The map the GPU chose: dQ of sampled query blocks (each depends only on
       its own kept keys) against the oracle, and the dK / dV sums that hold
       at any size (sum dV = sum dO over rows that keep a key; sum dK = 0).
    2. A map keeping only a few query blocks of a few heads: every element of
       dQ, dK and dV against the oracle (only those blocks contribute)."""
    w = W.BY_NAME[name]
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp, fused=True)
    gm = run.level_map.cpu().numpy()
    dO, dO32 = _grad_out(w, 2024, wide=False)
    gq, gk, gv = _run_backward(w, inp, run, dO, None, host=False)
    grp = w.Hq // w.Hkv
    rng = np.random.default_rng(3)
    heads = sorted({0, w.Hq // 2, w.Hq - 1})
    blocks = sorted({0, w.Nq - 1, int(rng.integers(1, w.Nq - 1))})
    s = 1.0 / np.sqrt(w.d)
    for h in heads:
        Q, dOh = inp.as_f64("q", 0, h), dO32[0, h].astype(np.float64)
        K, V = inp.as_f64("k", 0, h // grp), inp.as_f64("v", 0, h // grp)
        sub = np.full_like(gm[0, h], -1)
        sub[blocks] = gm[0, h][blocks]
        ref = OB.pyramid_attention_backward(Q, K, V, sub, dOh, w.q_blk, w.kv_blk, s, w.causal)
        rows = np.concatenate([np.arange(a * w.q_blk, min((a + 1) * w.q_blk, w.N)) for a in blocks])
        compare_grad(G.to_f64(gq[0, h])[rows], ref.dQ[rows], w.dtype, f"dQ head {h}")
    live = torch.isfinite(run.lse[0]).to(torch.float64)                        # [Hq, N]
    dO_dev = dO[0].to(torch.float64) * live[:, :, None]
    for hk in range(w.Hkv):
        want = dO_dev[hk * grp:(hk + 1) * grp].sum((0, 1))
        v64, k64 = gv[0, hk].to(torch.float64), gk[0, hk].to(torch.float64)
        assert float((v64.sum(0) - want).abs().max()) <= 1e-2 * float(v64.abs().sum(0).max()), hk
        assert float(k64.sum(0).abs().max()) <= 1e-2 * float(k64.abs().sum(0).max()), hk
    del gq, gk, gv, dO_dev

    # 2. a few query blocks of a few heads, every gradient element
    sub = np.full_like(gm, -1)
    for h in heads:
        sub[0, h, blocks] = gm[0, h, blocks]
    del run
    run2 = G.run_stages(w, inp, external_map=sub)
    gq, gk, gv = _run_backward(w, inp, run2, dO, sub, host=False)
    kv_heads = sorted({h // grp for h in heads})
    for hk in kv_heads:
        K, V = inp.as_f64("k", 0, hk), inp.as_f64("v", 0, hk)
        dK = np.zeros((w.N, w.d))
        dV = np.zeros((w.N, w.d))
        for h in [h for h in heads if h // grp == hk]:
            ref = OB.pyramid_attention_backward(inp.as_f64("q", 0, h), K, V, sub[0, h],
                                                dO32[0, h].astype(np.float64), w.q_blk, w.kv_blk,
                                                s, w.causal)
            compare_grad(G.to_f64(gq[0, h]), ref.dQ, w.dtype, f"dQ head {h}")
            dK += ref.dK
            dV += ref.dV
        compare_grad(G.to_f64(gk[0, hk]), dK, w.dtype, f"dK kv head {hk}")
        compare_grad(G.to_f64(gv[0, hk]), dV, w.dtype, f"dV kv head {hk}")
    others = [h for h in range(w.Hkv) if h not in kv_heads]
    if others:
        assert bool((gk[0, others] == 0).all()) and bool((gv[0, others] == 0).all())


def test_autograd_entry_point_matches_direct_calls():
    """psa_attention: O and dQ equal psa_forward's and psa_backward's on the
    same map, bit for bit.  dK and dV are sums by float atomics, whose order
    varies between calls, so they agree to rounding: within one bf16 ulp after
    the final rounding."""
    w = CASES["bf16_gqa_causal"]
    inp = W.make_inputs(w)
    tau = W.thresholds(w)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = P.psa_attention(qg, kg, vg, w.q_blk, w.kv_blk, tau, w.causal)
    dO, _ = _grad_out(w, 11)
    o.backward(dO)
    out, lse, lm = P.psa_forward(q, k, v, w.q_blk, w.kv_blk, tau, w.causal, return_map=True)
    assert torch.equal(o.detach(), out)
    p = G.params_for(w)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    P.backward(p, q, k, v, out, lse, dO, P.new_workspace(p), P.new_backward_workspace(p),
               dq, dk, dv, level_map=lm)
    torch.cuda.synchronize()
    assert torch.equal(qg.grad, dq)
    for a, b in ((kg.grad, dk), (vg.grad, dv)):
        a, b = a.float(), b.float()
        assert bool(((a - b).abs() <= 2.0 ** -7 * b.abs() + 1e-6 * b.abs().max()).all())
