"""GPU parity of every stage of the PSA forward pass against the CPU oracle,
through the C ABI, at sizes the oracle finishes in seconds (several tiles and
ragged tails in every case)."""
import zlib

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
    # the tiny fp32 workload as specified (64-row query blocks, CUDA-core path)
    "tiny_f32": BASE["tiny_f32"],
    # tensor-core path, d = 128, ragged N = 1000 (last query block 104 rows, last KV block 40)
    "bf16_d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 20, 50),
                                  coarse=(1, 5, 13), seed=11, target="fixed"),
    # tensor-core path, d = 64, text prefix forced to level 0, N = 226 + 760
    "bf16_d64_text": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, grid=(1, 20, 38),
                                      coarse=(1, 5, 10), seed=12, target="fixed"),
    # grouped queries (2 per KV head), causal, N = 1000
    "bf16_gqa_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=4, Hkv=2, grid=(1, 25, 40),
                                        coarse=(1, 7, 10), seed=13, target="fixed"),
    # 64-row query blocks (rows 64-127 of the tensor-core tiles idle), causal
    "bf16_q64_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=2, Hkv=1, grid=(1, 20, 33),
                                        coarse=(1, 5, 9), seed=14, q_blk=64, target="fixed"),
    # d = 64 (products of keys 0-63 issued before the rest of the softmax) with 64-row
    # query blocks, text prefix forced to level 0
    "bf16_d64_q64": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, grid=(1, 20, 38),
                                     coarse=(1, 5, 10), seed=18, q_blk=64, target="fixed"),
    # CUDA-core path, fp32, d = 128, 128-row query blocks
    "f32_d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=2, Hkv=2, dtype="f32",
                                 grid=(1, 18, 40), coarse=(1, 5, 10), seed=15, target="fixed"),
    # 150 KV blocks per row (N = 9541, ragged): the assignment's candidate cut
    # (a small tau_3, so only the top blocks are sorted)
    "bf16_cand": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=0, grid=(1, 47, 203),
                                  coarse=(1, 12, 51), forced_prefix_tokens=0, seed=16,
                                  target="alpha:0.15"),
    # the same length, causal with grouped queries, through the candidate cut
    "bf16_cand_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=2, Hkv=1, grid=(1, 47, 203),
                                         coarse=(1, 12, 51), seed=17, target="alpha:0.3"),
    # tau_3 = 1: every visible block is ranked, the full sort of the row
    "bf16_full_sort": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=0,
                                       grid=(1, 47, 203), coarse=(1, 12, 51),
                                       forced_prefix_tokens=0, seed=18, target="alpha:1.0"),
    # quantile rule (per-level quotas of blocks by rank): 16 blocks per row,
    # one per lane, with fractional quotas
    "f32_tiny_quantile": W.with_overrides(BASE["tiny_f32"], assign="quantile", seed=19),
    # quantile rule through the candidate cut (K_3 = 23 of 150), text prefix forced
    "bf16_quantile_cut": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=226,
                                          grid=(1, 42, 222), coarse=(1, 11, 56),
                                          forced_prefix_tokens=226, seed=20, target="alpha:0.15",
                                          assign="quantile"),
    # quantile rule, causal with grouped queries (quotas of each row's visible blocks)
    "bf16_quantile_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=2, Hkv=1, grid=(1, 47, 203),
                                             coarse=(1, 12, 51), seed=21, target="alpha:0.3",
                                             assign="quantile"),
    # quantile rule with tau_3 = 1: every visible block kept, the full sort
    "bf16_quantile_full": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=0,
                                           grid=(1, 47, 203), coarse=(1, 12, 51),
                                           forced_prefix_tokens=0, seed=22, target="alpha:1.0",
                                           assign="quantile"),
    # binary keep/drop (tau_0 = ... = tau_3: every kept block at level 0, the
    # baseline the method generalises), 150 blocks per row through the
    # candidate cut (small tau)
    "bf16_binary_cut": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=0,
                                        grid=(1, 47, 203), coarse=(1, 12, 51),
                                        forced_prefix_tokens=0, seed=24, target="binary:0.15"),
    # binary keep/drop, causal with grouped queries, through the candidate cut
    "bf16_binary_causal": W.with_overrides(BASE["qwen2.5_vl_7b"], Hq=2, Hkv=1, grid=(1, 47, 203),
                                           coarse=(1, 12, 51), seed=25, target="binary:0.3"),
    # binary keep/drop with tau = 1: every visible block kept at level 0 (dense
    # attention), the full sort of every row
    "bf16_binary_full": W.with_overrides(BASE["cogvideox_5b"], Hq=2, Hkv=2, n_text=0,
                                         grid=(1, 47, 203), coarse=(1, 12, 51),
                                         forced_prefix_tokens=0, seed=26, target="binary:1.0"),
}

_cache = {}


def setup(name):
    if name not in _cache:
        w = CASES[name]
        inp = W.make_inputs(w)
        heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
        ref = G.oracle_heads(w, inp, heads)
        run = G.run_stages(w, inp)
        _cache[name] = (w, inp, ref, run)
    return _cache[name]


@pytest.mark.parametrize("name", sorted(CASES))
def test_pyramid_levels(name):
    w, inp, _, run = setup(name)
    L = P.workspace_layout(run.p)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    for hk in range(w.Hkv):
        pyr = O.build_pyramid(inp.as_f64("k", 0, hk), inp.as_f64("v", 0, hk))
        for l in range(1, 4):
            shape = (w.B, w.Hkv, L["rows"][l], w.d)
            for key, ref in (("kp", pyr.keys[l]), ("vp", pyr.values[l])):
                got = G.to_f64(run.view(key, shape, tdt, l)[0, hk])
                tol = (2.0 ** -8 if w.dtype == "bf16" else 1e-6) * np.abs(ref) + 1e-6
                assert np.all(np.abs(got - ref) <= tol), (key, l, np.abs(got - ref).max())
        shape3 = (w.B, w.Hkv, L["rows"][3], w.d)
        head = run.view("k3h", shape3, torch.float32)[0, hk]
        tail = run.view("k3l", shape3, torch.float32)[0, hk]
        # the head is a tf32 value (low 13 mantissa bits clear); head + tail is
        # the fp32 level-3 key
        assert int((head.view(torch.int32) & 0x1FFF).abs().max()) == 0
        k3 = G.to_f64(head) + G.to_f64(tail)
        assert np.abs(k3 - pyr.keys[3]).max() <= 1e-5


@pytest.mark.parametrize("name", sorted(CASES))
def test_query_block_means(name):
    w, inp, ref, run = setup(name)
    L = P.workspace_layout(run.p)
    shape = (w.B, w.Hq, L["Nq"], w.d)
    head = run.view("qmh", shape, torch.float32)
    tail = run.view("qml", shape, torch.float32)
    assert int((head.view(torch.int32) & 0x1FFF).abs().max()) == 0
    qm = G.to_f64(head) + G.to_f64(tail)
    for (b, h), _ in ref.items():
        want = O.query_block_means(inp.as_f64("q", b, h), w.q_blk)
        assert np.abs(qm[b, h] - want).max() <= 1e-5 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("name", sorted(CASES))
def test_block_logits(name):
    w, inp, ref, run = setup(name)
    L = P.workspace_layout(run.p)
    z = G.to_f64(run.view("zlog", (w.B, w.Hq, L["Nq"], L["Nk"]), torch.float32))
    for (b, h), r in ref.items():
        vis = np.array([[O.visible(a, j, w.N, w.q_blk, w.kv_blk, w.causal) for j in range(L["Nk"])]
                        for a in range(L["Nq"])])
        err = np.abs(z[b, h] - r.z)[vis]
        assert err.max() <= 1e-4, err.max()


@pytest.mark.parametrize("name", sorted(CASES))
def test_level_map(name):
    w, inp, ref, run = setup(name)
    gm = run.level_map.cpu().numpy()
    tau = W.thresholds(w)
    for (b, h), r in ref.items():
        unexplained, thr, tie = G.map_mismatch_report(gm[b, h], r.mask, tau, w.assign)
        assert unexplained == 0, (b, h, unexplained, thr, tie)
        mass = G.to_f64(run.mass[b, h])
        assert np.abs(mass - r.mask.mass).max() <= 1e-5


@pytest.mark.parametrize("name", sorted(CASES))
def test_work_list_matches_map(name):
    w, inp, ref, run = setup(name)
    L = P.workspace_layout(run.p)
    Nq, Nk = L["Nq"], L["Nk"]
    gm = run.level_map.cpu().numpy()
    counts = run.view("counts", (w.B, w.Hq, Nq, 4), torch.int32).cpu().numpy()
    lst = run.view("list", (w.B, w.Hq, Nq, Nk), torch.int32).cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hq):
            for a in range(Nq):
                want = [j for l in range(4) for j in range(Nk) if gm[b, h, a, j] == l]
                n = [int((gm[b, h, a] == l).sum()) for l in range(4)]
                assert counts[b, h, a].tolist() == n
                assert lst[b, h, a, :len(want)].tolist() == want


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_on_oracle_map(name):
    """Attention alone: the kernel is fed the oracle's own map."""
    w, inp, ref, _ = setup(name)
    omap = np.zeros((w.B, w.Hq) + ref[(0, 0)].mask.level_map.shape, dtype=np.int8)
    for (b, h), r in ref.items():
        omap[b, h] = r.mask.level_map
    run = G.run_stages(w, inp, external_map=omap)
    gO, glse = G.to_f64(run.O), run.lse.cpu().numpy().astype(np.float64)
    for (b, h), r in ref.items():
        G.compare_out(gO[b, h], r.O, w.dtype)
        G.compare_lse(glse[b, h], r.lse, w.dtype)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("kind", ["random", "all_level3", "all_level0", "pruned_rows", "binary"])
def test_attention_on_external_maps(name, kind):
    w, inp, _, _ = setup(name)
    Nq, Nk = w.Nq, w.Nk
    rng = np.random.default_rng(zlib.crc32(f"{name}/{kind}".encode()))
    m = np.empty((w.B, w.Hq, Nq, Nk), dtype=np.int8)
    for b in range(w.B):
        for h in range(w.Hq):
            if kind == "random":
                m[b, h] = G.rand_map(rng, Nq, Nk)
            elif kind == "all_level3":
                m[b, h] = 3
            elif kind == "all_level0":
                m[b, h] = 0
            elif kind == "pruned_rows":
                m[b, h] = G.rand_map(rng, Nq, Nk, 0, 4)
                m[b, h, ::2] = -1
            else:
                m[b, h] = np.where(rng.random((Nq, Nk)) < 0.4, 0, -1)
    run = G.run_stages(w, inp, external_map=m)
    ref = G.oracle_heads(w, inp, [(0, h) for h in range(w.Hq)], level_map=m)
    gO, glse = G.to_f64(run.O), run.lse.cpu().numpy().astype(np.float64)
    for (b, h), r in ref.items():
        G.compare_out(gO[b, h], r.O, w.dtype)
        G.compare_lse(glse[b, h], r.lse, w.dtype)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_forward(name):
    """psa_forward end to end; its attention is checked against the oracle's
    attention on the map the GPU chose (map parity is checked above)."""
    w, inp, ref, _ = setup(name)
    run = G.run_stages(w, inp, fused=True)
    gm = run.level_map.cpu().numpy()
    tau = W.thresholds(w)
    for (b, h), r in ref.items():
        assert G.map_mismatch_report(gm[b, h], r.mask, tau, w.assign)[0] == 0
    ref_g = G.oracle_heads(w, inp, list(ref), level_map=gm)
    gO = G.to_f64(run.O)
    for (b, h), r in ref_g.items():
        G.compare_out(gO[b, h], r.O, w.dtype)


def test_quantile_long_rows_shared_memory_sort():
    """Rows of more than 1024 KV blocks sort in shared memory: the quantile
    rule there (one head, N = 66000: 1032 blocks per row), the map only."""
    w = W.with_overrides(BASE["cogvideox_5b"], Hq=1, Hkv=1, n_text=0, grid=(4, 110, 150),
                         coarse=(1, 28, 38), forced_prefix_tokens=0, seed=23,
                         target="alpha:0.2", assign="quantile")
    assert w.Nk == 1032
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp)
    gm = run.level_map.cpu().numpy()[0, 0]
    Q, K = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0)
    pyr = O.build_pyramid(K, K)
    z = O.block_logits(O.query_block_means(Q, w.q_blk), pyr, w.kv_blk, 1.0 / np.sqrt(w.d))
    mask = O.assign_levels(z, W.thresholds(w), w.N, w.q_blk, w.kv_blk, w.causal, 0, "quantile")
    assert G.map_mismatch_report(gm, mask, W.thresholds(w), "quantile")[0] == 0
    # every row keeps exactly K_3 blocks
    K3 = O.quotas(w.Nk, W.thresholds(w))[3]
    assert np.all((gm >= 0).sum(-1) == K3)


@pytest.mark.parametrize("assign", ["threshold", "quantile"])
@pytest.mark.parametrize("tau", [0.05, 1.0])
def test_long_rows_binary_and_quantile_shared_memory_path(assign, tau):
    """Rows of more than 1024 KV blocks (one head, N = 66000: 1032 blocks per
    row) sort in shared memory; binary keep/drop (tau_0 = ... = tau_3) through
    the candidate cut (tau = 0.05) and the full sort (tau = 1), under both
    rules.  The map against the oracle's."""
    w = W.with_overrides(BASE["cogvideox_5b"], Hq=1, Hkv=1, n_text=0, grid=(4, 110, 150),
                         coarse=(1, 28, 38), forced_prefix_tokens=0, seed=27,
                         target=f"binary:{tau}", assign=assign)
    assert w.Nk == 1032
    inp = W.make_inputs(w)
    run = G.run_stages(w, inp)
    gm = run.level_map.cpu().numpy()[0, 0]
    Q, K = inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0)
    pyr = O.build_pyramid(K, K)
    z = O.block_logits(O.query_block_means(Q, w.q_blk), pyr, w.kv_blk, 1.0 / np.sqrt(w.d))
    tau4 = W.thresholds(w)
    mask = O.assign_levels(z, tau4, w.N, w.q_blk, w.kv_blk, w.causal, 0, assign)
    assert G.map_mismatch_report(gm, mask, tau4, assign)[0] == 0
    assert set(np.unique(gm).tolist()) <= {-1, 0}
    if tau == 1.0:
        assert np.all(gm == 0)


@pytest.mark.parametrize("name", ["bf16_gqa_causal", "bf16_q64_causal"])
def test_causal_caller_map_is_corrected(name):
    """A caller's causal map that breaks the contract: future blocks at level 2,
    diagonal blocks at level 3, a value of 7 and one of -5.  The kernels attend
    to the corrected map (future blocks pruned, diagonal blocks at level 0,
    out-of-range values pruned), equal to the oracle's, and the error word
    reports the correction as PSA_ERR_LEVEL_MAP, which the check clears."""
    w, inp, _, _ = setup(name)
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    m = rng.integers(-1, 4, size=(w.B, w.Hq, w.Nq, w.Nk)).astype(np.int8)
    m[..., -1] = 2                            # the future of every query block but the last
    for a in range(w.Nq):                     # diagonal blocks at a pooled level
        for j in range(w.Nk):
            if O.straddles(a, j, w.N, w.q_blk, w.kv_blk):
                m[:, :, a, j] = 3
    m[0, 0, 1, 0], m[0, w.Hq - 1, 2, 1] = 7, -5
    p = G.params_for(w)
    ws = P.new_workspace(p)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    P.build_pyramid(p, k, v, ws)
    P.attention_fwd(p, q, k, v, ws, out, lse, torch.from_numpy(m).cuda())
    torch.cuda.synchronize()
    with pytest.raises(P.PSAError) as e:
        P.check_device(p, ws)
    assert e.value.status == 7
    P.check_device(p, ws)                     # cleared
    fixed = np.stack([np.stack([O.correct_map(m[b, h], w.N, w.q_blk, w.kv_blk, True)[0]
                                for h in range(w.Hq)]) for b in range(w.B)])
    assert int((fixed != m).sum()) > 0
    # the list the kernel built is the corrected map's
    counts = run_view(ws, p, "counts", (w.B, w.Hq, w.Nq, 4), torch.int32)
    lst = run_view(ws, p, "list", (w.B, w.Hq, w.Nq, w.Nk), torch.int32)
    for h in range(w.Hq):
        for a in range(w.Nq):
            want = [j for l in range(4) for j in range(w.Nk) if fixed[0, h, a, j] == l]
            assert counts[0, h, a].tolist() == [int((fixed[0, h, a] == l).sum()) for l in range(4)]
            assert lst[0, h, a, :len(want)].tolist() == want
    ref = G.oracle_heads(w, inp, [(0, h) for h in range(w.Hq)], level_map=m)
    gO, glse = G.to_f64(out), lse.cpu().numpy().astype(np.float64)
    for (b, h), r in ref.items():
        G.compare_out(gO[b, h], r.O, w.dtype)
        G.compare_lse(glse[b, h], r.lse, w.dtype)
    # a map that keeps the contract is not flagged
    P.attention_fwd(p, q, k, v, ws, out, lse, torch.from_numpy(fixed).cuda())
    torch.cuda.synchronize()
    P.check_device(p, ws)


def run_view(ws, p, key, shape, dtype):
    return P.workspace_view(ws, P.workspace_layout(p)[key], shape, dtype).cpu().numpy()


def test_no_device_timeouts_recorded():
    w, inp, _, run = setup("bf16_d128")
    P.check_device(run.p, run.ws)


@pytest.mark.parametrize("boost", [40.0, 600.0])
def test_attention_logit_jumps_across_tiles(boost):
    """A row's largest logits arrive on a later tile of its stream: keys of
    some coarser-level blocks are set to `boost` along the query direction
    (exact in bf16, and so are their pooled means), about +20 (boost 40: a
    rescale deferred to the stream's next tile) or about +300 (boost 600: past
    the direct-exponential range, so the tile half is redone after an
    immediate rescale, after the tile's first half of P was stored) in log2
    units.  External map: block j at level j // 8 (N = 2048, 32 blocks), so
    each query block has 8 tiles; the boosted blocks 10, 11 and 14, 15 fill
    the second halves of tiles 4 and 5 (one per stream), 30, 31 sit in tile 7."""
    N, d, bq, bk = 2048, 128, 128, 64
    rng = np.random.default_rng(41)
    Q = rng.standard_normal((N, d)) * 0.1
    Q[:, 0] += 4.0
    K = rng.standard_normal((N, d)) * 0.1
    V = rng.standard_normal((N, d))
    for j in (10, 11, 14, 15, 30, 31):
        K[j * bk:(j + 1) * bk, 0] = boost
    to_bf16 = lambda x: W.bf16_bits_to_f32(W.f32_to_bf16_bits(x.astype(np.float32))).astype(np.float64)
    Q, K, V = to_bf16(Q), to_bf16(K), to_bf16(V)
    Nq, Nk = N // bq, N // bk
    lm = np.repeat((np.arange(Nk) // 8).astype(np.int8)[None, :], Nq, axis=0)
    p = P.make_params(1, 1, 1, N, d, bq, bk)
    dev = lambda x: torch.from_numpy(W.f32_to_bf16_bits(x.astype(np.float32)).view(np.int16)) \
        .view(torch.bfloat16).reshape(1, 1, N, d).cuda()
    q, k, v = dev(Q), dev(K), dev(V)
    ws = P.new_workspace(p)
    out = torch.zeros_like(q)
    lse = torch.zeros((1, 1, N), dtype=torch.float32, device="cuda")
    P.build_pyramid(p, k, v, ws)
    P.attention_fwd(p, q, k, v, ws, out, lse, torch.from_numpy(lm[None, None]).cuda())
    torch.cuda.synchronize()
    P.check_device(p, ws)
    ref_O, ref_lse = O.pyramid_attention(Q, O.build_pyramid(K, V), lm, bq, bk, 1.0 / np.sqrt(d))
    G.compare_out(G.to_f64(out[0, 0]), ref_O, "bf16")
    G.compare_lse(lse[0, 0].cpu().numpy().astype(np.float64), ref_lse, "bf16")


SEQUENCE_CASES = {
    # d = 128, 128-row query blocks; N = 1000 (last query block 104 rows, last KV block 40)
    "d128": W.with_overrides(BASE["wan2.1_1.3b"], Hq=192, Hkv=192, grid=(1, 20, 50),
                             coarse=(1, 5, 13), seed=31, target="fixed"),
    # d = 64 (the split PV), N = 986
    "d64": W.with_overrides(BASE["cogvideox_5b"], Hq=192, Hkv=192, n_text=0, grid=(1, 29, 34),
                            coarse=(1, 8, 9), forced_prefix_tokens=0, seed=32, target="fixed"),
    # 64-row query blocks (rows 64-127 of each tile idle), grouped queries
    "q64_gqa": W.with_overrides(BASE["wan2.1_1.3b"], Hq=96, Hkv=48, grid=(1, 20, 50),
                                coarse=(1, 5, 13), seed=33, q_blk=64, target="fixed"),
}


@pytest.mark.parametrize("name", sorted(SEQUENCE_CASES))
def test_attention_block_sequences(name):
    """Each persistent CTA walks about ten query blocks in a row here, with tile
    counts from 0 to 8 in random order.  At the end of each block one softmax
    warpgroup hands its stream's (max, sum) to the other and starts the next
    block while the other writes O, through buffers and barriers that
    alternate by block; blocks without keys take no part in the alternation.
    Every row of every head against the oracle on the same map."""
    w = SEQUENCE_CASES[name]
    inp = W.make_inputs(w)
    rng = np.random.default_rng(zlib.crc32(f"sequences/{name}".encode()))
    m = np.stack([G.sequence_map(rng, w.Nq, w.Nk) for _ in range(w.B * w.Hq)])
    m = m.reshape(w.B, w.Hq, w.Nq, w.Nk)
    assert w.B * w.Hq * w.Nq >= 8 * 148
    run = G.run_stages(w, inp, external_map=m)
    ref = G.oracle_heads(w, inp, [(b, h) for b in range(w.B) for h in range(w.Hq)], level_map=m)
    gO, glse = G.to_f64(run.O), run.lse.cpu().numpy().astype(np.float64)
    for (b, h), r in ref.items():
        G.compare_out(gO[b, h], r.O, w.dtype)
        G.compare_lse(glse[b, h], r.lse, w.dtype)
