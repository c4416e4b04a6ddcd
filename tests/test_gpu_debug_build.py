"""The PSA_DEBUG build (libpsa_debug.so): device-side bounds checks of the
work lists, reported through the error word, never a trap.

A workspace whose work list was corrupted between calls (an entry past the
last KV block, counts adding up to more than the row holds, entries out of
order) is fed to psa_attention_fwd and psa_backward with level_map = NULL,
through the debug library only.  The corrupted query blocks are skipped (O = 0,
lse = -inf, no gradient), psa_check_device returns PSA_ERR_DEVICE_BOUNDS, and
every other query block equals the oracle.  The release library is never given
a corrupted list."""
import ctypes

import numpy as np
import pytest
import torch

import level_sparse_attention_b200 as P
import oracle as O
import workloads as W
from oracle import psa_backward as OB
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

W_CASE = W.with_overrides(W.BY_NAME["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 20, 50),
                          coarse=(1, 5, 13), seed=71, target="fixed")
BAD_ROWS = (3, 5, 7)                       # query blocks of head 0
PSA_ERR_DEVICE_BOUNDS = 8


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _st():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _corrupt(p, ws, Nq, Nk):
    L = P.workspace_layout(p)
    counts = P.workspace_view(ws, L["counts"], (p.B * p.Hq * Nq, 4), torch.int32)
    lst = P.workspace_view(ws, L["list"], (p.B * p.Hq * Nq, Nk), torch.int32)
    a, b, c = BAD_ROWS
    assert int(counts[a].sum()) >= 3 and int(counts[c, 0]) >= 2
    lst[a, 1] = Nk + 5                                  # past the last KV block
    counts[b] = torch.tensor([Nk, Nk, 0, 0], dtype=torch.int32)   # more entries than the row
    lst[c, 0], lst[c, 1] = lst[c, 1].clone(), lst[c, 0].clone()   # level 0 out of order
    torch.cuda.synchronize()


def test_corrupted_list_is_skipped_and_reported():
    w = W_CASE
    inp = W.make_inputs(w)
    p = G.params_for(w)
    D = P.debug_lib()
    ws = P.new_workspace(p)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    lm = torch.empty(P.map_shape(p), dtype=torch.int8, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    n = ws.numel()
    assert D.psa_build_pyramid(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(ws), n, _st()) == 0
    assert D.psa_score_and_mask(ctypes.byref(p), _ptr(q), _ptr(ws), n, _ptr(lm), None, _st()) == 0
    torch.cuda.synchronize()
    assert D.psa_check_device(ctypes.byref(p), _ptr(ws), n, _st()) == 0
    _corrupt(p, ws, w.Nq, w.Nk)
    assert D.psa_attention_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws), n, None,
                               _ptr(out), _ptr(lse), _st()) == 0
    torch.cuda.synchronize()
    assert D.psa_check_device(ctypes.byref(p), _ptr(ws), n, _st()) == PSA_ERR_DEVICE_BOUNDS
    assert D.psa_check_device(ctypes.byref(p), _ptr(ws), n, _st()) == 0     # cleared
    gm = lm.cpu().numpy()
    gO, glse = G.to_f64(out), lse.cpu().numpy().astype(np.float64)
    for h in range(w.Hq):
        sub = gm[0, h].copy()
        if h == 0:
            sub[list(BAD_ROWS)] = -1                   # skipped blocks: O = 0, lse = -inf
        ref = O.psa_head(inp.as_f64("q", 0, h), inp.as_f64("k", 0, h), inp.as_f64("v", 0, h),
                         w.q_blk, w.kv_blk, W.thresholds(w), level_map=sub)
        G.compare_out(gO[0, h], ref.O, w.dtype)
        G.compare_lse(glse[0, h], ref.lse, w.dtype)

    # the backward pass walks the same (sanitised) list: the skipped blocks
    # pass no gradient, and the rest equals the oracle on that map
    g = np.random.default_rng(5).standard_normal((w.B, w.Hq, w.N, w.d)).astype(np.float32)
    bits = W.f32_to_bf16_bits(g)
    dO, dO64 = G.to_device(bits, "bf16"), W.bf16_bits_to_f32(bits).astype(np.float64)
    # a fresh list from the mask stage, corrupted again
    assert D.psa_score_and_mask(ctypes.byref(p), _ptr(q), _ptr(ws), n, _ptr(lm), None, _st()) == 0
    _corrupt(p, ws, w.Nq, w.Nk)
    dQ, dK, dV = (torch.full_like(t, float("nan")) for t in (q, k, v))
    bws = P.new_backward_workspace(p)
    assert D.psa_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                          _ptr(dO), None, _ptr(ws), n, _ptr(bws), bws.numel(), _ptr(dQ), _ptr(dK),
                          _ptr(dV), _st()) == 0
    torch.cuda.synchronize()
    assert D.psa_check_device(ctypes.byref(p), _ptr(ws), n, _st()) == PSA_ERR_DEVICE_BOUNDS
    sub = gm.copy()
    sub[0, 0, list(BAD_ROWS)] = -1
    Q, K, V = (np.stack([np.stack([inp.as_f64(nm, 0, h) for h in range(w.Hq)])])
               for nm in ("q", "k", "v"))
    ref = OB.psa_backward(Q, K, V, dO64, sub, w.q_blk, w.kv_blk)
    for got, want in ((dQ, ref.dQ), (dK, ref.dK), (dV, ref.dV)):
        got = G.to_f64(got)
        err = np.abs(got - want)
        assert np.all(np.isfinite(got))
        assert err.max() <= 3e-2 * np.abs(want).max() and err.mean() <= 1e-2 * np.abs(want).mean()
    for a in BAD_ROWS:
        assert bool((dQ[0, 0, a * w.q_blk:(a + 1) * w.q_blk] == 0).all())

    # a clean list afterwards: no report
    assert D.psa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), None,
                         _ptr(ws), n, _st()) == 0
    torch.cuda.synchronize()
    assert D.psa_check_device(ctypes.byref(p), _ptr(ws), n, _st()) == 0
