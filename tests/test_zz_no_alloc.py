"""psa_forward_noalloc: the allocation-free forward pass.

It serves callers that may not allocate device memory while they run (a host
framework that plans memory ahead and gives a plugin only its inputs and
outputs, or a loop that cannot afford cudaMalloc's device-wide
synchronisation).  Its scratch is a 32 MiB device array inside the library,
so the GPU test checks, through the C ABI, that two calls in a row (the second
one finding the first one's leftovers in that array) give the same outputs as
psa_forward with a caller-provided workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import level_sparse_attention_b200 as P
import workloads as W
from tests import gpu_common as G


def _call(p, q, k, v, o, lse, lm):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return P.lib().psa_forward_noalloc(ctypes.byref(p), ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse),
                                       ptr(lm), stream)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # Wan2.1-1.3B shape: 217 MB of scratch > 32 MiB; rejected before any CUDA call
    big = P.make_params(1, 12, 12, 32760, 128)
    assert P.workspace_size(big) > 32 << 20
    A = ctypes.c_void_p(0x10000)
    st = P.lib().psa_forward_noalloc(ctypes.byref(big), A, A, A, A, None, None, None)
    assert st == 4, P.status_string(st)                      # PSA_ERR_WORKSPACE_TOO_SMALL
    bad = P.make_params(1, 12, 12, 32760, 96)
    assert P.lib().psa_forward_noalloc(ctypes.byref(bad), A, A, A, A, None, None, None) == 2


CASES = [
    W.with_overrides(W.BY_NAME["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 20, 50), coarse=(1, 5, 13),
                     seed=41, target="fixed"),
    W.with_overrides(W.BY_NAME["qwen2.5_vl_7b"], Hq=4, Hkv=2, grid=(1, 24, 40), coarse=(1, 6, 10),
                     seed=42, target="fixed"),
]


@pytest.mark.gpu
def test_noalloc_matches_psa_forward_twice_in_a_row():
    for w in CASES:                       # two calls in a row, different problems
        inp = W.make_inputs(w)
        p = G.params_for(w)
        assert P.workspace_size(p) <= 32 << 20
        q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
        shape = P.map_shape(p)
        o_ref, o_na = torch.empty_like(q), torch.full_like(q, float("nan"))
        lse_ref = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
        lse_na = torch.full_like(lse_ref, float("nan"))
        lm_ref = torch.empty(shape, dtype=torch.int8, device="cuda")
        lm_na = torch.full(shape, -7, dtype=torch.int8, device="cuda")
        ws = P.new_workspace(p)
        P.forward(p, q, k, v, o_ref, ws, lse_ref, lm_ref)
        assert _call(p, q, k, v, o_na, lse_na, lm_na) == 0
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bits, so a region of
        # the shared array that a call failed to rewrite would show
        assert torch.equal(lm_na, lm_ref)
        assert torch.equal(o_na, o_ref)
        assert torch.equal(lse_na, lse_ref)
