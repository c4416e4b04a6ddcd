"""Failure detection on the GPU without a fault.

Every mbarrier wait in the tensor-core kernels is bounded; a wait that runs
out records a timeout in the workspace's error word, the kernel winds down,
and psa_check_device reports PSA_ERR_DEVICE_TIMEOUT.  The self-test entry
point makes such a wait run out (a barrier nothing arrives at, a 20 ms limit)
through the same wait code; these tests check that the host sees the status,
that the check clears it, and that the context stays usable: a forward pass
right after it runs and matches the oracle-checked output of a clean run.
"""
import time

import numpy as np
import pytest
import torch

import level_sparse_attention_b200 as P
import workloads as W
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

TIMEOUT = 6   # PSA_ERR_DEVICE_TIMEOUT


def _case():
    w = W.with_overrides(W.BY_NAME["wan2.1_1.3b"], Hq=2, Hkv=2, grid=(1, 20, 50),
                         coarse=(1, 5, 13), seed=11, target="fixed")
    return w, G.params_for(w)


def test_wait_that_runs_out_is_reported_and_cleared():
    w, p = _case()
    ws = P.new_workspace(p)
    P.check_device(p, ws)                          # clean to begin with
    t0 = time.perf_counter()
    P.selftest_wait_timeout(p, ws, 20_000_000)     # 20 ms
    with pytest.raises(P.PSAError) as e:
        P.check_device(p, ws)
    elapsed = time.perf_counter() - t0
    assert e.value.status == TIMEOUT
    assert 0.015 < elapsed < 5.0                   # the wait ran out on its own limit
    P.check_device(p, ws)                          # the check cleared the word


def test_context_usable_after_a_timeout():
    w, p = _case()
    inp = W.make_inputs(w)
    clean = G.run_stages(w, inp, fused=True)
    ws = P.new_workspace(p)
    P.selftest_wait_timeout(p, ws, 10_000_000)
    with pytest.raises(P.PSAError):
        P.check_device(p, ws)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    P.forward(p, q, k, v, out, ws, lse)
    torch.cuda.synchronize()
    P.check_device(p, ws)
    assert torch.equal(out, clean.O)
    assert torch.equal(lse, clean.lse)


def test_selftest_rejects_bad_arguments():
    w, p = _case()
    ws = P.new_workspace(p)
    for limit in (0, 2_000_000_000):
        with pytest.raises(P.PSAError) as e:
            P.selftest_wait_timeout(p, ws, limit)
        assert e.value.status == 1                 # PSA_ERR_INVALID_ARG
    with pytest.raises(P.PSAError) as e:
        P.selftest_wait_timeout(p, ws[: ws.numel() // 2], 1000)
    assert e.value.status == 4                     # PSA_ERR_WORKSPACE_TOO_SMALL
