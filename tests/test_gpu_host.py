"""psa_forward_host: the forward pass from pinned host buffers, with per-head-
group copies pipelined behind the kernels.  Its outputs must equal one
psa_forward over the whole problem bit for bit (every (batch, head) is
computed the same way whichever heads share a call)."""
import pytest
import torch

import level_sparse_attention_b200 as P
import workloads as W
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


def _case(name):
    if name == "gqa_causal_b2":       # 2 KV heads, 8 groups: each KV head's 4 query heads split
        return W.with_overrides(W.BY_NAME["qwen2.5_vl_7b"], B=2, Hq=8, Hkv=2, grid=(1, 25, 40),
                                coarse=(1, 7, 10), seed=33, target="fixed")
    return W.with_overrides(W.BY_NAME["wan2.1_1.3b"], Hq=12, Hkv=12, grid=(1, 20, 50),
                            coarse=(1, 5, 13), seed=34, target="fixed")


@pytest.mark.parametrize("name,groups", [("gqa_causal_b2", 8), ("gqa_causal_b2", 2),
                                         ("mha", 8), ("mha", 5), ("mha", 1)])
def test_forward_host_equals_forward(name, groups):
    w = _case(name)
    inp = W.make_inputs(w)
    whole = G.run_stages(w, inp, fused=True)
    p = G.params_for(w)
    host = lambda x: torch.from_numpy(x.view("int16")).view(torch.bfloat16).pin_memory()
    hq, hk, hv = host(inp.q), host(inp.k), host(inp.v)
    hout = torch.zeros(hq.shape, dtype=hq.dtype).pin_memory()
    hlse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32).pin_memory()
    q, k, v = (torch.empty(t.shape, dtype=t.dtype, device="cuda") for t in (hq, hk, hv))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    ws = P.new_workspace(p)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    P.forward_host(p, hq, hk, hv, hout, q, k, v, out, ws, h2d, d2h, hlse=hlse, lse=lse,
                   groups=groups)
    torch.cuda.synchronize()
    P.check_device(p, ws)
    assert torch.equal(hout, whole.O.cpu())
    assert torch.equal(hlse, whole.lse.cpu())
