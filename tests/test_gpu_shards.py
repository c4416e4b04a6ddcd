"""Head-sharded forward (one problem's heads split among ranks): the shards,
run one after another on one GPU, give bit-identical outputs to the whole
forward pass, since every (batch, head) is computed the same way whichever
heads share a call.  The multi-process side (plan, oracle on shards) is
covered on the CPU by test_multirank_host.py."""
import pytest
import torch

import level_sparse_attention_b200 as P
import workloads as W
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", ["gqa_causal", "text_prefix"])
def test_head_shards_equal_whole_forward(case, world):
    if case == "gqa_causal":
        w = W.with_overrides(W.BY_NAME["qwen2.5_vl_7b"], B=2, Hq=8, Hkv=2, grid=(1, 25, 40),
                             coarse=(1, 7, 10), seed=31, target="fixed")
    else:
        w = W.with_overrides(W.BY_NAME["cogvideox_5b"], Hq=4, Hkv=4, grid=(1, 20, 38),
                             coarse=(1, 5, 10), seed=32, target="fixed")
    inp = W.make_inputs(w)
    whole = G.run_stages(w, inp, fused=True)
    p = G.params_for(w)
    q, k, v = (G.to_device(x, w.dtype) for x in (inp.q, inp.k, inp.v))
    out = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    for rank in range(world):
        P.psa_forward_heads(q, k, v, out, lse, p, rank, world)
    torch.cuda.synchronize()
    assert torch.equal(out, whole.O)
    assert torch.equal(lse, whole.lse)
