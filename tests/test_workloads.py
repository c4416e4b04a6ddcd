"""The seeded input generator: shapes, determinism, and bf16 rounding (checked
against torch's own float32 -> bfloat16 conversion)."""
import numpy as np
import torch

import workloads as W


def test_shapes_match_the_workload_table():
    want = {"tiny_f32": 1024, "wan2.1_1.3b": 32760, "cogvideox_5b": 17776,
            "wan2.1_14b_720p": 75600, "qwen2.5_vl_7b": 16384}
    for w in W.WORKLOADS:
        assert w.N == want[w.name]
    assert W.BY_NAME["tiny_f32"].coarse == (1, 4, 4)
    assert W.BY_NAME["qwen2.5_vl_7b"].Hq // W.BY_NAME["qwen2.5_vl_7b"].Hkv == 7


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0], np.float32)])
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_generator_is_deterministic_and_smooth():
    w = W.BY_NAME["tiny_f32"]
    a = W.make_inputs(w)
    b = W.make_inputs(w)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.v, b.v)
    assert not np.array_equal(a.q, a.k)
    # neighbouring tokens along w share the field: correlation well above zero
    q = a.q[0, 0].astype(np.float64)
    corr = np.mean(np.sum(q[:-1] * q[1:], 1)) / np.mean(np.sum(q * q, 1))
    assert corr > 0.5
    sub = W.make_inputs(w, heads_q=[1], heads_kv=[1])
    assert np.array_equal(sub.q[0, 1], a.q[0, 1]) and np.all(sub.q[0, 0] == 0)


def test_text_prefix_is_iid():
    w = W.with_overrides(W.BY_NAME["cogvideox_5b"], Hq=1, Hkv=1, grid=(2, 4, 4), coarse=(1, 1, 1))
    x = W.head_values(w, 0, 0)
    assert x.shape == (226 + 32, 64)
