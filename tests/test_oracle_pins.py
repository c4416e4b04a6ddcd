"""The CPU oracle against its pins (closed forms, library routines, invariants,
hand-worked cases, scalar brute force).  CPU only."""
import math

import numpy as np
import pytest

import oracle as O
from tests import oracle_pins as P
from tests.bruteforce import psa_bruteforce


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O)


@pytest.mark.parametrize("rule", ["threshold", "quantile"])
@pytest.mark.parametrize("N,d,bq,causal,forced", [
    (256, 8, 64, False, 0), (200, 8, 64, False, 70), (256, 4, 128, True, 0),
    (184, 8, 64, True, 0), (64, 8, 64, False, 0), (9, 4, 64, False, 0)])
def test_bruteforce_matches_oracle(N, d, bq, causal, forced, rule):
    rng = np.random.default_rng(N + d)
    Q, K, V = (rng.standard_normal((N, d)) * 1.5 for _ in range(3))
    tau = (0.5, 0.7, 0.85, 0.95) if rule == "threshold" else (0.2, 0.4, 0.6, 0.8)
    O_b, lse_b, lv_b = psa_bruteforce(Q.tolist(), K.tolist(), V.tolist(), bq, 64, tau,
                                      causal, forced, rule=rule)
    r = O.psa_head(Q, K, V, bq, 64, tau, causal, forced, rule=rule)
    assert r.mask.level_map.tolist() == lv_b
    assert np.allclose(r.O, np.array(O_b), atol=1e-12)
    assert np.allclose(r.lse, np.array(lse_b), atol=1e-12)


def test_forward_gqa_routes_kv_heads():
    """Query head h reads KV head h // (Hq / Hkv)."""
    rng = np.random.default_rng(1)
    B, Hq, Hkv, N, d = 1, 4, 2, 128, 8
    Q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    r = O.psa_forward(Q, K, V, 64, 64, (0.5, 0.7, 0.9, 0.95))
    for h in range(Hq):
        one = O.psa_head(Q[0, h], K[0, h // 2], V[0, h // 2], 64, 64, (0.5, 0.7, 0.9, 0.95))
        assert np.array_equal(r.O[0, h], one.O)


def test_executed_flops_dense_and_causal():
    N, d, bq, bk = 1000, 8, 128, 64
    Nq, Nk = -(-N // bq), -(-N // bk)
    assert O.executed_flops(np.zeros((Nq, Nk), np.int8), N, d, bq, bk) == 4 * d * N * N
    lmc = np.array([[0 if O.visible(a, j, N, bq, bk, True) else -1 for j in range(Nk)]
                    for a in range(Nq)], dtype=np.int8)
    assert O.executed_flops(lmc, N, d, bq, bk, causal=True) == 4 * d * N * (N + 1) / 2
    lm3 = np.full((Nq, Nk), 3, np.int8)
    # every level-3 block of 64 tokens keeps 8 keys; the 40-token tail keeps 5
    assert O.executed_flops(lm3, N, d, bq, bk) == 4 * d * N * (8 * 15 + 5)
