"""The backward-pass oracle against its pins (library autograd, finite
differences, exact invariants), and planted mistakes that the pins must
catch.  CPU only."""
import os
import sys
import types

import pytest

from oracle import psa_backward as OB
from tests import backward_pins as BP

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "psa_backward.py")

MUTATIONS = {
    "drops the D term": ("dX = P * (dP - Di[:, None])", "dX = P * dP"),
    "D from dO . dO": ("Di = (g * O).sum(axis=1)", "Di = (g * g).sum(axis=1)"),
    "unpool forgets the count": ("out[lo:hi] = g[r] / counts[r]", "out[lo:hi] = g[r]"),
    "dK forgets the scale": ("dKk = s * (dX.T @ Q[ri])", "dKk = (dX.T @ Q[ri])"),
    "dV from dX": ("dVk = P.T @ g", "dVk = dX.T @ g"),
    "dQ reads V": ("dQ[ri] = s * (dX @ Kk)", "dQ[ri] = s * (dX @ Vk)"),
    "level gradients land on level 0": ("dVl[l][r0:r1] += dVk[off:off + n]",
                                        "dVl[0][r0:r1] += dVk[off:off + n]"),
    "causal mask off by one": ("kpos_a[None, :] > rows_i[:, None]",
                               "kpos_a[None, :] >= rows_i[:, None]"),
    "bias dropped": ("+ bias_a[None, :]", ""),
    "grouped queries sum into the wrong KV head": ("dK[b, h // grp] += g.dK",
                                                   "dK[b, h % Hkv] += g.dK"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new).replace("from .psa_oracle import", "from oracle.psa_oracle import")
    name = "backward_mutant_%d" % abs(hash((old, new)))
    mod = types.ModuleType(name)
    sys.modules[name] = mod
    try:
        exec(compile(src, name, "exec"), mod.__dict__)
    finally:
        sys.modules.pop(name, None)
    return mod


@pytest.mark.parametrize("pin", BP.ALL_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    pin(OB)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_backward_mutation_is_caught(name):
    M = _mutant(*MUTATIONS[name])
    caught = []
    for pin in BP.ALL_PINS:
        try:
            pin(M)
        except Exception:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation '{name}'"
