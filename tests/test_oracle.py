"""The fp64 oracle against its pins (no GPU needed)."""

import pytest

from oracle import infini_ref
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    fails = pin(infini_ref)
    assert not fails, "\n".join(fails)


def test_hand_examples_through_brute_force():
    """The token-loop evaluations reproduce the hand-worked examples too."""
    import json
    import os

    import numpy as np

    from oracle import brute

    with open(os.path.join(oracle_pins.GOLDEN, "hand_examples.json")) as f:
        data = json.load(f)
    for ex in data["examples"]:
        q = [[[[oracle_pins._expr(x) for x in row] for row in ex["q"]]]]
        k = [[[[oracle_pins._expr(x) for x in row] for row in ex["k"]]]]
        v = [[[[oracle_pins._expr(x) for x in row] for row in ex["v"]]]]
        beta = [oracle_pins._expr(ex["beta"])]
        want = np.array([[oracle_pins._frac(x) for x in r] for r in ex["out"]])
        out, M, _ = brute.forward_linear_closed_form(q, k, v, beta, ex["N"])
        assert np.allclose(np.array(out[0][0]), want, atol=1e-12, rtol=0)
        wantM = np.array([[oracle_pins._frac(x) for x in r] for r in ex["linear"]["M"]])
        assert np.allclose(np.array(M[0][0]), wantM, atol=1e-12, rtol=0)
        out, M, _ = brute.forward_delta_loops(q, k, v, beta, ex["N"])
        assert np.allclose(np.array(out[0][0]), want, atol=1e-12, rtol=0)
        wantM = np.array([[oracle_pins._frac(x) for x in r] for r in ex["delta"]["M"]])
        assert np.allclose(np.array(M[0][0]), wantM, atol=1e-12, rtol=0)


def test_empty_memory_retrieval_is_zero():
    """Reading for the first segment: a zero denominator retrieves the zero row."""
    import numpy as np

    sq = np.ones((3, 4))
    r = infini_ref.memory_retrieval(sq, np.ones((4, 2)), np.zeros(4))
    assert np.all(r == 0.0)
