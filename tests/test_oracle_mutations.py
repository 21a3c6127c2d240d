"""Plant plausible mistakes in the oracle's transition (on the CPU, in a patched copy) and check
that the hand-worked examples and the defining properties reject every one of them."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import gdn_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _mutants():
    def transposed(S, k, v, a, b):       # writes k v^T instead of v k^T (square states)
        u = S @ k
        return a * (S - b * np.outer(u, k)) + b * np.outer(k, v)

    def no_alpha_on_erase(S, k, v, a, b):
        u = S @ k
        return a * S - b * np.outer(u, k) + b * np.outer(v, k)

    def alpha_on_write(S, k, v, a, b):
        u = S @ k
        return a * (S - b * np.outer(u, k)) + a * b * np.outer(v, k)

    def sign_flip(S, k, v, a, b):
        u = S @ k
        return a * (S + b * np.outer(u, k)) + b * np.outer(v, k)

    def dropped_write(S, k, v, a, b):
        u = S @ k
        return a * (S - b * np.outer(u, k))

    def wrong_projection(S, k, v, a, b):
        u = S.T @ k[: S.shape[0]] if S.shape[0] == S.shape[1] else S @ k
        return a * (S - b * np.outer(u, k)) + b * np.outer(v, k)

    return {"transposed": transposed, "no_alpha_on_erase": no_alpha_on_erase,
            "alpha_on_write": alpha_on_write, "sign_flip": sign_flip,
            "dropped_write": dropped_write, "wrong_projection": wrong_projection}


def _golden_fails():
    for case in json.load(open(GOLDEN))["cases"]:
        f = lambda a: np.array([[float(Fraction(x)) for x in row] for row in a])
        steps = case["steps"]
        q = np.stack([f(s["q"]) for s in steps])
        k = np.stack([f(s["k"]) for s in steps])
        v = np.stack([f(s["v"]) for s in steps])
        al = np.stack([[float(Fraction(a)) for a in s["alpha"]] for s in steps])
        be = np.stack([[float(Fraction(a)) for a in s["beta"]] for s in steps])
        par = np.array([s["parents"] for s in steps], dtype=np.int32)
        exp = np.stack([f(s["o"]) for s in steps])
        o = oracle.full_state_decode(f(case["S_ctx"]), q, k, v, np.log(al), be, par)
        if not np.allclose(o, exp, rtol=0, atol=1e-12):
            return True
    return False


def _property_fails():
    rng = np.random.default_rng(1)
    S = rng.standard_normal((5, 5))
    k = rng.standard_normal(5)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(5)
    a, b = 0.6, 0.3
    S1 = gdn_oracle.gdn_transition(S, k, v, a, b)
    if not np.allclose(S1 @ k, a * (1 - b) * (S @ k) + b * v, atol=1e-12):
        return True
    x = rng.standard_normal(5)
    x -= (x @ k) * k
    return not np.allclose(S1 @ x, a * (S @ x), atol=1e-12)


@pytest.mark.parametrize("name", list(_mutants()))
def test_pins_reject_mutant(name, monkeypatch):
    monkeypatch.setattr(gdn_oracle, "gdn_transition", _mutants()[name])
    assert _golden_fails() or _property_fails(), f"mutant {name} slipped through"


def test_pins_accept_original():
    assert not _golden_fails() and not _property_fails()


def _ancestry_mutants():
    original = gdn_oracle.ancestry_table

    def first_request_only(parents):        # every request takes request 0's parents
        T, R, B = parents.shape
        out = np.zeros((R, B, T), dtype=np.int32)
        for r in range(R):
            out[r] = np.array(gdn_oracle.chains(parents[:, 0])[T - 1], dtype=np.int32)
        return out

    def slots_reversed(parents):             # newest record first
        return original(parents)[:, :, ::-1]

    def own_index_everywhere(parents):       # beam b at every slot: parents never followed
        T, R, B = parents.shape
        out = np.zeros((R, B, T), dtype=np.int32)
        out[:] = np.arange(B, dtype=np.int32)[None, :, None]
        return out

    return {"first_request_only": first_request_only, "slots_reversed": slots_reversed,
            "own_index_everywhere": own_index_everywhere}


@pytest.mark.parametrize("name", list(_ancestry_mutants()))
def test_ancestry_pin_rejects_mutant(name, monkeypatch):
    import test_oracle_pins as pins
    monkeypatch.setattr(oracle, "ancestry_table", _ancestry_mutants()[name])
    with pytest.raises(AssertionError):
        pins.test_ancestry_table_by_walking_parent_pointers()


def test_ancestry_pin_accepts_original():
    import test_oracle_pins as pins
    pins.test_ancestry_table_by_walking_parent_pointers()
