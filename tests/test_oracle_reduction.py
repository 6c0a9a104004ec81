"""Pins of the oracle's reduction-aware planner (the MegaFlux summary's C_lambda proxy):
hand-computed trajectories, the proxy's closed forms, and its limits lambda = 0 and
lambda beyond the fixed-placement makespan; no GPU."""
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O


def test_hand_computed_cases(golden_dir):
    with open(os.path.join(golden_dir, "reduction_hand.json")) as fh:
        cases = json.load(fh)["cases"]
    for case in cases:
        for lam, spec in case["lambdas"].items():
            lam = int(lam)
            for v, want in spec["variants"].items():
                res = O.plan_variant(case["b"], case["P"], case["s"], int(v), lam)
                assert res["q"][0].tolist() == want["q0"], (case["name"], lam, v)
                if "q1" in want:
                    assert res["q"][1].tolist() == want["q1"], (case["name"], lam, v)
                for key in ("cost", "makespan", "replicas", "rounds"):
                    assert res[key] == want[key], (case["name"], lam, v, key)
            assert O.plan(case["b"], case["P"], case["s"], lam=lam)["variant"] == spec["best"]


def test_cost_closed_forms():
    # home placement: no replica, C = the fixed-placement makespan for every lambda
    b = [5, 1, 0, 2, 7, 3]
    home = np.zeros((6, 3), np.int32)
    for e in range(6):
        home[e, O.owner(e, 6, 3)] = b[e]
    for lam in (0, 1, 12, 1000):
        assert O.reduction_cost(home, 3, lam) == O.fixed_makespan(b, 3)
    # E = 4 on P = 3 (h = [0, 0, 1, 2]): e0 copied to slot 1, e1 to slot 2, so n = [2, 0, 0],
    # loads [3, 4, 4]
    q = np.array([[1, 2, 0], [2, 0, 2], [0, 2, 0], [0, 0, 2]])
    assert O.reduction_cost(q, 3, 0) == 4
    assert O.reduction_cost(q, 3, 1) == max(3 + 2, 4, 4)
    assert O.reduction_cost(q, 3, 12) == 3 + 24


def _random_b(rng, E, scale):
    zipf = 1.0 / np.arange(1, E + 1) ** rng.uniform(0, 2)
    return [int(x) for x in rng.multinomial(scale, zipf / zipf.sum())]


@pytest.mark.parametrize("E,P,s", [(8, 4, 1), (64, 8, 2), (128, 8, 2), (256, 8, 4)])
def test_limits_and_monotonicity(E, P, s):
    rng = np.random.default_rng(E + P + s)
    for _ in range(8):
        b = _random_b(rng, E, int(rng.integers(P, 30 * E)))
        fixed = O.fixed_makespan(b, P)
        for v in range(4):
            plain = O.plan_variant(b, P, s, v)
            zero = O.plan_variant(b, P, s, v, 0)
            # lambda = 0: C is the makespan, which the search never raises, so the result
            # reaches the plain makespan, at its first plan doing so
            assert zero["makespan"] == plain["makespan"] == zero["cost"]
            assert zero["replicas"] <= plain["replicas"]
            # a copy costing more than the whole fixed makespan never pays
            big = O.plan_variant(b, P, s, v, fixed + 1)
            assert big["replicas"] == 0 and big["cost"] == fixed
            # C of the returned plan is its own C, and it never rises with lambda
            costs = []
            for lam in (0, 1, 3, 12, 40):
                r = O.plan_variant(b, P, s, v, lam)
                assert r["cost"] == O.reduction_cost(r["q"], P, lam)
                assert r["cost"] <= O.reduction_cost(plain["q"], P, lam)
                assert r["cost"] <= fixed
                assert r["q"].sum(axis=1).tolist() == b
                costs.append(r["cost"])
            assert costs == sorted(costs)
