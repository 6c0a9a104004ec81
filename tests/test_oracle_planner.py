"""Pins of the oracle's bounded greedy planner: hand-worked cases, the ILP constraints,
the two cases whose optimum is known in closed form (s = 0 and a non-binding budget), and
brute force over every feasible q on tiny instances; no GPU."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O


def _cases(golden_dir):
    with open(os.path.join(golden_dir, "planner_hand.json")) as fh:
        return json.load(fh)["cases"]


def test_hand_worked_cases(golden_dir):
    for case in _cases(golden_dir):
        for v, want in case["variants"].items():
            res = O.plan_variant(case["b"], case["P"], case["s"], int(v))
            assert res["q"].tolist() == want["q"], (case["name"], v)
            assert res["makespan"] == want["makespan"], (case["name"], v)
            assert res["replicas"] == want["replicas"], (case["name"], v)
            if "rounds" in want:
                assert res["rounds"] == want["rounds"], (case["name"], v)
        assert O.plan(case["b"], case["P"], case["s"])["variant"] == case["best"]


def _check_constraints(q, b, P, s):
    q = np.asarray(q)
    E = len(b)
    assert (q >= 0).all()
    assert q.sum(axis=1).tolist() == list(b)                      # sum_r q_er = b_e
    for r in range(P):
        remote = sum(1 for e in range(E) if O.owner(e, E, P) != r and q[e, r] > 0)
        assert remote <= s                                         # replica budget
    for e in range(E):                                             # only home blocks move
        for r in range(P):
            if q[e, r] > 0 and r != O.owner(e, E, P):
                assert q[e, r] <= b[e]


def _random_b(rng, E, scale):
    zipf = 1.0 / np.arange(1, E + 1) ** rng.uniform(0, 2)
    c = rng.multinomial(scale, zipf / zipf.sum())
    return [int(x) for x in c]


@pytest.mark.parametrize("E,P,s", [(8, 4, 1), (64, 8, 2), (128, 8, 2), (256, 8, 4), (12, 5, 3)])
def test_constraints_and_bounds_random(E, P, s):
    rng = np.random.default_rng(E * 100 + P)
    for _ in range(15):
        b = _random_b(rng, E, rng.integers(1, 40 * E))
        B = sum(b)
        tau = -(-B // P)
        fixed = O.fixed_makespan(b, P)
        for v in range(4):
            res = O.plan_variant(b, P, s, v)
            _check_constraints(res["q"], b, P, s)
            assert sum(res["load"]) == B
            assert res["q"].sum(axis=0).tolist() == res["load"]
            assert tau <= res["makespan"] <= fixed
            assert res["tau"] == tau and res["B"] == B
        greedy = min(O.plan_variant(b, P, s, v)["makespan"] for v in range(4))
        assert O.plan(b, P, s)["makespan"] == greedy          # default: the greedy searches
        assert O.plan(b, P, s, variant_mask=O.ALL_VARIANTS)["makespan"] == min(
            greedy, O.plan_quota(b, P, s)["makespan"])


def test_zero_budget_is_fixed_placement():
    rng = np.random.default_rng(7)
    for _ in range(20):
        E, P = 16, 4
        b = _random_b(rng, E, 300)
        for v in range(4):
            res = O.plan_variant(b, P, 0, v)
            want = np.zeros((E, P), np.int32)
            for e in range(E):
                want[e, O.owner(e, E, P)] = b[e]
            assert (res["q"] == want).all()
            assert res["makespan"] == O.fixed_makespan(b, P)


def test_non_binding_budget_reaches_tau():
    rng = np.random.default_rng(8)
    for E, P in [(8, 4), (64, 8), (128, 8), (256, 8)]:
        for _ in range(8):
            b = _random_b(rng, E, int(rng.integers(P, 30 * E)))
            tau = -(-sum(b) // P)
            for v in (1, 3):  # several copies per round: the budget s >= E never binds
                assert O.plan_variant(b, P, E, v)["makespan"] == tau
            # fan-out one also reaches tau, over more rounds
            assert O.plan_variant(b, P, E, 0)["makespan"] == tau


def _brute_force_optimum(b, P, s):
    E = len(b)

    def splits(n):
        for cut in itertools.combinations(range(n + P - 1), P - 1):
            parts, prev = [], -1
            for c in cut + (n + P - 1,):
                parts.append(c - prev - 1)
                prev = c
            yield parts

    best = None
    for rows in itertools.product(*(list(splits(x)) for x in b)):
        q = np.array(rows).reshape(E, P)
        ok = all(sum(1 for e in range(E) if O.owner(e, E, P) != r and q[e, r] > 0) <= s
                 for r in range(P))
        if ok:
            m = int(q.sum(axis=0).max())
            best = m if best is None else min(best, m)
    return best


def test_brute_force_tiny_instances():
    rng = np.random.default_rng(9)
    gaps = []
    for _ in range(150):
        E = int(rng.integers(2, 5))
        P = int(rng.integers(2, 4))
        s = int(rng.integers(0, 3))
        b = [int(x) for x in rng.integers(0, 4, size=E)]
        opt = _brute_force_optimum(b, P, s)
        res = O.plan(b, P, s)
        assert res["makespan"] >= opt
        assert res["makespan"] >= -(-sum(b) // P)
        gaps.append(res["makespan"] - opt)
        if s == 0:
            assert res["makespan"] == opt
    # the heuristic is not optimal everywhere, but it is on the vast majority
    assert np.mean(np.array(gaps) == 0) > 0.9


def test_variants_differ_on_real_shapes():
    # the four searches must really be different rules; on a skewed 128-expert route
    # the fan-out rule changes the result
    rng = np.random.default_rng(11)
    seen = set()
    for _ in range(30):
        b = _random_b(rng, 128, 9000)
        res = [O.plan_variant(b, 8, 2, v) for v in range(4)]
        seen.add(tuple(r["makespan"] for r in res))
        if res[0]["q"].tolist() != res[1]["q"].tolist():
            break
    else:
        pytest.fail("fan-out one and multi never differed")


def test_block_list_order_and_coverage():
    rng = np.random.default_rng(12)
    b = _random_b(rng, 64, 3000)
    res = O.plan(b, 8, 2)
    blocks, slot_off = O.block_list(res["q"])
    assert len(blocks) == sum(b) and slot_off[-1] == sum(b)
    assert sorted(blocks) == [(e, j) for e in range(64) for j in range(b[e])]
    for r in range(8):
        seg = blocks[slot_off[r]:slot_off[r + 1]]
        assert len(seg) == res["load"][r]
        assert [e for e, _ in seg] == sorted(e for e, _ in seg)   # experts ascending


def test_deterministic():
    rng = np.random.default_rng(13)
    b = _random_b(rng, 256, 20000)
    a1 = O.plan(b, 8, 4)
    a2 = O.plan(list(b), 8, 4)
    assert a1["q"].tobytes() == a2["q"].tobytes() and a1["variant"] == a2["variant"]
