"""Pins of the oracle's quota solver (the UltraEP notes' Algorithm 1, planner variant 4):
hand-worked cases, the plan's constraints, the search's end point, the closed form of a
single hot expert, and the zero-budget and balanced special cases; no GPU."""
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O


def _cases(golden_dir):
    with open(os.path.join(golden_dir, "quota_hand.json")) as fh:
        return json.load(fh)["cases"]


def test_hand_worked_cases(golden_dir):
    for case in _cases(golden_dir):
        res = O.plan_quota(case["b"], case["P"], case["s"], case["u_min"])
        assert res["q"].tolist() == case["q"], case["name"]
        for key in ("makespan", "replicas", "tau_star", "rounds"):
            assert res[key] == case[key], (case["name"], key)


def _random_b(rng, E, scale):
    zipf = 1.0 / np.arange(1, E + 1) ** rng.uniform(0, 2)
    return [int(x) for x in rng.multinomial(scale, zipf / zipf.sum())]


@pytest.mark.parametrize("E,P,s,u_min", [(8, 4, 1, 1), (64, 8, 2, 1), (128, 8, 2, 3),
                                         (256, 8, 4, 1), (12, 5, 3, 2), (7, 1, 2, 1)])
def test_constraints_and_search_end(E, P, s, u_min):
    rng = np.random.default_rng(E * 10 + P + u_min)
    for _ in range(15):
        b = _random_b(rng, E, int(rng.integers(1, 40 * E)))
        B = sum(b)
        res = O.plan_quota(b, P, s, u_min)
        q = res["q"]
        h = [O.owner(e, E, P) for e in range(E)]
        assert (q >= 0).all() and q.sum(axis=1).tolist() == b     # sum_r u_er = b_e
        assert q.sum(axis=0).tolist() == res["load"] and sum(res["load"]) == B
        for r in range(P):                                         # N_slot per rank
            assert sum(1 for e in range(E) if h[e] != r and q[e, r] > 0) <= s
        for e in range(E):
            remote = [r for r in range(P) if r != h[e] and q[e, r] > 0]
            assert len(remote) <= 1                                # one transfer per expert
            assert all(q[e, r] >= u_min for r in remote)           # the quota floor
        lo, fixed = -(-B // P), O.fixed_makespan(b, P)
        assert lo <= res["makespan"] <= res["tau_star"] <= fixed
        assert res["tau"] == lo and res["B"] == B
        assert res["rounds"] <= (math.ceil(math.log2(fixed - lo + 1)) if fixed > lo else 0)
        # the search ends on a threshold the oracle satisfies, just above one it does not
        assert O.quota_feasible(b, P, s, u_min, res["tau_star"])["feasible"]
        if res["tau_star"] > lo:
            assert not O.quota_feasible(b, P, s, u_min, res["tau_star"] - 1)["feasible"]


@pytest.mark.parametrize("m", [1, 2, 3, 7, 10, 101, 256])
@pytest.mark.parametrize("u_min", [1, 3])
def test_single_hot_expert_closed_form(m, u_min):
    # one loaded expert on slot 0 of P = E = 4 slots: one transfer of delta = m - tau to
    # the emptiest slot is feasible iff delta <= tau (slack) and delta >= u_min (or
    # delta = 0), so tau* = ceil(m / 2) when m - ceil(m / 2) >= u_min, else m (no split)
    b = [m, 0, 0, 0]
    res = O.plan_quota(b, 4, 2, u_min)
    half = -(-m // 2)
    want = half if (m - half >= u_min or m - half == 0) else m
    assert res["tau_star"] == want and res["makespan"] == want
    assert res["replicas"] == (1 if want < m else 0)


def test_zero_budget_is_fixed_placement():
    rng = np.random.default_rng(7)
    for _ in range(20):
        b = _random_b(rng, 16, 300)
        res = O.plan_quota(b, 4, 0)
        assert res["replicas"] == 0 and res["makespan"] == O.fixed_makespan(b, 4)
        for e in range(16):
            assert res["q"][e, O.owner(e, 16, 4)] == b[e]


def test_balanced_homes_need_no_search():
    b = [5] * 32
    res = O.plan_quota(b, 8, 2)
    assert res["rounds"] == 0 and res["replicas"] == 0 and res["makespan"] == 20


def test_plan_picks_among_five_variants():
    rng = np.random.default_rng(21)
    picked = set()
    for _ in range(60):
        b = _random_b(rng, 64, int(rng.integers(50, 4000)))
        s = int(rng.integers(0, 4))
        allres = O.plan(b, 8, s, variant_mask=O.ALL_VARIANTS)
        assert O.plan(b, 8, s)["variant"] < 4  # the default is the four greedy searches
        greedy = [O.plan_variant(b, 8, s, v) for v in range(4)]
        quota = O.plan_quota(b, 8, s)
        key = lambda r: (r["makespan"], r["replicas"], r["variant"])
        assert allres["variant"] == min(greedy + [quota], key=key)["variant"]
        assert O.plan(b, 8, s, variant_mask=0x10)["q"].tolist() == quota["q"].tolist()
        picked.add(allres["variant"])
    assert O.QUOTA_VARIANT in picked  # the quota solver wins some of these plans
