"""Pins of the oracle's routing stages (top-k, gates, histogram, kappa, blocks) against
closed forms, brute force and hand-worked values; no GPU."""
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "routing_closed_forms.json")) as fh:
        return json.load(fh)


def test_topk_golden(golden_dir):
    for case in _golden(golden_dir)["topk"]:
        ids, gates = O.route_topk(np.array([case["logits"]], np.float32), case["k"])
        assert ids[0].tolist() == case["ids"], case["why"]
        np.testing.assert_allclose(gates[0], case["gates"], rtol=1e-7, err_msg=case["why"])


def test_topk_matches_brute_force_sort():
    rng = np.random.default_rng(1)
    for E, k in [(8, 2), (64, 8), (128, 8), (256, 8), (5, 5)]:
        L = rng.standard_normal((40, E)).astype(np.float32)
        L[:, 3] = L[:, 1]  # planted ties
        L[::3] = np.round(L[::3])  # many ties
        ids, gates = O.route_topk(L, k)
        for t in range(L.shape[0]):
            want = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k]
            assert ids[t].tolist() == want


def test_gates_equal_full_softmax_renormalised():
    # an independent formula: the softmax over all E experts, restricted to the top-k and
    # renormalised, equals the softmax over the k chosen logits
    rng = np.random.default_rng(2)
    L = (3 * rng.standard_normal((64, 32))).astype(np.float32)
    ids, gates = O.route_topk(L, 6)
    full = np.exp(L.astype(np.float64) - L.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(full, ids.astype(np.int64), axis=1)
    np.testing.assert_allclose(gates, sel / sel.sum(axis=1, keepdims=True), rtol=1e-6)
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, rtol=1e-6)
    assert np.all(np.diff(gates, axis=1) <= 0)  # gates follow the descending logit order


def test_topk_rejects_non_finite():
    L = np.zeros((2, 4), np.float32)
    L[1, 2] = np.nan
    with pytest.raises(ValueError):
        O.route_topk(L, 2)
    L[1, 2] = np.inf
    with pytest.raises(ValueError):
        O.route_topk(L, 2)


def test_kappa_golden(golden_dir):
    for case in _golden(golden_dir)["kappa"]:
        S, kappa = O.skew_kappa(case["counts"])
        assert S == case["sumsq"]
        assert kappa == case["kappa"], case["why"]


def test_kappa_uniform_is_one_and_concentrated_is_E_over_k():
    for E, k, T in [(8, 2, 256), (64, 8, 4096), (128, 8, 8192), (256, 8, 16384)]:
        N = T * k
        assert O.skew_kappa([N // E] * E)[1] == 1.0
        # every token picks the same k experts: k counts of T, the rest zero
        c = [T] * k + [0] * (E - k)
        assert O.skew_kappa(c)[1] == E / k


def test_kappa_bounds_on_random_routes():
    rng = np.random.default_rng(3)
    for _ in range(20):
        E, k, T = 32, 4, 200
        L = rng.standard_normal((T, E)).astype(np.float32) + np.log(
            1.0 / np.arange(1, E + 1)).astype(np.float32) * rng.uniform(0, 3)
        ids, _ = O.route_topk(L, k)
        c = O.expert_counts(ids, E)
        assert c.sum() == T * k
        S, kappa = O.skew_kappa(c)
        assert S == int((c.astype(np.int64) ** 2).sum())
        assert 1.0 - 1e-12 <= kappa <= E / k + 1e-12
        assert math.isclose(kappa, E * float(((c / c.sum()) ** 2).sum()), rel_tol=1e-12)


def test_counts_match_loop_and_reject_bad_ids():
    rng = np.random.default_rng(4)
    ids = rng.integers(0, 10, size=(50, 3))
    c = O.expert_counts(ids, 10)
    for e in range(10):
        assert c[e] == sum(1 for v in ids.ravel() if v == e)
    with pytest.raises(ValueError):
        O.expert_counts(np.array([[0, 10]]), 10)


def test_block_counts_and_offsets():
    for beta in (64, 128):
        c = [0, 1, beta - 1, beta, beta + 1, 5 * beta, 5 * beta + 3]
        b = O.block_counts(c, beta)
        assert b == [0, 1, 1, 1, 2, 5, 6]
        for ce, be in zip(c, b):
            assert ce <= beta * be < ce + beta or (ce == 0 and be == 0)
        off = O.block_offsets(b)
        assert off[0] == 0 and off[-1] == sum(b) and len(off) == len(b) + 1
        assert all(off[i + 1] - off[i] == b[i] for i in range(len(b)))


def test_owner_map_contiguous_ranges():
    for E, P in [(8, 4), (64, 8), (128, 8), (256, 8), (6, 4), (5, 3)]:
        h = [O.owner(e, E, P) for e in range(E)]
        assert h == sorted(h) and h[0] == 0 and h[-1] == P - 1
        sizes = [h.count(r) for r in range(P)]
        assert max(sizes) - min(sizes) <= 1
