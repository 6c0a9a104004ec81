"""Pins of the oracle's backward (the MegaFlux summary's backward gradients): central
finite differences of the forward oracle in fp64 for dx, dW1 and dW2, the SiLU
derivative, and bf16 requantization against torch's conversion; no GPU."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def _tiny(seed, T=6, d=8, E=4, k=2, f=4):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, d))
    w1 = rng.standard_normal((E, 2 * f, d)) / np.sqrt(d)
    w2 = rng.standard_normal((E, d, f)) / np.sqrt(f)
    dy = rng.standard_normal((T, d))
    return logits, x, w1, w2, dy, k


def _loss(logits, x, w1, w2, dy, k):
    """L = sum_t <dy_t, y_t>, y_t = sum_j g_tj O_{e_tj}(x_t), all fp64."""
    ids, gates = O.route_topk(logits, k)
    y = np.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(k):
            e = ids[t, j]
            y[t] += float(gates[t, j]) * O.expert_ffn(x[t:t + 1], w1[e], w2[e], np.float64)[0]
    return float(np.sum(dy * y))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gradients_match_finite_differences(seed):
    logits, x, w1, w2, dy, k = _tiny(seed)
    g = O.moe_backward(logits, x, lambda e: (w1[e], w2[e]), dy, k, beta=2,
                       dtype=np.float64, requant=False)
    eps = 1e-6

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + eps
        lp = _loss(logits, x, w1, w2, dy, k)
        arr[idx] = old - eps
        lm = _loss(logits, x, w1, w2, dy, k)
        arr[idx] = old
        return (lp - lm) / (2 * eps)

    for idx in np.ndindex(x.shape):
        assert abs(fd(x, idx) - g["dx"][idx]) < 1e-6 * (1 + abs(g["dx"][idx])), ("dx", idx)
    used = set(O.route_topk(logits, k)[0].ravel().tolist())
    for e in range(w1.shape[0]):
        for idx in np.ndindex(w1.shape[1:]):
            want = fd(w1, (e,) + idx)
            assert abs(want - g["dW1"][e][idx]) < 1e-6 * (1 + abs(want)), ("dW1", e, idx)
        for idx in np.ndindex(w2.shape[1:]):
            want = fd(w2, (e,) + idx)
            assert abs(want - g["dW2"][e][idx]) < 1e-6 * (1 + abs(want)), ("dW2", e, idx)
        if e not in used:
            assert not g["dW1"][e].any() and not g["dW2"][e].any()


def test_silu_derivative():
    g = np.linspace(-12, 12, 97)
    h = 1e-6
    fd = (O.silu(g + h) - O.silu(g - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_grad(g), fd, rtol=1e-7, atol=1e-9)
    assert O.silu_grad(np.zeros(1))[0] == 0.5


def test_round_bf16_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(3)
    a = (rng.standard_normal(10000) * 10.0 ** rng.uniform(-6, 6, 10000)).astype(np.float32)
    want = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    assert np.array_equal(O.round_bf16(a), want)
    one = np.float32(1.0)
    ties = np.array([one + 2 ** -8, one + 3 * 2 ** -8, one - 2 ** -9], np.float32)
    assert O.round_bf16(ties).tolist() == [1.0, 1.0 + 2 ** -6, 1.0]


def test_requantized_operands_are_bf16_values():
    logits, x, w1, w2, dy, k = _tiny(5, T=20, d=16, f=8)
    g = O.moe_backward(logits, x.astype(np.float32), lambda e: (w1[e], w2[e]),
                       dy.astype(np.float32), k, beta=4)
    for name in ("D", "dZ"):
        assert np.array_equal(O.round_bf16(g[name]), g[name]), name
    # padding rows carry nothing
    pad = g["row_token"] < 0
    assert pad.any() and not g["D"][pad].any() and not g["dX"][pad].any()
