"""Pins of the oracle's dispatch, FFN and combine: permutation invariants, the dense
SwiGLU special case, identical and scaled experts, exact linearity, token-permutation
equivariance, and an fp64 evaluation that bounds the oracle's own rounding; no GPU."""
import numpy as np
import torch

from oracle import moe_oracle as O


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def _dense_swiglu_f64(x, w1, w2):
    """Independent fp64 dense SwiGLU MLP: (silu(x Wg^T) * (x Wu^T)) W2^T via torch."""
    f = w1.shape[0] // 2
    xt = torch.from_numpy(np.asarray(x, np.float64))
    g = xt @ torch.from_numpy(np.asarray(w1[:f], np.float64)).T
    u = xt @ torch.from_numpy(np.asarray(w1[f:], np.float64)).T
    return (torch.nn.functional.silu(g) * u @ torch.from_numpy(np.asarray(w2, np.float64)).T).numpy()


def _setup(T=64, E=6, k=2, d=64, f=128, beta=64, seed=0):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = _bf16(rng.standard_normal((T, d)))
    W1 = _bf16(rng.standard_normal((E, 2 * f, d)) / np.sqrt(d))
    W2 = _bf16(rng.standard_normal((E, d, f)) / np.sqrt(f))
    return logits, x, W1, W2


def test_dispatch_invariants():
    rng = np.random.default_rng(1)
    for T, E, k, beta in [(256, 8, 2, 64), (999, 16, 4, 128), (7, 8, 8, 64), (0, 4, 2, 64)]:
        L = rng.standard_normal((T, E)).astype(np.float32)
        ids, gates = O.route_topk(L, k) if T else (np.zeros((0, k), np.int32),
                                                  np.zeros((0, k), np.float32))
        c = O.expert_counts(ids, E)
        boff = O.block_offsets(O.block_counts(c, beta))
        row_token, row_gate, tok_row = O.dispatch(ids, gates, boff, beta)
        R = beta * boff[-1]
        assert len(row_token) == R
        # tok_row is a bijection onto the valid rows, and row_token inverts it
        valid = np.nonzero(row_token >= 0)[0]
        assert sorted(tok_row.ravel().tolist()) == valid.tolist()
        for t in range(T):
            for j in range(k):
                r = tok_row[t, j]
                assert row_token[r] == t and row_gate[r] == gates[t, j]
                e = ids[t, j]
                assert beta * boff[e] <= r < beta * boff[e] + c[e]   # expert e's rows
        # stable: tokens ascend inside each expert; padding rows carry -1 / 0
        for e in range(E):
            rows = row_token[beta * boff[e]: beta * boff[e + 1]]
            assert (rows[:c[e]] >= 0).all() and (rows[c[e]:] == -1).all()
            assert (np.diff(rows[:c[e]]) > 0).all()
        assert (row_gate[row_token < 0] == 0).all()


def test_gather_rows_copies_exactly():
    x = np.arange(5 * 4, dtype=np.float32).reshape(5, 4)
    rt = np.array([3, -1, 0, 0, -1, 4], np.int32)
    xp = O.gather_rows(x, rt)
    assert (xp[0] == x[3]).all() and (xp[2] == x[0]).all() and (xp[5] == x[4]).all()
    assert (xp[1] == 0).all() and (xp[4] == 0).all()


def test_silu_matches_torch():
    g = np.linspace(-120, 60, 20001).astype(np.float32)
    want = torch.nn.functional.silu(torch.from_numpy(g.astype(np.float64))).numpy()
    np.testing.assert_allclose(O.silu(g), want, rtol=2e-6, atol=1e-30)


def test_single_expert_top1_is_dense_swiglu():
    logits, x, W1, W2 = _setup(T=37, E=1, k=1)
    out = O.moe_forward(logits, x, lambda e: (W1[e], W2[e]), k=1, beta=64, P=1, s=0)
    assert (out["gates"] == 1.0).all()
    np.testing.assert_allclose(out["y"], _dense_swiglu_f64(x, W1[0], W2[0]), rtol=2e-4,
                               atol=2e-5)


def test_identical_experts_reduce_to_dense():
    logits, x, W1, W2 = _setup(T=80, E=6, k=3)
    out = O.moe_forward(logits, x, lambda e: (W1[0], W2[0]), k=3, beta=64, P=3, s=1)
    # gates sum to one, so every token sees the dense MLP
    np.testing.assert_allclose(out["y"], _dense_swiglu_f64(x, W1[0], W2[0]), rtol=2e-4,
                               atol=2e-5)


def test_scaled_experts_weight_the_gates():
    logits, x, W1, W2 = _setup(T=80, E=6, k=3, seed=3)
    scale = np.arange(1, 7, dtype=np.float32)
    out = O.moe_forward(logits, x, lambda e: (W1[0], W2[0] * scale[e]), k=3, beta=64, P=3,
                        s=1)
    dense = _dense_swiglu_f64(x, W1[0], W2[0])
    ids, gates = out["ids"], out["gates"].astype(np.float64)
    want = (gates * (ids + 1)).sum(axis=1, keepdims=True) * dense
    np.testing.assert_allclose(out["y"], want, rtol=2e-4, atol=2e-5)


def test_doubling_w2_doubles_y_exactly():
    logits, x, W1, W2 = _setup(seed=4)
    a = O.moe_forward(logits, x, lambda e: (W1[e], W2[e]), k=2, beta=64, P=2, s=1)
    b = O.moe_forward(logits, x, lambda e: (W1[e], 2 * W2[e]), k=2, beta=64, P=2, s=1)
    assert np.array_equal(b["y"], 2 * a["y"])


def test_token_permutation_equivariance():
    logits, x, W1, W2 = _setup(T=90, seed=5)
    perm = np.random.default_rng(6).permutation(90)
    a = O.moe_forward(logits, x, lambda e: (W1[e], W2[e]), k=2, beta=64, P=3, s=1)
    b = O.moe_forward(logits[perm], x[perm], lambda e: (W1[e], W2[e]), k=2, beta=64, P=3, s=1)
    np.testing.assert_allclose(b["y"], a["y"][perm], rtol=1e-5, atol=1e-6)


def test_fp64_bound_on_tiny_shape():
    """A per-token fp64 evaluation of y_t = sum_j p_tj O_e(x_t) written as a loop bounds the
    fp32 oracle's own error far inside the GPU tolerance 1e-2 + 2e-2|ref|."""
    logits, x, W1, W2 = _setup(T=48, E=8, k=2, d=512, f=256, seed=7)
    out = O.moe_forward(logits, x, lambda e: (W1[e], W2[e]), k=2, beta=64, P=4, s=1)
    y64 = np.zeros_like(out["y"], dtype=np.float64)
    for t in range(48):
        for j in range(2):
            e = out["ids"][t, j]
            y64[t] += float(out["gates"][t, j]) * _dense_swiglu_f64(x[t:t + 1], W1[e], W2[e])[0]
    err = np.abs(out["y"] - y64)
    assert err.max() <= 1e-4 + 1e-4 * np.abs(y64).max()


def test_token_output_matches_full_forward():
    logits, x, W1, W2 = _setup(T=30, E=5, k=2, seed=8)
    out = O.moe_forward(logits, x, lambda e: (W1[e], W2[e]), k=2, beta=64, P=5, s=1)
    for t in (0, 7, 29):
        y_t = O.token_output(x[t], out["ids"][t], out["gates"][t], lambda e: (W1[e], W2[e]))
        np.testing.assert_allclose(y_t, out["y"][t], rtol=1e-5, atol=1e-6)
