"""GPU parity of the backward pass (moe_dispatch_grad + moe_expert_ffn_backward) against
the oracle, through the C ABI.

Stage by stage, each GPU stage is compared with the oracle's arithmetic applied to that
stage's own GPU inputs: D bit-exact; dZ against the SwiGLU backward of (D w2, saved Z)
within bf16 rounding; dX / dx, dW2 and dW1 against fp32 products of the GPU's bf16
operands within the fp32 accumulation bound 2^-12 * sum_k |a_k||b_k|.  End to end, dx,
dW1 and dW2 against the oracle's whole backward (with A and Z kept in bf16, as the forward
stores them) within 2^-5 * rms(ref) + 2e-2 * |ref|: the two sides round Z, A and dZ from
values that differ in the fp32 accumulation order, so an operand element differs by at
most one bf16 step (relative 2^-8) and rarely; summed with random signs over the
contraction, the output error's standard deviation is below 2^-8 * rms(ref), and
2^-5 * rms(ref) is eight of them."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import WORKLOADS, Workload

from gpu_common import f32, host_inputs

pytestmark = pytest.mark.gpu

CASES = [
    WORKLOADS["tiny"],
    Workload("ragged128", T=1111, d=512, E=12, k=4, f=384, beta=128, P=4, s=2, alpha=0.5),
    Workload("one_expert", T=200, d=256, E=1, k=1, f=128, beta=128, P=1, s=0),
    Workload("hot_all", T=515, d=256, E=16, k=4, f=128, beta=64, P=8, s=2, hot_p=1.0,
             hot_mode="all4"),
    Workload("idle_experts", T=24, d=256, E=32, k=1, f=256, beta=64, P=4, s=1, alpha=2.0),
    # every product on whole 256-row tiles, several n- and m-tiles, skewed experts
    Workload("wide_skew", T=2048, d=1024, E=16, k=4, f=512, beta=128, P=4, s=2, alpha=1.0),
    # f not a multiple of 256: dW2 on 128-column items, several of them per expert
    Workload("wide_skew_f384", T=1536, d=768, E=12, k=4, f=384, beta=64, P=4, s=2, alpha=1.0),
]


def _bound_check(got, want, absprod, what, c=2.0 ** -12):
    err = np.abs(got - want)
    bad = err > c * absprod + 1e-6
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside the accumulation "
                           f"bound (max err {err.max():.3e})")


def _e2e_check(got, ref, what):
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2))) or 1.0
    err = np.abs(got - ref)
    bad = err > 2.0 ** -5 * rms + 2e-2 * np.abs(ref)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside 2^-5 rms + "
                           f"2e-2|ref| (max err {err.max():.3e}, rms {rms:.3e})")


def _run(wl):
    logits, x = host_inputs(wl)
    dy = synth.make_dy(wl)
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda", train=True)
    layer.clear_status()
    layer(logits.cuda(), x.cuda(), w1, w2)
    for name in ("dx", "dw1", "dw2"):
        getattr(layer, name).fill_(float("nan"))  # every element must be written
    layer.backward(dy.cuda(), w1, w2)
    torch.cuda.synchronize()
    assert layer.read_status() == 0
    return layer, logits, x, dy, w1, w2


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_backward_stages_and_end_to_end(wl):
    layer, logits, x, dy, w1, w2 = _run(wl)
    B = int(layer.plan_info[0])
    R = wl.beta * B
    row_token = layer.view("row_token")[:R].cpu().numpy()
    row_gate = f32(layer.view("row_gate")[:R])
    valid = row_token >= 0
    boff = layer.view("block_off").cpu().tolist()
    dyn = dy.numpy()
    W1, W2 = f32(w1), f32(w2)

    # D = bf16(row_gate * dy[row_token]), zero on padding rows: bit-exact
    D = f32(layer.view("d_rows")[:R])
    D_ref = np.zeros_like(D)
    D_ref[valid] = O.round_bf16(row_gate[valid, None] * dyn[row_token[valid]])
    assert np.array_equal(D, D_ref)

    A = f32(layer.view("a_scratch")[:R])
    Z = f32(layer.view("z")[:R])
    dZ = f32(layer.view("dz")[:R])
    Xp = f32(layer.view("xp")[:R])
    dW1 = f32(layer.view("dw1"))
    dW2 = f32(layer.view("dw2"))
    f = wl.f
    for e in range(wl.E):
        rows = slice(wl.beta * boff[e], wl.beta * boff[e + 1])
        if boff[e + 1] == boff[e]:
            assert not dW1[e].any() and not dW2[e].any(), f"idle expert {e} not zero"
            continue
        De, Ze = D[rows], Z[rows]
        # dZ from the GPU's own D and saved Z: SwiGLU backward, then one bf16 rounding
        dA = De @ W2[e]
        G, U = Ze[:, :f], Ze[:, f:]
        dZ_ref = np.concatenate([dA * U * O.silu_grad(G), dA * O.silu(G)], axis=1)
        absdA = np.abs(De) @ np.abs(W2[e])
        scale = np.concatenate([absdA * np.abs(U) * 1.2, absdA * np.abs(G)], axis=1)
        err = np.abs(dZ[rows] - dZ_ref)
        assert not (err > 2.0 ** -7 * np.abs(dZ_ref) + 2.0 ** -12 * scale + 1e-6).any(), \
            f"dZ expert {e}"
        # weight gradients from the GPU's bf16 operands
        _bound_check(dW2[e], De.T @ A[rows], np.abs(De).T @ np.abs(A[rows]), f"dW2 {e}")
        _bound_check(dW1[e], dZ[rows].T @ Xp[rows], np.abs(dZ[rows]).T @ np.abs(Xp[rows]),
                     f"dW1 {e}")
    # dx = sum over each token's rows of dZ w1_e
    tok_row = layer.view("tok_row").cpu().numpy()
    ids = layer.view("topk_ids").cpu().numpy()
    dx_ref = np.zeros((wl.T, wl.d), np.float32)
    dx_abs = np.zeros((wl.T, wl.d), np.float32)
    for j in range(wl.k):
        for e in np.unique(ids[:, j]):
            sel = ids[:, j] == e
            r = tok_row[sel, j]
            dx_ref[sel] += dZ[r] @ W1[e]
            dx_abs[sel] += np.abs(dZ[r]) @ np.abs(W1[e])
    _bound_check(f32(layer.view("dx")), dx_ref, dx_abs, "dx")

    # end to end against the oracle's backward (its own fp32 forward quantities)
    ref = O.moe_backward(logits.numpy(), x.float().numpy(), lambda e: (W1[e], W2[e]),
                         dyn, wl.k, wl.beta, saved_bf16=True)
    _e2e_check(f32(layer.view("dx")), ref["dx"], "dx end to end")
    _e2e_check(dW1, ref["dW1"], "dW1 end to end")
    _e2e_check(dW2, ref["dW2"], "dW2 end to end")


def test_backward_repeatable_and_forward_unchanged():
    """A training forward gives the inference forward's y; two backward calls agree."""
    wl = CASES[1]
    layer, logits, x, dy, w1, w2 = _run(wl)
    y_train = layer.view("y").clone()
    dw1 = layer.view("dw1").clone()
    infer = MoeLayer(wl, "cuda")
    infer(logits.cuda(), x.cuda(), w1, w2)
    torch.cuda.synchronize()
    torch.testing.assert_close(infer.view("y"), y_train, rtol=1e-5, atol=1e-6)
    layer.backward(dy.cuda(), w1, w2)
    torch.cuda.synchronize()
    assert torch.equal(layer.view("dw1"), dw1)  # no atomics in the weight gradients


def test_backward_empty_input():
    """A layer with no tokens: the weight gradients come out zero and the status stays
    clean (one-element buffers stand in for the empty inputs)."""
    wl = CASES[0].with_(T=0)
    layer = MoeLayer(wl, "cuda", train=True)
    layer.clear_status()
    w1 = torch.zeros(wl.E, 2 * wl.f, wl.d, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros(wl.E, wl.d, wl.f, dtype=torch.bfloat16, device="cuda")
    layer(torch.zeros(1, wl.E, device="cuda"),
          torch.zeros(1, wl.d, dtype=torch.bfloat16, device="cuda"), w1, w2)
    layer.dw1.fill_(float("nan"))
    layer.dw2.fill_(float("nan"))
    layer.backward(torch.zeros(1, wl.d, device="cuda"), w1, w2)
    torch.cuda.synchronize()
    assert layer.read_status() == 0
    assert not layer.view("dw1").any() and not layer.view("dw2").any()
