"""GPU parity of the expert FFN and the combine through the C ABI against the oracle:
every element of y on shapes the oracle finishes in seconds (several tiles, ragged
tails, beta = 64 and 128, both FFN modes, strict slots), and sampled tokens at the full
sizes of the large workloads.  Bar: |gpu - ref| <= 1e-2 + 2e-2|ref| per element."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import native as N
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import WORKLOADS, Workload

from gpu_common import check_y, f32, host_inputs, run_gpu

pytestmark = pytest.mark.gpu

FULL_CASES = [
    WORKLOADS["tiny"],
    Workload("ragged64", T=333, d=256, E=6, k=2, f=256, beta=64, P=3, s=1, alpha=1.0),
    Workload("ragged128", T=1111, d=512, E=12, k=4, f=384, beta=128, P=4, s=2, alpha=0.5),
    Workload("one_expert", T=200, d=256, E=1, k=1, f=128, beta=128, P=1, s=0),
    Workload("hot_all", T=515, d=256, E=16, k=4, f=128, beta=64, P=8, s=2, hot_p=1.0,
             hot_mode="all4"),
    WORKLOADS["olmoe_a1"],
]
MODES = [N.MOE_FFN_FUSED_COMBINE, N.MOE_FFN_WRITE_O,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_STRICT_SLOTS,
         N.MOE_FFN_WRITE_O | N.MOE_FFN_STRICT_SLOTS,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_SM_PAIR,
         N.MOE_FFN_WRITE_O | N.MOE_FFN_SM_PAIR | N.MOE_FFN_STRICT_SLOTS,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_ONE_LAUNCH,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_TWO_LAUNCHES,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_TWO_LAUNCHES | N.MOE_FFN_FC1_M128,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_TWO_LAUNCHES | N.MOE_FFN_FC2_WHOLE,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_FC2_WHOLE | N.MOE_FFN_STRICT_SLOTS,
         N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_FC1_M128 | N.MOE_FFN_STRICT_SLOTS,
         N.MOE_FFN_WRITE_O | N.MOE_FFN_FC1_M128 | N.MOE_FFN_STRICT_SLOTS]


_ORACLE = {}


def _oracle_full(wl, w1, w2):
    """The oracle's whole layer on the workload's inputs (weights are a function of the
    workload, so the result is kept for the next test of the same workload)."""
    if wl not in _ORACLE:
        _ORACLE.clear()
        _ORACLE[wl] = _oracle_run(wl, w1, w2)
    return _ORACLE[wl]


def _oracle_run(wl, w1, w2):
    logits, x = host_inputs(wl)
    W1 = f32(w1)
    W2 = f32(w2)
    return O.moe_forward(logits.numpy(), x.float().numpy(), lambda e: (W1[e], W2[e]),
                         k=wl.k, beta=wl.beta, P=wl.P, s=wl.s)


@pytest.mark.parametrize("gather_x", [True, False], ids=["gather_x", "xp"])
@pytest.mark.parametrize("wl", FULL_CASES, ids=lambda w: w.name)
def test_ffn_every_element(wl, gather_x):
    """Both A sources of FC1: rows gathered from x by row_token, and the dispatched Xp."""
    w1, w2 = synth.make_weights(wl, "cuda")
    ref = _oracle_full(wl, w1, w2)
    # o_rows=False: each mode runs as written (the layer's own choice would add O rows)
    layer = MoeLayer(wl, "cuda", write_o=True, gather_x=gather_x, o_rows=False)
    for mode in MODES:
        if gather_x and mode & (N.MOE_FFN_ONE_LAUNCH | N.MOE_FFN_TWO_LAUNCHES |
                                N.MOE_FFN_FC1_M128 | N.MOE_FFN_FC2_WHOLE):
            continue  # launch-count and FC1 tile flags are for the Xp path
        layer.y.fill_(float("nan"))
        run_gpu(wl, w1, w2, mode=mode, layer=layer)
        assert layer.read_status() == 0, (mode, N.moe_status_string(layer.read_status()))
        check_y(f32(layer.view("y")), ref["y"], f"{wl.name} mode {mode}")
        if mode & N.MOE_FFN_WRITE_O:
            # O rows of valid pairs against the oracle's per-row expert outputs
            rows = ref["row_token"] >= 0
            o = f32(layer.view("o"))[: len(rows)]
            check_y(o[rows], ref["O"][rows], f"{wl.name} O rows")


@pytest.mark.parametrize("mode", [N.MOE_FFN_ONE_LAUNCH, N.MOE_FFN_TWO_LAUNCHES,
                                  N.MOE_FFN_TWO_LAUNCHES | N.MOE_FFN_FC1_M128],
                         ids=["one_launch", "fc1_whole_tiles", "fc1_tile_halves"])
@pytest.mark.parametrize("wl", [FULL_CASES[1], FULL_CASES[2]], ids=lambda w: w.name)
def test_intermediate_a_matches_swiglu(wl, mode):
    """FC1's output A on every valid row, for each FC1 kernel (tile halves in one launch or
    two, whole 256-row tiles)."""
    w1, w2 = synth.make_weights(wl, "cuda")
    ref = _oracle_full(wl, w1, w2)
    layer = run_gpu(wl, w1, w2, mode=mode)
    rows = np.nonzero(ref["row_token"] >= 0)[0]
    A = f32(layer.view("a_scratch"))[rows]
    _, x = host_inputs(wl)
    W1 = f32(w1)
    xr = x.float().numpy()[ref["row_token"][rows]]
    want = np.empty_like(A)
    for e in range(wl.E):
        sel = (rows >= wl.beta * ref["block_off"][e]) & (rows < wl.beta * ref["block_off"][e + 1])
        Z = xr[sel] @ W1[e].T
        want[sel] = O.silu(Z[:, : wl.f]) * Z[:, wl.f:]
    # A is rounded to bf16 on the GPU: 2^-8 relative plus accumulation-order noise
    check_y(A, want, "A = SiLU(G) * U")


@pytest.mark.parametrize("name", ["qwen3_a1.5", "dsv3_a1"])
def test_one_launch_full_size_sampled_tokens(name):
    """FC1 and FC2 in one launch at full size: sampled tokens against the oracle, and the
    whole y against the two-launch FFN on the same 128-row FC1 tiles (same arithmetic,
    atomics may reorder last bits)."""
    wl = WORKLOADS[name]
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = run_gpu(wl, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_TWO_LAUNCHES |
                    N.MOE_FFN_FC1_M128)
    y2 = layer.view("y").clone()
    run_gpu(wl, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_ONE_LAUNCH, layer=layer)
    assert layer.read_status() == 0
    torch.testing.assert_close(layer.view("y"), y2, rtol=1e-5, atol=1e-5)
    logits, x = host_inputs(wl)
    ids_ref, gates_ref = O.route_topk(logits.numpy(), wl.k)
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, 24, replace=False)]))
    y = f32(layer.view("y")[torch.from_numpy(sample).cuda()])
    xs = x.float().numpy()
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = (f32(w1[e]), f32(w2[e]))
        return cache[e]

    for i, t in enumerate(sample):
        check_y(y[i], O.token_output(xs[t], ids_ref[t], gates_ref[t], expert), f"{name} {t}")


@pytest.mark.parametrize("name,gather_x", [
    ("qwen3_a1.5", False), ("sweep_all4_p0.5_b128", False), ("sweep_one_p0.3_b64", False),
    ("sweep_all4_p1_b128_zipf1.5", False), ("dsv3_a1", False),
    ("sweep_all4_p1_b128_zipf1.5", True), ("dsv3_a1", True)])
def test_full_size_sampled_tokens(name, gather_x):
    """Full-size layers in the benchmark's launch configuration (and with FC1 gathering
    its rows from x); the oracle recomputes a sample of tokens one by one (rows of the
    FFN are independent)."""
    wl = WORKLOADS[name]
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = run_gpu(wl, w1, w2, layer=MoeLayer(wl, "cuda", gather_x=gather_x))
    assert layer.read_status() == 0
    logits, x = host_inputs(wl)
    ids = layer.view("topk_ids").cpu().numpy()
    ids_ref, gates_ref = O.route_topk(logits.numpy(), wl.k)
    assert np.array_equal(ids, ids_ref)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, 48, replace=False)]))
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = (f32(w1[e]), f32(w2[e]))
        return cache[e]

    y = f32(layer.view("y")[torch.from_numpy(sample).cuda()])
    xs = x.float().numpy()
    for i, t in enumerate(sample):
        y_ref = O.token_output(xs[t], ids_ref[t], gates_ref[t], expert)
        check_y(y[i], y_ref, f"{name} token {t}")
    # the whole output is finite and every token got its k contributions
    assert torch.isfinite(layer.view("y")).all()


def test_concurrent_planner_matches_sequential_stages():
    """The layer call runs the planner's search on a side stream beside the dispatch; the
    result must be the stage-by-stage one (the same plan, tiles, rows and y)."""
    wl = FULL_CASES[2]
    w1, w2 = synth.make_weights(wl, "cuda")
    logits, x = host_inputs(wl)
    a = MoeLayer(wl, "cuda")
    a(logits.cuda(), x.cuda(), w1, w2)
    b = MoeLayer(wl, "cuda")
    b.route(logits.cuda())
    b.plan(0)
    b.dispatch(x.cuda())
    b.ffn(w1, w2)
    torch.cuda.synchronize()
    assert a.read_status() == 0 and b.read_status() == 0
    for name in ("block_off", "q", "tiles", "row_token", "tok_row"):
        assert torch.equal(a.view(name), b.view(name)), name
    torch.testing.assert_close(a.view("y"), b.view("y"), rtol=1e-5, atol=1e-6)


def test_repeated_calls_reuse_buffers():
    wl = FULL_CASES[1]
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = run_gpu(wl, w1, w2)
    y1 = layer.view("y").clone()
    for _ in range(3):
        run_gpu(wl, w1, w2, layer=layer)
    assert layer.read_status() == 0
    # fp32 atomic accumulation order may differ in the last bits only
    torch.testing.assert_close(layer.view("y"), y1, rtol=1e-5, atol=1e-6)


def test_host_pipeline_matches_direct_calls():
    """The overlapped host-buffer runner gives, batch by batch, what direct calls give."""
    from skew_aware_token_b200.layer import HostPipeline
    wl = FULL_CASES[1]
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda")
    pipe = HostPipeline(layer)
    batches = []
    for seed in range(5):
        b = wl.with_(seed=seed)
        batches.append((synth.make_logits(b).pin_memory(), synth.make_x(b).pin_memory(),
                        torch.empty(wl.T, wl.d).pin_memory()))
    for logits_h, x_h, y_h in batches:
        pipe.submit(logits_h, x_h, y_h, w1, w2)
    pipe.drain()
    assert layer.read_status() == 0
    for logits_h, x_h, y_h in batches:
        want = layer(logits_h.cuda(), x_h.cuda(), w1, w2).cpu()
        torch.testing.assert_close(y_h, want, rtol=1e-5, atol=1e-6)


def test_graph_replay_matches_direct_calls():
    """The whole layer captured into a CUDA graph gives, batch by batch, what direct calls
    give (the fused combine's atomics may reorder the last bits)."""
    from skew_aware_token_b200.layer import LayerGraph
    wl = FULL_CASES[2]
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda")
    g = LayerGraph(layer, w1, w2)
    direct = MoeLayer(wl, "cuda")
    for seed in range(3):
        b = wl.with_(seed=seed)
        logits, x = synth.make_logits(b).cuda(), synth.make_x(b).cuda()
        g.logits.copy_(logits)
        g.x.copy_(x)
        g.replay()
        want = direct(logits, x, w1, w2)
        torch.cuda.synchronize()
        assert layer.read_status() == 0
        torch.testing.assert_close(layer.view("y"), want, rtol=1e-5, atol=1e-6)
        assert torch.equal(layer.view("q"), direct.view("q"))
