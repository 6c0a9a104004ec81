"""GPU parity of the integer stages through the C ABI: top-k, gates, counts, S and kappa;
block offsets, the planner's q for every variant, the block and tile lists; dispatch
indices and the gathered rows.  Integer results are compared bit for bit."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import native as N
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import WORKLOADS, Workload

from gpu_common import GATE_RTOL, expected_tiles, f32, host_inputs

pytestmark = pytest.mark.gpu

ROUTE_CASES = ["tiny", "olmoe_a0", "olmoe_a0.5", "olmoe_a1", "qwen3_a0", "qwen3_a1",
               "qwen3_a1.5", "sweep_one_p0.3_b128", "sweep_all4_p0.5_b64",
               "sweep_all4_p1_b128_zipf1.5", "dsv3_a1"]
SMALL = [
    Workload("e5k3", T=301, d=256, E=5, k=3, f=128, beta=64, P=3, s=1),
    Workload("e33k8", T=777, d=256, E=33, k=8, f=128, beta=128, P=5, s=2),
    Workload("e1k1", T=130, d=256, E=1, k=1, f=128, beta=64, P=1, s=0),
    Workload("e256k8", T=1000, d=256, E=256, k=8, f=128, beta=128, P=8, s=4, alpha=1.0),
    Workload("t1_all", T=1, d=256, E=8, k=8, f=128, beta=64, P=4, s=1),
]


ALL5 = N.variant_mask(range(N.N_VARIANTS))


def _wl(name):
    return WORKLOADS[name] if isinstance(name, str) else name


@pytest.mark.parametrize("case", ROUTE_CASES + SMALL, ids=lambda c: c if isinstance(c, str) else c.name)
def test_route_hist_and_plan_and_dispatch(case):
    wl = _wl(case)
    logits, x = host_inputs(wl)
    layer = MoeLayer(wl, "cuda", gather_x=False)  # materialise Xp to check its rows
    layer.clear_status()
    layer.route(logits.cuda())
    layer.plan(ALL5)
    layer.dispatch(x.cuda())
    torch.cuda.synchronize()
    assert layer.read_status() == 0

    # S1/S2: top-k, gates, histogram, kappa
    ids_ref, gates_ref = O.route_topk(logits.numpy(), wl.k)
    ids = layer.view("topk_ids").cpu().numpy()
    assert np.array_equal(ids, ids_ref)
    gates = f32(layer.view("topk_gates"))
    np.testing.assert_allclose(gates, gates_ref, rtol=GATE_RTOL, atol=0)
    counts_ref = O.expert_counts(ids_ref, wl.E)
    assert np.array_equal(layer.view("counts").cpu().numpy(), counts_ref)
    S_ref, kappa_ref = O.skew_kappa(counts_ref)
    assert int(layer.sumsq[0]) == S_ref
    assert float(layer.kappa[0]) == kappa_ref  # same exact integers, one rounding

    # S3/S4: blocks and the plan of the best variant
    b = O.block_counts(counts_ref, wl.beta)
    boff = O.block_offsets(b)
    assert layer.view("block_off").cpu().tolist() == boff
    assert layer.block_off_plan[:wl.E + 1].cpu().tolist() == boff  # the planner's copy
    ref = O.plan(b, wl.P, wl.s, variant_mask=ALL5)  # all five variants, best kept
    q = layer.view("q").cpu().numpy()
    assert np.array_equal(q, ref["q"])
    pi = layer.plan_info.cpu().tolist()
    assert pi[N.PI["B"]] == ref["B"] and pi[N.PI["TAU"]] == ref["tau"]
    assert pi[N.PI["MAKESPAN"]] == ref["makespan"] and pi[N.PI["VARIANT"]] == ref["variant"]
    assert pi[N.PI["REPLICAS"]] == ref["replicas"] and pi[N.PI["ROUNDS"]] == ref["rounds"]
    assert pi[N.PI["FIXED_MAKESPAN"]] == ref["fixed_makespan"]
    for v in range(N.N_VARIANTS):
        assert pi[N.PI["VAR_MAKESPAN"] + v] == ref["all"][v]["makespan"]
        assert pi[N.PI["VAR_REPLICAS"] + v] == ref["all"][v]["replicas"]
        assert pi[N.PI["VAR_ROUNDS"] + v] == ref["all"][v]["rounds"]
    assert pi[N.PI["QUOTA_TAU"]] == ref["all"][N.QUOTA_VARIANT]["tau_star"]
    assert layer.view("slot_load").cpu().tolist() == ref["load"]
    blocks_ref, slot_off_ref = O.block_list(ref["q"])
    assert layer.view("slot_off").cpu().tolist() == slot_off_ref
    B = ref["B"]
    assert [tuple(r) for r in layer.view("blocks")[:B].cpu().tolist()] == blocks_ref
    tiles_ref, sto_ref = expected_tiles(ref["q"], boff, wl.beta)
    nt = pi[N.PI["NTILES"]]
    assert nt == len(tiles_ref)
    assert [tuple(r) for r in layer.view("tiles")[:nt].cpu().tolist()] == tiles_ref
    assert pi[N.PI["SLOT_TILE_OFF"]:N.PI["SLOT_TILE_OFF"] + wl.P + 1] == sto_ref

    # S6: dispatch indices (bit-exact), gates carried with their pair, rows copied exactly
    rt_ref, _, tr_ref = O.dispatch(ids_ref, gates, boff, wl.beta)
    R = wl.beta * boff[-1]
    row_token = layer.view("row_token")[:R].cpu().numpy()
    assert np.array_equal(row_token, rt_ref)
    assert np.array_equal(layer.view("tok_row").cpu().numpy(), tr_ref)
    row_gate = f32(layer.view("row_gate")[:R])
    valid = rt_ref >= 0
    assert np.array_equal(row_gate[tr_ref.ravel()], gates.ravel())
    assert (row_gate[~valid] == 0).all()
    xp = layer.view("xp")[:R].cpu()
    xv = x.view(torch.int16)
    assert torch.equal(xp.view(torch.int16)[torch.from_numpy(valid)],
                       xv[torch.from_numpy(rt_ref[valid]).long()])
    assert (xp.view(torch.int16)[torch.from_numpy(~valid)] == 0).all()


@pytest.mark.parametrize("E,P", [(8, 4), (64, 8), (128, 8), (256, 8), (12, 5), (256, 2), (7, 1)])
def test_planner_every_variant_bit_exact(E, P):
    rng = np.random.default_rng(E * 10 + P)
    for trial in range(6):
        s = [0, 1, 2, 4, E, 3][trial]
        beta = (64, 128)[trial % 2]
        zipf = 1.0 / np.arange(1, E + 1) ** rng.uniform(0, 2.5)
        T = int(rng.integers(1, 3000))
        k = int(min(E, 8))
        counts = rng.multinomial(T * k, zipf / zipf.sum()).astype(np.int32)
        wl = Workload("rand", T=T, d=256, E=E, k=k, f=128, beta=beta, P=P, s=s)
        layer = MoeLayer(wl, "cuda")
        layer.counts[:E] = torch.from_numpy(counts).cuda()
        b = O.block_counts(counts, beta)
        # the four greedy searches, then the quota solver with three quota floors
        for v, u_min in [(0, 1), (1, 1), (2, 1), (3, 1), (4, 1), (4, 2), (4, 7)]:
            layer.clear_status()
            layer.plan(N.variant_mask([v], u_min=u_min))
            torch.cuda.synchronize()
            ref = O.plan_variant(b, P, s, v) if v < 4 else O.plan_quota(b, P, s, u_min)
            assert np.array_equal(layer.view("q").cpu().numpy(), ref["q"]), (E, P, s, v, u_min)
            pi = layer.plan_info.cpu().tolist()
            assert pi[N.PI["MAKESPAN"]] == ref["makespan"] and pi[N.PI["VARIANT"]] == v
            assert pi[N.PI["REPLICAS"]] == ref["replicas"]
            assert pi[N.PI["ROUNDS"]] == ref["rounds"]
            if v == 4:
                assert pi[N.PI["QUOTA_TAU"]] == ref["tau_star"]
            assert layer.read_status() == 0


@pytest.mark.parametrize("E,P", [(8, 4), (64, 8), (256, 8), (12, 5), (256, 2)])
def test_reduction_aware_plans_bit_exact(E, P):
    """C_lambda selection: every variant's least-C_lambda plan and the best of five."""
    rng = np.random.default_rng(E * 7 + P)
    for trial in range(5):
        s = [1, 2, 4, 3, E][trial]
        beta = (64, 128)[trial % 2]
        zipf = 1.0 / np.arange(1, E + 1) ** rng.uniform(0.5, 2.5)
        T = int(rng.integers(100, 3000))
        k = int(min(E, 8))
        counts = rng.multinomial(T * k, zipf / zipf.sum()).astype(np.int32)
        wl = Workload("rand", T=T, d=256, E=E, k=k, f=128, beta=beta, P=P, s=s)
        layer = MoeLayer(wl, "cuda")
        layer.counts[:E] = torch.from_numpy(counts).cuda()
        b = O.block_counts(counts, beta)
        for lam in (3, 12):
            for v in range(N.N_VARIANTS):
                layer.clear_status()
                layer.plan(N.variant_mask([v], lam=lam))
                torch.cuda.synchronize()
                if v < 4:
                    ref = O.plan_variant(b, P, s, v, lam)
                else:
                    ref = O.plan_quota(b, P, s)
                    ref["cost"] = O.reduction_cost(ref["q"], P, lam)
                assert np.array_equal(layer.view("q").cpu().numpy(), ref["q"]), (E, P, s, v, lam)
                pi = layer.plan_info.cpu().tolist()
                assert pi[N.PI["COST"]] == ref["cost"] and pi[N.PI["VARIANT"]] == v
                assert pi[N.PI["MAKESPAN"]] == ref["makespan"]
                assert pi[N.PI["REPLICAS"]] == ref["replicas"]
                assert pi[N.PI["ROUNDS"]] == ref["rounds"]
                assert layer.read_status() == 0
            layer.plan(N.variant_mask(range(N.N_VARIANTS), lam=lam))
            torch.cuda.synchronize()
            ref = O.plan(b, P, s, variant_mask=O.ALL_VARIANTS, lam=lam)
            assert np.array_equal(layer.view("q").cpu().numpy(), ref["q"])
            pi = layer.plan_info.cpu().tolist()
            assert pi[N.PI["VARIANT"]] == ref["variant"] and pi[N.PI["COST"]] == ref["cost"]
            assert pi[N.PI["VAR_COST"]:N.PI["VAR_COST"] + 5] == [ref["all"][v]["cost"]
                                                                for v in range(5)]
            # the tile list follows the chosen plan
            nt = pi[N.PI["NTILES"]]
            want, _ = expected_tiles(ref["q"], O.block_offsets(b), beta)
            assert [tuple(r) for r in layer.view("tiles")[:nt].cpu().tolist()] == want


def test_plan_is_deterministic():
    wl = WORKLOADS["dsv3_a1"]
    logits, _ = host_inputs(wl)
    layer = MoeLayer(wl, "cuda")
    layer.route(logits.cuda())
    outs = []
    for _ in range(3):
        layer.plan(0)
        torch.cuda.synchronize()
        outs.append((layer.q.clone(), layer.blocks.clone(), layer.tiles.clone(),
                     layer.plan_info.clone()))
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))


def test_empty_input():
    wl = WORKLOADS["tiny"].with_(T=0)
    layer = MoeLayer(wl, "cuda")
    layer.clear_status()
    # one-element buffers: valid, aligned pointers for a layer with no tokens
    layer(torch.zeros(1, wl.E, device="cuda"), torch.zeros(1, wl.d, dtype=torch.bfloat16,
                                                            device="cuda"),
          torch.zeros(wl.E, 2 * wl.f, wl.d, dtype=torch.bfloat16, device="cuda"),
          torch.zeros(wl.E, wl.d, wl.f, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert layer.read_status() == 0
    assert float(layer.kappa[0]) == 0.0 and int(layer.sumsq[0]) == 0
    assert layer.plan_info[N.PI["B"]].item() == 0 and layer.plan_info[N.PI["NTILES"]].item() == 0


def test_nonfinite_logit_sets_status():
    wl = WORKLOADS["tiny"]
    logits, _ = host_inputs(wl)
    bad = logits.clone()
    bad[17, 3] = float("nan")
    bad[90, 0] = float("inf")
    layer = MoeLayer(wl, "cuda")
    layer.clear_status()
    layer.route(bad.cuda())
    torch.cuda.synchronize()
    assert layer.read_status() & N.MOE_STATUS_NONFINITE


def test_bad_ids_and_overflow_are_reported_not_written_out_of_bounds():
    wl = WORKLOADS["tiny"]
    logits, x = host_inputs(wl)
    layer = MoeLayer(wl, "cuda", guard=256, gather_x=False)
    layer.route(logits.cuda())
    layer.plan(0)
    torch.cuda.synchronize()
    # out-of-range ids
    ids = layer.view("topk_ids")
    saved = ids.clone()
    ids[5, 1] = wl.E + 3
    ids[9, 0] = -2
    layer.clear_status()
    layer.dispatch(x.cuda())
    torch.cuda.synchronize()
    assert layer.read_status() & N.MOE_STATUS_BAD_ID
    ids.copy_(saved)
    # block offsets too small for the counts: rows are dropped, never written past R_max
    canary = 0x5A5A5A5A
    R = layer.R_max
    layer.row_token[R:] = canary
    layer.xp[R * wl.d:] = 7
    boff = layer.view("block_off")
    boff.copy_(torch.div(boff, 2, rounding_mode="floor"))
    layer.clear_status()
    layer.dispatch(x.cuda())
    torch.cuda.synchronize()
    assert layer.read_status() & N.MOE_STATUS_OVERFLOW
    assert (layer.row_token[R:] == canary).all()
    assert (layer.xp[R * wl.d:] == 7).all()
