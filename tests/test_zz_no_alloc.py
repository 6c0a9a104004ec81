"""The allocation-free FFN entry point (moe_expert_ffn_noalloc), for callers that cannot
allocate device memory: a plugin or custom operator that its host framework hands only
inputs and outputs, or a deployment that forbids cudaMalloc after start-up.

Through the C ABI it must give what moe_expert_ffn gives (with the caller's scratch), and
what the CPU oracle gives, on two calls in a row (the library's array keeps the previous
call's contents), within the parity tolerance 1e-2 + 2e-2|ref|, and refuse a problem whose
FC1 output does not fit its fixed array.  This file is collected last and runs the same
alone or after the others."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import native as N
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-2
CASES = [WORKLOADS["tiny"],
         Workload("ragged128", T=1111, d=512, E=12, k=4, f=384, beta=128, P=4, s=2, alpha=0.5)]


def _within(got: torch.Tensor, ref: torch.Tensor) -> bool:
    g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
    return bool(np.all(np.abs(g - r) <= ATOL + RTOL * np.abs(r)))


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [N.MOE_FFN_FUSED_COMBINE, N.MOE_FFN_WRITE_O])
def test_noalloc_matches_scratch_entry_point_twice(wl, mode):
    assert N.moe_workspace_size(wl, N.MOE_WS_FFN_SCRATCH) <= N.MOE_NOALLOC_SCRATCH_BYTES
    torch.manual_seed(0)
    logits, x = synth.make_logits(wl).cuda(), synth.make_x(wl).cuda()
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda", write_o=True, gather_x=False)
    layer.clear_status()
    layer.route(logits)
    layer.plan(0)
    layer.dispatch(x)
    out = layer.o if mode & N.MOE_FFN_WRITE_O else layer.y
    layer.ffn(w1, w2, mode)                         # caller-provided scratch
    torch.cuda.synchronize()
    ref = out.clone()
    W1, W2 = w1.float().cpu().numpy(), w2.float().cpu().numpy()
    oracle = O.moe_forward(synth.make_logits(wl).numpy(), synth.make_x(wl).float().numpy(),
                           lambda e: (W1[e], W2[e]), k=wl.k, beta=wl.beta, P=wl.P, s=wl.s)
    for call in range(2):
        out.fill_(float("nan"))
        N.moe_expert_ffn_noalloc(layer.cfg, layer.xp, w1, w2, layer.tiles, layer.plan_info,
                                 layer.row_token, layer.row_gate, mode, out, layer.status)
        torch.cuda.synchronize()
        assert layer.read_status() == 0, N.moe_status_string(layer.read_status())
        if mode & N.MOE_FFN_WRITE_O:
            R = wl.beta * int(layer.plan_info[N.PI["B"]])
            rows = layer.row_token[:R] >= 0
            got = out[: R * wl.d].view(R, wl.d)[rows]
            want = ref[: R * wl.d].view(R, wl.d)[rows]
            want_oracle = torch.from_numpy(oracle["O"][rows.cpu().numpy()])
        else:
            got = out[: wl.T * wl.d]
            want = ref[: wl.T * wl.d]
            want_oracle = torch.from_numpy(oracle["y"]).reshape(-1)
        assert _within(got, want), f"call {call}: against moe_expert_ffn"
        assert _within(got, want_oracle), f"call {call}: against the oracle"


def test_noalloc_refuses_a_problem_larger_than_its_array():
    wl = WORKLOADS["olmoe_a1"]
    assert N.moe_workspace_size(wl, N.MOE_WS_FFN_SCRATCH) > N.MOE_NOALLOC_SCRATCH_BYTES
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda", gather_x=False)
    cfg = N.MoeCfg.of(wl)
    rc = N.lib().moe_expert_ffn_noalloc(
        ctypes.byref(cfg), layer.xp.data_ptr(), w1.data_ptr(), w2.data_ptr(),
        layer.tiles.data_ptr(), layer.plan_info.data_ptr(), layer.row_token.data_ptr(),
        layer.row_gate.data_ptr(), 0, layer.y.data_ptr(), layer.status.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert rc == N.MOE_ERR_TOO_LARGE
    assert "too large" in N.moe_status_string(rc)
