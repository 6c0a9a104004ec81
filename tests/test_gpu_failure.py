"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The one-launch FFN's FC2 producers wait (bounded) for FC1 to publish each tile half's
activation rows.  MOE_FFN_TEST_WAIT_TIMEOUT sets the readiness target one above what FC1
reaches and limits waits to 10 ms: every such wait gives up, the kernel's roles drop out,
drain their own copies and MMAs, free TMEM and return.  The call must report
MOE_STATUS_TIMEOUT, and the next normal call on the same context must be correct."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import native as N
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import Workload

from gpu_common import check_y, f32, host_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    wl = Workload("ragged128", T=1111, d=512, E=12, k=4, f=384, beta=128, P=4, s=2, alpha=0.5)
    logits, x = host_inputs(wl)
    w1, w2 = synth.make_weights(wl, "cuda")
    layer = MoeLayer(wl, "cuda")
    layer.route(logits.cuda())
    layer.plan(0)
    layer.dispatch(x.cuda())
    layer.clear_status()
    layer.ffn(w1, w2, N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_TEST_WAIT_TIMEOUT)
    torch.cuda.synchronize()
    status = layer.read_status()
    assert status & N.MOE_STATUS_TIMEOUT, N.moe_status_string(status)
    # the context is intact: the same buffers, a normal call, the oracle's y
    layer.clear_status()
    layer.ffn(w1, w2, N.MOE_FFN_FUSED_COMBINE | N.MOE_FFN_ONE_LAUNCH)
    torch.cuda.synchronize()
    assert layer.read_status() == 0
    W1, W2 = f32(w1), f32(w2)
    ref = O.moe_forward(logits.numpy(), x.float().numpy(), lambda e: (W1[e], W2[e]),
                        k=wl.k, beta=wl.beta, P=wl.P, s=wl.s)
    check_y(f32(layer.view("y")), ref["y"], "after a timed-out call")
