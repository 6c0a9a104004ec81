"""The P virtual execution slots on one GPU ("MegaFlux" summary, Methodology 1, "Problem
Formulation": q_er blocks of expert e run on GPU r; here GPU r is slot r).

With MOE_FFN_STRICT_SLOTS the FFN's execution unit u (an SM, or an SM pair) only runs tiles
of slot u mod P, so the layer time follows the plan's makespan.  The kernels' slot record
(MOE_FFN_RECORD_SLOTS) shows which slots' units ran each tile: strict mode must confine
every tile's FC1 and FC2 items to its own slot, in every FFN configuration; the default
work-conserving mode lets units of any slot take a tile."""
import numpy as np
import pytest
import torch

from skew_aware_token_b200 import native as N
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer
from skew_aware_token_b200.synth import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

CASES = [WORKLOADS["olmoe_a1"],
         Workload("ragged128", T=1111, d=512, E=12, k=4, f=384, beta=128, P=4, s=2, alpha=0.5),
         Workload("hot_all", T=515, d=256, E=16, k=4, f=128, beta=64, P=8, s=2, hot_p=1.0,
                  hot_mode="all4")]
CONFIGS = {
    "default": 0,
    "fc1_tile_halves": N.MOE_FFN_FC1_M128,
    "o_rows": N.MOE_FFN_WRITE_O,
    "fc2_whole": N.MOE_FFN_FC2_WHOLE,
    "sm_pair": N.MOE_FFN_SM_PAIR,
}


def _run(wl, mode, layer=None):
    w1, w2 = synth.make_weights(wl, "cuda")
    logits, x = synth.make_logits(wl).cuda(), synth.make_x(wl).cuda()
    # o_rows=False: each configuration runs as written (the layer's own choice would add O
    # rows to the fused-combine ones)
    layer = layer or MoeLayer(wl, "cuda", write_o=True, o_rows=False)
    layer.clear_status()
    layer(logits, x, w1, w2, mode=mode | N.MOE_FFN_RECORD_SLOTS)
    torch.cuda.synchronize()
    assert layer.read_status() == 0, N.moe_status_string(layer.read_status())
    ntiles = int(layer.plan_info[N.PI["NTILES"]])
    tiles = layer.view("tiles").cpu().numpy()[:ntiles]
    rec = layer.view("slot_record").cpu().numpy()[:ntiles]
    return layer, tiles, rec


@pytest.mark.parametrize("cfg", list(CONFIGS), ids=list(CONFIGS))
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_strict_slots_confine_every_tile_to_its_slot(wl, cfg):
    layer, tiles, rec = _run(wl, CONFIGS[cfg] | N.MOE_FFN_STRICT_SLOTS)
    slot = tiles[:, 3]
    want = (1 << slot) | (1 << (8 + slot))  # FC1 and FC2 items ran on units of its slot only
    bad = np.nonzero(rec != want)[0]
    assert bad.size == 0, (f"{wl.name} {cfg}: tiles {bad[:8]} slots {slot[bad[:8]]} "
                           f"record {[hex(v) for v in rec[bad[:8]]]}")
    # tiles of every slot the plan gave work to were run
    assert set(np.unique(slot)) == {r for r in range(wl.P) if layer.view("slot_load")[r] > 0}


@pytest.mark.parametrize("wl", [CASES[0]], ids=lambda w: w.name)
def test_default_mode_shares_tiles_across_slots(wl):
    """Without strict slots any unit takes any tile: every tile still runs both GEMMs, and
    units of slots other than the tile's own take part."""
    _, tiles, rec = _run(wl, 0)
    assert np.all(rec & 0xFF) and np.all(rec >> 8)
    foreign = (rec & ~((1 << tiles[:, 3]) | (1 << (8 + tiles[:, 3])))) != 0
    assert foreign.mean() > 0.5


def test_recording_does_not_change_the_output():
    wl = CASES[1]
    layer, _, _ = _run(wl, N.MOE_FFN_STRICT_SLOTS)
    y_rec = layer.view("y").clone()
    w1, w2 = synth.make_weights(wl, "cuda")
    layer(synth.make_logits(wl).cuda(), synth.make_x(wl).cuda(), w1, w2,
          mode=N.MOE_FFN_STRICT_SLOTS)
    torch.cuda.synchronize()
    torch.testing.assert_close(layer.view("y"), y_rec, rtol=1e-5, atol=1e-6)
