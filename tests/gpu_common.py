"""Helpers shared by the GPU parity tests: run the oracle on a workload's inputs and run the
CUDA path on the same inputs through the C ABI."""
from __future__ import annotations

import functools

import numpy as np
import torch

from oracle import moe_oracle as O
from skew_aware_token_b200 import native as N
from skew_aware_token_b200 import synth
from skew_aware_token_b200.layer import MoeLayer

# |gpu - ref| <= ATOL + RTOL * |ref| per element of y (bf16 inputs, fp32 accumulation)
ATOL, RTOL = 1e-2, 2e-2
# gates: the GPU evaluates exp in fp32 from an fp32 logit difference (|diff| < 20 here),
# the oracle in fp64; relative error <= (|diff| + 8) * 2^-24 < 2e-6
GATE_RTOL = 4e-6


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


@functools.lru_cache(maxsize=8)
def host_inputs(wl):
    return synth.make_logits(wl), synth.make_x(wl)


def expected_tiles(q, block_off, beta):
    """The executor's tiles: per slot, experts ascending, each run of q[e][r] blocks
    (q[e][r] * beta consecutive rows) cut into tiles of 256 rows, the last possibly
    shorter."""
    q = np.asarray(q)
    E, P = q.shape
    tiles, slot_tile_off = [], [0]
    for r in range(P):
        for e in range(E):
            j0 = int(q[e, :r].sum())
            rows = int(q[e, r]) * beta
            for i in range(0, rows, 256):
                tiles.append((e, beta * (block_off[e] + j0) + i, min(256, rows - i), r))
        slot_tile_off.append(len(tiles))
    return tiles, slot_tile_off


def run_gpu(wl, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE, variant_mask=0, layer=None):
    logits, x = host_inputs(wl)
    # the test's mode runs as given (no switch to O rows for a large y)
    layer = layer or MoeLayer(wl, "cuda", write_o=bool(mode & N.MOE_FFN_WRITE_O), o_rows=False)
    layer.clear_status()
    layer(logits.cuda(), x.cuda(), w1, w2, mode=mode, variant_mask=variant_mask)
    torch.cuda.synchronize()
    return layer


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, what: str):
    err = np.abs(y_gpu - y_ref)
    bound = ATOL + RTOL * np.abs(y_ref)
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} of {bad.size} elements outside 1e-2 + 2e-2|ref| "
        f"(max err {err.max():.3e}, at {np.unravel_index(np.argmax(err - bound), err.shape)})")
    return float(err.max())
