"""Host-side checks of the C ABI: the library loads, exports every entry point the header
declares, sizes its workspaces by the stated bounds, and rejects bad arguments before
launching anything.  No GPU: the argument checks run before any CUDA call."""
import ctypes
import subprocess

import pytest
import torch

from skew_aware_token_b200 import build as B
from skew_aware_token_b200 import native as N
from skew_aware_token_b200.synth import WORKLOADS

NO_GPU = not torch.cuda.is_available()


@pytest.fixture(scope="module", autouse=True)
def built_library():
    B.build()
    return N.lib()


def test_exports_every_declared_symbol():
    declared = N.declared_symbols()
    assert set(declared) == {"moe_workspace_size", "moe_route_hist", "moe_plan_blocks",
                             "moe_dispatch_permute", "moe_expert_ffn", "moe_combine",
                             "moe_status_string", "moe_expert_ffn_noalloc",
                             "moe_dispatch_grad", "moe_expert_ffn_backward",
                             "moe_block_offsets"}
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared:
        assert name in exported, name
        assert hasattr(N.lib(), name)
    # nothing but the declared API is exported
    assert {s for s in exported if s.startswith("moe_")} == set(declared)


def test_workspace_sizes_follow_the_block_bound():
    for wl in WORKLOADS.values():
        Nr = wl.T * wl.k
        b_max = (Nr + min(wl.E, Nr) * (wl.beta - 1)) // wl.beta
        assert N.moe_workspace_size(wl, N.MOE_WS_BLOCKS) == b_max
        assert N.moe_workspace_size(wl, N.MOE_WS_ROWS) == b_max * wl.beta
        a_bytes = (b_max * wl.beta * wl.f * 2 + 255) // 256 * 256
        ready_bytes = (2 * b_max * 4 + 255) // 256 * 256  # one-launch readiness counters
        record_bytes = (b_max * 4 + 255) // 256 * 256     # slot record
        assert N.moe_workspace_size(wl, N.MOE_WS_FFN_RECORD) == a_bytes + 256 + ready_bytes
        assert N.moe_workspace_size(wl, N.MOE_WS_FFN_SCRATCH) == (a_bytes + 256 + ready_bytes +
                                                                   record_bytes)
        # the bound holds for the worst routing: every expert one row past a block
        worst = [wl.beta + 1] * wl.E
        if sum(worst) <= Nr:
            assert sum(-(-c // wl.beta) for c in worst) <= b_max


@pytest.mark.parametrize("field,value,code", [
    ("k", 9, N.MOE_ERR_INVALID_ARG), ("k", 0, N.MOE_ERR_INVALID_ARG),
    ("beta", 96, N.MOE_ERR_INVALID_ARG), ("P", 9, N.MOE_ERR_INVALID_ARG),
    ("P", 0, N.MOE_ERR_INVALID_ARG), ("s", -1, N.MOE_ERR_INVALID_ARG),
    ("T", -1, N.MOE_ERR_INVALID_ARG), ("E", 300, N.MOE_ERR_UNSUPPORTED),
    ("T", (1 << 21) + 1, N.MOE_ERR_UNSUPPORTED),
])
def test_bad_config_rejected_everywhere(field, value, code):
    wl = WORKLOADS["tiny"].with_(**{field: value})
    cfg = N.MoeCfg.of(wl)
    fake = 1 << 20  # never dereferenced: the config check comes first
    lib = N.lib()
    p = ctypes.byref(cfg)
    assert lib.moe_workspace_size(p, 0) == 0
    assert lib.moe_route_hist(p, *[fake] * 7, None) == code
    assert lib.moe_plan_blocks(p, fake, 0, *[fake] * 8, None) == code
    assert lib.moe_dispatch_permute(p, *[fake] * 9, None) == code
    assert lib.moe_expert_ffn(p, *[fake] * 7, 0, *[fake] * 3, None) == code
    assert lib.moe_combine(p, *[fake] * 5, None) == code


@pytest.mark.skipif(not NO_GPU, reason="fake pointers are only passed where no GPU exists")
def test_null_and_misaligned_pointers_rejected():
    cfg = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"]))
    lib = N.lib()
    ok = 1 << 20
    for i in range(7):
        args = [ok] * 7
        args[i] = None
        assert lib.moe_route_hist(cfg, *args, None) == N.MOE_ERR_INVALID_ARG
        args[i] = ok + 4
        assert lib.moe_route_hist(cfg, *args, None) == N.MOE_ERR_UNSUPPORTED
    for i in range(10):
        args = [ok] * 10
        args[i] = ok + 8
        assert lib.moe_expert_ffn(cfg, *args[:7], 0, *args[7:], None) == N.MOE_ERR_UNSUPPORTED
    # dispatch: xp may be NULL (row maps only), but not misaligned; the rest are required
    disp = [ok] * 9  # x, ids, gates, block_off, xp, row_token, row_gate, tok_row, status
    disp[4], disp[5] = None, None
    assert lib.moe_dispatch_permute(cfg, *disp, None) == N.MOE_ERR_INVALID_ARG
    disp[4], disp[5] = ok + 8, ok
    assert lib.moe_dispatch_permute(cfg, *disp, None) == N.MOE_ERR_UNSUPPORTED
    for bad_mask in (1 << 6, 1 << 7, 1 << 24, 0xFFFFFFFF):  # bits 6, 7 and 24..31 are unused
        assert lib.moe_plan_blocks(cfg, ok, bad_mask, *[ok] * 8, None) == N.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(cfg, *[ok] * 7, 2048, *[ok] * 3, None) == N.MOE_ERR_INVALID_ARG
    bad_d = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"].with_(d=320)))
    assert lib.moe_expert_ffn(bad_d, *[ok] * 7, 0, *[ok] * 3, None) == N.MOE_ERR_UNSUPPORTED
    bad_f = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"].with_(f=192)))
    assert lib.moe_expert_ffn(bad_f, *[ok] * 7, 0, *[ok] * 3, None) == N.MOE_ERR_UNSUPPORTED


def test_status_strings():
    assert N.moe_status_string(0) == "ok"
    for code in (-1, -2, -3, -4, 1, 2, 4, 8, 16):
        assert N.moe_status_string(code) not in ("", "unknown code")


def test_binding_refuses_host_tensors():
    with pytest.raises(TypeError):
        N.moe_route_hist(WORKLOADS["tiny"], torch.zeros(4), *[torch.zeros(4)] * 6)


def test_layer_api_surface():
    from skew_aware_token_b200.layer import HostPipeline, MoeLayer
    for name in ("route", "plan", "dispatch", "ffn", "combine", "forward_host", "clear_status",
                 "read_status", "view", "__call__"):
        assert callable(getattr(MoeLayer, name)), name
    for name in ("submit", "drain"):
        assert callable(getattr(HostPipeline, name)), name


def test_header_constants_match_binding():
    """plan_info indices, FFN modes and error codes: the header's enums and the binding's
    constants are the same numbers."""
    import re
    text = open(N.HEADER_PATH).read()
    enum = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(MOE_\w+)\s*=\s*(-?\d+)", text)}
    for key, val in N.PI.items():
        assert enum["MOE_PI_" + key] == val, key
    for name in ("MOE_FFN_FUSED_COMBINE", "MOE_FFN_WRITE_O", "MOE_FFN_STRICT_SLOTS",
                 "MOE_FFN_SM_PAIR", "MOE_FFN_GATHER_X", "MOE_ERR_TOO_LARGE"):
        assert enum[name] == getattr(N, name), name
    assert N.variant_mask() == 0 and N.variant_mask([4], u_min=3) == (1 << 4) | (3 << 8)


@pytest.mark.skipif(not NO_GPU, reason="fake pointers are only passed where no GPU exists")
def test_backward_entry_points_reject_bad_arguments():
    cfg = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"]))
    lib = N.lib()
    ok = 1 << 20
    for i in range(14):
        args = [ok] * 14
        args[i] = None
        assert lib.moe_expert_ffn_backward(cfg, *args, None) == N.MOE_ERR_INVALID_ARG, i
        args[i] = ok + 8
        assert lib.moe_expert_ffn_backward(cfg, *args, None) == N.MOE_ERR_UNSUPPORTED, i
    for i in range(6):
        args = [ok] * 6
        args[i] = None
        assert lib.moe_dispatch_grad(cfg, *args, None) == N.MOE_ERR_INVALID_ARG, i
    bad_d = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"].with_(d=320)))
    assert lib.moe_expert_ffn_backward(bad_d, *[ok] * 14, None) == N.MOE_ERR_UNSUPPORTED
    # the allocation-free forward cannot keep Z for a backward pass
    assert lib.moe_expert_ffn_noalloc(cfg, *[ok] * 7, N.MOE_FFN_SAVE_Z, *[ok] * 2,
                                      None) == N.MOE_ERR_INVALID_ARG


def test_training_workspace_sizes():
    for wl in (WORKLOADS["tiny"], WORKLOADS["olmoe_a1"], WORKLOADS["dsv3_a1"]):
        R = N.moe_workspace_size(wl, N.MOE_WS_ROWS)
        base = N.moe_workspace_size(wl, N.MOE_WS_FFN_SCRATCH)
        z_bytes = -(-R * 2 * wl.f * 2 // 256) * 256
        assert N.moe_workspace_size(wl, N.MOE_WS_FFN_SCRATCH_Z) == base + z_bytes
        assert N.moe_workspace_size(wl, N.MOE_WS_BWD_SCRATCH) == z_bytes + 256


@pytest.mark.skipif(not NO_GPU, reason="fake pointers are only passed where no GPU exists")
def test_one_launch_rejects_unsupported_combinations():
    cfg = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"]))
    lib = N.lib()
    ok = 1 << 20
    for other in (N.MOE_FFN_WRITE_O, N.MOE_FFN_STRICT_SLOTS, N.MOE_FFN_SM_PAIR,
                  N.MOE_FFN_GATHER_X, N.MOE_FFN_TWO_LAUNCHES):
        for flag in (N.MOE_FFN_ONE_LAUNCH, N.MOE_FFN_TEST_WAIT_TIMEOUT):
            assert lib.moe_expert_ffn(cfg, *[ok] * 7, flag | other, *[ok] * 3,
                                      None) == N.MOE_ERR_INVALID_ARG
        mode = N.MOE_FFN_ONE_LAUNCH | other
        assert lib.moe_expert_ffn_noalloc(cfg, *[ok] * 7, mode, *[ok] * 2,
                                          None) == N.MOE_ERR_INVALID_ARG


@pytest.mark.skipif(not NO_GPU, reason="fake pointers are only passed where no GPU exists")
def test_noalloc_refuses_modes_its_fixed_array_cannot_serve():
    """MOE_FFN_SAVE_Z (Z belongs in the caller's scratch) and MOE_FFN_RECORD_SLOTS (the
    record could not be read back) are refused before any CUDA call."""
    cfg = ctypes.byref(N.MoeCfg.of(WORKLOADS["tiny"]))
    ok = 1 << 20
    lib = N.lib()
    for flag in (N.MOE_FFN_SAVE_Z, N.MOE_FFN_RECORD_SLOTS):
        assert lib.moe_expert_ffn_noalloc(cfg, *[ok] * 7, flag, ok, ok, None) == \
            N.MOE_ERR_INVALID_ARG
