"""ctypes binding of libmoeskew.so: the C ABI of include/moeskew.h, same names, argument
marshalling only (torch tensors -> device pointers, the current CUDA stream).

Every step of the layer runs in the library's CUDA kernels.  There is no fallback: if the
library is missing this module raises, and every pointer argument must be a CUDA tensor.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoeskew.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "include", "moeskew.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, -1, -2, -3
MOE_ERR_TOO_LARGE = -4
MOE_NOALLOC_SCRATCH_BYTES = 64 << 20
MOE_STATUS_BAD_ID, MOE_STATUS_OVERFLOW, MOE_STATUS_NONFINITE = 1, 2, 4
MOE_STATUS_TIMEOUT, MOE_STATUS_PLAN = 8, 16
MOE_WS_ROWS, MOE_WS_BLOCKS, MOE_WS_FFN_SCRATCH = 0, 1, 2
MOE_WS_FFN_SCRATCH_Z, MOE_WS_BWD_SCRATCH, MOE_WS_FFN_RECORD = 3, 4, 5
MOE_FFN_FUSED_COMBINE, MOE_FFN_WRITE_O, MOE_FFN_STRICT_SLOTS, MOE_FFN_SM_PAIR = 0, 1, 2, 4
MOE_FFN_GATHER_X = 8
MOE_FFN_SAVE_Z = 16
MOE_FFN_ONE_LAUNCH = 32
MOE_FFN_TWO_LAUNCHES = 64
MOE_FFN_TEST_WAIT_TIMEOUT = 128
MOE_FFN_FC1_M128 = 256
MOE_FFN_FC2_WHOLE = 512
MOE_FFN_RECORD_SLOTS = 1024
PI = dict(B=0, TAU=1, MAKESPAN=2, VARIANT=3, NTILES=4, FIXED_MAKESPAN=5, REPLICAS=6,
          ROUNDS=7, SLOT_TILE_OFF=8, VAR_MAKESPAN=17, VAR_REPLICAS=22, VAR_ROUNDS=27,
          QUOTA_TAU=32, COST=33, VAR_COST=34, LEN=40)
N_VARIANTS = 5          # planner variants: 0..3 bounded greedy, 4 quota solver
QUOTA_VARIANT = 4


def variant_mask(variants=(), u_min: int = 1, lam: int | None = None) -> int:
    """moe_plan_blocks's variant_mask: enabled variants (none = the four greedy searches),
    the quota solver's floor u_min in blocks and, with `lam`, reduction-aware selection
    with that lambda (1..255; 12 on the pages)."""
    m = 0
    for v in variants:
        m |= 1 << v
    if not 1 <= u_min <= 255:
        raise ValueError("u_min must be in 1..255 blocks")
    if u_min != 1:
        m |= u_min << 8
    if lam is not None:
        if not 1 <= lam <= 255:
            raise ValueError("lambda must be in 1..255")
        m |= 1 << 5 | (0 if lam == 12 else lam << 16)
    return m


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code}: {moe_status_string(code)}")
        self.code = code


class MoeCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "d", "E", "k", "f", "beta", "P", "s")]

    @classmethod
    def of(cls, wl) -> "MoeCfg":
        return cls(wl.T, wl.d, wl.E, wl.k, wl.f, wl.beta, wl.P, wl.s)


_VP = ctypes.c_void_p
_SIGNATURES = {
    "moe_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(MoeCfg), ctypes.c_int]),
    "moe_route_hist": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 8),
    "moe_block_offsets": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 3),
    "moe_plan_blocks": (ctypes.c_int, [ctypes.POINTER(MoeCfg), _VP, ctypes.c_uint32] + [_VP] * 9),
    "moe_dispatch_permute": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 10),
    "moe_expert_ffn": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 7 + [ctypes.c_int] +
                       [_VP] * 4),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 6),
    "moe_expert_ffn_noalloc": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 7 +
                               [ctypes.c_int] + [_VP] * 3),
    "moe_dispatch_grad": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 7),
    "moe_expert_ffn_backward": (ctypes.c_int, [ctypes.POINTER(MoeCfg)] + [_VP] * 15),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m skew_aware_token_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def declared_symbols() -> list[str]:
    """Names of the entry points include/moeskew.h declares."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def _dev(t, name):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def _cfg(cfg) -> MoeCfg:
    return cfg if isinstance(cfg, MoeCfg) else MoeCfg.of(cfg)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def moe_workspace_size(cfg, which: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(_cfg(cfg)), which))


def moe_route_hist(cfg, logits, topk_ids, topk_gates, counts, sumsq, kappa, status,
                   stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_route_hist", lib().moe_route_hist(
        ctypes.byref(c), _dev(logits, "logits"), _dev(topk_ids, "topk_ids"),
        _dev(topk_gates, "topk_gates"), _dev(counts, "counts"), _dev(sumsq, "sumsq"),
        _dev(kappa, "kappa"), _dev(status, "status"), _stream(stream)))


def moe_block_offsets(cfg, counts, block_off, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_block_offsets", lib().moe_block_offsets(
        ctypes.byref(c), _dev(counts, "counts"), _dev(block_off, "block_off"), _stream(stream)))


def moe_plan_blocks(cfg, counts, variant_mask, block_off, q, slot_load, slot_off, blocks,
                    tiles, plan_info, status, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_plan_blocks", lib().moe_plan_blocks(
        ctypes.byref(c), _dev(counts, "counts"), int(variant_mask), _dev(block_off, "block_off"),
        _dev(q, "q"), _dev(slot_load, "slot_load"), _dev(slot_off, "slot_off"),
        _dev(blocks, "blocks"), _dev(tiles, "tiles"), _dev(plan_info, "plan_info"),
        _dev(status, "status"), _stream(stream)))


def moe_dispatch_permute(cfg, x, topk_ids, topk_gates, block_off, xp, row_token, row_gate,
                         tok_row, status, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_dispatch_permute", lib().moe_dispatch_permute(
        ctypes.byref(c), _dev(x, "x"), _dev(topk_ids, "topk_ids"), _dev(topk_gates, "topk_gates"),
        _dev(block_off, "block_off"), _dev(xp, "xp"), _dev(row_token, "row_token"),
        _dev(row_gate, "row_gate"), _dev(tok_row, "tok_row"), _dev(status, "status"),
        _stream(stream)))


def moe_expert_ffn(cfg, xp, w1, w2, tiles, plan_info, row_token, row_gate, mode, a_scratch,
                   out, status, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(c), _dev(xp, "xp"), _dev(w1, "w1"), _dev(w2, "w2"), _dev(tiles, "tiles"),
        _dev(plan_info, "plan_info"), _dev(row_token, "row_token"), _dev(row_gate, "row_gate"),
        int(mode), _dev(a_scratch, "a_scratch"), _dev(out, "out"), _dev(status, "status"),
        _stream(stream)))


def moe_dispatch_grad(cfg, dy, row_token, row_gate, plan_info, d_rows, status,
                      stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_dispatch_grad", lib().moe_dispatch_grad(
        ctypes.byref(c), _dev(dy, "dy"), _dev(row_token, "row_token"),
        _dev(row_gate, "row_gate"), _dev(plan_info, "plan_info"), _dev(d_rows, "d_rows"),
        _dev(status, "status"), _stream(stream)))


def moe_expert_ffn_backward(cfg, xp, w1, w2, tiles, plan_info, block_off, row_token, d_rows,
                            saved, bwd_scratch, dx, dw1, dw2, status, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_expert_ffn_backward", lib().moe_expert_ffn_backward(
        ctypes.byref(c), _dev(xp, "xp"), _dev(w1, "w1"), _dev(w2, "w2"), _dev(tiles, "tiles"),
        _dev(plan_info, "plan_info"), _dev(block_off, "block_off"),
        _dev(row_token, "row_token"), _dev(d_rows, "d_rows"), _dev(saved, "saved"),
        _dev(bwd_scratch, "bwd_scratch"), _dev(dx, "dx"), _dev(dw1, "dw1"), _dev(dw2, "dw2"),
        _dev(status, "status"), _stream(stream)))


def moe_combine(cfg, o, tok_row, topk_gates, y, status, stream=None) -> None:
    c = _cfg(cfg)
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(c), _dev(o, "o"), _dev(tok_row, "tok_row"), _dev(topk_gates, "topk_gates"),
        _dev(y, "y"), _dev(status, "status"), _stream(stream)))


def moe_expert_ffn_noalloc(cfg, xp, w1, w2, tiles, plan_info, row_token, row_gate, mode, out,
                           status, stream=None) -> None:
    """moe_expert_ffn without a caller scratch buffer (the library's fixed array holds A)."""
    c = _cfg(cfg)
    _check("moe_expert_ffn_noalloc", lib().moe_expert_ffn_noalloc(
        ctypes.byref(c), _dev(xp, "xp"), _dev(w1, "w1"), _dev(w2, "w2"), _dev(tiles, "tiles"),
        _dev(plan_info, "plan_info"), _dev(row_token, "row_token"), _dev(row_gate, "row_gate"),
        int(mode), _dev(out, "out"), _dev(status, "status"), _stream(stream)))
