"""The forward MoE layer as one call: owns the device buffers of one configuration and
strings the C-ABI calls together (route + histogram, block offsets, plan, dispatch, expert
FFN, and the combine when the FFN writes O) on the current CUDA stream, the planner's search
on a second stream beside the dispatch.

    layer = MoeLayer(workload, device="cuda")
    y = layer(logits, x, w1, w2)          # device tensors in, y fp32 [T, d] out
    y_host = layer.forward_host(...)      # pinned host tensors in and out (end to end)
"""
from __future__ import annotations

import torch

from . import native as N


# From this size of y on, a fused-combine call of the layer runs FC2 with O rows plus the
# ordered combine instead: the fused combine's fp32 reductions compete with the operand
# copies for L2 (and go to DRAM once y outgrows it), while O rows leave through TMA stores
# (the epilogue frees each accumulator half before staging them) and the combine reads them
# once.  Measured FFN + combine times against the fused combine: DeepSeek-V3-shaped layer with
# 32 experts (59 MB y) 3 % faster, 4096-token layers (32 MiB y) 1-4 % faster, and the larger
# layers as fast or faster; the 256-token layer stays fused.  The ordered combine also makes
# y independent of the reduction order.
O_ROWS_MIN_Y_BYTES = 32 << 20


class MoeLayer:
    def __init__(self, wl, device="cuda", write_o: bool = False, guard: int = 0,
                 gather_x: bool = False, train: bool = False, o_rows: bool | None = None):
        """`guard` adds that many spare elements after every buffer (canary checks).
        `write_o`: also hold the O buffer (bf16 [R_max, d]) for MOE_FFN_WRITE_O calls.
        `o_rows`: how a call in the fused-combine mode runs the combine: True, FC2 writes O
        rows and moe_combine adds each token's k rows in order; False, FC2 adds into y
        itself; None (default), O rows when y (T x d fp32) holds at least
        O_ROWS_MIN_Y_BYTES.
        `gather_x`: FC1 gathers its rows from x by row_token (MOE_FFN_GATHER_X) and the
        dispatched copy Xp is neither allocated nor written (saves R_max * d * 2 bytes; as
        fast while x stays resident in L2, slower once it does not); False (default)
        materialises Xp with the dispatch gather.
        `train`: the forward keeps Z = [G, U] (MOE_FFN_SAVE_Z) and the layer holds the
        backward's buffers (D rows, dZ scratch, dx, dW1, dW2); needs the Xp path."""
        if train and gather_x:
            raise ValueError("the backward pass reads Xp: train=True needs gather_x=False")
        self.cfg = N.MoeCfg.of(wl)
        self.wl = wl
        dev = torch.device(device)
        T, d, E, k, f, P = wl.T, wl.d, wl.E, wl.k, wl.f, wl.P
        R = N.moe_workspace_size(self.cfg, N.MOE_WS_ROWS)
        Bm = N.moe_workspace_size(self.cfg, N.MOE_WS_BLOCKS)
        if R == 0 and T > 0:
            raise ValueError("configuration rejected by moe_workspace_size")
        self.R_max, self.B_max = R, Bm
        i32, f32 = torch.int32, torch.float32
        z = lambda n, dt=i32: torch.zeros(n + guard, dtype=dt, device=dev)
        # at least one 16-byte granule per buffer so every pointer is valid and aligned
        self.topk_ids = z(max(T * k, 4))
        self.topk_gates = z(max(T * k, 4), dt=f32)
        self.counts = z(max(E, 4))
        self.sumsq = z(2, dt=torch.int64)
        self.kappa = z(2, dt=torch.float64)
        self.status = z(4)
        self.block_off = z(E + 4)       # written by moe_block_offsets, read by the dispatch
        self.block_off_plan = z(E + 4)  # the planner's own copy (same values)
        self.q = z(max(E * P, 4))
        self.slot_load = z(8)
        self.slot_off = z(12)
        self.blocks = z(max(2 * Bm, 4))
        self.tiles = z(max(4 * Bm, 4))
        self.plan_info = z(N.PI["LEN"])
        self.gather_x = gather_x
        self.xp = None if gather_x else z(max(R * d, 8), dt=torch.bfloat16)
        self.row_token = z(max(R, 4))
        self.row_gate = z(max(R, 4), dt=f32)
        self.tok_row = z(max(T * k, 4))
        self.train = train
        ws = N.moe_workspace_size(self.cfg, N.MOE_WS_FFN_SCRATCH_Z if train
                                  else N.MOE_WS_FFN_SCRATCH)
        self.a_scratch = z(max(ws // 2, 8), dt=torch.bfloat16)
        if train:
            self.d_rows = z(max(R * d, 8), dt=torch.bfloat16)
            bws = N.moe_workspace_size(self.cfg, N.MOE_WS_BWD_SCRATCH)
            self.bwd_scratch = z(max(bws // 2, 8), dt=torch.bfloat16)
            self.dx = z(max(T * d, 4), dt=f32)
            self.dw1 = z(max(E * 2 * f * d, 4), dt=f32)
            self.dw2 = z(max(E * d * f, 4), dt=f32)
        self.y = z(max(T * d, 4), dt=f32)
        self.o_rows = (T * d * 4 >= O_ROWS_MIN_Y_BYTES) if o_rows is None else bool(o_rows)
        self.o = z(max(R * d, 8), dt=torch.bfloat16) if (write_o or self.o_rows) else None
        self.device = dev
        self._side = torch.cuda.Stream(dev) if dev.type == "cuda" else None

    # ------------------------------------------------------------------ stages
    def route(self, logits, stream=None):
        N.moe_route_hist(self.cfg, logits, self.topk_ids, self.topk_gates, self.counts,
                         self.sumsq, self.kappa, self.status, stream)

    def block_offsets(self, stream=None):
        N.moe_block_offsets(self.cfg, self.counts, self.block_off, stream)

    def plan(self, variant_mask=0, stream=None):
        """Block offsets (what the dispatch needs), then the plan."""
        self.block_offsets(stream)
        self._search(variant_mask, stream)

    def _search(self, variant_mask, stream):
        N.moe_plan_blocks(self.cfg, self.counts, variant_mask, self.block_off_plan, self.q,
                          self.slot_load, self.slot_off, self.blocks, self.tiles,
                          self.plan_info, self.status, stream)

    def dispatch(self, x, stream=None):
        """Row maps (and, without gather_x, the dispatched rows Xp)."""
        N.moe_dispatch_permute(self.cfg, x, self.topk_ids, self.topk_gates, self.block_off,
                               self.xp, self.row_token, self.row_gate, self.tok_row,
                               self.status, stream)

    def ffn_mode(self, mode=N.MOE_FFN_FUSED_COMBINE) -> int:
        """The mode a layer call runs the FFN in: with o_rows, MOE_FFN_WRITE_O is added to a
        fused-combine mode (the layer then runs moe_combine after the FFN), except to one
        that asks for the one-launch FFN, which fuses the combine by design."""
        if self.o_rows and not mode & N.MOE_FFN_ONE_LAUNCH:
            return mode | N.MOE_FFN_WRITE_O
        return mode

    def ffn(self, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE, stream=None, y=None, x=None):
        """The expert FFN; `x` (the token rows) is needed when the layer gathers them."""
        out = self.o if mode & N.MOE_FFN_WRITE_O else (self.y if y is None else y)
        if out is None:
            raise ValueError("layer built without an O buffer (write_o=False)")
        if self.gather_x:
            if x is None:
                raise ValueError("gather_x layer: ffn() needs the token rows x")
            src, mode = x, mode | N.MOE_FFN_GATHER_X
        else:
            src = self.xp
        if self.train:
            mode |= N.MOE_FFN_SAVE_Z
        N.moe_expert_ffn(self.cfg, src, w1, w2, self.tiles, self.plan_info,
                         self.row_token, self.row_gate, mode, self.a_scratch, out,
                         self.status, stream)

    def combine(self, stream=None, y=None):
        N.moe_combine(self.cfg, self.o, self.tok_row, self.topk_gates,
                      self.y if y is None else y, self.status, stream)

    # ------------------------------------------------------------------ whole layer
    def __call__(self, logits, x, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE, variant_mask=0,
                 stream=None, y=None):
        """Route, plan, dispatch, FFN (+ combine): returns y fp32 [T, d], by default a view
        of the layer's buffer (valid until the next call), or the caller's `y`."""
        mode = self.ffn_mode(mode)
        self.pre_ffn(logits, x, variant_mask, stream)
        self.ffn(w1, w2, mode, stream, y, x)
        if mode & N.MOE_FFN_WRITE_O:
            self.combine(stream, y)
        out = self.y if y is None else y
        return out[: self.wl.T * self.wl.d].view(self.wl.T, self.wl.d)

    def pre_ffn(self, logits, x, variant_mask=0, stream=None):
        """The stages before the FFN: route + histogram, block offsets, then the planner's
        search on a side stream while the dispatch runs (the dispatch needs only the block
        offsets); both join on the main stream."""
        self.route(logits, stream)
        self.block_offsets(stream)
        main = stream if isinstance(stream, torch.cuda.Stream) else \
            torch.cuda.current_stream(self.device) if stream is None else None
        if main is not None:
            self._side.wait_stream(main)
            with torch.cuda.stream(self._side):
                self._search(variant_mask, None)
            self.dispatch(x, main)
            main.wait_stream(self._side)
        else:  # a raw stream handle: one stream
            self._search(variant_mask, stream)
            self.dispatch(x, stream)

    def backward(self, dy, w1, w2, stream=None):
        """Gradients of the expert computation for dL/dy = dy (fp32 [T, d]) after a forward
        call of this layer: returns views of dx [T, d], dW1 [E, 2f, d], dW2 [E, d, f]."""
        if not self.train:
            raise ValueError("layer built without train=True")
        N.moe_dispatch_grad(self.cfg, dy, self.row_token, self.row_gate, self.plan_info,
                            self.d_rows, self.status, stream)
        N.moe_expert_ffn_backward(self.cfg, self.xp, w1, w2, self.tiles, self.plan_info,
                                  self.block_off, self.row_token, self.d_rows, self.a_scratch,
                                  self.bwd_scratch, self.dx, self.dw1, self.dw2, self.status,
                                  stream)
        return self.view("dx"), self.view("dw1"), self.view("dw2")

    def forward_host(self, logits_h, x_h, w1, w2, y_h, logits_d, x_d, mode=0, stream=None):
        """End to end from pinned host buffers: copies logits and x in, runs the layer,
        copies y out (all asynchronous on the current stream)."""
        logits_d.copy_(logits_h, non_blocking=True)
        x_d.copy_(x_h, non_blocking=True)
        y = self(logits_d, x_d, w1, w2, mode=mode, stream=stream)
        y_h.copy_(y, non_blocking=True)
        return y_h


    def clear_status(self):
        self.status.zero_()

    def read_status(self) -> int:
        return int(self.status[0].item())

    def view(self, name):
        """Typed views of the layer's buffers (for tests and reports)."""
        wl = self.wl
        T, d, E, k, P = wl.T, wl.d, wl.E, wl.k, wl.P
        R, Bm = self.R_max, self.B_max
        shapes = {
            "topk_ids": (self.topk_ids, (T, k)), "topk_gates": (self.topk_gates, (T, k)),
            "counts": (self.counts, (E,)), "block_off": (self.block_off, (E + 1,)),
            "q": (self.q, (E, P)), "slot_load": (self.slot_load, (P,)),
            "slot_off": (self.slot_off, (P + 1,)), "blocks": (self.blocks, (Bm, 2)),
            "tiles": (self.tiles, (Bm, 4)),
            "row_token": (self.row_token, (R,)), "row_gate": (self.row_gate, (R,)),
            "tok_row": (self.tok_row, (T, k)), "a_scratch": (self.a_scratch, (R, wl.f)),
            "y": (self.y, (T, d)),
        }
        if self.o is not None:
            shapes["o"] = (self.o, (R, d))
        if self.xp is not None:
            shapes["xp"] = (self.xp, (R, d))
        if self.train:
            f = wl.f
            z_off = N.moe_workspace_size(self.cfg, N.MOE_WS_FFN_SCRATCH) // 2
            shapes.update({
                "z": (self.a_scratch[z_off:], (R, 2 * f)), "d_rows": (self.d_rows, (R, d)),
                "dz": (self.bwd_scratch, (R, 2 * f)), "dx": (self.dx, (T, d)),
                "dw1": (self.dw1, (E, 2 * f, d)), "dw2": (self.dw2, (E, d, f))})
        if name == "slot_record":
            # int32 [B_max] at a byte offset of the FFN scratch (MOE_FFN_RECORD_SLOTS)
            off = N.moe_workspace_size(self.cfg, N.MOE_WS_FFN_RECORD) // 2
            return self.a_scratch[off: off + 2 * Bm].view(torch.int32)
        buf, shape = shapes[name]
        n = 1
        for s in shape:
            n *= s
        return buf[:n].view(*shape)


class LayerGraph:
    """One forward of a MoeLayer (route, plan, dispatch, FFN and, unfused, the combine)
    captured into a CUDA graph: replay() runs it again on whatever `logits` and `x` hold,
    with one launch from the host.  The layer's own buffers hold the results.

        g = LayerGraph(layer, w1, w2)
        g.logits.copy_(logits); g.x.copy_(x); g.replay(); y = layer.view("y")
    """

    def __init__(self, layer: MoeLayer, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE, variant_mask=0,
                 warmup: int = 2):
        wl, dev = layer.wl, layer.device
        self.layer = layer
        self.logits = torch.zeros(wl.T, wl.E, device=dev)
        self.x = torch.zeros(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
        run = lambda: layer(self.logits, self.x, w1, w2, mode=mode, variant_mask=variant_mask)
        # warm up off the capture (the library sets its kernels' attributes on first use)
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for _ in range(warmup):
                run()
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            run()

    def replay(self):
        self.graph.replay()


class HostPipeline:
    """Runs a MoeLayer over a stream of batches held in pinned host memory, overlapping
    the host-to-device copy of batch i+1 and the device-to-host copy of batch i-1 with the
    layer's work on batch i (three CUDA streams, two device buffer sets).

        pipe = HostPipeline(layer)
        for logits_h, x_h, y_h in batches:
            pipe.submit(logits_h, x_h, y_h, w1, w2)
        pipe.drain()
    """

    def __init__(self, layer: MoeLayer, depth: int = 2):
        wl, dev = layer.wl, layer.device
        self.layer, self.depth = layer, depth
        self.s_in = torch.cuda.Stream(dev)
        self.s_run = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.logits = [torch.empty(wl.T, wl.E, device=dev) for _ in range(depth)]
        self.x = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=dev)
                  for _ in range(depth)]
        self.y = [torch.empty(max(wl.T * wl.d, 4), device=dev) for _ in range(depth)]
        ev = lambda: torch.cuda.Event()
        self.in_done = [ev() for _ in range(depth)]    # inputs of slot landed
        self.run_done = [ev() for _ in range(depth)]   # layer finished with slot
        self.out_done = [ev() for _ in range(depth)]   # y of slot read back
        self.used = [False] * depth
        self.i = 0

    def submit(self, logits_h, x_h, y_h, w1, w2, mode=N.MOE_FFN_FUSED_COMBINE):
        b = self.i % self.depth
        self.i += 1
        if self.used[b]:
            # the slot's inputs are free once the layer ran, its y once it was read back
            self.s_in.wait_event(self.run_done[b])
            self.s_run.wait_event(self.out_done[b])
        self.used[b] = True
        with torch.cuda.stream(self.s_in):
            self.logits[b].copy_(logits_h, non_blocking=True)
            self.x[b].copy_(x_h, non_blocking=True)
            self.in_done[b].record(self.s_in)
        self.s_run.wait_event(self.in_done[b])
        with torch.cuda.stream(self.s_run):
            y = self.layer(self.logits[b], self.x[b], w1, w2, mode=mode, y=self.y[b])
            self.run_done[b].record(self.s_run)
        self.s_out.wait_event(self.run_done[b])
        with torch.cuda.stream(self.s_out):
            y_h.copy_(y, non_blocking=True)
            self.out_done[b].record(self.s_out)

    def drain(self):
        for s in (self.s_in, self.s_run, self.s_out):
            s.synchronize()
