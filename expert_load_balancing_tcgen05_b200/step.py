"""The routing step over batches of T tokens, every buffer allocated once:
gate GEMM and scores, selection, load statistics, bias step, dispatch.

Two schedules of the same library calls:

* serial -- the calls in order on the caller's stream;
* pipelined -- the routing of batch i+1 (gate, selection, load statistics,
  bias step and, with several ranks, the all-reduce of the expert counts)
  runs on a high-priority stream beside the dispatch (and, when asked, the
  combine) of batch i on the caller's stream.  Batch i+1 depends on batch i
  only through the bias, which its routing stream updates in order, so every
  result equals the serial schedule's.  Everything a batch's routing writes
  and its dispatch or combine reads (scores, indices, weights, slots, counts,
  offsets, ranks, stats) is double-buffered; a buffer set is reused only
  after the dispatch and combine that read it have finished.  The gate GEMM
  gets a budget of SMs (``gate_max_ctas``) so that the dispatch, which is
  bound by HBM bandwidth, keeps the rest of the GPU.

Combine runs on identity experts here (it gathers the dispatched rows back),
the step having no expert FFNs.

Host-side orchestration only: streams, events and buffers.  Every step of the
path runs in the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe

# SMs the gate GEMM may use while it runs beside a dispatch (pipelined schedule)
PIPELINED_GATE_CTAS = 64


def fused_routing_supported(wl, x) -> bool:
    """Whether moe_route_tiles takes this workload: bf16 tokens on the
    tensor-core gate (64, 128 or 256 experts), K <= 8, and one group or
    sigmoid groups of 32 experts scored by their top one or two keys."""
    xs = x[0] if isinstance(x, (list, tuple)) else x
    if xs.dtype != torch.bfloat16 or wl.N not in (64, 128, 256) or wl.K > 8:
        return False
    return wl.n_groups == 1 or (wl.fn == moe.MOE_SIGMOID and wl.N // wl.n_groups == 32 and wl.group_topn <= 2)


class RoutingStep:
    """x: the token batch [T, d], or a list of batches that step() cycles
    through when it is given none (consecutive batches then live in
    different buffers, as in a stream of distinct batches)."""

    def __init__(self, wl, x, w_gate, bias, logit_offset, device, world: int = 1, pipelined: bool = True,
                 gate_max_ctas: int | None = None, bias_rate: float = 0.001, fused: bool | None = None):
        T, d, N, K = wl.T, wl.d, wl.N, wl.K
        self.wl, self.dev, self.world, self.pipelined, self.u = wl, device, world, pipelined, bias_rate
        # fused: the selection and a per-tile histogram in the gate's epilogue
        # (moe_route_tiles, no scores in memory), statistics from those
        # histograms (moe_load_stats_tiles).  Default: wherever the epilogue
        # can select (the shapes moe_route_tiles accepts).
        if fused is None:
            fused = fused_routing_supported(wl, x)
        self.fused = fused
        self.batches = list(x) if isinstance(x, (list, tuple)) else [x]
        x = self.batches[0]
        self.x, self.W, self.bias, self.off = x, w_gate, bias, logit_offset
        f32, i32 = torch.float32, torch.int32
        self.sets = [dict(scores=(torch.empty(moe.tile_counts_shape(T, N), dtype=i32, device=device) if fused
                                  else torch.empty(T, N, dtype=f32, device=device)),
                          idx=torch.empty(T, K, dtype=i32, device=device),
                          w=torch.empty(T, K, dtype=f32, device=device),
                          slot=torch.empty(T, K, dtype=i32, device=device),
                          counts=torch.empty(N, dtype=i32, device=device),
                          offsets=torch.empty(N + 1, dtype=i32, device=device),
                          rank=torch.empty(T, K, dtype=i32, device=device),
                          stats=moe.empty_stats(device))
                     for _ in range(2 if pipelined else 1)]
        self.ws = moe.workspace(T, K, N, N, device=device)
        self.rows = torch.empty(T * K, d, dtype=x.dtype, device=device)
        self.pos = torch.empty(T, K, dtype=i32, device=device)
        if gate_max_ctas is None:
            gate_max_ctas = PIPELINED_GATE_CTAS if pipelined else 0
        self.cfg = moe.route_cfg(T, d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm,
                                 wl.scale, moe.MOE_BF16 if x.dtype == torch.bfloat16 else moe.MOE_F32,
                                 gate_max_ctas=gate_max_ctas)
        self.i = 0
        if pipelined:
            _, highest = torch.cuda.Stream.priority_range()
            self.route_stream = torch.cuda.Stream(device=device, priority=highest)
            self.ev_routed = [torch.cuda.Event() for _ in range(2)]
            self.ev_dispatched = [torch.cuda.Event() for _ in range(2)]
        self.fence()

    # ------------------------------------------------------------------ parts
    def _route_part(self, s, x, stream, stage_events=None):
        wl = self.wl
        if stage_events is not None:
            stage_events[0].record(stream)
        if self.fused:
            # s["scores"] holds the per-tile histograms on this path
            moe.moe_route_tiles(self.cfg, x, self.W, self.off, self.bias, s["idx"], s["w"], s["scores"], self.ws,
                                stream=stream)
        else:
            moe.moe_route(self.cfg, x, self.W, self.off, self.bias, s["scores"], s["idx"], s["w"], self.ws,
                          stream=stream)
        if stage_events is not None:
            stage_events[1].record(stream)
        if self.fused:
            moe.moe_load_stats_tiles(s["idx"], wl.T, wl.K, wl.N, s["scores"], None, wl.N, s["slot"], s["counts"],
                                     s["offsets"], s["rank"], s["stats"], self.ws, stream=stream)
        else:
            moe.moe_load_stats(s["idx"], wl.T, wl.K, wl.N, None, wl.N, s["slot"], s["counts"], s["offsets"],
                               s["rank"], None, wl.fn, s["stats"], self.ws, stream=stream)
        total = wl.T * wl.K
        if self.world > 1:
            # the bias is shared by every rank: its step uses the global counts
            with torch.cuda.stream(stream):
                dist.all_reduce(s["counts"], op=dist.ReduceOp.SUM)
            total *= self.world
        moe.moe_bias_update(s["counts"], wl.N, total, self.u, 0, self.bias, stream=stream)

    def _dispatch_part(self, s, x, stream, combine_out=None):
        wl = self.wl
        moe.moe_dispatch(x, wl.T, wl.d, wl.K, s["slot"], s["offsets"], s["rank"], self.rows, None, None, self.pos,
                         None, stream=stream)
        if combine_out is not None:
            # identity experts: the expert outputs are the dispatched rows
            moe.moe_combine(self.rows, wl.T, wl.d, wl.K, self.pos, s["w"], combine_out, stream=stream)

    # the last batch's routing outputs (scores: the per-tile histograms on the fused path)
    @property
    def scores(self):
        return self.last()["scores"]

    @property
    def idx(self):
        return self.last()["idx"]

    @property
    def w(self):
        return self.last()["w"]

    # ------------------------------------------------------------------ api
    def fence(self):
        """Order the routing stream after everything already on the caller's
        stream (inputs written there, the start of a timed region)."""
        if self.pipelined:
            self.route_stream.wait_stream(torch.cuda.current_stream(self.dev))

    def results(self, s):
        """The routing result of a batch: indices, weights, offsets, counts, stats."""
        return [s["idx"], s["w"], s["offsets"], s["counts"], s["stats"]]

    def _copy_out(self, s, host_out, stream):
        with torch.cuda.stream(stream):
            for src, dst in zip(self.results(s), host_out):
                dst.copy_(src, non_blocking=True)

    def step(self, x=None, dispatch_events=None, stage_events=None, ready=None, host_out=None, combine_out=None):
        """Enqueue one batch.

        x: the batch's tokens (default: the next of the batches given at
        construction);
        ready: an event after which x is valid (e.g. the end of its copy from
        the host on another stream); host_out: pinned host tensors shaped like
        results(), filled with this batch's routing result (indices and
        weights are copied before the next batch overwrites them).
        combine_out: optional [T, d] tensor; when given, the batch's rows are
        combined back into it (identity experts) on the caller's stream
        right after its dispatch.
        dispatch_events: optional (start, end) CUDA events recorded around the
        dispatch on the caller's stream.  stage_events (serial schedule only):
        four events recorded before the gate, after the selection, after the
        bias step and after the dispatch."""
        x = self.batches[self.i % len(self.batches)] if x is None else x
        main = torch.cuda.current_stream(self.dev)
        if not self.pipelined:
            s = self.sets[0]
            if ready is not None:
                main.wait_event(ready)
            self._route_part(s, x, main, stage_events)
            if stage_events is not None:
                stage_events[2].record(main)
            if host_out is not None:
                self._copy_out(s, host_out, main)
            if dispatch_events is not None:
                dispatch_events[0].record(main)
            self._dispatch_part(s, x, main, combine_out)
            if dispatch_events is not None:
                dispatch_events[1].record(main)
            if stage_events is not None:
                stage_events[3].record(main)
            self.i += 1
            return
        b = self.i % 2
        s = self.sets[b]
        rs = self.route_stream
        if self.i >= 2:
            rs.wait_event(self.ev_dispatched[b])  # the dispatch that read this buffer set is done
        if ready is not None:
            rs.wait_event(ready)
        self._route_part(s, x, rs)
        if host_out is not None:
            self._copy_out(s, host_out, rs)
        self.ev_routed[b].record(rs)
        main.wait_event(self.ev_routed[b])
        if dispatch_events is not None:
            dispatch_events[0].record(main)
        self._dispatch_part(s, x, main, combine_out)
        if dispatch_events is not None:
            dispatch_events[1].record(main)
        self.ev_dispatched[b].record(main)  # buffer set b: its dispatch and combine are done with it
        self.i += 1

    def last(self):
        """Buffer set (slots, counts, offsets, ranks, stats) of the last batch."""
        return self.sets[(self.i - 1) % len(self.sets)]
