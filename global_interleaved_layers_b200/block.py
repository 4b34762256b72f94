"""Interleaved block runner: the attention calls of a block of layers as one CUDA graph.

Gemma-4-style models interleave several sliding-window layers with one global layer
("Visual guide to Gemma 4", section "Interleaving Layers": the 4:1
and 5:1 patterns, the last layer of a block global). Each layer's prefill is two launches
(rotated side copy, attention); a block of five layers is ten launches whose gaps the
GPU otherwise spends idle between kernels. `InterleavedBlock` records the calls once and
replays them as a CUDA graph: the buffers are fixed at construction, so new inputs are
written into the same tensors between replays.

Only orchestration lives here: every step runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import (GemmaAttnParams, gemma_attn_last_launch_count, gemma_attn_prefill_attend,
               gemma_attn_prefill_rotate, gemma_attn_prefill_workspace_size)


@dataclass
class BlockLayer:
    """One layer's prefill call: its parameters and device buffers (owned by the caller)."""
    params: GemmaAttnParams
    q: torch.Tensor                 # [T, Hq, d] bf16
    k: torch.Tensor                 # [T, Hkv, d] bf16 (global layers: the K=V tensor)
    v: Optional[torch.Tensor]       # [T, Hkv, d] bf16, None for global layers
    out: torch.Tensor               # [T, Hq, d] bf16 or fp32 per params.out_dtype
    lse: Optional[torch.Tensor]     # [Hq, T] fp32 or None
    positions: torch.Tensor         # [T] int32
    cu_seqlens: torch.Tensor        # [S + 1] int32
    num_seqs: int
    total_tokens: int
    max_seqlen: int
    workspace: Optional[torch.Tensor] = None  # allocated by the runner when None


class InterleavedBlock:
    def __init__(self, layers: List[BlockLayer]):
        self.layers = layers
        for ly in layers:
            need = gemma_attn_prefill_workspace_size(ly.params, ly.total_tokens)
            if ly.workspace is None or ly.workspace.numel() < need:
                ly.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=ly.q.device)
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def run(self, stream=None, events=None) -> int:
        """The block's calls in order, launched eagerly on `stream` (default: current).
        events: optional per layer (start, between rotate and attend, end) CUDA events to
        record, any of them None (created with external=True when the run is captured;
        each recorded event costs the stream a few microseconds). Returns the number of
        kernels launched."""
        s = torch.cuda.current_stream() if stream is None else stream
        n = 0
        for li, ly in enumerate(self.layers):
            args = (ly.params, ly.q, ly.k, ly.v, ly.out, ly.lse, ly.positions, ly.cu_seqlens, ly.num_seqs,
                    ly.total_tokens, ly.max_seqlen, ly.workspace, ly.workspace.numel())
            ev = (None, None, None) if events is None or events[li] is None else events[li]
            if ev[0] is not None:
                ev[0].record(s)
            gemma_attn_prefill_rotate(*args, stream=s)
            n += gemma_attn_last_launch_count()
            if ev[1] is not None:
                ev[1].record(s)
            gemma_attn_prefill_attend(*args, stream=s)
            n += gemma_attn_last_launch_count()
            if ev[2] is not None:
                ev[2].record(s)
        return n

    def capture(self, events=None) -> int:
        """Record the block as a CUDA graph (one eager run first sets the library's
        per-device kernel attributes, which capture must not do). Returns the kernels one
        replay launches."""
        self.run(events=events)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            n = self.run(events=events)
        torch.cuda.synchronize()
        self.graph = g
        return n

    def replay(self) -> None:
        if self.graph is None:
            raise RuntimeError("capture() first")
        self.graph.replay()
