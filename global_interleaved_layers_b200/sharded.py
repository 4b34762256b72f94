"""Split-KV decode of a long global-layer history spread over several GPUs.

The medium models' context reaches 256K tokens ("Visão geral do modelo Gemma 4", section
"Recursos": the context window); a global layer's K=V cache for a batch of such sequences
is tens of GB per layer. Here each rank (one process per GPU) holds a contiguous range of
every sequence's cached tokens and decodes against it alone:

1. ``gemma_attn_decode_shard`` on the rank's range: fp32 partial outputs and log-sum-exps
   for every query row, the queries placed ``q_pos_offset`` tokens after the range's end
   (the tokens other ranks hold), the new tokens among the keys only on the last rank;
2. an all-gather of the partials (NCCL over NVLink / NVSwitch between GPUs), stacked
   rank-major as splits;
3. ``gemma_attn_combine`` of all the splits: the attention over the whole history, since
   the rotated scores depend only on the distance between query and key ("Visual guide to
   Gemma 4", section "p-RoPE").

Only step 2 crosses GPUs, and it moves splits x rows x (head_dim + 1) x 4 bytes per rank
(about 0.5 MB for 8 sequences x 32 query heads at head dim 512 with one split), into each
rank's own memory: no kernel reads another GPU's memory. This module holds host plumbing
only; every step of the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

KEY_TILE = 128  # shard boundaries fall on the kernels' key tiles


def shard_ranges(length: int, world: int, align: int = KEY_TILE) -> List[Tuple[int, int]]:
    """Contiguous ranges [lo, hi) of a history of `length` cached tokens, one per rank in
    rank order, covering it exactly; inner boundaries are multiples of `align`."""
    if world < 1 or length < 0:
        raise ValueError("world >= 1 and length >= 0 required")
    bounds = [0]
    for r in range(1, world):
        cut = (length * r // world) // align * align
        bounds.append(max(bounds[-1], min(cut, length)))
    bounds.append(length)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def query_offsets(lengths: Sequence[int], world: int, rank: int, align: int = KEY_TILE):
    """Per sequence: (shard lo, shard length, q_pos_offset) of `rank`'s range, where
    q_pos_offset counts the cached tokens after the range (held by later ranks)."""
    out = []
    for n in lengths:
        lo, hi = shard_ranges(int(n), world, align)[rank]
        out.append((lo, hi - lo, int(n) - hi))
    return out


class _LibraryBackend:
    """The CUDA library: the decode over one shard and the combine."""

    def __init__(self):
        from . import gemma_attn_combine, gemma_attn_decode_shard  # raises ImportError without the library
        self.decode_shard = gemma_attn_decode_shard
        self.combine = gemma_attn_combine


class ShardedDecode:
    """One rank's part of a split-KV decode over a history spread across `world` ranks.

    Buffers (fp32 partials of this rank and of all ranks) are allocated once here, on the
    given device; a call launches the shard decode, the all-gather and the combine on the
    current stream. `group` is a torch.distributed process group (None: the default one,
    when torch.distributed is initialised; a single rank otherwise). `backend` replaces the
    library's entry points (tests run the host plumbing on CPU ranks this way)."""

    def __init__(self, params, batch: int, n_q: int, splits_per_rank: int, device, out_dtype: int = 0,
                 group=None, backend=None):
        import torch
        import torch.distributed as dist
        self.torch = torch
        self.dist = dist if (dist.is_available() and dist.is_initialized()) else None
        self.group = group
        self.world = self.dist.get_world_size(group) if self.dist else 1
        self.rank = self.dist.get_rank(group) if self.dist else 0
        self.params = params
        self.batch, self.n_q, self.splits = batch, n_q, splits_per_rank
        self.d = params.head_dim
        self.rows = batch * n_q * params.num_q_heads
        self.out_dtype = out_dtype
        self.backend = backend if backend is not None else _LibraryBackend()
        f32 = torch.float32
        self.po_local = torch.empty((self.splits, self.rows, self.d), dtype=f32, device=device)
        self.pl_local = torch.empty((self.splits, self.rows), dtype=f32, device=device)
        if self.world > 1:
            self.po_all = torch.empty((self.world * self.splits, self.rows, self.d), dtype=f32, device=device)
            self.pl_all = torch.empty((self.world * self.splits, self.rows), dtype=f32, device=device)
        else:
            self.po_all, self.pl_all = self.po_local, self.pl_local

    @property
    def holds_end(self) -> bool:
        """The last rank holds the end of every history: its keys include the new tokens."""
        return self.rank == self.world - 1

    def _gather(self, dst, src):
        try:
            self.dist.all_gather_into_tensor(dst, src, group=self.group)
        except (RuntimeError, AttributeError, NotImplementedError):  # backends without the fused form
            parts = list(dst.chunk(self.world, dim=0))
            self.dist.all_gather(parts, src, group=self.group)

    def __call__(self, q, new_k, k_shard, cache_capacity: int, shard_seqlens, q_pos_offset, max_shard_len: int,
                 out, lse=None, stream=None) -> int:
        """Attention of the n_q new tokens over the whole history into `out` (and `lse`).

        q [batch, n_q, Hq, d] and new_k [batch, n_q, Hkv, d] bf16 (new_k is read on the last
        rank only); k_shard [batch, Hkv, cache_capacity, d] bf16: this rank's range of each
        history at rows 0 .. shard_seqlens[b] - 1; shard_seqlens and q_pos_offset [batch]
        int32 device arrays (see query_offsets). Every rank gets the full result. Returns
        the number of kernel launches."""
        self.backend.decode_shard(self.params, q, new_k if self.holds_end else None, k_shard, cache_capacity,
                                  shard_seqlens, q_pos_offset, self.holds_end, self.batch, self.n_q, max_shard_len,
                                  self.po_local, self.pl_local, self.splits, stream)
        if self.world > 1:
            self._gather(self.po_all, self.po_local)
            self._gather(self.pl_all, self.pl_local)
        self.backend.combine(self.po_all, self.pl_all, self.world * self.splits, self.rows, self.d, self.out_dtype,
                             out, lse, stream)
        return 2
