"""Seeded synthetic inputs and workload shapes for the interleaved-attention path.

This module is shared by the tests, the bench and the oracle's callers. It holds
only random-number generation and shape bookkeeping: none of the attention
arithmetic (no rotation, no masking, no softmax) lives here.

Inputs are i.i.d. N(0, 1) draws from ``numpy.random.default_rng(seed + index)``
(index 0 = q, 1 = k or the single K=V tensor, 2 = v), drawn in float32 and
rounded to bfloat16 with round-to-nearest-even. Arrays of bf16 values are
carried as ``numpy.uint16`` bit patterns so that every consumer sees exactly
the same bits.

The architecture parameters (window 512/1024, 4:1 and 5:1 interleave, 8:1
global GQA, 512 vs 256 head dim, p = 0.25) come from "Visual guide to Gemma 4"
(sections "Interleaving Layers" and "Efficiency of global attention") and from
the DeepMind talk summary "Gemma 4: how Google DeepMind rethinks open models"
(section "Optimised attention: local and global layers").
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

LOCAL = 0
GLOBAL = 1
BIDIR = 2  # the vision encoder's bidirectional 2D-RoPE attention over an image's patches


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, index: int, shape: Sequence[int]) -> np.ndarray:
    """N(0,1) float32 draws from default_rng(seed + index), rounded to bf16 bits."""
    rng = np.random.default_rng(seed + index)
    return f32_to_bf16_bits(rng.standard_normal(tuple(shape), dtype=np.float32))


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One attention layer's shape: kind, heads, head dim, window and rotary setup."""
    kind: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    window: int = 0
    rope_p: float = 1.0
    rope_base: float = 10000.0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def k_eq_v(self) -> bool:
        return self.kind == GLOBAL


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """A prefill block: ragged sequences, and a stack of layers run over them."""
    name: str
    seq_lens: tuple
    layers: tuple
    seed: int = 0

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seq_lens)]).astype(np.int32)

    def positions(self, start: int = 0) -> np.ndarray:
        return np.concatenate([np.arange(n, dtype=np.int32) + start for n in self.seq_lens]).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Decode (n_q = 1) or speculative verify (n_q > 1) against per-sequence caches."""
    name: str
    batch: int
    cache_lens: tuple
    n_q: int
    layers: tuple
    seed: int = 0


def layer_inputs(layer: LayerSpec, total_tokens: int, seed: int, layer_index: int = 0):
    """q [T, Hq, d], k (or K=V) [T, Hkv, d] and v (None for K=V) as bf16 bits."""
    base = seed + 16 * layer_index
    q = normal_bf16(base, 0, (total_tokens, layer.num_q_heads, layer.head_dim))
    k = normal_bf16(base, 1, (total_tokens, layer.num_kv_heads, layer.head_dim))
    v = None if layer.k_eq_v else normal_bf16(base, 2, (total_tokens, layer.num_kv_heads, layer.head_dim))
    return q, k, v


def ragged_lengths(n: int, lo: int, hi: int, seed: int) -> List[int]:
    """Lengths round(exp(U(ln lo, ln hi))) from default_rng(seed)."""
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return [int(round(math.exp(x))) for x in u]


# ---------------------------------------------------------------------------
# The workloads. Sizes follow the Gemma-4 parameters named in the module doc.
# ---------------------------------------------------------------------------

def tiny_ref() -> PrefillWorkload:
    """Batch 1, L = 64: a W=16 local layer (4/2 heads, d=32) and a K=V p-RoPE global layer (8/1, d=64)."""
    return PrefillWorkload(
        name="tiny_L64", seq_lens=(64,), seed=0,
        layers=(LayerSpec(LOCAL, 4, 2, 32, window=16, rope_p=1.0, rope_base=1e4),
                LayerSpec(GLOBAL, 8, 1, 64, rope_p=0.25, rope_base=1e4)))


def e2b_block() -> PrefillWorkload:
    """L = 8192, 4 local (W=512, 8/4 heads, d=256) + 1 global (8/1 heads, d=512, K=V, p=0.25)."""
    loc = LayerSpec(LOCAL, 8, 4, 256, window=512, rope_p=1.0, rope_base=1e4)
    glo = LayerSpec(GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
    return PrefillWorkload(name="e2b_block_L8192", seq_lens=(8192,), seed=0,
                           layers=(loc, loc, loc, loc, glo))


def b31_block() -> PrefillWorkload:
    """L = 32768, 5 local (W=1024, 32/16 heads, d=256) + 1 global (32/4 heads, d=512, K=V, p=0.25)."""
    loc = LayerSpec(LOCAL, 32, 16, 256, window=1024, rope_p=1.0, rope_base=1e4)
    glo = LayerSpec(GLOBAL, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    return PrefillWorkload(name="31b_block_L32768", seq_lens=(32768,), seed=0,
                           layers=(loc, loc, loc, loc, loc, glo))


def long_decode() -> DecodeWorkload:
    """Batch 8, one query token: global K=V cache of 131072 tokens (d=512) and a 1024-slot local ring."""
    glo = LayerSpec(GLOBAL, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    loc = LayerSpec(LOCAL, 32, 16, 256, window=1024, rope_p=1.0, rope_base=1e4)
    return DecodeWorkload(name="decode_b8_ctx131072", batch=8, cache_lens=(131072,) * 8, n_q=1,
                          layers=(glo, loc), seed=0)


def ragged_31b(seed: int = 7):
    """16 sequences, lengths log-uniform in [1024, 65536]; 31B shapes; then a 4-token verify."""
    lens = tuple(ragged_lengths(16, 1024, 65536, seed))
    loc = LayerSpec(LOCAL, 32, 16, 256, window=1024, rope_p=1.0, rope_base=1e4)
    glo = LayerSpec(GLOBAL, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    pre = PrefillWorkload(name="ragged16_31b", seq_lens=lens, seed=0, layers=(loc, glo))
    ver = DecodeWorkload(name="verify4_ragged16_31b", batch=16, cache_lens=lens, n_q=4,
                         layers=(glo, loc), seed=0)
    return pre, ver


def vision_batch() -> PrefillWorkload:
    """4 images of 2520 patches (the pages' largest patch count: 9 x 280 at a soft-token
    budget of 280), bidirectional 2D-RoPE attention with 12 heads of 64 dims (a ViT-B-sized
    encoder; the pages give the encoder's parameter count, not its attention shape)."""
    layer = LayerSpec(BIDIR, 12, 12, 64, rope_p=1.0, rope_base=1e4)
    return PrefillWorkload(name="vision_4x2520", seq_lens=(2520,) * 4, seed=0, layers=(layer,))


def unmasked_pairs(seq_lens: Sequence[int], kind: int, window: int) -> int:
    """Number of visible (query, key) pairs for prefill with consecutive positions."""
    total = 0
    for n in seq_lens:
        if kind == BIDIR:  # every patch sees every patch of its image
            total += n * n
            continue
        if kind == GLOBAL or window >= n:
            total += n * (n + 1) // 2
        else:
            w = window
            # rows 0..w-1 see i+1 keys, the rest see w keys
            total += w * (w + 1) // 2 + (n - w) * w
    return total


def prefill_flops(seq_lens: Sequence[int], layer: LayerSpec) -> int:
    """Unmasked FLOPs: 4 * d * Hq * visible pairs (QK^T and PV, two FLOPs per MAC)."""
    return 4 * layer.head_dim * layer.num_q_heads * unmasked_pairs(seq_lens, layer.kind, layer.window)


def decode_cache_bytes(batch: int, cache_lens: Sequence[int], layer: LayerSpec) -> int:
    """Algorithmic bytes of one decode step: every visible cache row read once (K=V counted once)."""
    per_row = layer.num_kv_heads * layer.head_dim * 2
    tensors = 1 if layer.k_eq_v else 2
    total = 0
    for n in cache_lens:
        # queries sit at positions n .. n+n_q-1; the oldest visible cached position
        # is n - W + 1 for a local layer, so a W-slot ring contributes W - 1 rows.
        rows = n if layer.kind == GLOBAL else min(n, layer.window - 1)
        total += rows * per_row * tensors
    return total
