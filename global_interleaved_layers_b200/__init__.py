"""Python binding of libgemma_attn.so (the C ABI in include/gemma_attn.h).

Argument marshalling only: every step of the attention path runs in the CUDA
library. Tensors may be torch tensors (device memory) or raw integer addresses;
``None`` passes a NULL pointer. Each wrapper raises ``GemmaAttnError`` on a
non-zero status. Importing this module raises ImportError when the library has
not been built (``python -m global_interleaved_layers_b200.build``): there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgemma_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python global_interleaved_layers_b200/build.py` "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

LOCAL = 0
GLOBAL = 1
BIDIR = 2  # vision patches: bidirectional, 2D RoPE; positions are [T, 2] (h, w); prefill only
CACHE_CONTIGUOUS = 0
CACHE_RING = 1
CACHE_KEYS_ROTATED = 0x100  # OR-ed into the layout (local layers): cached keys stored rotated
OUT_BF16 = 0
OUT_F32 = 1

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_MISALIGNED = -4
ERR_LAUNCH = -5
ERR_TIMEOUT = -6
ERR_DEVICE = -7
ERR_SEQLEN = -8


class GemmaAttnParams(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("window", ctypes.c_int32), ("rope_p", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32)]


class GemmaAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gemma_attn_error_string(status)} ({status})")


_P = ctypes.c_void_p
_I = ctypes.c_int32
_PP = ctypes.POINTER(GemmaAttnParams)

_lib.gemma_attn_error_string.argtypes = [ctypes.c_int]
_lib.gemma_attn_error_string.restype = ctypes.c_char_p
_lib.gemma_attn_last_launch_count.argtypes = []
_lib.gemma_attn_last_launch_count.restype = ctypes.c_int
_lib.gemma_attn_prefill_workspace_size.argtypes = [_PP, _I, ctypes.POINTER(ctypes.c_size_t)]
_lib.gemma_attn_prefill.argtypes = [_PP, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, ctypes.c_size_t, _P]
_lib.gemma_attn_prefill_rotate.argtypes = _lib.gemma_attn_prefill.argtypes
_lib.gemma_attn_prefill_attend.argtypes = _lib.gemma_attn_prefill.argtypes
_lib.gemma_attn_decode.argtypes = [_PP, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _P, _P, _I, _P]
_lib.gemma_attn_decode_num_splits.argtypes = [_PP, _I, _I, _I, ctypes.POINTER(ctypes.c_int32)]
_lib.gemma_attn_combine.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P]
_lib.gemma_attn_tile_plan.argtypes = [_I, _I, _P, _I, _I, _I, _P, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
_lib.gemma_attn_decode_noalloc.argtypes = [_PP, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _P, _P, _P]
_lib.gemma_attn_cache_append.argtypes = [_PP, _P, _P, _P, _P, _I, _I, _P, _I, _I, _P]
_lib.gemma_attn_decode_shard.argtypes = [_PP, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P]
_lib.gemma_attn_check.argtypes = [_P]
_lib.gemma_attn_selftest_umma.argtypes = [_I, _P, _P, _P, _P, _P]
_lib.gemma_attn_selftest_timeout.argtypes = [_P, _P]
for _f in ("gemma_attn_prefill_workspace_size", "gemma_attn_prefill", "gemma_attn_decode",
           "gemma_attn_decode_num_splits", "gemma_attn_combine", "gemma_attn_tile_plan", "gemma_attn_check",
           "gemma_attn_selftest_umma", "gemma_attn_decode_noalloc", "gemma_attn_selftest_timeout",
           "gemma_attn_cache_append", "gemma_attn_decode_shard",
           "gemma_attn_prefill_rotate", "gemma_attn_prefill_attend"):
    getattr(_lib, _f).restype = ctypes.c_int


def params(kind: int, num_q_heads: int, num_kv_heads: int, head_dim: int, window: int = 0,
           rope_p: float = 1.0, rope_base: float = 10000.0, softmax_scale: Optional[float] = None,
           out_dtype: int = OUT_BF16) -> GemmaAttnParams:
    if softmax_scale is None:
        softmax_scale = head_dim ** -0.5
    return GemmaAttnParams(kind, window, rope_p, rope_base, softmax_scale, num_q_heads, num_kv_heads, head_dim,
                           out_dtype)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):          # numpy (host) arrays, for the host-only entry points
        return x.ctypes.data
    raise TypeError(f"cannot pass {type(x)} as a pointer")


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:  # no torch / no device: the legacy default stream
            return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != OK:
        raise GemmaAttnError(rc, where)


def gemma_attn_error_string(status: int) -> str:
    return _lib.gemma_attn_error_string(status).decode()


def gemma_attn_last_launch_count() -> int:
    return int(_lib.gemma_attn_last_launch_count())


def gemma_attn_prefill_workspace_size(p: GemmaAttnParams, total_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.gemma_attn_prefill_workspace_size(ctypes.byref(p), total_tokens, ctypes.byref(n)),
           "gemma_attn_prefill_workspace_size")
    return int(n.value)


def gemma_attn_prefill(p: GemmaAttnParams, q, k, v, out, lse, positions, cu_seqlens, num_seqs: int,
                       total_tokens: int, max_seqlen: int, workspace, workspace_bytes: int, stream=None) -> None:
    _check(_lib.gemma_attn_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                   _ptr(positions), _ptr(cu_seqlens), num_seqs, total_tokens, max_seqlen,
                                   _ptr(workspace), workspace_bytes, _stream(stream)), "gemma_attn_prefill")


def gemma_attn_prefill_rotate(p: GemmaAttnParams, q, k, v, out, lse, positions, cu_seqlens, num_seqs: int,
                              total_tokens: int, max_seqlen: int, workspace, workspace_bytes: int,
                              stream=None) -> None:
    _check(_lib.gemma_attn_prefill_rotate(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                          _ptr(positions), _ptr(cu_seqlens), num_seqs, total_tokens, max_seqlen,
                                          _ptr(workspace), workspace_bytes, _stream(stream)),
           "gemma_attn_prefill_rotate")


def gemma_attn_prefill_attend(p: GemmaAttnParams, q, k, v, out, lse, positions, cu_seqlens, num_seqs: int,
                              total_tokens: int, max_seqlen: int, workspace, workspace_bytes: int,
                              stream=None) -> None:
    _check(_lib.gemma_attn_prefill_attend(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                          _ptr(positions), _ptr(cu_seqlens), num_seqs, total_tokens, max_seqlen,
                                          _ptr(workspace), workspace_bytes, _stream(stream)),
           "gemma_attn_prefill_attend")


def gemma_attn_decode(p: GemmaAttnParams, q, new_k, new_v, k_cache, v_cache, cache_layout: int,
                      cache_capacity: int, cache_seqlens, batch: int, n_q: int, max_cache_len: int,
                      partial_o, partial_lse, num_splits: int, stream=None) -> None:
    _check(_lib.gemma_attn_decode(ctypes.byref(p), _ptr(q), _ptr(new_k), _ptr(new_v), _ptr(k_cache),
                                  _ptr(v_cache), cache_layout, cache_capacity, _ptr(cache_seqlens), batch, n_q,
                                  max_cache_len, _ptr(partial_o), _ptr(partial_lse), num_splits, _stream(stream)),
           "gemma_attn_decode")


def gemma_attn_decode_shard(p: GemmaAttnParams, q, new_k, k_cache, cache_capacity: int, shard_seqlens,
                            q_pos_offset, include_new: bool, batch: int, n_q: int, max_shard_len: int, partial_o,
                            partial_lse, num_splits: int, stream=None) -> None:
    """Split-KV partials over one key-range shard of a longer K=V history (global layers)."""
    _check(_lib.gemma_attn_decode_shard(ctypes.byref(p), _ptr(q), _ptr(new_k), _ptr(k_cache), cache_capacity,
                                        _ptr(shard_seqlens), _ptr(q_pos_offset), 1 if include_new else 0, batch,
                                        n_q, max_shard_len, _ptr(partial_o), _ptr(partial_lse), num_splits,
                                        _stream(stream)), "gemma_attn_decode_shard")


NOALLOC_SCRATCH_BYTES = 16 << 20


def gemma_attn_decode_noalloc(p: GemmaAttnParams, q, new_k, new_v, k_cache, v_cache, cache_layout: int,
                              cache_capacity: int, cache_seqlens, batch: int, n_q: int, max_cache_len: int,
                              num_splits: int, out, lse, stream=None) -> None:
    """Decode + combine with the split partials in the library's static device array (no allocation)."""
    _check(_lib.gemma_attn_decode_noalloc(ctypes.byref(p), _ptr(q), _ptr(new_k), _ptr(new_v), _ptr(k_cache),
                                          _ptr(v_cache), cache_layout, cache_capacity, _ptr(cache_seqlens), batch,
                                          n_q, max_cache_len, num_splits, _ptr(out), _ptr(lse), _stream(stream)),
           "gemma_attn_decode_noalloc")


def gemma_attn_cache_append(p: GemmaAttnParams, new_k, new_v, k_cache, v_cache, cache_layout: int,
                            cache_capacity: int, cache_seqlens, batch: int, n_q: int, stream=None) -> None:
    """New tokens' K (and V) rows into the cache at slot position mod window (ring) or row position."""
    _check(_lib.gemma_attn_cache_append(ctypes.byref(p), _ptr(new_k), _ptr(new_v), _ptr(k_cache), _ptr(v_cache),
                                        cache_layout, cache_capacity, _ptr(cache_seqlens), batch, n_q,
                                        _stream(stream)), "gemma_attn_cache_append")


def gemma_attn_decode_num_splits(p: GemmaAttnParams, batch: int, n_q: int, max_cache_len: int) -> int:
    n = ctypes.c_int32(0)
    _check(_lib.gemma_attn_decode_num_splits(ctypes.byref(p), batch, n_q, max_cache_len, ctypes.byref(n)),
           "gemma_attn_decode_num_splits")
    return int(n.value)


def gemma_attn_combine(partial_o, partial_lse, num_splits: int, rows: int, head_dim: int, out_dtype: int, out,
                       lse, stream=None) -> None:
    _check(_lib.gemma_attn_combine(_ptr(partial_o), _ptr(partial_lse), num_splits, rows, head_dim, out_dtype,
                                   _ptr(out), _ptr(lse), _stream(stream)), "gemma_attn_combine")


def gemma_attn_tile_plan(kind: int, window: int, cu_seqlens_host, bm: int, bn: int):
    """Host-side tile plan; cu_seqlens_host is a numpy int32 array. Returns an int32 [n, 4] numpy array."""
    import numpy as np
    cu = np.ascontiguousarray(cu_seqlens_host, dtype=np.int32)
    n = ctypes.c_int64(0)
    _check(_lib.gemma_attn_tile_plan(kind, window, _ptr(cu), cu.shape[0] - 1, bm, bn, None, 0, ctypes.byref(n)),
           "gemma_attn_tile_plan")
    out = np.zeros((max(int(n.value), 1), 4), dtype=np.int32)
    _check(_lib.gemma_attn_tile_plan(kind, window, _ptr(cu), cu.shape[0] - 1, bm, bn, _ptr(out), n.value,
                                     ctypes.byref(n)), "gemma_attn_tile_plan")
    return out[: int(n.value)]


def gemma_attn_check(stream=None) -> None:
    _check(_lib.gemma_attn_check(_stream(stream)), "gemma_attn_check")


def gemma_attn_selftest_umma(mode: int, a, b, p, d, stream=None) -> None:
    _check(_lib.gemma_attn_selftest_umma(mode, _ptr(a), _ptr(b), _ptr(p), _ptr(d), _stream(stream)),
           "gemma_attn_selftest_umma")


def gemma_attn_selftest_timeout(gave_up, stream=None) -> None:
    _check(_lib.gemma_attn_selftest_timeout(_ptr(gave_up), _stream(stream)), "gemma_attn_selftest_timeout")


def raw_call(name: str, *args) -> int:
    """Call an entry point with raw ctypes arguments and return its status (for contract tests)."""
    return int(getattr(_lib, name)(*args))
