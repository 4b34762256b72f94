"""fp64 CPU oracle for Gemma-4-style interleaved attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use this package. The product path (the CUDA library and its
Python binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``attn_oracle.c`` (plain C, double precision, OpenMP over
query rows); this module only builds it and marshals numpy arrays. Its header
comment names the passages each step follows and the readings taken where the
pages are silent.

Pinned by ``tests/test_oracle_pins.py`` (closed forms for the rotation sign, pair
layout, frequencies and the p cut-off; window and causal special cases; GQA
replication; shift invariance; an independent SDPA special case; split/combine
equivalence; brute-force tile counts), and the bidirectional 2D-RoPE routine by
``tests/test_oracle_pins_2d.py`` (each half a 1D rotation, shift invariance, SDPA
without a mask, patch permutation, GQA, the all-full tile plan).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

LOCAL = 0
GLOBAL = 1
BIDIR = 2  # bidirectional attention over an image's patches, 2D RoPE


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        lib.oracle_attention.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, P, P]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_combine.argtypes = [P, P, ctypes.c_int, ctypes.c_longlong, ctypes.c_int, P, P]
        lib.oracle_combine.restype = ctypes.c_int
        lib.oracle_tile_plan.argtypes = [ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, P, ctypes.c_longlong]
        lib.oracle_tile_plan.restype = ctypes.c_longlong
        lib.oracle_rope.argtypes = [P, P, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double]
        lib.oracle_rope.restype = None
        lib.oracle_rope2d.argtypes = [P, P, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double]
        lib.oracle_rope2d.restype = None
        lib.oracle_attention_2d.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P, P]
        lib.oracle_attention_2d.restype = ctypes.c_int
        lib.oracle_rotated_pairs.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_rotated_pairs.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def rotated_pairs(rope_p: float, head_dim: int) -> int:
    return int(_load().oracle_rotated_pairs(float(rope_p), int(head_dim)))


def rope(x: np.ndarray, rope_p: float, rope_base: float, pos: float) -> np.ndarray:
    """Rotate one vector (float64, even length) for position ``pos``."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().oracle_rope(_ptr(x), _ptr(y), x.shape[0], float(rope_p), float(rope_base), float(pos))
    return y


def attention(kind: int, window: int, rope_p: float, rope_base: float, scale: float,
              q: np.ndarray, k: np.ndarray, v: Optional[np.ndarray],
              positions: np.ndarray, cu_seqlens: np.ndarray,
              rows: Optional[np.ndarray] = None, key_range: Optional[tuple] = None):
    """Masked attention in fp64 for the selected query tokens.

    q [T, Hq, d], k [T, Hkv, d], v [T, Hkv, d] or None (K=V), all bf16 bit arrays (uint16).
    Returns (out [R, Hq, d] float64, lse [R, Hq] float64) for R = len(rows) (or T).
    """
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = None if v is None else np.ascontiguousarray(v, dtype=np.uint16)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    positions = np.ascontiguousarray(positions, dtype=np.int32)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = T if rr is None else rr.shape[0]
    out = np.zeros((n, Hq, d), dtype=np.float64)
    lse = np.zeros((n, Hq), dtype=np.float64)
    klo, khi = (0, 0) if key_range is None else key_range
    rc = lib.oracle_attention(int(kind), int(window), float(rope_p), float(rope_base), float(scale),
                              Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(v), _ptr(positions), _ptr(cu),
                              cu.shape[0] - 1, _ptr(rr), n, int(klo), int(khi), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")
    return out, lse


def rope2d(x: np.ndarray, rope_base: float, pos_h: float, pos_w: float) -> np.ndarray:
    """2D rotation of one vector (float64, length divisible by 4): first half for w, second for h."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().oracle_rope2d(_ptr(x), _ptr(y), x.shape[0], float(rope_base), float(pos_h), float(pos_w))
    return y


def attention_2d(rope_base: float, scale: float, q: np.ndarray, k: np.ndarray, v: Optional[np.ndarray],
                 positions_hw: np.ndarray, cu_seqlens: np.ndarray, rows: Optional[np.ndarray] = None):
    """Bidirectional attention with 2D RoPE in fp64 (every key of the query's sequence).

    q [T, Hq, d], k / v [T, Hkv, d] bf16 bits (v None: K=V); positions_hw [T, 2] int (h, w).
    Returns (out [R, Hq, d], lse [R, Hq]) float64 for R = len(rows) (or T).
    """
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = None if v is None else np.ascontiguousarray(v, dtype=np.uint16)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    hw = np.ascontiguousarray(positions_hw, dtype=np.int32).reshape(T, 2)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n = T if rr is None else rr.shape[0]
    out = np.zeros((n, Hq, d), dtype=np.float64)
    lse = np.zeros((n, Hq), dtype=np.float64)
    rc = lib.oracle_attention_2d(float(rope_base), float(scale), Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(v), _ptr(hw),
                                 _ptr(cu), cu.shape[0] - 1, _ptr(rr), n, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_2d rejected its arguments")
    return out, lse


def combine(partial_o: np.ndarray, partial_lse: np.ndarray):
    """partial_o [S, R, d], partial_lse [S, R] (float64) -> (out [R, d], lse [R])."""
    po = np.ascontiguousarray(partial_o, dtype=np.float64)
    pl = np.ascontiguousarray(partial_lse, dtype=np.float64)
    S, R, d = po.shape
    out = np.zeros((R, d), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    rc = _load().oracle_combine(_ptr(po), _ptr(pl), S, R, d, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_combine rejected its arguments")
    return out, lse


def tile_plan(kind: int, window: int, positions: np.ndarray, cu_seqlens: np.ndarray, bm: int, bn: int):
    """Brute-force tile list: int32 [n, 4] rows of (seq, q_tile, kv_tile, class), class 1 partial, 2 full."""
    lib = _load()
    positions = np.ascontiguousarray(positions, dtype=np.int32)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n = lib.oracle_tile_plan(int(kind), int(window), _ptr(positions), _ptr(cu), cu.shape[0] - 1,
                             int(bm), int(bn), None, 0)
    out = np.zeros((max(n, 1), 4), dtype=np.int32)
    lib.oracle_tile_plan(int(kind), int(window), _ptr(positions), _ptr(cu), cu.shape[0] - 1,
                         int(bm), int(bn), _ptr(out), n)
    return out[:n]


def decode(kind: int, window: int, rope_p: float, rope_base: float, scale: float,
           q_new: np.ndarray, k_hist: list, v_hist: Optional[list], cache_lens):
    """Decode / verify reference over each sequence's full token history.

    q_new [B, n_q, Hq, d]; k_hist[b] / v_hist[b]: [cache_lens[b] + n_q, Hkv, d] bf16 bits holding
    the cached tokens followed by the n_q new tokens (positions 0 .. len + n_q - 1).
    Queries sit at positions len .. len + n_q - 1. Returns out [B, n_q, Hq, d], lse [B, n_q, Hq].
    The cache layout (ring or contiguous) is a GPU-side detail and plays no part here.
    """
    B, n_q, Hq, d = q_new.shape
    outs, lses = [], []
    for b in range(B):
        L = int(cache_lens[b]) + n_q
        q = np.zeros((L, Hq, d), dtype=np.uint16)
        q[L - n_q:] = q_new[b]
        pos = np.arange(L, dtype=np.int32)
        cu = np.array([0, L], dtype=np.int32)
        rows = np.arange(L - n_q, L, dtype=np.int32)
        o, l = attention(kind, window, rope_p, rope_base, scale, q, k_hist[b],
                         None if v_hist is None else v_hist[b], pos, cu, rows=rows)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)
