"""Helpers for the GPU parity tests: marshal bf16 bit arrays to the device, call the
C-ABI through the binding, and compare with the fp64 oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import workloads as W

# Acceptance bounds: max-abs error 1e-2 and relative RMS error 5e-3 against the fp64
# oracle (bf16 inputs, fp32 accumulation, bf16 output).
TOL_MAX_ABS = 1e-2
TOL_REL_RMS = 5e-3
TOL_LSE = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = math.sqrt(float(np.sum(ref * ref))) or 1.0
    rel_rms = math.sqrt(float(np.sum(diff * diff))) / denom
    return max_abs, rel_rms


def assert_close(got, ref, what=""):
    max_abs, rel_rms = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert max_abs <= TOL_MAX_ABS and rel_rms <= TOL_REL_RMS, \
        f"{what}: max_abs={max_abs:.3e} rel_rms={rel_rms:.3e}"
    return max_abs, rel_rms


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 (round to nearest even) -> float32."""
    return W.bf16_bits_to_f32(W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def run_prefill(G, layer: W.LayerSpec, q, k, v, positions, cu_seqlens, with_lse=True, out_f32=False,
                out_offset_bytes=0):
    """q/k/v: bf16 bit arrays (host) or bf16 device tensors. Returns (out device tensor, lse device).

    out is bf16 unless out_f32 (then float32, the accumulator precision)."""
    qd = q if isinstance(q, torch.Tensor) else dev_bf16(q)
    kd = k if isinstance(k, torch.Tensor) else dev_bf16(k)
    vd = None if v is None else (v if isinstance(v, torch.Tensor) else dev_bf16(v))
    T, Hq, d = qd.shape
    cu = np.asarray(cu_seqlens, dtype=np.int32)
    S = cu.shape[0] - 1
    max_len = int(np.max(np.diff(cu)))
    p = G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, window=layer.window,
                 rope_p=layer.rope_p, rope_base=layer.rope_base, softmax_scale=layer.softmax_scale,
                 out_dtype=G.OUT_F32 if out_f32 else G.OUT_BF16)
    odt = torch.float32 if out_f32 else torch.bfloat16
    if out_offset_bytes:  # an output that is only 16-byte aligned
        esz = 4 if out_f32 else 2
        extra = out_offset_bytes // esz
        out = torch.empty((qd.numel() + extra,), dtype=odt, device="cuda")[extra:].view(qd.shape)
    else:
        out = torch.empty(qd.shape, dtype=odt, device="cuda")
    lse = torch.empty((Hq, T), dtype=torch.float32, device="cuda") if with_lse else None
    ws_bytes = G.gemma_attn_prefill_workspace_size(p, T)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    G.gemma_attn_prefill(p, qd, kd, vd, out, lse, dev_i32(positions), dev_i32(cu), S, T, max_len, ws, ws_bytes)
    G.gemma_attn_check()
    return out, lse


def ring_from_history(hist: np.ndarray, window: int) -> np.ndarray:
    """Place tokens of a [len, Hkv, d] history into a window-slot ring [Hkv, window, d] (slot = pos mod W)."""
    L, Hkv, d = hist.shape
    ring = np.zeros((Hkv, window, d), dtype=hist.dtype)
    for p in range(max(0, L - window), L):
        ring[:, p % window] = hist[p]
    return ring
