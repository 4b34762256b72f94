"""Pins for the oracle's bidirectional 2D-RoPE attention (the vision encoder's patches),
checked against facts that do not come from that routine itself:

* the 2D rotation of each half of the dims equals the 1D rotation (itself pinned by
  closed forms in test_oracle_pins.py) of that half-vector for w (first half) and h
  (second half); a zero position leaves its half unchanged; the norm is preserved;
* scores depend only on position differences: shifting every h, or every w, by a
  constant leaves the output unchanged; with all positions equal the rotation drops out;
* an independent routine: torch's SDPA in float64 without a mask, on q and k rotated by
  complex multiplication written here, per image;
* permuting the patches of an image (with their positions) permutes the outputs;
* GQA equals explicitly replicated KV heads; images do not see each other;
* the tile plan of a bidirectional layer: every tile of an image, each full (every
  in-image pair of it visible).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def _rand(L, Hq, Hkv, d, seed, kv_equal=False):
    q = W.normal_bf16(seed, 0, (L, Hq, d))
    k = W.normal_bf16(seed, 1, (L, Hkv, d))
    v = None if kv_equal else W.normal_bf16(seed, 2, (L, Hkv, d))
    return q, k, v


def _grid(n, width, h0=0, w0=0):
    """(h, w) of n patches laid out row by row in an image `width` patches wide."""
    idx = np.arange(n)
    return np.stack([h0 + idx // width, w0 + idx % width], axis=1).astype(np.int32)


def test_rope2d_halves_are_1d_rotations():
    rng = np.random.default_rng(3)
    for d in (16, 64, 128):
        x = rng.standard_normal(d)
        for h, w in ((0, 0), (3, 0), (0, 7), (11, 5), (40000, 123)):
            y = oracle.rope2d(x, 1e4, h, w)
            np.testing.assert_allclose(y[:d // 2], oracle.rope(x[:d // 2], 1.0, 1e4, w), rtol=0, atol=1e-12)
            np.testing.assert_allclose(y[d // 2:], oracle.rope(x[d // 2:], 1.0, 1e4, h), rtol=0, atol=1e-12)
            assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
            if w == 0:
                np.testing.assert_array_equal(y[:d // 2], x[:d // 2])
            if h == 0:
                np.testing.assert_array_equal(y[d // 2:], x[d // 2:])


@pytest.mark.parametrize("dh,dw", [(1, 0), (0, 1), (1000, 0), (0, 1000), (37, 91)])
def test_shift_of_h_or_w_leaves_output_unchanged(dh, dw):
    L, d = 23, 32
    q, k, v = _rand(L, 2, 1, d, 5)
    cu = np.array([0, L], np.int32)
    hw = _grid(L, 5)
    out0, lse0 = oracle.attention_2d(1e4, 1 / math.sqrt(d), q, k, v, hw, cu)
    out1, lse1 = oracle.attention_2d(1e4, 1 / math.sqrt(d), q, k, v, hw + np.array([dh, dw], np.int32), cu)
    np.testing.assert_allclose(out1, out0, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(lse1, lse0, rtol=1e-10, atol=1e-10)


def _complex_rope2d(x, hw, base):
    """Each half rotated as complex numbers (x_j + i x_{j+d/4}) times exp(i pos theta_j)."""
    L, H, d = x.shape
    half, q4 = d // 2, d // 4
    th = base ** (-2.0 * np.arange(q4) / half)
    out = np.empty_like(x)
    for part, pos in ((0, hw[:, 1]), (1, hw[:, 0])):  # first half w, second half h
        seg = x[..., part * half:(part + 1) * half]
        z = (seg[..., :q4] + 1j * seg[..., q4:]) * np.exp(1j * pos[:, None, None] * th[None, None, :])
        out[..., part * half:part * half + q4] = z.real
        out[..., part * half + q4:(part + 1) * half] = z.imag
    return out


@pytest.mark.parametrize("kv_eq", [False, True])
def test_against_torch_sdpa_without_mask(kv_eq):
    lens = (13, 21)
    Hq, Hkv, d = 4, 2, 16
    T = sum(lens)
    q, k, v = _rand(T, Hq, Hkv, d, 8, kv_equal=kv_eq)
    cu = np.array([0, lens[0], T], np.int32)
    hw = np.concatenate([_grid(lens[0], 4, 2, 1), _grid(lens[1], 7)])
    scale = 1 / math.sqrt(d)
    out, lse = oracle.attention_2d(1e4, scale, q, k, v, hw, cu)
    qf = W.bf16_bits_to_f32(q).astype(np.float64)
    kf = W.bf16_bits_to_f32(k).astype(np.float64)
    vf = kf if kv_eq else W.bf16_bits_to_f32(v).astype(np.float64)
    qr = _complex_rope2d(qf, hw.astype(np.float64), 1e4)
    kr = _complex_rope2d(kf, hw.astype(np.float64), 1e4)
    rep = np.repeat(np.arange(Hkv), Hq // Hkv)
    for s in range(2):
        a, b = cu[s], cu[s + 1]
        Q = torch.from_numpy(qr[a:b].transpose(1, 0, 2).copy())
        K = torch.from_numpy(kr[a:b][:, rep].transpose(1, 0, 2).copy())
        V = torch.from_numpy(vf[a:b][:, rep].transpose(1, 0, 2).copy())
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)
        np.testing.assert_allclose(out[a:b], ref.numpy().transpose(1, 0, 2), rtol=1e-11, atol=1e-11)
        sc = torch.einsum("hid,hjd->hij", Q, K) * scale
        np.testing.assert_allclose(lse[a:b], torch.logsumexp(sc, dim=-1).numpy().T, rtol=1e-11, atol=1e-11)


def test_equal_positions_drop_the_rotation():
    """All patches at one (h, w): the rotation is the same for q and k and cancels."""
    L, d = 17, 32
    q, k, v = _rand(L, 2, 2, d, 9)
    cu = np.array([0, L], np.int32)
    at = np.tile(np.array([[6, 9]], np.int32), (L, 1))
    zero = np.zeros((L, 2), np.int32)
    out_a, _ = oracle.attention_2d(1e4, 0.3, q, k, v, at, cu)
    out_0, _ = oracle.attention_2d(1e4, 0.3, q, k, v, zero, cu)
    np.testing.assert_allclose(out_a, out_0, rtol=1e-11, atol=1e-11)


def test_patch_permutation_permutes_outputs():
    L, d = 19, 16
    q, k, v = _rand(L, 2, 1, d, 10)
    cu = np.array([0, L], np.int32)
    hw = _grid(L, 6)
    perm = np.random.default_rng(4).permutation(L)
    out, lse = oracle.attention_2d(1e4, 0.25, q, k, v, hw, cu)
    out_p, lse_p = oracle.attention_2d(1e4, 0.25, q[perm], k[perm], v[perm], hw[perm], cu)
    np.testing.assert_allclose(out_p, out[perm], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(lse_p, lse[perm], rtol=1e-11, atol=1e-11)


def test_gqa_and_images_apart():
    lens = (9, 14)
    T, Hq, Hkv, d = sum(lens), 4, 2, 16
    q, k, v = _rand(T, Hq, Hkv, d, 12)
    cu = np.array([0, lens[0], T], np.int32)
    hw = np.concatenate([_grid(lens[0], 3), _grid(lens[1], 4)])
    out, _ = oracle.attention_2d(1e4, 0.25, q, k, v, hw, cu)
    rep = np.repeat(np.arange(Hkv), Hq // Hkv)
    out_r, _ = oracle.attention_2d(1e4, 0.25, q, k[:, rep], v[:, rep], hw, cu)
    np.testing.assert_allclose(out, out_r, rtol=1e-12, atol=1e-12)
    # the second image alone gives the same rows
    out2, _ = oracle.attention_2d(1e4, 0.25, q[lens[0]:], k[lens[0]:], v[lens[0]:], hw[lens[0]:],
                                  np.array([0, lens[1]], np.int32))
    np.testing.assert_allclose(out[lens[0]:], out2, rtol=1e-12, atol=1e-12)


def test_bidirectional_tile_plan():
    lens = (200, 64, 129)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    tiles = oracle.tile_plan(oracle.BIDIR, 0, pos, cu, 128, 128)
    want = []
    for s, n in enumerate(lens):
        nt = (n + 127) // 128
        for qt in range(nt):
            for kt in range(nt):
                want.append((s, qt, kt, 2))
    assert [tuple(t) for t in tiles] == want
