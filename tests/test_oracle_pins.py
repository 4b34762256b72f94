"""Pins for the fp64 oracle, checked against facts that do not come from the oracle itself.

Each test fixes one part of the definition so that a plausible slip (a wrong rotation
sign, pair layout, frequency, cut-off, window edge, head mapping, rotated values, a
dropped softmax term) fails at least one of them:

* closed forms of the rotation for basis vectors (sign, half-split pairs, theta_j, p);
* recovery of the visible key set by brute force on L <= 8 for every W in 1..9;
* special cases with a known answer (W = 1, position 0, equal keys, all-ones values);
* GQA against explicitly replicated heads, W >= L against global;
* invariance of scores to a shift of all positions, and to positions at all when p = 0;
* an independent routine: torch's SDPA in float64 on CPU, with the rotation applied by
  complex multiplication written here;
* split-then-combine against the unsplit result; decode rows against prefill rows;
* tile counts against closed forms.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def one_seq(L):
    return np.arange(L, dtype=np.int32), np.array([0, L], dtype=np.int32)


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("pos", [0.0, 1.0, 7.0, 123456.0])
def test_rope_basis_closed_form(pos):
    d, base = 8, 1e4
    # theta_j = base^(-2j/d) = 10^(-j) for d = 8, base = 1e4
    for j in range(4):
        th = 10.0 ** (-j)
        e = np.zeros(d); e[j] = 1.0
        y = oracle.rope(e, 1.0, base, pos)
        want = np.zeros(d); want[j] = math.cos(pos * th); want[j + 4] = math.sin(pos * th)
        np.testing.assert_allclose(y, want, atol=1e-12)
        e2 = np.zeros(d); e2[j + 4] = 1.0
        y2 = oracle.rope(e2, 1.0, base, pos)
        want2 = np.zeros(d); want2[j] = -math.sin(pos * th); want2[j + 4] = math.cos(pos * th)
        np.testing.assert_allclose(y2, want2, atol=1e-12)


def test_rope_p_cutoff_rotates_highest_frequency_pairs_only():
    d = 16
    assert oracle.rotated_pairs(0.25, d) == 2
    assert oracle.rotated_pairs(0.25, 512) == 64
    assert oracle.rotated_pairs(0.25, 64) == 8
    assert oracle.rotated_pairs(1.0, 256) == 128
    assert oracle.rotated_pairs(0.0, 256) == 0
    rng = np.random.default_rng(3)
    x = rng.standard_normal(d)
    y = oracle.rope(x, 0.25, 1e4, 37.0)
    # pairs j = 2..7 (dims 2..7 and 10..15) pass through unchanged
    np.testing.assert_array_equal(y[2:8], x[2:8])
    np.testing.assert_array_equal(y[10:16], x[10:16])
    # pairs 0 and 1 are rotated, with theta = 1 and 1e4^(-1/8)
    for j, th in ((0, 1.0), (1, 1e4 ** (-2.0 / 16))):
        a = 37.0 * th
        assert abs(y[j] - (x[j] * math.cos(a) - x[j + 8] * math.sin(a))) < 1e-12
        assert abs(y[j + 8] - (x[j] * math.sin(a) + x[j + 8] * math.cos(a))) < 1e-12


def test_rope_preserves_norm():
    rng = np.random.default_rng(5)
    for d in (8, 64, 512):
        x = rng.standard_normal(d)
        for p in (0.25, 0.5, 1.0):
            y = oracle.rope(x, p, 1e6, 98765.0)
            assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-10


# ---------------------------------------------------------------- scores through attention

def _two_key_out(d, q, k0, k1, v0, v1, pos, rope_p, base=1e4, scale=1.0):
    """Row 1 of a 2-token global sequence; every vector exactly representable in bf16."""
    qq = np.zeros((2, 1, d), np.float32); qq[1, 0] = q
    kk = np.stack([k0, k1])[:, None, :].astype(np.float32)
    vv = np.stack([v0, v1])[:, None, :].astype(np.float32)
    out, lse = oracle.attention(W.GLOBAL, 0, rope_p, base, scale, bits(qq), bits(kk), bits(vv),
                                np.array(pos, np.int32), np.array([0, 2], np.int32), rows=np.array([1], np.int32))
    return out[0, 0], lse[0, 0]


def test_score_sign_and_unrotated_values():
    # d = 2: q = (1,0) at position 6, k0 = (0,1) at 5, k1 = (1,0) at 6.
    # <R_6 q, R_5 k0> = sin(6 - 5) (counter-clockwise); <R_6 q, R_6 k1> = 1.
    e0, e1 = np.array([1.0, 0.0]), np.array([0.0, 1.0])
    out, lse = _two_key_out(2, e0, e1, e0, e0, e1, [5, 6], 1.0)
    z0, z1 = math.sin(1.0), 1.0
    w0 = math.exp(z0) / (math.exp(z0) + math.exp(z1))
    # values are the un-rotated tensors: out = w0 * (1,0) + w1 * (0,1)
    np.testing.assert_allclose(out, [w0, 1.0 - w0], atol=1e-12)
    assert abs(lse - math.log(math.exp(z0) + math.exp(z1))) < 1e-12


def test_half_split_pairs_and_frequency_in_scores():
    # d = 8, base 1e4: pair 1 is (dim 1, dim 5) with theta_1 = 0.1.
    d = 8
    e = np.eye(d)
    out, _ = _two_key_out(d, e[1], e[5], np.zeros(d), e[0], e[2], [0, 3], 1.0)
    z0 = math.sin(3 * 0.1)          # <R_3 e1, R_0 e5> = sin(3 * theta_1); z1 = 0
    w0 = math.exp(z0) / (math.exp(z0) + 1.0)
    np.testing.assert_allclose(out, w0 * e[0] + (1 - w0) * e[2], atol=1e-12)


def test_p_rope_leaves_low_frequency_pairs_in_scores():
    # d = 8, p = 0.25 -> one rotated pair (dims 0 and 4). Pair 1 passes through: <e1, e5> = 0 always,
    # while pair 0 gives sin((a - b) * theta_0) = sin(3).
    d = 8
    e = np.eye(d)
    out_low, _ = _two_key_out(d, e[1], e[5], np.zeros(d), e[0], e[2], [0, 3], 0.25)
    np.testing.assert_allclose(out_low, 0.5 * e[0] + 0.5 * e[2], atol=1e-12)
    out_high, _ = _two_key_out(d, e[0], e[4], np.zeros(d), e[0], e[2], [0, 3], 0.25)
    w0 = math.exp(math.sin(3.0)) / (math.exp(math.sin(3.0)) + 1.0)
    np.testing.assert_allclose(out_high, w0 * e[0] + (1 - w0) * e[2], atol=1e-12)


# ---------------------------------------------------------------- visibility by brute force

@pytest.mark.parametrize("L", [1, 2, 5, 8])
def test_visible_sets_brute_force(L):
    """q = 0 makes every visible key weigh the same; one-hot values then reveal the visible set."""
    d = 8
    q = np.zeros((L, 1, d), np.float32)
    k = np.random.default_rng(L).standard_normal((L, 1, d)).astype(np.float32)
    v = np.zeros((L, 1, d), np.float32)
    for t in range(L):
        v[t, 0, t] = 1.0
    pos, cu = one_seq(L)
    for kind, windows in ((W.LOCAL, range(1, 10)), (W.GLOBAL, [0])):
        for w in windows:
            out, _ = oracle.attention(kind, w, 1.0, 1e4, 1.0, bits(q), bits(k), bits(v), pos, cu)
            for i in range(L):
                vis = [t for t in range(L) if t <= i and (kind == W.GLOBAL or i - w < t)]
                want = np.zeros(d)
                want[vis] = 1.0 / len(vis)
                np.testing.assert_allclose(out[i, 0], want, atol=1e-15)


def test_sequences_do_not_see_each_other():
    d = 8
    lens = [3, 5]
    T = sum(lens)
    q = np.zeros((T, 1, d), np.float32)
    k = np.ones((T, 1, d), np.float32)
    v = np.zeros((T, 1, d), np.float32)
    for t in range(T):
        v[t, 0, t] = 1.0
    pos = np.array([0, 1, 2, 0, 1, 2, 3, 4], np.int32)
    cu = np.array([0, 3, 8], np.int32)
    out, _ = oracle.attention(W.GLOBAL, 0, 0.25, 1e4, 1.0, bits(q), bits(k), bits(v), pos, cu)
    np.testing.assert_allclose(out[3, 0], np.eye(d)[3], atol=1e-15)   # first token of seq 1 sees only itself
    np.testing.assert_allclose(out[2, 0], np.eye(d)[:3].mean(0), atol=1e-15)


# ---------------------------------------------------------------- special cases

def _rand_layer(L, Hq, Hkv, d, seed, kv_equal=False):
    q = W.normal_bf16(seed, 0, (L, Hq, d))
    k = W.normal_bf16(seed, 1, (L, Hkv, d))
    v = None if kv_equal else W.normal_bf16(seed, 2, (L, Hkv, d))
    return q, k, v


def test_window_one_returns_own_value():
    L, d = 12, 16
    q, k, v = _rand_layer(L, 2, 1, d, 11)
    pos, cu = one_seq(L)
    out, _ = oracle.attention(W.LOCAL, 1, 1.0, 1e4, 0.25, q, k, v, pos, cu)
    vf = W.bf16_bits_to_f32(v).astype(np.float64)
    for h in range(2):
        np.testing.assert_array_equal(out[:, h], vf[:, 0])


def test_first_position_and_equal_keys():
    L, d = 9, 16
    q, k, v = _rand_layer(L, 4, 2, d, 12)
    pos, cu = one_seq(L)
    vf = W.bf16_bits_to_f32(v).astype(np.float64)
    out, _ = oracle.attention(W.GLOBAL, 0, 0.25, 1e6, 0.25, q, k, v, pos, cu)
    for h in range(4):
        np.testing.assert_array_equal(out[0, h], vf[0, h // 2])
    # all keys equal and p = 0 -> equal scores -> mean of the visible values
    k_eq = np.repeat(k[:1], L, axis=0)
    for kind, w in ((W.GLOBAL, 0), (W.LOCAL, 4)):
        out, _ = oracle.attention(kind, w, 0.0, 1e4, 0.25, q, k_eq, v, pos, cu)
        for i in range(L):
            lo = 0 if kind == W.GLOBAL else max(0, i - w + 1)
            np.testing.assert_allclose(out[i, 1], vf[lo:i + 1, 0].mean(0), atol=1e-13)


def test_weights_sum_to_one():
    L, d = 20, 32
    q, k, _ = _rand_layer(L, 2, 2, d, 13)
    ones = bits(np.ones((L, 2, d)))
    pos, cu = one_seq(L)
    for kind, w in ((W.GLOBAL, 0), (W.LOCAL, 5)):
        out, _ = oracle.attention(kind, w, 1.0, 1e4, 0.2, q, k, ones, pos, cu)
        np.testing.assert_allclose(out, 1.0, atol=1e-12)


def test_gqa_equals_replicated_heads():
    L, d, Hq, Hkv = 17, 16, 8, 2
    q, k, v = _rand_layer(L, Hq, Hkv, d, 14)
    pos, cu = one_seq(L)
    rep = np.repeat(np.arange(Hkv), Hq // Hkv)   # head h -> kv head h // (Hq/Hkv)
    for kind, w, kv_eq in ((W.LOCAL, 6, False), (W.GLOBAL, 0, True)):
        vv = None if kv_eq else v
        a, la = oracle.attention(kind, w, 0.25, 1e4, 0.25, q, k, vv, pos, cu)
        b, lb = oracle.attention(kind, w, 0.25, 1e4, 0.25, q, k[:, rep], None if kv_eq else v[:, rep], pos, cu)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)
        np.testing.assert_allclose(la, lb, rtol=0, atol=1e-14)


def test_wide_window_equals_global():
    L, d = 23, 16
    q, k, v = _rand_layer(L, 2, 1, d, 15)
    pos, cu = one_seq(L)
    for w in (L, L + 7):
        a, la = oracle.attention(W.LOCAL, w, 0.25, 1e4, 0.25, q, k, v, pos, cu)
        b, lb = oracle.attention(W.GLOBAL, 0, 0.25, 1e4, 0.25, q, k, v, pos, cu)
        np.testing.assert_array_equal(a, b)
        np.testing.assert_array_equal(la, lb)


def test_p_zero_ignores_absolute_position():
    L, d = 15, 16
    q, k, v = _rand_layer(L, 2, 1, d, 16)
    pos, cu = one_seq(L)
    a, _ = oracle.attention(W.LOCAL, 5, 0.0, 1e4, 0.25, q, k, v, pos, cu)
    b, _ = oracle.attention(W.LOCAL, 5, 0.0, 1e4, 0.25, q, k, v, pos + 98765, cu)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("shift", [1, 1000, 100000])
def test_scores_depend_only_on_relative_position(shift):
    L, d = 13, 32
    q, k, v = _rand_layer(L, 2, 1, d, 17)
    pos, cu = one_seq(L)
    for p, base in ((1.0, 1e4), (0.25, 1e6)):
        a, la = oracle.attention(W.GLOBAL, 0, p, base, 0.2, q, k, v, pos, cu)
        b, lb = oracle.attention(W.GLOBAL, 0, p, base, 0.2, q, k, v, pos + shift, cu)
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(la, lb, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- independent routine

def _complex_rope(x, pos, p, base):
    """Rotation written as complex multiplication of (x_j + i x_{j+d/2}) by exp(i pos theta_j)."""
    L, H, d = x.shape
    half = d // 2
    r = int(math.floor(p * d / 2))
    z = x[..., :half] + 1j * x[..., half:]
    th = base ** (-2.0 * np.arange(half) / d)
    ang = np.where(np.arange(half) < r, 1.0, 0.0)[None, :] * (pos[:, None] * th[None, :])
    z = z * np.exp(1j * ang)[:, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("kind,w,p,base,kv_eq", [
    (W.GLOBAL, 0, 0.0, 1e4, True),
    (W.GLOBAL, 0, 0.25, 1e6, True),
    (W.LOCAL, 7, 1.0, 1e4, False),
    (W.LOCAL, 1, 0.5, 1e4, False),
])
def test_against_torch_sdpa(kind, w, p, base, kv_eq):
    L, Hq, Hkv, d = 29, 4, 2, 16
    q, k, v = _rand_layer(L, Hq, Hkv, d, 18, kv_equal=kv_eq)
    pos, cu = one_seq(L)
    pos = pos + 40
    scale = 1.0 / math.sqrt(d)
    out, lse = oracle.attention(kind, w, p, base, scale, q, k, v, pos, cu)
    qf = W.bf16_bits_to_f32(q).astype(np.float64)
    kf = W.bf16_bits_to_f32(k).astype(np.float64)
    vf = kf if kv_eq else W.bf16_bits_to_f32(v).astype(np.float64)
    qr = _complex_rope(qf, pos.astype(np.float64), p, base)
    kr = _complex_rope(kf, pos.astype(np.float64), p, base)
    rep = np.repeat(np.arange(Hkv), Hq // Hkv)
    Q = torch.from_numpy(qr.transpose(1, 0, 2))
    K = torch.from_numpy(kr[:, rep].transpose(1, 0, 2))
    V = torch.from_numpy(vf[:, rep].transpose(1, 0, 2))
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    allowed = (j <= i) if kind == W.GLOBAL else ((j <= i) & (i - w < j))
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(allowed), scale=scale)
    np.testing.assert_allclose(out, ref.numpy().transpose(1, 0, 2), rtol=1e-11, atol=1e-11)
    s = torch.einsum("hid,hjd->hij", Q, K) * scale
    s = s.masked_fill(~torch.from_numpy(allowed), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy().T, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- splits, combine, decode

def test_split_and_combine_equals_unsplit():
    L, d = 40, 16
    q, k, v = _rand_layer(L, 4, 2, d, 19)
    pos, cu = one_seq(L)
    full, lfull = oracle.attention(W.LOCAL, 13, 1.0, 1e4, 0.25, q, k, v, pos, cu)
    for cuts in ([0, 40], [0, 7, 40], [0, 10, 20, 30, 40], [0, 1, 2, 39, 40]):
        parts = [oracle.attention(W.LOCAL, 13, 1.0, 1e4, 0.25, q, k, v, pos, cu, key_range=(a, b))
                 for a, b in zip(cuts[:-1], cuts[1:])]
        po = np.stack([p_[0].reshape(-1, d) for p_ in parts])
        pl = np.stack([p_[1].reshape(-1) for p_ in parts])
        o, l = oracle.combine(po, pl)
        np.testing.assert_allclose(o.reshape(full.shape), full, atol=1e-12)
        np.testing.assert_allclose(l.reshape(lfull.shape), lfull, atol=1e-12)


def test_combine_closed_form():
    # two splits with lse 0 and log 3 -> weights 1/4 and 3/4
    po = np.array([[[4.0, 0.0]], [[0.0, 8.0]]])
    pl = np.array([[0.0], [math.log(3.0)]])
    o, l = oracle.combine(po, pl)
    np.testing.assert_allclose(o, [[1.0, 6.0]], atol=1e-15)
    assert abs(l[0] - math.log(4.0)) < 1e-15
    o, l = oracle.combine(np.zeros((2, 1, 2)), np.full((2, 1), -np.inf))
    assert l[0] == -np.inf and np.all(o == 0)
    # the weights depend on lse differences only: a common shift by +-1e4 (exp of which
    # overflows or underflows fp64) leaves the merge unchanged and shifts the lse
    for shift in (1e4, -1e4):
        o, l = oracle.combine(po, pl + shift)
        np.testing.assert_allclose(o, [[1.0, 6.0]], atol=1e-12)
        assert abs(l[0] - (shift + math.log(4.0))) < 1e-9


def test_decode_equals_prefill_rows():
    Hq, Hkv, d, n_q = 4, 2, 16, 3
    lens = [5, 11]
    qs, ks, vs, rows_out = [], [], [], []
    for b, n in enumerate(lens):
        L = n + n_q
        q, k, v = _rand_layer(L, Hq, Hkv, d, 30 + b)
        qs.append(q[n:]); ks.append(k); vs.append(v)
        pos, cu = one_seq(L)
        o, _ = oracle.attention(W.LOCAL, 6, 1.0, 1e4, 0.25, q, k, v, pos, cu)
        rows_out.append(o[n:])
    out, _ = oracle.decode(W.LOCAL, 6, 1.0, 1e4, 0.25, np.stack(qs), ks, vs, lens)
    for b in range(2):
        np.testing.assert_array_equal(out[b], rows_out[b])


# ---------------------------------------------------------------- tile plan

def test_tile_plan_closed_form_counts():
    for L, bm in ((1000, 128), (64, 16), (300, 64)):
        pos, cu = one_seq(L)
        nt = (L + bm - 1) // bm
        plan = oracle.tile_plan(W.GLOBAL, 0, pos, cu, bm, bm)
        assert len(plan) == nt * (nt + 1) // 2
        for s, qt, kt, c in plan:
            assert kt <= qt
            assert c == (1 if kt == qt else 2)
        for w in (1, bm, 3 * bm, 3 * bm + 5):
            plan = oracle.tile_plan(W.LOCAL, w, pos, cu, bm, bm)
            want = 0
            for qt in range(nt):
                lo_key = max(0, qt * bm - w + 1)
                want += qt - lo_key // bm + 1
            assert len(plan) == want, (L, bm, w)


# ---------------------------------------------------------------- page parameters

def test_workload_shapes_follow_page_parameters():
    g = json.load(open(os.path.join(HERE, "golden", "architecture_params.json")))
    e2b = W.e2b_block()
    kinds = [l.kind for l in e2b.layers]
    assert kinds == [W.LOCAL] * g["interleave_e2b"]["value"][0] + [W.GLOBAL] * g["interleave_e2b"]["value"][1]
    b31 = W.b31_block()
    assert [l.kind for l in b31.layers] == [W.LOCAL] * g["interleave_others"]["value"][0] + [W.GLOBAL]
    for blk, win in ((e2b, g["sliding_window_small_models"]["value"]), (b31, g["sliding_window_large_models"]["value"])):
        assert blk.layers[-1].kind == W.GLOBAL
        for l in blk.layers:
            if l.kind == W.LOCAL:
                assert l.window == win and l.head_dim == g["local_head_dim"]["value"]
                assert l.num_q_heads // l.num_kv_heads == g["local_q_per_kv"]["value"]
            else:
                assert l.head_dim == g["global_head_dim"]["value"] and l.k_eq_v
                assert l.num_q_heads // l.num_kv_heads == g["global_q_per_kv"]["value"]
                assert l.rope_p == g["p_rope_p"]["value"]
    assert W.long_decode().cache_lens[0] == g["context_small"]["value"]
