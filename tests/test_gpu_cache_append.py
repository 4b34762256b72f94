"""KV-cache append through the C-ABI, against the oracle.

gemma_attn_cache_append writes the new tokens' rows into a decode cache. Checked here:
  - un-rotated caches (global K=V contiguous, local ring): the rows land bit-exactly at
    slot position mod window / row position; every other row is untouched;
  - a ring that keeps keys rotated: the stored key is the oracle's p-RoPE rotation of the
    new key for its position, rounded to bf16, within one bf16 ulp (fp32 against fp64
    arithmetic before the rounding); values are copied bit-exactly;
  - a full decode loop: decode token t (new rows beside the cache), append, decode token
    t + 1 from the extended cache -- each step equals the oracle over the whole history,
    including steps where the ring wraps;
  - a contiguous cache without room records GEMMA_ATTN_ERR_SEQLEN and writes nothing;
  - more new tokens than ring slots: the ring holds the newest window positions.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import assert_close, dev_bf16, dev_i32, host_bits, ring_from_history  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _params(layer):
    return G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, window=layer.window,
                    rope_p=layer.rope_p, rope_base=layer.rope_base, softmax_scale=layer.softmax_scale)


def _rotate_rows(rows_bits, layer, positions):
    """[n, Hkv, d] bf16 bits rotated by the oracle's p-RoPE for each row's position, rounded to bf16."""
    out = rows_bits.copy()
    for n, pos in enumerate(positions):
        for h in range(rows_bits.shape[1]):
            x = W.bf16_bits_to_f32(rows_bits[n, h]).astype(np.float64)
            out[n, h] = W.f32_to_bf16_bits(oracle.rope(x, layer.rope_p, layer.rope_base, pos).astype(np.float32))
    return out


@pytest.mark.parametrize("layer,layout,cache_lens,n_q", [
    (W.LayerSpec(W.GLOBAL, 8, 2, 512, rope_p=0.25, rope_base=1e6), G.CACHE_CONTIGUOUS, (0, 37, 300), 4),
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=64, rope_p=1.0, rope_base=1e4), G.CACHE_RING, (0, 62, 200), 4),
    (W.LayerSpec(W.LOCAL, 2, 1, 128, window=16, rope_p=1.0, rope_base=1e4), G.CACHE_RING, (5, 15), 1),
])
def test_append_places_rows_and_leaves_the_rest(layer, layout, cache_lens, n_q):
    B, Hkv, d = len(cache_lens), layer.num_kv_heads, layer.head_dim
    cap = layer.window if layout == G.CACHE_RING else max(cache_lens) + n_q
    rng = np.random.default_rng(5)
    kc0 = rng.integers(0, 1 << 16, size=(B, Hkv, cap, d), dtype=np.uint16) & np.uint16(0x7F7F)  # finite bf16
    vc0 = None if layer.k_eq_v else rng.integers(0, 1 << 16, size=(B, Hkv, cap, d), dtype=np.uint16) & np.uint16(0x7F7F)
    nk = W.normal_bf16(21, 1, (B, n_q, Hkv, d))
    nv = None if layer.k_eq_v else W.normal_bf16(21, 2, (B, n_q, Hkv, d))
    kc, vc = dev_bf16(kc0), (None if vc0 is None else dev_bf16(vc0))
    G.gemma_attn_cache_append(_params(layer), dev_bf16(nk), None if nv is None else dev_bf16(nv), kc, vc, layout, cap,
                              dev_i32(cache_lens), B, n_q)
    G.gemma_attn_check()
    exp_k, exp_v = kc0.copy(), (None if vc0 is None else vc0.copy())
    for b, n in enumerate(cache_lens):
        for i in range(n_q):
            slot = (n + i) % cap if layout == G.CACHE_RING else n + i
            exp_k[b, :, slot] = nk[b, i]
            if exp_v is not None:
                exp_v[b, :, slot] = nv[b, i]
    np.testing.assert_array_equal(host_bits(kc), exp_k)
    if vc is not None:
        np.testing.assert_array_equal(host_bits(vc), exp_v)


def test_append_rotates_keys_for_a_rotated_ring():
    layer = W.LayerSpec(W.LOCAL, 4, 2, 256, window=32, rope_p=1.0, rope_base=1e4)
    B, Hkv, d, n_q, cap = 3, 2, 256, 4, 32
    cache_lens = (0, 31, 1000)
    nk = W.normal_bf16(22, 1, (B, n_q, Hkv, d))
    nv = W.normal_bf16(22, 2, (B, n_q, Hkv, d))
    kc = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    G.gemma_attn_cache_append(_params(layer), dev_bf16(nk), dev_bf16(nv), kc, vc, G.CACHE_RING | G.CACHE_KEYS_ROTATED,
                              cap, dev_i32(cache_lens), B, n_q)
    G.gemma_attn_check()
    got_k, got_v = host_bits(kc), host_bits(vc)
    for b, n in enumerate(cache_lens):
        pos = [n + i for i in range(n_q)]
        want = _rotate_rows(nk[b], layer, pos)
        for i, p in enumerate(pos):
            g = W.bf16_bits_to_f32(got_k[b, :, p % cap]).astype(np.float64)
            w = W.bf16_bits_to_f32(want[i]).astype(np.float64)
            # at most one bf16 ulp apart (an ulp is at most 2^-7 of the magnitude)
            tol = np.maximum(np.abs(g), np.abs(w)) * 2.0 ** -7
            assert np.all(np.abs(g - w) <= tol), f"seq {b} position {p}"
            np.testing.assert_array_equal(got_v[b, :, p % cap], nv[b, i])


@pytest.mark.parametrize("layer,layout,rotated,start", [
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=16, rope_p=1.0, rope_base=1e4), G.CACHE_RING, True, (3, 14)),
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=16, rope_p=1.0, rope_base=1e4), G.CACHE_RING, False, (0, 20)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), G.CACHE_CONTIGUOUS, False, (1, 40)),
])
def test_decode_append_loop_matches_oracle(layer, layout, rotated, start):
    """Decode one token per step for several steps, appending after each; every step
    equals the oracle over the full history (the ring wraps during the loop)."""
    B, Hq, Hkv, d = len(start), layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    steps = 6
    hist_len = [n + steps for n in start]
    k_hist = [W.normal_bf16(31 + b, 1, (hist_len[b], Hkv, d)) for b in range(B)]
    v_hist = [None if layer.k_eq_v else W.normal_bf16(31 + b, 2, (hist_len[b], Hkv, d)) for b in range(B)]
    cap = layer.window if layout == G.CACHE_RING else max(hist_len)
    # initial cache: the first start[b] tokens (rotated for their positions when asked)
    k_src = [(_rotate_rows(k_hist[b][:start[b]], layer, range(start[b])) if rotated else k_hist[b][:start[b]])
             for b in range(B)]
    if layout == G.CACHE_RING:
        kc0 = np.stack([ring_from_history(k_src[b], cap) for b in range(B)])
        vc0 = None if layer.k_eq_v else np.stack([ring_from_history(v_hist[b][:start[b]], cap) for b in range(B)])
    else:
        kc0 = np.zeros((B, Hkv, cap, d), np.uint16)
        vc0 = None
        for b in range(B):
            kc0[b, :, :start[b]] = k_src[b].transpose(1, 0, 2)
    kc, vc = dev_bf16(kc0), (None if vc0 is None else dev_bf16(vc0))
    lay = layout | (G.CACHE_KEYS_ROTATED if rotated else 0)
    p = _params(layer)
    for s in range(steps):
        lens = [n + s for n in start]
        q = W.normal_bf16(77 + s, 0, (B, 1, Hq, d))
        nk = np.stack([k_hist[b][lens[b]:lens[b] + 1] for b in range(B)])
        nv = None if layer.k_eq_v else np.stack([v_hist[b][lens[b]:lens[b] + 1] for b in range(B)])
        ref, _ = oracle.decode(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale, q,
                               [k_hist[b][:lens[b] + 1] for b in range(B)],
                               None if layer.k_eq_v else [v_hist[b][:lens[b] + 1] for b in range(B)], lens)
        out = torch.empty((B, 1, Hq, d), dtype=torch.float32, device="cuda")
        pf = G.params(layer.kind, Hq, Hkv, d, window=layer.window, rope_p=layer.rope_p, rope_base=layer.rope_base,
                      softmax_scale=layer.softmax_scale, out_dtype=G.OUT_F32)
        nkd, nvd, lensd = dev_bf16(nk), (None if nv is None else dev_bf16(nv)), dev_i32(lens)
        G.gemma_attn_decode_noalloc(pf, dev_bf16(q), nkd, nvd, kc, vc, lay, cap, lensd, B, 1, max(lens), 1, out, None)
        G.gemma_attn_cache_append(p, nkd, nvd, kc, vc, lay, cap, lensd, B, 1)
        G.gemma_attn_check()
        assert_close(out.cpu().numpy(), ref, f"decode step {s} lens={lens}")


def test_append_without_room_records_seqlen_and_writes_nothing():
    layer = W.LayerSpec(W.GLOBAL, 8, 1, 64, rope_p=0.25, rope_base=1e4)
    B, Hkv, d, cap, n_q = 2, 1, 64, 10, 2
    kc = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    nk = dev_bf16(W.normal_bf16(3, 1, (B, n_q, Hkv, d)))
    G.gemma_attn_check()  # clear any earlier status
    # sequence 1 has 9 cached tokens: its second new token (position 10) has no row
    G.gemma_attn_cache_append(_params(layer), nk, None, kc, None, G.CACHE_CONTIGUOUS, cap, dev_i32([3, 9]), B, n_q)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_check()
    assert e.value.status == G.ERR_SEQLEN
    got = host_bits(kc)
    nk_h = host_bits(nk)
    np.testing.assert_array_equal(got[0, :, 3], nk_h[0, 0])
    np.testing.assert_array_equal(got[0, :, 4], nk_h[0, 1])
    np.testing.assert_array_equal(got[1, :, 9], nk_h[1, 0])
    assert not got[1, :, :9].any() and not got[0, :, 5:].any()


@pytest.mark.parametrize("rotated", [False, True])
def test_ring_append_with_more_tokens_than_slots_keeps_the_newest(rotated):
    """n_q > window: tokens i and i + W share a slot; the ring must end up holding the
    newest W positions (what ring_from_history builds from the whole history)."""
    layer = W.LayerSpec(W.LOCAL, 4, 2, 128, window=8, rope_p=1.0, rope_base=1e4)
    B, Hkv, d, cap, n_q = 2, 2, 128, 8, 19
    start = [5, 30]
    k_hist = [W.normal_bf16(51 + b, 1, (start[b] + n_q, Hkv, d)) for b in range(B)]
    v_hist = [W.normal_bf16(51 + b, 2, (start[b] + n_q, Hkv, d)) for b in range(B)]
    k_src = [(_rotate_rows(k_hist[b], layer, range(start[b] + n_q)) if rotated else k_hist[b]) for b in range(B)]
    kc0 = np.stack([ring_from_history(k_src[b][:start[b]], cap) for b in range(B)])
    vc0 = np.stack([ring_from_history(v_hist[b][:start[b]], cap) for b in range(B)])
    kc, vc = dev_bf16(kc0), dev_bf16(vc0)
    nk = np.stack([k_hist[b][start[b]:] for b in range(B)])
    nv = np.stack([v_hist[b][start[b]:] for b in range(B)])
    lay = G.CACHE_RING | (G.CACHE_KEYS_ROTATED if rotated else 0)
    G.gemma_attn_cache_append(_params(layer), dev_bf16(nk), dev_bf16(nv), kc, vc, lay, cap, dev_i32(start), B, n_q)
    G.gemma_attn_check()
    for b in range(B):
        np.testing.assert_array_equal(host_bits(vc)[b], ring_from_history(v_hist[b], cap))
        want_k = ring_from_history(k_src[b], cap)
        got_k = host_bits(kc)[b]
        if rotated:  # fp32 rotation against the oracle's fp64 one, then bf16: within one ulp
            g = W.bf16_bits_to_f32(got_k).astype(np.float64)
            w = W.bf16_bits_to_f32(want_k).astype(np.float64)
            assert np.all(np.abs(g - w) <= np.maximum(np.abs(g), np.abs(w)) * 2.0 ** -7)
        else:
            np.testing.assert_array_equal(got_k, want_k)
