"""GPU parity: the CUDA path (called through the C-ABI) against the fp64 oracle.

Bounds (from the acceptance criteria, bf16 in, fp32 accumulate): max-abs <= 1e-2 and
relative RMS <= 5e-3 on the fp32 outputs; lse within 1e-2. The bf16 output mode must
equal the fp32 output rounded to nearest even, bit for bit (a bf16 half-ulp alone is
1.6e-2 for |o| in [4, 8), so the bound is applied before that final rounding). Shapes span several 128-row tiles with ragged tails, GQA
ratios 2:1 and 8:1, head dims 32..512, windows from 1 to beyond the length,
K=V with p-RoPE, and position offsets.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import (assert_close, bf16_round, dev_bf16, dev_i32, host_bits, ring_from_history,  # noqa: E402
                      run_prefill)


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _bf16_to_f64(bits):
    return W.bf16_bits_to_f32(bits).astype(np.float64)


# ------------------------------------------------------------------ tensor-core operand forms

def test_umma_selftest_ss_kmajor():
    rng = np.random.default_rng(1)
    a = W.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    b = W.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    d = torch.zeros((128, 128), dtype=torch.float32, device="cuda")
    G.gemma_attn_selftest_umma(0, dev_bf16(a), dev_bf16(b), None, d)
    torch.cuda.synchronize()
    ref = _bf16_to_f64(a) @ _bf16_to_f64(b).T
    np.testing.assert_allclose(d.cpu().numpy(), ref, rtol=1e-4, atol=1e-3)


def test_umma_selftest_ts_mnmajor():
    rng = np.random.default_rng(2)
    p = W.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    v = W.f32_to_bf16_bits(rng.standard_normal((128, 64), dtype=np.float32))
    d = torch.zeros((128, 64), dtype=torch.float32, device="cuda")
    G.gemma_attn_selftest_umma(1, None, dev_bf16(v), dev_bf16(p), d)
    torch.cuda.synchronize()
    ref = _bf16_to_f64(p) @ _bf16_to_f64(v)
    np.testing.assert_allclose(d.cpu().numpy(), ref, rtol=1e-4, atol=1e-3)


def test_bounded_wait_times_out_and_context_survives():
    # A wait on a barrier nothing arrives at gives up after its limit, the status word
    # reports the timeout once, and later launches run normally.
    G.gemma_attn_check()
    flag = torch.zeros((1,), dtype=torch.int32, device="cuda")
    G.gemma_attn_selftest_timeout(flag)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_check()
    assert e.value.status == G.ERR_TIMEOUT
    assert int(flag.item()) == 1
    G.gemma_attn_check()  # cleared
    test_umma_selftest_ss_kmajor()


def test_umma_selftest_ts_mnmajor_two_chunks():
    # N = 128: the second 64-column chunk is reached through the descriptor's leading
    # byte offset, as in the paired kernel's N = 256 value product.
    rng = np.random.default_rng(3)
    p = W.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    v = W.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    d = torch.zeros((128, 128), dtype=torch.float32, device="cuda")
    G.gemma_attn_selftest_umma(2, None, dev_bf16(v), dev_bf16(p), d)
    torch.cuda.synchronize()
    ref = _bf16_to_f64(p) @ _bf16_to_f64(v)
    np.testing.assert_allclose(d.cpu().numpy(), ref, rtol=1e-4, atol=1e-3)


# ------------------------------------------------------------------ prefill

def _check_prefill(layer, seq_lens, seed=0, pos_start=0, rows=None):
    T = int(sum(seq_lens))
    q, k, v = W.layer_inputs(layer, T, seed)
    cu = np.concatenate([[0], np.cumsum(seq_lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) + pos_start for n in seq_lens]).astype(np.int32)
    out32, lse = run_prefill(G, layer, q, k, v, pos, cu, out_f32=True)
    out16, _ = run_prefill(G, layer, q, k, v, pos, cu, with_lse=False)
    got = out32.cpu().numpy()
    got_lse = lse.cpu().numpy()
    np.testing.assert_array_equal(W.bf16_bits_to_f32(host_bits(out16)), bf16_round(got))
    ref, ref_lse = oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                                    q, k, v, pos, cu, rows=rows)
    if rows is not None:
        got = got[rows]
        got_lse = got_lse[:, rows]
    assert_close(got, ref, f"prefill {layer} lens={seq_lens}")
    np.testing.assert_allclose(got_lse.T, ref_lse, atol=1e-2, rtol=0)


def test_prefill_tiny_config_both_layers():
    wl = W.tiny_ref()
    for layer in wl.layers:
        _check_prefill(layer, wl.seq_lens, seed=wl.seed)


@pytest.mark.parametrize("layer,lens", [
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=300, rope_p=1.0, rope_base=1e4), (700,)),
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=512, rope_p=1.0, rope_base=1e4), (1, 129, 300, 513)),
    (W.LayerSpec(W.LOCAL, 2, 1, 256, window=1, rope_p=1.0, rope_base=1e4), (257,)),
    (W.LayerSpec(W.LOCAL, 2, 1, 256, window=5000, rope_p=1.0, rope_base=1e4), (300,)),
    (W.LayerSpec(W.LOCAL, 4, 2, 128, window=200, rope_p=1.0, rope_base=1e4), (450,)),
    (W.LayerSpec(W.LOCAL, 4, 2, 64, window=100, rope_p=0.5, rope_base=1e4), (333,)),
    (W.LayerSpec(W.LOCAL, 4, 2, 32, window=40, rope_p=1.0, rope_base=1e4), (200, 77)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (600,)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (1, 200, 257)),
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.0, rope_base=1e6), (300,)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 256, rope_p=0.25, rope_base=1e4), (390,)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 64, rope_p=0.25, rope_base=1e4), (260,)),
    (W.LayerSpec(W.LOCAL, 4, 2, 512, window=150, rope_p=0.25, rope_base=1e4), (333, 64)),
    (W.LayerSpec(W.GLOBAL, 4, 2, 512, rope_p=1.0, rope_base=1e4), (129, 65)),
])
def test_prefill_shapes(layer, lens):
    _check_prefill(layer, lens, seed=3)


# The single-CTA kernel at head dims >= 128: it runs when a query head has no partner that
# shares its KV head (an odd GQA group: 1 or 3 query heads per KV head here), and for every
# group when GEMMA_ATTN_NO_PAIR=1 is set (GQA mapping: "Visual guide to Gemma 4", section
# "GQA").
@pytest.mark.parametrize("layer,lens", [
    (W.LayerSpec(W.LOCAL, 3, 3, 128, window=200, rope_p=1.0, rope_base=1e4), (300, 129)),
    (W.LayerSpec(W.LOCAL, 3, 1, 256, window=300, rope_p=1.0, rope_base=1e4), (1, 400, 257)),
    (W.LayerSpec(W.LOCAL, 2, 2, 512, window=150, rope_p=0.25, rope_base=1e4), (333,)),
    (W.LayerSpec(W.GLOBAL, 1, 1, 128, rope_p=0.25, rope_base=1e6), (390, 7)),
    (W.LayerSpec(W.GLOBAL, 3, 3, 256, rope_p=0.25, rope_base=1e4), (260, 1)),
    (W.LayerSpec(W.GLOBAL, 3, 1, 512, rope_p=0.25, rope_base=1e6), (1, 200, 333)),
])
def test_prefill_single_cta_kernel_odd_group(layer, lens):
    _check_prefill(layer, lens, seed=6)


@pytest.mark.parametrize("layer,lens", [
    (W.LayerSpec(W.LOCAL, 4, 2, 256, window=512, rope_p=1.0, rope_base=1e4), (1, 129, 300, 513)),
    (W.LayerSpec(W.LOCAL, 4, 2, 128, window=200, rope_p=1.0, rope_base=1e4), (450,)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (1, 200, 257)),
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.0, rope_base=1e6), (300,)),
    (W.LayerSpec(W.GLOBAL, 8, 1, 256, rope_p=0.25, rope_base=1e4), (390,)),
])
def test_prefill_even_group_on_the_single_cta_kernel(layer, lens, monkeypatch):
    # the library reads the variable at every call
    monkeypatch.setenv("GEMMA_ATTN_NO_PAIR", "1")
    _check_prefill(layer, lens, seed=3)


@pytest.mark.parametrize("out_f32", [False, True])
def test_prefill_output_only_16_byte_aligned(out_f32):
    # 32-byte output stores are used only where the output allows them; a 16-byte aligned
    # output takes 16-byte stores and gives the same values
    layer = W.LayerSpec(W.LOCAL, 4, 2, 256, window=100, rope_p=1.0, rope_base=1e4)
    q, k, v = W.layer_inputs(layer, 300, 8)
    cu = np.array([0, 300], np.int32)
    pos = np.arange(300, dtype=np.int32)
    a, _ = run_prefill(G, layer, q, k, v, pos, cu, out_f32=out_f32)
    b, _ = run_prefill(G, layer, q, k, v, pos, cu, out_f32=out_f32, out_offset_bytes=16)
    assert b.data_ptr() % 32 == 16
    assert torch.equal(a, b)


def test_prefill_rotate_then_attend_equals_prefill():
    layer = W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
    T = 400
    q, k, _ = W.layer_inputs(layer, T, 12)
    full, _ = run_prefill(G, layer, q, k, None, np.arange(T, dtype=np.int32), np.array([0, T], np.int32))
    p = G.params(layer.kind, 8, 1, 512, rope_p=0.25, rope_base=1e6, softmax_scale=layer.softmax_scale)
    ws_bytes = G.gemma_attn_prefill_workspace_size(p, T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((T, 8, 512), dtype=torch.bfloat16, device="cuda")
    args = (dev_bf16(q), dev_bf16(k), None, out, None, dev_i32(np.arange(T)), dev_i32(np.array([0, T])), 1, T, T,
            ws, ws_bytes)
    G.gemma_attn_prefill_rotate(p, *args)
    assert G.gemma_attn_last_launch_count() == 1
    G.gemma_attn_prefill_attend(p, *args)
    assert G.gemma_attn_last_launch_count() == 1
    G.gemma_attn_check()
    assert torch.equal(out, full)


def test_prefill_position_offset():
    layer = W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
    _check_prefill(layer, (300,), seed=4, pos_start=100000)
    layer = W.LayerSpec(W.LOCAL, 4, 2, 256, window=128, rope_p=1.0, rope_base=1e4)
    _check_prefill(layer, (300,), seed=5, pos_start=60000)


def test_prefill_seqlen_violation_reported():
    layer = W.LayerSpec(W.LOCAL, 2, 1, 64, window=16)
    q, k, v = W.layer_inputs(layer, 300, 0)
    p = G.params(layer.kind, 2, 1, 64, window=16)
    ws_bytes = G.gemma_attn_prefill_workspace_size(p, 300)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty((300, 2, 64), dtype=torch.bfloat16, device="cuda")
    G.gemma_attn_prefill(p, dev_bf16(q), dev_bf16(k), dev_bf16(v), out, None, dev_i32(np.arange(300)),
                         dev_i32([0, 300]), 1, 300, 100, ws, ws_bytes)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_check()
    assert e.value.status == G.ERR_SEQLEN
    G.gemma_attn_check()  # cleared


# ------------------------------------------------------------------ decode / verify + combine

def _rotated_history(k_hist_b, n, layer):
    """Cached rows 0..n-1 of one sequence's key history rotated for their positions by the
    oracle's p-RoPE and rounded to bf16 (the pre-rotated cache layout); new rows stay."""
    out = k_hist_b.copy()
    for p in range(n):
        for h in range(k_hist_b.shape[1]):
            x = W.bf16_bits_to_f32(k_hist_b[p, h]).astype(np.float64)
            out[p, h] = W.f32_to_bf16_bits(oracle.rope(x, layer.rope_p, layer.rope_base, p).astype(np.float32))
    return out


def _check_decode(layer, cache_lens, n_q, layout, num_splits=None, seed=11, keys_rotated=False, junk=False):
    B = len(cache_lens)
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    rng_seed = seed
    k_hist, v_hist = [], []
    for b, n in enumerate(cache_lens):
        k_hist.append(W.normal_bf16(rng_seed + 100 * b, 1, (n + n_q, Hkv, d)))
        v_hist.append(None if layer.k_eq_v else W.normal_bf16(rng_seed + 100 * b, 2, (n + n_q, Hkv, d)))
    q = W.normal_bf16(rng_seed, 0, (B, n_q, Hq, d))
    ref, ref_lse = oracle.decode(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                                 q, k_hist, None if layer.k_eq_v else v_hist, cache_lens)
    max_len = max(cache_lens)
    # the oracle always gets the un-rotated history; the GPU cache may hold rotated keys
    k_cache_src = [_rotated_history(k_hist[b], cache_lens[b], layer) for b in range(B)] if keys_rotated else k_hist
    if layout == G.CACHE_RING:
        cap = layer.window
        kc = np.stack([ring_from_history(k_cache_src[b][:cache_lens[b]], cap) for b in range(B)])
        vc = None if layer.k_eq_v else np.stack([ring_from_history(v_hist[b][:cache_lens[b]], cap) for b in range(B)])
    else:
        cap = max(max_len, 1) + (200 if junk else 0)
        kc = np.zeros((B, Hkv, cap, d), np.uint16)
        vc = None if layer.k_eq_v else np.zeros((B, Hkv, cap, d), np.uint16)
        if junk:  # rows past each sequence's cached tokens hold NaNs: the kernels must not read them
            kc[:] = 0x7FC0
            if vc is not None:
                vc[:] = 0x7FC0
        for b, n in enumerate(cache_lens):
            kc[b, :, :n] = k_cache_src[b][:n].transpose(1, 0, 2)
            if vc is not None:
                vc[b, :, :n] = v_hist[b][:n].transpose(1, 0, 2)
    new_k = np.stack([k_hist[b][cache_lens[b]:] for b in range(B)])
    new_v = None if layer.k_eq_v else np.stack([v_hist[b][cache_lens[b]:] for b in range(B)])
    p = G.params(layer.kind, Hq, Hkv, d, window=layer.window, rope_p=layer.rope_p, rope_base=layer.rope_base,
                 softmax_scale=layer.softmax_scale)
    if num_splits is None:
        num_splits = G.gemma_attn_decode_num_splits(p, B, n_q, max_len)
    rows = B * n_q * Hq
    po = torch.empty((num_splits, rows, d), dtype=torch.float32, device="cuda")
    pl = torch.empty((num_splits, rows), dtype=torch.float32, device="cuda")
    G.gemma_attn_decode(p, dev_bf16(q), dev_bf16(new_k), None if new_v is None else dev_bf16(new_v), dev_bf16(kc),
                        None if vc is None else dev_bf16(vc), layout | (G.CACHE_KEYS_ROTATED if keys_rotated else 0),
                        cap, dev_i32(cache_lens), B, n_q, max_len, po, pl, num_splits)
    out = torch.empty((B, n_q, Hq, d), dtype=torch.float32, device="cuda")
    out16 = torch.empty((B, n_q, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    G.gemma_attn_combine(po, pl, num_splits, rows, d, G.OUT_F32, out, lse)
    G.gemma_attn_combine(po, pl, num_splits, rows, d, G.OUT_BF16, out16, None)
    G.gemma_attn_check()
    got = out.cpu().numpy()
    np.testing.assert_array_equal(W.bf16_bits_to_f32(host_bits(out16)), bf16_round(got))
    assert_close(got, ref, f"decode {layer} lens={cache_lens} n_q={n_q} splits={num_splits}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=1e-2, rtol=0)


LOC = W.LayerSpec(W.LOCAL, 8, 4, 256, window=64, rope_p=1.0, rope_base=1e4)
GLO = W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.25, rope_base=1e6)


@pytest.mark.parametrize("cache_lens,n_q,splits", [
    ((0, 5, 63, 64, 200), 1, None),
    ((1000, 130), 1, 3),
    ((77, 300), 4, 1),
    ((77, 300), 4, 5),
])
def test_decode_local_ring(cache_lens, n_q, splits):
    _check_decode(LOC, cache_lens, n_q, G.CACHE_RING, splits)


@pytest.mark.parametrize("cache_lens,n_q,splits,layout", [
    ((0, 5, 63, 64, 200), 1, None, G.CACHE_RING),       # warp kernel, split key / value stages
    ((77, 300), 4, 3, G.CACHE_RING),                    # 8 rows per KV head
    ((40, 150), 8, 2, G.CACHE_CONTIGUOUS),              # 16 rows: the CTA-wide kernel
])
def test_decode_local_prerotated_keys(cache_lens, n_q, splits, layout):
    _check_decode(LOC, cache_lens, n_q, layout, splits, keys_rotated=True)


def test_decode_local_contiguous():
    _check_decode(LOC, (10, 250), 2, G.CACHE_CONTIGUOUS, 4)


@pytest.mark.parametrize("cache_lens,n_q,splits", [
    ((0, 1, 300), 1, None),
    ((2000, 513), 1, 7),
    ((150, 400), 4, 3),
])
def test_decode_global(cache_lens, n_q, splits):
    _check_decode(GLO, cache_lens, n_q, G.CACHE_CONTIGUOUS, splits)


def test_decode_global_gqa8():
    _check_decode(W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (1500,), 1, G.CACHE_CONTIGUOUS)


@pytest.mark.parametrize("kind,hq,hkv,d,p,n_q", [
    (W.GLOBAL, 4, 1, 32, 1.0, 1),     # r = 16: every k-step rotated
    (W.GLOBAL, 2, 1, 64, 0.5, 3),     # r = 16
    (W.GLOBAL, 8, 2, 128, 0.3, 1),    # r = 19: odd, rotated k-steps partly pass-through
    (W.GLOBAL, 4, 1, 256, 0.1, 2),    # r = 12
    (W.LOCAL, 4, 2, 32, 1.0, 2),
    (W.LOCAL, 8, 4, 64, 0.75, 4),     # r = 24
    (W.LOCAL, 2, 2, 128, 0.3, 1),     # r = 19
    (W.LOCAL, 8, 1, 512, 1.0, 1),     # separate-V d = 512: one ring stage per warp
    # up to 2 rows per KV head
    (W.GLOBAL, 2, 1, 512, 0.25, 1),   # K=V, rotated k-steps read from the rotated copy
    (W.GLOBAL, 1, 1, 128, 0.3, 1),    # one row, r = 19
    (W.GLOBAL, 2, 1, 256, 1.0, 1),    # every k-step rotated
    (W.LOCAL, 2, 1, 512, 1.0, 1),     # separate-V d = 512
    (W.LOCAL, 1, 1, 256, 0.5, 2),     # 2 rows from 2 new tokens of one head
])
def test_decode_head_dims_and_partial_rotation(kind, hq, hkv, d, p, n_q):
    window = 48 if kind == W.LOCAL else 0
    layer = W.LayerSpec(kind, hq, hkv, d, window=window, rope_p=p, rope_base=1e4)
    layout = G.CACHE_RING if kind == W.LOCAL else G.CACHE_CONTIGUOUS
    _check_decode(layer, (0, 37, 130), n_q, layout, 3)


def test_combine_against_oracle():
    rng = np.random.default_rng(9)
    S, R, d = 5, 37, 64
    po = rng.standard_normal((S, R, d)).astype(np.float32)
    pl = (rng.standard_normal((S, R)) * 3).astype(np.float32)
    pl[1, :5] = -np.inf
    pl[:, 7] = -np.inf  # a row with every split empty
    ref, ref_lse = oracle.combine(po.astype(np.float64), pl.astype(np.float64))
    out = torch.empty((R, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((R,), dtype=torch.float32, device="cuda")
    G.gemma_attn_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(), S, R, d, G.OUT_F32, out, lse)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert_close(got, ref, "combine")
    got_lse = lse.cpu().numpy()
    assert got_lse[7] == -np.inf
    np.testing.assert_allclose(got_lse[np.isfinite(ref_lse)], ref_lse[np.isfinite(ref_lse)], atol=1e-5)


@pytest.mark.parametrize("S,R,d", [(5, 37, 64), (18, 2048, 512), (3, 2100, 36), (2, 4096, 32)])
@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_combine_vector_and_element_forms_agree(S, R, d, out_dtype):
    # 16-byte aligned buffers with at least 2048 warps of work (rows x ceil(d / 128)) take
    # the vectorized kernel (a warp per 128 columns of a row); buffers one element off, or
    # fewer rows, take the per-element kernel. Both merge in split order, so the outputs
    # are identical bit for bit, and both match the oracle.
    rng = np.random.default_rng(S * 1000 + R)
    po = rng.standard_normal((S, R, d)).astype(np.float32)
    pl = (rng.standard_normal((S, R)) * 3).astype(np.float32)
    pl[S - 1, : R // 2] = -np.inf
    pl[:, R // 3] = -np.inf
    f32 = out_dtype == "f32"
    flag = G.OUT_F32 if f32 else G.OUT_BF16
    tdt = torch.float32 if f32 else torch.bfloat16
    pl_d = torch.from_numpy(pl).cuda()
    outs = []
    for off in (0, 1):
        po_buf = torch.empty(S * R * d + 1, dtype=torch.float32, device="cuda")
        po_buf[off:off + S * R * d] = torch.from_numpy(po.reshape(-1)).cuda()
        out_buf = torch.full((R * d + 1,), 7.0, dtype=tdt, device="cuda")
        lse = torch.empty((R,), dtype=torch.float32, device="cuda")
        G.gemma_attn_combine(po_buf[off:], pl_d, S, R, d, flag, out_buf[off:], lse)
        torch.cuda.synchronize()
        outs.append((out_buf[off:off + R * d].float().cpu().numpy().reshape(R, d), lse.cpu().numpy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    ref, _ = oracle.combine(po.astype(np.float64), pl.astype(np.float64))
    if f32:
        assert_close(outs[0][0], ref, "combine vector form")


def test_prefill_divergent_rescale_within_warp():
    """One key with a huge score: rows at or after it raise their running max by far more
    than 2^8 mid-sequence, rows before it do not, so lanes of one warp disagree."""
    T, d = 400, 64
    layer = W.LayerSpec(W.GLOBAL, 2, 1, d, rope_p=0.0, rope_base=1e4)
    rng = np.random.default_rng(31)
    qf = np.zeros((T, 2, d), np.float32)
    qf[:, :, 0] = 4.0
    kf = (rng.standard_normal((T, 1, d)) * 0.1).astype(np.float32)
    kf[300, 0, 0] = 40.0
    q = W.f32_to_bf16_bits(qf)
    k = W.f32_to_bf16_bits(kf)
    pos = np.arange(T, dtype=np.int32)
    cu = np.array([0, T], np.int32)
    out, lse = run_prefill(G, layer, q, k, None, pos, cu, out_f32=True)
    ref, ref_lse = oracle.attention(layer.kind, 0, 0.0, 1e4, layer.softmax_scale, q, k, None, pos, cu)
    assert_close(out.cpu().numpy(), ref, "divergent rescale")
    np.testing.assert_allclose(lse.cpu().numpy().T, ref_lse, atol=1e-2, rtol=0)


# 9-32 query rows per KV head of a global layer (the speculative verify of 4 draft tokens
# with 8 query heads per KV head is 32): the tcgen05 kernel (keys on M, rows on N), and with
# GEMMA_ATTN_DECODE_MMA_SYNC=1 the mma.sync kernel, against the oracle. Cache rows past each
# sequence's tokens hold NaNs; lengths straddle the 128-key tiles.
GLO8 = W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)


@pytest.mark.parametrize("mma_sync", [False, True])
@pytest.mark.parametrize("layer,cache_lens,n_q,splits", [
    (GLO8, (0, 1, 127, 128, 129, 1000), 4, None),
    (GLO8, (255, 256, 3000), 4, 3),
    (GLO8, (700, 40), 2, 1),
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.0, rope_base=1e6), (300, 129), 3, 2),
    (W.LayerSpec(W.GLOBAL, 8, 1, 256, rope_p=0.25, rope_base=1e4), (500, 64), 4, 2),
    (W.LayerSpec(W.GLOBAL, 4, 1, 512, rope_p=0.125, rope_base=1e6), (333,), 3, 1),
])
def test_decode_verify_rows_kernels(layer, cache_lens, n_q, splits, mma_sync, monkeypatch):
    if mma_sync:
        monkeypatch.setenv("GEMMA_ATTN_DECODE_MMA_SYNC", "1")
    _check_decode(layer, cache_lens, n_q, G.CACHE_CONTIGUOUS, splits, seed=13, junk=True)


@pytest.mark.parametrize("batch,splits", [(40, 5), (2060, 2)])
def test_verify_work_items_over_ragged_batches(batch, splits):
    """The tcgen05 verify kernel's work items (equal tile counts per split, longest sequence
    first, unused splits left at -inf): a ragged batch with empty, one-tile and multi-tile
    sequences, and a batch past the 2048 sequences the kernel ranks by length (those keep
    their index order)."""
    rng = np.random.default_rng(batch)
    lens = rng.integers(0, 130, batch)
    lens[:3] = (0, 1, 129)
    if batch < 100:
        lens[3:6] = (1500, 700, 2000)
    _check_decode(GLO8, tuple(int(n) for n in lens), 4, G.CACHE_CONTIGUOUS, splits, seed=17, junk=batch < 100)
