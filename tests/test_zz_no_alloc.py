"""The allocation-free decode entry point against the regular decode + combine path.

gemma_attn_decode_noalloc is for callers that cannot allocate device memory (an op
inside a framework that owns all device allocations, or a caller capturing a CUDA
graph): it keeps the split partials in a static device array inside the library
instead of caller-provided buffers. These checks call it through the C-ABI twice in a
row, on different inputs so that stale contents of the shared array would show, and
compare each result with gemma_attn_decode + gemma_attn_combine on the same inputs
within the bounds the parity tests use. The file runs last (its name sorts last) and
also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import assert_close, dev_bf16, dev_i32  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _inputs(layer, cache_lens, n_q, seed, ring):
    B = len(cache_lens)
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    cap = layer.window if ring else max(cache_lens)
    q = dev_bf16(W.normal_bf16(seed, 0, (B, n_q, Hq, d)))
    nk = dev_bf16(W.normal_bf16(seed, 1, (B, n_q, Hkv, d)))
    nv = None if layer.k_eq_v else dev_bf16(W.normal_bf16(seed, 2, (B, n_q, Hkv, d)))
    kc = dev_bf16(W.normal_bf16(seed, 3, (B, Hkv, cap, d)))
    vc = None if layer.k_eq_v else dev_bf16(W.normal_bf16(seed, 4, (B, Hkv, cap, d)))
    return q, nk, nv, kc, vc, cap


@pytest.mark.parametrize("layer,cache_lens,n_q,ring,splits", [
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.25, rope_base=1e6), (300, 1000), 2, False, 4),
    (W.LayerSpec(W.LOCAL, 8, 4, 256, window=128, rope_p=1.0, rope_base=1e4), (50, 700), 1, True, 3),
])
def test_noalloc_decode_matches_regular_path_twice(layer, cache_lens, n_q, ring, splits):
    B = len(cache_lens)
    Hq, d = layer.num_q_heads, layer.head_dim
    rows = B * n_q * Hq
    layout = G.CACHE_RING if ring else G.CACHE_CONTIGUOUS
    p = G.params(layer.kind, Hq, layer.num_kv_heads, d, window=layer.window, rope_p=layer.rope_p,
                 rope_base=layer.rope_base, softmax_scale=layer.softmax_scale, out_dtype=G.OUT_F32)
    max_len = max(cache_lens)
    lens = dev_i32(cache_lens)
    for call, seed in enumerate((41, 42)):  # two calls in a row, different inputs
        q, nk, nv, kc, vc, cap = _inputs(layer, cache_lens, n_q, seed, ring)
        # regular path: caller-provided partials, then the combine
        po = torch.empty((splits, rows, d), dtype=torch.float32, device="cuda")
        pl = torch.empty((splits, rows), dtype=torch.float32, device="cuda")
        G.gemma_attn_decode(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, max_len, po, pl, splits)
        ref = torch.empty((B, n_q, Hq, d), dtype=torch.float32, device="cuda")
        ref_lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
        G.gemma_attn_combine(po, pl, splits, rows, d, G.OUT_F32, ref, ref_lse)
        # allocation-free path
        out = torch.empty((B, n_q, Hq, d), dtype=torch.float32, device="cuda")
        lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
        G.gemma_attn_decode_noalloc(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, max_len, splits, out, lse)
        assert G.gemma_attn_last_launch_count() == 2  # the decode kernel, then the combine
        G.gemma_attn_check()
        assert_close(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), f"noalloc call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=1e-2, rtol=0)


def test_noalloc_rejects_requests_beyond_the_static_buffer():
    layer = W.LayerSpec(W.GLOBAL, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    p = G.params(layer.kind, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    B, n_q = 16, 4
    rows = B * n_q * 32
    splits = G.NOALLOC_SCRATCH_BYTES // (rows * 513 * 4) + 1   # one split more than fits
    fake = 1 << 20  # never dereferenced: the size check fails first
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode_noalloc(p, fake, fake, None, fake, None, G.CACHE_CONTIGUOUS, 1000, fake, B, n_q, 1000,
                                    splits, fake, None)
    assert e.value.status == G.ERR_WORKSPACE


@pytest.mark.parametrize("layer,cache_lens,n_q,ring,out_dtype", [
    # 8 rows per KV head and 2 new tokens: 16 rows, the tensor-core split kernel
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.25, rope_base=1e6), (300, 1000), 2, False, "f32"),
    # 2 rows per KV head: the warp-split kernel, bf16 output, keys stored rotated
    (W.LayerSpec(W.LOCAL, 8, 4, 256, window=128, rope_p=1.0, rope_base=1e4), (50, 700), 1, True, "bf16"),
    (W.LayerSpec(W.LOCAL, 8, 4, 256, window=128, rope_p=1.0, rope_base=1e4), (0, 129), 1, True, "f32"),
])
def test_noalloc_single_split_writes_the_combined_result_directly(layer, cache_lens, n_q, ring, out_dtype):
    """One split: the decode kernel writes out and lse itself, bit for bit what the combine
    of its single partial writes (exp(0) = 1 weights, division by 1)."""
    B = len(cache_lens)
    Hq, d = layer.num_q_heads, layer.head_dim
    rows = B * n_q * Hq
    layout = (G.CACHE_RING | G.CACHE_KEYS_ROTATED) if ring else G.CACHE_CONTIGUOUS
    od = G.OUT_F32 if out_dtype == "f32" else G.OUT_BF16
    tdt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    p = G.params(layer.kind, Hq, layer.num_kv_heads, d, window=layer.window, rope_p=layer.rope_p,
                 rope_base=layer.rope_base, softmax_scale=layer.softmax_scale, out_dtype=od)
    max_len = max(cache_lens)
    lens = dev_i32(cache_lens)
    q, nk, nv, kc, vc, cap = _inputs(layer, cache_lens, n_q, 43, ring)
    po = torch.empty((1, rows, d), dtype=torch.float32, device="cuda")
    pl = torch.empty((1, rows), dtype=torch.float32, device="cuda")
    G.gemma_attn_decode(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, max_len, po, pl, 1)
    ref = torch.empty((B, n_q, Hq, d), dtype=tdt, device="cuda")
    ref_lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    G.gemma_attn_combine(po, pl, 1, rows, d, od, ref, ref_lse)
    out = torch.full((B, n_q, Hq, d), float("nan"), dtype=tdt, device="cuda")
    lse = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    G.gemma_attn_decode_noalloc(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, max_len, 1, out, lse)
    assert G.gemma_attn_last_launch_count() == 1  # the decode kernel alone
    out_nolse = torch.full_like(out, float("nan"))
    G.gemma_attn_decode_noalloc(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, max_len, 1, out_nolse, None)
    G.gemma_attn_check()
    assert torch.equal(out, ref)
    assert torch.equal(out_nolse, ref)
    assert torch.equal(lse, ref_lse)
