"""The vision encoder's attention (bidirectional, 2D RoPE) through the C-ABI against the
oracle: every patch of an image sees every patch of it and nothing of the other images;
q and k are rotated for the patch's (h, w) by the 2D rule. Ragged images with partial
last tiles, head dims 64 to 512, the paired (two query heads per KV head) and unpaired
kernels; patch order and coordinates arbitrary."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import assert_close, run_prefill  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _grid(n, width, h0=0, w0=0):
    idx = np.arange(n)
    return np.stack([h0 + idx // width, w0 + idx % width], axis=1).astype(np.int32)


@pytest.mark.parametrize("hq,hkv,d,lens,widths", [
    (4, 4, 64, (300, 45), (20, 9)),          # one query head per KV head: unpaired kernel
    (8, 4, 128, (129, 256, 7), (16, 16, 7)),  # paired kernel, a 1-row last tile and a 7-patch image
    (4, 2, 256, (200,), (14,)),
    (2, 1, 512, (130, 64), (13, 8)),          # two output halves per query tile
])
def test_bidir_prefill_matches_oracle(hq, hkv, d, lens, widths):
    layer = W.LayerSpec(W.BIDIR, hq, hkv, d, rope_p=1.0, rope_base=1e4)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    hw = np.concatenate([_grid(n, w, 3 * s, s) for s, (n, w) in enumerate(zip(lens, widths))])
    q = W.normal_bf16(60, 0, (T, hq, d))
    k = W.normal_bf16(60, 1, (T, hkv, d))
    v = W.normal_bf16(60, 2, (T, hkv, d))
    out, lse = run_prefill(G, layer, q, k, v, hw, cu, out_f32=True)
    ref, ref_lse = oracle.attention_2d(layer.rope_base, layer.softmax_scale, q, k, v, hw, cu)
    assert_close(out.cpu().numpy(), ref, f"bidir {hq}/{hkv} d={d} lens={lens}")
    np.testing.assert_allclose(lse.cpu().numpy().T, ref_lse, atol=1e-2, rtol=0)


def test_bidir_patch_order_and_coordinates_are_free():
    """Shuffled patches with scattered coordinates (a sparse, pooled layout): still the oracle."""
    hq, hkv, d = 4, 2, 128
    lens = (180, 77)
    T = sum(lens)
    cu = np.array([0, lens[0], T], np.int32)
    rng = np.random.default_rng(8)
    hw = rng.integers(0, 500, size=(T, 2)).astype(np.int32)
    q = W.normal_bf16(61, 0, (T, hq, d))
    k = W.normal_bf16(61, 1, (T, hkv, d))
    v = W.normal_bf16(61, 2, (T, hkv, d))
    layer = W.LayerSpec(W.BIDIR, hq, hkv, d, rope_p=1.0, rope_base=1e4)
    out, _ = run_prefill(G, layer, q, k, v, hw, cu, out_f32=True)
    ref, _ = oracle.attention_2d(1e4, 1 / math.sqrt(d), q, k, v, hw, cu)
    assert_close(out.cpu().numpy(), ref, "bidir shuffled")


def test_bidir_at_the_benchmark_shape_sampled_rows():
    """4 images x 2520 patches, 12 heads of 64 dims (the measured vision batch): sampled
    rows of every image against the oracle."""
    wl = W.vision_batch()
    layer = wl.layers[0]
    T = wl.total_tokens
    cu = wl.cu_seqlens()
    idx = np.concatenate([np.arange(n) for n in wl.seq_lens])
    hw = np.stack([idx // 56, idx % 56], axis=1).astype(np.int32)
    q = W.normal_bf16(62, 0, (T, layer.num_q_heads, layer.head_dim))
    k = W.normal_bf16(62, 1, (T, layer.num_kv_heads, layer.head_dim))
    v = W.normal_bf16(62, 2, (T, layer.num_kv_heads, layer.head_dim))
    out, lse = run_prefill(G, layer, q, k, v, hw, cu, out_f32=True)
    rng = np.random.default_rng(3)
    rows = np.sort(np.concatenate([cu[s] + np.concatenate([[0, n - 1], rng.integers(0, n, 14)])
                                   for s, n in enumerate(wl.seq_lens)])).astype(np.int32)
    ref, ref_lse = oracle.attention_2d(layer.rope_base, layer.softmax_scale, q, k, v, hw, cu, rows=rows)
    assert_close(out.cpu().numpy()[rows], ref, "vision batch, sampled rows")
    np.testing.assert_allclose(lse.cpu().numpy().T[rows], ref_lse, atol=1e-2, rtol=0)
