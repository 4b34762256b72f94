"""Launches with more CTAs than SMs (several waves per SM), at small per-CTA work.

Every CTA of a wave must release its tensor memory so the next wave's CTA on that SM
can allocate; these shapes exercise that hand-over for each head-dim variant."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import assert_close, run_prefill  # noqa: E402


@pytest.mark.parametrize("layer,lens", [
    (W.LayerSpec(W.LOCAL, 16, 8, 64, window=64, rope_p=1.0, rope_base=1e4), (4096,)),      # 512 CTAs
    (W.LayerSpec(W.LOCAL, 8, 4, 256, window=128, rope_p=1.0, rope_base=1e4), (3000,)),     # 192 CTAs
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (1300,)),               # 176 CTAs
])
def test_multi_wave_prefill(layer, lens):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T = sum(lens)
    q, k, v = W.layer_inputs(layer, T, 21)
    cu = np.array([0, T], np.int32)
    pos = np.arange(T, dtype=np.int32)
    out, _ = run_prefill(G, layer, q, k, v, pos, cu, out_f32=True)
    rows = np.concatenate([np.arange(0, T, 97), [T - 1]]).astype(np.int32)
    ref, _ = oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                              q, k, v, pos, cu, rows=rows)
    assert_close(out.cpu().numpy()[rows], ref, f"multi-wave {layer}")


@pytest.mark.parametrize("layer,lens", [
    # many short sequences: most units have one or two key tiles
    (W.LayerSpec(W.LOCAL, 16, 8, 128, window=16, rope_p=1.0, rope_base=1e4),
     tuple(int(n) for n in np.random.default_rng(5).integers(1, 300, 60))),
    (W.LayerSpec(W.LOCAL, 8, 4, 256, window=256, rope_p=1.0, rope_base=1e4), (5000, 77, 1, 640, 129, 2000)),
    (W.LayerSpec(W.GLOBAL, 16, 2, 128, rope_p=0.25, rope_base=1e6), (3000, 1, 130, 900)),
    (W.LayerSpec(W.GLOBAL, 12, 12, 64, rope_p=0.25, rope_base=1e4), (2500, 64, 700)),          # single-CTA form
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (900, 1, 300, 129)),
])
def test_many_units_per_cta(layer, lens):
    """Persistent CTAs walking many work units back to back (units of one key tile
    included): the query tiles of consecutive units share the tile stream, so every unit
    boundary is checked against the oracle on sampled rows of every sequence."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T = sum(lens)
    q, k, v = W.layer_inputs(layer, T, 23)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    out, _ = run_prefill(G, layer, q, k, v, pos, cu, out_f32=True)
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([cu[s] + np.concatenate([[0, n - 1], rng.integers(0, n, 6)])
                                     for s, n in enumerate(lens)])).astype(np.int32)
    ref, _ = oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                              q, k, v, pos, cu, rows=rows)
    assert_close(out.cpu().numpy()[rows], ref, f"many units {layer} lens={lens[:8]}")
