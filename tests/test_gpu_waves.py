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
