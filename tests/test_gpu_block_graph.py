"""Interleaved block runner: the block's calls replayed from a CUDA graph equal the same
calls launched eagerly, bit for bit, and a replay after new inputs are written into the
block's tensors equals an eager run on those inputs. One layer is also checked against
the oracle, so that the block wiring (positions, cu_seqlens, K=V) is the tested one."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from global_interleaved_layers_b200.block import BlockLayer, InterleavedBlock  # noqa: E402
from gpu_util import assert_close, dev_bf16, dev_i32  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


SPECS = [
    W.LayerSpec(W.LOCAL, 4, 2, 128, window=64, rope_p=1.0, rope_base=1e4),
    W.LayerSpec(W.LOCAL, 4, 2, 128, window=64, rope_p=1.0, rope_base=1e4),
    W.LayerSpec(W.GLOBAL, 8, 1, 256, rope_p=0.25, rope_base=1e6),
]
LENS = (170, 300)


def _layer(spec, seed):
    T = sum(LENS)
    cu = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in LENS]).astype(np.int32)
    q = dev_bf16(W.normal_bf16(seed, 0, (T, spec.num_q_heads, spec.head_dim)))
    k = dev_bf16(W.normal_bf16(seed, 1, (T, spec.num_kv_heads, spec.head_dim)))
    v = None if spec.k_eq_v else dev_bf16(W.normal_bf16(seed, 2, (T, spec.num_kv_heads, spec.head_dim)))
    # the global layer writes fp32 (checked against the oracle below: bf16 output rounding
    # alone would reach 1.6e-2 at |o| >= 4); the local layers write bf16
    f32 = spec.kind == W.GLOBAL
    p = G.params(spec.kind, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, window=spec.window,
                 rope_p=spec.rope_p, rope_base=spec.rope_base, softmax_scale=spec.softmax_scale,
                 out_dtype=G.OUT_F32 if f32 else G.OUT_BF16)
    out = torch.zeros((T, spec.num_q_heads, spec.head_dim), dtype=torch.float32 if f32 else torch.bfloat16,
                      device="cuda")
    lse = torch.zeros((spec.num_q_heads, T), dtype=torch.float32, device="cuda")
    return BlockLayer(p, q, k, v, out, lse, dev_i32(pos), dev_i32(cu), len(LENS), T, max(LENS))


def _outputs(block):
    return [(ly.out.clone(), ly.lse.clone()) for ly in block.layers]


def test_graph_replay_equals_eager_and_follows_new_inputs():
    block = InterleavedBlock([_layer(s, 40 + i) for i, s in enumerate(SPECS)])
    block.run()
    G.gemma_attn_check()
    eager = _outputs(block)
    block.capture()
    for ly in block.layers:
        ly.out.zero_()
        ly.lse.zero_()
    block.replay()
    G.gemma_attn_check()
    for (o, l), ly in zip(eager, block.layers):
        assert torch.equal(ly.out, o) and torch.equal(ly.lse, l)
    # new inputs into the same tensors: the replay computes on them
    for i, ly in enumerate(block.layers):
        spec = SPECS[i]
        ly.q.copy_(dev_bf16(W.normal_bf16(90 + i, 0, tuple(ly.q.shape))))
        ly.k.copy_(dev_bf16(W.normal_bf16(90 + i, 1, tuple(ly.k.shape))))
        if ly.v is not None:
            ly.v.copy_(dev_bf16(W.normal_bf16(90 + i, 2, tuple(ly.v.shape))))
        assert spec.k_eq_v == (ly.v is None)
    block.replay()
    G.gemma_attn_check()
    replayed = _outputs(block)
    block.run()
    G.gemma_attn_check()
    for (o, l), ly in zip(replayed, block.layers):
        assert torch.equal(ly.out, o) and torch.equal(ly.lse, l)
    # the global layer against the oracle on the new inputs
    spec, ly = SPECS[2], block.layers[2]
    qh = ly.q.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    kh = ly.k.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    pos = np.concatenate([np.arange(n) for n in LENS]).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    ref, _ = oracle.attention(spec.kind, spec.window, spec.rope_p, spec.rope_base, spec.softmax_scale, qh, kh, None,
                              pos, cu)
    assert_close(ly.out.cpu().numpy(), ref, "global layer of the replayed block")
