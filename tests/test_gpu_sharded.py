"""Key-range shards of a global-layer history through gemma_attn_decode_shard, on one GPU.

A history spread over W GPUs is decoded rank by rank here, one shard after another on the
same GPU (no kernel waits on another): each shard's partials come from the library's
decode kernels with the queries placed after the later shards' tokens and the new tokens
among the keys of the last shard only; the stacked partials go through gemma_attn_combine
and must match the oracle's attention over the whole history. Cache rows past each
shard's tokens hold NaNs. Shapes cover the warp kernel (8 query rows per KV head) and the
tcgen05 verify kernel (16-32 rows). ShardedDecode with a single rank is checked on the same
inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from global_interleaved_layers_b200.sharded import ShardedDecode, query_offsets  # noqa: E402
from gpu_util import assert_close, dev_bf16, dev_i32  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _case(layer, lengths, n_q, world, splits, seed):
    B = len(lengths)
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    hist = [W.normal_bf16(seed + b, 1, (n + n_q, Hkv, d)) for b, n in enumerate(lengths)]
    qn = W.normal_bf16(seed, 0, (B, n_q, Hq, d))
    ref, ref_lse = oracle.decode(layer.kind, 0, layer.rope_p, layer.rope_base, layer.softmax_scale, qn, hist, None,
                                 list(lengths))
    p = G.params(layer.kind, Hq, Hkv, d, rope_p=layer.rope_p, rope_base=layer.rope_base,
                 softmax_scale=layer.softmax_scale, out_dtype=G.OUT_F32)
    rows = B * n_q * Hq
    new_k = dev_bf16(np.stack([hist[b][n:] for b, n in enumerate(lengths)]))
    return hist, qn, ref, ref_lse, p, rows, new_k


@pytest.mark.parametrize("layer,lengths,n_q,world,splits", [
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (5000, 300, 1), 1, 2, 2),    # warp kernel
    (W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6), (5000, 300, 1), 4, 3, 1),    # tcgen05 kernel
    (W.LayerSpec(W.GLOBAL, 16, 2, 512, rope_p=0.25, rope_base=1e6), (2000, 129), 2, 4, 2),      # 16 rows
    (W.LayerSpec(W.GLOBAL, 8, 1, 256, rope_p=0.25, rope_base=1e4), (700, 64), 3, 2, 1),         # head dim 256
])
def test_shards_combined_equal_the_whole_history(layer, lengths, n_q, world, splits):
    B = len(lengths)
    Hkv, d = layer.num_kv_heads, layer.head_dim
    hist, qn, ref, ref_lse, p, rows, new_k = _case(layer, lengths, n_q, world, splits, seed=90)
    po_all, pl_all = [], []
    for rank in range(world):
        offs = query_offsets(lengths, world, rank)
        cap = max(max(o[1] for o in offs), 1) + 100
        kc = np.full((B, Hkv, cap, d), 0x7FC0, np.uint16)  # NaN past each shard's tokens
        for b, (lo, ln, _) in enumerate(offs):
            kc[b, :, :ln] = hist[b][lo:lo + ln].transpose(1, 0, 2)
        po = torch.empty((splits, rows, d), dtype=torch.float32, device="cuda")
        pl = torch.empty((splits, rows), dtype=torch.float32, device="cuda")
        last = rank == world - 1
        G.gemma_attn_decode_shard(p, dev_bf16(qn), new_k if last else None, dev_bf16(kc), cap,
                                  dev_i32([o[1] for o in offs]), dev_i32([o[2] for o in offs]), last, B, n_q,
                                  max(o[1] for o in offs), po, pl, splits)
        po_all.append(po)
        pl_all.append(pl)
    po_all = torch.cat(po_all)
    pl_all = torch.cat(pl_all)
    out = torch.empty((B, n_q, layer.num_q_heads, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    G.gemma_attn_combine(po_all, pl_all, world * splits, rows, d, G.OUT_F32, out, lse)
    G.gemma_attn_check()
    assert_close(out.cpu().numpy(), ref, f"{world} shards {layer} lens={lengths} n_q={n_q}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(ref_lse.shape), ref_lse, atol=1e-2, rtol=0)


def test_single_rank_sharded_decode_is_the_plain_decode():
    layer = W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
    lengths, n_q = (3000, 17), 4
    B, Hkv, d = len(lengths), layer.num_kv_heads, layer.head_dim
    hist, qn, ref, ref_lse, p, rows, new_k = _case(layer, lengths, n_q, 1, 2, seed=95)
    cap = max(lengths)
    kc = np.zeros((B, Hkv, cap, d), np.uint16)
    for b, n in enumerate(lengths):
        kc[b, :, :n] = hist[b][:n].transpose(1, 0, 2)
    dec = ShardedDecode(p, B, n_q, 2, "cuda", out_dtype=G.OUT_F32)
    assert dec.world == 1 and dec.holds_end
    out = torch.empty((B, n_q, layer.num_q_heads, d), dtype=torch.float32, device="cuda")
    dec(dev_bf16(qn), new_k, dev_bf16(kc), cap, dev_i32(lengths), dev_i32([0] * B), cap, out)
    G.gemma_attn_check()
    assert_close(out.cpu().numpy(), ref, "single-rank sharded decode")
