"""GPU parity at the full workload sizes, in the launch configuration the bench times.

Each case compares sampled outputs with the fp64 oracle. Device tensors are first
filled with device-side random data, then the slices that the sampled outputs depend on
(the sampled query rows, and every key/value row of the KV head they read) are
overwritten with seeded host data that the oracle also receives. The sampled outputs
therefore depend only on oracle-visible inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

G = pytest.importorskip("global_interleaved_layers_b200")
from gpu_util import assert_close, dev_bf16, dev_i32, run_prefill  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _rows_sample(lens, per_seq_first=32, per_seq_last=32, n_rand=32, seed=1):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)])
    rows = []
    for s, n in enumerate(lens):
        r = set(range(min(per_seq_first, n))) | set(range(max(0, n - per_seq_last), n))
        r |= set(int(x) for x in rng.integers(0, n, size=n_rand))
        rows.extend(int(cu[s]) + x for x in sorted(r))
    return np.array(rows, dtype=np.int32)


def _prefill_case(layer: W.LayerSpec, lens, seed, q_heads_checked=None, rows=None):
    """Run the full-size layer; check query heads of KV head 0 on sampled rows."""
    lens = tuple(int(x) for x in lens)
    T = sum(lens)
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    group = Hq // Hkv
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    if rows is None:
        rows = _rows_sample(lens)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    q = torch.randn((T, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    k = torch.randn((T, Hkv, d), generator=gen, device="cuda").to(torch.bfloat16)
    v = None if layer.k_eq_v else torch.randn((T, Hkv, d), generator=gen, device="cuda").to(torch.bfloat16)
    # oracle-visible slices: the sampled rows of query heads 0..group-1 and all rows of KV head 0
    q_rows = W.normal_bf16(seed, 0, (rows.shape[0], group, d))
    k0 = W.normal_bf16(seed, 1, (T, 1, d))
    v0 = None if layer.k_eq_v else W.normal_bf16(seed, 2, (T, 1, d))
    q[torch.from_numpy(rows.astype(np.int64)).cuda(), 0:group] = dev_bf16(q_rows)
    k[:, 0:1] = dev_bf16(k0)
    if v is not None:
        v[:, 0:1] = dev_bf16(v0)
    out, lse = run_prefill(G, layer, q, k, v, pos, cu, out_f32=True)
    got = out[torch.from_numpy(rows.astype(np.int64)).cuda(), 0:group].cpu().numpy()
    del q, k, v, out
    torch.cuda.empty_cache()
    # oracle on the same values: a one-KV-head problem with `group` query heads
    qo = np.zeros((T, group, d), np.uint16)
    qo[rows] = q_rows
    ref, _ = oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                              qo, k0, v0, pos, cu, rows=rows)
    return assert_close(got, ref, f"full-size prefill {layer} T={T}")


def test_e2b_block_layers():
    wl = W.e2b_block()
    for li in (0, 4):  # the local and the global layer shapes of the block
        _prefill_case(wl.layers[li], wl.seq_lens, seed=100 + li)


def test_31b_block_global_layer():
    wl = W.b31_block()
    rows = _rows_sample(wl.seq_lens, 16, 16, 16)
    _prefill_case(wl.layers[-1], wl.seq_lens, seed=200, rows=rows)


def test_31b_block_global_layer_every_query_head():
    """Sampled rows of all 32 query heads (every KV head's group), not only KV head 0's."""
    layer = W.b31_block().layers[-1]
    T = 32768
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    rows = np.array(sorted({0, 1, 127, 128, 4095, 16384, 32766, 32767} |
                           set(int(x) for x in np.random.default_rng(2).integers(0, T, 4))), np.int32)
    cu = np.array([0, T], np.int32)
    pos = np.arange(T, dtype=np.int32)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(210)
    q = torch.randn((T, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    k_host = W.normal_bf16(210, 1, (T, Hkv, d))
    q_rows = W.normal_bf16(210, 0, (rows.shape[0], Hq, d))
    ridx = torch.from_numpy(rows.astype(np.int64)).cuda()
    q[ridx] = dev_bf16(q_rows)
    out, _ = run_prefill(G, layer, q, dev_bf16(k_host), None, pos, cu, out_f32=True)
    got = out[ridx].cpu().numpy()
    del q, out
    torch.cuda.empty_cache()
    qo = np.zeros((T, Hq, d), np.uint16)  # only the sampled rows are read
    qo[rows] = q_rows
    ref, _ = oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                              qo, k_host, None, pos, cu, rows=rows)
    assert_close(got, ref, "31B global layer, every query head")


def test_31b_block_local_layer():
    wl = W.b31_block()
    _prefill_case(wl.layers[0], wl.seq_lens, seed=201)


def test_ragged_prefill_both_kinds():
    pre, _ = W.ragged_31b()
    rows = _rows_sample(pre.seq_lens, 2, 2, 2)
    for li, layer in enumerate(pre.layers):
        _prefill_case(layer, pre.seq_lens, seed=300 + li, rows=rows)


def _decode_case(layer: W.LayerSpec, cache_lens, n_q, seed, check_batches=(0,), all_heads=False):
    """Full-size decode/verify; checks the query heads of KV head 0 (every KV head with
    all_heads) for the given sequences."""
    B = len(cache_lens)
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    group = Hq // Hkv
    hk = Hkv if all_heads else 1      # KV heads and query heads with oracle-visible data
    hq = Hq if all_heads else group
    max_len = max(cache_lens)
    local = layer.kind == W.LOCAL
    cap = layer.window if local else max_len
    layout = G.CACHE_RING if local else G.CACHE_CONTIGUOUS
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    kc = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    kc.normal_(generator=gen)
    vc = None
    if not layer.k_eq_v:
        vc = torch.empty_like(kc)
        vc.normal_(generator=gen)
    q = torch.randn((B, n_q, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    nk = torch.randn((B, n_q, Hkv, d), generator=gen, device="cuda").to(torch.bfloat16)
    nv = None if layer.k_eq_v else torch.randn((B, n_q, Hkv, d), generator=gen, device="cuda").to(torch.bfloat16)
    hists = {}
    for b in check_batches:
        n = cache_lens[b]
        kh = W.normal_bf16(seed + b, 1, (n + n_q, hk, d))
        vh = None if layer.k_eq_v else W.normal_bf16(seed + b, 2, (n + n_q, hk, d))
        qb = W.normal_bf16(seed + b, 0, (1, n_q, hq, d))
        hists[b] = (kh, vh, qb)
        q[b, :, 0:hq] = dev_bf16(qb[0])
        nk[b, :, 0:hk] = dev_bf16(kh[n:])
        if nv is not None:
            nv[b, :, 0:hk] = dev_bf16(vh[n:])
        if local:
            lo = max(0, n - cap)
            slots = torch.from_numpy(np.arange(lo, n) % cap).cuda()
            kc[b, 0:hk, slots] = dev_bf16(kh[lo:n]).transpose(0, 1)
            vc[b, 0:hk, slots] = dev_bf16(vh[lo:n]).transpose(0, 1)
        else:
            kc[b, 0:hk, :n] = dev_bf16(kh[:n]).transpose(0, 1)
    p = G.params(layer.kind, Hq, Hkv, d, window=layer.window, rope_p=layer.rope_p, rope_base=layer.rope_base,
                 softmax_scale=layer.softmax_scale)
    splits = G.gemma_attn_decode_num_splits(p, B, n_q, max_len)
    rows = B * n_q * Hq
    po = torch.empty((splits, rows, d), dtype=torch.float32, device="cuda")
    pl = torch.empty((splits, rows), dtype=torch.float32, device="cuda")
    G.gemma_attn_decode(p, q, nk, nv, kc, vc, layout, cap, dev_i32(cache_lens), B, n_q, max_len, po, pl, splits)
    out = torch.empty((B, n_q, Hq, d), dtype=torch.float32, device="cuda")
    G.gemma_attn_combine(po, pl, splits, rows, d, G.OUT_F32, out, None)
    G.gemma_attn_check()
    got_all = out.cpu().numpy()
    del kc, vc, q, nk, nv, po, pl, out
    torch.cuda.empty_cache()
    for b in check_batches:
        kh, vh, qb = hists[b]
        ref, _ = oracle.decode(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                               qb, [kh], None if vh is None else [vh], [cache_lens[b]])
        assert_close(got_all[b:b + 1, :, 0:hq], ref, f"full-size decode {layer} b={b}")


def test_long_context_decode_global():
    wl = W.long_decode()
    _decode_case(wl.layers[0], list(wl.cache_lens), wl.n_q, seed=400, check_batches=(0, 7))


def test_long_context_decode_local_ring():
    wl = W.long_decode()
    _decode_case(wl.layers[1], list(wl.cache_lens), wl.n_q, seed=401, check_batches=(0, 3))


def test_ragged_verify_both_kinds():
    _, ver = W.ragged_31b()
    for li, layer in enumerate(ver.layers):
        _decode_case(layer, list(ver.cache_lens), ver.n_q, seed=500 + li, check_batches=(0, 1, 7))


def test_ragged_verify_global_every_kv_head():
    """The tcgen05 verify kernel at full size: every KV head's group (CTAs of every
    blockIdx.y), on the longest sequence and a short one."""
    _, ver = W.ragged_31b()
    layer = [l for l in ver.layers if l.kind == W.GLOBAL][0]
    lens = list(ver.cache_lens)
    b_long = int(np.argmax(lens))
    b_short = int(np.argmin(lens))
    _decode_case(layer, lens, ver.n_q, seed=520, check_batches=(b_long, b_short), all_heads=True)
