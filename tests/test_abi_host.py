"""C-ABI contract checks that need no GPU: the library loads, exports every function the
header declares, rejects bad arguments before launching anything, and its host tile
planner matches the oracle's brute-force tile classification exactly."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
G = pytest.importorskip("global_interleaved_layers_b200")


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gemma_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gemma_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(G.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_error_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert G.gemma_attn_error_string(code) != "unknown status"
    assert G.gemma_attn_error_string(-99) == "unknown status"


def _p(**kw):
    base = dict(kind=G.LOCAL, num_q_heads=4, num_kv_heads=2, head_dim=256, window=16, rope_p=1.0,
                rope_base=1e4, softmax_scale=0.0625)
    base.update(kw)
    return G.params(base.pop("kind"), base.pop("num_q_heads"), base.pop("num_kv_heads"), base.pop("head_dim"),
                    **base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), G.ERR_UNSUPPORTED),
    (dict(num_q_heads=3), G.ERR_INVALID_ARG),
    (dict(window=0), G.ERR_INVALID_ARG),
    (dict(rope_p=1.5), G.ERR_INVALID_ARG),
    (dict(rope_base=0.0), G.ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), G.ERR_INVALID_ARG),
])
def test_bad_params_rejected(kw, code):
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill_workspace_size(_p(**kw), 100)
    assert e.value.status == code


def test_prefill_argument_errors_launch_nothing():
    p = _p()
    fake = 1 << 20  # never dereferenced: validation fails first
    # v missing on a local layer
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill(p, fake, fake, None, fake, None, fake, fake, 1, 10, 10, fake, 1 << 20, 0)
    assert e.value.status == G.ERR_INVALID_ARG
    # misaligned q
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill(p, fake + 2, fake, fake, fake, None, fake, fake, 1, 10, 10, fake, 1 << 20, 0)
    assert e.value.status == G.ERR_MISALIGNED
    # workspace too small
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill(p, fake, fake, fake, fake, None, fake, fake, 1, 10, 10, fake, 16, 0)
    assert e.value.status == G.ERR_WORKSPACE
    # K=V layer given a separate v
    pg = _p(kind=G.GLOBAL, num_q_heads=8, num_kv_heads=1, head_dim=512, rope_p=0.25)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill(pg, fake, fake, fake, fake, None, fake, fake, 1, 10, 10, fake, 1 << 30, 0)
    assert e.value.status == G.ERR_INVALID_ARG


def test_decode_argument_errors():
    p = _p(window=64)
    fake = 1 << 20
    # ring capacity must equal the window
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(p, fake, fake, fake, fake, fake, G.CACHE_RING, 32, fake, 1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_INVALID_ARG
    pg = _p(kind=G.GLOBAL, num_q_heads=8, num_kv_heads=1, head_dim=512, rope_p=0.25)
    # no ring for a global layer
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(pg, fake, fake, None, fake, None, G.CACHE_RING, 64, fake, 1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_INVALID_ARG
    # too many query rows per KV head
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(pg, fake, fake, None, fake, None, G.CACHE_CONTIGUOUS, 64, fake, 1, 5, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_UNSUPPORTED
    # a global layer's K=V cache cannot hold rotated keys (they are also the values)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(pg, fake, fake, None, fake, None, G.CACHE_CONTIGUOUS | G.CACHE_KEYS_ROTATED, 64, fake,
                            1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_INVALID_ARG
    # unknown layout bits
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(p, fake, fake, fake, fake, fake, G.CACHE_RING | 0x40, 64, fake, 1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_INVALID_ARG
    # 16 rows of a separate-V d = 512 layer: no decode variant fits in shared memory
    pl = _p(num_q_heads=16, num_kv_heads=1, head_dim=512, window=64)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(pl, fake, fake, fake, fake, fake, G.CACHE_RING, 64, fake, 1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_UNSUPPORTED


def test_combine_argument_errors():
    fake = 1 << 20
    bad = [
        (0, fake, 2, 8, 64, G.OUT_BF16, fake),      # no partial_o
        (fake, 0, 2, 8, 64, G.OUT_BF16, fake),      # no partial_lse
        (fake, fake, 2, 8, 64, G.OUT_BF16, 0),      # no out
        (fake, fake, 0, 8, 64, G.OUT_BF16, fake),   # no split
        (fake, fake, 2, -1, 64, G.OUT_BF16, fake),  # negative row count
        (fake, fake, 2, 8, 0, G.OUT_BF16, fake),    # empty head dim
        (fake, fake, 2, 8, 64, 7, fake),            # unknown output type
    ]
    for po, pl, s, rows, d, dt, out in bad:
        with pytest.raises(G.GemmaAttnError) as e:
            G.gemma_attn_combine(po, pl, s, rows, d, dt, out, None)
        assert e.value.status == G.ERR_INVALID_ARG
    # no rows: nothing to merge, nothing launched
    G.gemma_attn_combine(fake, fake, 2, 0, 64, G.OUT_F32, fake, None)
    assert G.gemma_attn_last_launch_count() == 0


def test_cache_append_argument_errors():
    p = _p(window=64)
    fake = 1 << 20
    pg = _p(kind=G.GLOBAL, num_q_heads=8, num_kv_heads=1, head_dim=512, rope_p=0.25)
    cases = [
        # ring capacity must equal the window
        ((p, fake, fake, fake, fake, G.CACHE_RING, 32, fake, 1, 1), G.ERR_INVALID_ARG),
        # a local layer needs its value rows, a global one has none
        ((p, fake, None, fake, fake, G.CACHE_RING, 64, fake, 1, 1), G.ERR_INVALID_ARG),
        ((pg, fake, fake, fake, None, G.CACHE_CONTIGUOUS, 64, fake, 1, 1), G.ERR_INVALID_ARG),
        # no ring and no rotated keys for a global layer's K=V cache
        ((pg, fake, None, fake, None, G.CACHE_RING, 64, fake, 1, 1), G.ERR_INVALID_ARG),
        ((pg, fake, None, fake, None, G.CACHE_CONTIGUOUS | G.CACHE_KEYS_ROTATED, 64, fake, 1, 1), G.ERR_INVALID_ARG),
        # empty batch, no new tokens, unknown layout bits
        ((p, fake, fake, fake, fake, G.CACHE_RING, 64, fake, 0, 1), G.ERR_INVALID_ARG),
        ((p, fake, fake, fake, fake, G.CACHE_RING, 64, fake, 1, 0), G.ERR_INVALID_ARG),
        ((p, fake, fake, fake, fake, G.CACHE_RING | 0x40, 64, fake, 1, 1), G.ERR_INVALID_ARG),
        # rows must be 16-byte aligned
        ((p, fake + 2, fake, fake, fake, G.CACHE_RING, 64, fake, 1, 1), G.ERR_MISALIGNED),
    ]
    for args, code in cases:
        with pytest.raises(G.GemmaAttnError) as e:
            G.gemma_attn_cache_append(*args, stream=0)
        assert e.value.status == code, args


def test_bidir_argument_rules():
    fake = 1 << 20
    # the 2D rotation turns every pair: rope_p must be 1
    p = _p(kind=G.BIDIR, num_q_heads=4, num_kv_heads=4, head_dim=64, rope_p=0.5)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill_workspace_size(p, 100)
    assert e.value.status == G.ERR_INVALID_ARG
    # whole 64-dim chunks
    p = _p(kind=G.BIDIR, num_q_heads=4, num_kv_heads=4, head_dim=32, rope_p=1.0)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_prefill_workspace_size(p, 100)
    assert e.value.status == G.ERR_UNSUPPORTED
    # no decode for the vision kind
    p = _p(kind=G.BIDIR, num_q_heads=4, num_kv_heads=4, head_dim=64, rope_p=1.0)
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode(p, fake, fake, fake, fake, fake, G.CACHE_CONTIGUOUS, 64, fake, 1, 1, 10, fake, fake, 1, 0)
    assert e.value.status == G.ERR_UNSUPPORTED
    with pytest.raises(G.GemmaAttnError) as e:
        G.gemma_attn_decode_num_splits(p, 1, 1, 10)
    assert e.value.status == G.ERR_UNSUPPORTED


@pytest.mark.parametrize("lens", [(200, 64, 129), (1,), (128, 256)])
def test_bidir_tile_plan_matches_oracle(lens):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    got = G.gemma_attn_tile_plan(G.BIDIR, 0, cu, 128, 128)
    want = oracle.tile_plan(oracle.BIDIR, 0, pos, cu, 128, 128)
    np.testing.assert_array_equal(np.asarray(got).reshape(-1, 4), np.asarray(want).reshape(-1, 4))


def test_workspace_sizes():
    # local p = 1: full rotated q and k copies; global p = 0.25, d = 512: 2 of 8 chunks
    T = 1000
    loc = _p(num_q_heads=8, num_kv_heads=4)
    assert G.gemma_attn_prefill_workspace_size(loc, T) == T * (8 + 4) * 256 * 2
    glo = _p(kind=G.GLOBAL, num_q_heads=8, num_kv_heads=1, head_dim=512, rope_p=0.25)
    assert G.gemma_attn_prefill_workspace_size(glo, T) == T * 8 * 128 * 2 + T * 1 * 128 * 2
    none = _p(kind=G.GLOBAL, num_q_heads=8, num_kv_heads=1, head_dim=512, rope_p=0.0)
    assert G.gemma_attn_prefill_workspace_size(none, T) == 0


@pytest.mark.parametrize("kind,window,lens,bm,bn", [
    (W.GLOBAL, 0, (1000,), 128, 128),
    (W.GLOBAL, 0, (1, 127, 128, 129, 700), 128, 128),
    (W.LOCAL, 1, (300,), 128, 128),
    (W.LOCAL, 300, (1000, 5, 640), 128, 128),
    (W.LOCAL, 512, (8192,), 128, 128),
    (W.LOCAL, 1024, (2048, 1500), 128, 128),
    (W.LOCAL, 70, (333,), 64, 32),
    (W.LOCAL, 2000, (333,), 128, 128),
])
def test_tile_plan_matches_oracle_brute_force(kind, window, lens, bm, bn):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    got = G.gemma_attn_tile_plan(kind, window, cu, bm, bn)
    want = oracle.tile_plan(kind, window, pos, cu, bm, bn)
    np.testing.assert_array_equal(got, want)


def test_decode_split_hint():
    glo = _p(kind=G.GLOBAL, num_q_heads=32, num_kv_heads=4, head_dim=512, rope_p=0.25)
    s = G.gemma_attn_decode_num_splits(glo, 8, 1, 131072)
    assert s >= 1 and 8 * 4 * s >= 148
    loc = _p(num_q_heads=32, num_kv_heads=16, window=1024)
    assert G.gemma_attn_decode_num_splits(loc, 8, 1, 5) == 1


def test_decode_split_hint_verify_shapes(monkeypatch):
    # the tcgen05 verify kernel's shapes (global, 9..32 rows per KV head) get twice the
    # uniform-length choice, at most one split per 128 keys; the legacy path keeps it
    glo = _p(kind=G.GLOBAL, num_q_heads=32, num_kv_heads=4, head_dim=512, rope_p=0.25)
    for batch, n_q, max_len in [(16, 4, 42740), (2, 4, 300), (8, 2, 131072)]:
        monkeypatch.setenv("GEMMA_ATTN_DECODE_MMA_SYNC", "1")
        uniform = G.gemma_attn_decode_num_splits(glo, batch, n_q, max_len)
        monkeypatch.delenv("GEMMA_ATTN_DECODE_MMA_SYNC")
        got = G.gemma_attn_decode_num_splits(glo, batch, n_q, max_len)
        assert got == min(2 * uniform, (max_len + n_q + 127) // 128)
    # 8 rows per KV head stay on the warp kernel: no doubling
    one = G.gemma_attn_decode_num_splits(glo, 8, 1, 131072)
    monkeypatch.setenv("GEMMA_ATTN_DECODE_MMA_SYNC", "1")
    assert G.gemma_attn_decode_num_splits(glo, 8, 1, 131072) == one


def test_shard_entry_point_argument_rules():
    # rejected before any launch: no device is needed
    loc = G.params(G.LOCAL, 8, 4, 256, window=64)
    glo = G.params(G.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
    fake = 1 << 20
    with pytest.raises(G.GemmaAttnError) as e:  # local layers hold only a window: no shards
        G.gemma_attn_decode_shard(loc, fake, fake, fake, 64, fake, fake, True, 1, 1, 64, fake, fake, 1)
    assert e.value.status == G.ERR_INVALID_ARG
    with pytest.raises(G.GemmaAttnError) as e:  # the shard that ends the history needs the new keys
        G.gemma_attn_decode_shard(glo, fake, None, fake, 64, fake, fake, True, 1, 1, 64, fake, fake, 1)
    assert e.value.status == G.ERR_INVALID_ARG
    with pytest.raises(G.GemmaAttnError) as e:  # no offsets
        G.gemma_attn_decode_shard(glo, fake, None, fake, 64, fake, None, False, 1, 1, 64, fake, fake, 1)
    assert e.value.status == G.ERR_INVALID_ARG
