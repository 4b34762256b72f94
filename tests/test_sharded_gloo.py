"""Split-KV decode across ranks, run as two gloo processes on the CPU.

Each rank holds one contiguous half of every sequence's history (a 256K-token sequence
and a 100,003-token one, global-layer shapes: 8 query heads per KV head, head dim 512,
p-RoPE p = 0.25), computes its partial outputs and log-sum-exps, the ranks all-gather
them and combine: every rank's result must equal the oracle's attention over the whole
history. The kernels are stood in for by the oracle itself (its key-range split and its
combine), so this checks the host plumbing of global_interleaved_layers_b200.sharded: the
ranges, the queries' position offsets, which rank sees the new tokens, and the rank-major
layout of the gathered splits. The GPU side of the same path is tests/test_gpu_sharded.py.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from global_interleaved_layers_b200.sharded import query_offsets, shard_ranges


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


LENGTHS = (262144, 100003)
N_Q = 2


def _rank_main(rank, world, port, q_out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch
    import torch.distributed as dist

    import global_interleaved_layers_b200 as G
    import oracle
    import workloads as W
    from global_interleaved_layers_b200.sharded import ShardedDecode

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        layer = W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6)
        Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
        B = len(LENGTHS)
        hist = [W.normal_bf16(70 + b, 1, (n + N_Q, Hkv, d)) for b, n in enumerate(LENGTHS)]
        qn = W.normal_bf16(70, 0, (B, N_Q, Hq, d))
        offs = query_offsets(LENGTHS, world, rank)

        class OracleBackend:
            """The oracle standing in for the kernels: this rank's keys of each history."""

            def decode_shard(self, p, q, new_k, k_shard, cap, shard_lens, q_off, include_new, batch, n_q,
                             max_len, po, pl, splits, stream):
                assert include_new == (rank == world - 1)
                assert (new_k is None) == (not include_new)
                assert list(shard_lens.tolist()) == [o[1] for o in offs]
                assert list(q_off.tolist()) == [o[2] for o in offs]
                assert splits == 1 and batch == B and n_q == N_Q
                for b, n in enumerate(LENGTHS):
                    lo, ln, _ = offs[b]
                    hi = lo + ln + (N_Q if include_new else 0)
                    T = n + N_Q
                    qfull = np.zeros((T, Hq, d), np.uint16)  # only the query rows are read
                    qfull[n:] = qn[b]
                    rows = np.arange(n, T, dtype=np.int32)
                    o, lse = oracle.attention(layer.kind, 0, layer.rope_p, layer.rope_base, layer.softmax_scale,
                                              qfull, hist[b], None, np.arange(T, dtype=np.int32),
                                              np.array([0, T], np.int32), rows=rows, key_range=(lo, hi))
                    r0 = b * N_Q * Hq
                    po[0, r0:r0 + N_Q * Hq] = torch.from_numpy(o.reshape(N_Q * Hq, d))
                    pl[0, r0:r0 + N_Q * Hq] = torch.from_numpy(lse.reshape(N_Q * Hq))

            def combine(self, po, pl, nsplit, rows, dd, out_dtype, out, lse, stream):
                assert nsplit == world and po.shape[0] == world
                o, l = oracle.combine(po.numpy(), pl.numpy())
                out.copy_(torch.from_numpy(o).reshape(out.shape))
                lse.copy_(torch.from_numpy(l))

        p = G.params(layer.kind, Hq, Hkv, d, rope_p=layer.rope_p, rope_base=layer.rope_base,
                     softmax_scale=layer.softmax_scale, out_dtype=G.OUT_F32)
        dec = ShardedDecode(p, B, N_Q, 1, "cpu", out_dtype=G.OUT_F32, backend=OracleBackend())
        # po / pl in float64 so the oracle's partials pass through the gather unrounded
        for name in ("po_local", "pl_local", "po_all", "pl_all"):
            setattr(dec, name, getattr(dec, name).double())
        shard_lens = torch.tensor([o[1] for o in offs], dtype=torch.int32)
        q_off = torch.tensor([o[2] for o in offs], dtype=torch.int32)
        new_k = torch.from_numpy(np.stack([hist[b][n:] for b, n in enumerate(LENGTHS)]).view(np.int16))
        out = torch.zeros((B, N_Q, Hq, d), dtype=torch.float64)
        lse = torch.zeros((B * N_Q * Hq,), dtype=torch.float64)
        dec(torch.from_numpy(qn.view(np.int16)), new_k, None, 0, shard_lens, q_off, max(o[1] for o in offs), out, lse)
        if rank == 0:
            ref, ref_lse = oracle.decode(layer.kind, 0, layer.rope_p, layer.rope_base, layer.softmax_scale, qn,
                                         hist, None, list(LENGTHS))
            q_out.put((rank, float(np.max(np.abs(out.numpy() - ref))),
                       float(np.max(np.abs(lse.numpy().reshape(ref_lse.shape) - ref_lse)))))
        else:
            q_out.put((rank, 0.0, 0.0))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_ranges_cover_the_history_on_tile_bounds():
    for n in (0, 1, 127, 128, 129, 100003, 262144):
        for world in (1, 2, 3, 4, 8):
            rr = shard_ranges(n, world)
            assert rr[0][0] == 0 and rr[-1][1] == n and len(rr) == world
            for (lo, hi), (lo2, _) in zip(rr, rr[1:]):
                assert hi == lo2 and lo <= hi and hi % 128 == 0
    # the queries sit after the tokens of later ranks
    offs = query_offsets((1000,), 2, 0)
    assert offs == [(0, 384, 616)]
    assert query_offsets((1000,), 2, 1) == [(384, 616, 0)]


def test_two_rank_split_kv_decode_over_a_256k_history():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    got = dict((r, (e, el)) for r, e, el in (q.get(timeout=5) for _ in range(world)))
    err, lse_err = got[0]
    assert err < 1e-9 and lse_err < 1e-9, (err, lse_err)
