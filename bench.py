"""Benchmark of the Gemma-4-style interleaved attention path on B200.

A step is one pass of the hot path over the 31B-shaped prefill block: L = 32768 tokens,
5 sliding-window layers (W = 1024, 32/16 heads, d = 256) and 1 global layer (32/4 heads,
d = 512, K=V, p-RoPE p = 0.25). `value` is unmasked prefill TFLOP/s of that block, its
twelve launches (rotated side copy + attention per layer) replayed as one CUDA graph; the
same calls launched one by one are reported as per_kind.b31_block_eager, and the
E2B-shaped block (L = 8192, 4 local + 1 global) and the ragged 16-sequence 31B-shaped
batch (both layer kinds) beside them.
In the same run the decode path (split-KV + combine) is timed on the long-context
decode shape (batch 8, 32/4 heads, global K=V cache of 131072 tokens at d = 512;
local 1024-slot ring at d = 256, 32/16 heads) and the 4-token verify of the ragged
batch, reported in HBM GB/s.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs an independent replica (weak scaling); rank 0 prints
one JSON line with the max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "prefill TFLOP/s (unmasked FLOPs) and decode HBM GB/s per layer kind, % roofline"
L2_FLUSH_BYTES = 256 << 20


# DRAM bytes (read + write) per launch of the global layer's attention kernel on the
# headline block: an ncu capture of the same sequence length with a quarter of the heads
# (8 query heads, 1 KV head), scaled by 4 (the work units and their bytes scale with the
# heads). Reported only while the kernel's sources (their code: comments and blank lines do
# not count) still hash to the captured state; any change makes it null until re-captured.
NCU_TRAFFIC = {"bytes": 4 * (334923776 + 233282048), "sources_sha256_16": "661f32af2124420b",
               "sources": ["global_interleaved_layers_b200/csrc/prefill.cu",
                           "global_interleaved_layers_b200/csrc/common.cuh",
                           "global_interleaved_layers_b200/csrc/tile_plan.h",
                           "global_interleaved_layers_b200/csrc/kernels.h"]}


def source_code_hash(paths):
    """sha256 (16 hex digits) of C/CUDA sources with comments, trailing blanks and empty
    lines removed: a comment edit leaves it unchanged, any change to the code does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in paths:
        with open(os.path.join(ROOT, f), "r", encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def ncu_traffic():
    try:
        digest = source_code_hash(NCU_TRAFFIC["sources"])
    except OSError:
        return None
    return NCU_TRAFFIC["bytes"] if digest == NCU_TRAFFIC["sources_sha256_16"] else None


def log(msg: str) -> None:
    print(f"[bench {time.strftime('%H:%M:%S')}] {msg}", file=sys.stderr, flush=True)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region.

    Polls NVML (the library nvidia-smi reads) from a thread every ~2 ms, so that even a
    region of a few tens of milliseconds gets samples; falls back to `nvidia-smi -lms`
    when NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.rows = []
        self.thread = None
        self.stop = False
        self.source = None

    def _nvml_start(self):
        import threading
        import pynvml as nv
        import torch
        nv.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
        h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        max_sm = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

        def sample():
            sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.rows.append((sm, max_sm, ["Active" if r & b else "Not Active" for b in bits]))

        def loop():
            while not self.stop:
                try:
                    sample()
                except Exception:
                    return
                time.sleep(0.002)

        sample()
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        self.source = "nvml"

    def __enter__(self):
        try:
            self._nvml_start()
            return self
        except Exception:
            self.rows = []
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.idx)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
            t0 = time.time()  # let the first sample land before the timed region starts
            while time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = list(self.rows)
        if self.path is not None:
            try:
                for line in open(self.path):
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                    except ValueError:
                        continue
            finally:
                try:
                    os.unlink(self.path)
                except Exception:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        reasons = sorted({self.NAMES[i] for _, _, flags in rows for i, f in enumerate(flags)
                          if f.lower().startswith("active")})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "source": self.source}


# ----------------------------------------------------------------------------- CPU oracle baseline

def sample_rows(L: int, n_first: int, n_last: int, n_rand: int, seed: int = 1):
    """First n_first, last n_last and n_rand rows from default_rng(seed), sorted, unique."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(n_first, L))) | set(range(max(0, L - n_last), L))
    rows |= set(int(x) for x in rng.integers(0, L, size=n_rand))
    return np.array(sorted(rows), dtype=np.int32)


def oracle_sample_flops(layer: W.LayerSpec, rows: np.ndarray) -> int:
    """Unmasked FLOPs of the sampled query rows (one sequence, positions 0 .. L-1)."""
    pairs = 0
    for i in rows.tolist():
        vis = i + 1 if layer.kind == W.GLOBAL else min(i + 1, layer.window)
        pairs += vis
    return 4 * layer.head_dim * layer.num_q_heads * pairs


class OracleBlockSample:
    """The fp64 oracle on a bounded row sample of each distinct layer shape of a block.

    Inputs: every key/value row (the sampled rows see any of them) and only the sampled
    query rows (the rest of q is never read: a zero array whose pages stay untouched)."""

    def __init__(self, wl: W.PrefillWorkload, rows: np.ndarray):
        import oracle
        oracle.build()
        self.oracle = oracle
        self.wl = wl
        self.rows = rows
        L = wl.total_tokens
        self.pos, self.cu = wl.positions(), wl.cu_seqlens()
        self.kinds = []  # (layer, count in the block, q, k, v)
        seen = {}
        for li, layer in enumerate(wl.layers):
            if layer in seen:
                seen[layer][1] += 1
                continue
            base = wl.seed + 16 * li
            q = np.zeros((L, layer.num_q_heads, layer.head_dim), np.uint16)
            q[rows] = W.normal_bf16(base, 0, (rows.shape[0], layer.num_q_heads, layer.head_dim))
            k = W.normal_bf16(base, 1, (L, layer.num_kv_heads, layer.head_dim))
            v = None if layer.k_eq_v else W.normal_bf16(base, 2, (L, layer.num_kv_heads, layer.head_dim))
            seen[layer] = [layer, 1, q, k, v]
        self.kinds = list(seen.values())

    def run(self):
        """Time one pass over each distinct layer shape; returns (seconds for the block's
        layers, each distinct shape's time counted once per layer of that shape, FLOPs of
        that much work, query-row x head units)."""
        sec = flops = units = 0
        for layer, count, q, k, v in self.kinds:
            t0 = time.perf_counter()
            self.oracle.attention(layer.kind, layer.window, layer.rope_p, layer.rope_base, layer.softmax_scale,
                                  q, k, v, self.pos, self.cu, rows=self.rows)
            sec += count * (time.perf_counter() - t0)
            flops += count * oracle_sample_flops(layer, self.rows)
            units += count * self.rows.shape[0] * layer.num_q_heads
        return sec, flops, units


def cpu_baseline(wl: W.PrefillWorkload):
    """The fp64 oracle on a bounded row sample of the headline block (about 10 s on 16
    host cores): its FLOP rate, query rows per second, and the full block's time
    extrapolated from that rate."""
    rows = sample_rows(wl.total_tokens, 32, 32, 64)
    smp = OracleBlockSample(wl, rows)
    sec, flops, units = smp.run()
    rate = flops / sec
    block_flops = sum(W.prefill_flops(wl.seq_lens, layer) for layer in wl.layers)
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": smp.oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(rows)} query rows (first 32, last 32, 64 from default_rng(1)) x all heads of "
                      f"each distinct layer shape of {wl.name}; the local shape's time counted once per local "
                      f"layer ({sum(1 for ly in wl.layers if ly.kind == W.LOCAL)} of them); fp64 C oracle with "
                      "OpenMP",
            "seconds": sec, "query_rows_per_s": units / sec, "query_rows_unit": "query row x head",
            "extrapolated_full_block_s": block_flops / rate,
            "extrapolated_note": "extrapolated: the full block's unmasked FLOPs / the sample's FLOP rate"}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, each step a bounded sample of
    the headline block (its first 16 and last 16 query rows of every layer shape)."""
    world, rank, local = dist_setup(args.gpus)
    if rank != 0:
        return
    wl = W.b31_block()
    L = wl.total_tokens
    rows = sample_rows(L, 16, 16, 0)
    smp = OracleBlockSample(wl, rows)
    for _ in range(args.warmup):
        smp.run()
    sec = flops = 0
    for _ in range(args.steps):
        s_, f_, _ = smp.run()
        sec += s_
        flops += f_
    value = flops / sec / 1e12
    sample = (f"{len(rows)} query rows (first 16, last 16) x all heads of each distinct layer shape of {wl.name} "
              "per step, the local shape's time counted once per local layer; fp64 C oracle with OpenMP")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": 1, "seq_len": L,
                   "layers": "5 local (W=1024, 32/16 heads, d=256) + 1 global (32/4 heads, d=512, K=V, p=0.25)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": smp.oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------- GPU arm

class BlockBench:
    """One prefill block's device buffers and its timings (graph replay and call by call)."""

    def __init__(self, G, torch, dev, wl: W.PrefillWorkload, seed: int):
        self.G, self.torch, self.wl = G, torch, wl
        L = wl.total_tokens
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        self.layers = []
        max_ws = 0
        for li, layer in enumerate(wl.layers):
            q = torch.randn((L, layer.num_q_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
            k = torch.randn((L, layer.num_kv_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
            v = None if layer.k_eq_v else torch.randn((L, layer.num_kv_heads, layer.head_dim), generator=gen,
                                                     device=dev).to(torch.bfloat16)
            out = torch.empty_like(q)
            p = G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, window=layer.window,
                         rope_p=layer.rope_p, rope_base=layer.rope_base, softmax_scale=layer.softmax_scale)
            max_ws = max(max_ws, G.gemma_attn_prefill_workspace_size(p, L))
            self.layers.append(dict(spec=layer, q=q, k=k, v=v, out=out, p=p,
                                    flops=W.prefill_flops(wl.seq_lens, layer)))
        self.ws = torch.empty(max(max_ws, 256), dtype=torch.uint8, device=dev)
        self.pos = torch.from_numpy(wl.positions()).to(dev)
        self.cu = torch.from_numpy(wl.cu_seqlens()).to(dev)
        self.total_flops = sum(ly["flops"] for ly in self.layers)
        self.glob = [li for li, ly in enumerate(self.layers) if ly["spec"].kind == W.GLOBAL]
        self.loc = [li for li, ly in enumerate(self.layers) if ly["spec"].kind == W.LOCAL]
        self.blk = None

    def call_args(self, li, stream):
        ly = self.layers[li]
        S = len(self.wl.seq_lens)
        L = self.wl.total_tokens
        return (ly["p"], ly["q"], ly["k"], ly["v"], ly["out"], None, self.pos, self.cu, S, L,
                max(self.wl.seq_lens), self.ws, self.ws.numel(), stream)

    def run_layer(self, li, stream):
        # one layer = the prefill's two phases back to back (exactly what gemma_attn_prefill runs)
        G = self.G
        call = self.call_args(li, stream)
        G.gemma_attn_prefill_rotate(*call)
        n = G.gemma_attn_last_launch_count()
        G.gemma_attn_prefill_attend(*call)
        return n + G.gemma_attn_last_launch_count()

    def capture(self, stream, warmup):
        """The block's launches recorded once as a CUDA graph, with two events around the
        global layer's attention kernel (each recorded event costs the stream microseconds,
        so there are no others)."""
        torch, G = self.torch, self.G
        from global_interleaved_layers_b200.block import BlockLayer, InterleavedBlock
        S, L = len(self.wl.seq_lens), self.wl.total_tokens
        self.blk = InterleavedBlock([BlockLayer(ly["p"], ly["q"], ly["k"], ly["v"], ly["out"], None, self.pos,
                                                self.cu, S, L, max(self.wl.seq_lens), self.ws)
                                     for ly in self.layers])
        self.att0 = torch.cuda.Event(enable_timing=True, external=True)
        self.att1 = torch.cuda.Event(enable_timing=True, external=True)
        g0 = self.glob[0]
        evs = [((None, self.att0, self.att1) if li == g0 else None) for li in range(len(self.layers))]
        self.launches_per_step = self.blk.capture(events=evs)
        for _ in range(warmup):
            self.blk.replay()
        torch.cuda.synchronize()
        G.gemma_attn_check()

    def time_graph(self, stream, steps, flush_l2):
        """Per-step ms of graph replays (L2 flushed before each) and the global attention
        kernel's ms inside each."""
        torch = self.torch
        step_ms, att_ms = [], []
        for _ in range(steps):
            flush_l2()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            self.blk.replay()
            s1.record(stream)
            # the graph's events are re-recorded by every replay: read them now
            s1.synchronize()
            step_ms.append(s0.elapsed_time(s1))
            att_ms.append(self.att0.elapsed_time(self.att1))
        self.G.gemma_attn_check()
        return step_ms, att_ms

    def release_graph(self):
        if self.blk is not None:
            self.blk.graph = None

    def time_eager(self, stream, steps, flush_l2):
        """The same step launched call by call (no graph), with events around every layer.
        Returns (mean step ms, {layer index: mean ms})."""
        torch = self.torch
        step, per = [], {}
        for _ in range(steps):
            flush_l2()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            evs = []
            for li in range(len(self.layers)):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                self.run_layer(li, stream)
                e1.record(stream)
                evs.append((e0, e1))
            s1.record(stream)
            torch.cuda.synchronize()
            step.append(s0.elapsed_time(s1))
            for li, (e0, e1) in enumerate(evs):
                per.setdefault(li, []).append(e0.elapsed_time(e1))
        self.G.gemma_attn_check()
        return float(np.mean(step)), {li: float(np.mean(v)) for li, v in per.items()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="only the headline block (no per_kind extras)")
    ap.add_argument("--case", default="block",
                    choices=["block", "global_prefill", "local_prefill", "global_prefill_31b_h8", "local_prefill_31b",
                             "global_decode", "local_decode", "global_verify", "vision_prefill"],
                    help="block: the benchmark (one JSON line). Any other value runs only that operation "
                         "(warmup + steps launches, no timing contract) for profiler captures.")
    ap.add_argument("--ctx", type=int, default=0, help="decode cases: cached tokens per sequence (0: 131072)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    if args.case != "block":
        run_case(args)
        return

    import torch
    import global_interleaved_layers_b200 as G

    from global_interleaved_layers_b200.replicas import Replicas

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    reps = Replicas(backend="nccl", timeout_s=120)  # process group only when WORLD_SIZE > 1
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    peak_t = peaks["bf16_tflops"]  # burst, until the clock record of the timed block says otherwise

    def barrier():
        reps.barrier()

    def max_over_ranks(x: float) -> float:
        return reps.max_over_ranks(x, dev)

    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write 256 MiB (evicts every line of the previous step), then read another 256 MiB:
        # the written lines leave L2 (written back) before the timed step, which then starts
        # with L2 holding only clean lines of neither input nor output
        flush_buf.fill_(1.0)
        torch.sum(flush_read, dim=0, out=flush_sink)

    stream = torch.cuda.current_stream()

    # ------------------------------------------------------------------ headline: the 31B-shaped block
    wl = W.b31_block()
    L = wl.total_tokens
    bb = BlockBench(G, torch, dev, wl, seed=1234 + rank)
    log("31B block warmup")
    for _ in range(args.warmup):
        for li in range(len(bb.layers)):
            bb.run_layer(li, stream)
    torch.cuda.synchronize()
    G.gemma_attn_check()
    bb.capture(stream, args.warmup)
    log("31B block timed")
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        step_ms, att_ms = bb.time_graph(stream, args.steps, flush_l2)
        torch.cuda.synchronize()
        barrier()
    clk = clocks.summary()
    # The peak the roofline divides by: the burst GEMM figure for kernels that ran at full
    # clock; the sustained one (a seconds-long GEMM loop under the power cap) when the timed
    # steps themselves ran under the power cap.
    power_capped = "sw_power_cap" in clk.get("reasons", [])
    peak_name = "bf16_tflops_sustained" if power_capped else "bf16_tflops"
    peak_t = peaks[peak_name]
    launches = bb.launches_per_step * args.steps
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / args.steps
    value = world * bb.total_flops * args.steps / (total_ms * 1e-3) / 1e12
    bb.release_graph()

    barrier()
    eager_ms, per_layer_ms = bb.time_eager(stream, max(3, args.steps // 2), flush_l2)
    eager_ms = max_over_ranks(eager_ms)
    barrier()
    g_ms = float(np.mean([per_layer_ms[i] for i in bb.glob]))
    l_ms = float(np.mean([per_layer_ms[i] for i in bb.loc]))
    g_flops = bb.layers[bb.glob[0]]["flops"]
    l_flops = bb.layers[bb.loc[0]]["flops"]
    g_tflops = g_flops / (g_ms * 1e-3) / 1e12
    l_tflops = l_flops / (l_ms * 1e-3) / 1e12
    # the dominant kernel (the global layer's attention) per launch, timed inside the step
    attend_ms = max_over_ranks(float(np.mean(att_ms)))
    attend_tflops = g_flops / (attend_ms * 1e-3) / 1e12
    loc_spec = bb.layers[bb.loc[0]]["spec"]
    local_ceiling = loc_spec.window / (loc_spec.window + 128 - 1)
    per_kind = {
        "local_prefill": {"tflops": l_tflops, "ms": l_ms, "frac_of_peak": l_tflops / peak_t,
                          "tile_geometry_ceiling": local_ceiling,
                          "shape": "31B local layer: L=32768, W=1024, 32/16 heads, d=256 (rotated copy + attention)"},
        "global_prefill": {"tflops": g_tflops, "ms": g_ms, "frac_of_peak": g_tflops / peak_t,
                           "shape": "31B global layer: L=32768, 32/4 heads, d=512, K=V, p=0.25 "
                                    "(rotated copy + attention)"},
        "b31_block_eager": {"ms": eager_ms, "tflops": world * bb.total_flops / (eager_ms * 1e-3) / 1e12,
                            "launches": bb.launches_per_step,
                            "note": "the timed step's calls launched one by one from Python (no CUDA graph), "
                                    "with events around every layer (per_kind.local_prefill / global_prefill)"},
    }

    # ------------------------------------------------------------------ e2e through host buffers
    e2e = bench_e2e(G, torch, dev, stream, bb, args, world, max_over_ranks, barrier)
    del bb
    torch.cuda.empty_cache()

    # ------------------------------------------------------------------ the other workloads
    if not args.no_extra:
        per_kind["e2b_block"] = bench_block_graph(G, torch, dev, stream, W.e2b_block(), args, world,
                                                  max_over_ranks, barrier, flush_l2, peak_t)
        per_kind.update(bench_ragged_prefill(G, torch, dev, stream, args, max_over_ranks, barrier, flush_l2, peak_t))
        if not args.no_decode:
            per_kind.update(bench_decode(G, torch, dev, stream, flush_l2, peaks, args, world, max_over_ranks,
                                         barrier))
            per_kind["sharded_global_decode_256k"] = bench_sharded_decode(G, torch, dev, stream, flush_l2, peaks,
                                                                          args, world, max_over_ranks, barrier)
        per_kind["vision_bidir_prefill"] = bench_vision(G, torch, dev, stream, flush_l2, peaks, args, world,
                                                        max_over_ranks, barrier)

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": 1, "seq_len": L,
                   "layers": "5 local (W=1024, 32/16 heads, d=256) + 1 global (32/4 heads, d=512, K=V, p=0.25)",
                   "l2": "inputs larger than L2, and L2 flushed before every timed step (256 MiB write, then a "
                         "256 MiB read of another buffer, so no dirty lines are left for the step to write back); "
                         "per-step CUDA events",
                   "parallelism": f"replicas x{world}"},
        "per_kind": per_kind,
        "roofline": {"bound": "tensor", "achieved": attend_tflops, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": attend_tflops / peak_t, "kernel_ms": attend_ms, "traffic": ncu_traffic(),
                     "traffic_unit": "bytes per launch",
                     "frac_of_burst_peak": attend_tflops / peaks["bf16_tflops"],
                     "frac_of_sustained_peak": attend_tflops / peaks["bf16_tflops_sustained"],
                     "kernel": "prefill_kernel<512>: the 31B global layer's attention phase (35.19 TFLOP of "
                               "unmasked work per launch), timed with CUDA events recorded inside the timed "
                               "step's graph (per_kind.global_prefill, from the call-by-call run, also counts "
                               "the rotated side copy)",
                     "peak_source": f"{peaks['source']} {peak_name} ("
                                    + ("sustained: the timed steps ran under sw_power_cap" if power_capped else
                                       "burst: the timed steps ran at full clock") + ")"},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        log("cpu baseline")
        result["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(result), flush=True)
    reps.close()


def bench_e2e(G, torch, dev, stream, bb, args, world, max_over_ranks, barrier):
    """The block through the public API with host buffers: every step copies each layer's
    q/k/v from pinned host memory and its output back, inside the timed region."""
    host = []
    h2d = d2h = 0
    for ly in bb.layers:
        hq = ly["q"].cpu().pin_memory()
        hk = ly["k"].cpu().pin_memory()
        hv = None if ly["v"] is None else ly["v"].cpu().pin_memory()
        ho = torch.empty(ly["out"].shape, dtype=torch.bfloat16).pin_memory()
        host.append((hq, hk, hv, ho))
        h2d += hq.numel() * 2 + hk.numel() * 2 + (0 if hv is None else hv.numel() * 2)
        d2h += ho.numel() * 2

    # Three streams, as a serving loop would run them: host->device copies of a layer's
    # inputs, the layer's attention call, and the device->host copy of its output, each
    # ordered after the step it depends on, so that copies of one layer overlap the
    # attention of another. Every step still moves all of its inputs and outputs.
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    nl = len(bb.layers)
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_done = [torch.cuda.Event() for _ in range(nl)]
    ev_out = [torch.cuda.Event() for _ in range(nl)]
    first_step = [True]

    def e2e_step():
        for li, ly in enumerate(bb.layers):
            hq, hk, hv, ho = host[li]
            with torch.cuda.stream(h2d_stream):
                if not first_step[0]:
                    h2d_stream.wait_event(ev_done[li])  # the previous step's call has read the inputs
                ly["q"].copy_(hq, non_blocking=True)
                ly["k"].copy_(hk, non_blocking=True)
                if hv is not None:
                    ly["v"].copy_(hv, non_blocking=True)
                ev_in[li].record(h2d_stream)
            stream.wait_event(ev_in[li])
            if not first_step[0]:
                stream.wait_event(ev_out[li])  # the previous step's output has been read back
            bb.run_layer(li, stream)
            ev_done[li].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_done[li])
                ho.copy_(ly["out"], non_blocking=True)
                ev_out[li].record(d2h_stream)
        first_step[0] = False

    log("e2e")
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e_steps = max(3, args.steps // 4)
    e0.record(h2d_stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(d2h_stream)  # after the last read-back, which follows every earlier operation
    torch.cuda.synchronize()
    G.gemma_attn_check()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e_steps
    value = world * bb.total_flops / (e2e_ms * 1e-3) / 1e12
    del host
    return {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms, "steps": e_steps}


def bench_block_graph(G, torch, dev, stream, wl, args, world, max_over_ranks, barrier, flush_l2, peak_t):
    """A block's step replayed as a CUDA graph (per_kind entry for a second block shape)."""
    bb = BlockBench(G, torch, dev, wl, seed=77)
    for li in range(len(bb.layers)):
        bb.run_layer(li, stream)
    torch.cuda.synchronize()
    bb.capture(stream, args.warmup)
    log(f"{wl.name} timed")
    barrier()
    step_ms, att_ms = bb.time_graph(stream, args.steps, flush_l2)
    barrier()
    ms = max_over_ranks(float(np.mean(step_ms)))
    att = max_over_ranks(float(np.mean(att_ms)))
    g_flops = bb.layers[bb.glob[0]]["flops"]
    bb.release_graph()
    res = {"ms": ms, "tflops": world * bb.total_flops / (ms * 1e-3) / 1e12, "launches": bb.launches_per_step,
           "global_attention_ms": att, "global_attention_tflops": g_flops / (att * 1e-3) / 1e12,
           "global_attention_frac_of_peak": g_flops / (att * 1e-3) / 1e12 / peak_t,
           "shape": f"{wl.name}: " + ", ".join(sorted({str(ly['spec']) for ly in bb.layers}))}
    del bb
    torch.cuda.empty_cache()
    return res


def bench_ragged_prefill(G, torch, dev, stream, args, max_over_ranks, barrier, flush_l2, peak_t):
    """The ragged 16-sequence 31B-shaped batch (229,704 tokens): one local and one global
    layer's prefill, each call timed alone."""
    pre, _ = W.ragged_31b()
    bb = BlockBench(G, torch, dev, pre, seed=91)
    res = {}
    steps = max(3, args.steps // 4)
    for li in range(len(bb.layers)):
        spec = bb.layers[li]["spec"]
        tag = "ragged_global_prefill" if spec.kind == W.GLOBAL else "ragged_local_prefill"
        for _ in range(2):
            bb.run_layer(li, stream)
        torch.cuda.synchronize()
        G.gemma_attn_check()
        log(tag)
        barrier()
        evs = []
        for _ in range(steps):
            flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            bb.run_layer(li, stream)
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        G.gemma_attn_check()
        barrier()
        ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])))
        tf = bb.layers[li]["flops"] / (ms * 1e-3) / 1e12
        res[tag] = {"tflops": tf, "ms": ms, "frac_of_peak": tf / peak_t, "steps": steps,
                    "tflop_per_call": bb.layers[li]["flops"] / 1e12,
                    "shape": f"16 sequences, {pre.total_tokens} tokens (lengths from default_rng(7)), {spec} "
                             "(rotated copy + attention)"}
    del bb
    torch.cuda.empty_cache()
    return res


def bench_decode(G, torch, dev, stream, flush_l2, peaks, args, world, max_over_ranks, barrier):
    res = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    # the long-context decode step, then the 4-token verify of the ragged 31B-shaped batch
    for wl, tag in ((W.long_decode(), "decode"), (W.ragged_31b()[1], "verify")):
        bench_decode_workload(G, torch, dev, stream, flush_l2, peaks, args, max_over_ranks, barrier, gen, wl, tag,
                              res)
    return res


def bench_decode_workload(G, torch, dev, stream, flush_l2, peaks, args, max_over_ranks, barrier, gen, wl, tag, res):
    B, n_q = wl.batch, wl.n_q
    for layer in wl.layers:
        Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
        ctx = max(wl.cache_lens)
        if layer.kind == W.GLOBAL:
            cap = ctx
            layout = G.CACHE_CONTIGUOUS
        else:
            cap = layer.window
            layout = G.CACHE_RING
        kc = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        kc.normal_(generator=gen)
        vc = None
        if not layer.k_eq_v:
            vc = torch.empty_like(kc)
            vc.normal_(generator=gen)
        q = torch.randn((B, n_q, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
        nk = torch.randn((B, n_q, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        nv = None if layer.k_eq_v else torch.randn((B, n_q, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        lens = torch.tensor(list(wl.cache_lens), dtype=torch.int32, device=dev)
        p = G.params(layer.kind, Hq, Hkv, d, window=layer.window, rope_p=layer.rope_p, rope_base=layer.rope_base,
                     softmax_scale=layer.softmax_scale)
        splits = G.gemma_attn_decode_num_splits(p, B, n_q, ctx)
        rows = B * n_q * Hq
        po = torch.empty((splits, rows, d), dtype=torch.float32, device=dev)
        pl = torch.empty((splits, rows), dtype=torch.float32, device=dev)
        out = torch.empty((B, n_q, Hq, d), dtype=torch.bfloat16, device=dev)

        log(f"{tag} kind={layer.kind}")

        def measure(layout):
            # one split: the one-call entry point, whose decode kernel writes the output itself;
            # several: the split partials, then the combine
            def dec():
                if splits == 1:
                    G.gemma_attn_decode_noalloc(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, ctx, 1, out,
                                                None, stream)
                else:
                    G.gemma_attn_decode(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, ctx, po, pl, splits,
                                        stream)

            def comb():
                if splits > 1:
                    G.gemma_attn_combine(po, pl, splits, rows, d, G.OUT_BF16, out, None, stream)

            def one():
                dec()
                comb()

            for _ in range(args.warmup):
                one()
            torch.cuda.synchronize()
            G.gemma_attn_check()

            # the whole call (decode + combine) and the decode kernel alone, each timed in its
            # own loop with two events, so no event sits inside the timed work
            def timed(fn):
                evs = []
                barrier()
                for _ in range(args.steps):
                    flush_l2()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                    evs.append((e0, e1))
                torch.cuda.synchronize()
                G.gemma_attn_check()
                barrier()
                return max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])))

            ms = timed(one)
            dec_ms = timed(dec) if splits > 1 else ms
            nbytes = W.decode_cache_bytes(B, wl.cache_lens, layer)
            gbs = nbytes / (ms * 1e-3) / 1e9
            rotated = bool(layout & G.CACHE_KEYS_ROTATED)
            return {"gbs": gbs, "ms": ms, "decode_kernel_ms": dec_ms, "bytes": nbytes, "splits": splits,
                    "launches": 1 if splits == 1 else 2,
                    "frac_of_hbm": gbs / peaks["hbm_gbs"],
                    "shape": f"B={B} n_q={n_q} Hq={Hq} Hkv={Hkv} d={d} cache lens "
                             f"{min(wl.cache_lens)}..{max(wl.cache_lens)} " + (
                        "K=V contiguous" if layer.k_eq_v else
                        f"ring W={layer.window}, cached keys {'stored rotated' if rotated else 'un-rotated'}")}

        if layer.kind == W.GLOBAL:
            res[f"global_{tag}"] = measure(layout)
        else:
            # the serving layout keeps local keys rotated in the cache; for the decode step
            # the un-rotated cache (the kernel rotates every key) is reported beside it
            res[f"local_{tag}"] = measure(layout | G.CACHE_KEYS_ROTATED)
            if tag == "decode":
                res["local_decode_unrotated_cache"] = measure(layout)
        if tag != "decode":
            del kc, vc
            torch.cuda.empty_cache()
            continue

        # the step's new rows into the cache (after the decode that read them beside it)
        app_layout = layout if layer.k_eq_v else (layout | G.CACHE_KEYS_ROTATED)
        # the contiguous cache is exactly full here: time the append over its last n_q rows
        app_lens = lens - n_q if layer.k_eq_v else lens
        for _ in range(args.warmup):
            G.gemma_attn_cache_append(p, nk, nv, kc, vc, app_layout, cap, app_lens, B, n_q, stream)
        torch.cuda.synchronize()
        app_evs = []
        barrier()
        for _ in range(args.steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            G.gemma_attn_cache_append(p, nk, nv, kc, vc, app_layout, cap, app_lens, B, n_q, stream)
            e1.record(stream)
            app_evs.append((e0, e1))
        torch.cuda.synchronize()
        G.gemma_attn_check()
        barrier()
        app_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in app_evs])))
        app_bytes = 2 * B * n_q * Hkv * d * 2 * (1 if layer.k_eq_v else 2)  # rows read + written
        res["global_cache_append" if layer.kind == W.GLOBAL else "local_cache_append"] = {
            "us": app_ms * 1e3, "bytes": app_bytes, "launches": 1,
            "note": "one launch per decode step; launch-bound (the rows are a few hundred KB)"}
        del kc, vc
        torch.cuda.empty_cache()


def bench_sharded_decode(G, torch, dev, stream, flush_l2, peaks, args, world, max_over_ranks, barrier):
    """One decode step of a global layer over 8 sequences of 262,144 cached tokens (the 256K
    context), the history split over the job's ranks by key range: each rank decodes its
    range, the fp32 partials are all-gathered (NCCL) and combined on every rank. With one
    rank this is the plain decode over the whole context."""
    from global_interleaved_layers_b200.sharded import ShardedDecode, query_offsets
    layer = W.LayerSpec(W.GLOBAL, 32, 4, 512, rope_p=0.25, rope_base=1e6)
    B, n_q, L = 8, 1, 262144
    Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
    rank = int(os.environ.get("RANK", "0"))
    offs = query_offsets([L] * B, world, rank)
    shard = max(o[1] for o in offs)
    gen = torch.Generator(device=dev)
    gen.manual_seed(55 + rank)
    kc = torch.empty((B, Hkv, max(shard, 1), d), dtype=torch.bfloat16, device=dev).normal_(generator=gen)
    q = torch.randn((B, n_q, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
    nk = torch.randn((B, n_q, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
    lens = torch.tensor([o[1] for o in offs], dtype=torch.int32, device=dev)
    qoff = torch.tensor([o[2] for o in offs], dtype=torch.int32, device=dev)
    p = G.params(layer.kind, Hq, Hkv, d, rope_p=layer.rope_p, rope_base=layer.rope_base,
                 softmax_scale=layer.softmax_scale)
    splits = G.gemma_attn_decode_num_splits(p, B, n_q, shard)
    dec = ShardedDecode(p, B, n_q, splits, dev)
    out = torch.empty((B, n_q, Hq, d), dtype=torch.bfloat16, device=dev)

    def one():
        dec(q, nk, kc, kc.shape[2], lens, qoff, shard, out, None, stream)

    log("sharded decode")
    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    G.gemma_attn_check()
    barrier()
    evs = []
    for _ in range(args.steps):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    G.gemma_attn_check()
    barrier()
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])))
    total_bytes = W.decode_cache_bytes(B, [L] * B, layer)  # every rank's range, read once
    gbs = total_bytes / (ms * 1e-3) / 1e9
    res = {"gbs": gbs, "ms": ms, "bytes": total_bytes, "ranks": world, "splits_per_rank": splits,
           "frac_of_hbm_per_gpu": gbs / world / peaks["hbm_gbs"],
           "gathered_bytes_per_rank": splits * B * n_q * Hq * (d + 1) * 4 * world,
           "shape": f"B={B} n_q={n_q} Hq={Hq} Hkv={Hkv} d={d}, {L} cached tokens per sequence, "
                    f"split by key range over {world} rank(s); decode + all-gather + combine"}
    del kc, dec
    torch.cuda.empty_cache()
    return res


def bench_vision(G, torch, dev, stream, flush_l2, peaks, args, world, max_over_ranks, barrier):
    """The vision encoder's attention: bidirectional, 2D RoPE, 4 images of 2520 patches."""
    wl = W.vision_batch()
    layer = wl.layers[0]
    T = wl.total_tokens
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    q = torch.randn((T, layer.num_q_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    k = torch.randn((T, layer.num_kv_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((T, layer.num_kv_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty_like(q)
    # patches of each image row by row, 56 wide (45 x 56 = 2520)
    idx = np.concatenate([np.arange(n) for n in wl.seq_lens])
    hw = torch.from_numpy(np.stack([idx // 56, idx % 56], axis=1).astype(np.int32)).to(dev)
    cu = torch.from_numpy(wl.cu_seqlens()).to(dev)
    p = G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, rope_p=1.0,
                 rope_base=layer.rope_base, softmax_scale=layer.softmax_scale)
    ws_bytes = G.gemma_attn_prefill_workspace_size(p, T)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    maxlen = max(wl.seq_lens)

    def one():
        G.gemma_attn_prefill(p, q, k, v, out, None, hw, cu, len(wl.seq_lens), T, maxlen, ws, ws_bytes, stream)

    log("vision prefill")
    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    G.gemma_attn_check()
    evs = []
    barrier()
    for _ in range(args.steps):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    G.gemma_attn_check()
    barrier()
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])))
    flops = W.prefill_flops(wl.seq_lens, layer)
    tflops = flops / (ms * 1e-3) / 1e12
    return {"tflops": tflops, "ms": ms, "frac_of_peak": tflops / peaks["bf16_tflops"],
            "launches": 2, "shape": f"{len(wl.seq_lens)} images x {maxlen} patches, {layer.num_q_heads} heads, "
                                    f"d={layer.head_dim}, bidirectional, 2D RoPE (rotated copy + attention)"}


def run_case(args):
    """One operation of the hot path on its benchmark shape, for profiler captures."""
    import torch
    import global_interleaved_layers_b200 as G
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    if args.case == "vision_prefill":
        wl = W.vision_batch()
        layer = wl.layers[0]
        T = wl.total_tokens
        q = torch.randn((T, layer.num_q_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
        k = torch.randn((T, layer.num_kv_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
        v = torch.randn_like(k)
        out = torch.empty_like(q)
        idx = np.concatenate([np.arange(n) for n in wl.seq_lens])
        hw = torch.from_numpy(np.stack([idx // 56, idx % 56], axis=1).astype(np.int32)).to(dev)
        cu = torch.from_numpy(wl.cu_seqlens()).to(dev)
        p = G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, rope_p=1.0,
                     rope_base=layer.rope_base, softmax_scale=layer.softmax_scale)
        ws_bytes = G.gemma_attn_prefill_workspace_size(p, T)
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

        def op():
            G.gemma_attn_prefill(p, q, k, v, out, None, hw, cu, len(wl.seq_lens), T, max(wl.seq_lens), ws, ws_bytes,
                                 stream)
    elif "prefill" in args.case:
        wl = W.e2b_block()
        layer = wl.layers[-1] if args.case == "global_prefill" else wl.layers[0]
        if args.case == "local_prefill_31b":
            wl = W.b31_block()
            layer = wl.layers[0]
        if args.case == "global_prefill_31b_h8":
            # the 31B global layer's sequence length with a quarter of its heads (8 query heads,
            # one KV head): DRAM traffic per launch scales with the heads, for a capture that
            # stays small
            wl = W.PrefillWorkload(name="31b_global_h8", seq_lens=(32768,), seed=0,
                                   layers=(W.LayerSpec(W.GLOBAL, 8, 1, 512, rope_p=0.25, rope_base=1e6),))
            layer = wl.layers[0]
        L = wl.total_tokens
        q = torch.randn((L, layer.num_q_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
        k = torch.randn((L, layer.num_kv_heads, layer.head_dim), generator=gen, device=dev).to(torch.bfloat16)
        v = None if layer.k_eq_v else torch.randn_like(k)
        out = torch.empty_like(q)
        p = G.params(layer.kind, layer.num_q_heads, layer.num_kv_heads, layer.head_dim, window=layer.window,
                     rope_p=layer.rope_p, rope_base=layer.rope_base, softmax_scale=layer.softmax_scale)
        ws_bytes = G.gemma_attn_prefill_workspace_size(p, L)
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        pos = torch.from_numpy(wl.positions()).to(dev)
        cu = torch.from_numpy(wl.cu_seqlens()).to(dev)

        def op():
            G.gemma_attn_prefill(p, q, k, v, out, None, pos, cu, 1, L, L, ws, ws_bytes, stream)
    elif args.case == "global_verify":
        _, ver = W.ragged_31b()
        layer = ver.layers[0]
        B, n_q = ver.batch, ver.n_q
        Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
        cap = max(ver.cache_lens)
        kc = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev).normal_(generator=gen)
        q = torch.randn((B, n_q, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
        nk = torch.randn((B, n_q, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        lens = torch.tensor(list(ver.cache_lens), dtype=torch.int32, device=dev)
        p = G.params(layer.kind, Hq, Hkv, d, rope_p=layer.rope_p, rope_base=layer.rope_base,
                     softmax_scale=layer.softmax_scale)
        splits = G.gemma_attn_decode_num_splits(p, B, n_q, cap)
        rows = B * n_q * Hq
        po = torch.empty((splits, rows, d), dtype=torch.float32, device=dev)
        pl = torch.empty((splits, rows), dtype=torch.float32, device=dev)
        out = torch.empty((B, n_q, Hq, d), dtype=torch.bfloat16, device=dev)

        def op():
            G.gemma_attn_decode(p, q, nk, None, kc, None, G.CACHE_CONTIGUOUS, cap, lens, B, n_q, cap, po, pl, splits,
                                stream)
            G.gemma_attn_combine(po, pl, splits, rows, d, G.OUT_BF16, out, None, stream)
    else:
        wl = W.long_decode()
        layer = wl.layers[0] if args.case == "global_decode" else wl.layers[1]
        B, n_q, ctx = wl.batch, wl.n_q, (args.ctx or wl.cache_lens[0])
        Hq, Hkv, d = layer.num_q_heads, layer.num_kv_heads, layer.head_dim
        cap = ctx if layer.k_eq_v else layer.window
        # local: the serving layout with keys stored rotated (what per_kind.local_decode times)
        layout = G.CACHE_CONTIGUOUS if layer.k_eq_v else (G.CACHE_RING | G.CACHE_KEYS_ROTATED)
        kc = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev).normal_(generator=gen)
        vc = None if layer.k_eq_v else torch.empty_like(kc).normal_(generator=gen)
        q = torch.randn((B, n_q, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
        nk = torch.randn((B, n_q, Hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        nv = None if layer.k_eq_v else torch.randn_like(nk)
        lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        p = G.params(layer.kind, Hq, Hkv, d, window=layer.window, rope_p=layer.rope_p, rope_base=layer.rope_base,
                     softmax_scale=layer.softmax_scale)
        splits = G.gemma_attn_decode_num_splits(p, B, n_q, ctx)
        rows = B * n_q * Hq
        po = torch.empty((splits, rows, d), dtype=torch.float32, device=dev)
        pl = torch.empty((splits, rows), dtype=torch.float32, device=dev)
        out = torch.empty((B, n_q, Hq, d), dtype=torch.bfloat16, device=dev)

        def op():
            if splits == 1:
                G.gemma_attn_decode_noalloc(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, ctx, 1, out, None,
                                            stream)
            else:
                G.gemma_attn_decode(p, q, nk, nv, kc, vc, layout, cap, lens, B, n_q, ctx, po, pl, splits, stream)
                G.gemma_attn_combine(po, pl, splits, rows, d, G.OUT_BF16, out, None, stream)
    for _ in range(args.warmup + args.steps):
        op()
    torch.cuda.synchronize()
    G.gemma_attn_check()
    print(json.dumps({"case": args.case, "launches": args.warmup + args.steps}), flush=True)


if __name__ == "__main__":
    main()
