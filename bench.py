#!/usr/bin/env python
"""Benchmark of the TurboQuant hot path on B200 (one process per GPU).

Workloads (`--config`), all seeded synthetic data of the shapes and distributions below:

  ragged   (default) ragged batched serving decode: batch 64, context lengths uniform in
           [1024, 32768] stored in 16-token paged blocks behind a shuffled block table, 32 query /
           8 KV heads, head_dim 128, bf16 K/V drawn N(0,1) x lognormal(0,1) per (KV head,
           channel); K 2 Lloyd-Max bits + QJL (m = 128), V 3 bits.  About 8.6 M (token, KV head)
           pairs, 0.93 GB of packed K+V per step.
  llama8b  Llama-3.1-8B-shaped decode layer: batch 1, context 32768, same heads and
           distribution, K `--kbits` (3: 2+QJL, 4: 3+QJL), V 3 bits; 48 layer caches cycled.
  longctx  long-context prefill + decode: batch 4, 8 KV heads (32 q), context 131072, K 3+QJL,
           V 2 bits: the whole prefill is encoded (timed as encode vectors/s), then 64 decode steps
           that each append one token per (sequence, KV head) and attend over the grown cache.
  search   10^6 unit vectors d 1024, 1000 unit queries, top-10, `--search-bits` 2 or 4 per
           coordinate (1 or 3 MSE bits + QJL m 1024): database encode and search.

A decode step appends the new token's K and V of every (sequence, KV head) to the compressed
cache and attends (`tq_decode_step`: one append/query-preparation launch and one attention launch).
`value` = decode keys scored per second over all ranks, a key being one (token, KV head) pair
scored against its 4 query heads.  The default run's single JSON line also carries, under
"encode", the bulk encode of the workload's cache, under "sparse_v", the same steps with value rows
below a 1e-6 softmax weight skipped (also with the queries scaled by 2 and 4, which sharpens the
softmax as a peaked long-context attention would), and, under "search", the search workload at 2 and
4 bits (each with its own roofline), so one run measures every half of the path.

Multi-GPU runs are weak scaling: every rank runs its own copy of the workload (independent
problems, no data-path collective); times are the max over ranks of device time.
`--impl reference` times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload and prints the same kind of line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config ragged|llama8b|longctx|search] [--kbits 3|4] [--search-bits 2|4]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CONFIGS = {
    "ragged": dict(name="ragged paged serving decode", batch=64, n_q_heads=32, n_kv_heads=8, d=128,
                   len_lo=1024, len_hi=32768, paged=True, k_bits=3, v_bits=3, qjl_m=128, caches=2),
    "llama8b": dict(name="llama3.1-8b decode layer", batch=1, n_q_heads=32, n_kv_heads=8, d=128, ctx=32768,
                    paged=False, k_bits=3, v_bits=3, qjl_m=128, caches=48),
    "longctx": dict(name="long-context prefill + decode", batch=4, n_q_heads=32, n_kv_heads=8, d=128,
                    ctx=131072, paged=False, k_bits=4, v_bits=2, qjl_m=128, caches=1, append_steps=64),
}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BLOCK = 16
DTYPE_DECODE = ("int8 tensor-core limbs: 32-bit fixed-point query terms x 0/1 key bit planes, 16-bit "
                "fixed-point value weights; fp32 softmax and accumulation")
# DRAM bytes (read + write) per launch of the attention kernel, from one ncu capture (one pass,
# `dram__bytes_read.sum` + `dram__bytes_write.sum`) of the kernel revision named in the library's
# version string, on the workload named; null for any other revision or workload
NCU_TRAFFIC = {
    ("attend_mma", "r14", "ragged"): 949.94e6 + 13.79e6,
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=["ragged", "llama8b", "longctx", "search"], default=None)
    ap.add_argument("--workload", choices=["decode", "search"], default=None,
                    help="older spelling: decode = --config llama8b, search = --config search")
    ap.add_argument("--kbits", type=int, choices=[3, 4], default=None,
                    help="llama8b: K bits per coordinate, (kbits-1) MSE bits + 1 QJL bit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default run: skip the encode and search sub-measurements")
    ap.add_argument("--cpu-sample-seconds", type=float, default=20.0)
    ap.add_argument("--search-bits", type=int, choices=[2, 4], default=2,
                    help="search: bits per coordinate, (bits-1) MSE bits + 1 QJL bit with m = d")
    ap.add_argument("--search-rows", type=int, default=1_000_000,
                    help="search: database rows (the workload is 10^6; smaller only for profiler captures)")
    ap.add_argument("--batch", type=int, default=None,
                    help="ragged: number of sequences (the workload is 64; smaller only for profiler captures)")
    ap.add_argument("--sparse-v", type=float, default=0.0,
                    help="decode: Sparse V threshold on the softmax weight (0 = off)")
    a = ap.parse_args(argv)
    if a.config is None:
        a.config = {"decode": "llama8b", "search": "search"}.get(a.workload, "ragged")
    return a


def workload(args) -> dict:
    cfg = dict(CONFIGS[args.config])
    if args.config == "llama8b" and args.kbits is not None:
        cfg["k_bits"] = args.kbits
    if args.config == "ragged" and args.batch is not None:
        cfg["batch"] = args.batch
    return cfg


def packed_bytes_per_key(d, mse_bits, m):
    code = (mse_bits * d // 8 + 15) // 16 * 16
    sign = (m // 8 + 15) // 16 * 16 if m > 0 else 0
    return code + sign + 4 + (4 if m > 0 else 0)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def recorded_traffic(kernel: str, config: str):
    from kv_cache_vector_06_b200 import tq
    ver = tq.version()
    for (name, rev, cfg), val in NCU_TRAFFIC.items():
        if name == kernel and cfg == config and f"{name} {rev}" in ver:
            return val
    return None


# ------------------------------------------------------------------------------ clocks (NVML)
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_r(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if self.nv is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------------------ distributed
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes units_per_step per step, and
    ms is the slowest rank's time for `steps` steps."""
    return world * units_per_step * steps / (ms / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


# ------------------------------------------------------------------------------ our arm: decode
def ragged_layout(cfg, seed: int):
    """Context lengths and one shuffled block table of the ragged workload (synth recipe)."""
    import synth
    lens = synth.ragged_lengths(cfg["batch"], cfg["len_lo"], cfg["len_hi"], seed=seed)
    table, nblocks = synth.shuffled_block_table(lens, seed=seed + 1)
    return lens, table, nblocks


def cache_block_table(lens, seed: int, ci: int):
    """Block table of cache `ci` of a paged workload: the same lengths as every other cache (so
    every step does the same work), another permutation of the physical blocks."""
    import synth
    tab, _ = synth.shuffled_block_table(lens, seed=seed + 1 + 17 * ci)
    return tab


class DecodeBench:
    """Device-resident compressed caches of one decode workload plus the per-step inputs.

    The caches are drawn on the device with a seeded generator (the synth recipe's distribution:
    N(0,1) x lognormal(0,1) per (KV head, channel), rounded to bf16) and encoded by the library;
    the first cache's encode is timed (`encode_timing`)."""

    def __init__(self, cfg: dict, rank: int, sparse_v: float = 0.0):
        import torch

        import synth
        from kv_cache_vector_06_b200 import tq
        self.tq, self.cfg = tq, cfg
        d, hq, hkv, B = cfg["d"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["batch"]
        self.d, self.hq, self.hkv, self.batch = d, hq, hkv, B
        self.kmse, self.m, self.vbits = cfg["k_bits"] - 1, cfg["qjl_m"], cfg["v_bits"]
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev = dev
        seed = 1000 * rank
        self.kctx = tq.Context(d, self.kmse, self.m, synth.rotation_signs(d, seed + 1),
                               synth.qjl_matrix(self.m, d, seed + 2), device=dev.index)
        self.vctx = tq.Context(d, self.vbits, 0, synth.rotation_signs(d, seed + 3), device=dev.index,
                               layout=tq.LAYOUT_BLOCK16)
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        self.sparse_v = sparse_v
        self.paged = cfg["paged"]
        self.append_steps = cfg.get("append_steps", 0)
        if self.paged:
            lens, _, nblocks = ragged_layout(cfg, 1102 + seed)
            self.lens = lens
            cap = nblocks * hkv * BLOCK
            self.max_len = int(lens.max())
            self.stride = None
        else:
            ctx = cfg["ctx"]
            self.stride = (ctx + self.append_steps + BLOCK - 1) // BLOCK * BLOCK
            self.lens = torch.full((B,), ctx, dtype=torch.int32)
            cap = B * hkv * self.stride
            self.max_len = ctx + self.append_steps
        self.cap = cap
        self.caches = []
        self.encode_timing = None
        for ci in range(cfg["caches"]):
            kp = tq.Packed.allocate(self.kctx, cap)
            vp = tq.Packed.allocate(self.vctx, cap)
            xs = []
            for role in range(2):
                scale = torch.exp(torch.randn(hkv, d, generator=g, device=dev))
                x = torch.empty(cap, d, dtype=torch.bfloat16, device=dev)
                ch = 1 << 20
                for r0 in range(0, cap, ch):
                    r1 = min(cap, r0 + ch)
                    idx = torch.arange(r0, r1, device=dev)
                    head = (idx // BLOCK) % hkv if self.paged else (idx // self.stride) % hkv
                    x[r0:r1] = (torch.randn(r1 - r0, d, generator=g, device=dev) * scale[head]).to(torch.bfloat16)
                xs.append(x)
            if ci == 0:
                self.encode_timing = self._time_encode(xs[0], xs[1], kp, vp)
            else:
                ws = torch.empty(tq.encode_workspace_size(self.kctx, cap), dtype=torch.uint8, device=dev)
                tq.encode_kv(self.kctx, xs[0], kp, ws=ws)
                tq.encode_kv(self.vctx, xs[1], vp, ws=ws)
                del ws
            del xs
            table = None
            if self.paged:
                table = cache_block_table(self.lens, 1102 + seed, ci).to(dev)
            self.caches.append((kp, vp, table))
        torch.cuda.synchronize()
        # per-step inputs: the queries and the new token's K/V of every (sequence, KV head)
        self.q = torch.randn(B, hq, d, generator=g, device=dev).to(torch.bfloat16)
        self.k_new = torch.randn(B * hkv, d, generator=g, device=dev).to(torch.bfloat16)
        self.v_new = torch.randn(B * hkv, d, generator=g, device=dev).to(torch.bfloat16)
        self.out = torch.empty(B, hq, d, dtype=torch.float32, device=dev)
        # steps: (cache index, seq_lens, slots of the appended rows); the ragged and llama8b steps
        # rewrite each sequence's last token, the long-context steps append at ctx + t
        self.steps = []
        nsteps = self.append_steps if self.append_steps else 1
        for ci, (kp, vp, table) in enumerate(self.caches):
            for t in range(nsteps):
                L = self.lens + (t + 1 if self.append_steps else 0)
                sl = []
                for b in range(B):
                    pos = int(L[b]) - 1
                    for h in range(hkv):
                        if self.paged:
                            blk = int(table[b, pos // BLOCK])
                            sl.append((blk * hkv + h) * BLOCK + pos % BLOCK)
                        else:
                            sl.append((b * hkv + h) * self.stride + pos)
                lens_dev = L.to(torch.int32).to(dev)
                slots = torch.tensor(sl, dtype=torch.int64, device=dev)
                desc = tq.make_attn_desc(self.kctx, self.vctx, (B, hq, d), kp, vp, lens_dev, self.max_len,
                                         ctx_stride=self.stride, block_table=table, n_kv_heads=hkv)
                self.steps.append((desc, lens_dev, slots, int(L.sum())))
        self.ws_step = torch.empty(tq.decode_step_workspace_size(self.kctx, self.vctx, self.steps[0][0], B * hkv),
                                   dtype=torch.uint8, device=dev)
        self.kv_bytes = packed_bytes_per_key(d, self.kmse, self.m) + packed_bytes_per_key(d, self.vbits, 0)
        # units: (token, KV head) pairs scored per step, averaged over the step cycle
        self.keys_per_step = hkv * sum(s[3] for s in self.steps) / len(self.steps)
        self.bytes_per_step = self.keys_per_step * self.kv_bytes

    def _time_encode(self, xk, xv, kp, vp, reps=3):
        """Bulk encode of the cache's K and V rows (the prefill encode): vectors/s and its HBM
        roofline (bf16 rows in, packed bytes out)."""
        import torch
        tq = self.tq
        n = xk.shape[0]
        ws = torch.empty(tq.encode_workspace_size(self.kctx, n), dtype=torch.uint8, device=self.dev)
        tq.encode_kv(self.kctx, xk, kp, ws=ws)
        tq.encode_kv(self.vctx, xv, vp, ws=ws)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(reps):
            tq.encode_kv(self.kctx, xk, kp, ws=ws)
            tq.encode_kv(self.vctx, xv, vp, ws=ws)
        end.record()
        torch.cuda.synchronize()
        ms = start.elapsed_time(end) / reps
        # per-kernel device times of one more encode, on the launching stream
        torch.cuda.synchronize()
        tq.profile_reset()
        tq.profile_enable(True)
        try:
            tq.encode_kv(self.kctx, xk, kp, ws=ws)
            tq.encode_kv(self.vctx, xv, vp, ws=ws)
            torch.cuda.synchronize()
        finally:
            tq.profile_enable(False)
        prof = {k: v for k, v in tq.profile_read().items() if v[0] > 0}
        tq.profile_reset()
        del ws
        kb = packed_bytes_per_key(self.d, self.kmse, self.m)
        vb = packed_bytes_per_key(self.d, self.vbits, 0)
        return {"n_vectors": 2 * n, "ms": ms, "bytes": n * (2 * 2 * self.d + kb + vb),
                "flop": 2.0 * self.m * self.d * n, "kernels": prof}

    def set_sparse_v(self, tau: float):
        """Sparse V threshold of every step's descriptor (0 = off)."""
        for desc, _, _, _ in self.steps:
            desc.sparse_v = tau

    def step(self, i: int, q=None, out=None, k_new=None, v_new=None):
        desc, _, slots, _ = self.steps[i % len(self.steps)]
        self.tq.decode_step(self.kctx, self.vctx, self.q if q is None else q,
                            self.k_new if k_new is None else k_new, self.v_new if v_new is None else v_new,
                            slots, desc, out=self.out if out is None else out, ws=self.ws_step)

    def capture_graphs(self):
        import torch
        graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(len(self.steps)):  # warm every step once outside capture
                self.step(i)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for i in range(len(self.steps)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(i)
            graphs.append(g)
        torch.cuda.synchronize()
        return graphs


def time_graph_steps(graphs, steps, warmup, world, sampler=None):
    import torch
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        start.record()
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)


def profile_kernels(bench, steps):
    """Per-kernel device times from the library's CUDA events on the kernels' own stream (eager
    steps).  A spin kernel first keeps the device busy while the host queues all the steps, so
    the device runs them back to back and no host launch gap falls between an event and its
    kernel."""
    import torch
    tq = bench.tq
    torch.cuda.synchronize()
    tq.profile_reset()
    tq.profile_enable(True)
    try:
        torch.cuda._sleep(20_000_000)  # about 10 ms of device time
        for i in range(steps):
            bench.step(i)
        torch.cuda.synchronize()
    finally:
        tq.profile_enable(False)
    prof = tq.profile_read()
    tq.profile_reset()
    return {k: v for k, v in prof.items() if v[0] > 0}


def time_e2e(bench, steps, warmup):
    """End to end through the public API with host buffers.  Per step: one H2D copy of the step's
    inputs (the query and the new token's K and V, packed in one pinned buffer; the library reads
    views of the one device buffer), append + attention, and a D2H copy of the output.  The output
    of step i is read back on a second stream while step i + 1 runs (two output buffers, so a
    buffer is written again only after its read-back); the timed region ends when the last
    read-back has landed."""
    import torch
    srcs = [bench.q, bench.k_new, bench.v_new]
    sizes = [t.numel() * t.element_size() for t in srcs]
    offs = [0]
    for sz in sizes[:-1]:
        offs.append((offs[-1] + sz + 255) // 256 * 256)
    total = offs[-1] + sizes[-1]
    h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o, sz in zip(srcs, offs, sizes):
        h_in[o:o + sz].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
    d_in = torch.empty(total, dtype=torch.uint8, device=bench.q.device)
    d_q, d_k, d_v = (d_in[o:o + sz].view(t.dtype).view(t.shape) for t, o, sz in zip(srcs, offs, sizes))
    d_out = [torch.empty_like(bench.out) for _ in range(2)]
    h_out = [torch.empty(bench.out.shape, dtype=bench.out.dtype).pin_memory() for _ in range(2)]
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    computed = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        b = i % 2
        main.wait_event(read[b])  # the previous read-back of this output buffer has landed
        d_in.copy_(h_in, non_blocking=True)
        bench.step(i, q=d_q, out=d_out[b], k_new=d_k, v_new=d_v)
        computed[b].record(main)
        side.wait_event(computed[b])
        with torch.cuda.stream(side):
            h_out[b].copy_(d_out[b], non_blocking=True)
        read[b].record(side)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(main)
    for i in range(steps):
        one(i)
    main.wait_stream(side)
    end.record(main)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    return ms, total, h_out[0].numel() * h_out[0].element_size()


def decode_config(args, cfg, bench=None) -> dict:
    kb, vb = cfg["k_bits"], cfg["v_bits"]
    shape = (f"batch {cfg['batch']}, {cfg['n_q_heads']} q / {cfg['n_kv_heads']} kv heads, head_dim {cfg['d']}, "
             f"K {kb - 1}+QJL(m={cfg['qjl_m']}) bits, V {vb} bits")
    if cfg["paged"]:
        ctx = f"context lengths U[{cfg['len_lo']}, {cfg['len_hi']}] in {BLOCK}-token paged blocks, shuffled block table"
    else:
        ctx = f"context {cfg['ctx']}" + (f" + {cfg['append_steps']} appended decode steps" if cfg.get("append_steps") else "")
    out = {"workload": f"{cfg['name']}: {shape}, {ctx}; step = append-encode one token per (sequence, KV head) "
                       f"+ decode attention",
           "batch": cfg["batch"], "n_q_heads": cfg["n_q_heads"], "n_kv_heads": cfg["n_kv_heads"],
           "head_dim": cfg["d"], "k_bits": kb, "v_bits": vb, "qjl_m": cfg["qjl_m"],
           "parallelism": "independent workload copy per GPU (weak scaling)"}
    if cfg["paged"]:
        out.update(context_min=cfg["len_lo"], context_max=cfg["len_hi"], block_tokens=BLOCK)
    else:
        out["context"] = cfg["ctx"]
    if bench is not None:
        out["keys_per_step"] = bench.keys_per_step
        out["packed_bytes_per_step"] = bench.bytes_per_step
        out["l2"] = ("inputs larger than L2: %.0f MB of packed K+V per step, %d distinct cache%s cycled"
                     % (bench.bytes_per_step / 1e6, len(bench.caches), "s" if len(bench.caches) > 1 else ""))
    if args.sparse_v > 0:
        out["sparse_v_threshold"] = args.sparse_v
    return out


def encode_summary(timing: dict, peaks: dict, src: str, d: int) -> dict:
    ms = timing["ms"]
    gbs = timing["bytes"] / (ms / 1e3) / 1e9
    tfl = timing["flop"] / (ms / 1e3) / 1e12
    return {"metric": "encode vectors/s", "value": timing["n_vectors"] / (ms / 1e3), "unit": "vectors/s",
            "ms": ms, "n_vectors": timing["n_vectors"],
            "workload": f"bulk encode of the cache: {timing['n_vectors'] // 2} K + {timing['n_vectors'] // 2} V "
                        f"bf16 rows, d {d}",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "note": "bf16 rows in + packed codes, signs and norms out per call, all encode "
                                 "kernels together; peak = %s burst copy" % src},
            "projection_tflops": tfl,
            "kernels": {k: {"launches": n, "ms": t} for k, (n, t) in timing["kernels"].items()}}


def ours_decode(args, world, rank):
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py --impl ours needs a CUDA device (there is no CPU fallback)")
    cfg = workload(args)
    bench = DecodeBench(cfg, rank, args.sparse_v)
    graphs = bench.capture_graphs()
    sampler = ClockSampler(torch.cuda.current_device())
    ms = time_graph_steps(graphs, args.steps, args.warmup, world, sampler)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = aggregate_rate(world, bench.keys_per_step, args.steps, ms)
    hbm_gbs = aggregate_rate(world, bench.bytes_per_step, args.steps, ms) / 1e9

    prof_steps = max(len(bench.steps), min(args.steps, 48))
    prof = profile_kernels(bench, prof_steps)
    launches_per_step = sum(n for n, _ in prof.values()) / prof_steps
    split_n, split_ms = prof.get("attend_split", (0, 0.0))  # the attention kernel
    peaks, src = measured_peaks()
    roof = None
    if split_n:
        per_launch_s = split_ms / split_n / 1e3
        achieved = bench.bytes_per_step / per_launch_s / 1e9
        roof = {"kernel": "attend_mma_kernel (tensor cores, streamed sub-chunks, fused split merge)", "bound": "hbm",
                "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic("attend_mma", args.config if args.batch is None else None),
                "peak_source": src + " (burst copy)", "us_per_launch": per_launch_s * 1e6,
                "algorithmic_bytes_per_launch": bench.bytes_per_step,
                "bytes_per_unit": bench.kv_bytes, "units_per_launch": bench.keys_per_step}
    kernel_share = {k: {"launches_per_step": n / prof_steps, "us_per_launch": 1e3 * t / n}
                    for k, (n, t) in prof.items()}

    e2e_steps = min(args.steps, 200)
    e_ms, h2d, d2h = time_e2e(bench, e2e_steps, min(args.warmup, 10))
    e_ms = max_over_ranks(e_ms, world)
    e2e_value = aggregate_rate(world, bench.keys_per_step, e2e_steps, e_ms)
    # Sparse V ("TurboQuant+ 深度解析" 第六部分) on the same steps: value rows whose softmax weight is
    # below 1e-6 are skipped; reported beside the plain step (the headline keeps every row)
    sparse = None
    if args.sparse_v == 0:
        tau = 1e-6

        def timed_ms(threshold):
            bench.set_sparse_v(threshold)
            g = bench.capture_graphs()
            t = max_over_ranks(time_graph_steps(g, args.steps, args.warmup, world), world)
            bench.set_sparse_v(0.0)
            del g
            return t

        s_ms = timed_ms(tau)
        sparse = {"threshold": tau, "ms_per_step": s_ms / args.steps,
                  "value": aggregate_rate(world, bench.keys_per_step, args.steps, s_ms), "unit": "keys/s",
                  "speedup_vs_all_rows": ms / s_ms, "peaked": []}
        # Peaked attention on the same caches: the queries scaled by a power of two (exact), so the
        # logits spread (their spread grows with the scale) and most rows of a long context fall below
        # the threshold; both steps are timed on the scaled queries, which are restored afterwards
        for scale in (2.0, 4.0):
            bench.q.mul_(scale)
            try:
                p_ms, ps_ms = timed_ms(0.0), timed_ms(tau)
            finally:
                bench.q.div_(scale)
            sparse["peaked"].append({"query_scale": scale, "ms_per_step_all_rows": p_ms / args.steps,
                                     "ms_per_step_sparse_v": ps_ms / args.steps, "speedup": p_ms / ps_ms})
    enc = encode_summary(bench.encode_timing, peaks, src, bench.d)
    enc_ms = max_over_ranks(enc["ms"], world)
    enc["value"] = world * bench.encode_timing["n_vectors"] / (enc_ms / 1e3)
    line = {
        "metric": "decode keys scored/s", "value": value, "unit": "keys/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_DECODE, "data": "synthetic",
        "config": decode_config(args, cfg, bench),
        "hbm_gbs": hbm_gbs, "hbm_frac_of_peak": hbm_gbs / (world * peaks["hbm_gbs"]), "peak_source": src,
        "roofline": roof,
        "kernels": kernel_share,
        "e2e": {"value": e2e_value, "unit": "keys/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "note": "eager tq.decode_step calls; per step one H2D of the packed inputs from pinned memory "
                        "and a D2H of the output, read back on a second stream during the next step"},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": sampler.summary(),
        "encode": enc,
        "sparse_v": sparse,
    }
    del graphs
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(cfg, args.cpu_sample_seconds)
        line["cpu_baseline"] = cpu
    del bench
    torch.cuda.empty_cache()
    if args.config == "ragged" and not args.no_extras:
        line["search"] = {}
        for bits in (2, 4):
            line["search"][f"{bits}bit"] = run_search(args, bits, world, rank, cpu_baseline=(cpu is not None))
            torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------ our arm: search
def run_search(args, bits: int, world=1, rank=0, cpu_baseline=True) -> dict:
    """Vector search at 10^6 rows x d 1024: encode the database (unit vectors, fp32), then top-10
    for 1000 queries.  Inputs are drawn on the device with a seeded generator (same recipe as the
    parity tests: N(0, I) rows L2-normalised).  Under torchrun every rank searches its own
    database (weak scaling); times are the slowest rank's."""
    import torch
    from kv_cache_vector_06_b200 import tq
    import synth
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py --config search needs a CUDA device (there is no CPU fallback)")
    d, n, nq, k = 1024, args.search_rows, 1000, 10
    mse, m = bits - 1, d
    dev = torch.device("cuda", torch.cuda.current_device())
    ctx = tq.Context(d, mse, m, synth.rotation_signs(d, 11), synth.qjl_matrix(m, d, 12), device=dev.index)
    g = torch.Generator(device=dev)
    g.manual_seed(13 + rank)
    X = torch.randn(n, d, generator=g, device=dev)
    X /= X.norm(dim=1, keepdim=True)
    Q = torch.randn(nq, d, generator=g, device=dev)
    Q /= Q.norm(dim=1, keepdim=True)
    db = tq.Packed.allocate(ctx, n)
    ws_e = torch.empty(tq.encode_workspace_size(ctx, n), dtype=torch.uint8, device=dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tq.encode_kv(ctx, X, db, ws=ws_e)  # warm-up
    torch.cuda.synchronize()
    reps = max(1, min(args.steps, 5))
    barrier(world)
    start.record()
    for _ in range(reps):
        tq.encode_kv(ctx, X, db, ws=ws_e)
    end.record()
    torch.cuda.synchronize()
    enc_ms = max_over_ranks(start.elapsed_time(end), world) / reps
    tq.profile_reset()
    tq.profile_enable(True)
    try:
        tq.encode_kv(ctx, X, db, ws=ws_e)
        torch.cuda.synchronize()
    finally:
        tq.profile_enable(False)
    enc_prof = {k: v for k, v in tq.profile_read().items() if v[0] > 0}
    tq.profile_reset()
    del X, ws_e
    row_bytes = packed_bytes_per_key(d, mse, m)
    ws_s = torch.empty(tq.search_workspace_size(ctx, nq, n, k), dtype=torch.uint8, device=dev)
    sc = torch.empty(nq, k, dtype=torch.float32, device=dev)
    ix = torch.empty(nq, k, dtype=torch.int64, device=dev)
    for _ in range(max(1, min(args.warmup, 3))):
        tq.search_topk(ctx, Q, db, k, out_scores=sc, out_idx=ix, ws=ws_s)
    torch.cuda.synchronize()
    barrier(world)
    sampler = ClockSampler(dev.index)
    with sampler:
        start.record()
        for _ in range(reps):
            tq.search_topk(ctx, Q, db, k, out_scores=sc, out_idx=ix, ws=ws_s)
        end.record()
        torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), world) / reps
    tq.profile_reset()
    tq.profile_enable(True)
    try:
        tq.search_topk(ctx, Q, db, k, out_scores=sc, out_idx=ix, ws=ws_s)
        torch.cuda.synchronize()
    finally:
        tq.profile_enable(False)
    scan_prof = {k2: v for k2, v in tq.profile_read().items() if v[0] > 0}
    tq.profile_reset()
    # end to end through the API: each call's queries from pinned host memory, its top-k back to
    # pinned host memory
    h_q = Q.cpu().pin_memory()
    h_s = torch.empty(nq, k, dtype=torch.float32).pin_memory()
    h_i = torch.empty(nq, k, dtype=torch.int64).pin_memory()
    d_q = torch.empty_like(Q)
    torch.cuda.synchronize()
    barrier(world)
    start.record()
    for _ in range(reps):
        d_q.copy_(h_q, non_blocking=True)
        tq.search_topk(ctx, d_q, db, k, out_scores=sc, out_idx=ix, ws=ws_s)
        h_s.copy_(sc, non_blocking=True)
        h_i.copy_(ix, non_blocking=True)
    end.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(start.elapsed_time(end), world) / reps
    peaks, src = measured_peaks()
    db_bytes = n * row_bytes
    # the method's own work per (query, row): the codebook dot over d coordinates and the sign
    # correction over m projected coordinates, one multiply-add each (2 (d + m) ops), against the
    # measured bf16 peak x 2 (the dense int8:bf16 ratio of the tensor cores the scan runs on)
    method_ops = 2.0 * (d + m) * nq * n
    int8_peak = peaks["bf16_tflops"] * 2
    scan_n, scan_ms = scan_prof.get("search_scan", (0, 0.0))
    scan_s = scan_ms / scan_n / 1e3 if scan_n else ms / 1e3
    enc_flop = 3 * 2.0 * m * d * n
    out = {
        "metric": "search queries/s", "value": aggregate_rate(world, nq, 1, ms), "unit": "queries/s",
        "n_gpus": world, "steps": reps, "warmup": max(1, min(args.warmup, 3)), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 tensor-core limbs (24-bit fixed-point query terms x 0/1 row bit planes), fp32 combine",
        "data": "synthetic",
        "config": search_config(bits, n, db_bytes),
        "scores_per_s": nq * n / (ms / 1e3),
        "database_passes_per_s": 1e3 / ms,
        "hbm": {"database_bytes": db_bytes, "gbs_one_read_per_query": nq * db_bytes / (ms / 1e3) / 1e9,
                "peak": peaks["hbm_gbs"], "peak_source": src},
        "encode": {"metric": "encode vectors/s", "value": n / (enc_ms / 1e3), "unit": "vectors/s", "ms": enc_ms,
                   "gbs": n * (4 * d + row_bytes) / (enc_ms / 1e3) / 1e9,
                   "roofline": {"bound": "tensor", "achieved": enc_flop / (enc_ms / 1e3) / 1e12,
                                "peak": peaks["bf16_tflops"] / 2, "unit": "TFLOP/s",
                                "frac": enc_flop / (enc_ms / 1e3) / 1e12 / (peaks["bf16_tflops"] / 2),
                                "traffic": None,
                                "note": "QJL projection S r as 3 TF32 tensor-core passes (2 m d flops each) per "
                                        "vector; peak = measured bf16 x 1/2 (the dense tf32:bf16 ratio), %s" % src},
                   "kernels": {k2: {"launches": a, "ms": b} for k2, (a, b) in enc_prof.items()}},
        "roofline": {"kernel": "search scan (bit-plane tensor-core MMAs)", "bound": "tensor",
                     "achieved": method_ops / scan_s / 1e12, "peak": int8_peak, "unit": "TOP/s",
                     "frac": method_ops / scan_s / 1e12 / int8_peak, "traffic": None,
                     "us_per_launch": scan_s * 1e6,
                     "note": "the method's ops, 2 (d + m) per (query, row), over the scan kernel's own time; "
                             "peak = measured bf16 x 2 (dense int8:bf16 ratio), %s" % src},
        "kernels": {k2: {"launches": a, "ms": b} for k2, (a, b) in scan_prof.items()},
        "e2e": {"value": aggregate_rate(world, nq, 1, e_ms), "unit": "queries/s",
                "h2d_bytes_per_step": h_q.numel() * h_q.element_size(),
                "d2h_bytes_per_step": h_s.numel() * 4 + h_i.numel() * 8},
        "gpu_launches": int(sum(a for a, _ in scan_prof.values())) * reps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and cpu_baseline:
        out["cpu_baseline"] = search_cpu_baseline(ctx_d=d, mse=mse, m=m, row_count=n)
    del db, ws_s
    return out


def ours_search(args, world, rank):
    line = run_search(args, args.search_bits, world, rank, cpu_baseline=not args.no_cpu_baseline)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def search_config(bits: int, n: int, db_bytes: int) -> dict:
    mse = bits - 1
    return {"workload": f"vector search: {'10^6' if n == 1_000_000 else n} unit vectors d 1024, "
                        f"{bits} bits/coord ({mse} MSE + QJL m 1024), 1000 queries, top-10",
            "rows": n, "d": 1024, "queries": 1000, "k": 10,
            "l2": "database (%.0f MB packed) %s than the 126 MB L2" % (
                db_bytes / 1e6, "larger" if db_bytes > 126e6 else "smaller")}


# ------------------------------------------------------------------------------ oracle (CPU) arm
class OracleDecode:
    """The fp64 oracle on one KV-head group (4 query heads) of a decode workload (host cores)."""

    def __init__(self, cfg: dict, ctx_tokens: int, seed: int = 0):
        import numpy as np

        import synth
        from oracle import attention as oattn
        from oracle import codebook as ocb
        from oracle import encode as oenc
        d, m = cfg["d"], cfg["qjl_m"]
        self.np, self.oattn, self.oenc = np, oattn, oenc
        self.d, self.G = d, cfg["n_q_heads"] // cfg["n_kv_heads"]
        self.L = ctx_tokens
        self.Dk = synth.rotation_signs(d, seed + 1).double().numpy()
        self.Sk = synth.qjl_matrix(m, d, seed + 2).double().numpy()
        self.Dv = synth.rotation_signs(d, seed + 3).double().numpy()
        self.ck, self.tk = ocb.codebook(d, cfg["k_bits"] - 1)
        self.cv, self.tv = ocb.codebook(d, cfg["v_bits"])
        K = synth.channel_scaled(1, 1, ctx_tokens, d, seed=seed + 4)[0, 0].double().numpy()
        V = synth.channel_scaled(1, 1, ctx_tokens, d, seed=seed + 5)[0, 0].double().numpy()
        ek = oenc.encode(K, self.Dk, self.Sk, self.ck, self.tk)
        ev = oenc.encode(V, self.Dv, np.zeros((0, d)), self.cv, self.tv)
        self.kc = oattn.Cache(norm=ek.norm, codes=ek.codes, rnorm=ek.rnorm, bits=ek.bits)
        self.vc = oattn.Cache(norm=ev.norm, codes=ev.codes)
        self.q = synth.decode_queries(1, self.G, d, seed=seed + 6).double().numpy()
        self.knew = synth.channel_scaled(1, 1, 1, d, seed=seed + 8)[0, 0].double().numpy()

    def step(self):
        """Append-encode one K and one V vector, then attention for the G query heads of the group
        over the sampled context."""
        ek = self.oenc.encode(self.knew, self.Dk, self.Sk, self.ck, self.tk)
        ev = self.oenc.encode(self.knew, self.Dv, self.np.zeros((0, self.d)), self.cv, self.tv)
        self.kc.norm[-1], self.kc.codes[-1], self.kc.rnorm[-1], self.kc.bits[-1] = ek.norm[0], ek.codes[0], ek.rnorm[0], ek.bits[0]
        self.vc.norm[-1], self.vc.codes[-1] = ev.norm[0], ev.codes[0]
        return self.oattn.attend_decode(self.q, self.kc, self.vc, [self.L], 1, self.Dk, self.Sk, self.ck, self.Dv,
                                        self.cv, ctx_stride=self.L)


def cpu_cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def typical_context(cfg) -> int:
    """The context of one (sequence, KV head) of the workload: the mean ragged length, else ctx."""
    if cfg["paged"]:
        return (cfg["len_lo"] + cfg["len_hi"]) // 2
    return cfg["ctx"]


def oracle_sample_plan(cfg, target_s: float):
    """Pick a context slice so that one oracle step takes about target_s seconds."""
    probe = OracleDecode(cfg, 4096)
    probe.step()
    t0 = time.perf_counter()
    probe.step()
    dt = time.perf_counter() - t0
    per_token = dt / 4096
    return int(min(typical_context(cfg), max(512, target_s / per_token)))


def run_cpu_baseline(cfg, target_s: float):
    """Repeat the oracle on one KV-head group over a typical context until about target_s."""
    L = typical_context(cfg)
    o = OracleDecode(cfg, L)
    reps = 0
    t0 = time.perf_counter()
    while True:
        o.step()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or reps >= 8 * cfg["n_kv_heads"]:  # the time target governs; the cap bounds it
            break
    return {"value": L * reps / dt, "unit": "keys/s", "cores": cpu_cores_used(), "kind": "oracle",
            "sample": f"{reps} x one KV-head group (4 query heads) over a {L}-token context (the workload's "
                      f"typical (sequence, KV head) length), each including append-encoding one K and one V "
                      f"vector; fp64 numpy oracle; {dt:.1f} s"}


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    cfg = workload(args)
    per_step_s = max(0.05, 90.0 / max(1, args.steps + args.warmup))
    L = oracle_sample_plan(cfg, per_step_s)
    o = OracleDecode(cfg, L)
    for _ in range(args.warmup):
        o.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.step()
    dt = time.perf_counter() - t0
    value = L * args.steps / dt
    cores = cpu_cores_used()
    line = {
        "impl": "reference", "metric": "decode keys scored/s", "value": value, "unit": "keys/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(args, cfg),
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: one KV-head group (4 query heads) over {L} of the workload's "
                                   f"{typical_context(cfg)}-token typical context, plus append-encoding one K "
                                   f"and one V vector"},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def reference_search_arm(args, world, rank):
    """The oracle on the search workload, on the host cores: each step scores one query against a
    4096-row sample of the database (encoded by the oracle beforehand, untimed) and takes its
    top-10; queries/s is scaled to the full database."""
    if rank != 0:
        return 0
    import synth
    from oracle import codebook as ocb, encode as oenc, estimate as oest, search as osearch
    d, n, rows, k = 1024, args.search_rows, 4096, 10
    mse, m = args.search_bits - 1, 1024
    D = synth.rotation_signs(d, 11).double().numpy()
    S = synth.qjl_matrix(m, d, 12).double().numpy()
    c, t = ocb.codebook(d, mse)
    enc = oenc.encode(synth.unit_rows(rows, d, seed=0).double().numpy(), D, S, c, t)
    Q = synth.unit_rows(max(1, args.steps + args.warmup), d, seed=1).double().numpy()

    def one(i):
        qr, p = oest.prepare_query(Q[i:i + 1], D, S)
        osearch.topk(oest.scores(qr, p, enc.norm, enc.codes, enc.rnorm, enc.bits, c), k)

    for i in range(args.warmup):
        one(args.steps + i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    dt = (time.perf_counter() - t0) / args.steps * (n / rows)  # seconds per query over n rows
    value = 1.0 / dt
    line = {
        "impl": "reference", "metric": "search queries/s", "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": search_config(args.search_bits, n, n * packed_bytes_per_key(d, mse, m)),
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": f"each step: one query scored against {rows} oracle-encoded rows and its "
                                   f"top-{k}, scaled to {n} rows; fp64 numpy oracle"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def search_cpu_baseline(ctx_d: int, mse: int, m: int, row_count: int):
    """The oracle on a bounded sample of the search workload: encode 4096 unit rows, score one
    query against them (timed separately), scaled to queries/s over the full database."""
    import synth
    from oracle import codebook as ocb, encode as oenc, estimate as oest
    rows = 4096
    D = synth.rotation_signs(ctx_d, 11).double().numpy()
    S = synth.qjl_matrix(m, ctx_d, 12).double().numpy()
    c, t = ocb.codebook(ctx_d, mse)
    X = synth.unit_rows(rows, ctx_d, seed=0).double().numpy()
    q = synth.unit_rows(1, ctx_d, seed=1).double().numpy()
    t0 = time.perf_counter()
    enc = oenc.encode(X, D, S, c, t)
    t_enc = time.perf_counter() - t0
    t0 = time.perf_counter()
    qr, p = oest.prepare_query(q, D, S)
    oest.scores(qr, p, enc.norm, enc.codes, enc.rnorm, enc.bits, c)
    t_sc = time.perf_counter() - t0
    return {"value": 1.0 / (t_sc * row_count / rows), "unit": "queries/s", "cores": cpu_cores_used(),
            "kind": "oracle", "encode_vectors_per_s": rows / t_enc,
            "sample": f"encode {rows} rows ({t_enc:.1f} s), score one query against them ({t_sc:.2f} s), "
                      f"scaled to {row_count} rows; fp64 numpy oracle"}


def main(argv=None):
    args = parse_args(argv)
    world, rank, _ = dist_setup(args)
    try:
        if args.impl == "reference":
            if args.config == "search":
                return reference_search_arm(args, world, rank)
            return reference_arm(args, world, rank)
        if args.config == "search":
            return ours_search(args, world, rank)
        return ours_decode(args, world, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
