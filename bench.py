#!/usr/bin/env python
"""Benchmark of the TurboQuant hot path on B200 (one process per GPU).

Default workload (the Llama-3.1-8B-shaped decode layer): batch 1, 32 query heads / 8 KV heads
(GQA 4), head_dim 128, context 32768, bf16 K/V drawn N(0,1) x lognormal(0,1) per (KV head,
channel); K encoded with 2 Lloyd-Max bits + a QJL sign sketch (m = 128), i.e. 3 bits/coordinate,
V with 3 MSE bits.  One step = one decode step of one layer: encode the new token's K and V for the
8 KV heads into the cache (append), then fused logits + softmax + V sum over the 32768 cached
tokens for the 32 query heads (query rotation and projection, split-context attention, combine).
Steps cycle over 48 distinct layer caches (1.36 GB of packed K+V), far larger than the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--kbits 3|4]

Prints one JSON line on rank 0.  `value` = decode keys scored per second over all ranks, a key
being one (token, KV head) pair scored against its 4 query heads.  Multi-GPU runs are weak
scaling: every rank decodes its own layers (independent problems, no data-path collective);
timing is the max over ranks of device time.  `--impl reference` times the fp64 CPU oracle on
the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import re
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = dict(name="llama3.1-8b decode layer", batch=1, n_q_heads=32, n_kv_heads=8, d=128, ctx=32768,
                v_bits=3, qjl_m=128)
N_LAYERS = 48
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--kbits", type=int, choices=[3, 4], default=3,
                    help="K bits per coordinate: (kbits-1) MSE bits + 1 QJL bit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=20.0)
    ap.add_argument("--workload", choices=["decode", "search"], default="decode",
                    help="decode: the Llama-3.1-8B decode layer (default); search: 10^6 x 1024 unit "
                         "vectors, 1000 queries, top-10 (encode and scan), one GPU")
    ap.add_argument("--search-bits", type=int, choices=[2, 4], default=2,
                    help="search: bits per coordinate, (bits-1) MSE bits + 1 QJL bit with m = d")
    ap.add_argument("--search-rows", type=int, default=1_000_000,
                    help="search: database rows (the workload is 10^6; smaller only for profiler captures)")
    return ap.parse_args(argv)


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


def recorded_traffic():
    """DRAM bytes per launch of the tensor-core attention kernel from the committed ncu summary,
    if it was taken on the kernel revision this library reports (else None)."""
    from kv_cache_vector_06_b200 import tq
    path = os.path.join(ROOT, "profiles", "attend_mma_llama8b_decode.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    rev = re.search(r"kernel revision: (\S+)", text)
    val = re.search(r"traffic_bytes_per_launch: (\d+)", text)
    if not rev or not val or f"attend_mma {rev.group(1)}" not in tq.version():
        return None
    return int(val.group(1))


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


# ------------------------------------------------------------------------------ our arm
class DecodeLayerBench:
    """Device-resident caches for N_LAYERS layers plus the per-step inputs."""

    def __init__(self, kbits: int, rank: int):
        import torch

        import synth
        from kv_cache_vector_06_b200 import tq
        self.tq = tq
        w = WORKLOAD
        self.d, self.hq, self.hkv, self.ctx, self.batch = w["d"], w["n_q_heads"], w["n_kv_heads"], w["ctx"], w["batch"]
        self.kmse = kbits - 1
        self.m = w["qjl_m"]
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev = dev
        seed = 1000 * rank
        self.kctx = tq.Context(self.d, self.kmse, self.m, synth.rotation_signs(self.d, seed + 1),
                               synth.qjl_matrix(self.m, self.d, seed + 2), device=dev.index)
        self.vctx = tq.Context(self.d, w["v_bits"], 0, synth.rotation_signs(self.d, seed + 3), device=dev.index,
                               layout=tq.LAYOUT_BLOCK16)
        cap = self.batch * self.hkv * self.ctx
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 7)
        self.layers = []
        ws_enc = torch.empty(tq.encode_workspace_size(self.kctx, self.hkv * self.ctx), dtype=torch.uint8, device=dev)
        for layer in range(N_LAYERS):
            kp = tq.Packed.allocate(self.kctx, cap)
            vp = tq.Packed.allocate(self.vctx, cap)
            for role, (ctx_, pk) in enumerate(((self.kctx, kp), (self.vctx, vp))):
                scale = torch.exp(torch.randn(self.hkv, 1, self.d, generator=g, device=dev))
                x = (torch.randn(self.batch * self.hkv, self.ctx, self.d, generator=g, device=dev)
                     * scale.repeat(self.batch, 1, 1)).to(torch.bfloat16).reshape(cap, self.d)
                tq.encode_kv(ctx_, x, pk, ws=ws_enc)
                del x
            self.layers.append((kp, vp))
        torch.cuda.synchronize()
        # per-step inputs: query and the new token's K/V (bf16), slots of the last position
        self.q = torch.randn(self.batch, self.hq, self.d, generator=g, device=dev).to(torch.bfloat16)
        self.k_new = torch.randn(self.batch * self.hkv, self.d, generator=g, device=dev).to(torch.bfloat16)
        self.v_new = torch.randn(self.batch * self.hkv, self.d, generator=g, device=dev).to(torch.bfloat16)
        self.slots = torch.tensor([(b * self.hkv + h) * self.ctx + self.ctx - 1 for b in range(self.batch)
                                   for h in range(self.hkv)], dtype=torch.int64, device=dev)
        self.seq_lens = torch.full((self.batch,), self.ctx, dtype=torch.int32, device=dev)
        self.out = torch.empty(self.batch, self.hq, self.d, dtype=torch.float32, device=dev)
        self.descs = [tq.make_attn_desc(self.kctx, self.vctx, (self.batch, self.hq, self.d), kp, vp, self.seq_lens,
                                        self.ctx, ctx_stride=self.ctx, n_kv_heads=self.hkv)
                      for kp, vp in self.layers]
        self.ws_step = torch.empty(tq.decode_step_workspace_size(self.kctx, self.vctx, self.descs[0],
                                                                 self.batch * self.hkv), dtype=torch.uint8, device=dev)
        self.keys_per_step = self.batch * self.hkv * self.ctx
        self.bytes_per_step = self.keys_per_step * (packed_bytes_per_key(self.d, self.kmse, self.m)
                                                    + packed_bytes_per_key(self.d, w["v_bits"], 0))

    def step(self, layer: int, q=None, out=None, k_new=None, v_new=None):
        # one decode step of one layer: append the new K and V token of every KV head, attend
        self.tq.decode_step(self.kctx, self.vctx, self.q if q is None else q, self.k_new if k_new is None else k_new,
                            self.v_new if v_new is None else v_new, self.slots, self.descs[layer],
                            out=self.out if out is None else out, ws=self.ws_step)

    def capture_graphs(self):
        import torch
        graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for layer in range(N_LAYERS):  # warm every layer once outside capture
                self.step(layer)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for layer in range(N_LAYERS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(layer)
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


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


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
            bench.step(i % N_LAYERS)
        torch.cuda.synchronize()
    finally:
        tq.profile_enable(False)
    prof = tq.profile_read()
    tq.profile_reset()
    return {k: v for k, v in prof.items() if v[0] > 0}


def time_e2e(bench, steps, warmup):
    """End to end through the public API with host buffers: per step, H2D of the query and the new
    token's K/V from pinned memory, encode + attention, D2H of the output."""
    import torch
    h_q = bench.q.cpu().pin_memory()
    h_k = bench.k_new.cpu().pin_memory()
    h_v = bench.v_new.cpu().pin_memory()
    h_out = torch.empty(bench.out.shape, dtype=torch.float32).pin_memory()
    d_q, d_k, d_v = torch.empty_like(bench.q), torch.empty_like(bench.k_new), torch.empty_like(bench.v_new)
    d_out = torch.empty_like(bench.out)

    def one(i):
        d_q.copy_(h_q, non_blocking=True)
        d_k.copy_(h_k, non_blocking=True)
        d_v.copy_(h_v, non_blocking=True)
        bench.step(i % N_LAYERS, q=d_q, out=d_out, k_new=d_k, v_new=d_v)
        h_out.copy_(d_out, non_blocking=True)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        one(i)
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    h2d = h_q.numel() * h_q.element_size() + h_k.numel() * h_k.element_size() + h_v.numel() * h_v.element_size()
    d2h = h_out.numel() * h_out.element_size()
    return ms, h2d, d2h


def time_encode(bench, reps=5):
    """Encode vectors/s: a full layer's K and V (2 x 262144 bf16 vectors) per rep."""
    import torch
    tq = bench.tq
    n = bench.batch * bench.hkv * bench.ctx
    g = torch.Generator(device=bench.dev)
    g.manual_seed(99)
    xk = torch.randn(n, bench.d, generator=g, device=bench.dev).to(torch.bfloat16)
    xv = torch.randn(n, bench.d, generator=g, device=bench.dev).to(torch.bfloat16)
    kp, vp = bench.layers[0]
    ws = torch.empty(tq.encode_workspace_size(bench.kctx, n), dtype=torch.uint8, device=bench.dev)
    for _ in range(2):
        tq.encode_kv(bench.kctx, xk, kp, ws=ws)
        tq.encode_kv(bench.vctx, xv, vp, ws=ws)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        tq.encode_kv(bench.kctx, xk, kp, ws=ws)
        tq.encode_kv(bench.vctx, xv, vp, ws=ws)
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / reps
    return 2 * n / (ms / 1e3), ms


# ------------------------------------------------------------------------------ oracle (CPU) arm
class OracleDecode:
    """The fp64 oracle on one KV-head group of the same workload (host cores)."""

    def __init__(self, kbits: int, ctx_tokens: int, seed: int = 0):
        import numpy as np

        import synth
        from oracle import attention as oattn
        from oracle import codebook as ocb
        from oracle import encode as oenc
        w = WORKLOAD
        d, m = w["d"], w["qjl_m"]
        self.np, self.oattn, self.oenc = np, oattn, oenc
        self.d, self.G = d, w["n_q_heads"] // w["n_kv_heads"]
        self.L = ctx_tokens
        self.Dk = synth.rotation_signs(d, seed + 1).double().numpy()
        self.Sk = synth.qjl_matrix(m, d, seed + 2).double().numpy()
        self.Dv = synth.rotation_signs(d, seed + 3).double().numpy()
        self.ck, self.tk = ocb.codebook(d, kbits - 1)
        self.cv, self.tv = ocb.codebook(d, w["v_bits"])
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


def oracle_sample_plan(target_s: float, kbits: int):
    """Pick a context slice so that one oracle step takes about target_s seconds."""
    probe = OracleDecode(kbits, 4096)
    probe.step()
    t0 = time.perf_counter()
    probe.step()
    dt = time.perf_counter() - t0
    per_token = dt / 4096
    L = int(min(WORKLOAD["ctx"], max(512, target_s / per_token)))
    return L


def run_cpu_baseline(kbits: int, target_s: float):
    """Repeat the oracle on one KV-head group over the full context until about target_s."""
    L = WORKLOAD["ctx"]
    o = OracleDecode(kbits, L)
    reps = 0
    t0 = time.perf_counter()
    while True:
        o.step()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or reps >= WORKLOAD["n_kv_heads"]:
            break
    return {"value": L * reps / dt, "unit": "keys/s", "cores": cpu_cores_used(), "kind": "oracle",
            "sample": f"{reps} x one KV-head group (4 query heads) over the full {L}-token context, each "
                      f"including append-encoding one K and one V vector; fp64 numpy oracle; {dt:.1f} s"}


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    kbits = args.kbits
    per_step_s = max(0.05, 90.0 / max(1, args.steps + args.warmup))
    L = oracle_sample_plan(per_step_s, kbits)
    o = OracleDecode(kbits, L)
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
        "config": workload_config(kbits),
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: one KV-head group (4 query heads) over {L} of the 32768 context "
                                   f"tokens, plus append-encoding one K and one V vector"},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(kbits):
    w = WORKLOAD
    return {"workload": f"{w['name']}: batch {w['batch']}, {w['n_q_heads']} q / {w['n_kv_heads']} kv heads, "
                        f"head_dim {w['d']}, context {w['ctx']}, K {kbits - 1}+QJL(m={w['qjl_m']}) bits, "
                        f"V {w['v_bits']} bits; step = append-encode + decode attention",
            "batch": w["batch"], "n_q_heads": w["n_q_heads"], "n_kv_heads": w["n_kv_heads"], "head_dim": w["d"],
            "context": w["ctx"], "k_bits": kbits, "v_bits": w["v_bits"], "qjl_m": w["qjl_m"],
            "parallelism": "independent layers per GPU (weak scaling)",
            "l2": f"inputs larger than L2: {N_LAYERS} distinct layer caches cycled"}


def ours_arm(args, world, rank):
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py --impl ours needs a CUDA device (there is no CPU fallback)")
    bench = DecodeLayerBench(args.kbits, rank)
    graphs = bench.capture_graphs()
    sampler = ClockSampler(torch.cuda.current_device())
    ms = time_graph_steps(graphs, args.steps, args.warmup, world, sampler)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = aggregate_rate(world, bench.keys_per_step, args.steps, ms)
    hbm_gbs = aggregate_rate(world, bench.bytes_per_step, args.steps, ms) / 1e9

    prof_steps = min(args.steps, N_LAYERS)
    prof = profile_kernels(bench, prof_steps)
    launches_per_step = sum(n for n, _ in prof.values()) / prof_steps
    split_n, split_ms = prof.get("attend_split", (0, 0.0))  # the split kernel (tensor-core path here)
    peaks, src = measured_peaks()
    roof = None
    if split_n:
        per_launch_s = split_ms / split_n / 1e3
        achieved = bench.bytes_per_step / per_launch_s / 1e9
        roof = {"kernel": "attend_mma_kernel (tensor cores, streamed sub-chunks, fused split merge)", "bound": "hbm",
                "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic(),
                "peak_source": src + " (burst copy)", "us_per_launch": per_launch_s * 1e6,
                "algorithmic_bytes_per_launch": bench.bytes_per_step}
    kernel_share = {k: {"launches_per_step": n / prof_steps, "us_per_launch": 1e3 * t / n}
                    for k, (n, t) in prof.items()}

    e2e_steps = min(args.steps, 500)
    e_ms, h2d, d2h = time_e2e(bench, e2e_steps, min(args.warmup, 20))
    e_ms = max_over_ranks(e_ms, world)
    e2e_value = aggregate_rate(world, bench.keys_per_step, e2e_steps, e_ms)

    enc_vps, enc_ms = time_encode(bench)
    enc_ms = max_over_ranks(enc_ms, world)
    enc_vps = 2 * bench.keys_per_step / (enc_ms / 1e3)
    line = {
        "metric": "decode keys scored/s", "value": value, "unit": "keys/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args.kbits),
        "hbm_gbs": hbm_gbs, "hbm_frac_of_peak": hbm_gbs / (world * peaks["hbm_gbs"]), "peak_source": src,
        "encode_vectors_per_s": world * enc_vps,
        "roofline": roof,
        "kernels": kernel_share,
        "e2e": {"value": e2e_value, "unit": "keys/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = run_cpu_baseline(args.kbits, args.cpu_sample_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    return 0


def search_arm(args, world=1, rank=0):
    """Vector search at 10^6 rows x d 1024: encode the database (unit vectors, fp32), then top-10
    for 1000 queries.  Inputs are drawn on the device with a seeded generator (same recipe as the
    parity tests: N(0, I) rows L2-normalised).  Under torchrun every rank searches its own
    database (weak scaling); times are the slowest rank's and rank 0 prints the line."""
    import torch
    from kv_cache_vector_06_b200 import tq
    import synth
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py --workload search needs a CUDA device (there is no CPU fallback)")
    d, n, nq, k = 1024, args.search_rows, 1000, 10
    mse, m = args.search_bits - 1, d
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
    # Tensor roofline of the scan: the estimate is a contraction of the rows' bit planes (mse code
    # planes, a parity plane at 3 MSE bits, the sign plane) with the queries' 24-bit fixed-point
    # values as three int8 limbs: 2 x planes x d x 3 int8 ops per (query, row), against the measured
    # bf16 peak x 2 (the dense int8:bf16 ratio)
    planes = mse + (1 if mse == 3 else 0) + 1
    int8_ops = 2.0 * planes * d * 3 * nq * n
    int8_peak = peaks["bf16_tflops"] * 2
    terms = nq * n * (d + m) / (ms / 1e3)
    line = {
        "metric": "search queries/s", "value": aggregate_rate(world, nq, 1, ms), "unit": "queries/s",
        "n_gpus": world,
        "steps": reps, "warmup": max(1, min(args.warmup, 3)), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": search_config(args, n, db_bytes),
        "scores_per_s": nq * n / (ms / 1e3),
        "database_passes_per_s": 1e3 / ms,
        "hbm": {"database_bytes": db_bytes, "gbs_one_read_per_query": nq * db_bytes / (ms / 1e3) / 1e9,
                "peak": peaks["hbm_gbs"], "peak_source": src},
        "encode": {"vectors_per_s": n / (enc_ms / 1e3), "ms": enc_ms,
                   "gbs": n * (4 * d + row_bytes) / (enc_ms / 1e3) / 1e9,
                   "roofline": {"bound": "tensor", "achieved": 3 * 2 * m * d * n / (enc_ms / 1e3) / 1e12,
                                "peak": peaks["bf16_tflops"] / 2, "unit": "TFLOP/s",
                                "frac": 3 * 2 * m * d * n / (enc_ms / 1e3) / 1e12 / (peaks["bf16_tflops"] / 2),
                                "traffic": None,
                                "note": "QJL projection as 3 x TF32 MMA passes; peak = measured bf16 x 1/2 "
                                        "(the dense tf32:bf16 ratio)"}},
        "terms_per_s": terms,
        "roofline": {"kernel": "search_tc_kernel (bit-plane tcgen05 kind::i8 MMAs)", "bound": "tensor",
                     "achieved": int8_ops / (ms / 1e3) / 1e12, "peak": int8_peak, "unit": "TOP/s",
                     "frac": int8_ops / (ms / 1e3) / 1e12 / int8_peak, "traffic": None,
                     "note": "int8 ops of the bit-plane contraction (2 x %d planes x d x 3 limbs per query and row) "
                             "per search call; peak = measured bf16 x 2 (dense int8:bf16 ratio), %s" % (planes, src)},
        "e2e": {"value": aggregate_rate(world, nq, 1, e_ms), "unit": "queries/s",
                "h2d_bytes_per_step": h_q.numel() * h_q.element_size(),
                "d2h_bytes_per_step": h_s.numel() * 4 + h_i.numel() * 8},
        # per call: query rotation, query projection, per-query scales, query operand, scan, merge
        "gpu_launches": 6 * reps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = search_cpu_baseline(ctx_d=d, mse=mse, m=m, row_count=n)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def search_config(args, n: int, db_bytes: int) -> dict:
    mse = args.search_bits - 1
    return {"workload": f"vector search: {'10^6' if n == 1_000_000 else n} unit vectors d 1024, "
                        f"{args.search_bits} bits/coord ({mse} MSE + QJL m 1024), 1000 queries, top-10",
            "rows": n, "d": 1024, "queries": 1000, "k": 10,
            "l2": "database (%.0f MB packed) %s than the 126 MB L2" % (
                db_bytes / 1e6, "larger" if db_bytes > 126e6 else "smaller")}


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
        "config": search_config(args, n, n * packed_bytes_per_key(d, mse, m)),
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
    import numpy as np
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
            if args.workload == "search":
                return reference_search_arm(args, world, rank)
            return reference_arm(args, world, rank)
        if args.workload == "search":
            return search_arm(args, world, rank)
        return ours_arm(args, world, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
