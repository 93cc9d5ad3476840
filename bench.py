"""Benchmark of the HSA denoising step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the full HSA loop of a 30-layer DiT (hidden 1536, 12 heads x 128,
MLP 8960, bf16 weights N(0, 1/fan_in)) on a 21x30x52 video latent (N = 32760
tokens x 16 channels), T = 40 flow-matching steps (sigma 1 -> 0, shift 5), K = 3
groups with budgets {40, 20, 10} holding 40/30/30% of the tokens, re-grouped by
L1 relative velocity change.  A step is one global iteration i of that loop
(schedule, embed, 30 sparse layers, head, cached Euler, re-grouping); step k
runs iteration k mod 40, so 40 steps are one whole loop.  All inputs are seeded
synthetic data resident in HBM before timing; every step touches > 8 GB
(weights 2.2 GB + KV caches 6 GB), far more than the 126 MB L2.

One JSON line is printed by rank 0.  ``value`` is ms per denoising step (max
over ranks; lower is better); extra keys carry the dense all-active step time,
active-query attention TFLOP/s at 100/50/25% active, cached-Euler GB/s, the
roofline of the dominant kernel (attention), the end-to-end figure through the
public call with host buffers, and the CPU oracle timed on a bounded sample.
With --gpus N > 1 each rank runs an independent replica (the method runs on one
GPU; there is no data-path collective).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSA denoise-step ms & active-query attn TFLOP/s at 25/50/100% active; Euler GB/s"
WORKLOAD = "dit30_1536"


def parse():
    ap = argparse.ArgumentParser(description="HSA denoising-step benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["replicas", "shard"], default="replicas",
                    help="replicas: one loop per GPU (weak scaling); shard: one loop split "
                         "over the GPUs by active-list chunks with a K/V all-gather per layer "
                         "(strong scaling)")
    ap.add_argument("--kv-exchange", choices=["gather", "peer"], default="gather",
                    help="shard mode: K|V rows by NCCL all-gather + scatter, or stored by the "
                         "QKV GEMM's epilogue straight into every rank's cache (peer memory)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the sub-benchmarks (profiling runs)")
    ap.add_argument("--profile-case", choices=["attention", "gemm", "euler", "rows", "tokens",
                                                "embed_head", "gemm_epi", "gemm1", "qkv_peers"],
                    default=None,
                    help="run three launches of one kernel at the workload shape and exit")
    return ap.parse_args()


# --------------------------------------------------------------------------- distributed

def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        pg = dist
    return rank, world, local, pg


def max_over_ranks(value: float, pg, device) -> float:
    if pg is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in self.rows for j in range(4)
                          if r[4 + j].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


# --------------------------------------------------------------------------- our arm

def build_loop(spec, seed, torch):
    from token_sparse_denoising_layer_b200 import synth
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    layers = [synth.device_layer_weights(sh.D, sh.F, seed * 1000 + l) for l in range(sh.L)]
    wf = synth.model_weights(synth.ModelShape(sh.N, sh.C, sh.D, sh.H, 64, 0), seed)
    w_in = torch.from_numpy(wf["w_in"]).cuda()
    w_head = torch.from_numpy(wf["w_head"]).cuda()
    loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, w_in, w_head, spec["T"], spec["budgets"],
                   counts, shift=spec["shift"])
    x0 = torch.from_numpy(synth.latent(sh.N, 16, seed)).cuda()
    g0 = torch.from_numpy(synth.random_split(sh.N, counts, seed)).cuda()
    return loop, x0, g0, counts, layers


def time_steps(loop, steps, torch, regroup=True, per_step_hook=None):
    """Time `steps` iterations (i = k mod T) with CUDA events on the launch stream."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    torch.cuda.synchronize()
    for k in range(steps):
        i = k % loop.T
        ev[k][0].record(stream)
        if per_step_hook is not None:
            per_step_hook(k, i)
        else:
            loop.step(i, regroup)
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def attention_sweep(torch, abi, synth):
    """Single DiT layer, N = 32760, hidden 1536, 12 x 128 heads: attention of
    |A| = f*N queries against the full cache, f in {1, .5, .25, .1}."""
    N, D, H = 32760, 1536, 12
    ctx = abi.hsa_create(N=N, D=D, H=H, F=6144, L=1, T=1, budgets=[1], counts=[N])
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    kc = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    o = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
    out = {}
    stream = torch.cuda.current_stream()
    for f in (1.0, 0.5, 0.25, 0.1):
        a = int(round(f * N))
        for _ in range(3):
            abi.hsa_attention(ctx, q, a, kc, vc, o)
        reps = 10
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            abi.hsa_attention(ctx, q, a, kc, vc, o)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        flop = 4.0 * a * N * D
        out[f"{int(f * 100)}%"] = {"active": a, "ms": round(ms, 4),
                                   "tflops": round(flop / ms / 1e9, 1)}
    abi.hsa_sync_check(ctx)
    ctx.close()
    del kc, vc, q, o
    # the 40-layer DiT's attention shape: N = 75600 (21x45x80), 40 heads x 128
    N, D, H = 75600, 5120, 40
    ctx = abi.hsa_create(N=N, D=D, H=H, F=64, L=1, T=1, budgets=[1], counts=[N])
    kc = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((N, D), generator=g, device="cuda").to(torch.bfloat16)
    o = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
    for f in (1.0, 0.25):
        a = int(round(f * N))
        ms = _time(lambda: abi.hsa_attention(ctx, q, a, kc, vc, o), torch, reps=3)
        out[f"dit40_{int(f * 100)}%"] = {"active": a, "N": N, "D": D, "ms": round(ms, 3),
                                         "tflops": round(4.0 * a * N * D / ms / 1e9, 1)}
    abi.hsa_sync_check(ctx)
    ctx.close()
    return out


def euler_bandwidth(torch, abi):
    """Cached-Euler kernel GB/s at the 21x30x52 and 21x45x80 latents (L2 flushed
    between samples) and at a 256M-float size (asymptotic)."""
    res = {}
    flush = _l2_flush(torch)
    stream = torch.cuda.current_stream()
    for N in (32760, 75600, 16 * 1024 * 1024):
        ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=40, budgets=[40, 20, 10],
                             counts=[N - 2 * (N * 3 // 10), N * 3 // 10, N * 3 // 10])
        x, vh, vp, vf = (torch.randn((N, 16), device="cuda") for _ in range(4))
        mask = (torch.rand(N, device="cuda") < 0.625).to(torch.uint8)
        a = int(mask.sum().item())
        times = []
        for r in range(13):
            _do_flush(flush, r)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            abi.hsa_euler_step(ctx, x, vh, vp, vf, mask, 0.5, 0.475)
            e1.record(stream)
            torch.cuda.synchronize()
            if r >= 3:
                times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
        bytes_ = N * 16 * 4 * 3 + a * 16 * 4 * 3 + N
        res[str(N)] = {"ms": round(ms, 5), "GBps": round(bytes_ / ms / 1e6, 1), "bytes": bytes_}
        ctx.close()
    del flush
    return res


def token_kernels_graph(torch, abi, synth):
    """Scheduler, re-grouping and cached Euler at the 21x30x52 and 21x45x80
    latents ({40,20,10} at 40/30/30%), each captured as a CUDA graph of
    back-to-back calls so the per-call figure carries no launch gaps: all 40
    schedule calls of a loop, 20 standalone re-groupings (score + radix select +
    assign), 100 Euler updates, 20 re-grouping steps' tail as the loop runs it
    (Euler pass that writes the scores, then radix select + assign), and, as the
    floor every launch pays, 100 empty kernels.  The buffers (<= 25 MB) stay in
    L2 across the calls."""
    out = {}
    stream = torch.cuda.current_stream()
    for name in ("select_euler_32760", "select_euler_75600"):
        spec = synth.WORKLOADS[name]
        N, T = spec["N"], spec["T"]
        counts = synth.group_counts(N, spec["fractions"])
        ctx = abi.hsa_create(N=N, D=128, H=1, F=64, L=0, T=T, budgets=spec["budgets"],
                             counts=counts)
        vp, vc, _ = synth.velocity_pair(N, 16, spec["seed"])
        v_prev, v_cur = torch.from_numpy(vp).cuda(), torch.from_numpy(vc).cuda()
        g = torch.from_numpy(synth.random_split(N, counts, spec["seed"])).cuda()
        mask = torch.zeros(N, dtype=torch.uint8, device="cuda")
        idx = torch.zeros(N, dtype=torch.int32, device="cuda")
        score = torch.zeros(N, dtype=torch.float32, device="cuda")
        x, vf = (torch.randn((N, 16), device="cuda") for _ in range(2))
        vh, vhp = v_cur.clone(), v_prev.clone()
        gsel = g.clone()
        calls = {
            "schedule": (T, lambda k: abi.hsa_schedule(ctx, k % T, g, mask, idx)),
            "regroup": (20, lambda k: abi.hsa_select_groups(ctx, v_prev, v_cur, score, gsel)),
            "euler": (100, lambda k: abi.hsa_euler_step(ctx, x, vh, vhp, vf, mask, 0.5, 0.475)),
            "euler_score+select": (20, lambda k: (
                abi.hsa_euler_step_score(ctx, x, vh, vhp, vf, mask, 0.5, 0.475, score),
                abi.hsa_select_from_score(ctx, score, gsel))),
            "empty_kernel": (100, lambda k: torch.cuda._sleep(0)),
        }
        res = {}
        for key, (n_calls, fn) in calls.items():
            for k in range(3):
                fn(k)
            torch.cuda.synchronize()
            side = torch.cuda.Stream()
            graph = torch.cuda.CUDAGraph()
            abi.hsa_set_stream(ctx, side)
            try:
                with torch.cuda.graph(graph, stream=side):
                    for k in range(n_calls):
                        fn(k)
            finally:
                abi.hsa_set_stream(ctx, None)
            graph.replay()
            times = []
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) / n_calls)
            us = float(np.median(times)) * 1e3
            res[key] = {"us_per_call": round(us, 2), "calls_per_graph": n_calls}
            del graph
        a = int(mask.sum().item())
        eb = N * 16 * 4 * 3 + a * 16 * 4 * 3 + N
        res["euler"]["GBps_l2_resident"] = round(eb / res["euler"]["us_per_call"] / 1e3, 1)
        floor = res["empty_kernel"]["us_per_call"]
        launches = {"schedule": 1, "regroup": 3, "euler": 1, "euler_score+select": 3}
        for key, nl in launches.items():
            res[key]["launches_per_call"] = nl
            res[key]["over_launch_floor_us"] = round(res[key]["us_per_call"] - nl * floor, 2)
        abi.hsa_sync_check(ctx)
        ctx.close()
        out[str(N)] = res
    return out


def attention_traffic():
    """DRAM bytes per launch of the attention kernel at N = |A| = 32760 from the
    committed ncu summary, or None if the kernel source changed since the capture."""
    import hashlib
    import re

    prof = os.path.join(ROOT, "profiles", "k_attn_128_n32760_a32760.md")
    src = os.path.join(ROOT, "token_sparse_denoising_layer_b200", "csrc", "k_attn.cu")
    try:
        text = open(prof).read()
        want = re.search(r"source_sha256_prefix: ([0-9a-f]+)", text).group(1)
        have = hashlib.sha256(open(src, "rb").read()).hexdigest()[: len(want)]
        if want != have:
            return None
        return int(re.search(r"traffic_bytes_per_launch: (\d+)", text).group(1))
    except (OSError, AttributeError):
        return None


def _peaks():
    """The measured peaks (HBM GB/s, bf16 TFLOP/s burst and sustained), or {}."""
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        with open(pp) as f:
            return json.load(f)
    return {}


def _l2_flush(torch):
    """Two 256 MB buffers: one written between samples (evicts every line), then
    one read, so the written lines are back in HBM before the sample starts and
    the timed kernel pays for no one else's write-back."""
    n = 256 * 1024 * 1024 // 4
    return (torch.empty(n, dtype=torch.float32, device="cuda"),
            torch.ones(n, dtype=torch.float32, device="cuda"))


def _do_flush(flush, r):
    wbuf, rbuf = flush
    wbuf.fill_(float(r))
    rbuf.sum()


def _time(fn, torch, reps=10, flush=None):
    """Median CUDA-event time (ms) of fn() on the current stream, after warm-up;
    with `flush` (see _l2_flush), L2 holds neither useful nor dirty lines when
    each sample starts."""
    stream = torch.cuda.current_stream()
    for _ in range(3):
        fn()
    times = []
    for r in range(reps):
        if flush is not None:
            _do_flush(flush, r)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return float(np.median(times))


def _sm_clock_mhz(index=0):
    """The SM clock now (MHz), read once through NVML, or None."""
    try:
        import pynvml

        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(index)
        return int(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
    except Exception:   # noqa: BLE001 - a missing NVML only loses the clock note
        return None


def gemm_sweep(torch, abi, synth, peak_tf=None):
    """The active-row GEMMs of a 1536-wide DiT layer as the step runs them, at
    each active-row count: QKV with the KV-cache scatter epilogue
    (hsa_qkv_project), out-projection with the residual add into scattered rows
    (hsa_out_proj_residual), and the MLP pair (GELU epilogue up, residual add
    down: hsa_mlp_residual less its LN gather, timed apart).  Beside each, the
    same product with the plain bf16 store (hsa_linear).  Shapes: the 30-layer
    DiT (F = 8960) at the step's 100/70/40% of 32760 rows, and the single layer
    (F = 6144) at 100/50/25/10%.  L2 is flushed between samples; the SM clock
    is read after each group."""
    N, D, H = 32760, 1536, 12
    flush = _l2_flush(torch)
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    rnd = lambda *sh: torch.randn(sh, generator=g, device="cuda").to(torch.bfloat16)
    out = {}
    for tag, F, Ms in (("dit30", 8960, (32760, 22932, 13104)),
                       ("layer_1536", 6144, (32760, 16380, 8190, 3276))):
        ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=1, T=1, budgets=[1], counts=[N])
        w_qkv, w_o, w_1, w_2 = rnd(3 * D, D), rnd(D, D), rnd(F, D), rnd(D, F)
        kc, vc = rnd(N, D), rnd(N, D)
        x = torch.randn((N, D), generator=g, device="cuda") * 0.0
        obuf = torch.empty((N, max(3 * D, F)), dtype=torch.bfloat16, device="cuda")
        u = rnd(N, D)
        hid = rnd(N, F)
        for M in Ms:
            idx = torch.from_numpy(synth.random_active_set(N, M, M)).cuda()
            t = {}
            t["qkv"] = _time(lambda: abi.hsa_qkv_project(ctx, w_qkv, u, idx, M, obuf, kc, vc),
                             torch, flush=flush)
            t["out_proj"] = _time(lambda: abi.hsa_out_proj_residual(ctx, w_o, u, idx, M, x),
                                  torch, flush=flush)
            mlp = _time(lambda: abi.hsa_mlp_residual(ctx, w_1, w_2, x, idx, M), torch,
                        flush=flush)
            ln = _time(lambda: abi.hsa_ln_gather(ctx, x, idx, M, u), torch, flush=flush)
            t["mlp_up+down"] = mlp - ln
            p = {}
            p["qkv"] = _time(lambda: abi.hsa_linear(ctx, u, M, D, w_qkv, 3 * D, obuf), torch,
                             flush=flush)
            p["out_proj"] = _time(lambda: abi.hsa_linear(ctx, u, M, D, w_o, D, obuf), torch,
                                  flush=flush)
            p["mlp_up+down"] = (_time(lambda: abi.hsa_linear(ctx, u, M, D, w_1, F, hid), torch,
                                      flush=flush) +
                                _time(lambda: abi.hsa_linear(ctx, hid, M, F, w_2, D, obuf),
                                      torch, flush=flush))
            mhz = _sm_clock_mhz()
            flops = {"qkv": 6.0 * M * D * D, "out_proj": 2.0 * M * D * D,
                     "mlp_up+down": 4.0 * M * D * F}
            row = {"sm_mhz_after": mhz}
            for k, fl in flops.items():
                tf, tp = fl / t[k] / 1e9, fl / p[k] / 1e9
                row[k] = {"ms": round(t[k], 4), "tflops": round(tf, 1),
                          "frac": round(tf / peak_tf, 3) if peak_tf else None,
                          "plain_ms": round(p[k], 4), "plain_tflops": round(tp, 1),
                          "fused_vs_plain": round(p[k] / t[k], 3)}
            out[f"{tag} M={M}"] = row
            del idx
        abi.hsa_sync_check(ctx)
        ctx.close()
        del w_qkv, w_o, w_1, w_2, kc, vc, x, obuf, u, hid
    del flush
    return out


def bandwidth_sweep(torch, abi):
    """HBM-bound row kernels at the workloads' sizes, L2 flushed between samples:
    the standalone KV-cache scatter (dit30 and dit40 shapes) and the LN gather."""
    flush = _l2_flush(torch)
    res = {}
    for name, N, D, a in (("kv_scatter_dit30_f1", 32760, 1536, 32760),
                          ("kv_scatter_dit40_f0.25", 75600, 5120, 18900)):
        ctx = abi.hsa_create(N=N, D=D, H=D // 128, F=64, L=1, T=1, budgets=[1], counts=[N])
        kr = torch.randn((a, D), device="cuda").to(torch.bfloat16)
        vr = torch.randn((a, D), device="cuda").to(torch.bfloat16)
        kc = torch.zeros((N, D), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros((N, D), dtype=torch.bfloat16, device="cuda")
        idx = torch.sort(torch.randperm(N, device="cuda")[:a]).values.to(torch.int32)
        ms = _time(lambda: abi.hsa_kv_scatter(ctx, kr, vr, idx, a, kc, vc), torch, flush=flush)
        nbytes = 4 * a * D * 2 + 4 * a
        res[name] = {"rows": a, "D": D, "ms": round(ms, 4), "GBps": round(nbytes / ms / 1e6, 1)}
        abi.hsa_sync_check(ctx)
        ctx.close()
        del kr, vr, kc, vc
    N, D = 32760, 1536
    ctx = abi.hsa_create(N=N, D=D, H=12, F=64, L=1, T=1, budgets=[1], counts=[N])
    x = torch.randn((N, D), device="cuda")
    u = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.arange(N, dtype=torch.int32, device="cuda")
    ms = _time(lambda: abi.hsa_ln_gather(ctx, x, idx, N, u), torch, flush=flush)
    nbytes = N * D * (4 + 2) + N * 4
    res["ln_gather_dit30_f1"] = {"rows": N, "D": D, "ms": round(ms, 4),
                                 "GBps": round(nbytes / ms / 1e6, 1)}
    ctx.close()
    del flush
    return res


def conditioned_layer(torch, abi):
    """One 1536-wide DiT layer (N = 32760, F = 8960) with 40% of the tokens
    active: the plain block against the conditioned one (timestep modulation
    plus cross-attention to 512 text tokens), ms per layer."""
    N, D, H, F, a, n_txt = 32760, 1536, 12, 8960, 13104, 512
    ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=1, T=1, budgets=[1], counts=[N])
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    rnd = lambda *sh, s=1.0: (torch.randn(sh, generator=g, device="cuda") * s).to(torch.bfloat16)
    lw = abi.layer_weights(rnd(3 * D, D, s=D ** -0.5), rnd(D, D, s=D ** -0.5),
                           rnd(F, D, s=D ** -0.5), rnd(D, F, s=F ** -0.5))
    xa = abi.cross_attn(rnd(D, D, s=D ** -0.5), rnd(D, D, s=D ** -0.5), rnd(n_txt, D),
                        rnd(n_txt, D), n_txt)
    mod = torch.randn((6, D), generator=g, device="cuda") * 0.5
    mod[2] += 1.0
    mod[5] += 1.0
    x = torch.randn((N, D), generator=g, device="cuda")
    kc, vc = rnd(N, D), rnd(N, D)
    idx = torch.sort(torch.randperm(N, generator=g, device="cuda")[:a]).values.to(torch.int32)
    plain = _time(lambda: abi.hsa_layer_forward(ctx, lw, x, idx, a, kc, vc), torch)
    cond = _time(lambda: abi.hsa_layer_forward_cond(ctx, lw, mod, xa, x, idx, a, kc, vc), torch)
    abi.hsa_sync_check(ctx)
    ctx.close()
    # cross-attention adds LN + a [a, D] x [D, D] projection twice + attention over n_txt keys
    extra_flop = 2 * 2.0 * a * D * D + 4.0 * a * n_txt * D
    return {"active": a, "n_txt": n_txt, "plain_ms": round(plain, 4), "cond_ms": round(cond, 4),
            "extra_ms": round(cond - plain, 4),
            "extra_tflops": round(extra_flop / max(cond - plain, 1e-6) / 1e9, 1)}


def dit40_steps(torch, synth):
    """The 40-layer DiT (N = 75600, D = 5120, 40 x 128 heads, F = 13824), budgets
    {40, 10} at 25/75%: one step at each of its two active patterns (i = 0: all
    tokens; i = 1: the 25% full-budget group), median of 3 after one warm-up,
    extrapolated to the 40-step loop (10 all-active steps + 30 at 25%)."""
    spec = synth.WORKLOADS["dit40_5120"]
    loop, x0, g0, counts, layers = build_loop(spec, 2, torch)
    loop.reset(x0, g0)
    per = {}
    for i in (0, 1):
        loop.step(i, False)
        ts = time_steps_at(loop, i, 3, torch)
        per[i] = float(np.median(ts))
    a = {i: loop.n_active(i) for i in (0, 1)}
    from token_sparse_denoising_layer_b200 import abi
    abi.hsa_sync_check(loop.ctx)
    loop.close()
    del loop, layers
    torch.cuda.empty_cache()
    n_full = sum(1 for i in range(spec["T"]) if i % 4 == 0)
    hsa_loop = n_full * per[0] + (spec["T"] - n_full) * per[1]
    return {"N": 75600, "D": 5120, "L": 40, "active_i0": a[0], "active_i1": a[1],
            "ms_step_100%": round(per[0], 1), "ms_step_25%": round(per[1], 1),
            "hsa_loop_s": round(hsa_loop / 1e3, 2), "dense_loop_s": round(spec["T"] * per[0] / 1e3, 2),
            "hsa_vs_dense": round(hsa_loop / (spec["T"] * per[0]), 3),
            "mean_active_fraction": 0.4375}


def time_steps_at(loop, i, reps, torch):
    """CUDA-event times (ms) of `reps` calls of step i (no re-grouping)."""
    stream = torch.cuda.current_stream()
    out = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        loop.step(i, False)
        e1.record(stream)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1))
    return out


def preset_sweep(torch, synth, spec, layers, w_in, w_head, x0_seed=0):
    """Budget presets and the static split on the 30-layer DiT: the whole 40-step
    loop per preset (ms per step, mean over the loop).  The pages evaluate four
    presets and four grouping strategies without defining them; these presets
    span mean active fractions from 0.75 to 0.44, and "static" keeps the initial
    seeded random split (no re-grouping) of the default preset."""
    from token_sparse_denoising_layer_b200.loop import HsaLoop
    sh = spec["shape"]
    presets = [("{40,20} 50/50", (40, 20), (0.5, 0.5), True),
               ("{40,20,10} 40/30/30", (40, 20, 10), (0.4, 0.3, 0.3), True),
               ("{40,20,10} 40/30/30 static", (40, 20, 10), (0.4, 0.3, 0.3), False),
               ("{40,10} 25/75", (40, 10), (0.25, 0.75), True),
               ("{40,20,10,5} 25/25/25/25", (40, 20, 10, 5), (0.25, 0.25, 0.25, 0.25), True)]
    out = {}
    for name, budgets, fr, regroup in presets:
        counts = synth.group_counts(sh.N, fr)
        loop = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, w_in, w_head, spec["T"], budgets, counts,
                       shift=spec["shift"])
        loop.reset(torch.from_numpy(synth.latent(sh.N, 16, x0_seed)).cuda(),
                   torch.from_numpy(synth.random_split(sh.N, counts, x0_seed)).cuda())
        ts = time_steps(loop, spec["T"], torch, regroup=regroup)
        mean_frac = sum(c * b for c, b in zip(counts, budgets)) / (sh.N * spec["T"])
        out[name] = {"ms_per_step": round(float(np.mean(ts)), 2),
                     "mean_active_fraction": round(mean_frac, 4)}
        loop.close()
        del loop
    torch.cuda.empty_cache()
    return out


def graph_replay(torch, synth, loop, x0, g0, eager_ms):
    """The loop recorded as one CUDA graph (40 steps, one launch from the host)
    against eager launches: the tiny DiT (N = 256, launch-bound) and the
    30-layer DiT (the bench loop itself)."""
    from token_sparse_denoising_layer_b200.loop import HsaLoop

    def time_replay(lp, reps):
        stream = torch.cuda.current_stream()
        out = []
        for _ in range(reps):
            lp.reset(x0_of[id(lp)], g0_of[id(lp)])
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            lp.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1) / lp.T)
        return float(np.median(out))

    spec = synth.WORKLOADS["tiny_dit"]
    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 0)
    layers = [tuple(torch.from_numpy(lw[k]).to(torch.bfloat16).cuda()
                    for k in ("w_qkv", "w_o", "w_1", "w_2")) for lw in w["layers"]]
    tiny = HsaLoop(sh.N, sh.D, sh.H, sh.F, layers, torch.from_numpy(w["w_in"]).cuda(),
                   torch.from_numpy(w["w_head"]).cuda(), spec["T"], spec["budgets"], counts,
                   shift=spec["shift"])
    tx0 = torch.from_numpy(synth.latent(sh.N, 16, 0)).cuda()
    tg0 = torch.from_numpy(synth.random_split(sh.N, counts, 0)).cuda()
    x0_of = {id(tiny): tx0, id(loop): x0}
    g0_of = {id(tiny): tg0, id(loop): g0}
    tiny.reset(tx0, tg0)
    tiny.run()
    tiny.reset(tx0, tg0)
    tiny_eager = float(np.median(time_steps(tiny, 5 * spec["T"], torch)))
    tiny.capture()
    tiny_graph = time_replay(tiny, 5)
    loop.reset(x0, g0)
    loop.capture()
    big_graph = time_replay(loop, 2)
    out = {"tiny_dit": {"eager_ms_per_step": round(tiny_eager, 4),
                        "graph_ms_per_step": round(tiny_graph, 4),
                        "launches_per_loop": tiny.graph_launches},
           "dit30_1536": {"eager_ms_per_step": round(eager_ms, 3),
                          "graph_ms_per_step": round(big_graph, 3),
                          "launches_per_loop": loop.graph_launches}}
    tiny.close()
    loop.graph = None
    return out


def conditioned_loop(torch, abi, loop, x0, g0, eager_ms):
    """The 30-layer DiT loop with conditioned blocks: every layer modulated
    with vectors that change each iteration, and cross-attention to 512 text
    tokens in every layer; ms per step over the whole 40-step loop."""
    T, L, D, n_txt = loop.T, loop.L, loop.D, 512
    g = torch.Generator(device="cuda")
    g.manual_seed(13)
    rnd = lambda *sh, s=1.0: (torch.randn(sh, generator=g, device="cuda") * s)
    mods = []
    for i in range(T):
        row = []
        for l in range(L):
            m = rnd(6, D, s=0.3)
            m[2] += 1.0
            m[5] += 1.0
            row.append(m.contiguous())
        mods.append(row)
    xa = [abi.cross_attn(rnd(D, D, s=D ** -0.5).to(torch.bfloat16),
                         rnd(D, D, s=D ** -0.5).to(torch.bfloat16),
                         rnd(n_txt, D).to(torch.bfloat16), rnd(n_txt, D).to(torch.bfloat16), n_txt)
          for _ in range(L)]
    conds = [abi.StepCond(mods[i], xa) for i in range(T)]
    loop.reset(x0, g0)
    loop.step(0, True, cond=conds[0])
    loop.reset(x0, g0)
    ts = time_steps(loop, T, torch, per_step_hook=lambda k, i: loop.step(i, True, cond=conds[i]))
    abi.hsa_sync_check(loop.ctx)
    ms = float(np.mean(ts))
    return {"n_txt": n_txt, "ms_per_step": round(ms, 3), "plain_ms_per_step": round(eager_ms, 3),
            "overhead": round(ms / eager_ms - 1.0, 4)}


def oracle_cores() -> dict:
    """Threads the oracle's numpy arithmetic can use: the BLAS pool size
    (threadpoolctl) capped by the CPUs this process may run on."""
    aff = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    blas = None
    try:
        from threadpoolctl import threadpool_info

        pools = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        blas = max(pools) if pools else None
    except Exception:   # noqa: BLE001 - without threadpoolctl the affinity stands
        blas = None
    eff = min(aff, blas) if blas else aff
    return {"cores": eff, "cpus_allowed": aff, "blas_threads": blas,
            "cores_note": "effective = min(CPUs in the process affinity mask, BLAS threads)"}


ORACLE_ROWS = 64   # active rows per sampled oracle layer call (both CPU legs)


def oracle_layer_sample(spec, seed, n_rows=ORACLE_ROWS):
    """State for one sampled oracle layer call of the workload: a layer's
    weights, x and a stale cache at full N, and a function that runs
    layer_forward on `n_rows` random active rows and returns its seconds."""
    from oracle import hsa_oracle as O
    from token_sparse_denoising_layer_b200 import synth

    sh = spec["shape"]
    r = synth.rng(seed)
    D, F, N = sh.D, sh.F, sh.N
    w = {"w_qkv": r.standard_normal((3 * D, D), dtype=np.float32) / np.sqrt(D),
         "w_o": r.standard_normal((D, D), dtype=np.float32) / np.sqrt(D),
         "w_1": r.standard_normal((F, D), dtype=np.float32) / np.sqrt(D),
         "w_2": r.standard_normal((D, F), dtype=np.float32) / np.sqrt(F)}
    x = r.standard_normal((N, D))
    kc, vc = r.standard_normal((N, D)), r.standard_normal((N, D))

    def call():
        idx = np.sort(r.permutation(N)[:n_rows]).astype(np.int32)
        t0 = time.perf_counter()
        O.layer_forward(w, x, idx, kc, vc, sh.H)
        return time.perf_counter() - t0

    return call


ORACLE_WORKLOAD = ("HSA loop, 30-layer DiT: N=32760 (21x30x52), C=16, D=1536, H=12x128, F=8960, "
                   "T=40, shift 5, budgets {40,20,10} at 40/30/30%, regroup by L1 relative "
                   "velocity change")


def oracle_beside(reps=3):
    """The oracle on the host cores for the smaller workloads, timed in the same
    run as the GPU figures for the same work: the whole tiny-DiT loop (ms per
    step), and one re-grouping (score + ranking) and one cached-Euler update at
    N = 32760 (ms per call).  Median of `reps`."""
    from oracle import hsa_oracle as O
    from token_sparse_denoising_layer_b200 import synth

    def med(fn):
        ts = []
        for _ in range(reps):
            t0 = time.perf_counter()
            fn()
            ts.append(time.perf_counter() - t0)
        return float(np.median(ts)) * 1e3

    spec = synth.WORKLOADS["tiny_dit"]
    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    w = synth.model_weights(sh, 0)
    x0 = synth.latent(sh.N, 16, 0)
    g0 = synth.random_split(sh.N, counts, 0)
    sig = O.sigma_schedule(spec["T"], spec["shift"])
    tiny = med(lambda: O.run_loop(w, x0, g0, spec["T"], list(spec["budgets"]), counts, sig,
                                  sh.H)) / spec["T"]
    s2 = synth.WORKLOADS["select_euler_32760"]
    N = s2["N"]
    vp, vc, _ = synth.velocity_pair(N, 16, s2["seed"])
    c2 = synth.group_counts(N, s2["fractions"])
    regroup = med(lambda: O.assign_groups(O.l1_relative_change(vp, vc), c2))
    r = synth.rng(3)
    x, vf = (r.standard_normal((N, 16)) for _ in range(2))
    mask = r.random(N) < 0.625
    euler = med(lambda: O.euler_step(x, vc, vp, vf, mask, 0.5, 0.475))
    return {**oracle_cores(), "kind": "oracle",
            "tiny_dit_loop_ms_per_step": round(tiny, 3),
            "regroup_32760_ms": round(regroup, 3),
            "euler_32760_ms": round(euler, 3)}


def cpu_baseline(spec, target_s=12.0):
    """The oracle on the host cores, on a bounded sample: one layer of the
    30-layer DiT for ORACLE_ROWS active rows against the full N = 32760 cache,
    repeated until about `target_s` seconds; extrapolated linearly in the
    active rows to a full step of the loop (cost is O(|A_i|) per layer)."""
    from oracle import hsa_oracle as O
    from token_sparse_denoising_layer_b200 import synth

    sh = spec["shape"]
    call = oracle_layer_sample(spec, 3)
    t0 = time.perf_counter()
    spent = []
    while True:
        spent.append(call())
        if time.perf_counter() - t0 >= target_s:
            break
    per_row_layer_s = float(np.mean(spent)) / ORACLE_ROWS
    counts = synth.group_counts(sh.N, spec["fractions"])
    mean_active = np.mean([O.n_active(i, spec["T"], spec["budgets"], counts)
                           for i in range(spec["T"])])
    ms_step = per_row_layer_s * mean_active * sh.L * 1e3
    return {"value": round(ms_step, 1), "unit": "ms/step", **oracle_cores(), "kind": "oracle",
            "sample": (f"{len(spent)} x oracle layer_forward on {ORACLE_ROWS} active rows vs the "
                       f"full N={sh.N} cache (D={sh.D}, F={sh.F}); "
                       f"{time.perf_counter() - t0:.1f} s; extrapolated (not run in full) "
                       f"x{mean_active:.0f} mean active rows x {sh.L} layers")}


def run_ours(args, rank, world, local, pg):
    import torch

    from token_sparse_denoising_layer_b200 import abi, synth

    torch.cuda.set_device(local)
    spec = synth.WORKLOADS[WORKLOAD]
    sh = spec["shape"]
    loop, x0, g0, counts, layers = build_loop(spec, seed=rank, torch=torch)

    # warm-up, then a fresh loop state for the timed region
    loop.reset(x0, g0)
    for k in range(args.warmup):
        loop.step(k % loop.T)
    abi.hsa_sync_check(loop.ctx)
    loop.reset(x0, g0)
    barrier(pg)
    launches0 = abi.hsa_kernel_launches(loop.ctx)
    # every launch in the timed region is bracketed by CUDA events on the
    # context's stream, so each kernel class's own time inside the step is known
    abi.hsa_kernel_times(loop.ctx)
    abi.hsa_time_kernels(loop.ctx, True)
    with ClockSampler(local) as clk:
        times = time_steps(loop, args.steps, torch)
    kernel_times = abi.hsa_kernel_times(loop.ctx)
    abi.hsa_time_kernels(loop.ctx, False)
    launches = abi.hsa_kernel_launches(loop.ctx) - launches0
    abi.hsa_sync_check(loop.ctx)
    ms_total = max_over_ranks(float(np.sum(times)), pg, torch.device("cuda", local))
    ms_step = ms_total / args.steps
    barrier(pg)

    # dense all-active loop on the same kernels (every token active every step)
    dense = None
    if not args.quick:
        dl = __import__("token_sparse_denoising_layer_b200.loop", fromlist=["HsaLoop"]).HsaLoop(
            sh.N, sh.D, sh.H, sh.F, layers, loop.model._keep[0], loop.model._keep[1], spec["T"],
            [spec["T"]], [sh.N], shift=spec["shift"])
        dl.reset(x0, torch.zeros_like(g0))
        for k in range(2):
            dl.step(k)
        dl.reset(x0, torch.zeros_like(g0))
        dt = time_steps(dl, min(args.steps, 8), torch)
        dense = float(np.mean(dt))
        dl.close()
        del dl

    # end to end through the public call with host buffers: H2D of the latent,
    # the step, D2H of the latent, every step
    # (two pinned host buffers ping-pong, so the latent really travels through host memory)
    x_host = [torch.empty((sh.N, 16), dtype=torch.float32).pin_memory() for _ in range(2)]
    x_host[0].copy_(x0.cpu())
    loop.reset(x0, g0)

    def e2e_hook(k, i):
        loop.x.copy_(x_host[k % 2], non_blocking=True)
        loop.step(i)
        x_host[(k + 1) % 2].copy_(loop.x, non_blocking=True)

    e2e_times = time_steps(loop, args.steps, torch, per_step_hook=e2e_hook)
    e2e_ms = max_over_ranks(float(np.sum(e2e_times)), pg, torch.device("cuda", local)) / args.steps

    # sub-benchmarks: one GPU only (with N ranks, rank 0 alone would hold the
    # others at teardown for minutes)
    sub = {}
    if not args.quick and world == 1:
        sub["attention"] = attention_sweep(torch, abi, synth)
        sub["gemm"] = gemm_sweep(torch, abi, synth, _peaks().get("bf16_tflops", 1590.0))
        sub["euler"] = euler_bandwidth(torch, abi)
        sub["token_kernels_graph"] = token_kernels_graph(torch, abi, synth)
        sub["bandwidth"] = bandwidth_sweep(torch, abi)
        sub["conditioned_layer"] = conditioned_layer(torch, abi)
        sub["presets_dit30"] = preset_sweep(torch, synth, spec, layers, loop.model._keep[0],
                                            loop.model._keep[1])
        sub["dit40"] = dit40_steps(torch, synth)
        sub["conditioned_loop"] = conditioned_loop(torch, abi, loop, x0, g0, ms_step)
        sub["cuda_graph"] = graph_replay(torch, synth, loop, x0, g0, ms_step)

    result = None
    if rank == 0:
        peaks = _peaks()
        hbm = peaks.get("hbm_gbs", 6650.0)
        for grp in ("euler", "bandwidth"):
            for v in sub.get(grp, {}).values():
                v["frac_of_hbm"] = round(v["GBps"] / hbm, 3)
        # In the step: each class's launches as timed by their own CUDA events
        # over the timed region.  A kernel timed inside a long step is compared
        # with the sustained peak; the isolated sweep (sub.attention, 10 launches
        # back to back) with the burst peak.
        # fallbacks when no measured file is present: 1590 TFLOP/s burst, and
        # about 1400 sustained under the 1000 W power cap (earlier measurements
        # on these B200s)
        peak_burst = peaks.get("bf16_tflops", 1590.0)
        peak_sus = peaks.get("bf16_tflops_sustained", 1400.0 if "bf16_tflops" not in peaks
                             else peak_burst)
        in_step = {}
        for cls, v in kernel_times.items():
            e = {"calls_per_step": round(v["calls"] / args.steps, 2),
                 "ms_per_step": round(v["ms"] / args.steps, 3),
                 "share_of_step": round(v["ms"] / float(np.sum(times)), 4)}
            if cls in ("attention", "gemm") and v["ms"] > 0:
                e["tflops"] = round(v["work"] / v["ms"] / 1e9, 1)
                e["frac_of_sustained"] = round(e["tflops"] / peak_sus, 3)
            elif cls == "rows" and v["ms"] > 0:
                e["GBps"] = round(v["work"] / v["ms"] / 1e6, 1)
                e["frac_of_hbm"] = round(e["GBps"] / hbm, 3)
            in_step[cls] = e
        at = kernel_times["attention"]
        a_tf = at["work"] / at["ms"] / 1e9 if at["ms"] > 0 else None
        roof = None
        if a_tf is not None:
            roof = {"bound": "tensor",
                    "kernel": "k_attn<128> + k_attn_combine (active-query attention), every "
                              "launch of the timed steps",
                    "achieved": round(a_tf, 1), "peak": peak_sus, "unit": "TFLOP/s",
                    "frac": round(a_tf / peak_sus, 3),
                    "peak_source": "MEASURED_PEAKS.json bf16_tflops_sustained: the kernel is "
                                   "timed inside the long step (of measured)"
                    if "bf16_tflops_sustained" in peaks else
                    ("fallback 1400 TFLOP/s sustained (of fallback)"
                     if "bf16_tflops" not in peaks else
                     "MEASURED_PEAKS.json bf16_tflops: no sustained figure (of measured)"),
                    "launches": at["calls"],
                    "ms_per_launch": round(at["ms"] / max(at["calls"], 1), 4),
                    "per_launch": "4*|A_i|*N*D FLOP, N = 32760, D = 1536; |A_i| = 32760, "
                                  "22932 or 13104 by iteration (6.594 TFLOP at |A_i| = N)",
                    "burst_peak": peak_burst}
            # bytes of the average attention launch of the step: Q and O rows
            # (2 B x D each per active row) and the K, V cache (2 B x D each per row)
            a_avg = at["work"] / (4.0 * sh.N * sh.D) / max(at["calls"], 1)
            algo_avg = 4.0 * sh.D * (a_avg + sh.N)
            algo_full = 4.0 * sh.D * (sh.N + sh.N)
            t_full = attention_traffic()
            roof["algorithmic_bytes"] = round(algo_avg)
            roof["traffic"] = round(t_full * algo_avg / algo_full) if t_full is not None else None
            roof["traffic_note"] = ("ncu DRAM bytes (read + write) of one launch at |A| = N = 32760 "
                                    f"({t_full} B against {round(algo_full)} B algorithmic), "
                                    "scaled to the step's average launch by its algorithmic bytes"
                                    if t_full is not None else "no capture of the current kernel")
            if "attention" in sub:
                a100 = sub["attention"]["100%"]
                roof["isolated_100pct"] = {"tflops": a100["tflops"],
                                           "frac_of_burst": round(a100["tflops"] / peak_burst, 3)}
        result = {
            "metric": METRIC, "value": round(ms_step, 3), "unit": "ms/step", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random N(0,1/fan_in) weights, x ~ N(0,1))",
            "config": {"workload": ORACLE_WORKLOAD,
                       "global_batch": 1, "seq_len": sh.N, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (>8 GB touched per step)",
                       "step": "one global iteration i = k mod 40; 40 steps = one loop",
                       "value": "ms per step, max over ranks; each rank runs its own replica"},
            "dense_ms_per_step": round(dense, 3) if dense else None,
            "hsa_vs_dense": round(ms_step / dense, 3) if dense else None,
            "mean_active_fraction": 0.625,
            "gpu_launches": launches * world,
            "job_steps_per_s": round(world * 1000.0 / ms_step, 3),
            "e2e": {"value": round(e2e_ms, 3), "unit": "ms/step",
                    "h2d_bytes_per_step": sh.N * 16 * 4, "d2h_bytes_per_step": sh.N * 16 * 4},
            "clocks": clk.summary(),
            "roofline": roof,
            "in_step_kernels": in_step,
            "sub": sub,
        }
        if not args.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = cpu_baseline(spec)
            if sub:
                # the oracle beside the GPU on the smaller workloads; the GPU
                # figures for the same work are sub.cuda_graph.tiny_dit and
                # sub.token_kernels_graph["32760"]
                sub["oracle_beside"] = oracle_beside()
    loop.close()
    return result


def run_shard(args, rank, world, local, pg):
    """One 30-layer DiT loop split over the ranks (sequence-sharded step):
    every rank runs its chunk of each step's active list; ms per step is the
    max over ranks of the device-timed region."""
    import torch

    from token_sparse_denoising_layer_b200 import abi, synth
    from token_sparse_denoising_layer_b200.shard import (ShardRank, link_ipc, link_local,
                                                         run_dist, run_local)

    torch.cuda.set_device(local)
    spec = synth.WORKLOADS[WORKLOAD]
    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    # the same seed on every rank: one model, one latent, one initial split
    layers = [synth.device_layer_weights(sh.D, sh.F, l) for l in range(sh.L)]
    wf = synth.model_weights(synth.ModelShape(sh.N, sh.C, sh.D, sh.H, 64, 0), 0)
    rk = ShardRank(rank, world, sh.N, sh.D, sh.H, sh.F, layers,
                   torch.from_numpy(wf["w_in"]).cuda(), torch.from_numpy(wf["w_head"]).cuda(),
                   spec["T"], spec["budgets"], counts, shift=spec["shift"])
    if args.kv_exchange == "peer":
        if pg is not None:
            link_ipc(rk, pg)
        else:
            link_local([rk])
    x0 = torch.from_numpy(synth.latent(sh.N, 16, 0)).cuda()
    g0 = torch.from_numpy(synth.random_split(sh.N, counts, 0)).cuda()

    def step(i):
        if pg is not None:
            run_dist(rk.steps(i, True))
        else:
            run_local([rk.steps(i, True)])

    def timed(k_steps, hook=None):
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(k_steps)]
        torch.cuda.synchronize()
        for k in range(k_steps):
            ev[k][0].record(stream)
            (hook or (lambda kk, ii: step(ii)))(k, k % spec["T"])
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    rk.reset(x0, g0)
    for k in range(args.warmup):
        step(k % spec["T"])
    abi.hsa_sync_check(rk.ctx)
    rk.reset(x0, g0)
    barrier(pg)
    launches0 = abi.hsa_kernel_launches(rk.ctx)
    with ClockSampler(local) as clk:
        times = timed(args.steps)
    launches = abi.hsa_kernel_launches(rk.ctx) - launches0
    abi.hsa_sync_check(rk.ctx)
    dev = torch.device("cuda", local)
    ms_step = max_over_ranks(float(np.sum(times)), pg, dev) / args.steps
    barrier(pg)
    x_host = [torch.empty((sh.N, 16), dtype=torch.float32).pin_memory() for _ in range(2)]
    x_host[0].copy_(x0.cpu())
    rk.reset(x0, g0)

    def e2e_hook(k, i):
        rk.x.copy_(x_host[k % 2], non_blocking=True)
        step(i)
        x_host[(k + 1) % 2].copy_(rk.x, non_blocking=True)

    e2e_ms = max_over_ranks(float(np.sum(timed(args.steps, e2e_hook))), pg, dev) / args.steps
    launches_all = max_over_ranks(float(launches), pg, dev) * world
    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": round(ms_step, 3), "unit": "ms/step", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
            "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random N(0,1/fan_in) weights, x ~ N(0,1))",
            "config": {"workload": ORACLE_WORKLOAD,
                       "global_batch": 1, "seq_len": sh.N,
                       "parallelism": f"sequence-shard x{world} (active-list chunks, " + (
                           "K|V all-gather per layer" if args.kv_exchange == "gather" else
                           "K|V stored into every rank's cache by the QKV epilogue + barrier "
                           "per layer") + ", velocity all-reduce per step)",
                       "l2": "inputs larger than L2 (>8 GB touched per step)",
                       "step": "one global iteration i = k mod 40; 40 steps = one loop",
                       "value": "ms per step of the one loop, max over ranks"},
            "mean_active_fraction": 0.625,
            "gpu_launches": int(launches_all),
            "e2e": {"value": round(e2e_ms, 3), "unit": "ms/step",
                    "h2d_bytes_per_step": sh.N * 16 * 4, "d2h_bytes_per_step": sh.N * 16 * 4},
            "clocks": clk.summary(),
        }
    rk.close()
    return result


# --------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step a bounded sample of the
    same workload (ORACLE_ROWS active rows of one layer against the full cache,
    the same sample as cpu_baseline), extrapolated to that iteration's |A_i|
    rows x 30 layers."""
    if rank != 0:
        return None
    from oracle import hsa_oracle as O
    from token_sparse_denoising_layer_b200 import synth

    spec = synth.WORKLOADS[WORKLOAD]
    sh = spec["shape"]
    counts = synth.group_counts(sh.N, spec["fractions"])
    call = oracle_layer_sample(spec, 4)
    t_start = time.perf_counter()
    per_step = []
    for k in range(args.warmup + args.steps):
        i = k % spec["T"]
        a = O.n_active(i, spec["T"], spec["budgets"], counts)
        t = call()
        if k >= args.warmup:
            per_step.append(t / ORACLE_ROWS * a * sh.L * 1e3)
    ms = float(np.mean(per_step))
    return {"impl": "reference", "metric": METRIC, "value": round(ms, 1), "unit": "ms/step",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 1), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": ORACLE_WORKLOAD, "global_batch": 1, "seq_len": sh.N,
                       "parallelism": "replicas x1 (oracle on rank 0 only)"},
            "cpu_baseline": {"value": round(ms, 1), "unit": "ms/step", **oracle_cores(),
                             "kind": "oracle",
                             "sample": f"per step: oracle layer_forward on {ORACLE_ROWS} active "
                                       f"rows of one layer vs the full N={sh.N} cache, "
                                       f"extrapolated (not run in full) by |A_i| x {sh.L} layers; "
                                       f"{time.perf_counter() - t_start:.1f} s for the run"},
            "e2e": {"value": round(ms, 1), "unit": "ms/step", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def profile_case(name):
    """A few launches of one kernel at the workload's shapes, for ncu captures."""
    import torch

    from token_sparse_denoising_layer_b200 import abi

    N, D, H, F = 32760, 1536, 12, 8960
    ctx = abi.hsa_create(N=N, D=D, H=H, F=F, L=1, T=40, budgets=[40, 20, 10],
                         counts=[13104, 9828, 9828])
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    rnd = lambda *s: torch.randn(s, generator=g, device="cuda")
    if name == "attention":
        kc, vc, q = (rnd(N, D).to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        for _ in range(3):
            abi.hsa_attention(ctx, q, N, kc, vc, o)
    elif name == "gemm":
        u = rnd(N, D).to(torch.bfloat16)
        w1 = (rnd(F, D) / D ** 0.5).to(torch.bfloat16)
        out = torch.empty((N, F), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            abi.hsa_linear(ctx, u, N, D, w1, F, out)
    elif name == "euler":
        x, vh, vp, vf = (rnd(N, 16) for _ in range(4))
        m = (torch.rand(N, device="cuda") < 0.6).to(torch.uint8)
        for _ in range(3):
            abi.hsa_euler_step(ctx, x, vh, vp, vf, m, 0.5, 0.45)
    elif name == "rows":
        # the HBM-bound row kernels on inputs larger than L2, two launches each:
        # cached Euler over 1M tokens (256 MB of latent and velocities), the LN
        # gather of all 32760 rows (D = 1536, 201 MB of fp32 rows), and the KV
        # scatter of 16380 fresh rows into 32760 x 1536 caches
        Ne = 1024 * 1024
        ce = abi.hsa_create(N=Ne, D=128, H=1, F=64, L=0, T=40, budgets=[40, 20, 10],
                            counts=[Ne - 2 * (Ne * 3 // 10), Ne * 3 // 10, Ne * 3 // 10])
        x, vh, vp, vf = (rnd(Ne, 16) for _ in range(4))
        m = (torch.rand(Ne, device="cuda") < 0.625).to(torch.uint8)
        for _ in range(2):
            abi.hsa_euler_step(ce, x, vh, vp, vf, m, 0.5, 0.45)
        abi.hsa_sync_check(ce)
        ce.close()
        del x, vh, vp, vf, m
        h = rnd(N, D)
        u = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
        idx = torch.arange(N, dtype=torch.int32, device="cuda")
        for _ in range(2):
            abi.hsa_ln_gather(ctx, h, idx, N, u)
        del h, u, idx
        a = N // 2
        kr, vr = (rnd(a, D).to(torch.bfloat16) for _ in range(2))
        kc, vc = (torch.zeros((N, D), dtype=torch.bfloat16, device="cuda") for _ in range(2))
        ik = torch.sort(torch.randperm(N, generator=g, device="cuda")[:a]).values.to(torch.int32)
        for _ in range(2):
            abi.hsa_kv_scatter(ctx, kr, vr, ik, a, kc, vc)
    elif name == "tokens":
        # the per-token kernels at the 21x45x80 latent (N = 75600, {40,20,10} at
        # 40/30/30%), two launches each: schedule (iteration 4: groups 1 and 2
        # active), the Euler pass that writes the scores, the standalone score,
        # and the selection (cluster cut search + assignment)
        from token_sparse_denoising_layer_b200 import synth

        spec = synth.WORKLOADS["select_euler_75600"]
        Nt = spec["N"]
        counts = synth.group_counts(Nt, spec["fractions"])
        ct = abi.hsa_create(N=Nt, D=128, H=1, F=64, L=0, T=spec["T"], budgets=spec["budgets"],
                            counts=counts)
        vp, vc, _ = synth.velocity_pair(Nt, 16, spec["seed"])
        v_prev, v_cur = torch.from_numpy(vp).cuda(), torch.from_numpy(vc).cuda()
        gg = torch.from_numpy(synth.random_split(Nt, counts, spec["seed"])).cuda()
        mask = torch.zeros(Nt, dtype=torch.uint8, device="cuda")
        idx = torch.zeros(Nt, dtype=torch.int32, device="cuda")
        score = torch.zeros(Nt, dtype=torch.float32, device="cuda")
        x, vf = rnd(Nt, 16), rnd(Nt, 16)
        for _ in range(2):
            abi.hsa_schedule(ct, 4, gg, mask, idx)
        for _ in range(2):
            abi.hsa_euler_step_score(ct, x, v_cur, v_prev, vf, mask, 0.5, 0.45, score)
        for _ in range(2):
            abi.hsa_score(ct, v_prev, v_cur, score)
        for _ in range(2):
            abi.hsa_select_from_score(ct, score, gg)
        abi.hsa_sync_check(ct)
        ct.close()
    elif name == "embed_head":
        # embed and velocity head of the 30-layer DiT's 40%-active iterations
        from token_sparse_denoising_layer_b200 import synth

        a = 13104
        w_in, w_head = rnd(D, 16) / 4.0, rnd(16, D) / D ** 0.5
        xl = rnd(N, 16)
        h = torch.zeros((N, D), dtype=torch.float32, device="cuda")
        vf = torch.zeros((N, 16), dtype=torch.float32, device="cuda")
        idx = torch.from_numpy(synth.random_active_set(N, a, 1)).cuda()
        for _ in range(2):
            abi.hsa_embed(ctx, w_in, xl, idx, a, h)
        for _ in range(2):
            abi.hsa_head(ctx, w_head, h, idx, a, vf)
    elif name == "gemm_epi":
        # the step's fused-epilogue GEMMs at 100% active (M = 32760): QKV with
        # the KV-cache scatter, out-projection with the residual add into
        # scattered rows, and the MLP (GELU epilogue up, residual add down)
        from token_sparse_denoising_layer_b200 import synth

        u = rnd(N, D).to(torch.bfloat16)
        w_qkv, w_o = (rnd(3 * D, D) / D ** 0.5).to(torch.bfloat16), (rnd(D, D) / D ** 0.5).to(torch.bfloat16)
        w1, w2 = (rnd(F, D) / D ** 0.5).to(torch.bfloat16), (rnd(D, F) / F ** 0.5).to(torch.bfloat16)
        kc, vc = (torch.zeros((N, D), dtype=torch.bfloat16, device="cuda") for _ in range(2))
        q = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
        x = rnd(N, D)
        idx = torch.from_numpy(synth.random_active_set(N, N, 1)).cuda()
        for _ in range(2):
            abi.hsa_qkv_project(ctx, w_qkv, u, idx, N, q, kc, vc)
        for _ in range(2):
            abi.hsa_out_proj_residual(ctx, w_o, u, idx, N, x)
        for _ in range(2):
            abi.hsa_mlp_residual(ctx, w1, w2, x, idx, N)
    elif name == "qkv_peers":
        # one rank's QKV launch of a 4-way sequence-sharded step at 100% active
        # (8190 rows of 32760), storing its fresh K/V rows into 4 cache copies
        # (all in this GPU's memory here)
        G, M = 4, N // 4
        u = rnd(M, D).to(torch.bfloat16)
        w_qkv = (rnd(3 * D, D) / D ** 0.5).to(torch.bfloat16)
        kcs = [torch.zeros((N, D), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        vcs = [torch.zeros((N, D), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        q = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
        idx = torch.arange(M, dtype=torch.int32, device="cuda")  # rank 0's chunk of A_i
        for _ in range(2):
            abi.hsa_qkv_project_peers(ctx, w_qkv, u, idx, M, q, kcs, vcs)
    elif name == "gemm1":
        # the 1-CTA GEMM, as the tiny DiT (N = 256, D = 128, F = 512) runs it
        c1 = abi.hsa_create(N=256, D=128, H=2, F=512, L=1, T=1, budgets=[1], counts=[256])
        u = rnd(256, 128).to(torch.bfloat16)
        w = (rnd(384, 128) / 128 ** 0.5).to(torch.bfloat16)
        out = torch.empty((256, 384), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            abi.hsa_linear(c1, u, 256, 128, w, 384, out)
        abi.hsa_sync_check(c1)
        c1.close()
    abi.hsa_sync_check(ctx)
    ctx.close()
    return 0


def main():
    args = parse()
    if args.profile_case:
        return profile_case(args.profile_case)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        res = run_reference(args, rank, world)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
        return 0
    rank, world, local, pg = dist_setup(args.gpus)
    res = (run_shard if args.mode == "shard" else run_ours)(args, rank, world, local, pg)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
