#!/usr/bin/env python
"""Benchmark: Wan2.2 DiT self-attention hot path on B200.

One step = the whole path on one batch of the workload: Q/K RMSNorm + bf16
round + 3D RoPE in place on the packed [Q|K|V] buffer, then softmax attention
(``wan_dit_attn``: two kernels chained on one stream). Default workload: the
Wan2.2-A14B 832x480, 81-frame clip with its CFG batch of 2 (grid 21x30x52 =
32760 tokens, 40 heads x 128), synthetic seeded data.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). ``value`` is attention TFLOP/s over whole steps
(4*B*heads*S^2*128 FLOP per step / device time per step, all ranks); the
line also carries per-kernel figures (attention TFLOP/s, norm+RoPE GB/s),
the roofline of the dominant kernel, an end-to-end figure through host
buffers, clocks seen during the timed region, and the oracle's CPU time.
With N > 1 every rank runs an independent replica (the path does not shard):
scaling is weak and ``value`` sums all ranks' work over the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle (the reference arm) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import wan_inputs as wi  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRC = os.path.join(ROOT, "video_diffusion_transformer_packed_b200", "csrc", "attn_fwd.cu")
NORM_SRC = os.path.join(ROOT, "video_diffusion_transformer_packed_b200", "csrc", "qk_norm_rope.cu")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=wi.BENCH_WORKLOAD.name, choices=sorted(wi.BY_NAME))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-skip", action="store_true", help="skip the Skip-Softmax side measurement")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 side measurement")
    ap.add_argument("--no-proj", action="store_true", help="skip the QKV projection side measurement")
    ap.add_argument("--no-ring", action="store_true", help="skip the ring context-parallel side measurement")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


SM100_HDR = os.path.join(ROOT, "video_diffusion_transformer_packed_b200", "csrc", "sm100.cuh")


def kernel_sha256(src):
    """sha256 of a kernel's source followed by the shared PTX-wrapper header:
    both decide the compiled kernel."""
    h = hashlib.sha256()
    for path in (src, SM100_HDR):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(kernel: str, src: str, tokens: int):
    """DRAM bytes per launch for a launch over `tokens` tokens (batch x S), from
    the committed ncu summary of `kernel` (bytes per token; both kernels move
    a fixed number of bytes per token), if the summary was taken on the
    current kernel source; else None."""
    pdir = os.path.join(ROOT, "profiles")
    for fn in sorted(os.listdir(pdir)) if os.path.isdir(pdir) else []:
        if not fn.startswith(kernel):
            continue
        txt = open(os.path.join(pdir, fn)).read()
        m_sha = re.search(r"kernel_source_sha256\s*[:=]\s*([0-9a-f]{64})", txt)
        m_tr = re.search(r"traffic_per_token_bytes\s*[:=]\s*([0-9.eE+]+)", txt)
        if m_sha and m_tr and m_sha.group(1) == kernel_sha256(src):
            return float(m_tr.group(1)) * tokens
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.device = device

    def start(self):
        try:
            props = torch.cuda.get_device_properties(self.device)
            ident = "GPU-" + str(props.uuid) if getattr(props, "uuid", None) else str(self.device)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", ident], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s, p in zip(sm, power) if p > 0.5 * max(power)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w, qkv, gq, gk, target_s: float):
    """Times the oracle on a bounded sample of the workload: attention for n
    query rows spread over (batch, head) pairs plus norm+RoPE for the matching
    share of tokens (n / heads). Returns (TFLOP/s, seconds, description)."""
    import numpy as np
    import oracle
    S, H = w.seq_len, w.heads
    g = torch.Generator().manual_seed(1234)

    def rows_for(n):
        b = torch.randint(w.batch, (n,), generator=g)
        h = torch.randint(H, (n,), generator=g)
        i = torch.randint(S, (n,), generator=g)
        return np.stack([b.numpy(), h.numpy(), i.numpy()], axis=1).astype(np.int64)

    def run(n):
        rows = rows_for(n)
        ntok = max(1, n // H)
        toks = np.stack([rows[:ntok, 0], rows[:ntok, 2]], axis=1)
        t0 = time.perf_counter()
        oracle.qk_norm_rope_tokens(qkv, w.grid, H, gq, gk, wi.EPS, wi.THETA, toks)
        oracle.attention_rows(qkv, H, rows, 1.0 / 128 ** 0.5)
        return time.perf_counter() - t0

    oracle.build()
    run(8)  # warm the library and threads
    n0 = 16
    t = run(n0)
    n = int(max(n0, min(200000, n0 * target_s / max(t, 1e-6))))
    t = run(n)
    flop = n * 4.0 * S * wi.HEAD_DIM
    desc = (f"{n} query rows of random (batch, head) pairs at S={S} plus norm+RoPE of {max(1, n // H)} "
            f"tokens (the same share of the step), fp64 oracle")
    return flop / t / 1e12, t, desc


def max_over_ranks(value: float, device, pg) -> float:
    """Largest `value` over all ranks (identity without a process group)."""
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flop_per_step: float, steps: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank's steps over the slowest rank's time."""
    return world * flop_per_step * steps / (ms / 1e3) / 1e12


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# -------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = wi.BY_NAME[args.workload]
    qkv, gq, gk = wi.inputs_for(w, seed=0)
    per_step = min(20.0, max(1.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, times, desc = [], [], ""
    for k in range(args.warmup + args.steps):
        v, t, desc = oracle_sample(w, qkv, gq, gk, per_step)
        if k >= args.warmup:
            vals.append(v)
            times.append(t)
    value = statistics.mean(vals)
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": "self-attn TFLOP/s (% of B200 bf16 peak) at Wan 480p/81f; norm+RoPE GB/s",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.mean(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        # the GPU arm's workload keys, plus what this arm actually timed
        "config": {**w.describe(), "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single",
                   "step": "norm+RoPE and attention of the step, fp64 oracle on a bounded sample", "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- our arm
def run_ours(args):
    import video_diffusion_transformer_packed_b200 as wan
    from video_diffusion_transformer_packed_b200 import build as wan_build
    from video_diffusion_transformer_packed_b200 import sp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        pg = dist
    if rank == 0:
        wan_build.build()
    if pg is not None:
        pg.barrier()
    wan.load_library()

    w = wi.BY_NAME[args.workload]
    qkv_h, gq_h, gk_h = wi.inputs_for(w, seed=0)
    qkv_pinned = torch.empty_like(qkv_h).pin_memory()
    qkv_pinned.copy_(qkv_h)
    pristine = qkv_pinned.to(dev)
    gq, gk = gq_h.to(dev), gk_h.to(dev)
    out = torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # The path works in place, so every timed step gets its own fresh copy of
    # the seeded input (re-normalising the same buffer again and again drifts
    # the data away from the workload's distribution). Copies are refreshed
    # outside the timed region; a buffer serves at most one timed step.
    nbuf = max(1, min(args.steps, int(os.environ.get("WAN_BENCH_BUFFERS", "32"))))
    bufs = [torch.empty_like(pristine) for _ in range(nbuf)]

    def refresh():
        with torch.cuda.stream(stream):
            for b_ in bufs:
                b_.copy_(pristine)
        stream.synchronize()

    def step(k):
        wan.dit_attn(bufs[k % nbuf], w.grid, w.heads, gq, gk, out=out, stream=stream)

    refresh()
    with torch.cuda.stream(stream):
        for k in range(max(3, args.warmup)):
            step(k)
    stream.synchronize()
    refresh()
    if wan.device_error(stream) != 0:
        raise SystemExit("attention kernel reported a device timeout during warm-up")

    # ---- timed region: K whole steps, barrier + sync on both sides, device events
    sampler = ClockSampler(local)
    sampler.start()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dev, pg)
    if wan.device_error(stream) != 0:
        raise SystemExit("attention kernel reported a device timeout during the timed region")
    ms_step = ms / args.steps
    value = job_throughput(world, w.attn_flop, args.steps, ms)

    # ---- per-kernel durations on the launching stream (separate calls, same work)
    refresh()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * args.steps)]
    for k in range(args.steps):
        ev[3 * k].record(stream)
        wan.qk_norm_rope(bufs[k % nbuf], w.grid, w.heads, gq, gk, stream=stream)
        ev[3 * k + 1].record(stream)
        wan.self_attention(bufs[k % nbuf], w.heads, out=out, stream=stream)
        ev[3 * k + 2].record(stream)
    stream.synchronize()
    t_norm = statistics.mean(ev[3 * k].elapsed_time(ev[3 * k + 1]) for k in range(args.steps))
    t_attn = statistics.mean(ev[3 * k + 1].elapsed_time(ev[3 * k + 2]) for k in range(args.steps))
    attn_tflops = w.attn_flop / (t_attn / 1e3) / 1e12
    norm_gbs = w.norm_rope_bytes / (t_norm / 1e3) / 1e9

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # wan_dit_attn_host: each step's input arrives from pinned host memory
        # and its output returns to pinned host memory, the copies overlapped
        # with the kernels inside the library; every byte of both crosses PCIe
        # inside the timed region. Two device buffer sets alternate between
        # steps, so a step's input transfer also overlaps the previous step's
        # kernels (WAN_HOST_OVERLAP_INPUT).
        sets = [(bufs[0], out), (bufs[1] if nbuf > 1 else torch.empty_like(bufs[0]), torch.empty_like(out))]
        outs_pinned = [torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for k in range(args.warmup + args.steps):
            if k == args.warmup:
                stream.synchronize()
                h0.record(stream)
            qd, od = sets[k % 2]
            wan.dit_attn_host(qkv_pinned, w.grid, w.heads, gq, gk, out_host=outs_pinned[k % 2], qkv_dev=qd,
                              out_dev=od, overlap_input=True, stream=stream)
        h1.record(stream)
        stream.synchronize()
        qkv = bufs[0]
        e2e_ms = max_over_ranks(h0.elapsed_time(h1), dev, pg)
        e2e = {"value": job_throughput(world, w.attn_flop, args.steps, e2e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": qkv.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
               "ms_per_step": e2e_ms / args.steps}

    # ---- Skip-Softmax side measurement (not the headline): same shape, inputs
    # with local, peaked attention (wan_inputs.local_peaked_qkv), dense kernel
    # vs threshold mode, device time of one launch each, skipped fractions
    # from the kernel's own counters.
    skip = None
    if not args.no_skip:
        loc = wi.local_peaked_qkv(w.batch, w.seq_len, w.heads, seed=5).to(dev)
        n_t = (w.seq_len + 127) // 128
        reps = 3

        def timed(thr):
            with torch.cuda.stream(stream):
                wan.self_attention_sparse(loc, w.heads, thr, out=out, stream=stream)
            wan.skip_stats(stream)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                wan.self_attention_sparse(loc, w.heads, thr, out=out, stream=stream)
            b_.record(stream)
            b_.synchronize()
            tiles, prods = wan.skip_stats(stream)
            return a.elapsed_time(b_) / reps, tiles / reps, prods / reps

        dense_ms, _, _ = timed(0.0)
        skip = {"workload": "local peaked synthetic (each query alpha=0.6 times a key within 8 tokens), "
                            + w.name, "dense_ms": dense_ms, "points": []}
        for thr in (0.02, 0.05):
            ms_, tiles, prods = timed(thr)
            skip["points"].append({"threshold": thr, "ms": ms_, "speedup_vs_dense": dense_ms / ms_,
                                   "group_tiles_skipped": tiles / (w.batch * w.heads * 4 * n_t * n_t),
                                   "products_skipped": prods / (w.batch * w.heads * n_t * n_t)})
        del loc

    # ---- FP8 (e4m3) side measurement (not the headline): the normalised
    # buffer of a step, per-tensor scales amax/448, the quantisation and the
    # FP8 attention timed separately, and the FP8 output's divergence from
    # the bf16 kernel's on the same buffer.
    fp8 = None
    if not args.no_fp8:
        src = bufs[0]  # normalised by the per-kernel pass above
        amax_d = wan.qkv_amax(src, w.heads, stream=stream)
        stream.synchronize()  # the maxima are written on `stream`; read them only after it
        amax = amax_d.cpu().numpy().astype("float32")
        sc = [float(a) / 448.0 for a in amax]
        inv = [448.0 / float(a) for a in amax]
        qk8, v8t = wan.quantize_fp8(src, w.heads, inv, stream=stream)
        out8 = torch.empty_like(out)
        wan.self_attention_fp8(qk8, v8t, w.heads, sc, out=out8, stream=stream)
        wan.self_attention(src, w.heads, out=out, stream=stream)
        stream.synchronize()
        rel = float((out8.float() - out.float()).norm() / out.float().norm())

        def timed_ms(fn, reps=3):
            fn()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b_.record(stream)
            b_.synchronize()
            return a.elapsed_time(b_) / reps

        q_ms = timed_ms(lambda: wan.quantize_fp8(src, w.heads, inv, qk8, v8t, stream=stream))
        a_ms = timed_ms(lambda: wan.self_attention_fp8(qk8, v8t, w.heads, sc, out=out8, stream=stream))
        if wan.device_error(stream) != 0:
            raise SystemExit("FP8 attention reported a device timeout")
        fp8 = {"scales": "per tensor, amax/448", "quantize_ms": q_ms, "attention_ms": a_ms,
               "attn_tflops_equiv": w.attn_flop / (a_ms / 1e3) / 1e12,
               "path_tflops_equiv": w.attn_flop / ((q_ms + a_ms) / 1e3) / 1e12,
               "rel_fro_vs_bf16": rel}
        del qk8, v8t, out8

    # ---- QKV projection side measurement (not the headline): the GEMM that
    # produces the packed buffer (tokens x D -> tokens x 3D, seeded synthetic
    # activations and weights), with and without its norm statistic, cuBLAS
    # on the same operands for reference, and norm+RoPE fed by the statistic
    # against the reducing kernel on the same buffer.
    proj = None
    if not args.no_proj:
        M, D = w.batch * w.seq_len, w.dim
        gen = torch.Generator(device=dev).manual_seed(11)
        xact = torch.randn(M, D, device=dev, generator=gen).to(torch.bfloat16)
        wqkv = (torch.randn(3 * D, D, device=dev, generator=gen) / D ** 0.5).to(torch.bfloat16)
        yqkv = bufs[0]

        def timed_p(fn, reps=3):
            fn()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b_.record(stream)
            b_.synchronize()
            return a.elapsed_time(b_) / reps

        g_ms = timed_p(lambda: wan.linear(xact, wqkv, yqkv, stream=stream))
        stats_box = {}

        def with_stats():
            _, stats_box["s"] = wan.linear(xact, wqkv, yqkv, stat_cols=2 * D, stream=stream)

        gs_ms = timed_p(with_stats)
        with torch.cuda.stream(stream):
            cb_ms = timed_p(lambda: torch.matmul(xact, wqkv.t(), out=yqkv.view(M, 3 * D)))
        with_stats()
        ns_ms = timed_p(lambda: wan.qk_norm_rope_stats(yqkv, w.grid, w.heads, gq, gk, stats_box["s"], stream=stream))
        n_ms = timed_p(lambda: wan.qk_norm_rope(yqkv, w.grid, w.heads, gq, gk, stream=stream))
        if wan.device_error(stream) != 0:
            raise SystemExit("projection kernels reported a device timeout")
        pflop = 2.0 * M * D * 3 * D
        # the output projection after the attention: tokens x D -> D
        wout = (torch.randn(D, D, device=dev, generator=gen) / D ** 0.5).to(torch.bfloat16)
        yout = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
        attn_in = out.view(M, D)
        o_ms = timed_p(lambda: wan.linear(attn_in, wout, yout, stream=stream))
        with torch.cuda.stream(stream):
            ocb_ms = timed_p(lambda: torch.matmul(attn_in, wout.t(), out=yout))
        if wan.device_error(stream) != 0:
            raise SystemExit("projection kernels reported a device timeout")
        oflop = 2.0 * M * D * D
        proj = {"shape": f"{M} x {D} -> {3 * D}", "gemm_ms": g_ms, "gemm_tflops": pflop / (g_ms / 1e3) / 1e12,
                "gemm_with_stats_ms": gs_ms, "cublas_ms": cb_ms, "cublas_tflops": pflop / (cb_ms / 1e3) / 1e12,
                "norm_from_stats_ms": ns_ms, "norm_from_stats_gbs": w.norm_rope_bytes / (ns_ms / 1e3) / 1e9,
                "norm_reducing_ms": n_ms,
                "out_projection": {"shape": f"{M} x {D} -> {D}", "ms": o_ms, "tflops": oflop / (o_ms / 1e3) / 1e12,
                                   "cublas_ms": ocb_ms, "cublas_tflops": oflop / (ocb_ms / 1e3) / 1e12}}
        del xact, wqkv, stats_box, wout, yout

    # ---- ring context parallelism, compute side (not the headline): the
    # rounds of 8 ranks run one after another on this GPU, each "remote" K|V
    # chunk a local buffer; partial-state attention per round, merge per
    # round, finalise per rank. Against the dense kernel on the same buffer:
    # the cost of cutting the keys into chunks and merging the states. The
    # NVLink exchange itself needs several GPUs and is not measured here.
    ring = None
    if not args.no_ring and w.seq_len % 8 == 0:
        nr = 8
        src = bufs[0]
        s_l = w.seq_len // nr
        shards = [src[:, r * s_l:(r + 1) * s_l].contiguous() for r in range(nr)]
        chunks = [sh[..., w.dim:].contiguous() for sh in shards]
        states = [(torch.empty((w.batch, s_l, w.heads, 128), dtype=torch.float32, device=dev),
                   torch.empty((w.batch, s_l, w.heads, 2), dtype=torch.float32, device=dev)) for _ in range(2)]
        outs_r = [torch.empty((w.batch, s_l, w.dim), dtype=torch.bfloat16, device=dev) for _ in range(nr)]

        def ring_all():
            # round 0 writes the state, later rounds merge into it in the
            # attention's epilogue, the final merge normalises it
            for r in range(nr):
                acc = states[0]
                for i, c in enumerate(sp.ring_order(nr, r)):
                    wan.self_attention_partial(shards[r], w.heads, chunks[c], o=acc[0], ml=acc[1], stream=stream,
                                               accumulate=i > 0)
                wan.attention_merge(acc[0], acc[1], out=outs_r[r], stream=stream)

        def timed_r(fn, reps=2):
            fn()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b_.record(stream)
            b_.synchronize()
            return a.elapsed_time(b_) / reps

        r_ms = timed_r(ring_all)
        d_ms = timed_r(lambda: wan.self_attention(src, w.heads, out=out, stream=stream))
        acc, part = states
        wan.self_attention_partial(shards[0], w.heads, chunks[1], o=part[0], ml=part[1], stream=stream)
        m_ms = timed_r(lambda: wan.attention_merge(acc[0], acc[1], part[0], part[1], stream=stream), reps=10)
        if wan.device_error(stream) != 0:
            raise SystemExit("ring kernels reported a device timeout")
        units = w.batch * s_l * w.heads
        merge_bytes = units * (3 * 128 * 4 + 3 * 8)  # read both states, write the accumulator
        ring = {"ranks_simulated": nr, "chunk_tokens": s_l, "all_ranks_ms": r_ms, "dense_ms": d_ms,
                "efficiency_vs_dense": d_ms / r_ms, "merge_ms": m_ms,
                "merge_gbs": merge_bytes / (m_ms / 1e3) / 1e9,
                "launches": nr * (nr + 1), "rounds_after_the_first": "merged in the attention's epilogue"}
        del shards, chunks, states, outs_r

    peaks, peak_src = load_peaks()
    # The attention is timed launch by launch (CUDA events around each
    # launch): the burst figure is its denominator; the sustained one (a
    # seconds-long GEMM loop under the power cap) is given beside it.
    tensor_peak = peaks["bf16_tflops"]
    roofline = {
        "kernel": "attn_fwd", "bound": "tensor", "achieved": attn_tflops, "peak": tensor_peak,
        "unit": "TFLOP/s", "frac": attn_tflops / tensor_peak,
        "traffic": profiled_traffic("attn_fwd", ATTN_SRC, w.batch * w.seq_len),
        "peak_source": f"{peak_src} bf16 burst (kernel timed per launch)",
        "frac_of_sustained_peak": attn_tflops / peaks["bf16_tflops_sustained"],
        "algorithmic_flop_per_launch": w.attn_flop, "avg_launch_ms": t_attn,
    }
    norm_roofline = {
        "kernel": "qk_norm_rope", "bound": "hbm", "achieved": norm_gbs, "peak": peaks["hbm_gbs"],
        "unit": "GB/s", "frac": norm_gbs / peaks["hbm_gbs"],
        "traffic": profiled_traffic("qk_norm_rope", NORM_SRC, w.batch * w.seq_len),
        "algorithmic_bytes_per_launch": w.norm_rope_bytes, "avg_launch_ms": t_norm,
        "peak_source": f"{peak_src} copy bandwidth",
    }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, desc = oracle_sample(w, qkv_h, gq_h, gk_h, args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc,
               "seconds": t}

    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "self-attn TFLOP/s (% of B200 bf16 peak) at Wan 480p/81f; norm+RoPE GB/s",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {**w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"inputs larger than L2 ({pristine.numel() * 2 / 1e9:.2f} GB packed QKV per step, "
                         f"a fresh copy per timed step)",
                   "step": "wan_dit_attn: qk_norm_rope in place, then attention (PDL-chained)"},
        "attn_tflops": attn_tflops, "attn_frac_of_peak": attn_tflops / tensor_peak,
        "norm_rope_gbs": norm_gbs, "norm_rope_frac_of_hbm": norm_gbs / peaks["hbm_gbs"],
        # the fused call (one step, PDL-chained) against its two kernels timed
        # as separate calls on the same stream
        "fused": {"step_ms": ms_step, "norm_ms": t_norm, "attn_ms": t_attn, "parts_sum_ms": t_norm + t_attn},
        "roofline": roofline, "roofline_norm_rope": norm_roofline,
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "skip_softmax": skip, "fp8": fp8,
        "qkv_projection": proj, "ring": ring,
        "gpu_launches": 2 * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
