#!/usr/bin/env python
"""Benchmark of packed MM-RoPE attention on B200.

One step = the whole hot path over one packed sequence: h3_build_coords ->
h3_mmrope_qk -> h3_packed_attention (coords, fused Q/K rotation, full
attention for all heads: "ms/layer" of the attention path).  Default
workload: the worked-example shape, 28,196 packed rows (512 text, 31 x 880
video latent tokens, 202 x 2 stereo audio tokens), 42 heads x 128, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs one independent packed sequence on its
own GPU (data parallel, no collective on the data path); the step time is the
max over ranks and `value` counts the FLOPs of all ranks ("scaling": "weak").
`--impl reference` times the fp64 CPU oracle (the only reference this path
has) on a bounded sample of query rows per step, on rank 0 only.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "packed MM-RoPE attention TFLOP/s & % bf16 peak (1 B200); ms/layer at 27.7k tokens"
UNIT = "TFLOP/s"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK), "fallback"


def pick_workload(args):
    import workload as W
    if args.video_frames:
        return W.worked_example_resized(args.video_frames)
    return W.workload(args.config)


def config_dict(wl, n_gpus):
    return {"workload": f"{wl.name}: {wl.n_rows} packed rows x {wl.heads} heads x {wl.head_dim}",
            "n_rows": wl.n_rows, "heads": wl.heads, "head_dim": wl.head_dim, "batch_per_gpu": 1,
            "global_batch": n_gpus, "seq_len": wl.n_rows,
            "parallelism": f"dp{n_gpus}" if n_gpus > 1 else "single",
            "rope": {"theta": wl.theta, "sections_thw": list(wl.sections), "pair_layout": "adjacent"},
            "l2": "inputs larger than L2: Q+K+V = %.0f MB per step vs 126 MB L2"
                  % (3 * wl.n_rows * wl.heads * wl.head_dim * 2 / 1e6)}


# ------------------------------------------------------------ clocks -------

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------- our GPU path ------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import packed_mm_rope_b200 as h3
    from packed_mm_rope_b200 import _lib
    from packed_mm_rope_b200 import dist as hdist
    import workload as W

    world, rank, local = hdist.world_from_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        hdist.init("nccl", device=dev, timeout_s=300)

    wl = pick_workload(args)
    N, H, D = wl.n_rows, wl.heads, wl.head_dim
    flops = wl.attention_flops
    q, k, v = W.qkv_bf16(wl)
    perm = W.permutation(wl)

    def host_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)

    hq, hk, hv = (host_bf16(a).pin_memory() for a in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    dq, dk, dv = (t.to(dev) for t in (hq, hk, hv))
    dqr, dkr, do = torch.empty_like(dq), torch.empty_like(dk), torch.empty_like(dq)
    coords = torch.empty((N, 3), dtype=torch.float32, device=dev)
    rope_cs = torch.empty((N, 64, 2), dtype=torch.float32, device=dev) if args.fused_q_rope else None
    hperm = None if perm is None else torch.from_numpy(perm.astype(np.int32)).pin_memory()
    dperm = None if perm is None else hperm.to(dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    cfg = h3.rope_cfg(wl.theta, D, wl.sections, 0)
    segs = _lib.segment_array(wl.segments)
    nseg = len(wl.segments)
    L = _lib.load()
    rs = H * D
    fused = args.fused_q_rope

    def call(status, what):
        if status != 0:
            raise RuntimeError(f"{what}: {h3.status_str(status)}")

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        call(L.h3_build_coords(segs, nseg, dperm.data_ptr() if dperm is not None else None, N,
                               coords.data_ptr(), s), "h3_build_coords")
        if evs is not None:
            evs[1].record(stream)
        if fused:
            # the rows' rotary table, K rotated by the rope kernel, Q rotated
            # inside the attention kernel from the table
            call(L.h3_rope_cos_sin(coords.data_ptr(), N, cfg, rope_cs.data_ptr(), s), "h3_rope_cos_sin")
            call(L.h3_mmrope_qk(None, dk.data_ptr(), None, dkr.data_ptr(), coords.data_ptr(),
                                N, H, rs, cfg, s), "h3_mmrope_qk")
        else:
            call(L.h3_mmrope_qk(dq.data_ptr(), dk.data_ptr(), dqr.data_ptr(), dkr.data_ptr(), coords.data_ptr(),
                                N, H, rs, cfg, s), "h3_mmrope_qk")
        if evs is not None:
            evs[2].record(stream)
        if fused:
            call(L.h3_packed_attention(dq.data_ptr(), dkr.data_ptr(), dv.data_ptr(), do.data_ptr(), None,
                                       rope_cs.data_ptr(), cfg, 1, N, H, D, rs, 0.0, s), "h3_packed_attention")
        else:
            call(L.h3_packed_attention(dqr.data_ptr(), dkr.data_ptr(), dv.data_ptr(), do.data_ptr(), None, None,
                                       None, 1, N, H, D, rs, 0.0, s), "h3_packed_attention")
        if evs is not None:
            evs[3].record(stream)

    work = h3.host_workspace(N, H, device=dev)

    def e2e_step():
        # the public host-buffer call: pinned Q/K/V in, O out, copies of one
        # chunk of heads overlapped with rope + attention of another
        call(L.h3_packed_mmrope_attention_host(segs, nseg, hperm.data_ptr() if hperm is not None else None,
                                               hq.data_ptr(), hk.data_ptr(), hv.data_ptr(), ho.data_ptr(),
                                               work.data_ptr(), N, H, 0, cfg, s), "h3_packed_mmrope_attention_host")

    barrier = hdist.barrier
    max_over_ranks = hdist.max_over_ranks

    # warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = h3.h3_check_device_error(s)
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {h3.status_str(st)}")

    # timed region: K steps, per-kernel events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1))
    st = h3.h3_check_device_error(s)
    if st != 0:
        raise RuntimeError(f"device error in timed region: {h3.status_str(st)}")
    coords_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    rope_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    attn_ms_max = max_over_ranks(attn_ms)
    ms_per_step = total_ms / args.steps

    # end to end through host buffers
    for _ in range(min(args.warmup, 2)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps
    h2d = 3 * N * H * D * 2 + (N * 4 if perm is not None else 0)
    d2h = N * H * D * 2

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    pk, src = peaks()
    value = hdist.weak_scaling_throughput(flops, world, ms_per_step * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms_max * 1e-3) / 1e12
    # fused: K read + written, coords read twice, the (cos, sin) table written
    rope_bytes = (2 * N * H * D * 2 + N * 24 + N * 512) if fused else (4 * N * H * D * 2 + N * 12)
    rope_gbs = rope_bytes / (rope_ms * 1e-3) / 1e9
    traffic = profiled_traffic(wl)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": config_dict(wl, world),
        "rope_fused_into_attention": "Q" if fused else "none",
        "pct_bf16_peak": round(100 * value / world / pk["bf16_tflops"], 2),
        "kernels_ms": {"h3_build_coords": round(coords_ms, 4), "h3_mmrope_qk": round(rope_ms, 4),
                       "h3_packed_attention": round(attn_ms, 4)},
        "roofline": {"kernel": "h3_packed_attention", "bound": "tensor", "achieved": round(attn_tflops, 2),
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(attn_tflops / pk["bf16_tflops"], 4),
                     "peak_source": f"{src} dense bf16 GEMM, burst (the attention kernel is timed in launches of "
                                    f"~{attn_ms:.0f} ms, {args.steps} back to back: a short region, not a "
                                    f"seconds-long power-capped loop)",
                     "frac_of_sustained_peak": round(attn_tflops / pk["bf16_tflops_sustained"], 4),
                     "sustained_peak": pk["bf16_tflops_sustained"],
                     "algorithmic": "4*N^2*D*H = %.4e FLOP per launch" % flops,
                     "traffic": traffic},
        "rope": {"kernel": "h3_mmrope_qk", "bound": "hbm", "achieved": round(rope_gbs, 1), "peak": pk["hbm_gbs"],
                 "unit": "GB/s", "frac": round(rope_gbs / pk["hbm_gbs"], 4),
                 "algorithmic": ("2*N*H*D*2 + 24*N + 512*N = %d bytes per step (table + K-only rope)" if fused
                                 else "4*N*H*D*2 + 12*N = %d bytes per launch") % rope_bytes},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "h3_packed_mmrope_attention_host (pinned host Q/K/V -> host O, copies overlapped with "
                       "compute over chunks of heads)"},
        "gpu_launches": (4 if fused else 3) * args.steps,
        "clocks": clk.summary(),
    }
    if args.adaln:
        line["adaln"] = time_adaln(h3, wl, dev, stream, pk["hbm_gbs"], args.steps)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, q, k, v, perm, rows=args.cpu_rows)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def time_adaln(h3, wl, dev, stream, hbm_gbs, steps):
    """h3_adaln_modulate on the workload's layer input [N, H*128] (not part of the step)."""
    import torch
    import workload as W
    n, c = wl.n_rows, wl.heads * wl.head_dim
    x = torch.from_numpy(W.normal_bf16(wl.seed, 9, (n, c)).view(np.int16)).view(torch.bfloat16).to(dev)
    tags = torch.tensor(sum(([s.kind] * s.rows for s in wl.segments), []), dtype=torch.int32, device=dev)
    ts = torch.zeros(n, dtype=torch.int32, device=dev)
    table = torch.randn((3, 2, c), dtype=torch.float32, device=dev) * 0.1
    y = torch.empty_like(x)
    for _ in range(3):
        h3.adaln_modulate(x, ts, tags, table, out=y, stream=stream)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        h3.adaln_modulate(x, ts, tags, table, out=y, stream=stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    nbytes = 2 * n * c * 2 + n * 8
    return {"kernel": "h3_adaln_modulate", "ms": round(ms, 4), "bound": "hbm",
            "achieved": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "peak": hbm_gbs,
            "frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "algorithmic": "2*N*C*2 + 8*N = %d bytes per launch (x read, y written, two int32 indices)" % nbytes}


def profiled_traffic(wl):
    """DRAM bytes per attention launch from the committed ncu summary.

    Only when the summary was taken on this workload AND on the current kernel
    source (hash match); otherwise null, as the counters no longer apply.
    """
    import hashlib
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    # the attention kernel is built from these three files
    srcs = [os.path.join(ROOT, "packed_mm_rope_b200", "csrc", n) for n in ("attention.cuh", "common.cuh", "rope.cuh")]
    try:
        with open(path) as f:
            d = json.load(f)
        h = hashlib.sha256()
        for src in srcs:
            with open(src, "rb") as f:
                h.update(f.read())
        sha = h.hexdigest()[:16]
        if d.get("n_rows") == wl.n_rows and d.get("heads") == wl.heads and d.get("source_sha256_16") == sha:
            return d.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


# ---------------------------------------------------------- oracle leg -----

def oracle_sample(wl, q, k, v, perm, rows):
    from oracle import pipeline as opipe
    t = time.perf_counter()
    opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections, rows=rows)
    return time.perf_counter() - t


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, q, k, v, perm, rows=768):
    import workload as W
    sample = np.sort(W.uniform01(wl.seed, 7, rows) * wl.n_rows).astype(np.int64)
    secs = oracle_sample(wl, q, k, v, perm, sample)
    flops = 4 * rows * wl.n_rows * wl.head_dim * wl.heads
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "seconds": round(secs, 3),
            "sample": f"{rows} seeded query rows x all {wl.heads} heads x all {wl.n_rows} keys of the "
                      f"{wl.name} workload, fp64 numpy oracle (coords, rotation, exact softmax); "
                      f"full-step time extrapolates to {secs * wl.n_rows / rows:.0f} s"}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import workload as W
    wl = pick_workload(args)
    q, k, v = W.qkv_bf16(wl)
    perm = W.permutation(wl)
    rows = args.ref_rows
    flops = 4 * rows * wl.n_rows * wl.head_dim * wl.heads
    u = W.uniform01(wl.seed, 8, rows * (args.steps + args.warmup)) * wl.n_rows
    samples = np.sort(u.astype(np.int64).reshape(args.steps + args.warmup, rows), axis=1)
    for i in range(args.warmup):
        oracle_sample(wl, q, k, v, perm, samples[i])
    secs = [oracle_sample(wl, q, k, v, perm, samples[args.warmup + i]) for i in range(args.steps)]
    total = sum(secs)
    value = flops * args.steps / total / 1e12
    desc = (f"{rows} seeded query rows x all {wl.heads} heads x all {wl.n_rows} keys per step, fp64 numpy "
            f"oracle; a full step would take {total / args.steps * wl.n_rows / rows:.0f} s")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16)", "config": config_dict(wl, args.gpus),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload index (default 2: 28,196 rows)")
    ap.add_argument("--video-frames", type=int, default=0,
                    help="resize the worked-example layout to this many latent frames (profiling cases)")
    ap.add_argument("--fused-q-rope", action="store_true",
                    help="rotate only K in h3_mmrope_qk and Q inside h3_packed_attention (from h3_rope_cos_sin)")
    ap.add_argument("--adaln", action="store_true", help="also time h3_adaln_modulate on [N, H*128]")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=768,
                    help="query rows of the timed oracle sample (768: about 10 s of host time at the worked example)")
    ap.add_argument("--ref-rows", type=int, default=16, help="query rows per reference-arm step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
