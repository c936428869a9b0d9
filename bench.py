"""Benchmark of the causal Conv3D hot path (libcc3d.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cc3d|reference]
                    [--quick-sweep|--no-sweep]

Workload (one "step"): the decoder latent-resolution causal conv,
bf16, C_in = C_out = 384 on x[1, 384, 5, 30, 52], 3x3x3, run once over the
whole sequence and once as 5 one-frame chunks that carry a 2-frame cache
(the outputs of the two are bitwise identical; the tests check that).
FLOP per step = 2 * (2 * C_out * C_in * 27 * T * H * W).  Inputs are 1.2 MB,
smaller than L2, so L2 is flushed (a 512 MiB buffer is rewritten) before
every timed step and the flush is outside the timed events.

The same JSON line carries the residual block (x[1, 192, 9, 240, 416]:
RMS_norm+SiLU -> conv -> RMS_norm+SiLU (fused) -> conv + x (fused)) as
``resblock`` with its latency, and as ``sweep`` the encoder convs (3 -> 96,
96 -> 96 at 17 x 480 x 832), the downsample path's time_conv (kernel
(3, 1, 1), stride 2 in time, at 192 and 384 channels) and its per-frame
3x3 stride-2 conv (96 channels, 480 x 832 -> 240 x 416), all nine rows of
the streaming channel/resolution sweep (C = 96, 192, 384 at three sizes, 21
one-frame chunks each, CUDA-graph captured) and the encoder's residual
blocks (96 -> 192, 192 -> 384 and a 384-channel one).  ``--quick-sweep``
keeps only the 384-channel rows and the 384-channel block; ``--no-sweep``
drops the sweep.

Multi-GPU: the path runs as independent replicas (one process per GPU, no
data-path collective); ``value`` is the FLOP all ranks processed divided by
the slowest rank's time ("scaling": "weak").

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (the only other place this script runs the oracle besides the
``cpu_baseline`` leg).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal Conv3D effective TFLOP/s and % of bf16 tensor roofline; resblock latency"
WORKLOAD = ("decoder latent-res causal conv bf16 384->384 k3x3x3, x[1,384,5,30,52], "
            "whole sequence + 5 one-frame chunks with 2-frame cache per step")
C2 = dict(c=384, t=5, h=30, w=52)
C4 = dict(c=192, t=9, h=240, w=416)


# DRAM bytes (read + write) per launch of the conv kernel on this workload,
# from one ncu capture of the current kernel (profiles/ holds the summaries
# and commands); None until captured.
NCU_TRAFFIC = {"whole": 14.03e6, "chunk": 10.09e6}


def conv_flop(n, cin, cout, t, h, w, taps=27):
    return 2.0 * n * cout * cin * taps * t * h * w


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---- clocks sampled during the timed region ---------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="cc3d_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        under_load = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(under_load) if under_load else None,
                "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ---- the reference arm: the fp64 oracle on a bounded sample -----------------------

def oracle_sample_rate(points_count, seed=11):
    """Time the oracle on `points_count` output voxels of the workload; returns
    (TFLOP/s, seconds, flop)."""
    import oracle
    from video_vae_causal_implicit_b200 import synth
    case = synth.conv_case(C2["c"], C2["c"], C2["t"], C2["h"], C2["w"])
    x = synth.ndhwc(case["x"])
    pts = synth.sample_points(1, C2["t"], C2["h"], C2["w"], points_count, seed)
    t0 = time.perf_counter()
    oracle.causal_conv3d_points(synth.ncthw_view(x), case["w"], case["b"].double().numpy(), None,
                                pts)
    dt = time.perf_counter() - t0
    flop = 2.0 * points_count * C2["c"] * C2["c"] * 27
    return flop / dt / 1e12, dt, flop


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    pts = 256  # about 2 GFLOP of fp64 work per step
    for _ in range(args.warmup):
        oracle_sample_rate(pts, seed=1)
    times, flops = [], 0.0
    for k in range(args.steps):
        _, dt, fl = oracle_sample_rate(pts, seed=100 + k)
        times.append(dt)
        flops += fl
    total = sum(times)
    value = flops / total / 1e12
    sample = (f"{pts} seeded output voxels (all 384 channels each) of the 384->384 conv on "
              f"[1,384,5,30,52] per step, fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- the CUDA arm ------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cc3d", choices=["cc3d", "reference"])
    ap.add_argument("--sweep", action="store_true",
                    help="(the default) time every sweep row: all nine config 5 rows and the "
                         "encoder blocks")
    ap.add_argument("--quick-sweep", action="store_true",
                    help="time only the 384-channel rows of config 5 and one encoder block")
    ap.add_argument("--no-sweep", action="store_true", help="skip the sweep rows")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from video_vae_causal_implicit_b200 import cc3d, replicas, synth

    rank, world, local = replicas.env_rank()
    torch.cuda.set_device(local)
    replicas.init("nccl", device=torch.device("cuda", local), timeout_s=120)
    barrier = replicas.barrier

    def max_over_ranks(v):
        return replicas.max_over_ranks(v, device=torch.device("cuda", local))

    peaks = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def flush_l2(k):
        flush.fill_(k & 0xFF)

    # --- workload: config 2 ---
    c, T, H, W = C2["c"], C2["t"], C2["h"], C2["w"]
    case = synth.conv_case(c, c, T, H, W, seed_base=replicas.replica_seed(0, rank))
    x = synth.ndhwc(case["x"]).to(dev)
    plan = cc3d.Plan(case["w"].to(dev), case["b"].to(dev), h=H, w=W, max_t=T)
    y_whole = torch.empty((1, T, H, W, c), dtype=torch.bfloat16, device=dev)
    xs = [x[:, k:k + 1].contiguous() for k in range(T)]
    ys = [torch.empty((1, 1, H, W, c), dtype=torch.bfloat16, device=dev) for _ in range(T)]
    caches = [torch.empty((1, 2, H, W, c), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    flop_step = 2 * conv_flop(1, c, c, T, H, W)

    def step(xin=None, marks=None):
        """One pass: the whole sequence, then 5 one-frame chunks carrying the
        cache.  `marks` (T + 2 events) bracket each forward call."""
        s = torch.cuda.current_stream()
        src = x if xin is None else xin
        if marks:
            marks[0].record(s)
        plan.forward(src, y_whole)
        if marks:
            marks[1].record(s)
        cache = None
        for k in range(T):
            xk = xs[k] if xin is None else src[:, k:k + 1]
            plan.forward(xk, ys[k], t=1, cache_in=cache, cache_out=caches[k % 2])
            cache = caches[k % 2]
            if marks:
                marks[2 + k].record(s)

    for k in range(args.warmup):
        flush_l2(k)
        step()
    cc3d.sync_status()

    # The timed step runs as one CUDA graph of the six forward calls,
    # captured once through the same C ABI calls: the GPU then runs the step
    # back to back, without the host time of six API calls between kernels
    # (each conv may start its setup while the previous one finishes:
    # programmatic dependent launch).  Its timing events are graph nodes at
    # its two ends only; the per-launch times come from a second graph of the
    # same step with an event between launches (event nodes between kernels
    # cost time of their own and stop the overlap, so that graph is not the
    # timed one).
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    graph = torch.cuda.CUDAGraph()
    n0 = cc3d.cc3d_launch_count()
    with torch.cuda.graph(graph):
        ends[0].record(torch.cuda.current_stream())
        step()
        ends[1].record(torch.cuda.current_stream())
    launches_per_step = cc3d.cc3d_launch_count() - n0
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(T + 2)]
    graph_marked = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_marked):
        step(marks=marks)
    for k in range(args.warmup):
        flush_l2(k)
        graph.replay()
        flush_l2(k)
        graph_marked.replay()
    torch.cuda.synchronize()
    cc3d.sync_status()

    sampler = ClockSampler(local)
    step_ms = []
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    for k in range(args.steps):
        flush_l2(k)  # untimed: the step's events are inside the graph
        graph.replay()
        torch.cuda.synchronize()
        step_ms.append(ends[0].elapsed_time(ends[1]))
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    launches = launches_per_step * args.steps
    cc3d.sync_status()
    # per-launch breakdown (untimed for the metric)
    whole_l, chunk_l = [], []
    for k in range(args.steps):
        flush_l2(k)
        graph_marked.replay()
        torch.cuda.synchronize()
        whole_l.append(marks[0].elapsed_time(marks[1]))
        chunk_l.extend(marks[1 + i].elapsed_time(marks[2 + i]) for i in range(T))
    cc3d.sync_status()
    whole_ms = statistics.mean(whole_l)
    chunk_ms = statistics.mean(chunk_l)
    plan_stats = plan.stats()

    # For context (not the timed step): the same layer planned for one-frame
    # calls only (max_t = 1); its 5 chunks as one graph.  Whatever tile shape
    # that plan picks, every output sums its taps in one accumulator in the
    # same order, so its bytes equal the whole-sequence plan's (the tests
    # check it).
    plan_s = cc3d.Plan(case["w"].to(dev), case["b"].to(dev), h=H, w=W, max_t=1)
    ys_s = [torch.empty_like(ys[0]) for _ in range(T)]
    smarks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(T + 1)]

    def stream_only():
        s = torch.cuda.current_stream()
        smarks[0].record(s)
        cache = None
        for k in range(T):
            plan_s.forward(xs[k], ys_s[k], t=1, cache_in=cache, cache_out=caches[k % 2])
            cache = caches[k % 2]
            smarks[1 + k].record(s)

    stream_only()
    sgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(sgraph):
        stream_only()
    s_chunks = []
    for k in range(args.warmup + args.steps):
        flush_l2(k)
        sgraph.replay()
        torch.cuda.synchronize()
        if k >= args.warmup:
            s_chunks.extend(smarks[i].elapsed_time(smarks[i + 1]) for i in range(T))
    cc3d.sync_status()
    stream_plan_ms = statistics.mean(s_chunks)
    stream_plan_stats = plan_s.stats()
    del sgraph
    plan_s.close()
    ms_local = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms_local)
    value = world * flop_step / (ms * 1e-3) / 1e12
    # the conv kernel over the timed region: the step is its 6 launches back
    # to back (the tensor-core conv writes its caches itself), so the average
    # launch lasts a sixth of the step
    flop_whole = conv_flop(1, c, c, T, H, W)
    flop_chunk = conv_flop(1, c, c, 1, H, W)
    avg_launch_ms = ms_local / (T + 1)
    achieved = (flop_step / (T + 1)) / (avg_launch_ms * 1e-3) / 1e12
    traffic_avg = None
    if NCU_TRAFFIC["whole"] is not None and NCU_TRAFFIC["chunk"] is not None:
        traffic_avg = (NCU_TRAFFIC["whole"] + T * NCU_TRAFFIC["chunk"]) / (T + 1)
    # FLOP the MMAs execute: a tap that reads a causal zero frame of a call
    # without a cache is skipped (output frame t of the whole sequence runs
    # min(t + 1, 3) of its 3 temporal taps; the first chunk, which has no
    # cache, runs 1 of 3; the later chunks multiply their cache frames)
    exec_whole = flop_whole * sum(min(t + 1, 3) for t in range(T)) / (3 * T)
    exec_step = exec_whole + flop_chunk * (1 / 3 + (T - 1))
    executed = (exec_step / (T + 1)) / (avg_launch_ms * 1e-3) / 1e12

    # --- end to end through the public API with host buffers ---
    # The step's six calls through cc3d_forward_host: each call's x comes
    # from pinned host memory and its y goes back to it; the library
    # overlaps one call's upload and another's download with the conv
    # between them.  Every step's result is read on the host at its end.
    x_host = x.cpu().pin_memory()
    xs_host = [xk.cpu().pin_memory() for xk in xs]
    y_host = torch.empty(tuple(y_whole.shape), dtype=torch.bfloat16).pin_memory()
    ys_host = [torch.empty(tuple(yk.shape), dtype=torch.bfloat16).pin_memory() for yk in ys]
    host_calls = [dict(x_host=x_host, y_host=y_host)]
    for k in range(T):
        host_calls.append(dict(x_host=xs_host[k], y_host=ys_host[k], t=1,
                               cache_in=caches[(k - 1) % 2] if k > 0 else None,
                               cache_out=caches[k % 2]))
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for k in range(args.warmup + args.steps):
        flush_l2(k)
        i = k - args.warmup
        if i >= 0:
            e0[i].record(stream)
        plan.forward_host(host_calls)
        if i >= 0:
            e1[i].record(stream)
    torch.cuda.synchronize()
    cc3d.sync_status()
    e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(e0, e1)))
    e2e = {"value": world * flop_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": sum(c["x_host"].numel() * 2 for c in host_calls),
           "d2h_bytes_per_step": sum(c["y_host"].numel() * 2 for c in host_calls),
           "ms_per_step": e2e_ms,
           "api": "cc3d_forward_host: six calls per step (whole sequence + 5 one-frame chunks), "
                  "x and y in pinned host memory, uploads and downloads overlapped with the convs"}

    # --- residual block (config 4): latency ---
    resblock = None
    cb, Tb, Hb, Wb = C4["c"], C4["t"], C4["h"], C4["w"]
    bc = synth.block_case(cb, Tb, Hb, Wb)
    blk = cc3d.Block(*(bc[k].to(dev) for k in ("w1", "b1", "g1", "w2", "b2", "g2")), h=Hb, w=Wb,
                     max_t=Tb)
    xb = synth.ndhwc(bc["x"]).to(dev)
    yb = torch.empty_like(xb)
    for _ in range(args.warmup):
        blk.forward(xb, yb)
    torch.cuda.synchronize()
    b0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    b1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for k in range(args.steps):
        b0[k].record(stream)
        blk.forward(xb, yb)
        b1[k].record(stream)
    torch.cuda.synchronize()
    cc3d.sync_status()
    blk_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in zip(b0, b1)))
    blk_flop = 2 * conv_flop(1, cb, cb, Tb, Hb, Wb)
    act_bytes = Tb * Hb * Wb * cb * 2
    blk_bytes = 7 * act_bytes  # x r, a0 w, a0 r, a1 w, a1 r, x r (residual), y w
    # the block is timed on its own (a few ms): the burst peak applies
    roof_ms = max(blk_flop / (peaks["bf16_tflops"] * 1e12),
                  blk_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    # the block's three kernels, timed one by one through the public API
    dv = {k: bc[k].to(dev) for k in ("w1", "b1", "g1", "w2", "b2", "g2")}
    conv1 = cc3d.Plan(dv["w1"], dv["b1"], h=Hb, w=Wb, max_t=Tb, epi=cc3d.EPI_BIAS_RMS_SILU,
                      gamma=dv["g2"])
    conv2 = cc3d.Plan(dv["w2"], dv["b2"], h=Hb, w=Wb, max_t=Tb, epi=cc3d.EPI_BIAS_RESIDUAL)
    a0 = torch.empty_like(xb)
    a1 = torch.empty_like(xb)
    parts = {"rmsnorm_silu": lambda: cc3d.rms_silu(xb, dv["g1"], a0),
             "conv1_rms_silu_epilogue": lambda: conv1.forward(a0, a1),
             "conv2_residual_epilogue": lambda: conv2.forward(a1, yb, residual=xb)}
    breakdown = {}
    for name, fn in parts.items():
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        ea = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        eb = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for k in range(args.steps):
            ea[k].record(stream)
            fn()
            eb[k].record(stream)
        torch.cuda.synchronize()
        pms = statistics.median(a.elapsed_time(b) for a, b in zip(ea, eb))
        if name == "rmsnorm_silu":
            gbs = 2 * act_bytes / pms / 1e6
            breakdown[name] = {"ms": pms, "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"]}
        else:
            tf = conv_flop(1, cb, cb, Tb, Hb, Wb) / pms / 1e9
            breakdown[name] = {"ms": pms, "tflops": tf, "frac": tf / peaks["bf16_tflops"]}
    cc3d.sync_status()
    resblock = {"workload": "Wan residual block bf16 192ch x[1,192,9,240,416]",
                "ms": blk_ms, "tflops": blk_flop / (blk_ms * 1e-3) / 1e12,
                "roofline_ms": roof_ms, "frac": roof_ms / blk_ms,
                "peak_basis": "burst bf16 (" + peaks["source"] + ")",
                "frac_vs_sustained": blk_flop / (peaks["bf16_tflops_sustained"] * 1e12) * 1e3 / blk_ms,
                "note": "effective FLOP = 2*Cout*Cin*27*T*H*W per conv; the taps that read the "
                        "causal zero frames (1/9 of the MMAs at T=9) are not executed",
                "kernels": breakdown}
    del conv1, conv2, a0, a1
    # two such blocks in a row: each running its own first norm, or the
    # first block's conv2 epilogue handing the second block its activation
    bc2 = synth.block_case(cb, Tb, Hb, Wb, seed_base=100)
    blk2 = cc3d.Block(*(bc2[k].to(dev) for k in ("w1", "b1", "g1", "w2", "b2", "g2")), h=Hb,
                      w=Wb, max_t=Tb)
    y2b, a_hand = torch.empty_like(xb), torch.empty_like(xb)
    chain = {"unfused": lambda: (blk.forward(xb, yb), blk2.forward(yb, y2b)),
             "fused": lambda: (blk.forward(xb, yb, g_next=blk2.g1, a0_next=a_hand),
                               blk2.forward(yb, y2b, a0_in=a_hand))}
    # (the two forms alternate step by step: run one after the other, the
    # second would run on a hotter, more power-capped GPU)
    for fn in chain.values():
        fn()
        fn()
    torch.cuda.synchronize()
    ev = {name: [] for name in chain}
    for k in range(args.steps):
        for name, fn in chain.items():
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record(stream)
            fn()
            eb.record(stream)
            ev[name].append((ea, eb))
    torch.cuda.synchronize()
    chain_ms = {name: statistics.median(a.elapsed_time(b) for a, b in pairs)
                for name, pairs in ev.items()}
    cc3d.sync_status()
    resblock["chain2"] = {"workload": "two 192ch blocks in a row, x[1,192,9,240,416]",
                          "unfused_ms": chain_ms["unfused"], "fused_ms": chain_ms["fused"],
                          "note": "fused: the first block's conv2 epilogue also writes the "
                                  "second block's SiLU(RMS_norm(y)), which then skips its "
                                  "stand-alone norm pass"}
    del blk, blk2, xb, yb, y2b, a_hand

    sweep = None if args.no_sweep else run_sweep(args, dev, stream, peaks, flush_l2,
                                                  full=not args.quick_sweep)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        # a bounded sample of the workload: about 10 s of the host cores' time
        pts = 16384
        rate, dt, fl = oracle_sample_rate(pts)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
               "kind": "oracle", "seconds": dt,
               "sample": f"{pts} seeded output voxels x 384 channels of the 384->384 conv "
                         f"on [1,384,5,30,52] ({fl / 1e9:.1f} GFLOP fp64)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) activations, Kaiming-uniform weights)",
            "config": {"workload": WORKLOAD, "global_batch": world, "parallelism": f"replicas{world}",
                       "l2": "flushed before every timed step (512 MiB rewrite, untimed)",
                       "launch": "the step's six forward calls captured once as a CUDA graph "
                                 "(timing events only at its ends), replayed per step",
                       "flop_per_step": flop_step},
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic_avg,
                         "kernel": "conv_umma_kernel, average over the 6 launches of the "
                                   "timed step; per_launch: a copy of the step graph with an "
                                   "event between launches (the events add time of their own)",
                         "executed_tflops": executed,
                         "executed_frac": executed / peaks["bf16_tflops"],
                         "executed_note": "FLOP of the MMAs run: the taps that read causal zero "
                                          "frames of a call without a cache are skipped "
                                          f"({exec_step / 1e9:.1f} of {flop_step / 1e9:.1f} "
                                          "GFLOP per step)",
                         "peak_basis": "burst bf16 (" + peaks["source"] + ")",
                         "per_launch": {
                             "whole_sequence": {"ms": whole_ms, "gflop": flop_whole / 1e9,
                                                "tflops": flop_whole / whole_ms / 1e9,
                                                "frac": flop_whole / whole_ms / 1e9 / peaks["bf16_tflops"],
                                                "traffic": NCU_TRAFFIC["whole"]},
                             "one_frame_chunk": {"ms": chunk_ms, "gflop": flop_chunk / 1e9,
                                                 "tflops": flop_chunk / chunk_ms / 1e9,
                                                 "frac": flop_chunk / chunk_ms / 1e9 / peaks["bf16_tflops"],
                                                 "traffic": NCU_TRAFFIC["chunk"]},
                             "plan": {"k_split": plan_stats.k_split,
                                      "mma_ctas": plan_stats.mma_ctas,
                                      "n_tile": plan_stats.n_tile,
                                      "second_tiles_mma_ctas": plan_stats.one_frame_mma_ctas,
                                      "calls_on_second_tiles": plan_stats.second_tile_calls,
                                      "note": "the uncached whole-sequence call and the one-frame "
                                              "chunks run on the plan's second tile choice "
                                              "(CTA pairs)"},
                             "one_frame_chunk_streaming_plan": {
                                 "ms": stream_plan_ms, "tflops": flop_chunk / stream_plan_ms / 1e9,
                                 "frac": flop_chunk / stream_plan_ms / 1e9 / peaks["bf16_tflops"],
                                 "n_tile": stream_plan_stats.n_tile,
                                 "mma_ctas": stream_plan_stats.mma_ctas,
                                 "note": "the layer planned for one-frame calls (max_t = 1); "
                                         "same bytes as the step's plan; context only, not in "
                                         "the timed step"}}},
            "resblock": resblock,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if sweep is not None:
            line["sweep"] = sweep
        print(json.dumps(line), flush=True)
    replicas.shutdown()
    return 0


def run_sweep(args, dev, stream, peaks, flush_l2, full=False):
    """Config 3 (encoder full-res convs), the downsample path's convs and the
    384-channel rows of config 5 (streaming sweep); with `full` also config
    5's 96- and 192-channel rows and the encoder's residual blocks."""
    import torch

    from video_vae_causal_implicit_b200 import cc3d, synth
    out = {}
    reps = max(3, min(args.steps, 10))

    def timed(fn, flush=False):
        # every row starts from an idle GPU (half a second), so that the
        # power and clock state a heavy row leaves behind does not carry
        # over into the next one
        torch.cuda.synchronize()
        time.sleep(0.5)
        for k in range(2):
            fn()
        torch.cuda.synchronize()
        ts = []
        for k in range(reps):
            if flush:
                flush_l2(k)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    g = torch.Generator(device=dev)
    g.manual_seed(0)
    # config 1: the fp32 causal conv, 16 -> 16 on x[1,16,5,16,16] (SIMT FFMA;
    # a launch-latency-bound 17.7 MFLOP, reported in microseconds)
    c1 = synth.conv_case(16, 16, 5, 16, 16, dtype=torch.float32)
    p1 = cc3d.Plan(c1["w"].to(dev), c1["b"].to(dev), h=16, w=16, max_t=5, dtype=cc3d.FP32)
    x1 = synth.ndhwc(c1["x"]).to(dev)
    y1 = torch.empty((1, 5, 16, 16, 16), dtype=torch.float32, device=dev)
    # the device time of one call (captured once as a CUDA graph and
    # replayed: a single call's events would mostly time the host's call
    # path, which is reported beside it)
    host_ms = timed(lambda: p1.forward(x1, y1))
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        p1.forward(x1, y1)
    ms = timed(g1.replay)
    out["cfg1_fp32_16to16_5x16x16"] = {"us": ms * 1e3,
                                       "gflops": conv_flop(1, 16, 16, 5, 16, 16) / ms / 1e6,
                                       "us_one_host_call": host_ms * 1e3}
    del g1, p1, x1, y1
    # config 3a: 3 -> 96 at 17 x 480 x 832 (HBM-bound on the output write)
    T, H, W = 17, 480, 832
    x3 = (torch.rand((1, T, H, W, 3), generator=g, device=dev) * 2 - 1).to(torch.bfloat16)
    w3 = synth.kaiming_uniform(96, 3, (3, 3, 3), 1).to(dev)
    b3 = synth.uniform((96,), -0.1, 0.1, 2).to(dev)
    p3 = cc3d.Plan(w3, b3, h=H, w=W, max_t=T)
    y3 = torch.empty((1, T, H, W, 96), dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: p3.forward(x3, y3), flush=True)
    fl = conv_flop(1, 3, 96, T, H, W)
    byts = x3.numel() * 2 + y3.numel() * 2
    # the layer's bytes are 97 % writes: its ceiling is the rate at which
    # HBM takes a pure write stream, measured here on the same buffer (a
    # torch fill of y), not the copy rate of the peak file
    wms = timed(lambda: y3.fill_(0.5), flush=True)
    write_gbs = y3.numel() * 2 / wms / 1e6
    out["cfg3a_3to96_17x480x832"] = {"ms": ms, "tflops": fl / ms / 1e9,
                                     "hbm_gbs": byts / ms / 1e6,
                                     "hbm_frac": byts / ms / 1e6 / peaks["hbm_gbs"],
                                     "write_peak_gbs": write_gbs,
                                     "frac_of_write_peak": byts / ms / 1e6 / write_gbs}
    del p3, x3, y3
    # config 3b: 96 -> 96 at 17 x 480 x 832
    x96 = torch.randn((1, T, H, W, 96), generator=g, device=dev).to(torch.bfloat16)
    w96 = synth.kaiming_uniform(96, 96, (3, 3, 3), 1).to(dev)
    b96 = synth.uniform((96,), -0.1, 0.1, 2).to(dev)
    p96 = cc3d.Plan(w96, b96, h=H, w=W, max_t=T)
    y96 = torch.empty_like(x96)
    ms = timed(lambda: p96.forward(x96, y96))
    fl = conv_flop(1, 96, 96, T, H, W)
    out["cfg3b_96to96_17x480x832"] = {"ms": ms, "tflops": fl / ms / 1e9,
                                      "frac": fl / ms / 1e9 / peaks["bf16_tflops"]}
    del p96, x96, y96
    # the downsample path's time_conv: kernel (3, 1, 1), temporal stride 2,
    # whole sequence (17 -> 9 frames at 192 channels, 9 -> 5 at 384)
    for (cc, T, H, W) in ((192, 17, 120, 208), (384, 9, 60, 104)):
        xs = torch.randn((1, T, H, W, cc), generator=g, device=dev).to(torch.bfloat16)
        ws = synth.kaiming_uniform(cc, cc, (3, 1, 1), 1).to(dev)
        bs = synth.uniform((cc,), -0.1, 0.1, 2).to(dev)
        ps = cc3d.Plan(ws, bs, h=H, w=W, max_t=T, stride_t=2)
        t_out = (T - 1) // 2 + 1
        ys = torch.empty((1, t_out, H, W, cc), dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: ps.forward(xs, ys), flush=True)
        fl = conv_flop(1, cc, cc, t_out, H, W, taps=3)
        out[f"time_conv_s2_c{cc}_{T}x{H}x{W}"] = {
            "ms": ms, "tflops": fl / ms / 1e9, "frac": fl / ms / 1e9 / peaks["bf16_tflops"],
            "tile": [ps.stats().mma_ctas, ps.stats().tile_w, ps.stats().k_split]}
        del ps, xs, ys
    # the downsample path's spatial step: ZeroPad2d(0, 1, 0, 1) + 3x3 stride 2
    # per frame, 96 channels, 17 x 480 x 832 -> 17 x 240 x 416
    T, H, W, cc = 17, 480, 832, 96
    xs = torch.randn((1, T, H, W, cc), generator=g, device=dev).to(torch.bfloat16)
    ws = synth.kaiming_uniform(cc, cc, (1, 3, 3), 1).to(dev)
    bs = synth.uniform((cc,), -0.1, 0.1, 2).to(dev)
    ps = cc3d.Plan(ws, bs, h=H, w=W, max_t=T, pad=(0, 0), stride_hw=2)
    ys = torch.empty((1, T, H // 2, W // 2, cc), dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: ps.forward(xs, ys), flush=True)
    fl = conv_flop(1, cc, cc, T, H // 2, W // 2, taps=9)
    byts = xs.numel() * 2 + ys.numel() * 2
    out[f"downsample_s2_c{cc}_{T}x{H}x{W}"] = {
        "ms": ms, "tflops": fl / ms / 1e9, "frac": fl / ms / 1e9 / peaks["bf16_tflops"],
        "hbm_gbs": byts / ms / 1e6, "hbm_frac": byts / ms / 1e6 / peaks["hbm_gbs"]}
    del ps, xs, ys
    # the downsample path as the page draws it: WanRMS_norm, the stride-2
    # conv, WanRMS_norm (the second one in the conv's epilogue)
    T, H, W, cc = 17, 480, 832, 96
    xs = torch.randn((1, T, H, W, cc), generator=g, device=dev).to(torch.bfloat16)
    ga = synth.uniform((cc,), 0.5, 1.5, 3).to(dev)
    gb = synth.uniform((cc,), 0.5, 1.5, 4).to(dev)
    ps = cc3d.Plan(ws, bs, h=H, w=W, max_t=T, pad=(0, 0), stride_hw=2, epi=cc3d.EPI_BIAS_RMS,
                   gamma=gb)
    xa = torch.empty_like(xs)
    ys = torch.empty((1, T, H // 2, W // 2, cc), dtype=torch.bfloat16, device=dev)

    def down_path():
        cc3d.rms(xs, ga, xa)
        ps.forward(xa, ys)

    ms = timed(down_path, flush=True)
    byts = 3 * xs.numel() * 2 + ys.numel() * 2  # norm r/w, conv r, conv w
    out[f"downsample_path_rms_s2conv_rms_c{cc}_{T}x{H}x{W}"] = {
        "ms": ms, "hbm_gbs": byts / ms / 1e6, "hbm_frac": byts / ms / 1e6 / peaks["hbm_gbs"],
        "tflops": fl / ms / 1e9}
    del ps, xs, ys, xa
    # FP8 (E4M3) operands: the config-2 step (whole sequence + 5 one-frame
    # chunks) and config 5's largest 384-channel row, against the fp8 peak
    # (the measured bf16 peak x the nominal fp8 / bf16 ratio of 2)
    fp8_peak = 2 * peaks["bf16_tflops"]
    c2, T2, H2, W2 = C2["c"], C2["t"], C2["h"], C2["w"]
    case = synth.conv_case(c2, c2, T2, H2, W2)
    w8 = case["w"].to(dev)
    s_w = (w8.float().abs().reshape(c2, -1).amax(dim=1) / 448.0).contiguous()
    xb = synth.ndhwc(case["x"]).to(dev)
    s_x = float(xb.float().abs().max()) / 448.0
    p8 = cc3d.Plan(w8, case["b"].to(dev), h=H2, w=W2, max_t=T2, dtype=cc3d.FP8_E4M3,
                   w_scale=s_w, x_scale=s_x)
    xq = torch.empty(xb.shape, dtype=torch.uint8, device=dev)
    cc3d.quantize_e4m3(xb, s_x, xq)
    y8 = torch.empty((1, T2, H2, W2, c2), dtype=torch.bfloat16, device=dev)
    xq1 = [xq[:, k:k + 1].contiguous() for k in range(T2)]
    y81 = [torch.empty((1, 1, H2, W2, c2), dtype=torch.bfloat16, device=dev) for _ in range(T2)]
    c8 = [torch.empty((1, 2, H2, W2, c2), dtype=torch.uint8, device=dev) for _ in range(2)]

    def fp8_step():
        p8.forward(xq, y8)
        cache = None
        for k in range(T2):
            p8.forward(xq1[k], y81[k], t=1, cache_in=cache, cache_out=c8[k % 2])
            cache = c8[k % 2]

    fp8_step()
    gr8 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr8):
        fp8_step()
    ms = timed(gr8.replay, flush=True)
    fl = 2 * conv_flop(1, c2, c2, T2, H2, W2)
    out["fp8_cfg2_step_whole_plus_5_chunks"] = {
        "ms": ms, "tflops": fl / ms / 1e9, "frac_of_fp8_peak": fl / ms / 1e9 / fp8_peak,
        "fp8_peak_basis": "2 x bf16 (" + peaks["source"] + ")"}
    del gr8, p8, xq, y8, xq1, y81, c8
    H5, W5 = 360, 640
    x5 = torch.randn((1, 21, H5, W5, 384), generator=g, device=dev).to(torch.bfloat16)
    w5 = synth.kaiming_uniform(384, 384, (3, 3, 3), 1).to(dev)
    s_w5 = (w5.float().abs().reshape(384, -1).amax(dim=1) / 448.0).contiguous()
    s_x5 = float(x5.float().abs().max()) / 448.0
    x5q = torch.empty(x5.shape, dtype=torch.uint8, device=dev)
    cc3d.quantize_e4m3(x5, s_x5, x5q)
    del x5
    p5 = cc3d.Plan(w5, synth.uniform((384,), -0.1, 0.1, 2).to(dev), h=H5, w=W5, max_t=1,
                   dtype=cc3d.FP8_E4M3, w_scale=s_w5, x_scale=s_x5)
    y5 = torch.empty((1, 21, H5, W5, 384), dtype=torch.bfloat16, device=dev)
    xs5 = [x5q[:, k:k + 1] for k in range(21)]
    ys5 = [y5[:, k:k + 1] for k in range(21)]
    cb5 = [torch.empty((1, 2, H5, W5, 384), dtype=torch.uint8, device=dev) for _ in range(2)]

    def run5():
        cache = None
        for k in range(21):
            p5.forward(xs5[k], ys5[k], t=1, cache_in=cache, cache_out=cb5[k % 2])
            cache = cb5[k % 2]

    run5()
    gr5 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr5):
        run5()
    ms = timed(gr5.replay, flush=True)
    fl = conv_flop(1, 384, 384, 21, H5, W5)
    out["fp8_cfg5_c384_360x640_21x1frame"] = {
        "ms": ms, "tflops": fl / ms / 1e9, "frac_of_fp8_peak": fl / ms / 1e9 / fp8_peak}
    del gr5, p5, x5q, y5, cb5
    # the encoder's other residual blocks (§8(f) NEXT-2): the two that change
    # the channel count (the 1x1x1 conv_shortcut fused into conv2) and a
    # 384-channel one (conv1's RMS_norm + SiLU fused into its epilogue as two
    # N = 192 MMAs per K step), whole sequence; the 384-channel one always
    for (ci, co, T, H, W) in (((96, 192, 17, 240, 416), (192, 384, 9, 120, 208),
                               (384, 384, 5, 60, 104)) if full else ((384, 384, 5, 60, 104),)):
        xb = torch.randn((1, T, H, W, ci), generator=g, device=dev).to(torch.bfloat16)
        wts = dict(w1=synth.kaiming_uniform(co, ci, (3, 3, 3), 11),
                   b1=synth.uniform((co,), -0.1, 0.1, 12), g1=synth.uniform((ci,), 0.5, 1.5, 13),
                   w2=synth.kaiming_uniform(co, co, (3, 3, 3), 14),
                   b2=synth.uniform((co,), -0.1, 0.1, 15), g2=synth.uniform((co,), 0.5, 1.5, 16))
        if ci != co:
            wts["w_sc"] = synth.kaiming_uniform(co, ci, (1, 1, 1), 17)
            wts["b_sc"] = synth.uniform((co,), -0.1, 0.1, 18)
        wts = {k: v.to(dev) for k, v in wts.items()}
        blk = cc3d.Block(**wts, h=H, w=W, max_t=T)
        yb = torch.empty((1, T, H, W, co), dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: blk.forward(xb, yb), flush=True)
        fl = conv_flop(1, ci, co, T, H, W) + conv_flop(1, co, co, T, H, W) + (
            conv_flop(1, ci, co, T, H, W, taps=1) if ci != co else 0)
        out[f"block_{ci}to{co}_{T}x{H}x{W}"] = {
            "ms": ms, "tflops": fl / ms / 1e9, "frac": fl / ms / 1e9 / peaks["bf16_tflops"]}
        del blk, xb, yb
    # config 5: C x resolution, 21 one-frame chunks, graph-captured
    for cc in ((96, 192, 384) if full else (384,)):
        for (H, W) in ((90, 160), (180, 320), (360, 640)):
            T = 21
            x5 = torch.randn((1, T, H, W, cc), generator=g, device=dev).to(torch.bfloat16)
            w5 = synth.kaiming_uniform(cc, cc, (3, 3, 3), 1).to(dev)
            b5 = synth.uniform((cc,), -0.1, 0.1, 2).to(dev)
            p5 = cc3d.Plan(w5, b5, h=H, w=W, max_t=1)
            y5 = torch.empty_like(x5)
            xsl = [x5[:, k:k + 1] for k in range(T)]
            ysl = [y5[:, k:k + 1] for k in range(T)]
            cbuf = [torch.empty((1, 2, H, W, cc), dtype=torch.bfloat16, device=dev)
                    for _ in range(2)]

            def run():
                cache = None
                for k in range(T):
                    p5.forward(xsl[k], ysl[k], t=1, cache_in=cache, cache_out=cbuf[k % 2])
                    cache = cbuf[k % 2]

            run()
            torch.cuda.synchronize()
            gs = torch.cuda.Stream(device=dev)
            graph = torch.cuda.CUDAGraph()
            gs.wait_stream(stream)
            with torch.cuda.stream(gs):
                graph.capture_begin()
                cache = None
                for k in range(T):
                    p5.forward(xsl[k], ysl[k], t=1, cache_in=cache, cache_out=cbuf[k % 2],
                               stream=gs)
                    cache = cbuf[k % 2]
                graph.capture_end()
            stream.wait_stream(gs)
            ms = timed(graph.replay, flush=True)
            fl = conv_flop(1, cc, cc, T, H, W)
            out[f"cfg5_c{cc}_{H}x{W}_21x1frame"] = {"ms": ms, "tflops": fl / ms / 1e9,
                                                    "frac": fl / ms / 1e9 / peaks["bf16_tflops"]}
            del graph, p5, x5, y5, cbuf
            torch.cuda.synchronize()
    cc3d.sync_status()
    return out


if __name__ == "__main__":
    sys.exit(main())
