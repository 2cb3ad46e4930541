"""Throughput of the vision-tower forward (32 bf16 blocks + final norm + aligner) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 4|5]

One step = one pass of the whole path over one batch: copy the resident patch states into the
working buffer, dsv4v_tower_forward, dsv4v_aligner_forward.  Default workload: one 28x28 image
(784 patches, 196 tokens), seeded synthetic inputs and random-init weights of the tower's shape.
Under torchrun each rank runs its own replica of the batch (images are independent, so the
path shards by image with no collective; weak scaling); the reported time is the max over
ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (the only other place this script runs the oracle besides the cpu_baseline leg).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vision_transformer_encoder_dsv4v_b200 import synth  # noqa: E402

METRIC = "ViT tower patches/sec and TFLOP/s (bf16, 1 B200) vs dense bf16 roofline"

# DRAM bytes per launch of each kernel class (dram__bytes_read.sum + dram__bytes_write.sum), from
# one-kernel ncu captures of the benchmark's step (-k regex:k_gemm_tc -s 8 -c 4 for the GEMMs of
# the third layer, -k regex:k_attn_tc -s 2 -c 1) of the kernels as they are now; an entry is
# removed when its kernel changes.
TRAFFIC_BYTES = {
    (4, "down"): 18.15e6, (4, "swiglu"): 19.01e6, (4, "attention"): 4.88e6, (4, "out"): 16.91e6, (4, "qkv"): 10.30e6,
}
UNIT = "patches/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=4, choices=[4, 5])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps as plain C-ABI calls (no graph, no extra passes) for ncu; "
                         "prints no bench line")
    ap.add_argument("--extra", choices=["patch_embed", "patch_merger", "bridge", "block_backward", "workload5"],
                    help="time only this one of the bench line's extras (for a profiler) and print it; "
                         "prints no bench line")
    return ap.parse_args()


def workload_desc(wl):
    return {"workload": f"{wl.name}: {len(wl.grids)} image(s), {wl.n_patches} patches -> {wl.n_tokens} tokens, "
                        f"D={wl.vision_dim} H={wl.n_heads} F={wl.mlp_hidden} r={wl.downsample_ratio} "
                        f"E={wl.llm_dim} L={wl.n_layers}",
            "grids": wl.grids, "patches_per_gpu": wl.n_patches, "tokens_per_gpu": wl.n_tokens,
            "flops_per_gpu_step": synth.algorithmic_flops(wl)}


# ------------------------------------------------------------------------------ CPU oracle timing
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def time_oracle(wl, inp, budget_s):
    """Runs the oracle on a bounded sample: whole layers of the tower (plus the aligner when the
    budget allows), and scales to patches/s of the full workload by the counted work."""
    from oracle import dsv4v_oracle as O
    layers = [{k: (v.values if hasattr(v, "values") else v) for k, v in l.items()} for l in inp.layers]
    cos, sin = O.packed_cos_sin(wl.grids, wl.head_dim // 2, wl.rope_theta)
    x = inp.x.values.astype(np.float64)
    t0 = time.perf_counter()
    done = 0
    while done < wl.n_layers:
        x = O.block_forward(x, layers[done], cos, sin, wl.grids, wl.n_heads, wl.eps)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    t_layers = time.perf_counter() - t0
    aligner_s = 0.0
    if done == wl.n_layers:
        t1 = time.perf_counter()
        x = O.rmsnorm(x, inp.final_norm_w, wl.eps)
        O.aligner_forward(x, inp.w_align.values, wl.grids, wl.downsample_ratio)
        aligner_s = time.perf_counter() - t1
    per_layer = t_layers / done
    full_s = per_layer * wl.n_layers + (aligner_s if done == wl.n_layers else
                                         per_layer * synth.algorithmic_flops(wl, 0, True) /
                                         synth.algorithmic_flops(wl, 1, False))
    sample = (f"{done} of {wl.n_layers} tower layers" + (" + final norm + aligner" if done == wl.n_layers else "") +
              f" of the same workload in {t_layers + aligner_s:.1f} s; full step extrapolated by counted work")
    return {"value": wl.n_patches / full_s, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": sample, "seconds_per_step_full": full_s}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = synth.workload(args.workload)
    inp = synth.draw(wl)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        r = time_oracle(wl, inp, budget)
        if i >= args.warmup:
            vals.append(r["value"])
        last = r
    v = statistics.median(vals) if vals else last["value"]
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wl.n_patches / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(wl),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": "each step: " + last["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        # the reader thread ends at EOF of the pipe; parse only once it has appended every line
        self.thread.join(timeout=5)
        return parse_clock_lines(list(self.lines))


def parse_clock_lines(lines):
    """Summary of `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,noheader,nounits`
    lines: median SM clock, the highest max clock seen, and every throttle reason that was active
    in any sample (malformed lines are skipped)."""
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            mx.append(float(parts[1]))
        except ValueError:
            continue
        for n, v in zip(names, parts[4:8]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch

    from vision_transformer_encoder_dsv4v_b200 import build as B
    from vision_transformer_encoder_dsv4v_b200 import dsv4v as A

    B.build()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if dist is not None:
            t = torch.ones(1, device="cuda")
            dist.all_reduce(t)
        torch.cuda.synchronize()

    wl = synth.workload(args.workload)
    inp = synth.draw(wl)
    cfg = A.make_config(wl.vision_dim, wl.n_heads, wl.mlp_hidden, wl.downsample_ratio, wl.llm_dim, wl.n_layers,
                        wl.eps, wl.rope_theta, A.DSV4V_BF16)
    batch = A.BatchRef(wl.grids)

    def dev(t):
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).cuda()

    layers = [{k: (torch.from_numpy(v).cuda() if isinstance(v, np.ndarray) else dev(v)) for k, v in l.items()}
              for l in inp.layers]
    lw = [A.block_weights(l) for l in layers]
    fnw = torch.from_numpy(inp.final_norm_w).cuda()
    wa = dev(inp.w_align)
    x0 = dev(inp.x)
    x = torch.empty_like(x0)
    T = A.dsv4v_aligner_tokens(cfg, batch)
    out = torch.empty(T, wl.llm_dim, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_workspace_size(cfg, batch), dtype=torch.uint8, device="cuda")
    flush = L2Flush(torch)
    stream = torch.cuda.Stream()

    # Launches of one step (the library's count for this batch and launch sequence): the rotary
    # table, the first norm operand, per layer either 4 GEMMs + attention or attention + one chain
    # launch (plus layer 0's q|k|v launch), the final norm, and the aligner's window index,
    # merged-row copy and GEMM.
    chain_path = A.dsv4v_tower_path(cfg, batch) == A.PATH_CHAIN
    launches_per_step = A.dsv4v_step_launches(cfg, batch, True, True)

    def step(s):
        x.copy_(x0)
        A.dsv4v_tower_forward(cfg, batch, lw, fnw, x, ws, stream=s.cuda_stream)
        A.dsv4v_aligner_forward(cfg, batch, x, wa, out, ws, stream=s.cuda_stream)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            with torch.cuda.stream(stream):
                step(stream)
        torch.cuda.synchronize()
        print(json.dumps({"profile_run": True, "device_error": A.dsv4v_device_error(),
                          "kernels_per_step": launches_per_step,
                          "path": "chain" if chain_path else "kernels"}), flush=True)
        return

    if args.extra:
        one = {"patch_embed": lambda: patch_embed_timing(A, torch, cfg, wl, stream, flush, args.steps),
               "patch_merger": lambda: patch_merger_timing(A, torch, cfg, batch, wl, stream, flush, args.steps),
               "bridge": lambda: bridge_timing(A, torch, cfg, stream, flush, args.steps),
               "block_backward": lambda: block_backward_timing(A, torch, cfg, batch, wl, lw, stream, flush,
                                                               args.steps),
               "workload5": lambda: workload5_timing(A, torch, lw, fnw, wa, stream, flush, args.steps)}[args.extra]()
        print(json.dumps({"extra": args.extra, **one}), flush=True)
        return

    # Capture one step (all kernels of the path, launched through the C ABI) in a CUDA graph.
    with torch.cuda.stream(stream):
        step(stream)  # warm the descriptor cache and function attributes
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step(stream)
    torch.cuda.synchronize()
    if A.dsv4v_device_error() != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            flush()
            graph.replay()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush()  # L2 flush between steps, outside the timed interval
            a.record(stream)
            graph.replay()
            b.record(stream)
    stream.synchronize()
    barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    if A.dsv4v_device_error() != 0:
        raise RuntimeError("device-side wait timed out")
    ms = total_ms / args.steps
    patches_all = wl.n_patches * world
    value = patches_all * args.steps / (total_ms / 1e3)
    tflops = synth.algorithmic_flops(wl) * world * args.steps / (total_ms / 1e3) / 1e12

    # ---- kernel timing pass: the same step as component calls, with events around each launch
    kern = kernel_timing(A, torch, cfg, batch, wl, lw, fnw, wa, x0, x, out, ws, stream, flush, args.steps)

    # ---- the step before the tower: patch embedding of the same patches (14 x 14 RGB patches)
    extras = {"patch_embed": patch_embed_timing(A, torch, cfg, wl, stream, flush, args.steps),
              "patch_merger": patch_merger_timing(A, torch, cfg, batch, wl, stream, flush, args.steps),
              "bridge": bridge_timing(A, torch, cfg, stream, flush, args.steps),
              "block_backward": block_backward_timing(A, torch, cfg, batch, wl, lw, stream, flush, args.steps)}
    if args.workload == 4:
        extras["workload5"] = workload5_timing(A, torch, lw, fnw, wa, stream, flush, min(args.steps, 10))

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region.
    # Serial: every step copies its input in, runs the two calls, copies its result out, and the
    # host waits for it.  Pipelined (the reported value): the same calls and copies for K steps on
    # a compute stream and two copy streams with two device buffer sets, so that one step's copies
    # overlap its neighbours' kernels, as a serving loop runs; one timed interval from the first
    # input copy to the last result copy.
    x_host = x0.cpu().pin_memory()
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(stream):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            x.copy_(x_host, non_blocking=True)
            A.dsv4v_tower_forward(cfg, batch, lw, fnw, x, ws, stream=stream.cuda_stream)
            A.dsv4v_aligner_forward(cfg, batch, x, wa, out, ws, stream=stream.cuda_stream)
            out_host[0].copy_(out, non_blocking=True)
            b.record(stream)
        stream.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_serial = sum(e2e_ms)
    ref_out = out_host[0].clone()

    xs, outs = [x, torch.empty_like(x)], [out, torch.empty_like(out)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "done", "out")}

    def pipelined(n):
        for i in range(n):
            k = i & 1
            if i >= 2:
                h2d.wait_event(ev["done"][k])  # step i-2 has finished reading xs[k]
            with torch.cuda.stream(h2d):
                xs[k].copy_(x_host, non_blocking=True)
            ev["in"][k].record(h2d)
            stream.wait_event(ev["in"][k])
            if i >= 2:
                stream.wait_event(ev["out"][k])  # step i-2's result has left outs[k]
            A.dsv4v_tower_forward(cfg, batch, lw, fnw, xs[k], ws, stream=stream.cuda_stream)
            A.dsv4v_aligner_forward(cfg, batch, xs[k], wa, outs[k], ws, stream=stream.cuda_stream)
            ev["done"][k].record(stream)
            d2h.wait_event(ev["done"][k])
            with torch.cuda.stream(d2h):
                out_host[k].copy_(outs[k], non_blocking=True)
            ev["out"][k].record(d2h)

    pipelined(args.warmup)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        flush()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    pipelined(args.steps)
    t1.record(d2h)
    torch.cuda.synchronize()
    e2e_total = t0.elapsed_time(t1)
    # both pipelined result buffers against the serial run's result (the path is deterministic)
    e2e_same = bool(torch.equal(out_host[0], ref_out) and torch.equal(out_host[1], ref_out))
    if dist is not None:
        t = torch.tensor([e2e_total, e2e_serial], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total, e2e_serial = float(t[0].item()), float(t[1].item())
    e2e_value = patches_all * args.steps / (e2e_total / 1e3)
    e2e_serial_value = patches_all * args.steps / (e2e_serial / 1e3)

    peaks = load_peaks()
    dom = kern["dominant"]
    # The per-class times are standalone kernel durations (events between launches) at full
    # clocks, so the burst GEMM peak is the denominator, for the dominant class and for the step.
    peak = peaks.get("bf16_tflops") or 1590.0
    traffic = TRAFFIC_BYTES.get((args.workload, dom["name"]))
    roof = {"bound": "tensor", "kernel": dom["name"], "achieved": dom["tflops"], "peak": peak, "unit": "TFLOP/s",
            "frac": dom["tflops"] / peak, "traffic": traffic,
            "traffic_unit": "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum, ncu); a GEMM's "
                            "figure includes the next GEMM's weights, which it prefetches into L2",
            "peak_source": ("MEASURED_PEAKS.json bf16_tflops, the burst cuBLAS bf16 rate (of measured)" if peaks
                            else "fallback 1.59 PF burst"),
            "peak_sustained": peaks.get("bf16_tflops_sustained"),
            "step_tflops": tflops, "step_frac": tflops / peak,
            "step_frac_of_sustained": tflops / peaks["bf16_tflops_sustained"] if peaks.get("bf16_tflops_sustained")
            else None,
            "path": kern["path"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(wl, inp, args.cpu_seconds)

    if rank == 0:
        cfgd = workload_desc(wl)
        cfgd.update({"parallelism": f"replicas x{world} (image-parallel, no collective)",
                     "l2": "flushed between timed steps (256 MB write, then a 256 MB read, outside the timed "
                           "interval); "
                           "weights (0.8 GB) exceed L2 anyway",
                     "timing": "CUDA events per step around a CUDA-graph replay of the C-ABI calls",
                     "graph": True})
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) patch states, N(0,0.02) "
                "random-init weights of the tower's shape)", "config": cfgd,
                "tflops": tflops, "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms),
                "roofline": roof, "kernels": kern["all"], "extras": extras, "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": x0.numel() * 2,
                        "d2h_bytes_per_step": out.numel() * 2,
                        "path": "dsv4v_tower_forward + dsv4v_aligner_forward C-ABI calls (the library replays "
                                "each call's CUDA graph from the second identical call on), "
                                "pinned host input/output copies of every step inside the timed region; "
                                "copies on two copy streams overlapping the neighbouring steps' kernels "
                                "(two device buffer sets), one interval over all steps",
                        "serial_value": e2e_serial_value,
                        "results_match_serial": e2e_same,
                        "serial_note": "each step alone: L2 flush, copy in, calls, copy out, host wait"},
                "gpu_launches": launches_per_step * args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


class L2Flush:
    """Evicts the 126 MB L2 between timed steps: writes a 256 MB buffer, then reads another one,
    so that the timed step starts with none of its inputs cached and with clean lines only (the
    read pass writes back the dirty lines of the write pass before the timed interval, as a
    profiler's cache flush does, instead of leaving up to 126 MB of write-backs to the step)."""

    def __init__(self, torch):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(32 << 20, dtype=torch.int64, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def kernel_timing(A, torch, cfg, batch, wl, lw, fnw, wa, x0, x, out, ws, stream, flush, steps):
    """Per-launch device time of each GEMM class and the attention kernel, from CUDA events that
    the library records on the launching stream around every launch of the step
    (dsv4v_tower_forward_profiled, same kernels and plans as dsv4v_tower_forward), captured in
    one CUDA graph and replayed `steps` times with an L2 flush between replays."""
    D, F, P, L = wl.vision_dim, wl.mlp_hidden, wl.n_patches, wl.n_layers
    kinds = A.PROFILE_KINDS
    flops = {"qkv": 2.0 * P * D * 3 * D, "out": 2.0 * P * D * D, "swiglu": 2.0 * P * D * 2 * F,
             "down": 2.0 * P * F * D, "attention": sum(4.0 * (a * b) ** 2 * D for a, b in wl.grids)}
    # the chain launch of layer l runs its output projection, SwiGLU and down projection and
    # layer l + 1's q|k|v projection (none after the last layer): average over the L launches
    flops["chain"] = flops["out"] + flops["swiglu"] + flops["down"] + flops["qkv"] * (L - 1) / L
    chain = A.dsv4v_tower_path(cfg, batch) == A.PATH_CHAIN
    active = ("attention", "chain") if chain else ("qkv", "attention", "out", "swiglu", "down")
    events = [torch.cuda.Event(enable_timing=True) for _ in range(wl.n_layers * len(kinds) * 2)]
    for e in events:  # creates the CUDA handles
        e.record(stream)
    torch.cuda.synchronize()

    def one_step():
        x.copy_(x0)
        A.dsv4v_tower_forward_profiled(cfg, batch, lw, fnw, x, ws, events, stream=stream.cuda_stream)
        A.dsv4v_aligner_forward(cfg, batch, x, wa, out, ws, stream=stream.cuda_stream)

    with torch.cuda.stream(stream):
        one_step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    times = {k: [] for k in active}
    for i in range(steps + 2):
        with torch.cuda.stream(stream):
            flush()
            g.replay()
        stream.synchronize()
        if i < 2:
            continue
        for l in range(wl.n_layers):
            for k in active:
                ki = kinds.index(k)
                a, b = events[(l * len(kinds) + ki) * 2], events[(l * len(kinds) + ki) * 2 + 1]
                times[k].append(a.elapsed_time(b))
    res = {}
    for k in active:
        ts = times[k]
        avg_us = 1e3 * sum(ts) / len(ts)
        res[k] = {"launches": len(ts), "avg_us": avg_us, "total_ms": sum(ts), "tflops": flops[k] / (avg_us * 1e-6) / 1e12}
    dom_name = max(active, key=lambda k: res[k]["total_ms"])
    return {"all": res, "dominant": {"name": dom_name, **res[dom_name]},
            "path": "chain" if chain else "kernels"}


def workload5_timing(A, torch, lw, fnw, wa, stream, flush, steps):
    """The high-resolution packed batch (16 images, 8..64 per side plus one 64x64, seed 4): the
    same tower + aligner step as the headline, CUDA-graph replay, L2 flushed between steps.  The
    patch states are the batch's own seeded draw; the weights are the headline workload's
    (same shapes; the kernels' timing does not depend on weight values).  Not in value."""
    wl = synth.workload(5)
    rng = np.random.default_rng(wl.seed)
    xv = synth._store(rng.standard_normal((wl.n_patches, wl.vision_dim), dtype=np.float32), "bf16")
    cfg = A.make_config(wl.vision_dim, wl.n_heads, wl.mlp_hidden, wl.downsample_ratio, wl.llm_dim, wl.n_layers,
                        wl.eps, wl.rope_theta, A.DSV4V_BF16)
    batch = A.BatchRef(wl.grids)
    x0 = torch.from_numpy(xv.bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    x = torch.empty_like(x0)
    out = torch.empty(A.dsv4v_aligner_tokens(cfg, batch), wl.llm_dim, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_workspace_size(cfg, batch), dtype=torch.uint8, device="cuda")

    def step():
        x.copy_(x0)
        A.dsv4v_tower_forward(cfg, batch, lw, fnw, x, ws, stream=stream.cuda_stream)
        A.dsv4v_aligner_forward(cfg, batch, x, wa, out, ws, stream=stream.cuda_stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    ts = []
    for i in range(steps + 2):
        with torch.cuda.stream(stream):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
        stream.synchronize()
        if i >= 2:
            ts.append(a.elapsed_time(b))
    if A.dsv4v_device_error() != 0:
        raise RuntimeError("device-side wait timed out (workload 5)")
    ms = statistics.median(ts)
    fl = synth.algorithmic_flops(wl)
    peaks = load_peaks()
    peak = peaks.get("bf16_tflops") or 1590.0
    del g
    return {"workload": f"{wl.name}: {len(wl.grids)} images, {wl.n_patches} patches -> {wl.n_tokens} tokens",
            "grids": wl.grids, "ms_per_step": ms, "patches_per_s": wl.n_patches / (ms * 1e-3),
            "tflops": fl / (ms * 1e-3) / 1e12, "frac_of_burst": fl / (ms * 1e-3) / 1e12 / peak,
            "path": "chain" if A.dsv4v_tower_path(cfg, batch) == A.PATH_CHAIN else "kernels", "steps": steps,
            "note": "CUDA-graph replay, median step, L2 flushed between steps; not in value"}


def patch_embed_timing(A, torch, cfg, wl, stream, flush, steps, patch=14):
    """dsv4v_patch_embed on the workload's patches (random bf16 pixels, 14 x 14 patches: K = 588
    with rows padded to 592 elements, with a bias): CUDA events around a CUDA-graph replay of
    20 calls, L2 flushed between replays.  Not part of the tower step above."""
    P, D = wl.n_patches, wl.vision_dim
    k = 3 * patch * patch
    ld = (k + 7) // 8 * 8
    g = torch.Generator(device="cuda").manual_seed(7)
    pix = torch.randn(P, ld, device="cuda", generator=g).to(torch.bfloat16)
    w = (torch.randn(D, ld, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    bias = torch.randn(D, device="cuda", generator=g)
    out = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    reps = 20
    with torch.cuda.stream(stream):
        A.dsv4v_patch_embed(cfg, P, patch, patch, pix, w, bias, out, ld, ld, stream=stream.cuda_stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(reps):
            A.dsv4v_patch_embed(cfg, P, patch, patch, pix, w, bias, out, ld, ld, stream=stream.cuda_stream)
    times = []
    for i in range(steps + 2):
        with torch.cuda.stream(stream):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
        stream.synchronize()
        if i >= 2:
            times.append(a.elapsed_time(b) / reps)
    avg_ms = sum(times) / len(times)
    flops = 2.0 * P * k * D
    return {"avg_us": avg_ms * 1e3, "tflops": flops / (avg_ms * 1e-3) / 1e12, "patch": patch, "k": k, "ld": ld,
            "bias": True, "launches_per_call": 1,
            "note": "standalone, 20 calls per graph replay; the step before the tower, not in value"}


def patch_merger_timing(A, torch, cfg, batch, wl, stream, flush, steps):
    """dsv4v_patch_merger_forward (the PatchMerger projector: LayerNorm per patch, r x r merge,
    Linear + GELU, Linear) on the workload's patches, timed like patch_embed_timing.  Not part of
    the tower step above."""
    P, D, E, r2 = wl.n_patches, wl.vision_dim, wl.llm_dim, wl.downsample_ratio ** 2
    T = wl.n_tokens
    g = torch.Generator(device="cuda").manual_seed(8)
    x = torch.randn(P, D, device="cuda", generator=g).to(torch.bfloat16)
    ln_w = 1 + 0.1 * torch.randn(D, device="cuda", generator=g)
    ln_b = 0.1 * torch.randn(D, device="cuda", generator=g)
    w1 = (torch.randn(r2 * D, r2 * D, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    b1 = 0.1 * torch.randn(r2 * D, device="cuda", generator=g)
    w2 = (torch.randn(E, r2 * D, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    b2 = 0.1 * torch.randn(E, device="cuda", generator=g)
    out = torch.empty(T, E, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_patch_merger_workspace_size(cfg, batch), dtype=torch.uint8, device="cuda")
    reps = 20

    def call():
        A.dsv4v_patch_merger_forward(cfg, batch, x, ln_w, ln_b, w1, b1, w2, b2, out, ws, stream=stream.cuda_stream)

    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(reps):
            call()
    times = []
    for i in range(steps + 2):
        with torch.cuda.stream(stream):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
        stream.synchronize()
        if i >= 2:
            times.append(a.elapsed_time(b) / reps)
    avg_ms = sum(times) / len(times)
    flops = 2.0 * T * (r2 * D) * (r2 * D) + 2.0 * T * (r2 * D) * E
    return {"avg_us": avg_ms * 1e3, "tflops": flops / (avg_ms * 1e-3) / 1e12, "tokens": T, "launches_per_call": 4,
            "note": "standalone, 20 calls per graph replay; the alternative projector, not in value"}


def graph_timed(torch, stream, flush, fn, steps):
    """Average ms of fn() captured in a CUDA graph: one replay per timed interval (CUDA events on
    the stream), each after an L2 flush outside the events; no host launch cost inside."""
    with torch.cuda.stream(stream):
        fn()  # warm descriptors and function attributes before the capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        fn()
    out = []
    for i in range(steps + 3):
        with torch.cuda.stream(stream):
            flush()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            graph.replay()
            ev1.record(stream)
        stream.synchronize()
        if i >= 3:
            out.append(ev0.elapsed_time(ev1))
    del graph
    return sum(out) / len(out)


def bridge_timing(A, torch, cfg, stream, flush, steps, n_seqs=4, seq_len=8192):
    """The image-token bridge on a language batch of n_seqs x seq_len positions holding the 16
    images of the high-resolution batch (N-layouts from dsv4v_image_layout, placed by
    synth.place_spans with text gaps, one image_pad in every fourth span), E = llm_dim bf16:
    dsv4v_merge_image_embeddings (2 launches) and dsv4v_image_visibility on an fp32
    [n_seqs, seq_len, seq_len] mask (3 launches).  Each timed call is preceded by an L2 flush
    outside its events.  Not part of the tower step above."""
    import numpy as np
    grids = synth.workload(5).grids
    r, E = cfg.downsample_ratio, cfg.llm_dim
    layouts = [A.dsv4v_image_layout(h, w, r) for h, w in grids]
    types_np = synth.place_spans(layouts, n_seqs, seq_len, seed=21, pad_every=4, balance=True)
    b = A.BatchRef(grids)
    T = A.dsv4v_aligner_tokens(cfg, b)
    g = torch.Generator(device="cuda").manual_seed(9)
    types = torch.from_numpy(types_np).cuda()
    embeds = torch.randn(n_seqs, seq_len, E, device="cuda", generator=g).to(torch.bfloat16)
    toks = torch.randn(T, E, device="cuda", generator=g).to(torch.bfloat16)
    sent = torch.randn(4, E, device="cuda", generator=g).to(torch.bfloat16)
    ws = torch.empty(A.dsv4v_bridge_workspace_size(n_seqs * seq_len), dtype=torch.uint8, device="cuda")
    mask = torch.full((n_seqs, seq_len, seq_len), float("-inf"), device="cuda")

    def timed(fn):
        return graph_timed(torch, stream, flush, fn, steps)

    merge_ms = timed(lambda: A.dsv4v_merge_image_embeddings(cfg, b, types, toks, sent, embeds, ws,
                                                            stream=stream.cuda_stream))
    vis_ms = timed(lambda: A.dsv4v_image_visibility(types, mask, ws, stream=stream.cuda_stream))
    if A.dsv4v_device_error(stream.cuda_stream) != 0:
        raise RuntimeError("bridge layout rejected on the device")
    n = n_seqs * seq_len
    pseudo = int((types_np != -1).sum())
    merge_bytes = 2.0 * pseudo * E * 2 + 2.0 * n * 4  # each pseudo row read and written; types read twice
    span_cells = 0
    for row in types_np:
        starts, ends = np.flatnonzero(row == 1), np.flatnonzero(row == 2)
        span_cells += int(((ends - starts + 1) ** 2).sum())
    vis_bytes = span_cells * 4.0  # the span blocks written; the type scans stay in L1/L2
    hbm = load_peaks().get("hbm_gbs")
    merge_gbs = merge_bytes / (merge_ms * 1e-3) / 1e9
    return {"workload": f"{len(grids)} images ({T} tokens) in {n_seqs} x {seq_len} positions, E={E} bf16",
            "pseudo_tokens": pseudo,
            "merge": {"avg_us": merge_ms * 1e3, "bytes": merge_bytes, "gbs": merge_gbs,
                      "frac_hbm": merge_gbs / hbm if hbm else None, "launches_per_call": 2},
            "visibility": {"avg_us": vis_ms * 1e3, "bytes_written": vis_bytes,
                           "gbs": vis_bytes / (vis_ms * 1e-3) / 1e9, "launches_per_call": 3},
            "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)" if hbm else None,
            "note": "standalone, the call captured in a CUDA graph, one replay per timed interval after an L2 "
                    "flush; not in value"}


def block_backward_timing(A, torch, cfg, batch, wl, lw, stream, flush, steps):
    """dsv4v_block_backward of the first block on the workload's patches (random input and output
    gradient): CUDA events around one call after an L2 flush.  The call recomputes the block's
    forward, then runs the backward; 'tflops' counts the backward's algorithmic work only (two
    GEMMs per forward GEMM, 8 N^2 D for the attention), without the recompute.  Not part of the
    tower step above."""
    P, D, F, H = wl.n_patches, wl.vision_dim, wl.mlp_hidden, wl.n_heads
    g = torch.Generator(device="cuda").manual_seed(10)
    x = torch.randn(P, D, device="cuda", generator=g).to(torch.bfloat16)
    do = torch.randn(P, D, device="cuda", generator=g).to(torch.bfloat16)
    dx = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    gb = {"norm1_w": torch.empty(D, device="cuda"), "norm2_w": torch.empty(D, device="cuda"),
          "wqkv": torch.empty(3 * D, D, dtype=torch.bfloat16, device="cuda"),
          "wo": torch.empty(D, D, dtype=torch.bfloat16, device="cuda"),
          "w_gate": torch.empty(F, D, dtype=torch.bfloat16, device="cuda"),
          "w_up": torch.empty(F, D, dtype=torch.bfloat16, device="cuda"),
          "w_down": torch.empty(D, F, dtype=torch.bfloat16, device="cuda")}
    grads = A.block_grads(gb["norm1_w"], gb["norm2_w"], gb["wqkv"], gb["wo"], gb["w_gate"], gb["w_up"], gb["w_down"])
    cos = torch.empty(P, D // H // 2, device="cuda")
    sin = torch.empty_like(cos)
    A.dsv4v_rope2d_table(cfg, batch, cos, sin, stream=stream.cuda_stream)
    ws = torch.empty(A.dsv4v_backward_workspace_size(cfg, batch), dtype=torch.uint8, device="cuda")
    def timed(fn):
        return graph_timed(torch, stream, flush, fn, steps)

    ms = timed(lambda: A.dsv4v_block_backward(cfg, batch, lw[0], cos, sin, x, do, dx, grads, ws,
                                              stream=stream.cuda_stream))
    # the attention backward alone, on the same shapes (its share of the call above)
    qkv = torch.randn(P, 3 * D, device="cuda", generator=g).to(torch.bfloat16)
    att = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    dqkv = torch.empty(P, 3 * D, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_attention(cfg, batch, qkv, att, stream=stream.cuda_stream)
    attn_ms = timed(lambda: A.dsv4v_attention_backward(cfg, batch, qkv, att, do, dqkv, ws, stream=stream.cuda_stream))
    if A.dsv4v_device_error(stream.cuda_stream) != 0:
        raise RuntimeError("device-side check failed in the block backward")
    attn_flops = sum(8.0 * (h * w) ** 2 * D for h, w in wl.grids)
    flops = 2.0 * P * (8 * D * D + 6 * D * F) + attn_flops
    return {"avg_us": ms * 1e3, "tflops": flops / (ms * 1e-3) / 1e12, "patches": P,
            "attention_backward": {"avg_us": attn_ms * 1e3, "tflops": attn_flops / (attn_ms * 1e-3) / 1e12,
                                   "launches_per_call": 4,
                                   "note": "dsv4v_attention_backward: forward attention rebuilding the row "
                                           "log-sum-exp, rowsum(do * o), dK/dV kernel, dQ kernel; flops counted "
                                           "are the backward's 8 N^2 D"},
            "note": "standalone, the call's launches captured in one CUDA graph, one replay per timed interval "
                    "after an L2 flush; recompute + backward of one block; attention backward on tcgen05; "
                    "not in value"}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh)
    except Exception:
        return {}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
