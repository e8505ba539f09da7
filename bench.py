"""Throughput of the BASED hot path on B200: Taylor linear attention + sliding-window attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

One step = one pass of the whole hot path over one batch of the 360M-shaped
workload (B=8 sequences, N=2048 tokens, 16 linear-attention heads with d'=16,
dv=64, 16 sliding-window heads of dim 64 with w=64, bf16 inputs):
  1. Taylor linear-attention prefill (y, final S and z),
  2. sliding-window prefill (y and the 64-slot ring KV cache),
  3. one generated token per sequence: linear-attention decode step and
     sliding-window decode step, continuing from the prefilled states.
Tokens per step = B*N (prefill) + B (decode). `value` is whole-job tokens/s
(all ranks) with inputs resident in HBM; `e2e` is the same through the public
API with pinned host inputs copied in and outputs copied back inside the
timed region. Multi-GPU: one process per GPU (torchrun), each rank runs its
own batch (weak scaling, no data-path collective); time is the max over ranks.

--impl reference times the CPU oracle (float64 NumPy) on a bounded sample of
the same workload: the comparison arm on the host cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill & decode tokens/s (Taylor LA + SWA) and % of roofline on 1 B200"
UNIT = "tokens/s"
WORKLOAD = dict(B=8, H=16, N=2048, d_feat=16, d_v=64, swa_heads=16, swa_dim=64, w=64)
N_INPUT_SETS = 3          # rotated so every step reads inputs last touched two steps earlier


def _feature_dim(d):
    return 1 + d + d * d


# ---------------------------------------------------------------- algorithmic work per launch
# Per head-token figures of the Taylor LA and SWA paths (bytes at bf16 inputs, fp32 state).

def la_prefill_work(B, H, N, d_feat, d_v, chunk):
    D = _feature_dim(d_feat)
    flops = B * H * N * (2 * chunk * d_feat + 2 * chunk * d_v + 2 * chunk + 4 * D * d_v + 4 * D)
    byts = B * H * N * (2 * d_feat + 2 * d_v) * 2 + B * H * (D * d_v + D) * 4
    return flops, byts


def la_backward_work(B, H, N, d_feat, d_v):
    """Gradients of the causal quadratic form: per query-key pair of the causal triangle
    the products s = q.k, g.v, ds k, ds q and a g (2(3d' + 2dv) flops); bytes: q, k, v,
    y, dy read and dq, dk, dv written once (bf16)."""
    flops = B * H * N * (N + 1) * (3 * d_feat + 2 * d_v)
    byts = B * H * N * (4 * d_feat + 4 * d_v) * 2
    return flops, byts


def swa_prefill_work(B, H, N, d, w):
    flops = B * H * N * 4 * w * d
    byts = B * H * N * 4 * d * 2 + B * H * 2 * w * d * 2      # q, k, v, y + ring cache
    return flops, byts


def la_decode_work(B, H, d_feat, d_v, packed=False):
    """Per step: read and write the fp32 state once (D rows, or D_s in the symmetric layout)."""
    D = (1 + d_feat + d_feat * (d_feat + 1) // 2) if packed else _feature_dim(d_feat)
    flops = B * H * (4 * D * d_v + 4 * D + d_feat * d_feat)
    byts = B * H * (2 * (D * d_v + D) * 4 + (2 * d_feat + 2 * d_v) * 2)
    return flops, byts


def swa_decode_work(B, H, d, w):
    flops = B * H * 4 * w * d
    byts = B * H * (2 * w * d * 2 + 2 * d * 2 + 4 * d * 2)   # ring read, slot write, q k v y
    return flops, byts


def baseconv_prefill_work(B, N, d, K):
    """u_gate and u_conv read and y written once (bf16), the state rows written once; per
    element K FMAs, the gate product and SiLU (counted as 4: negate, exp, add, divide)."""
    flops = B * N * d * (2 * K + 5)
    byts = B * N * d * 3 * 2 + B * (K - 1) * d * 2 + d * (K + 1) * 4
    return flops, byts


def baseconv_decode_work(B, d, K):
    """Per step: the K-1 state rows read and written, u_gate and u_conv read, y written (bf16)."""
    flops = B * d * (2 * K + 5)
    byts = B * d * (2 * (K - 1) + 3) * 2 + d * (K + 1) * 4
    return flops, byts


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


KERNEL_SOURCES = {
    "la_prefill": ["la_prefill_tc.cu", "tcgen05.cuh", "common.cuh", "tma_host.cu"],
    "swa_prefill": ["swa_tc.cu", "tcgen05.cuh", "common.cuh", "tma_host.cu"],
    "la_decode": ["la_decode.cu", "common.cuh"],
    "swa_decode": ["swa.cu", "common.cuh"],
}


def kernel_source_hash(kind):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "linear_attention_sequence_causal_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def measured_traffic(kind):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(p):
        return None
    pat = re.compile(r"^\|\s*%s\s*\|\s*([0-9a-f]{12})\s*\|\s*([0-9.eE+]+)\s*\|" % re.escape(kind))
    with open(p) as f:
        for line in f:
            m = pat.match(line.strip())
            if m and m.group(1) == kernel_source_hash(kind):
                return float(m.group(2))
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(self.NAMES, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus, backend="nccl"):
    """Join the job launched by torchrun (one process per GPU); returns (rank, world, local rank)."""
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, dev):
    """The slowest rank's value (timing is the max over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank, input_set):
    """Seed of one rank's input set: every rank draws its own batch (weak scaling)."""
    return 1000 * rank + input_set


def whole_job_rate(world, units_per_step, steps, max_elapsed_ms):
    """Units of all ranks per second over the slowest rank's time."""
    return world * units_per_step * steps / (max_elapsed_ms / 1e3)


# ---------------------------------------------------------------- the GPU arm

def run_mine(args):
    import torch

    import linear_attention_sequence_causal_b200 as based
    from linear_attention_sequence_causal_b200 import synthetic

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    W = WORKLOAD
    B, H, N, df, dv, Hs, ds, w = (W[k] for k in ("B", "H", "N", "d_feat", "d_v", "swa_heads", "swa_dim", "w"))
    D = _feature_dim(df)
    scale = 1.0 / math.sqrt(ds)
    chunk = 128

    # Inputs: N_INPUT_SETS seeded sets per rank, resident in HBM; one more token per
    # sequence for the decode step.
    sets = []
    for s in range(N_INPUT_SETS):
        seed = rank_seed(rank, s)
        la = synthetic.la_inputs(B, H, N + 1, df, dv, "bf16", seed=seed)
        sw = synthetic.swa_inputs(B, Hs, N + 1, ds, "bf16", seed=seed + 500)
        d = {}
        for name, t in (("q", la.q), ("k", la.k), ("v", la.v)):
            d[name] = t[:, :, :N].contiguous().to(dev)
            d[name + "1"] = t[:, :, N].contiguous().to(dev)
        for name, t in (("sq", sw.q), ("sk", sw.k), ("sv", sw.v)):
            d[name] = t[:, :, :N].contiguous().to(dev)
            d[name + "1"] = t[:, :, N].contiguous().to(dev)
        sets.append(d)
    y = torch.empty((B, H, N, dv), dtype=torch.bfloat16, device=dev)
    S = torch.empty((B, H, D, dv), dtype=torch.float32, device=dev)
    z = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    ys = torch.empty((B, Hs, N, ds), dtype=torch.bfloat16, device=dev)
    kc = torch.empty((B, Hs, w, ds), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    y1 = torch.empty((B, H, dv), dtype=torch.bfloat16, device=dev)
    ys1 = torch.empty((B, Hs, ds), dtype=torch.bfloat16, device=dev)
    ws_bytes = based.la_prefill_workspace(B, H, N, df, dv, torch.bfloat16, chunk)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def calls(d):
        return [
            lambda: based.la_prefill(d["q"], d["k"], d["v"], chunk=chunk, y=y, S=S, z=z, workspace=ws),
            lambda: based.swa_prefill(d["sq"], d["sk"], d["sv"], w=w, scale=scale, y=ys, k_cache=kc, v_cache=vc),
            lambda: based.la_decode_step(S, z, d["q1"], d["k1"], d["v1"], y=y1),
            lambda: based.swa_decode(kc, vc, N, d["sq1"], d["sk1"], d["sv1"], w=w, scale=scale, y=ys1),
        ]

    launches_per_step = 1 + (1 if ws_bytes else 0) + 1 + 1 + 1

    # Eager warm-up (also the first use of each kernel), then one CUDA graph per
    # input set holding the whole step (the four API calls): replaying it keeps
    # host launch overhead out of the device timeline of the small decode kernels.
    for i in range(args.warmup):
        for f in calls(sets[i % N_INPUT_SETS]):
            f()
    torch.cuda.synchronize(dev)
    if based.get_last_error(dev) != 0:
        raise SystemExit("device status error after warm-up")
    side = torch.cuda.Stream(dev)

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.graph(g, stream=side):
            for f in fns:
                f()
        torch.cuda.current_stream(dev).wait_stream(side)
        return g

    step_graphs = [capture(calls(d)) for d in sets]

    def step(i):
        step_graphs[i % N_INPUT_SETS].replay()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)

    gpu_index = local
    try:
        p = torch.cuda.get_device_properties(dev)
        gpu_index = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        pass
    clocks = ClockSampler(gpu_index)
    clocks.start()
    # pre-roll under load for about a second so the clock samples cover a loaded GPU
    t_pre = time.perf_counter()
    i = 0
    while time.perf_counter() - t_pre < args.preroll_s:
        step(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(args.steps):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    if based.get_last_error(dev) != 0:
        raise SystemExit("device status error in the timed region")

    # Per-kernel launch durations: one graph per API call holding its launches
    # over the rotated input sets, replayed back to back; CUDA events on the
    # launching stream around the replays.
    names = ("la_prefill", "swa_prefill", "la_decode", "swa_decode")
    per_kernel = {}
    reps = max(3, min(args.steps, 50))
    for j, name in enumerate(names):
        g = capture([calls(d)[j] for d in sets])
        g.replay()
        torch.cuda.synchronize(dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        per_kernel[name] = a.elapsed_time(b) / (reps * N_INPUT_SETS)
        del g
    clk = clocks.stop()
    clk["window"] = f"{args.preroll_s:.1f} s pre-roll of identical steps + the timed region + per-kernel replays"
    if based.get_last_error(dev) != 0:
        raise SystemExit("device status error in the per-kernel replays")
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    del step_graphs

    tokens_per_step = B * N + B
    value = whole_job_rate(world, tokens_per_step, args.steps, elapsed_ms)
    ms_per_step = elapsed_ms / args.steps

    # ---- roofline of the dominant kernel (algorithmic work / measured launch time)
    peaks = load_peaks()
    work = {
        "la_prefill": la_prefill_work(B, H, N, df, dv, chunk),
        "swa_prefill": swa_prefill_work(B, Hs, N, ds, w),
        "la_decode": la_decode_work(B, H, df, dv),
        "swa_decode": swa_decode_work(B, Hs, ds, w),
    }
    dom = max(per_kernel, key=per_kernel.get)
    flops, byts = work[dom]
    t_s = per_kernel[dom] / 1e3
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    t_byte = byts / (peaks["hbm_gbs"] * 1e9)
    if t_flop > t_byte:
        roof = {"bound": "tensor", "achieved": flops / t_s / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": byts / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(dom)
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"] + (" burst" if roof["bound"] == "tensor" else " copy")
    roof["algorithmic_per_launch"] = {"flops": flops, "bytes": byts}

    kernels = {}
    for name, ms in per_kernel.items():
        f_, b_ = work[name]
        kernels[name] = {"us": round(ms * 1e3, 2), "GB_s": round(b_ / (ms / 1e3) / 1e9, 1),
                         "TFLOP_s": round(f_ / (ms / 1e3) / 1e12, 1),
                         "roofline_frac": round(max(f_ / (peaks["bf16_tflops"] * 1e12),
                                                    b_ / (peaks["hbm_gbs"] * 1e9)) / (ms / 1e3), 3)}
    prefill_ms = per_kernel["la_prefill"] + per_kernel["swa_prefill"]
    decode_ms = per_kernel["la_decode"] + per_kernel["swa_decode"]

    # ---- end to end through the public API with pinned host buffers
    e2e = run_e2e(based, dev, stream, B, H, N, df, dv, Hs, ds, w, scale, chunk, y, S, z, ys, kc, vc, y1, ys1,
                  ws, min(args.steps, 20), world)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "360M-shaped: B=8, N=2048; Taylor LA 16 heads d'=16 dv=64; "
                               "SWA 16 heads d=64 w=64; + 1 decode token per sequence",
                   "B": B, "N": N, "la_heads": H, "d_feat": df, "d_v": dv, "swa_heads": Hs,
                   "swa_head_dim": ds, "w": w, "chunk": chunk, "tokens_per_step": tokens_per_step,
                   "l2": f"inputs rotated over {N_INPUT_SETS} sets (>{N_INPUT_SETS * 0.23:.1f} GB); "
                         "each step's inputs were last read two steps earlier",
                   "parallelism": f"dp{world}"},
        "prefill": {"tokens_per_s": world * B * N / (prefill_ms / 1e3), "ms": prefill_ms},
        "decode": {"tokens_per_s": world * B / (decode_ms / 1e3), "ms": decode_ms, "batch": B},
        "kernels": kernels,
        "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clk,
    }
    if not args.no_workloads:
        result["workloads"] = run_workloads(based, dev, stream, peaks, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(based, dev, stream, B, H, N, df, dv, Hs, ds, w, scale, chunk, y, S, z, ys, kc, vc, y1, ys1, ws,
            steps, world):
    """The bench step through the public API from pinned host buffers.

    Every step copies its own inputs host -> device and its four outputs device
    -> host. As in a serving loop, the copies of neighbouring steps run on
    their own streams (double-buffered device inputs and outputs), so step
    i+1's upload and step i-1's download overlap step i's kernels; the timed
    region runs from the first upload to the last download."""
    import torch
    from linear_attention_sequence_causal_b200 import synthetic

    la = synthetic.la_inputs(B, H, N + 1, df, dv, "bf16", seed=77)
    sw = synthetic.swa_inputs(B, Hs, N + 1, ds, "bf16", seed=78)
    host = {}
    for name, t in (("q", la.q), ("k", la.k), ("v", la.v), ("sq", sw.q), ("sk", sw.k), ("sv", sw.v)):
        host[name] = t[:, :, :N].contiguous().pin_memory()
        host[name + "1"] = t[:, :, N].contiguous().pin_memory()
    dev_in = [{n: torch.empty_like(t, device=dev) for n, t in host.items()} for _ in range(2)]
    # Every result of the step's calls: y, the final state S and z (updated by the
    # decode step), the sliding-window outputs and ring caches, the decode outputs.
    dev_out = [{"y": y, "S": S, "z": z, "ys": ys, "kc": kc, "vc": vc, "y1": y1, "ys1": ys1}]
    dev_out.append({n: torch.empty_like(t) for n, t in dev_out[0].items()})
    host_out = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in dev_out[0].items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i & 1
        d, o = dev_in[b], dev_out[b]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev_done[b])                # step i-2's kernels have read set b
            for n in host:
                d[n].copy_(host[n], non_blocking=True)
            ev_in[b].record(up)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_read[b])            # step i-2's outputs have been read back
            based.la_prefill(d["q"], d["k"], d["v"], chunk=chunk, y=o["y"], S=o["S"], z=o["z"], workspace=ws)
            based.swa_prefill(d["sq"], d["sk"], d["sv"], w=w, scale=scale, y=o["ys"], k_cache=o["kc"],
                              v_cache=o["vc"])
            based.la_decode_step(o["S"], o["z"], d["q1"], d["k1"], d["v1"], y=o["y1"])
            based.swa_decode(o["kc"], o["vc"], N, d["sq1"], d["sk1"], d["sv1"], w=w, scale=scale, y=o["ys1"])
            ev_done[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[b])
            for n in host_out:
                host_out[n].copy_(o[n], non_blocking=True)
            ev_read[b].record(down)

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(up)
    for i in range(3, 3 + steps):
        step(i)
    b.record(down)
    torch.cuda.synchronize(dev)
    if based.get_last_error(dev) != 0:
        raise SystemExit("device status error in the end-to-end steps")
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    return {"value": world * (B * N + B) * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "returned": sorted(host_out),
            "overlap": "uploads and downloads of neighbouring steps on their own streams"}


# ---------------------------------------------------------------- the other configurations

def graph_time_ms(fns, reps, dev, stream):
    """Average device time of one call of a list of calls (run in turn) captured in a
    CUDA graph and replayed `reps` times; CUDA events on the launching stream."""
    import torch
    for f in fns:
        f()
    torch.cuda.synchronize(dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for f in fns:
            f()
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    del g
    return a.elapsed_time(b) / (reps * len(fns))


def _frac(flops, byts, ms, peaks):
    """Fraction of the roofline: the slower of flops at the tensor peak and bytes at the
    HBM peak, over the measured time."""
    return max(flops / (peaks["bf16_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9)) / (ms / 1e3)


def run_workloads(based, dev, stream, peaks, world):
    """The other configurations of the workload list, each against its roofline:
      decode: H=16, d'=16, dv=64 (LA) and 16 SWA heads of 64 with w=64, batch
        1/16/64/128/256, states prefilled from a 512-token prompt; steps in a CUDA
        graph cycling over three state sets (three batch-64 LA states are 437 MB,
        so a step does not find the previous step's state in the 126 MB L2);
      long prefill: B=2, H=16, N=16384, d'=16, dv=64 at chunk 64, 128 and 256;
      large state: d'=32, dv=128, H=8, B=4, N=8192 prefill (the library's chunk),
        then decode at batch 64 (256 steps, two state sets of 277 MB).
    Prefill inputs are rotated over two sets (2 x 100 MB). Tokens/s are whole-job
    (all ranks; every rank runs its own copy)."""
    import torch
    from linear_attention_sequence_causal_b200 import synthetic

    out = {}
    H, df, dv, Hs, ds, w = 16, 16, 64, 16, 64, 64
    D = _feature_dim(df)
    scale = 1.0 / math.sqrt(ds)
    prompt, nsets, steps_per_set = 512, 3, 32
    dec = {}
    for batch in (1, 16, 64, 128, 256):
        sets = []
        for si in range(nsets):
            q, k, v = synthetic.device_la_inputs(batch, H, prompt + steps_per_set, df, dv, dev, seed=900 + si)
            sq, sk, sv = synthetic.device_swa_inputs(batch, Hs, prompt + steps_per_set, ds, dev, seed=950 + si)
            _, S, z = based.la_prefill(q[:, :, :prompt].contiguous(), k[:, :, :prompt].contiguous(),
                                       v[:, :, :prompt].contiguous())
            _, kc, vc = based.swa_prefill(sq[:, :, :prompt].contiguous(), sk[:, :, :prompt].contiguous(),
                                          sv[:, :, :prompt].contiguous(), w=w, scale=scale)
            step_in = [tuple(x[:, :, prompt + t].contiguous() for x in (q, k, v, sq, sk, sv))
                       for t in range(steps_per_set)]
            sets.append(dict(S=S, z=z, kc=kc, vc=vc, inp=step_in,
                             y=torch.empty(batch, H, dv, dtype=torch.bfloat16, device=dev),
                             ys=torch.empty(batch, Hs, ds, dtype=torch.bfloat16, device=dev)))
            del q, k, v, sq, sk, sv
        torch.cuda.synchronize(dev)

        def la_step(st, t):
            qi, ki, vi = st["inp"][t][:3]
            return lambda: based.la_decode_step(st["S"], st["z"], qi, ki, vi, y=st["y"])

        def swa_step(st, t):
            qi, ki, vi = st["inp"][t][3:]
            return lambda: based.swa_decode(st["kc"], st["vc"], prompt + t, qi, ki, vi, w=w, scale=scale, y=st["ys"])

        order = [(t, si) for t in range(steps_per_set) for si in range(nsets)]
        la_ms = graph_time_ms([la_step(sets[si], t) for t, si in order], 3, dev, stream)
        swa_ms = graph_time_ms([swa_step(sets[si], t) for t, si in order], 3, dev, stream)
        both = []
        for t, si in order:
            both += [la_step(sets[si], t), swa_step(sets[si], t)]
        step_ms = graph_time_ms(both, 3, dev, stream) * 2        # per step of both layer types
        lf, lb = la_decode_work(batch, H, df, dv)
        sf, sb = swa_decode_work(batch, Hs, ds, w)
        dec[str(batch)] = {
            "la": {"us_per_step": round(la_ms * 1e3, 2), "tokens_per_s": world * batch / (la_ms / 1e3),
                   "roofline_frac": round(_frac(lf, lb, la_ms, peaks), 3)},
            "swa": {"us_per_step": round(swa_ms * 1e3, 2), "tokens_per_s": world * batch / (swa_ms / 1e3),
                    "roofline_frac": round(_frac(sf, sb, swa_ms, peaks), 3)},
            "based_step": {"us_per_step": round(step_ms * 1e3, 2), "tokens_per_s": world * batch / (step_ms / 1e3),
                           "roofline_frac": round(_frac(lf + sf, lb + sb, step_ms, peaks), 3)},
        }
        del sets
    out["decode"] = {"workload": f"H=16 d'=16 dv=64 LA + 16 SWA heads d=64 w=64; {prompt}-token prompt "
                                 f"prefilled; {nsets} state sets rotated per step", "bound": "hbm",
                     "batches": dec}

    # long prefill
    B, N = 2, 16384
    ins = [synthetic.device_la_inputs(B, H, N, df, dv, dev, seed=30 + i) for i in range(2)]
    y = torch.empty(B, H, N, dv, dtype=torch.bfloat16, device=dev)
    S = torch.empty(B, H, D, dv, device=dev)
    z = torch.empty(B, H, D, device=dev)
    lp = {}
    for chunk in (64, 128, 256):
        wsb = based.la_prefill_workspace(B, H, N, df, dv, torch.bfloat16, chunk)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        ms = graph_time_ms([lambda qkv=qkv: based.la_prefill(*qkv, chunk=chunk, y=y, S=S, z=z, workspace=ws)
                            for qkv in ins], 5, dev, stream)
        fl, by = la_prefill_work(B, H, N, df, dv, chunk)
        lp[str(chunk)] = {"us": round(ms * 1e3, 2), "tokens_per_s": world * B * N / (ms / 1e3),
                          "TFLOP_s": round(fl / (ms / 1e3) / 1e12, 1),
                          "roofline_frac": round(_frac(fl, by, ms, peaks), 3)}
    out["long_prefill"] = {"workload": "B=2 H=16 N=16384 d'=16 dv=64 bf16, final S and z", "chunks": lp}
    del ins, y, S, z

    # large state
    Bl, Hl, Nl, dfl, dvl = 4, 8, 8192, 32, 128
    Dl = _feature_dim(dfl)
    ins = [synthetic.device_la_inputs(Bl, Hl, Nl, dfl, dvl, dev, seed=40 + i) for i in range(2)]
    y = torch.empty(Bl, Hl, Nl, dvl, dtype=torch.bfloat16, device=dev)
    S = torch.empty(Bl, Hl, Dl, dvl, device=dev)
    z = torch.empty(Bl, Hl, Dl, device=dev)
    wsb = based.la_prefill_workspace(Bl, Hl, Nl, dfl, dvl, torch.bfloat16, 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    ms = graph_time_ms([lambda qkv=qkv: based.la_prefill(*qkv, y=y, S=S, z=z, workspace=ws) for qkv in ins],
                       5, dev, stream)
    # flops at the survey's C=64 count (the smallest of the chunk-dependent counts)
    fl, by = la_prefill_work(Bl, Hl, Nl, dfl, dvl, 64)
    large = {"prefill": {"us": round(ms * 1e3, 2), "tokens_per_s": world * Bl * Nl / (ms / 1e3),
                         "TFLOP_s": round(fl / (ms / 1e3) / 1e12, 1),
                         "roofline_frac": round(_frac(fl, by, ms, peaks), 3),
                         "chunk": "library default (1024)", "flops_counted_at_chunk": 64}}
    del ins, y, S, z, ws
    lsets = []
    for si in range(2):
        q, k, v = synthetic.device_la_inputs(64, Hl, 512 + 8, dfl, dvl, dev, seed=60 + si)
        _, S, z = based.la_prefill(q[:, :, :512].contiguous(), k[:, :, :512].contiguous(), v[:, :, :512].contiguous())
        lsets.append(dict(S=S, z=z, inp=[tuple(x[:, :, 512 + t].contiguous() for x in (q, k, v)) for t in range(8)],
                          y=torch.empty(64, Hl, dvl, dtype=torch.bfloat16, device=dev)))
        del q, k, v
    fns = [lambda st=lsets[t % 2], t8=(t // 2) % 8: based.la_decode_step(st["S"], st["z"], *st["inp"][t8], y=st["y"])
           for t in range(256)]
    ms = graph_time_ms(fns, 2, dev, stream)
    fl, by = la_decode_work(64, Hl, dfl, dvl)
    large["decode"] = {"batch": 64, "steps": 256, "us_per_step": round(ms * 1e3, 2),
                       "tokens_per_s": world * 64 / (ms / 1e3), "roofline_frac": round(_frac(fl, by, ms, peaks), 3)}
    del lsets
    out["large_state"] = dict(workload="d'=32 dv=128 H=8: B=4 N=8192 prefill; decode batch 64, 256 steps", **large)
    return out


# ---------------------------------------------------------------- the CPU oracle arm

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(n_heads, seed=0):
    """Time the oracle on n_heads heads of one sequence (LA prefill + SWA prefill + decode
    token for those heads). Returns (seconds, tokens) with tokens = n_heads * (N + 1) / H."""
    import numpy as np

    import oracle
    from linear_attention_sequence_causal_b200 import synthetic

    W = WORKLOAD
    N, df, dv, ds, w = W["N"], W["d_feat"], W["d_v"], W["swa_dim"], W["w"]
    la = synthetic.la_inputs(1, n_heads, N + 1, df, dv, "bf16", seed=seed)
    sw = synthetic.swa_inputs(1, n_heads, N + 1, ds, "bf16", seed=seed + 1)
    scale = 1.0 / math.sqrt(ds)
    t0 = time.perf_counter()
    oracle.la_quadratic(la.q64[..., :N, :], la.k64[..., :N, :], la.v64[..., :N, :])
    S, z = oracle.la_state(la.k64[..., :N, :], la.v64[..., :N, :])
    oracle.la_recurrent(la.q64[..., N:, :], la.k64[..., N:, :], la.v64[..., N:, :], S, z)
    oracle.swa(sw.q64[..., :N, :], sw.k64[..., :N, :], sw.v64[..., :N, :], w, scale)
    kc, vc = oracle.swa_ring_after_prefill(sw.k64[..., :N, :], sw.v64[..., :N, :], w)
    oracle.swa_decode_step(kc, vc, N, sw.q64[..., N, :], sw.k64[..., N, :], sw.v64[..., N, :], w, scale)
    dt = time.perf_counter() - t0
    return dt, n_heads * (N + 1) / W["H"]


def cpu_baseline(seconds):
    # calibrate on one head, then size the sample to about `seconds` of CPU work
    dt1, _ = oracle_sample(1, seed=1)
    heads = max(1, min(WORKLOAD["H"] * WORKLOAD["B"], int(seconds / max(dt1, 1e-3))))
    dt, tokens = oracle_sample(heads, seed=2)
    return {"value": tokens / dt, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{heads} of {WORKLOAD['B'] * WORKLOAD['H']} (sequence, head) pairs of the "
                      f"workload (LA + SWA prefill of N={WORKLOAD['N']} plus one decode token each), "
                      f"{dt:.1f} s; tokens = heads x (N+1) / {WORKLOAD['H']}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = 150.0 / max(1, args.steps + args.warmup)          # seconds per step, whole run < ~3 min
    dt1, _ = oracle_sample(1, seed=1)
    heads = max(1, min(WORKLOAD["H"] * WORKLOAD["B"], int(budget / max(dt1, 1e-3))))
    for i in range(args.warmup):
        oracle_sample(heads, seed=10 + i)
    tot_t, tot_tok = 0.0, 0.0
    for i in range(args.steps):
        dt, tok = oracle_sample(heads, seed=100 + i)
        tot_t += dt
        tot_tok += tok
    value = tot_tok / tot_t
    sample = (f"per step {heads} (sequence, head) pairs of the workload through the float64 oracle "
              f"(LA + SWA prefill of N={WORKLOAD['N']} plus one decode token)")
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "360M-shaped: B=8, N=2048; Taylor LA 16 heads d'=16 dv=64; "
                               "SWA 16 heads d=64 w=64; + 1 decode token per sequence",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": _blas_threads(),
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------- ncu capture cases

PROFILE_CASES = {
    # inputs larger than the 126 MB L2 so DRAM counters mean something; a few hundred MB at most
    "la_prefill": "B=32 H=16 N=2048 d'=16 dv=64 bf16 (q,k,v,y 335 MB)",
    # quadratic-form kernel: K and V tiles are re-read from L2 by design, so a small
    # case (one eighth of the large-state workload, y only) shows its SM behaviour
    "la_prefill_large": "B=1 H=8 N=8192 d'=32 dv=128 bf16, y only (q,k,v,y 42 MB)",
    "swa_prefill": "B=16 H=16 N=2048 d=64 w=64 bf16 (q,k,v,y 268 MB)",
    "la_decode": "batch 256, H=16, d'=16, dv=64 (fp32 state 286 MB)",
    "swa_decode": "batch 1024, H=16, d=64, w=64 (ring caches 268 MB)",
    "la_backward": "B=8 H=16 N=2048 d'=16 dv=64 bf16 (q,k,v,y,dy,dq,dk,dv 168 MB)",
    # below L2 size, but ncu flushes the caches before every pass, so DRAM counters still count
    "baseconv": "B=8 N=2048 d=1024 K=4 bf16 (u_gate,u_conv,y 100 MB)",
}


def run_profile(kind, reps):
    """Launch one kernel `reps` times on its capture case (for ncu; prints timings only)."""
    import torch

    import linear_attention_sequence_causal_b200 as based
    from linear_attention_sequence_causal_b200 import synthetic

    dev = torch.device("cuda", 0)
    if kind == "la_prefill":
        inp = synthetic.la_inputs(32, 16, 2048, 16, 64, "bf16", seed=0)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        fn = lambda: based.la_prefill(q, k, v)
    elif kind == "la_prefill_large":
        inp = synthetic.la_inputs(1, 8, 8192, 32, 128, "bf16", seed=0)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        fn = lambda: based.la_prefill(q, k, v, want_state=False)
    elif kind == "swa_prefill":
        inp = synthetic.swa_inputs(16, 16, 2048, 64, "bf16", seed=0)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        fn = lambda: based.swa_prefill(q, k, v, w=64)
    elif kind == "la_backward":
        inp = synthetic.la_inputs(8, 16, 2048, 16, 64, "bf16", seed=0)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        dy = synthetic.upstream_grad((8, 16, 2048, 64), "bf16", seed=1)[0].to(dev)
        y, _, _ = based.la_prefill(q, k, v, want_state=False)
        fn = lambda: based.la_backward(q, k, v, y, dy)
    elif kind == "baseconv":
        c = synthetic.conv_inputs(8, 2048, 1024, 4, "bf16", seed=0)
        g, x, h, bias = (t.to(dev) for t in (c.u_gate, c.u_conv, c.h, c.bias))
        fn = lambda: based.baseconv_prefill(g, x, h, bias)
    elif kind == "la_decode":
        S = torch.randn(256, 16, 273, 64, device=dev)
        z = torch.rand(256, 16, 273, device=dev) + 300.0
        x = torch.randn(256, 16, 16, device=dev).bfloat16()
        vv = torch.randn(256, 16, 64, device=dev).bfloat16()
        fn = lambda: based.la_decode_step(S, z, x, x, vv)
    else:
        kc = torch.randn(1024, 16, 64, 64, device=dev).bfloat16()
        vc = torch.randn(1024, 16, 64, 64, device=dev).bfloat16()
        x = torch.randn(1024, 16, 64, device=dev).bfloat16()
        fn = lambda: based.swa_decode(kc, vc, 1000, x, x, x)
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    if based.get_last_error() != 0:
        raise SystemExit("device status error")
    print(json.dumps({"profile": kind, "case": PROFILE_CASES[kind], "ms": ts}))


def run_sweep(reps, only=None):
    """Extra lines beside the headline: the short gated convolution, the decode batch
    sweep (a CUDA graph of 32 steps per replay) and the long-prefill workload, each
    against its roofline. only="baseconv" stops after the convolution lines."""
    import torch

    import linear_attention_sequence_causal_b200 as based
    from linear_attention_sequence_causal_b200 import synthetic

    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)

    def timed(fn, n_inner):
        fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.graph(g, stream=side):
            for _ in range(n_inner):
                fn()
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize(dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / (reps * n_inner)

    # short gated convolution (BaseConv) at the 360M model width d=1024, K=4. The graph
    # runs three input sets in turn, so each launch reads inputs evicted from the
    # 126 MB L2 by the two launches before it (3 x 100 MB).
    Bc, Nc, dc, Kc = 8, 2048, 1024, 4
    cs = [synthetic.conv_inputs(Bc, Nc, dc, Kc, "bf16", seed=s) for s in range(3)]
    hc, bc = cs[0].h.to(dev), cs[0].bias.to(dev)
    bufs = [(c.u_gate.to(dev), c.u_conv.to(dev), torch.empty(Bc, Nc, dc, dtype=torch.bfloat16, device=dev),
             torch.empty(Bc, Kc - 1, dc, dtype=torch.bfloat16, device=dev)) for c in cs]
    del cs

    def conv_sets():
        for g, x, y, st in bufs:
            based.baseconv_prefill(g, x, hc, bc, state=st, y=y)

    ms = timed(conv_sets, 1) / len(bufs)
    flops, byts = baseconv_prefill_work(Bc, Nc, dc, Kc)
    print(json.dumps({"sweep": "baseconv_prefill", "shape": f"B={Bc} N={Nc} d={dc} K={Kc}", "us": ms * 1e3,
                      "tokens_per_s": Bc * Nc / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                      "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                      "l2": "3 input sets rotated"}), flush=True)
    del bufs
    for batch in (64, 128, 256):
        c = synthetic.conv_inputs(batch, Kc, dc, Kc, "bf16", seed=batch)
        g, x = c.u_gate[:, 0].contiguous().to(dev), c.u_conv[:, 0].contiguous().to(dev)
        st = c.u_conv[:, 1:].contiguous().to(dev)
        y = torch.empty_like(g)
        ms = timed(lambda: based.baseconv_decode(st, g, x, hc, bc, y=y), 32)
        _, byts = baseconv_decode_work(batch, dc, Kc)
        print(json.dumps({"sweep": "baseconv_decode", "batch": batch, "us_per_step": ms * 1e3,
                          "tokens_per_s": batch / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                          "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
    if only == "baseconv":
        return

    H, df, dv, D = 16, 16, 64, _feature_dim(16)
    for batch in (1, 16, 64, 128, 256):
        S = torch.randn(batch, H, D, dv, device=dev) * 0.01
        z = torch.rand(batch, H, D, device=dev) + 600.0
        inp = synthetic.la_inputs(batch, H, 1, df, dv, "bf16", seed=batch)
        q, k, v = (t[:, :, 0].contiguous().to(dev) for t in (inp.q, inp.k, inp.v))
        y = torch.empty(batch, H, dv, dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: based.la_decode_step(S, z, q, k, v, y=y), 32)
        _, byts = la_decode_work(batch, H, df, dv)
        print(json.dumps({"sweep": "la_decode", "batch": batch, "us_per_step": ms * 1e3,
                          "tokens_per_s": batch / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                          "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
        Dp = based.packed_dim(df)
        Sp = torch.randn(batch, H, Dp, dv, device=dev) * 0.01
        zp = torch.rand(batch, H, Dp, device=dev) + 600.0
        ms = timed(lambda: based.la_decode_step(Sp, zp, q, k, v, y=y, packed=True), 32)
        _, byts = la_decode_work(batch, H, df, dv, packed=True)
        print(json.dumps({"sweep": "la_decode_packed", "batch": batch, "us_per_step": ms * 1e3,
                          "tokens_per_s": batch / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                          "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
        del Sp, zp
        kc = torch.randn(batch, H, 64, 64, device=dev).bfloat16()
        vc = torch.randn(batch, H, 64, 64, device=dev).bfloat16()
        sq = torch.randn(batch, H, 64, device=dev).bfloat16()
        ys = torch.empty_like(sq)
        ms = timed(lambda: based.swa_decode(kc, vc, 1000, sq, sq, sq, w=64, scale=0.125, y=ys), 32)
        _, byts = swa_decode_work(batch, H, 64, 64)
        print(json.dumps({"sweep": "swa_decode", "batch": batch, "us_per_step": ms * 1e3,
                          "tokens_per_s": batch / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                          "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
        # one BASED decode step: the linear-attention and sliding-window layers on the same batch
        ms = timed(lambda: (based.la_decode_step(S, z, q, k, v, y=y),
                            based.swa_decode(kc, vc, 1000, sq, sq, sq, w=64, scale=0.125, y=ys)), 32)
        byts = la_decode_work(batch, H, df, dv)[1] + swa_decode_work(batch, H, 64, 64)[1]
        print(json.dumps({"sweep": "based_decode_step", "batch": batch, "us_per_step": ms * 1e3,
                          "tokens_per_s": batch / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                          "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
        del S, z, kc, vc
    # large state: d'=32 (D=1057), dv=128, H=8, B=4, N=8192 prefill, then decode at batch 64
    Bl, Hl, Nl, dfl, dvl = 4, 8, 8192, 32, 128
    Dl = _feature_dim(dfl)
    inp = synthetic.la_inputs(Bl, Hl, Nl, dfl, dvl, "bf16", seed=0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    y = torch.empty(Bl, Hl, Nl, dvl, dtype=torch.bfloat16, device=dev)
    S = torch.empty(Bl, Hl, Dl, dvl, device=dev)
    z = torch.empty(Bl, Hl, Dl, device=dev)
    wsl = torch.empty(max(16, based.la_prefill_workspace(Bl, Hl, Nl, dfl, dvl, torch.bfloat16, 0)),
                      dtype=torch.uint8, device=dev)
    ms = timed(lambda: based.la_prefill(q, k, v, y=y, S=S, z=z, workspace=wsl), 1)
    flops, byts = la_prefill_work(Bl, Hl, Nl, dfl, dvl, 64)
    print(json.dumps({"sweep": "la_prefill_large_state", "us": ms * 1e3, "tokens_per_s": Bl * Nl / (ms / 1e3),
                      "TFLOP_s": flops / (ms / 1e3) / 1e12,
                      "tensor_frac": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                      "GB_s": byts / (ms / 1e3) / 1e9}), flush=True)
    del q, k, v, y
    S = torch.randn(64, Hl, Dl, dvl, device=dev) * 0.01
    z = torch.rand(64, Hl, Dl, device=dev) + 600.0
    inp = synthetic.la_inputs(64, Hl, 1, dfl, dvl, "bf16", seed=1)
    q, k, v = (t[:, :, 0].contiguous().to(dev) for t in (inp.q, inp.k, inp.v))
    y = torch.empty(64, Hl, dvl, dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: based.la_decode_step(S, z, q, k, v, y=y), 32)
    _, byts = la_decode_work(64, Hl, dfl, dvl)
    print(json.dumps({"sweep": "la_decode_large_state", "batch": 64, "us_per_step": ms * 1e3,
                      "tokens_per_s": 64 / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                      "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
    del S, z
    Dpl = based.packed_dim(dfl)
    S = torch.randn(64, Hl, Dpl, dvl, device=dev) * 0.01
    z = torch.rand(64, Hl, Dpl, device=dev) + 600.0
    ms = timed(lambda: based.la_decode_step(S, z, q, k, v, y=y, packed=True), 32)
    _, byts = la_decode_work(64, Hl, dfl, dvl, packed=True)
    print(json.dumps({"sweep": "la_decode_large_state_packed", "batch": 64, "us_per_step": ms * 1e3,
                      "tokens_per_s": 64 / (ms / 1e3), "GB_s": byts / (ms / 1e3) / 1e9,
                      "hbm_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}), flush=True)
    del S, z
    # coarse decay (one gamma per 128-token tile): the quadratic-form path at the 360M and large shapes
    for (Bd, Hd, Nd, dfd, dvd, cd) in ((8, 16, 2048, 16, 64, 128), (4, 8, 8192, 32, 128, 32)):
        inp = synthetic.la_inputs(Bd, Hd, Nd, dfd, dvd, "bf16", seed=4)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        gam = torch.full((Bd, Hd, (Nd + 127) // 128), 0.95, dtype=torch.float32, device=dev)
        yd = torch.empty(Bd, Hd, Nd, dvd, dtype=torch.bfloat16, device=dev)
        Dd = _feature_dim(dfd)
        Sd = torch.empty(Bd, Hd, Dd, dvd, device=dev)
        zd = torch.empty(Bd, Hd, Dd, device=dev)
        wsd = torch.empty(max(16, based.lib().based_la_prefill_decay_workspace(Bd, Hd, Nd, dfd, dvd)),
                          dtype=torch.uint8, device=dev)
        ms = timed(lambda: based.la_prefill_decay(q, k, v, gam, y=yd, S=Sd, z=zd, workspace=wsd), 1)
        flops, byts = la_prefill_work(Bd, Hd, Nd, dfd, dvd, cd)
        print(json.dumps({"sweep": "la_prefill_decay", "shape": f"B={Bd} H={Hd} N={Nd} d'={dfd} dv={dvd}",
                          "us": ms * 1e3, "tokens_per_s": Bd * Nd / (ms / 1e3),
                          "TFLOP_s": flops / (ms / 1e3) / 1e12,
                          "tensor_frac": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]}), flush=True)
        del q, k, v, gam, yd, Sd, zd, wsd
    # backward (training) pass at the 360M shape and the large-state shape
    for (Bb, Hb, Nb, dfb, dvb) in ((8, 16, 2048, 16, 64), (4, 8, 8192, 32, 128)):
        inp = synthetic.la_inputs(Bb, Hb, Nb, dfb, dvb, "bf16", seed=2)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        dy = synthetic.upstream_grad((Bb, Hb, Nb, dvb), "bf16", seed=3)[0].to(dev)
        y, _, _ = based.la_prefill(q, k, v, want_state=False)
        grads = tuple(torch.empty_like(t) for t in (q, k, v))
        ws = torch.empty(based.la_backward_workspace(Bb, Hb, Nb, dfb, dvb), dtype=torch.uint8, device=dev)
        ms = timed(lambda: based.la_backward(q, k, v, y, dy, *grads, workspace=ws), 1)
        flops, byts = la_backward_work(Bb, Hb, Nb, dfb, dvb)
        print(json.dumps({"sweep": "la_backward", "shape": f"B={Bb} H={Hb} N={Nb} d'={dfb} dv={dvb}",
                          "us": ms * 1e3, "tokens_per_s": Bb * Nb / (ms / 1e3),
                          "TFLOP_s": flops / (ms / 1e3) / 1e12,
                          "tensor_frac": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                          "GB_s": byts / (ms / 1e3) / 1e9}), flush=True)
        del q, k, v, dy, y, grads, ws
    # long prefill: B=2, H=16, N=16384
    B, N = 2, 16384
    inp = synthetic.la_inputs(B, H, N, df, dv, "bf16", seed=0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    for chunk in (64, 128, 256):
        try:
            ws_bytes = based.la_prefill_workspace(B, H, N, df, dv, torch.bfloat16, chunk)
            ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
            y = torch.empty(B, H, N, dv, dtype=torch.bfloat16, device=dev)
            S = torch.empty(B, H, D, dv, device=dev)
            z = torch.empty(B, H, D, device=dev)
            ms = timed(lambda: based.la_prefill(q, k, v, chunk=chunk, y=y, S=S, z=z, workspace=ws), 1)
        except based.BasedError as e:
            print(json.dumps({"sweep": "la_prefill_long", "chunk": chunk, "unsupported": str(e)}), flush=True)
            continue
        flops, byts = la_prefill_work(B, H, N, df, dv, chunk)
        print(json.dumps({"sweep": "la_prefill_long", "chunk": chunk, "us": ms * 1e3,
                          "tokens_per_s": B * N / (ms / 1e3), "TFLOP_s": flops / (ms / 1e3) / 1e12,
                          "tensor_frac": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                          "GB_s": byts / (ms / 1e3) / 1e9}), flush=True)


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=("mine", "reference"), default="mine")
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU oracle sample size")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-workloads", action="store_true", help="skip the other configurations' lines")
    p.add_argument("--preroll-s", type=float, default=1.0, help="loaded seconds before the timed region")
    p.add_argument("--profile", choices=sorted(PROFILE_CASES), help="run one kernel on its ncu capture case")
    p.add_argument("--profile-reps", type=int, default=3)
    p.add_argument("--sweep", nargs="?", const="all", choices=("all", "baseconv"),
                   help="decode batch sweep and long-prefill lines (baseconv: the convolution lines only)")
    args = p.parse_args(argv)
    if args.profile:
        run_profile(args.profile, args.profile_reps)
        return
    if args.sweep:
        run_sweep(max(3, min(args.steps, 20)), only=args.sweep)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mine(args)


if __name__ == "__main__":
    main()
