"""Benchmark of the ternary GEMV hot path on B200 (one JSON line on rank 0).

Default workload (the headline): the decode layer stack -- 30 independently
seeded copies of a BitNet-b1.58-2B-4T decoder layer, 7 ternary projections
each (210 projections, 2.08e9 weights, 521 MB packed), M = 1. One step is one
pass of the whole path over that stack: absmax-int8 quantisation of 210 fresh
bf16 activation vectors and the 210 GEMVs with their scale epilogues, in one
persistent launch (tq_gemv_stack with TQ_STACK_QUANTIZE). The weight stream is
larger than L2, so no flush is needed between steps. Other workloads of several
projections group them the same way: one quantising stack launch at M = 1, the
stack quantiser plus tq_gemv_stack_batch at M = 2..32 (the streaming kernel up
to 2 tokens, the warp-MMA kernel for 3..24, the tensor-core group plan from
25); single projections and
prefill run one quantiser launch and one GEMV launch per projection.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

value  = algorithmic bytes of a step (all ranks) / device time per step, GB/s
e2e    = the same metric through the same calls with host buffers: each step
         copies the activations in from pinned host memory and the outputs back
roofline = the dominant kernel (the quantising stack GEMV for the stack; the
         GEMV or prefill GEMM otherwise): its algorithmic bytes (or int8 ops)
         over its average CUDA-event duration inside the timed region, against
         the measured HBM copy bandwidth (or int8 tensor peak).
--impl reference times the oracle (plain C, one host thread) on a bounded
sample of the same workload; it is the CPU baseline, not a GPU arm.
With N > 1 (torchrun) every rank runs its own replica of the workload
(replicas only: the path has no exchange step); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import (HADAMARD_BLOCK, NEXT_WORKLOADS, WORKLOADS, algorithmic_bytes,  # noqa: E402
                       binary_bytes, make_binary_projections, make_projections)

METRIC = ("ternary GEMV achieved HBM GB/s (% of B200 peak) at M=1; layer-stack passes/s")
PEAK_FALLBACK_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
STACK_KERNEL_SRC = os.path.join(ROOT, "ternary_absmax_int8_b200", "csrc", "gemv_stream.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
TRAFFIC_BINARY_FILE = os.path.join(ROOT, "profiles", "traffic_binary.json")

DESCRIPTIONS = {
    "stack30_m1": "decode layer stack: 30 x BitNet-b1.58-2B-4T decoder layer (q,k,v,o,gate,up,"
                  "down ternary projections), M=1, 210 projections, 2.08e9 weights",
    "stack10_m1": "decode layer stack: 10 x BitNet-b1.58-2B-4T decoder layer, M=1 "
                  "(profiling case)",
    "stack30_m2": "decode layer stack (30 layers, 210 projections) at M=2 tokens per projection",
    "stack30_m4": "decode layer stack (30 layers, 210 projections) at M=4 tokens per projection",
    "stack30_m8": "decode layer stack (30 layers, 210 projections) at M=8 tokens per projection",
    "stack30_m16": "decode layer stack (30 layers, 210 projections) at M=16 tokens per "
                   "projection",
    "stack30_m24": "decode layer stack (30 layers, 210 projections) at M=24 tokens per "
                   "projection",
    "layer_m1": "one BitNet-b1.58-2B-4T decoder layer, 7 ternary projections, M=1",
    "single_640x2560_m1": "one ternary projection N=640 K=2560, M=1",
    "prefill_m512": "prefill M=512 through ternary 6912x2560, 2560x6912, 17408x5120",
    "prefill_had4_m512": "prefill M=512 through ternary 6912x2560, 2560x6912, 17408x5120 with "
                         "Hadamard-rotated 4-bit activations (blockwise rotation, n=256)",
    "binary_ffn27b_m1": "binary g128 decode: 8 x 27B-scale FFN layer (gate/up 17408x5120, down "
                        "5120x17408), 1 bit + fp16 scale per 128 weights, M=1, 24 projections, "
                        "2.14e9 weights",
}


def quant_bytes(K: int, M: int) -> int:
    """bf16 in, int8 out, fp32 scale + int32 sum out."""
    return M * K * 2 + M * K + M * 8


def step_bytes(projs) -> int:
    """Quantiser launch + GEMV launch per projection."""
    return sum(quant_bytes(p.K, p.M) + algorithmic_bytes(p.N, p.K, p.M) for p in projs)


def step_mode(projs) -> str:
    """How a step launches: "fused" -- one quantising stack launch for every
    projection (M = 1, also a single projection); "batch" -- the stack
    quantiser, then tq_gemv_stack_batch (M = 2..32); "prefill" -- the stack
    quantiser, then tq_gemm_prefill_stack (M >= 33, several projections);
    "per_projection" -- a quantiser launch and a GEMV launch per projection
    (a single projection of several tokens)."""
    M = projs[0].M
    if M == 1:
        return "fused"
    if len(projs) > 1 and M <= 32:
        return "batch"
    if len(projs) > 1:
        return "prefill"
    return "per_projection"


def batch_launches(n: int, M: int) -> int:
    """Kernel launches of tq_quantize_act_stack_batch + tq_gemv_stack_batch
    over n projections of M tokens: 512 projections per quantiser launch; 256
    projections per streaming or warp-MMA launch, 64 per tensor-core group
    launch."""
    per = 64 if batch_kernel_name(M, "batch") == "smallm_group_kernel" else 256
    return -(-n // 512) + -(-n // per)


def prefill_launches(n: int, M: int) -> int:
    """Kernel launches of tq_quantize_act_stack_batch + tq_gemm_prefill_stack
    over n projections of M >= 33 tokens: 512 projections per quantiser
    launch, 16 projections per prefill launch (up to 4096 tiles each, which
    every measured shape stays within)."""
    return -(-n // 512) + -(-n // 16)


def workload_step_bytes(workload: str, projs) -> int:
    """Algorithmic bytes of one step of `workload` over `projs` (both arms)."""
    return fused_step_bytes(projs) if step_mode(projs) == "fused" else step_bytes(projs)


def fused_step_bytes(projs) -> int:
    """One quantising GEMV launch per projection: the GEMV's bytes with bf16
    activations read (2K) and int8 codes written (K) instead of int8 codes
    read (K), plus the scale and sum written (8) instead of read (8)."""
    return sum(algorithmic_bytes(p.N, p.K, p.M) + 2 * p.M * p.K for p in projs)


# ----------------------------------------------------------------- helpers
def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank timings (one collective; identity at N=1)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Units of all ranks per second of the slowest rank's time (ms)."""
    return world * units_per_rank / (ms * 1e-3)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"tq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 10:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        busy = [r for r in rows if r[4].isdigit() and int(r[4]) > 0] or rows
        sm = [int(r[1]) for r in busy if r[1].isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": int(rows[0][2]) if rows[0][2].isdigit() else None,
                "reasons": reasons, "samples": len(busy)}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return PEAK_FALLBACK_GBS, "fallback"


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return 2.0 * float(d["bf16_tflops"]), "measured bf16 burst x 2 (nominal int8:bf16)"
    except (OSError, KeyError, ValueError):
        return 2.0 * 1590.0, "fallback 1.59 PFLOP/s bf16 x 2"


def stack_kernel_sha() -> str:
    """Hash of the stack kernel's sources: its file, the headers it uses and
    the streaming section of the launch-parameter header (other kernels'
    declarations there do not change it)."""
    d = os.path.dirname(STACK_KERNEL_SRC)
    h = hashlib.sha256()
    for name in ("gemv_stream.cu", "quant_core.cuh", "tq_device.cuh"):
        h.update(open(os.path.join(d, name), "rb").read())
    text = open(os.path.join(d, "tq_internal.h"), "rb").read()
    start = text.index(b"// ------------------------------------------------- streaming GEMV")
    end = text.index(b"\n// ------", start + 1)
    h.update(text[start:end])
    return h.hexdigest()[:16]


def binary_kernel_sha() -> str:
    """Hash of the binary g128 kernels' sources (their file, the headers they
    use and the binary section of the launch-parameter header)."""
    d = os.path.dirname(STACK_KERNEL_SRC)
    h = hashlib.sha256()
    for name in ("gemv_binary.cu", "mma_common.cuh", "tq_device.cuh"):
        h.update(open(os.path.join(d, name), "rb").read())
    text = open(os.path.join(d, "tq_internal.h"), "rb").read()
    start = text.index(b"// --------------------------------------------- binary g128 GEMV")
    end = text.index(b"\n// Device address of the library's error word", start + 1)
    h.update(text[start:end])
    return h.hexdigest()[:16]


def recorded_binary_traffic(workload: str, kernel: str):
    """DRAM bytes of one binary GEMV launch from a committed ncu summary of
    the same kernel version and workload; None otherwise."""
    try:
        d = json.load(open(TRAFFIC_BINARY_FILE))
    except (OSError, ValueError):
        return None
    if (d.get("kernel_sha") != binary_kernel_sha() or d.get("workload") != workload
            or d.get("kernel") != kernel):
        return None
    return float(d["dram_bytes_read"] + d["dram_bytes_write"])


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the stack kernel from a committed ncu summary,
    scaled to this workload; None if absent or taken on another kernel version."""
    try:
        d = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    if d.get("kernel_sha") != stack_kernel_sha() or workload != "stack30_m1":
        return None
    return float(d["bytes_per_packed_byte"]) * d["full_packed_bytes"]


def step_spread(marks, steps_per_chunk: int):
    """Median, 10th and 90th percentile of the time per step (ms) over the
    chunks between consecutive recorded events (None for fewer than two
    chunks). The machine's GPUs are shared, so the spread is part of the
    record."""
    if len(marks) < 3:
        return None
    per = sorted(a.elapsed_time(b) / steps_per_chunk for a, b in zip(marks, marks[1:]))
    return {"median_ms": round(percentile(per, 50), 5), "p10_ms": round(percentile(per, 10), 5),
            "p90_ms": round(percentile(per, 90), 5), "chunks": len(per),
            "steps_per_chunk": steps_per_chunk}


def percentile(sorted_vals, q: float) -> float:
    """Linear-interpolated percentile q (0..100) of an ascending list."""
    if not sorted_vals:
        raise ValueError("no values")
    x = (len(sorted_vals) - 1) * q / 100.0
    lo = int(x)
    hi = min(lo + 1, len(sorted_vals) - 1)
    return sorted_vals[lo] + (sorted_vals[hi] - sorted_vals[lo]) * (x - lo)


def pipelined_steps(steps: int, stream, up, down, h2d, compute, d2h):
    """Enqueue `steps` end-to-end steps on two buffer sets: step i's
    host-to-device copy (h2d(i, b) on stream `up`) overlaps step i - 1's
    compute (compute(i, b, stream)), and its device-to-host copy (d2h(i, b)
    on stream `down`) overlaps step i + 1's compute; buffer b = i % 2 is
    reused only after step i - 2's compute and download are done. Every
    step's inputs are uploaded and its outputs read back."""
    import torch

    computed = [torch.cuda.Event(), torch.cuda.Event()]
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    downloaded = [torch.cuda.Event(), torch.cuda.Event()]
    up.wait_stream(stream)
    down.wait_stream(stream)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])  # step i - 2 has read buffer b's inputs
            h2d(i, b)
            uploaded[b].record(up)
        stream.wait_event(uploaded[b])
        if i >= 2:
            stream.wait_event(downloaded[b])  # step i - 2's outputs are on the host
        compute(i, b, stream)
        computed[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            d2h(i, b)
            downloaded[b].record(down)
    stream.wait_stream(up)
    stream.wait_stream(down)


def pipelined_e2e(steps: int, stream, h2d, compute, d2h, chunk: int = 64) -> float:
    """Device time (ms) of `steps` (a multiple of `chunk`) end-to-end steps:
    pipelined_steps over `chunk` steps captured once in a CUDA graph (the
    copies from and to pinned host memory, the library calls and the
    cross-stream events), replayed steps / chunk times."""
    import torch

    cs, up, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    cs.wait_stream(stream)
    with torch.cuda.stream(cs):
        pipelined_steps(2, cs, up, down, h2d, compute, d2h)  # eager warm-up
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        pipelined_steps(chunk, cs, up, down, h2d, compute, d2h)
    stream.wait_stream(cs)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps // chunk):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1)


# -------------------------------------------------------------- our arm
def run_ours(args, rank: int, world: int):
    import torch

    import ternary_absmax_int8_b200 as tq

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    shapes, M = WORKLOADS[args.workload]
    projs = list(make_projections(shapes, M=M, seed=args.seed))
    mode = step_mode(projs)
    stack = mode == "fused"
    # The fused stack quantises inside its GEMV launch; the other modes run a
    # quantiser launch first.
    sb = workload_step_bytes(args.workload, projs)
    gemv_bytes = sb if stack else sum(algorithmic_bytes(p.N, p.K, p.M) for p in projs)
    packed_bytes = sum(p.N * p.K // 4 for p in projs)

    # Weights: packed on the host by the library's packer, then resident in
    # HBM. Small workloads rotate several copies so a step's weights are never
    # still in L2 from the previous step.
    copies = 1 if packed_bytes > 2 * L2_BYTES else -(-2 * L2_BYTES // packed_bytes)
    packed = []
    for p in projs:
        P = np.empty((p.N // 4, p.K), dtype=np.uint8)
        tq.tq_pack_host(p.w, P, p.M, p.N, p.K)
        packed.append([torch.from_numpy(P).cuda() for _ in range(copies)])
    w_scales = [float(p.w_scale) for p in projs]

    # Activations and outputs: one contiguous buffer each, per-projection views.
    kx = [p.M * p.K for p in projs]
    ny = [p.M * p.N for p in projs]
    ox = np.concatenate([[0], np.cumsum(kx)]).astype(np.int64)
    oy = np.concatenate([[0], np.cumsum(ny)]).astype(np.int64)
    x_host = torch.empty(int(ox[-1]), dtype=torch.int16).pin_memory()
    for j, p in enumerate(projs):
        x_host[ox[j]:ox[j + 1]] = torch.from_numpy(p.x_bf16.view(np.int16).reshape(-1))
    x_dev = x_host.cuda()
    xq = torch.empty(int(ox[-1]), dtype=torch.int8, device="cuda")
    y_dev = torch.empty(int(oy[-1]), dtype=torch.float32, device="cuda")
    y_host = torch.empty(int(oy[-1]), dtype=torch.float32).pin_memory()
    moff = np.concatenate([[0], np.cumsum([p.M for p in projs])]).astype(np.int64)
    xs = torch.empty(int(moff[-1]), dtype=torch.float32, device="cuda")
    xsum = torch.empty(int(moff[-1]), dtype=torch.int32, device="cuda")

    # a second activation / output buffer pair for the end-to-end pipeline
    # (step i's inputs upload while step i - 1 computes)
    x_dev_b = torch.empty_like(x_dev)
    y_dev_b = torch.empty_like(y_dev)
    y_host_b = torch.empty_like(y_host).pin_memory()

    def table(c, xb=x_dev, yb=y_dev):
        return [tq.make_proj(packed=packed[j][c], x=xb.data_ptr() + 2 * int(ox[j]),
                             xq=xq.data_ptr() + int(ox[j]),
                             x_scale=xs.data_ptr() + 4 * int(moff[j]),
                             x_sum=xsum.data_ptr() + 4 * int(moff[j]),
                             y=yb.data_ptr() + 4 * int(oy[j]), w_scale=w_scales[j],
                             N=p.N, K=p.K) for j, p in enumerate(projs)]

    tables = [table(c) for c in range(copies)]
    tables_b = [table(c, x_dev_b, y_dev_b) for c in range(copies)]
    stream = torch.cuda.current_stream()

    def quant(c, s, tabs=None):
        tabs = tabs or tables
        if stack:
            return  # quantised inside the stack launch
        if mode in ("batch", "prefill"):
            tq.tq_quantize_act_stack_batch(tabs[c], M, stream=s)
            return
        for j, p in enumerate(projs):
            t = tabs[c][j]
            tq.tq_quantize_act(t.x, t.xq, t.x_scale, t.x_sum, p.M, p.N, p.K, stream=s)

    def gemv(c, s, first=True, tabs=None):
        tabs = tabs or tables
        if stack:
            # Consecutive stack launches may overlap (the next one streams
            # weights while the previous one drains); the first launch of a
            # captured sequence has no predecessor to overlap.
            flags = tq.TQ_STACK_QUANTIZE | (0 if first else tq.TQ_STACK_OVERLAP_PREV)
            tq.tq_gemv_stack(tabs[c], flags=flags, stream=s)
            return
        if mode == "batch":
            # weights may stream while the quantiser drains
            tq.tq_gemv_stack_batch(tabs[c], M, flags=tq.TQ_STACK_OVERLAP_PREV, stream=s)
            return
        if mode == "prefill":
            tq.tq_gemm_prefill_stack(tabs[c], M, stream=s)
            return
        for j, p in enumerate(projs):
            t = tabs[c][j]
            call = tq.tq_gemv if p.M <= 24 else tq.tq_gemm_prefill
            call(t.packed, t.w_scale, t.xq, t.x_scale, t.x_sum, t.y, None, p.M, p.N, p.K, stream=s)

    def step(c, s, first=True, tabs=None):
        quant(c, s, tabs)
        gemv(c, s, first, tabs)

    launches_per_step = {"fused": 1, "batch": batch_launches(len(projs), M),
                         "prefill": prefill_launches(len(projs), M)}.get(
        mode, sum(1 + gemv_launches(p.M) for p in projs))

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for i in range(args.warmup):
        step(i % copies, stream)
    torch.cuda.synchronize()

    # The timed steps replay CUDA graphs of the same library calls, so host
    # launch overhead does not stretch the device time: a chunk graph holds
    # S consecutive steps (a multiple of the rotated weight copies), and
    # single-step graphs cover a remainder, so exactly K steps run.
    K = args.steps
    S = copies * max(1, 16 // copies)
    n_chunks, rem = divmod(K, S)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=cs):
            fn(cs)
        return g

    chunk_graph = capture(lambda cs: [step(i % copies, cs, first=(i == 0)) for i in range(S)])
    single = [capture(lambda cs, c=c: step(c, cs)) for c in range(copies)] if rem else []
    chunk_graph.replay()
    for g in single:
        g.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # an event after every chunk (between graph replays, which do not overlap
    # anyway): the spread of the time per step across the chunks
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(n_chunks)]
    barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for c in range(n_chunks):
        chunk_graph.replay()
        marks[c].record(stream)
    for i in range(rem):
        single[(n_chunks * S + i) % copies].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = t0.elapsed_time(t1)
    spread = step_spread([t0] + marks, S)

    # The split between quantiser and GEMV launches (non-stack workloads):
    # graphs of S steps' quantiser calls alone and GEMV calls alone.
    def graph_ms(fn, reps=3):
        g = capture(fn)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    if stack:
        quant_ms_step, gemv_ms_step = 0.0, total_ms / K
    else:
        quant_ms_step = graph_ms(lambda cs: [quant(i % copies, cs) for i in range(S)]) / S
        gemv_ms_step = graph_ms(lambda cs: [gemv(i % copies, cs) for i in range(S)]) / S

    # End to end through the library calls themselves: host activations in,
    # host outputs out, every step, double-buffered so that step i + 1's
    # upload and step i - 1's download overlap step i, replayed from a CUDA
    # graph of 64 such steps (replays run one after another, so each costs
    # one upload and one download that overlap no compute). At least half a
    # second of it, so that the clock samples see the GPU under load.
    chunk = 64
    e2e_steps = -(-max(K, int(0.5e3 / max(total_ms / K, 1e-3))) // chunk) * chunk
    xb, yb, yh = (x_dev, x_dev_b), (y_dev, y_dev_b), (y_host, y_host_b)
    tb = (tables, tables_b)
    io = dict(h2d=lambda i, b: xb[b].copy_(x_host, non_blocking=True),
              compute=lambda i, b, s: step(i % copies, s, tabs=tb[b]),
              d2h=lambda i, b: yh[b].copy_(yb[b], non_blocking=True))
    barrier()
    e2e_ms = pipelined_e2e(e2e_steps, stream, chunk=chunk, **io)
    barrier()
    # both buffer sets carry the same step (same inputs, copies of the same
    # weights): equal host outputs show that the pipeline kept its order
    assert torch.equal(y_host, y_host_b), "end-to-end pipeline outputs differ"

    # Per-projection GEMM timing (workloads of separate calls, and the small
    # batches for comparison with their grouped launch): a graph of R calls of
    # one projection over the rotated weight copies, time per call.
    per_proj = []
    if (not stack or len(projs) == 1) and len(projs) <= 8:
        R = copies * max(1, 32 // copies)
        for j, p in enumerate(projs):
            call = tq.tq_gemv if p.M <= 24 else tq.tq_gemm_prefill

            def proj_calls(cs, j=j, p=p, call=call):
                for r in range(R):
                    t_ = tables[r % copies][j]
                    call(t_.packed, t_.w_scale, t_.xq, t_.x_scale, t_.x_sum, t_.y, None, p.M,
                         p.N, p.K, stream=cs)

            us = graph_ms(proj_calls) / R * 1e3
            entry = {"name": p.name, "N": p.N, "K": p.K, "M": p.M, "us": round(us, 3),
                     "GB_s": round(algorithmic_bytes(p.N, p.K, p.M) / (us * 1e3), 1)}
            if p.M > 24:
                entry["TOPS"] = round(2.0 * p.M * p.N * p.K / (us * 1e6), 1)
            else:
                entry["token_proj_per_s"] = round(p.M / (us * 1e-6), 1)
            per_proj.append(entry)
    time.sleep(0.3)
    clk = clocks.stop()
    assert tq.tq_device_error(reset=True) == 0, "a kernel reported a device error"

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device="cuda")
    if rank != 0:
        return None

    ms_step = total_ms / K
    value = whole_job_rate(world, sb, ms_step) / 1e9
    peak, peak_kind = measured_peak()
    gemv_avg = gemv_ms_step
    achieved = gemv_bytes / (gemv_avg * 1e6)
    traffic = recorded_traffic(args.workload)
    prefill = M > 24
    flops = sum(2.0 * p.M * p.N * p.K for p in projs)
    if prefill:
        # int8 contraction: tensor-bound. Peak = measured dense bf16 x the
        # nominal int8 : bf16 ratio (4.5 : 2.25 PFLOP/s).
        tpeak, tkind = measured_tensor_peak()
        roof = {"kernel": prefill_kernel_name(M), "bound": "tensor",
                "achieved": round(flops / (gemv_avg * 1e9), 1), "peak": tpeak,
                "peak_kind": tkind, "unit": "TOPS (int8)",
                "frac": round(flops / (gemv_avg * 1e9) / tpeak, 4), "traffic": None,
                "algorithmic_ops_per_step": flops}
    else:
        roof = {
            "kernel": batch_kernel_name(M, mode),
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs copy bandwidth)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "algorithmic_bytes_per_launch": gemv_bytes,
        }
    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "step_spread": spread,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 (bf16 activations in, int8 x ternary -> int32, fp32 out)",
        "data": "synthetic (seeded ternary weights P=0.3/0.4/0.3, bf16 N(0,1) activations "
                "with 1% x20 outliers)",
        "config": {
            "workload": f"{args.workload}: {DESCRIPTIONS.get(args.workload, args.workload)}",
            "projections": len(projs),
            "tokens_M": M,
            "packed_weight_bytes": packed_bytes,
            "step_bytes": sb,
            "weight_copies_rotated": copies,
            "l2": ("inputs larger than L2 (weight stream > 126 MB), no flush" if copies == 1 else
                   f"{copies} rotated weight copies, {copies * packed_bytes / 2**20:.0f} MiB > L2"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "seed": args.seed,
        },
        "passes_per_s": round(whole_job_rate(world, 1.0, ms_step), 1),
        # tokens through every projection of the workload per second
        "token_passes_per_s": round(whole_job_rate(world, float(M), ms_step), 1),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "us_per_projection": round(ms_step * 1e3 / len(projs), 4),
        "quant_us_per_step": round(quant_ms_step * 1e3, 3),
        "gemv_us_per_step": round(gemv_avg * 1e3, 3),
        "quantiser": {"fused": "fused into the stack launch",
                      "batch": "one stack quantiser launch for all projections",
                      "prefill": "one stack quantiser launch for all projections"}.get(
                          mode, "separate launch per projection"),
        "launch_form": {"fused": "one quantising tq_gemv_stack launch",
                        "batch": "tq_quantize_act_stack_batch + tq_gemv_stack_batch",
                        "prefill": "tq_quantize_act_stack_batch + tq_gemm_prefill_stack"}
        .get(mode, "tq_quantize_act + tq_gemv / tq_gemm_prefill per projection"),
        "roofline": roof,
        "e2e": {
            "value": round(whole_job_rate(world, sb, e2e_ms / e2e_steps) / 1e9, 1),
            "unit": "GB/s",
            "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
            "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
            "ms_per_step": round(e2e_ms / e2e_steps, 5),
        },
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
        "impl": "ours",
    }
    if per_proj:
        out["per_projection"] = per_proj
    if prefill:
        out["tops"] = round(world * flops / (ms_step * 1e9), 1)
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(projs, args, budget_s=args.cpu_seconds)
    return out


def batch_kernel_name(M: int, mode: str) -> str:
    """The kernel the library runs for M tokens per projection (its default
    choice by M, or the one TQ_BATCH_KERNEL forces)."""
    forced = os.environ.get("TQ_BATCH_KERNEL", "")
    if M == 1:
        return "stream_gemv_kernel"
    if forced == "stream" and M <= 4 or forced == "" and M <= 2:
        return "stream_gemv_kernel"
    if forced == "mma" or forced == "" and M <= 24:
        return "mma_gemv_kernel"
    return "smallm_group_kernel" if mode == "batch" else "smallm_tc_kernel"


def prefill_kernel_name(M: int) -> str:
    """The prefill GEMM kernel the library runs for M tokens: CTA pairs from
    129 tokens unless TQ_PREFILL_PAIR=0, single CTAs otherwise."""
    if M > 128 and os.environ.get("TQ_PREFILL_PAIR", "") != "0":
        return "prefill_pair_kernel"
    return "prefill_tc_kernel"


def binary_kernel_name(M: int) -> str:
    """The binary g128 kernel the library runs for M tokens (the warp-MMA
    kernel for one token unless TQ_BINARY_KERNEL=dp4a forces the dp4a one)."""
    if M == 1 and os.environ.get("TQ_BINARY_KERNEL", "") != "dp4a":
        return "binary_mma_kernel"
    return "binary_gemv_kernel"


def gemv_launches(M: int) -> int:
    """Kernel launches of one tq_gemv / tq_gemm_prefill call at M tokens: one
    (the streaming kernel up to 4 tokens, the batched-decode tensor-core
    kernel up to 32, the prefill GEMM beyond)."""
    return 1


# ------------------------------------------------------------ CPU / oracle
def cpu_baseline(projs, args, budget_s: float = 10.0):
    """Time the oracle (one host thread) on whole passes over the workload's
    projections until budget_s has elapsed (at least one pass); report GB/s
    with the same algorithmic-byte count as the GPU arm. Prefill keeps the
    first 16 tokens of each projection so one pass stays within seconds."""
    import oracle

    sp = projs
    if projs[0].M > 24:
        import copy
        sp = []
        for p in projs:
            q = copy.copy(p)
            q.M, q.x_bf16 = 16, p.x_bf16[:16]
            sp.append(q)
    packed = [(oracle.pack(p.w), p) for p in sp]
    sb = workload_step_bytes(args.workload, sp)
    passes, t0 = 0, time.perf_counter()
    while True:
        for P, p in packed:
            oracle.forward(P, p.N, p.w_scale, p.x_bf16, threads=1)
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": round(sb * passes / el / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{passes} full pass(es) of the oracle over {len(sp)} projections of "
                      f"{args.workload} ({sb} algorithmic bytes per pass) in {el:.1f} s, "
                      f"one thread, on {os.cpu_count()} host cores",
            "passes_per_s": round(passes / el, 4)}


def run_reference(args, rank: int, world: int):
    """The oracle as the reference arm: rank 0 only, a bounded sample per step."""
    if rank != 0:
        return None
    import oracle

    shapes, M = WORKLOADS[args.workload]
    # One decoder layer's projections (or the whole workload if smaller) per step.
    sample = shapes[:7] if len(shapes) > 7 else shapes
    if M > 24:  # prefill: a 16-token slice per step keeps a step to seconds
        M = 16
    sp = list(make_projections(sample, M=M, seed=args.seed))
    packed = [(oracle.pack(p.w), p) for p in sp]
    sb = workload_step_bytes(args.workload, sp)

    def step():
        for P, p in packed:
            oracle.forward(P, p.N, p.w_scale, p.x_bf16, threads=1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    ms = el * 1e3 / args.steps
    value = sb / (ms * 1e6)
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 (oracle: int32 accumulate, fp64 epilogue)", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {DESCRIPTIONS.get(args.workload, '')}",
                   "sample_per_step": f"{len(sp)} projections, M={M}",
                   "parallelism": "host, one thread"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{len(sp)} projections (M={M}) of {args.workload} per step, "
                                   f"one thread, on {os.cpu_count()} host cores"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# --------------------------------------- Hadamard prefill, binary g128 decode
def run_next(args, rank: int, world: int):
    """prefill_had4_m512: the grouped Hadamard rotation + 4-bit quantiser
    launch and the grouped prefill GEMM on its codes; binary_ffn27b_m1: the
    stack quantiser and one binary g128 GEMV launch over the 24 projections.
    Same JSON line as the other workloads."""
    import torch

    import ternary_absmax_int8_b200 as tq

    shapes, M = NEXT_WORKLOADS[args.workload]
    if args.impl == "reference":
        return next_reference(args, shapes, M, rank, world)
    dev_i = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev_i)
    stream = torch.cuda.current_stream()
    had = args.workload == "prefill_had4_m512"
    if had:
        projs = list(make_projections(shapes, M=M, seed=args.seed))
        wbytes = sum(p.N * p.K // 4 for p in projs)
    else:
        projs = list(make_binary_projections(shapes, M=M, seed=args.seed))
        wbytes = sum(p.N * p.K // 8 + p.N * p.K // 64 for p in projs)
    copies = 1 if wbytes > 2 * L2_BYTES else -(-2 * L2_BYTES // wbytes)
    n = len(projs)
    x_host = torch.from_numpy(np.concatenate([p.x_bf16.view(np.int16).reshape(-1)
                                              for p in projs])).pin_memory()
    x_dev = x_host.cuda()
    kx = np.concatenate([[0], np.cumsum([p.M * p.K for p in projs])]).astype(np.int64)
    ny = np.concatenate([[0], np.cumsum([p.M * p.N for p in projs])]).astype(np.int64)
    xq = torch.empty(int(kx[-1]), dtype=torch.int8, device="cuda")
    xs = torch.empty(n * M, device="cuda")
    xsum = torch.empty(n * M, dtype=torch.int32, device="cuda")
    y_dev = torch.empty(int(ny[-1]), device="cuda")
    y_host = torch.empty(int(ny[-1])).pin_memory()
    # second activation / output buffers for the end-to-end pipeline
    xbufs = (x_dev, torch.empty_like(x_dev))
    ybufs = (y_dev, torch.empty_like(y_dev))
    yhosts = (y_host, torch.empty_like(y_host).pin_memory())
    if had:
        W = []
        for p in projs:
            P = np.empty((p.N // 4, p.K), np.uint8)
            tq.tq_pack_host(p.w, P, p.M, p.N, p.K)
            W.append([torch.from_numpy(P).cuda() for _ in range(copies)])

        htabs = [[tq.make_proj(x=xb.data_ptr() + 2 * int(kx[j]), xq=xq.data_ptr() + int(kx[j]),
                               x_scale=xs.data_ptr() + 4 * j * M,
                               x_sum=xsum.data_ptr() + 4 * j * M, K=p.K)
                  for j, p in enumerate(projs)] for xb in xbufs]

        def quant(c, s_, k=0):
            tq.tq_hadamard_quantize_act_stack(htabs[k], M, HADAMARD_BLOCK, stream=s_)

        ptabs = [[[tq.make_proj(packed=W[j][c], xq=xq.data_ptr() + int(kx[j]),
                                x_scale=xs.data_ptr() + 4 * j * M,
                                x_sum=xsum.data_ptr() + 4 * j * M,
                                y=yb.data_ptr() + 4 * int(ny[j]), w_scale=float(p.w_scale),
                                N=p.N, K=p.K) for j, p in enumerate(projs)] for c in range(copies)]
                 for yb in ybufs]

        def gemv(c, s_, k=0):
            tq.tq_gemm_prefill_stack(ptabs[k][c], M, stream=s_)

        sb = sum(quant_bytes(p.K, p.M) + algorithmic_bytes(p.N, p.K, p.M) for p in projs)
        gemv_units = sum(2.0 * p.M * p.N * p.K for p in projs)
        launches = -(-n // 512) + -(-n // 16)
        kernel = prefill_kernel_name(M)
    else:
        B = []
        for p in projs:
            bits = np.empty((p.N // 8, p.K), np.uint8)
            sp = np.empty((p.N // 8, p.K // 128, 8), np.uint16)
            tq.tq_pack_binary_host(p.w, p.s_f16, bits, sp, p.N, p.K)
            B.append([(torch.from_numpy(bits).cuda(), torch.from_numpy(sp.view(np.int16)).cuda())
                      for _ in range(copies)])
        qtabs = [[tq.make_proj(x=xb.data_ptr() + 2 * int(kx[j]), xq=xq.data_ptr() + int(kx[j]),
                               x_scale=xs.data_ptr() + 4 * j * M,
                               x_sum=xsum.data_ptr() + 4 * j * M, N=p.N, K=p.K)
                  for j, p in enumerate(projs)] for xb in xbufs]
        btabs = [[[tq.make_binary_proj(bits=B[j][c][0], scales_packed=B[j][c][1],
                                       xq=xq.data_ptr() + int(kx[j]),
                                       x_scale=xs.data_ptr() + 4 * j * M,
                                       y=yb.data_ptr() + 4 * int(ny[j]), N=p.N, K=p.K)
                   for j, p in enumerate(projs)] for c in range(copies)] for yb in ybufs]

        def quant(c, s_, k=0):
            tq.tq_quantize_act_stack_batch(qtabs[k], M, stream=s_)

        def gemv(c, s_, k=0):
            tq.tq_gemv_binary_stack(btabs[k][c], M, stream=s_)

        sb = sum(quant_bytes(p.K, p.M) + binary_bytes(p.N, p.K, p.M) for p in projs)
        gemv_units = float(sum(binary_bytes(p.N, p.K, p.M) for p in projs))
        launches = 2
        kernel = binary_kernel_name(M)

    def step(c, s_, k=0):
        quant(c, s_, k)
        gemv(c, s_, k)

    for i in range(args.warmup):
        step(i % copies, stream)
    torch.cuda.synchronize()
    K_ = args.steps
    S = copies * max(1, 8 // copies)
    n_chunks, rem = divmod(K_, S)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=cs):
            fn(cs)
        return g

    chunk = capture(lambda cs: [step(i % copies, cs) for i in range(S)])
    single = [capture(lambda cs, c=c: step(c, cs)) for c in range(copies)] if rem else []
    chunk.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev_i)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(n_chunks):
        chunk.replay()
    for i in range(rem):
        single[(n_chunks * S + i) % copies].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)

    def graph_ms(fn, reps=3):
        g = capture(fn)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    quant_ms = graph_ms(lambda cs: [quant(i % copies, cs) for i in range(S)]) / S
    gemv_ms = graph_ms(lambda cs: [gemv(i % copies, cs) for i in range(S)]) / S
    # end to end: uploads, library calls and downloads, double-buffered and
    # replayed from a CUDA graph of 16 steps (pipelined_e2e)
    chunk = 64
    e2e_steps = -(-max(K_, int(0.5e3 / max(total_ms / K_, 1e-3))) // chunk) * chunk
    e2e_ms = pipelined_e2e(
        e2e_steps, stream, chunk=chunk,
        h2d=lambda i, b: xbufs[b].copy_(x_host, non_blocking=True),
        compute=lambda i, b, s_: step(i % copies, s_, b),
        d2h=lambda i, b: yhosts[b].copy_(ybufs[b], non_blocking=True))
    assert torch.equal(yhosts[0], yhosts[1]), "end-to-end pipeline outputs differ"
    time.sleep(0.3)
    clk = clocks.stop()
    assert tq.tq_device_error(reset=True) == 0, "a kernel reported a device error"
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device="cuda")
    if rank != 0:
        return None
    ms_step = total_ms / K_
    value = whole_job_rate(world, sb, ms_step) / 1e9
    if had:
        tpeak, tkind = measured_tensor_peak()
        achieved = gemv_units / (gemv_ms * 1e9)
        roof = {"kernel": kernel, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": tpeak, "peak_kind": tkind, "unit": "TOPS (int8)",
                "frac": round(achieved / tpeak, 4), "traffic": None,
                "algorithmic_ops_per_step": gemv_units}
    else:
        peak, peak_kind = measured_peak()
        achieved = gemv_units / (gemv_ms * 1e6)
        roof = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs copy bandwidth)",
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "traffic": recorded_binary_traffic(args.workload, kernel),
                "algorithmic_bytes_per_launch": int(gemv_units)}
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K_, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("int8 codes -7..7 (bf16 in, fp64 rotation) x ternary -> int32, fp32 out"
                  if had else "int8 x binary (1 bit) -> int32 per group, fp64 group scaling, "
                              "fp32 out"),
        "data": ("synthetic (seeded ternary weights P=0.3/0.4/0.3, bf16 N(0,1) activations "
                 "with 1% x20 outliers)" if had else
                 "synthetic (seeded binary weights P=1/2, fp16 group scales U(0.012, 0.020), "
                 "bf16 N(0,1) activations with 1% x20 outliers)"),
        "config": {"workload": f"{args.workload}: {DESCRIPTIONS[args.workload]}",
                   "projections": n, "tokens_M": M, "weight_bytes": wbytes, "step_bytes": sb,
                   "weight_copies_rotated": copies,
                   "l2": ("inputs larger than L2 (weight stream > 126 MB), no flush"
                          if copies == 1 else f"{copies} rotated weight copies, "
                          f"{copies * wbytes / 2**20:.0f} MiB > L2"),
                   "parallelism": "single GPU" if world == 1 else f"replicas x{world}",
                   "seed": args.seed},
        "quant_us_per_step": round(quant_ms * 1e3, 3),
        "gemv_us_per_step": round(gemv_ms * 1e3, 3),
        "roofline": roof,
        "e2e": {"value": round(whole_job_rate(world, sb, e2e_ms / e2e_steps) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 4),
                "ms_per_step": round(e2e_ms / e2e_steps, 5)},
        "gpu_launches": launches * K_,
        "clocks": clk,
        "impl": "ours",
    }
    if had:
        out["tops"] = round(world * gemv_units / (ms_step * 1e9), 1)
    else:
        out["passes_per_s"] = round(whole_job_rate(world, 1.0, ms_step), 1)
    if world == 1 and not args.no_cpu_baseline:
        sample = dict(args.__dict__)
        sample["impl"], sample["steps"], sample["warmup"] = "reference", 1, 0
        ref = next_reference(argparse.Namespace(**sample), shapes, M, 0, 1)
        out["cpu_baseline"] = dict(ref["cpu_baseline"])
    return out


def next_reference(args, shapes, M, rank, world):
    """The oracle on a bounded sample per step: 16 tokens of each prefill shape
    (Hadamard route), or one layer's three binary projections."""
    if rank != 0:
        return None
    import oracle

    had = args.workload == "prefill_had4_m512"
    if had:
        sp = list(make_projections(shapes, M=16, seed=args.seed))
        packed = [oracle.pack(p.w) for p in sp]
        sb = sum(quant_bytes(p.K, p.M) + algorithmic_bytes(p.N, p.K, p.M) for p in sp)

        def one():
            for P, p in zip(packed, sp):
                oracle.forward_had4(P, p.N, p.w_scale, p.x_bf16, HADAMARD_BLOCK)
    else:
        sp = list(make_binary_projections(shapes[:3], M=M, seed=args.seed))
        packed = [oracle.pack_binary(p.w) for p in sp]
        sb = sum(quant_bytes(p.K, p.M) + binary_bytes(p.N, p.K, p.M) for p in sp)

        def one():
            for B, p in zip(packed, sp):
                oracle.forward_binary(B, p.N, p.s_f16, p.x_bf16)

    for _ in range(args.warmup):
        one()
    n = max(1, args.steps)
    t0 = time.perf_counter()
    for _ in range(n):
        one()
    el = time.perf_counter() - t0
    value = sb * n / el / 1e9
    sample = (f"{len(sp)} projections, {sp[0].M} tokens each, of {args.workload} per step, one "
              f"thread, on {os.cpu_count()} host cores")
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / n * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "oracle (int32 accumulate, fp64 scaling)", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {DESCRIPTIONS[args.workload]}",
                   "parallelism": "host, one thread"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------ decoder-layer chains
CHAIN_WORKLOADS = {
    "ffn_block30_m1": "30 x BitNet-b1.58-2B-4T FFN block, M=1, real dependencies, two launches "
                      "per layer: [input RMSNorm + quantiser + gate and up GEMVs] -> "
                      "[relu^2(gate)*up + ffn_sub_norm + quantiser + down GEMV, weights "
                      "streamed while the first drains]; 90 projections, 398 MB packed",
    "absmean_pack_27b": "absmean ternary quantisation + packing of bf16 latent weights "
                        "17408x5120 (N(0, 0.02)), two passes",
}
FFN_H, FFN_I, FFN_LAYERS, RMS_EPS = 2560, 6912, 30, 1e-5


def ffn_block_bytes(M: int) -> int:
    """Algorithmic bytes of one FFN block: rms+quant (x bf16, gain, codes,
    scale+sum), gate and up GEMVs, relu^2*up + sub-norm + quant (two fp32
    rows, gain, codes, scale+sum), down GEMV."""
    H, I = FFN_H, FFN_I
    rms = M * H * 2 + H * 4 + M * H + M * 8
    relu = 2 * M * I * 4 + I * 4 + M * I + M * 8
    return rms + 2 * algorithmic_bytes(I, H, M) + relu + algorithmic_bytes(H, I, M)


def absmean_bytes(N: int, K: int) -> int:
    """Two reads of the bf16 weights (the sum must be complete before any
    weight is quantised and 178 MB does not stay on chip), the packed bytes
    and the scale."""
    return 2 * 2 * N * K + N * K // 4 + 4


def run_chain(args, rank: int, world: int):
    """The decoder-layer chain or the absmean packer: same JSON line as the
    stack; CUDA-graph replays, e2e through the library calls with host
    buffers, the oracle on a bounded sample as the CPU baseline."""
    import torch

    import ternary_absmax_int8_b200 as tq

    dev_i = int(os.environ.get("LOCAL_RANK", "0"))
    rng = np.random.default_rng(args.seed)
    if args.impl == "reference" and rank != 0:
        return None
    if args.impl == "ours":
        torch.cuda.set_device(dev_i)
    stream = torch.cuda.current_stream() if args.impl == "ours" else None
    if args.workload == "ffn_block30_m1":
        M, H, I, L = 1, FFN_H, FFN_I, FFN_LAYERS
        shapes = [(f"L{l}.{n}", a, b) for l in range(L)
                  for (n, a, b) in (("gate_proj", I, H), ("up_proj", I, H), ("down_proj", H, I))]
        projs = list(make_projections(shapes, M=M, seed=args.seed))
        g_in = rng.uniform(0.5, 1.5, (L, H)).astype(np.float32)
        g_ffn = rng.uniform(0.5, 1.5, (L, I)).astype(np.float32)
        sb = L * ffn_block_bytes(M)
        if args.impl == "reference":
            return chain_reference(args, projs, g_in, g_ffn, sb, world)
        packed = []
        for p in projs:
            P = np.empty((p.N // 4, p.K), np.uint8)
            tq.tq_pack_host(p.w, P, M, p.N, p.K)
            packed.append(torch.from_numpy(P).cuda())
        x_host = torch.from_numpy(np.stack([projs[3 * l].x_bf16.view(np.int16)
                                            for l in range(L)])).pin_memory()
        x_dev = x_host.cuda()
        gi, gf = torch.from_numpy(g_in).cuda(), torch.from_numpy(g_ffn).cuda()
        xq = torch.empty((L, M, H), dtype=torch.int8, device="cuda")
        xs = torch.empty((L, M), device="cuda")
        xsum = torch.empty((L, M), dtype=torch.int32, device="cuda")
        yg = torch.empty((L, M, I), device="cuda")
        yu = torch.empty((L, M, I), device="cuda")
        xq2 = torch.empty((L, M, I), dtype=torch.int8, device="cuda")
        xs2 = torch.empty((L, M), device="cuda")
        xsum2 = torch.empty((L, M), dtype=torch.int32, device="cuda")
        yd = torch.empty((L, M, H), device="cuda")
        y_host = torch.empty_like(yd, device="cpu").pin_memory()
        tabs = [[tq.make_proj(packed=packed[3 * l + j], xq=xq[l], x_scale=xs[l], x_sum=xsum[l],
                              y=(yg if j == 0 else yu)[l], w_scale=projs[3 * l + j].w_scale,
                              N=I, K=H) for j in (0, 1)] for l in range(L)]
        xq_b = torch.empty((L, M, H), dtype=torch.int8, device="cuda")
        xs_b = torch.empty((L, M), device="cuda")
        xsum_b = torch.empty((L, M), dtype=torch.int32, device="cuda")
        # gate + up: one launch that normalises (gain g_in) and quantises the
        # shared input itself; down: one launch that computes relu^2(gate) *
        # up, normalises (g_ffn) and quantises, streaming its weights while
        # the first launch drains.
        tabs = [[tq.make_proj(packed=packed[3 * l], x=x_dev[l], xq=xq[l], x_scale=xs[l],
                              x_sum=xsum[l], y=yg[l], w_scale=projs[3 * l].w_scale, N=I, K=H,
                              gain=gi[l], eps=RMS_EPS),
                 tq.make_proj(packed=packed[3 * l + 1], x=x_dev[l], xq=xq_b[l], x_scale=xs_b[l],
                              x_sum=xsum_b[l], y=yu[l], w_scale=projs[3 * l + 1].w_scale, N=I,
                              K=H, gain=gi[l], eps=RMS_EPS)] for l in range(L)]
        dtabs = [[tq.make_proj(packed=packed[3 * l + 2], x_f32=yg[l], up=yu[l], xq=xq2[l],
                               x_scale=xs2[l], x_sum=xsum2[l], y=yd[l],
                               w_scale=projs[3 * l + 2].w_scale, N=H, K=I, gain=gf[l],
                               eps=RMS_EPS)] for l in range(L)]
        ov = tq.TQ_STACK_OVERLAP_PREV

        def step(s_):
            for l in range(L):
                tq.tq_gemv_stack(tabs[l], flags=tq.TQ_STACK_RMSNORM, stream=s_)
                tq.tq_gemv_stack(dtabs[l], flags=tq.TQ_STACK_RELU2_MUL | ov, stream=s_)

        launches, kernel = 2 * L, "stream_gemv_kernel (normalising + quantising prologue)"
        bytes_in = int(x_host.numel() * x_host.element_size())
        bytes_out = int(y_host.numel() * y_host.element_size())
        config = {"layers": L, "projections": 3 * L, "tokens_M": M,
                  "packed_weight_bytes": sum(p.N * p.K // 4 for p in projs), "rms_eps": RMS_EPS,
                  "l2": "inputs larger than L2 (weight stream 398 MB), no flush"}
    else:
        N, K = 17408, 5120
        W = (rng.standard_normal((N, K), dtype=np.float32) * 0.02)
        Wb = torch.from_numpy(W).to(torch.bfloat16)
        sb = absmean_bytes(N, K)
        if args.impl == "reference":
            return absmean_reference(args, Wb.view(torch.int16).numpy().view(np.uint16), sb)
        x_host = Wb.view(torch.int16).pin_memory()
        x_dev = x_host.cuda()
        packed_dev = torch.empty((N // 4, K), dtype=torch.uint8, device="cuda")
        ws = torch.empty(1, device="cuda")
        y_host = torch.empty((N // 4, K), dtype=torch.uint8).pin_memory()
        yd = packed_dev

        def step(s_):
            tq.tq_absmean_pack(x_dev, packed_dev, ws, N, K, stream=s_)

        launches, kernel = 2, "absmean_sum_kernel + absmean_pack_kernel"
        bytes_in = int(x_host.numel() * 2)
        bytes_out = int(y_host.numel())
        config = {"N": N, "K": K, "weight_bytes_bf16": 2 * N * K,
                  "l2": "weights (178 MB) larger than L2; the second pass re-reads them, part "
                        "from L2"}

    for _ in range(args.warmup):
        step(stream)
    torch.cuda.synchronize()
    K_ = args.steps
    S = 4 if args.workload == "ffn_block30_m1" else 8
    n_chunks, rem = divmod(K_, S)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=cs):
            fn(cs)
        return g

    chunk = capture(lambda cs: [step(cs) for _ in range(S)])
    single = capture(step) if rem else None
    chunk.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev_i)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(n_chunks):
        chunk.replay()
    for _ in range(rem):
        single.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    e2e_steps = max(K_, int(0.5e3 / max(total_ms / K_, 1e-3)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        step(stream)
        y_host.copy_(yd, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    time.sleep(0.3)
    clk = clocks.stop()
    assert tq.tq_device_error(reset=True) == 0, "a kernel reported a device error"
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device="cuda")
    if rank != 0:
        return None
    ms_step = total_ms / K_
    value = whole_job_rate(world, sb, ms_step) / 1e9
    peak, peak_kind = measured_peak()
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K_, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 codes / ternary (bf16 and fp32 rows in, fp64 norm statistics)",
        "data": "synthetic (seeded ternary weights P=0.3/0.4/0.3, bf16 N(0,1) activations "
                "with 1% x20 outliers; gains U(0.5,1.5); latent weights N(0,0.02))",
        "config": {"workload": f"{args.workload}: {CHAIN_WORKLOADS[args.workload]}",
                   "step_bytes": sb, "parallelism": "single GPU" if world == 1 else
                   f"replicas x{world}", "seed": args.seed, **config},
        "roofline": {"kernel": kernel, "bound": "hbm", "achieved": round(value / world, 1),
                     "peak": peak, "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs copy "
                                                f"bandwidth)", "unit": "GB/s",
                     "frac": round(value / world / peak, 4), "traffic": None,
                     "algorithmic_bytes_per_step": sb},
        "e2e": {"value": round(whole_job_rate(world, sb, e2e_ms / e2e_steps) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": bytes_in, "d2h_bytes_per_step": bytes_out,
                "ms_per_step": round(e2e_ms / e2e_steps, 5)},
        "gpu_launches": launches * K_,
        "clocks": clk,
        "impl": "ours",
    }
    if world == 1 and not args.no_cpu_baseline:
        sample = dict(args.__dict__)
        sample["impl"] = "reference"
        sample["steps"], sample["warmup"] = 1, 0
        ref = run_chain(argparse.Namespace(**sample), 0, 1)
        out["cpu_baseline"] = dict(ref["cpu_baseline"])
    return out


def chain_reference(args, projs, g_in, g_ffn, sb, world):
    """The oracle on one FFN block per step (a bounded sample), the same chain
    as the GPU step."""
    import oracle

    H, I = FFN_H, FFN_I
    gate, up, down = projs[0], projs[1], projs[2]
    P = [oracle.pack(p.w) for p in (gate, up, down)]
    xb = gate.x_bf16
    f32 = (xb.astype(np.uint32) << 16).view(np.float32)

    def one():
        q, s, t = oracle.quant_f32(oracle.rmsnorm(f32, g_in[0], RMS_EPS))
        yg = oracle.epilogue(oracle.gemv(P[0], I, q), gate.w_scale, s).astype(np.float32)
        yu = oracle.epilogue(oracle.gemv(P[1], I, q), up.w_scale, s).astype(np.float32)
        q2, s2, t2 = oracle.quant_f32(oracle.rmsnorm(oracle.relu2_mul(yg, yu), g_ffn[0],
                                                     RMS_EPS))
        oracle.epilogue(oracle.gemv(P[2], H, q2), down.w_scale, s2)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    n = max(1, args.steps)
    for _ in range(n):
        one()
    el = time.perf_counter() - t0
    per_block = sb // FFN_LAYERS
    value = per_block * n / el / 1e9
    return _ref_line(args, world, value, el / n * 1e3,
                     f"one FFN block (layer 0) of {args.workload} per step, one thread, on "
                     f"{os.cpu_count()} host cores")


def absmean_reference(args, Wb, sb):
    """The oracle absmean + pack on a 1/16 row slice per step (bounded)."""
    import oracle

    rows = Wb.shape[0] // 16
    sub = np.ascontiguousarray(Wb[:rows])
    for _ in range(args.warmup):
        oracle.pack(oracle.absmean(sub)[0])
    t0 = time.perf_counter()
    n = max(1, args.steps)
    for _ in range(n):
        oracle.pack(oracle.absmean(sub)[0])
    el = time.perf_counter() - t0
    value = (sb / 16) * n / el / 1e9
    return _ref_line(args, 1, value, el / n * 1e3,
                     f"rows 0..{rows - 1} of the 17408x5120 weights per step, one thread, on "
                     f"{os.cpu_count()} host cores")


def _ref_line(args, world, value, ms, sample):
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "oracle (int32 accumulate, fp64 statistics)", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {CHAIN_WORKLOADS[args.workload]}",
                   "parallelism": "host, one thread"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# Workloads measured after the headline in the default run, in the same
# process, each with its own clock record: the single projection, one decoder
# layer, the batched-decode FFN sweep, prefill, the small-batch stacks and the
# two further paths.
EXTRA_CONFIGS = (["single_640x2560_m1", "layer_m1"] + [f"ffn_m{m}" for m in (1, 2, 4, 8, 16, 24)]
                 + ["prefill_m512", "stack30_m4", "stack30_m16", "prefill_had4_m512",
                    "binary_ffn27b_m1"])


def summarise(line):
    """The figures of one workload's JSON line kept under "configs"."""
    r = line["roofline"]
    out = {"us_per_step": round(line["ms_per_step"] * 1e3, 3), "GB_s": line["value"],
           "roofline_kernel": r["kernel"], "roofline_achieved": r["achieved"],
           "roofline_unit": r["unit"], "frac": r["frac"], "steps": line["steps"],
           "sm_mhz": line["clocks"].get("sm_mhz"), "reasons": line["clocks"].get("reasons")}
    for k in ("tops", "token_passes_per_s", "passes_per_s"):
        if k in line:
            out[k] = line[k]
    if "per_projection" in line:
        out["per_projection"] = line["per_projection"]
    return out


def run_extra_configs(args):
    res = {}
    for w in EXTRA_CONFIGS:
        heavy = w.startswith("prefill") or w.startswith("stack30") or w.startswith("binary")
        a = argparse.Namespace(**dict(args.__dict__, workload=w, steps=50 if heavy else 200,
                                      warmup=3, no_cpu_baseline=True))
        if w in NEXT_WORKLOADS:
            line = run_next(a, 0, 1)
        else:
            line = run_ours(a, 0, 1)
        res[w] = summarise(line)
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(CHAIN_WORKLOADS) +
                    sorted(NEXT_WORKLOADS), default="stack30_m1")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads measured after the default one")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.workload in CHAIN_WORKLOADS:
            out = run_chain(args, rank, world)
        elif args.workload in NEXT_WORKLOADS:
            out = run_next(args, rank, world)
        elif args.impl == "ours":
            out = run_ours(args, rank, world)
        else:
            out = run_reference(args, rank, world)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()
    if (out is not None and world == 1 and args.impl == "ours" and not args.no_configs
            and args.workload == "stack30_m1"):
        out["configs"] = run_extra_configs(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
