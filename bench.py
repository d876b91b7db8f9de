#!/usr/bin/env python
"""Throughput of the butterfly transform + quantize path on B200.

Default workload (N=1 line): the LLaMA-2-7B activation shape, n = 4096,
2048 rows of bf16 input, fused Q x + INT4 asymmetric RTN in groups of 128
(packed 2 codes/byte, fp16 scale/zero).  One step = one bq_transform_quantize
call over the batch, inputs resident in HBM; the per-layer angle table is
prepared once before timing (the angles are fixed at inference).  The input
(16.8 MB) is smaller than L2, so the timed steps cycle over enough copies of
the batch (and of its outputs) that together exceed twice the L2: every step
reads an input that is not in L2.  The K timed steps are one CUDA graph of K
launches replayed between two CUDA events.

Multi-GPU (torchrun, one process per GPU): rows are independent, so every
rank processes its own batch of the same shape (weak scaling, no collective
on the data path); the step time is the max over ranks.

--impl reference times the float64 CPU oracle (tests' ground truth) on a
bounded sample of the same workload on the host cores.
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

FP32_PEAK_DERIVED = 148 * 128 * 2 * 1.965e9   # SMs x FP32 lanes x 2 flop x max SM clock
L2_FLUSH_BYTES = 1 << 30   # also gives the host time to enqueue the step before the GPU reaches it
L2_BYTES = 126 * 1000 * 1000


# ----------------------------------------------------------------------------- workloads

def workload_spec(name: str):
    from rotation_bit_quantization_b200 import workloads as wl
    if name == "act4096":
        return dict(make=lambda rank: wl.act_4096(2048, seed_offset=rank), kind="quant", rows=2048, n=4096,
                    bits=4, group=128, label="act n=4096 rows=2048 bf16 -> Qx + INT4 RTN g128 (LLaMA-2-7B activation shape)")
    if name == "fwd4096":
        return dict(make=lambda rank: wl.act_4096(2048, seed_offset=rank), kind="fwd", rows=2048, n=4096,
                    bits=4, group=128, label="act n=4096 rows=2048 bf16 -> Qx float32 (forward only)")
    if name == "inv4096":
        return dict(make=lambda rank: wl.act_4096(2048, seed_offset=rank), kind="inv", rows=2048, n=4096,
                    bits=4, group=128, label="act n=4096 rows=2048 bf16 -> Q^T y bf16 (inverse)")
    if name == "inv5120":
        return dict(make=lambda rank: wl.act_5120(8192), kind="inv", rows=8192, n=5120, bits=4, group=128,
                    label="act n=5120 = B_1024 (x) O_5, rows=8192 bf16 -> Q^T y bf16 (inverse)")
    if name == "weight4096":
        return dict(make=lambda rank: wl.weight_4096(11008), kind="quant", rows=11008, n=4096, bits=2, group=128,
                    label="weight n=4096 rows=11008 bf16 -> W Q^T + INT2 RTN g128 (W2A16)")
    if name == "bwd":
        return dict(make=None, kind="bwd", rows=65536, n=4096, bits=0, group=0, layers=32,
                    label="calibration backward: 32 layers x 65536 tokens x n=4096, X bf16, dY fp32 -> Y bf16, dX fp32, dtheta (one launch)")
    if name == "uniformity":
        return dict(make=None, kind="uniformity", rows=65536, n=4096, bits=4, group=128, layers=1,
                    label="uniformity regulariser: 65536 tokens x n=4096 float32 rotated activations -> "
                          "per-group KL to uniform over the INT4 g128 levels + dL/dY (one calibration batch of one layer)")
    if name == "w2a16":
        return dict(make=None, kind="gemm", rows=2048, n=4096, bits=2, group=128, out_features=11008,
                    label="W2A16 linear: rotated activations 2048 x 4096 bf16 times INT2 g128 weights 11008 x 4096 "
                          "-> 2048 x 11008 bf16 (LLaMA-2-7B MLP up-projection shape)")
    if name == "wush4096":
        return dict(make=None, kind="block", rows=2048, n=4096, bits=4, group=32, fmt="mxfp4",
                    label="block transform + MXFP4: 2048 x 4096 bf16 activations, 128 per-block 32 x 32 transforms "
                          "(tcgen05), E2M1 codes with E8M0 scales per 32 (WUSH workload shape)")
    if name == "act5120":
        return dict(make=lambda rank: wl.act_5120(8192), kind="quant", rows=8192, n=5120, bits=4, group=128,
                    label="act n=5120 = B_1024 (x) O_5, rows=8192 bf16 -> INT4 RTN g128 (LLaMA-2-13B shape)")
    raise SystemExit(f"unknown workload {name}")


def flops_per_row(m: int, r: int) -> float:
    """Algorithmic flops of one row: 6 per rotation (4 mul + 2 add), (m/2) log2 m rotations per sub-row,
    plus 2 r^2 per contiguous group for a dense Kronecker factor."""
    L = m.bit_length() - 1
    f = 6.0 * (m // 2) * L * r
    if r > 1:
        f += 2.0 * r * r * m
    return f


def bytes_per_row(n: int, in_bytes: int, bits: int, group: int) -> float:
    """Algorithmic HBM bytes of one row: input + packed codes + fp16 scale and zero per group."""
    return n * in_bytes + n * bits / 8 + 4 * (n // group)


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def kernel_source_hash(files) -> str:
    """Hash of the CUDA sources a profiled kernel is built from (paths relative to csrc/)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rotation_bit_quantization_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode()); h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if it was
    captured on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        rec = json.load(f).get(workload)
    if not rec or rec.get("source_hash") != kernel_source_hash(rec.get("sources", [])):
        return None, None
    return rec.get("dram_bytes_per_launch"), rec.get("kernel")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.raw = ""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-i", gpu_id,
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, err = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, err = self.proc.communicate()
        self.raw = (out or "")[-2000:] + (err or "")[-500:]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1])); mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"error": "no nvidia-smi samples", "raw": self.raw[-300:]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "window": "from 0.5 s of continuous steps before the timed region to its end"}


def gpu_id_for(device) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(device.index if hasattr(device, "index") else 0)


class GpuLocalCpus:
    """Context manager: while it is open the process runs on the CPUs NVML reports as
    local to the GPU, so that pinned host buffers allocated inside it sit on the GPU's
    NUMA node (host-device copies then do not cross the inter-socket link).  The
    previous affinity is restored on exit; without NVML it changes nothing.  `cpus` is
    the number of CPUs used (None when unchanged)."""

    def __init__(self, device):
        self.device = device
        self.saved = None
        self.cpus = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(gpu_id_for(self.device))
                words = pynvml.nvmlDeviceGetCpuAffinity(h, 64)
            finally:
                pynvml.nvmlShutdown()
            local = {64 * i + b for i, wd in enumerate(words) for b in range(64) if (int(wd) >> b) & 1}
            self.saved = os.sched_getaffinity(0)
            use = local & self.saved
            if use and use != self.saved:
                os.sched_setaffinity(0, use)
                self.cpus = len(use)
            else:
                self.saved = None
        except Exception:
            self.saved = None
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False


def cpu_oracle_rate(w, rows_target_s: float, max_rows: int, inverse: bool = False):
    """Rows/s of the float64 oracle (transform + float32-step quantizer, or the inverse
    transform alone) on the host cores."""
    from concurrent.futures import ThreadPoolExecutor

    from oracle import butterfly as ob
    from oracle import quant as oq
    from rotation_bit_quantization_b200 import workloads as wl

    cores = len(os.sched_getaffinity(0))
    src = w.x if w.x is not None else w.w
    dt = w.x_dtype if w.x is not None else w.w_dtype
    chunk = 32

    def one(lo):
        xs = src[lo:lo + chunk]
        xf = (wl.f32_from_bf16_bits(xs) if dt == "bf16" else xs).astype(np.float64)
        if inverse:
            ob.inverse(w.theta, xf) if w.r == 1 else ob.kron_inverse(w.theta, w.O, xf, w.m)
            return xs.shape[0]
        y = ob.forward(w.theta, xf) if w.r == 1 else ob.kron_forward(w.theta, w.O, xf, w.m)
        oq.quantize_pack(y.astype(np.float32), w.bits, w.group)
        return xs.shape[0]

    # calibrate on one chunk, then run a bounded sample on all cores
    t0 = time.perf_counter(); one(0); t1 = time.perf_counter()
    per_chunk = t1 - t0
    nchunks = max(cores, int(rows_target_s * cores / max(per_chunk, 1e-6)))
    nchunks = min(nchunks, max_rows // chunk)
    starts = [(k * chunk) % (src.shape[0] - chunk + 1) for k in range(nchunks)]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=cores) as ex:
        done = sum(ex.map(one, starts))
    el = time.perf_counter() - t0
    return done / el, cores, f"{done} rows of the workload ({nchunks} chunks of {chunk}), {el:.1f} s on {cores} threads"


def cpu_dense_rate(w, rows_sample: int):
    """Rows/s of the materialised-Q path on the host: Q built once (the stage-wise float64
    oracle applied to the identity, not timed), then y = X Q^T as one float64 matmul and the
    float32-step quantizer, on a sample of rows."""
    from oracle import butterfly as ob
    from oracle import quant as oq
    from rotation_bit_quantization_b200 import workloads as wl

    src = w.x if w.x is not None else w.w
    dt = w.x_dtype if w.x is not None else w.w_dtype
    n = w.m * w.r
    eye = np.eye(n)
    qt = ob.forward(w.theta, eye) if w.r == 1 else ob.kron_forward(w.theta, w.O, eye, w.m)   # row j = Q e_j
    xs = src[:rows_sample]
    xf = (wl.f32_from_bf16_bits(xs) if dt == "bf16" else xs).astype(np.float64)
    t0 = time.perf_counter()
    y = xf @ qt
    oq.quantize_pack(y.astype(np.float32), w.bits, w.group)
    el = time.perf_counter() - t0
    return xs.shape[0] / el, len(os.sched_getaffinity(0)), (
        f"{xs.shape[0]} rows, dense {n} x {n} float64 Q (built once, not timed) times the rows on the host's "
        f"BLAS threads plus the quantizer, {el:.2f} s")


def cpu_bwd_rate(layer: int, tokens_sample: int, m: int = 4096):
    """Tokens/s of the float64 oracle backward (Y, dX, dtheta) on a sample of one layer's tokens."""
    from oracle import butterfly as ob
    from rotation_bit_quantization_b200 import workloads as wl

    w = wl.backward_layer_host(layer, tokens_sample, m)
    x = wl.f32_from_bf16_bits(w.x).astype(np.float64)
    t0 = time.perf_counter()
    ob.backward(w.theta, x, w.dy.astype(np.float64))
    el = time.perf_counter() - t0
    return tokens_sample / el, (f"{tokens_sample} tokens of layer {layer} (stage-wise float64 numpy), {el:.1f} s; "
                                f"the per-token rate applies to all 32 layers (an extrapolation)")


# ----------------------------------------------------------------------------- our arm

E2E_CHUNKS = 4


def pipelined_e2e(torch, dev, stream, x_pin, outs_pin, make_dev, call, steps, warmup, nchunk=E2E_CHUNKS):
    """(milliseconds per step, method) of `steps` end-to-end steps through the public API with
    host buffers: every step copies its whole input from pinned host memory, runs `call` and
    copies every output back, all inside the timed region.  The batch goes in `nchunk` row
    chunks and three streams: the copy-in of chunk c, the call on it and the copy-out of its
    results are ordered by events, so the two PCIe directions and the kernels overlap,
    within a step and across steps; two device buffer sets alternate by step, each chunk's
    reuse waiting for the call and the copy-out that last used it.  The timed steps are
    captured in one CUDA graph (copies, calls and their cross-stream dependencies), so that
    host-side launch work stays out of the time; if the capture fails, they run eagerly.

    make_dev() -> (x_dev, [out_dev, ...]) with rows in dimension 0; outs_pin the matching
    pinned host outputs; call(x_chunk, [out_chunk, ...]) runs the library on the current
    stream."""
    rows = x_pin.shape[0]
    bounds = [(rows * c // nchunk, rows * (c + 1) // nchunk) for c in range(nchunk)]
    bounds = [b for b in bounds if b[1] > b[0]]
    sets = [make_dev() for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = {k: [[torch.cuda.Event() for _ in bounds] for _ in range(2)] for k in ("in", "cmp", "out")}

    def one(step, fresh):
        # fresh: the buffer set has no earlier use in this sequence (nothing to wait for)
        k = step % 2
        xd, od = sets[k]
        for c, (r0, r1) in enumerate(bounds):
            with torch.cuda.stream(s_in):
                if not fresh:
                    s_in.wait_event(ev["cmp"][k][c])   # the call two steps back has read this chunk
                xd[r0:r1].copy_(x_pin[r0:r1], non_blocking=True)
                ev["in"][k][c].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev["in"][k][c])
                if not fresh:
                    s_cmp.wait_event(ev["out"][k][c])  # the copy-out two steps back has read its outputs
                call(xd[r0:r1], [o[r0:r1] for o in od])
                ev["cmp"][k][c].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["cmp"][k][c])
                for o, h in zip(od, outs_pin):
                    h[r0:r1].copy_(o[r0:r1], non_blocking=True)
                ev["out"][k][c].record(s_out)

    def run(n):
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_stream(torch.cuda.current_stream())
        for i in range(n):
            one(i, i < 2)
        for s_ in (s_in, s_cmp, s_out):
            torch.cuda.current_stream().wait_stream(s_)

    run(max(warmup, 2))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            run(steps)
        torch.cuda.synchronize()
        method = "one CUDA graph of the timed steps (copies, calls, cross-stream dependencies)"
    except RuntimeError as exc:  # capture refused: time the same steps eagerly
        graph = None
        torch.cuda.synchronize()
        method = f"eager (graph capture failed: {str(exc).splitlines()[0][:80]})"
    e0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) / steps, method


def run_ours(args, spec, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build as bq_build

    bq_build.build()
    bq.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = spec["make"](rank)
    rows, n, bits, group = spec["rows"], spec["n"], spec["bits"], spec["group"]
    src = w.x if w.x is not None else w.w
    src_dtype = w.x_dtype if w.x is not None else w.w_dtype
    assert src_dtype == "bf16"
    x_host = torch.from_numpy(src.view(np.int16)).view(torch.bfloat16)
    x = x_host.to(dev)
    theta = torch.from_numpy(w.theta).to(dev)
    O = None if w.O is None else torch.from_numpy(w.O).to(dev)
    layer = bq.Layer(theta, O)
    fwd = spec["kind"] == "fwd"
    inv = spec["kind"] == "inv"
    out_row_bytes = n * 4 if fwd else (n * 2 if inv else bytes_per_row(n, 0, bits, group))
    # Every timed step reads an input set that is not in L2: NS copies of the batch
    # (and NS output sets), cycled, with NS sets together more than twice the L2.
    set_bytes = rows * (n * 2 + out_row_bytes)
    NS = max(2, int(np.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x] + [x.clone() for _ in range(NS - 1)]
    if fwd or inv:
        outs = [torch.empty((rows, n), dtype=torch.float32 if fwd else torch.bfloat16, device=dev)
                for _ in range(NS)]
    else:
        outs = [bq.quant_outputs(rows, n, bits, group, dev) for _ in range(NS)]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        if fwd:
            bq.bq_butterfly_fwd(layer, xs[i % NS], outs[i % NS])
        elif inv:
            bq.bq_butterfly_inv(layer, xs[i % NS], outs[i % NS])
        else:
            bq.bq_transform_quantize(layer, xs[i % NS], bits, group, *outs[i % NS])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # The K timed steps are one CUDA graph of K launches (step i on set i mod NS),
    # replayed once between the two events: one launch per step, no host work or
    # flush between steps.
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            for i in range(args.steps):
                step(i)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    # the clock sampler needs more time than the timed region takes: keep the GPU
    # busy with the same graph for 0.5 s while it starts
    sampler = ClockSampler(gpu_id_for(dev))
    t_busy = time.perf_counter()
    while time.perf_counter() - t_busy < 0.5:
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    total_ms = float(e0.elapsed_time(e1))
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_total_ms = float(t.item())
    ms_per_step = max_total_ms / args.steps
    value = rows * world / (ms_per_step * 1e-3)
    del graph

    # Secondary: the latency of one launch on its own (L2 flushed by a 1 GiB write, the
    # launch alone between two events), which carries the launch and event overhead
    step_ms = []
    for i in range(max(args.warmup, 5)):
        flush.zero_()
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_.record(stream)
        step(0)
        e_.record(stream)
        torch.cuda.synchronize()
        step_ms.append(s_.elapsed_time(e_))
    del flush

    # end to end through the public API with host buffers: H2D input, kernel, D2H codes/scale/zero
    e2e = None
    if not args.no_e2e:
        with GpuLocalCpus(dev) as host_cpus:  # pinned buffers on the GPU's NUMA node
            x_pin = x_host.pin_memory()
            if fwd or inv:
                outs_pin = [torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory()]

                def make_dev():
                    return torch.empty_like(x), [torch.empty_like(outs[0])]

                def call(xc, oc):
                    (bq.bq_butterfly_fwd if fwd else bq.bq_butterfly_inv)(layer, xc, oc[0])
            else:
                outs_pin = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs[0]]

                def make_dev():
                    return torch.empty_like(x), list(bq.quant_outputs(rows, n, bits, group, dev))

                def call(xc, oc):
                    bq.bq_transform_quantize(layer, xc, bits, group, *oc)

            if world > 1:
                dist.barrier()
            e2e_ms, e2e_method = pipelined_e2e(torch, dev, stream, x_pin, outs_pin, make_dev, call, args.steps,
                                               args.warmup)
            te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            e2e_ms = float(te.item())
            e2e = {"value": rows * world / (e2e_ms * 1e-3), "unit": "rows/s", "host_cpus": host_cpus.cpus,
                   "h2d_bytes_per_step": int(x_pin.numel() * x_pin.element_size()),
                   "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outs_pin)),
                   "ms_per_step": e2e_ms,
                   "pipeline": f"{E2E_CHUNKS} row chunks per step on three streams (copy-in, the library call, "
                               f"copy-out), two device buffer sets alternating by step; timed as {e2e_method}"}

    peaks, peak_src = load_peaks()
    fl_launch = flops_per_row(w.m, w.r) * rows
    by_launch = (n * 2 + out_row_bytes) * rows
    avg_launch_s = (total_ms / args.steps) * 1e-3
    achieved_tf = fl_launch / avg_launch_s / 1e12
    traffic, traffic_kernel = recorded_traffic(args.workload) if not (args.rows or args.layers) else (None, None)
    result = {
        "metric": "butterfly fwd+quant rows/s and GB/s at n=4096 on 1 B200; % of FP32/HBM roofline",
        "value": value,
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; bf16 input, Student-t nu=3 with outlier channels)",
        "config": {"workload": spec["label"], "rows_per_gpu": rows, "n": n, "bits": bits, "group": group,
                   "global_batch": rows * world, "parallelism": f"rows sharded, dp{world}",
                   "l2": (f"inputs larger than L2: step i reads input set i mod {NS}, {NS} sets of "
                          f"{set_bytes / 1e6:.1f} MB (input + outputs) cycled, {NS * set_bytes / 1e6:.0f} MB in "
                          f"total > 2 x the 126 MB L2; no flush"),
                   "timing": (f"the {args.steps} timed steps are one CUDA graph of {args.steps} launches replayed "
                              f"once between two CUDA events on the launching stream"),
                   "angle_table": "prepared once per layer before timing"},
        "gbs": by_launch * world / (ms_per_step * 1e-3) / 1e9,
        "roofline": {
            "bound": "alu",
            "achieved": achieved_tf,
            "peak": FP32_PEAK_DERIVED / 1e12,
            "unit": "TFLOP/s",
            "frac": achieved_tf / (FP32_PEAK_DERIVED / 1e12),
            "traffic": traffic,
            "peak_note": "FP32 FMA peak derived: 148 SMs x 128 lanes x 2 flop x 1.965 GHz",
            "algorithmic_flops_per_launch": fl_launch,
            "algorithmic_bytes_per_launch": by_launch,
            "hbm_frac": (by_launch / avg_launch_s / 1e9) / peaks["hbm_gbs"],
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "hbm_peak_source": peak_src,
            "kernel": traffic_kernel,
        },
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
        "wall_s_timed_region": wall,
        "single_launch_ms": {"median": statistics.median(step_ms), "min": min(step_ms),
                             "note": "one launch alone between two events after a 1 GiB L2 flush "
                                     "(carries the launch and event overhead; not the bench value)"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = cpu_oracle_rate(w, rows_target_s=10.0, max_rows=rows * 8, inverse=inv)
        result["cpu_baseline"] = {"value": rate, "unit": "rows/s", "cores": cores, "kind": "oracle", "sample": sample}
        rate, cores, sample = cpu_dense_rate(w, rows_sample=min(rows, 512))
        result["cpu_baseline_dense"] = {"value": rate, "unit": "rows/s", "cores": cores, "kind": "oracle (dense Q)",
                                        "sample": sample}
    return result


def run_bwd_bench(args, spec, rank, world, local_rank):
    """The calibration backward: one bq_butterfly_bwd launch over all layers per step."""
    import torch
    import torch.distributed as dist

    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build as bq_build
    from rotation_bit_quantization_b200 import workloads as wl

    bq_build.build()
    bq.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    L_total, T, m = spec["layers"], spec["rows"], spec["n"]
    # the layers are independent: under torchrun rank r takes layers r, r + N, ... of the
    # same workload (angles and inputs depend on the layer index only); no collective
    mine = wl.shard_layers(L_total, world, rank)
    L = len(mine)
    if L == 0:
        raise SystemExit(f"rank {rank}: no layer of {L_total} left for {world} ranks")
    thetas = wl.backward_angles(mine, m)
    layers = [bq.Layer(torch.from_numpy(thetas[l]).to(dev)) for l in range(L)]
    x, dy = wl.backward_inputs_device(mine, T, m, dev)
    y = torch.empty((L, T, m), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((L, T, m), dtype=torch.float32, device=dev)
    dth = torch.empty((L, 12 * m // 2), dtype=torch.float32, device=dev)
    ws = torch.empty(bq.bq_butterfly_bwd_workspace_size(m, L, T), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        bq.bq_butterfly_bwd(layers, x, y, dy, dx, dth, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id_for(dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for s_, e_ in evs:
        s_.record(stream)
        step()
        e_.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = float(sum(s_.elapsed_time(e_) for s_, e_ in evs))
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / args.steps
    tokens = L_total * T    # all ranks together
    by_tok = m * (2 + 2 + 4 + 4)
    traffic, traffic_kernel = recorded_traffic("bwd") if not (args.rows or args.layers) else (None, None)
    peaks, peak_src = load_peaks()
    achieved = L * T * by_tok / (ms * 1e-3) / 1e9    # this rank's kernel

    # end to end through the public API with host buffers, on one layer of the workload
    # (the whole 103 GB batch does not fit a host round trip per step): H2D of X and dY,
    # the launch, D2H of Y, dX and dtheta
    e2e = None
    if not args.no_e2e:
        with GpuLocalCpus(dev) as host_cpus:  # pinned buffers on the GPU's NUMA node
            x1 = x[0].cpu().pin_memory()
            dy1 = dy[0].cpu().pin_memory()
            y1h = torch.empty(y[0].shape, dtype=y.dtype).pin_memory()
            dx1h = torch.empty(dx[0].shape, dtype=dx.dtype).pin_memory()
            dth1h = torch.empty(dth[0:1].shape, dtype=dth.dtype).pin_memory()
            x1d, dy1d = torch.empty_like(x[0:1]), torch.empty_like(dy[0:1])
            y1d, dx1d, dth1d = torch.empty_like(y[0:1]), torch.empty_like(dx[0:1]), torch.empty_like(dth[0:1])
            ws1 = torch.empty(bq.bq_butterfly_bwd_workspace_size(m, 1, T), dtype=torch.uint8, device=dev)

            def e2e_step():
                x1d[0].copy_(x1, non_blocking=True)
                dy1d[0].copy_(dy1, non_blocking=True)
                bq.bq_butterfly_bwd(layers[:1], x1d, y1d, dy1d, dx1d, dth1d, ws1)
                y1h.copy_(y1d[0], non_blocking=True)
                dx1h.copy_(dx1d[0], non_blocking=True)
                dth1h.copy_(dth1d, non_blocking=True)

            e2e_step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            n_e2e = min(args.steps, 3)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n_e2e):
                e2e_step()
            e1.record(stream)
            torch.cuda.synchronize()
            te = torch.tensor([e0.elapsed_time(e1) / n_e2e], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            e2e = {"value": T * world / (float(te.item()) * 1e-3), "unit": "tokens/s", "host_cpus": host_cpus.cpus,
                   "h2d_bytes_per_step": x1.numel() * 2 + dy1.numel() * 4,
                   "d2h_bytes_per_step": y1h.numel() * 2 + dx1h.numel() * 4 + dth1h.numel() * 4,
                   "scope": f"one layer of the workload ({T} tokens), host buffers pinned"}
            del x1, dy1, y1h, dx1h, x1d, dy1d, y1d, dx1d
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, sample = cpu_bwd_rate(0, 256, m)
        cpu = {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample}
    return {
        "metric": "butterfly backward tokens/s (Y, dX, dtheta), n=4096", "value": tokens / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong" if world > 1 else "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded on device)", "config": {"workload": spec["label"], "layers": L_total, "tokens_per_layer": T,
                                                           "parallelism": f"layers split over {world} rank(s), "
                                                                          f"{L} on rank {rank}, no collective",
                                                           "l2": "inputs 103 GB, far larger than L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                     "algorithmic_bytes_per_token": by_tok, "algorithmic_flops_per_token": 368640,
                     "kernel": traffic_kernel},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": args.steps, "clocks": clocks,
    }


def run_uniformity_bench(args, spec, rank, world, local_rank):
    """The calibration regulariser: one bq_uniformity_loss over a batch of rotated activations."""
    import torch
    import torch.distributed as dist

    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build as bq_build

    bq_build.build()
    bq.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    rows, n, bits, group = spec["rows"], spec["n"], spec["bits"], spec["group"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(11 + rank)
    y = torch.randn((rows, n), generator=gen, device=dev) * 0.5
    y[:, torch.randperm(n, generator=gen, device=dev)[:6]] *= 40.0     # outlier channels
    kl = torch.empty((rows, n // group), dtype=torch.float32, device=dev)
    dy = torch.empty_like(y)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        bq.bq_uniformity_loss(y, bits, group, 1e-4, kl, dy, loss)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id_for(dev))
    t_busy = time.perf_counter()
    while time.perf_counter() - t_busy < 0.5:
        for _ in range(10):
            step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for s_, e_ in evs:
        s_.record(stream)
        step()
        e_.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = float(sum(s_.elapsed_time(e_) for s_, e_ in evs))
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / args.steps
    by_row = 4 * n + 4 * n + 4 * (n // group)
    peaks, peak_src = load_peaks()
    achieved = rows * by_row / (ms * 1e-3) / 1e9
    # end to end through the public API with host buffers: H2D of y, the launch, D2H of
    # dL/dY, the per-group KL and the loss
    e2e = None
    if not args.no_e2e:
        with GpuLocalCpus(dev) as host_cpus:  # pinned buffers on the GPU's NUMA node
            y_pin = y.cpu().pin_memory()
            dy_pin = torch.empty(dy.shape, dtype=dy.dtype).pin_memory()
            kl_pin = torch.empty(kl.shape, dtype=kl.dtype).pin_memory()
            loss_pin = torch.empty(1, dtype=torch.float32).pin_memory()
            y_dev = torch.empty_like(y)

            def e2e_step():
                y_dev.copy_(y_pin, non_blocking=True)
                bq.bq_uniformity_loss(y_dev, bits, group, 1e-4, kl, dy, loss)
                dy_pin.copy_(dy, non_blocking=True)
                kl_pin.copy_(kl, non_blocking=True)
                loss_pin.copy_(loss, non_blocking=True)

            e2e_step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            n_e2e = min(args.steps, 5)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n_e2e):
                e2e_step()
            e1.record(stream)
            torch.cuda.synchronize()
            te = torch.tensor([e0.elapsed_time(e1) / n_e2e], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            e2e = {"value": rows * world / (float(te.item()) * 1e-3), "unit": "rows/s", "host_cpus": host_cpus.cpus,
                   "h2d_bytes_per_step": y.numel() * 4, "d2h_bytes_per_step": dy.numel() * 4 + kl.numel() * 4 + 4}
            del y_pin, dy_pin, y_dev
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import calib as oc
        sample = y[:512].cpu().numpy()
        t0 = time.perf_counter()
        oc.uniformity_loss(sample, bits, group, 1e-4)
        el = time.perf_counter() - t0
        cpu = {"value": sample.shape[0] / el, "unit": "rows/s", "cores": 1, "kind": "oracle",
               "sample": f"{sample.shape[0]} rows of the batch (float64 numpy), {el:.1f} s"}
    traffic, traffic_kernel = recorded_traffic("uniformity") if not args.rows else (None, None)
    return {
        "metric": "uniformity regulariser rows/s (per-group KL + dL/dY), n=4096 INT4 g128", "value": rows * world / (ms * 1e-3),
        "unit": "rows/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded on device)", "config": {"workload": spec["label"], "rows": rows,
                                                           "l2": "input 1 GiB, larger than L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                     "algorithmic_bytes_per_row": by_row, "kernel": traffic_kernel or "k_uniformity"},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": 2 * args.steps, "clocks": clocks,
    }


def oracle_gemm_rate(x_bits, codes, s16, z16, bits, group, tokens_sample):
    """Output elements/s of the float64 oracle GEMM on a bounded sample of tokens (all features),
    counting the dequantization of the whole weight matrix."""
    from oracle import w2a16 as ow
    from rotation_bit_quantization_b200 import workloads as wl
    xs = wl.f32_from_bf16_bits(x_bits[:tokens_sample])
    t0 = time.perf_counter()
    ow.w2a16_gemm(xs, codes, s16, z16, bits, group)
    el = time.perf_counter() - t0
    flops = 2.0 * tokens_sample * x_bits.shape[1] * codes.shape[0]
    return flops / el, el


def run_block_bench(args, spec, rank, world, local_rank):
    """The block transform + MXFP4 quantizer (bq_block_transform_quantize) over a batch of
    activations, timed like the transform line: K launches in one CUDA graph over input
    sets cycled so that every step reads an input that is not in L2."""
    import torch
    import torch.distributed as dist

    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build as bq_build
    from rotation_bit_quantization_b200 import workloads as wl

    bq_build.build()
    bq.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    rows, C, G, fmt = spec["rows"], spec["n"], spec["group"], spec["fmt"]
    w = wl.act_4096(rows, seed_offset=rank)
    x_host = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16)
    x = x_host.to(dev)
    Tb = wl.block_transforms(C, G)
    T = torch.from_numpy(Tb.view(np.int16)).to(dev).view(torch.bfloat16).view(C // G, G, G)
    bt = bq.BlockTransform(T)
    out_bytes = C // 2 + C // G
    set_bytes = rows * (C * 2 + out_bytes)
    NS = max(2, int(np.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x] + [x.clone() for _ in range(NS - 1)]
    outs = [bq.block_outputs(rows, C, fmt, dev) for _ in range(NS)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        bq.bq_block_transform_quantize(bt, xs[i % NS], fmt, *outs[i % NS], status=status)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            for i in range(args.steps):
                step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id_for(dev))
    t_busy = time.perf_counter()
    while time.perf_counter() - t_busy < 0.5:
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    del graph
    if int(status.item()) != 0:
        raise SystemExit(f"block kernel reported a wait timeout (status {int(status.item())})")
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / args.steps
    by_launch = rows * (C * 2 + out_bytes)
    flops = 2.0 * rows * C * G
    peaks, peak_src = load_peaks()
    gbs = by_launch / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        with GpuLocalCpus(dev) as host_cpus:  # pinned buffers on the GPU's NUMA node
            codes, scales = outs[0]
            x_pin = x_host.pin_memory()
            outs_pin = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (codes, scales)]

            def make_dev():
                return torch.empty_like(x), list(bq.block_outputs(rows, C, fmt, dev))

            def call(xc, oc):
                bq.bq_block_transform_quantize(bt, xc, fmt, *oc, status=status)

            if world > 1:
                dist.barrier()
            e2e_ms, e2e_method = pipelined_e2e(torch, dev, stream, x_pin, outs_pin, make_dev, call, args.steps,
                                               args.warmup)
            te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            e2e = {"value": rows * world / (float(te.item()) * 1e-3), "unit": "rows/s", "host_cpus": host_cpus.cpus,
                   "h2d_bytes_per_step": int(x_pin.numel() * 2),
                   "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outs_pin)),
                   "ms_per_step": float(te.item()),
                   "pipeline": f"{E2E_CHUNKS} row chunks per step on three streams (copy-in, the library call, "
                               f"copy-out), two device buffer sets alternating by step; timed as {e2e_method}"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import blockq as obq
        xs_h = wl.f32_from_bf16_bits(w.x[:256]).astype(np.float64)
        Tf = wl.f32_from_bf16_bits(Tb).astype(np.float64)
        t0 = time.perf_counter()
        obq.quantize(obq.block_transform(Tf, xs_h).astype(np.float32), fmt)
        el = time.perf_counter() - t0
        cpu = {"value": 256 / el, "unit": "rows/s", "cores": 1, "kind": "oracle",
               "sample": f"256 rows (float64 numpy einsum + the MXFP4 quantizer), {el:.2f} s"}
    return {
        "metric": "block transform + MXFP4 rows/s, n=4096 (per-block 32 x 32 transforms on tcgen05)",
        "value": rows * world / (ms * 1e-3), "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 operands, f32 accumulate", "data": "synthetic (seeded)",
        "config": {"workload": spec["label"], "rows": rows, "C": C, "G": G, "format": fmt,
                   "l2": f"inputs larger than L2: {NS} input/output sets cycled ({NS * set_bytes / 1e6:.0f} MB)",
                   "timing": f"{args.steps} launches in one CUDA graph between two CUDA events"},
        "gbs": gbs,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None, "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": by_launch, "algorithmic_flops_per_launch": flops,
                     "tensor_tflops": flops / (ms * 1e-3) / 1e12, "kernel": "k_blockq<MXFP4, G=32>"},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": args.steps, "clocks": clocks,
    }


def run_gemm_bench(args, spec, rank, world, local_rank):
    """The W2A16 consumer GEMM (bq_w2a16_gemm) on the LLaMA-2-7B MLP shape."""
    import torch
    import torch.distributed as dist

    import rotation_bit_quantization_b200 as bq
    from rotation_bit_quantization_b200 import build as bq_build
    from rotation_bit_quantization_b200 import workloads as wl

    bq_build.build()
    bq.load()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tokens = spec["rows"]
    xb, codes_h, s16, z16, bits, group = wl.w2a16_4096(tokens, spec["out_features"], seed=6 + rank)
    n, out_f = xb.shape[1], codes_h.shape[0]
    x_host = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    x = x_host.to(dev)
    codes = torch.from_numpy(codes_h).to(dev)
    scale = torch.from_numpy(s16.view(np.int16)).to(dev)
    zero = torch.from_numpy(z16.view(np.int16)).to(dev)
    out = torch.empty((tokens, out_f), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    ws_bytes = bq.bq_w2a16_gemm_workspace_size(tokens, n, out_f)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step():
        bq.bq_w2a16_gemm(x, codes, scale, zero, bits, group, out, workspace=ws, status=status)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id_for(dev))
    t_busy = time.perf_counter()
    while time.perf_counter() - t_busy < 0.5:
        for _ in range(10):
            flush.zero_()
            step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for s_, e_ in evs:
        flush.zero_()
        s_.record(stream)
        step()
        e_.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise SystemExit(f"w2a16 kernel reported a wait timeout (status {int(status.item())})")
    total_ms = float(sum(s_.elapsed_time(e_) for s_, e_ in evs))
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / args.steps
    flops = 2.0 * tokens * n * out_f
    tflops = flops * world / (ms * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        with GpuLocalCpus(dev) as host_cpus:  # pinned buffers on the GPU's NUMA node
            x_pin = x_host.pin_memory()
            o_pin = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            # token chunks of the same GEMM (the weights stay on the device, as for a served layer)
            chunk_tokens = -(-tokens // E2E_CHUNKS)
            ws_c = torch.empty(max(256, bq.bq_w2a16_gemm_workspace_size(chunk_tokens, n, out_f)), dtype=torch.uint8,
                               device=dev)

            def make_dev():
                return torch.empty_like(x), [torch.empty_like(out)]

            def call(xc, oc):
                bq.bq_w2a16_gemm(xc, codes, scale, zero, bits, group, oc[0],
                                 workspace=ws_c if xc.shape[0] == chunk_tokens else None, status=status)

            if world > 1:
                dist.barrier()
            e2e_ms, e2e_method = pipelined_e2e(torch, dev, stream, x_pin, [o_pin], make_dev, call, args.steps,
                                               args.warmup)
            te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            e2e = {"value": flops * world / (float(te.item()) * 1e-3) / 1e12, "unit": "TFLOP/s", "host_cpus": host_cpus.cpus,
                   "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                   "ms_per_step": float(te.item()),
                   "pipeline": f"{E2E_CHUNKS} token chunks per step on three streams (copy-in, the GEMM, copy-out), "
                               f"two device buffer sets alternating by step; timed as {e2e_method}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, el = oracle_gemm_rate(xb, codes_h, s16, z16, bits, group, tokens_sample=256)
        cpu = {"value": rate / 1e12, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"256 of {tokens} tokens x all {out_f} features, dequantization of the whole weight "
                         f"matrix included, {el:.1f} s (numpy float64 matmul on the host's BLAS threads)"}
    peaks, peak_src = load_peaks()
    traffic, traffic_kernel = recorded_traffic("w2a16")
    return {
        "metric": "W2A16 GEMM TFLOP/s (bf16 x INT2 g128 on tcgen05), 2048 x 4096 x 11008", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)", "config": {"workload": spec["label"], "tokens": tokens, "n": n,
                                                 "out_features": out_f, "bits": bits, "group": group,
                                                 "l2": "1 GiB written between timed steps (L2 flushed)"},
        "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": peaks.get("bf16_tflops", 1590.0),
                     "unit": "TFLOP/s", "frac": tflops / world / peaks.get("bf16_tflops", 1590.0),
                     "traffic": traffic, "peak_source": peak_src + " (bf16 burst)",
                     "algorithmic_flops_per_launch": flops, "kernel": traffic_kernel or "k_w2a16"},
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": args.steps, "clocks": clocks,
    }


# ----------------------------------------------------------------------------- reference arm

def _reference_line(args, spec, metric, unit, value, el, cores, sample, config):
    return {
        "impl": "reference",
        "metric": metric,
        "value": value,
        "unit": unit,
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": config,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, spec):
    """The float64 oracle, as it stands, on the host cores: each step a bounded sample of
    the workload, the metric and unit of our arm's line for that workload."""
    kind = spec["kind"]
    t0 = time.perf_counter()
    if kind in ("quant", "fwd", "inv"):
        w = spec["make"](0)
        for _ in range(args.warmup):
            cpu_oracle_rate(w, rows_target_s=1.0, max_rows=256, inverse=kind == "inv")
        rates = []
        sample = cores = None
        t0 = time.perf_counter()
        for _ in range(args.steps):
            rate, cores, sample = cpu_oracle_rate(w, rows_target_s=3.0, max_rows=spec["rows"], inverse=kind == "inv")
            rates.append(rate)
        el = time.perf_counter() - t0
        return _reference_line(args, spec, "butterfly fwd+quant rows/s and GB/s at n=4096 on 1 B200; % of FP32/HBM roofline",
                               "rows/s", statistics.median(rates), el, cores, sample,
                               {"workload": spec["label"], "rows_per_gpu": spec["rows"], "n": spec["n"],
                                "bits": spec["bits"], "group": spec["group"]})
    if kind == "bwd":
        for i in range(args.warmup):
            cpu_bwd_rate(i, 16)
        rates = []
        t0 = time.perf_counter()
        for i in range(args.steps):
            rate, sample = cpu_bwd_rate(i % spec["layers"], 512)
            rates.append(rate)
        el = time.perf_counter() - t0
        return _reference_line(args, spec, "butterfly backward tokens/s (Y, dX, dtheta), n=4096", "tokens/s",
                               statistics.median(rates), el, 1, sample,
                               {"workload": spec["label"], "layers": spec["layers"], "tokens_per_layer": spec["rows"]})
    if kind == "uniformity":
        from oracle import calib as oc
        n, bits, group = spec["n"], spec["bits"], spec["group"]

        def rows_sample(seed, rows):
            # our arm's distribution: N(0, 0.5^2) with six outlier channels x40
            rng = np.random.default_rng(seed)
            y = (rng.standard_normal((rows, n)) * 0.5).astype(np.float32)
            y[:, rng.choice(n, 6, replace=False)] *= 40.0
            return y

        for i in range(args.warmup):
            oc.uniformity_loss(rows_sample(100 + i, 64), bits, group, 1e-4)
        rates = []
        t0 = time.perf_counter()
        for i in range(args.steps):
            y = rows_sample(i, 2048)
            ts = time.perf_counter()
            oc.uniformity_loss(y, bits, group, 1e-4)
            rates.append(y.shape[0] / (time.perf_counter() - ts))
        el = time.perf_counter() - t0
        return _reference_line(args, spec, "uniformity regulariser rows/s (per-group KL + dL/dY), n=4096 INT4 g128",
                               "rows/s", statistics.median(rates), el, 1,
                               "2048 rows per step (float64 numpy), the batch's distribution",
                               {"workload": spec["label"], "rows": spec["rows"]})
    if kind == "gemm":
        from rotation_bit_quantization_b200 import workloads as wl
        xb, codes, s16, z16, bits, group = wl.w2a16_4096(256, spec["out_features"], seed=6)
        oracle_gemm_rate(xb, codes, s16, z16, bits, group, 8)
        rates = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            rate, _ = oracle_gemm_rate(xb, codes, s16, z16, bits, group, 256)
            rates.append(rate / 1e12)
        el = time.perf_counter() - t0
        return _reference_line(args, spec, "W2A16 GEMM TFLOP/s (bf16 x INT2 g128 on tcgen05), 2048 x 4096 x 11008",
                               "TFLOP/s", statistics.median(rates), el, 1,
                               "256 tokens x 4096 x 11008 per step (float64 numpy, the whole weight matrix dequantized)",
                               {"workload": spec["label"], "tokens": spec["rows"], "out_features": spec["out_features"]})
    if kind == "block":
        from oracle import blockq as obq
        from rotation_bit_quantization_b200 import workloads as wl
        C, G, fmt = spec["n"], spec["group"], spec["fmt"]
        Tf = wl.f32_from_bf16_bits(wl.block_transforms(C, G)).astype(np.float64)
        w = wl.act_4096(256)
        xs = wl.f32_from_bf16_bits(w.x).astype(np.float64)
        obq.quantize(obq.block_transform(Tf, xs[:16]).astype(np.float32), fmt)
        rates = []
        t0 = time.perf_counter()
        for _ in range(args.steps):
            ts = time.perf_counter()
            obq.quantize(obq.block_transform(Tf, xs).astype(np.float32), fmt)
            rates.append(xs.shape[0] / (time.perf_counter() - ts))
        el = time.perf_counter() - t0
        return _reference_line(args, spec, "block transform + MXFP4 rows/s, n=4096 (per-block 32 x 32 transforms on tcgen05)",
                               "rows/s", statistics.median(rates), el, 1,
                               "256 rows per step (float64 numpy einsum + the MXFP4 quantizer)",
                               {"workload": spec["label"], "rows": spec["rows"]})
    raise SystemExit(f"no reference arm for workload kind {kind}")


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="act4096",
                    choices=["act4096", "fwd4096", "inv4096", "inv5120", "weight4096", "act5120", "bwd",
                             "uniformity", "w2a16", "wush4096"])
    ap.add_argument("--rows", type=int, default=0, help="override the workload's rows (tokens per layer for bwd)")
    ap.add_argument("--layers", type=int, default=0, help="override the backward workload's layer count")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    spec = workload_spec(args.workload)
    if args.rows or args.layers:
        # a smaller (or larger) instance of the same workload, e.g. for an ncu capture
        # that has to fit the profiling size rules; never the bench line's size
        from rotation_bit_quantization_b200 import workloads as wl
        rows = args.rows or spec["rows"]
        if spec["kind"] in ("bwd", "uniformity", "gemm", "block"):
            spec = dict(spec, rows=rows, layers=args.layers or spec.get("layers", 1))
        else:
            base = {"act4096": lambda r, k: wl.act_4096(r, seed_offset=k), "fwd4096": lambda r, k: wl.act_4096(r, seed_offset=k),
                    "inv4096": lambda r, k: wl.act_4096(r, seed_offset=k), "inv5120": lambda r, k: wl.act_5120(r),
                    "weight4096": lambda r, k: wl.weight_4096(r), "act5120": lambda r, k: wl.act_5120(r)}[args.workload]
            spec = dict(spec, rows=rows, make=lambda rank, b=base, r=rows: b(r, rank))
        spec["label"] = spec["label"] + f" [resized: rows={spec['rows']}" + (
            f", layers={spec['layers']}]" if spec["kind"] == "bwd" else "]")

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, spec)))
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if spec["kind"] == "bwd":
            res = run_bwd_bench(args, spec, rank, world, local_rank)
        elif spec["kind"] == "uniformity":
            res = run_uniformity_bench(args, spec, rank, world, local_rank)
        elif spec["kind"] == "block":
            res = run_block_bench(args, spec, rank, world, local_rank)
        elif spec["kind"] == "gemm":
            res = run_gemm_bench(args, spec, rank, world, local_rank)
        else:
            res = run_ours(args, spec, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
