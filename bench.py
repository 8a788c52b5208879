"""Benchmark of libqmm's hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_m1|...]

One JSON line on rank 0.  The headline workload is the decode GEMV: x bf16
[1, 4096] against W [14336, 4096] quantized affine int4, group size 64,
transpose=true; the metric is weight+scale+bias bytes per second (GB/s).  The
same line carries the prefill GEMM (x [2048, 4096], int4) in TFLOP/s, both as
fractions of their rooflines, the end-to-end number through host buffers,
clocks sampled during the timed region, and the CPU oracle's throughput.

A step is one call of the hot path on one batch.  Weight copies rotate so the
bytes a step reads are never L2-resident (8 copies x 33 MB > 126 MB L2).  At
N > 1 (torchrun) every rank runs an independent replica (no data-path
collective), timing is the max over ranks, and the value is the sum of the
work all ranks did.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from quantized_matmul_03_b200 import workloads as wl  # noqa: E402

N_OUT, K_IN, GS = 14336, 4096, 64
L2_ROTATE = 8


def weight_bytes(n, k, bits, gs, elt=2):
    """Algorithmic bytes of one packed weight: codes + scales + biases."""
    return n * k * bits // 8 + 2 * n * (k // gs) * elt


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:  # host-only runs (the reference arm, CPU tests of the rank logic)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def whole_job_rate(world, steps, units_per_step, slowest_total_ms):
    """Units per second of the whole job: every rank does `steps` steps of
    `units_per_step`, and the job takes as long as its slowest rank."""
    return world * steps * units_per_step / (slowest_total_ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return None
        self.file.flush()
        rows = [r.split(",") for r in Path(self.file.name).read_text().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

# Device-side spin queued ahead of the start event (about 0.2 ms at 1.9 GHz):
# while it runs, the host finishes submitting the graph, so the start event
# marks the device starting the first timed step rather than the host
# enqueueing it (the same holding kernel benchmark harnesses such as nvbench
# use).  The spin itself is outside the timed region.
HOLD_CYCLES = 400_000


def timed_launches(fns, steps, warmup, world):
    """Run fns[i % len(fns)] for `warmup` eager iterations, then capture `steps`
    iterations into one CUDA graph and time its replay with CUDA events on the
    replay stream, bracketed by a barrier and a synchronize on both sides.
    Graph replay keeps host launch cost (~15 us per ctypes call) out of the
    device time.  Returns (total ms over the timed steps, mean ms per step,
    library kernel launches inside the timed region)."""
    from quantized_matmul_03_b200 import binding as qb
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(warmup):
            fns[i % len(fns)]()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = qb.qmm_launch_count()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(steps):
            fns[i % len(fns)]()
    launches = qb.qmm_launch_count() - n0
    graph.replay()                            # upload + one untimed replay
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(HOLD_CYCLES)
        t0.record(stream)
        graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total = t0.elapsed_time(t1)
    del graph
    return total, total / steps, launches


def timed_eager(fns, steps, warmup, world):
    """Eager loop through the public API (for the end-to-end number): total ms."""
    for i in range(warmup):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        fns[i % len(fns)]()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1)


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "src": "fallback"}


def strip_comments(text: str) -> str:
    """C/C++ source without its comments and blank lines (the kernel sources
    hold no string literal with comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(files) -> str:
    """Hash of the CUDA sources a kernel is built from (its .cu and the
    device headers it includes), comments removed: an edit to a comment does
    not change the kernel, an edit to the code does."""
    h = hashlib.sha256()
    for name in sorted(files):
        h.update(strip_comments((ROOT / "quantized_matmul_03_b200" / "csrc" / name).read_text()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, when the kernel's
    sources have not changed since it was taken; else None."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(e.get("source_files", [])):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

def make_packed(w_cpu, gs, bits, copies, device):
    from quantized_matmul_03_b200 import binding as qb
    w = w_cpu.to(device)
    wq, s, b = qb.qmm_quantize(w, gs, bits)
    out = [(wq, s, b)]
    for _ in range(copies - 1):
        out.append((wq.clone(), s.clone(), b.clone()))
    del w
    torch.cuda.synchronize()
    return out


def bench_decode(m, steps, warmup, world, device, bits=4, packs=None):
    from quantized_matmul_03_b200 import binding as qb
    c = wl.decode_case(m, bits=bits)
    if packs is None:
        packs = make_packed(c.w, c.group_size, c.bits, L2_ROTATE, device)
    x = c.x.to(device)
    y = torch.empty((m, N_OUT), dtype=torch.bfloat16, device=device)
    fns = [lambda p=p: qb.qmm_quantized_matmul(x, *p, True, c.group_size, c.bits, out=y)
           for p in packs]
    total_ms, per_ms, launches = timed_launches(fns, steps, warmup, world)
    nbytes = weight_bytes(N_OUT, K_IN, c.bits, c.group_size)
    return dict(case=c, packs=packs, x=x, y=y, total_ms=total_ms, per_ms=per_ms,
                launches=launches, bytes=nbytes, flops=2 * m * N_OUT * K_IN)


def bench_decode_e2e(d, steps, warmup, world, device):
    """Same decode step through the C-ABI call with host buffers
    (qmm_quantized_matmul_host, one prepared call per weight copy): each step
    copies pinned x in, runs the product and copies y out, all inside the
    timed region."""
    from quantized_matmul_03_b200 import binding as qb
    c = d["case"]
    x_host = c.x.clone().pin_memory()
    y_host = torch.empty(tuple(d["y"].shape), dtype=torch.bfloat16).pin_memory()
    x_dev, y_dev = d["x"], d["y"]
    packs = d["packs"]
    fns = [qb.HostMatmul(x_host, x_dev, *p, y_dev, y_host, True, c.group_size, c.bits)
           for p in packs]
    total_ms = timed_eager(fns, steps, warmup, world)
    total_ms = max_over_ranks(world, total_ms)
    gbs = world * steps * d["bytes"] / (total_ms * 1e-3) / 1e9
    return {"value": gbs, "unit": "GB/s",
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host.numel() * y_host.element_size()}


def bench_prefill(bits, steps, warmup, world, device):
    from quantized_matmul_03_b200 import binding as qb
    c = wl.prefill_case(bits)
    packs = make_packed(c.w, c.group_size, c.bits, 2, device)
    x = c.x.to(device)
    y = torch.empty((x.shape[0], N_OUT), dtype=torch.bfloat16, device=device)
    fns = [lambda p=p: qb.qmm_quantized_matmul(x, *p, True, c.group_size, c.bits, out=y)
           for p in packs]
    total_ms, per_ms, launches = timed_launches(fns, steps, warmup, world)
    flops = 2 * x.shape[0] * N_OUT * K_IN
    return dict(total_ms=total_ms, per_ms=per_ms, launches=launches, flops=flops)


def roofline_frac(t_ms, nbytes, flops, pk):
    """Fraction of max(bytes / HBM bandwidth, flops / bf16 peak) achieved."""
    t_roof = max(nbytes / (pk["hbm_gbs"] * 1e9), flops / (pk["bf16_tflops"] * 1e12))
    return t_roof / (t_ms * 1e-3), ("hbm" if nbytes / (pk["hbm_gbs"] * 1e9) >=
                                     flops / (pk["bf16_tflops"] * 1e12) else "tensor")


def bench_moe(steps, warmup, world, device):
    """gather_qmm on the MoE workload: 8 experts W [14336, 4096] int4 gs 64,
    x [512, 1, 4096], rhs Zipf(1.2).  The stacked experts (264 MB) exceed L2,
    so one copy suffices.  A step is the whole call (prepare, gather, product)."""
    from quantized_matmul_03_b200 import binding as qb
    c = wl.moe_case()
    wq, s, b = make_packed(c.w, c.group_size, c.bits, 1, device)[0]
    del c.w
    x = c.x.to(device)
    rhs = c.rhs_indices.to(device)
    batch, k = x.shape[0], x.shape[2]
    ws = torch.empty(qb.qmm_gather_qmm_workspace_size(batch, 1, k, wq.shape[0]),
                     dtype=torch.uint8, device=device)
    y = torch.empty((batch, 1, N_OUT), dtype=torch.bfloat16, device=device)
    fns = [lambda: qb.qmm_gather_qmm(x, wq, s, b, None, rhs, True, c.group_size, c.bits,
                                     workspace=ws, out=y)]
    total_ms, per_ms, launches = timed_launches(fns, steps, warmup, world)
    nbytes = wq.shape[0] * weight_bytes(N_OUT, K_IN, c.bits, c.group_size)
    return dict(total_ms=total_ms, per_ms=per_ms, launches=launches, bytes=nbytes,
                flops=2 * batch * N_OUT * K_IN)


def bench_next_rows(steps, warmup, world, device, pk):
    """The rows beyond the headline, each timed on the decode weight's shape
    (W [14336, 4096]): dense with a bias, the microscaled modes, 3-/6-bit codes
    and qqmm at M = 1 (weights rotating through copies larger than L2) and
    M = 2048, plus the quantize kernel.  Returns {name: result}."""
    from quantized_matmul_03_b200 import binding as qb
    out = {}
    c = wl.decode_case(1)
    w = c.w.to(device)
    x1 = c.x.to(device)
    x2048 = wl.prefill_case(4).x.to(device)

    def wbytes(bits, gs, sb_bytes):
        return N_OUT * K_IN * bits // 8 + N_OUT * (K_IN // gs) * sb_bytes

    def record(name, per_ms, nbytes, m):
        flops = 2 * m * N_OUT * K_IN
        f, bound = roofline_frac(per_ms, nbytes, flops, pk)
        out[name] = {"us": per_ms * 1e3, "frac": f, "bound": bound,
                     "GB/s": nbytes / (per_ms * 1e-3) / 1e9,
                     "TFLOP/s": flops / (per_ms * 1e-3) / 1e12}

    def copies(packed, n):
        return [packed] + [tuple(t.clone() if t is not None else None for t in packed)
                           for _ in range(n - 1)]

    # quantize (row a1): bf16 weight in, codes + scales + biases out
    wq4 = qb.qmm_quantize(w, 64, 4)
    _, q_ms, _ = timed_launches([lambda: qb.qmm_quantize(w, 64, 4, out=wq4)], steps, warmup, world)
    qbytes = N_OUT * K_IN * 2 + wbytes(4, 64, 4)
    out["quantize_int4_gs64"] = {"us": q_ms * 1e3, "GB/s": qbytes / (q_ms * 1e-3) / 1e9,
                                 "frac": qbytes / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"], "bound": "hbm"}
    # quantized_dense: the affine product plus a bias vector in the epilogue
    bias = torch.randn(N_OUT, device=device).to(torch.bfloat16)
    packs = copies(wq4, L2_ROTATE)
    y1 = torch.empty((1, N_OUT), dtype=torch.bfloat16, device=device)
    _, ms, _ = timed_launches([lambda p=p: qb.qmm_quantized_dense(x1, *p, bias, True, 64, 4, out=y1)
                               for p in packs], steps, warmup, world)
    record("dense_bias_m1_int4", ms, wbytes(4, 64, 4), 1)
    y2048 = torch.empty((2048, N_OUT), dtype=torch.bfloat16, device=device)
    _, ms, _ = timed_launches([lambda: qb.qmm_quantized_dense(x2048, *wq4, bias, True, 64, 4, out=y2048)],
                              max(3, steps // 4), warmup, world)
    record("dense_bias_m2048_int4", ms, wbytes(4, 64, 4), 2048)
    del packs
    # microscaled modes and affine 3-/6-bit codes
    specs = [("mxfp4", 32, 4, 1), ("mxfp8", 32, 8, 1), ("nvfp4", 16, 4, 1),
             ("affine", 64, 3, 4), ("affine", 64, 6, 4)]
    for mode, gs, bits, sbb in specs:
        name = mode if mode != "affine" else f"affine_int{bits}"
        packed = qb.qmm_quantize(w, gs, bits, mode)
        nb = wbytes(bits, gs, sbb)
        packs = copies(packed, max(2, -(-256_000_000 // nb)))
        _, ms, _ = timed_launches([lambda p=p: qb.qmm_quantized_matmul(x1, *p, True, gs, bits, mode, out=y1)
                                   for p in packs], steps, warmup, world)
        record(f"{name}_m1", ms, nb, 1)
        _, ms, _ = timed_launches([lambda: qb.qmm_quantized_matmul(x2048, *packed, True, gs, bits, mode,
                                                                   out=y2048)],
                                  max(3, steps // 4), warmup, world)
        record(f"{name}_m2048", ms, nb, 2048)
        if mode in ("nvfp4", "mxfp8"):
            for m, x, y in ((1, x1, y1), (2048, x2048, y2048)):
                wsz = int(qb.lib().qmm_qqmm_workspace_size(m, K_IN, gs, bits, 1))
                ws = torch.empty(wsz, dtype=torch.uint8, device=device)
                _, ms, _ = timed_launches(
                    [lambda p=p, x=x, y=y, ws=ws: qb.qmm_qqmm(x, p[0], p[1], gs, bits, mode, out=y, workspace=ws)
                     for p in (packs if m == 1 else [packed])], steps if m == 1 else max(3, steps // 4),
                    warmup, world)
                record(f"qqmm_{mode}_m{m}", ms, nb, m)
        del packs, packed
        torch.cuda.empty_cache()
    return out


def run_suite(args, world, device, pk):
    """Every measured configuration, one entry each (not the headline line)."""
    from quantized_matmul_03_b200 import binding as qb
    out = []
    for m in (1, 4, 8, 16):
        d = bench_decode(m, args.steps, args.warmup, world, device)
        nb = d["bytes"] + 2 * m * (K_IN + N_OUT)
        f, bound = roofline_frac(d["per_ms"], nb, d["flops"], pk)
        out.append({"workload": f"decode_m{m}_int4_gs64", "us": d["per_ms"] * 1e3,
                    "GB/s": d["bytes"] / (d["per_ms"] * 1e-3) / 1e9, "frac": f, "bound": bound})
        del d
    for bits in (4, 8):
        pre = bench_prefill(bits, max(3, min(args.steps, 20)), args.warmup, world, device)
        tf = pre["flops"] / (pre["per_ms"] * 1e-3) / 1e12
        out.append({"workload": f"prefill_m2048_int{bits}_gs64", "us": pre["per_ms"] * 1e3,
                    "TFLOP/s": tf, "frac": tf / pk["bf16_tflops"], "bound": "tensor"})
    w = wl.sweep_weight()
    for bits in (2, 4, 8):
        for gs in (32, 64, 128):
            for transpose in (True, False):
                wb = weight_bytes(4096, 4096, bits, gs)
                copies = max(2, -(-256_000_000 // wb))  # > 2x L2 per rotation
                packs = make_packed(w, gs, bits, copies, device)
                for m in (1, 16, 256):
                    x = wl.sweep_x(m).to(device)
                    y = torch.empty((m, 4096), dtype=torch.bfloat16, device=device)
                    fns = [lambda p=p: qb.qmm_quantized_matmul(x, *p, transpose, gs, bits, out=y)
                           for p in packs]
                    _, per_ms, _ = timed_launches(fns, args.steps, args.warmup, world)
                    flops = 2 * m * 4096 * 4096
                    f, bound = roofline_frac(per_ms, wb + 4 * m * 4096, flops, pk)
                    out.append({"workload": f"sweep_b{bits}_gs{gs}_{'t' if transpose else 'n'}_m{m}",
                                "us": per_ms * 1e3, "frac": f, "bound": bound})
                del packs
                torch.cuda.empty_cache()
    moe = bench_moe(max(3, min(args.steps, 50)), args.warmup, world, device)
    f, bound = roofline_frac(moe["per_ms"], moe["bytes"], moe["flops"], pk)
    out.append({"workload": "moe_e8_t512_int4_gs64", "us": moe["per_ms"] * 1e3,
                "GB/s": moe["bytes"] / (moe["per_ms"] * 1e-3) / 1e9,
                "TFLOP/s": moe["flops"] / (moe["per_ms"] * 1e-3) / 1e12, "frac": f,
                "bound": bound, "launches_per_step": moe["launches"] / max(3, min(args.steps, 50))})
    return out


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the decode workload)
# ---------------------------------------------------------------------------

def oracle_decode_sample(budget_s: float, rows: int = N_OUT):
    """Time the oracle's quantized_matmul on the decode workload (M = 1, the
    first `rows` weight rows), repeating until `budget_s` of CPU time."""
    import oracle
    c = wl.decode_case(1)
    w = c.w[:rows].contiguous()
    wq, s, b = oracle.quantize(w, c.group_size, c.bits)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.quantized_matmul(c.x, wq, s, b, True, c.group_size, c.bits)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    nbytes = weight_bytes(rows, K_IN, c.bits, c.group_size)
    return {"value": reps * nbytes / el / 1e9, "unit": "GB/s",
            "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": (f"oracle quantized_matmul, x [1,4096] x W[{rows},4096] int4 gs64, "
                       f"{reps} passes in {el:.1f} s (dequantize in C on 1 thread, float64 "
                       f"matmul on {torch.get_num_threads()} threads)")}


# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, timed on this host's cores."""
    if rank != 0:
        return 0
    import oracle
    rows = 1792        # 1/8 of the decode weight per step keeps a step ~0.1-0.3 s
    c = wl.decode_case(1)
    w = c.w[:rows].contiguous()
    wq, s, b = oracle.quantize(w, c.group_size, c.bits)
    for _ in range(args.warmup):
        oracle.quantized_matmul(c.x, wq, s, b, True, c.group_size, c.bits)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.quantized_matmul(c.x, wq, s, b, True, c.group_size, c.bits)
    el = time.perf_counter() - t0
    nbytes = weight_bytes(rows, K_IN, c.bits, c.group_size)
    v = args.steps * nbytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode_m1_int4_gs64 (rows sampled)", "rows_per_step": rows,
                   "M": 1, "N": N_OUT, "K": K_IN, "bits": 4, "group_size": GS},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": torch.get_num_threads(),
                         "kind": "oracle",
                         "sample": f"W rows [0,{rows}) of the decode weight per step"},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


PROFILE_CASES = ("decode_m1", "decode_m16", "decode_tc_m16", "prefill", "moe", "quantize", "kn_m256",
                 "decode_m1_mxfp4", "decode_m1_nvfp4")


def profile_case(name, steps, warmup, device):
    """Run one workload's call `warmup + steps` times and nothing else (for a
    profiler's launch filter): the decode weight (14336 x 4096 bf16, int4
    gs64) at M = 1, at M = 16 on the automatic path and on the forced decode
    tensor-core path; the prefill product (M = 2048); the MoE gather; the
    quantize of the decode weight; the 4096^2 sweep weight stored [K, N] at
    M = 256; the decode weight in mxfp4 / nvfp4 at M = 1."""
    from quantized_matmul_03_b200 import binding as qb
    if name == "moe":
        c = wl.moe_case()
        wq, s, b = make_packed(c.w, c.group_size, c.bits, 1, device)[0]
        x, rhs = c.x.to(device), c.rhs_indices.to(device)
        fn = lambda: qb.qmm_gather_qmm(x, wq, s, b, None, rhs, True, c.group_size, c.bits)
    elif name in ("decode_m1_mxfp4", "decode_m1_nvfp4"):
        mode = name.rsplit("_", 1)[1]
        c = wl.decode_case(1)
        gs = 32 if mode == "mxfp4" else 16
        wq, s, _ = qb.qmm_quantize(c.w.to(device), gs, 4, mode)
        x = c.x.to(device)
        fn = lambda: qb.qmm_quantized_matmul(x, wq, s, None, True, gs, 4, mode)
    elif name == "kn_m256":
        w = wl.with_outliers((K_IN, K_IN), seed=3, dtype=torch.bfloat16)
        wq, s, b = make_packed(w, 64, 4, 1, device)[0]
        x = wl.normal((256, K_IN), 4, 1.0, torch.bfloat16).to(device)
        fn = lambda: qb.qmm_quantized_matmul(x, wq, s, b, False, 64, 4)
    else:
        c = wl.decode_case(1) if name != "prefill" else wl.prefill_case(4)
        if name == "quantize":
            w = c.w.to(device)
            fn = lambda: qb.qmm_quantize(w, c.group_size, c.bits)
        else:
            wq, s, b = make_packed(c.w, c.group_size, c.bits, 1, device)[0]
            m = {"decode_m1": 1, "decode_m16": 16, "decode_tc_m16": 16}.get(name, 2048)
            x = (c.x if name == "prefill" else wl.decode_case(m).x).to(device)
            if name == "decode_tc_m16":
                qb.qmm_set_path("decode_tc")
            fn = lambda: qb.qmm_quantized_matmul(x, wq, s, b, True, c.group_size, c.bits)
    for _ in range(warmup + steps):
        fn()
    torch.cuda.synchronize()
    qb.qmm_device_status()
    qb.qmm_set_path("auto")
    print(json.dumps({"case": name, "calls": warmup + steps}), flush=True)


METRIC = "int4 qmm weight GB/s at M=1 and TFLOP/s at M=2048, % of roofline"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the rows beyond the headline (dense, microscaled, 3/6-bit, qqmm)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the prefill GEMM (for profiling); prints its own line")
    ap.add_argument("--prefill-bits", type=int, default=4)
    ap.add_argument("--suite", action="store_true",
                    help="time every configuration (decode M 1/4/8/16, prefill int4/int8, "
                         "the 54-point sweep, MoE) and print one JSON line of results")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=PROFILE_CASES,
                    help="run one workload's call warmup + steps times and print nothing else "
                         "(for a profiler); no timing")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        barrier(world)
        dist_teardown(world)
        return rc

    from quantized_matmul_03_b200 import binding as qb
    qb.lib()  # fails loudly if the library was not built
    device = torch.device("cuda", local)
    pk = peaks()

    if args.case:
        profile_case(args.case, args.steps, args.warmup, device)
        return 0

    if args.suite:
        with ClockSampler(local) as clk:
            suite = run_suite(args, world, device, pk)
        if rank == 0:
            print(json.dumps({"suite": suite, "peaks": pk, "clocks": clk.summary()}), flush=True)
        return 0

    if args.prefill_only:
        pre = bench_prefill(args.prefill_bits, args.steps, args.warmup, world, device)
        p_ms = max_over_ranks(world, pre["per_ms"])
        tf = pre["flops"] / (p_ms * 1e-3) / 1e12
        if rank == 0:
            print(json.dumps({"workload": f"prefill_m2048_int{args.prefill_bits}_gs64",
                              "value": tf, "unit": "TFLOP/s", "kernel_us": p_ms * 1e3,
                              "frac": tf / pk["bf16_tflops"], "launches": pre["launches"]}))
        return 0

    with ClockSampler(local) as clk:
        d = bench_decode(1, args.steps, args.warmup, world, device)
        d16 = bench_decode(16, args.steps, args.warmup, world, device, packs=d["packs"])
        pre = moe = None
        if not args.no_prefill:
            psteps = max(3, min(args.steps, 20))
            pre = bench_prefill(4, psteps, max(3, args.warmup // 4), world, device)
        if not args.no_moe:
            moe = bench_moe(max(3, min(args.steps, 20)), max(3, args.warmup // 4), world, device)
        nxt = None
        if not args.no_next:
            nxt = bench_next_rows(max(3, min(args.steps, 20)), max(3, args.warmup // 4), world, device, pk)
    clocks = clk.summary()

    total_ms = max_over_ranks(world, d["total_ms"])
    per_ms = max_over_ranks(world, d["per_ms"])
    value = whole_job_rate(world, args.steps, d["bytes"], total_ms) / 1e9
    achieved = d["bytes"] / (per_ms * 1e-3) / 1e9
    e2e = bench_decode_e2e(d, args.steps, args.warmup, world, device)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "decode_m1_int4_gs64", "M": 1, "N": N_OUT, "K": K_IN,
                   "bits": 4, "group_size": GS, "transpose": True,
                   "l2": f"rotating {L2_ROTATE} weight copies ({L2_ROTATE * d['bytes'] / 1e6:.0f}"
                         " MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                     "peak_src": pk["src"], "kernel_us": per_ms * 1e3,
                     "traffic": profiled_traffic("gemv", "decode_m1_int4_gs64")},
        "e2e": e2e,
        "gpu_launches": d["launches"],
    }
    if pre is not None:
        p_ms = max_over_ranks(world, pre["per_ms"])
        tf = pre["flops"] / (p_ms * 1e-3) / 1e12
        line["prefill"] = {
            "workload": "prefill_m2048_int4_gs64", "value": tf, "unit": "TFLOP/s",
            "kernel_us": p_ms * 1e3, "launches": pre["launches"],
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                         "peak_src": pk["src"]}}
        line["gpu_launches"] += pre["launches"]
    m16_ms = max_over_ranks(world, d16["per_ms"])
    m16_gbs = d16["bytes"] / (m16_ms * 1e-3) / 1e9
    line["decode_m16"] = {
        "workload": "decode_m16_int4_gs64", "value": m16_gbs, "unit": "GB/s",
        "kernel_us": m16_ms * 1e3, "launches": d16["launches"],
        "roofline": {"bound": "hbm", "achieved": m16_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": m16_gbs / pk["hbm_gbs"], "peak_src": pk["src"]}}
    line["gpu_launches"] += d16["launches"]
    if moe is not None:
        moe_ms = max_over_ranks(world, moe["per_ms"])
        f, bound = roofline_frac(moe_ms, moe["bytes"], moe["flops"], pk)
        line["moe"] = {
            "workload": "moe_e8_t512_int4_gs64", "value": moe["bytes"] / (moe_ms * 1e-3) / 1e9,
            "unit": "GB/s", "tflops": moe["flops"] / (moe_ms * 1e-3) / 1e12,
            "kernel_us": moe_ms * 1e3, "launches": moe["launches"],
            "roofline": {"bound": bound, "frac": f,
                         "definition": "max(weight bytes / HBM peak, flops / bf16 peak) / time",
                         "peak_src": pk["src"]}}
        line["gpu_launches"] += moe["launches"]
    if nxt is not None:
        line["next_rows"] = {k: {kk: round(vv, 4) if isinstance(vv, float) else vv for kk, vv in v.items()}
                             for k, v in nxt.items()}
    if clocks:
        line["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_decode_sample(args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_teardown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
