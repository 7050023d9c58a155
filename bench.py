"""Throughput benchmark of the scaled low-precision GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the operation on one batch of synthetic inputs that are
already resident in HBM.  The default workload is the FP8 block-scaled GEMM
M=16640, N=5120, K=8192 (bf16 out).  Rank 0 prints one JSON line.

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica of the workload on its own GPU -- the operation has no exchange step --
and ``value`` is the total work of all ranks over the slowest rank's time
("scaling": "weak").

``--impl reference`` times the CPU oracle on the host cores instead (bounded
row sample per step); it is a reported baseline, not an optimisation target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 blockwise GEMM TFLOP/s at 16640x5120x8192; % of B200 dense FP8 peak"
DEFAULT_WORKLOAD = "fp8_16640x5120x8192"
L2_BYTES = 126 * 1024 * 1024
FP8_PER_BF16 = 2.0  # nominal dense fp8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
# B200 datasheet figures (dense): FP8 and INT8 tensor 4.5 PFLOP/s (POPS), HBM3e 8 TB/s
DENSE_TENSOR_TFLOPS = 4500.0
DATASHEET_HBM_GBS = 8000.0


# ---------------------------------------------------------------------------
# helpers that need no GPU (covered by tests/test_bench_host.py)
# ---------------------------------------------------------------------------
def load_peaks(path=os.path.join(ROOT, "MEASURED_PEAKS.json")):
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


SUSTAINED_AFTER_S = 0.5  # a timed region this long runs under the power cap, like the sustained peak loop


def tensor_peak(peaks: dict, timed_s: float):
    """FP8/INT8 dense tensor peak in TFLOP/s: the measured bf16 GEMM rate times the nominal fp8:bf16 ratio,
    burst for a short timed region, sustained (seconds-long loop under the power cap) for a long one."""
    sustained = timed_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    kind = "sustained" if sustained else "burst"
    return bf16 * FP8_PER_BF16, f"{peaks.get('source')}: bf16 {kind} x 2 (fp8:bf16 nominal ratio)"


# The device-code files of each kernel (its template, the PTX helpers it includes,
# the translation unit that instantiates and launches it, and the compile-time
# constants in launch.h).
KERNEL_SOURCES = {
    "wide": ["sm100.cuh", "tile_order.h", "wide_kernel.cuh", "skinny_kernel.cuh", "kernels_wide.cu", "launch.h"],
    "skinny": ["sm100.cuh", "tile_order.h", "wide_kernel.cuh", "skinny_kernel.cuh", "kernels_skinny.cu", "launch.h"],
    "gemv": ["sm100.cuh", "tile_order.h", "wide_kernel.cuh", "skinny_kernel.cuh", "kernels_gemv.cu", "launch.h"],
    "quantize": ["sm100.cuh", "group_quant.cuh", "tile_ring.cuh", "quant_ring.cuh", "quantize.h", "kernels_quantize.cu"],
    "quantize_t": ["sm100.cuh", "group_quant.cuh", "tile_ring.cuh", "quantize.h", "kernels_quantize_t.cu"],
    "quantize_blocks": ["sm100.cuh", "group_quant.cuh", "tile_ring.cuh", "quant_ring.cuh", "quantize.h",
                        "kernels_quantize_blocks.cu"],
}


def source_digest(kernel: str = "wide") -> str:
    """Hash of one kernel's CUDA sources: a stored ncu traffic figure is only valid for the kernel it was taken on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_gemm_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str):
    """dram read+write bytes per launch from the committed ncu summary, or None if stale/absent."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload)
    if not e or e.get("kernel") not in KERNEL_SOURCES or e.get("source_digest") != source_digest(e["kernel"]):
        return None
    return e.get("dram_bytes_per_launch")


def aggregate(local_ms: float, units_per_rank: float, world: int, reduce_max=None):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    t = reduce_max(local_ms) if reduce_max else local_ms
    return t, units_per_rank * world / (t / 1e3)


def parse_clock_csv(text: str):
    rows = []
    for line in text.strip().splitlines():
        if not line or line.startswith("index") or "clocks" in line:
            continue
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm = float(parts[1].split()[0])
            smax = float(parts[2].split()[0])
            pw = float(parts[3].split()[0]) if parts[3].split()[0] not in ("[N/A]", "N/A") else float("nan")
        except ValueError:
            continue
        rows.append({"sm": sm, "max": smax, "power": pw, "active": parts[4], "hw_slowdown": parts[5],
                     "hw_thermal": parts[6], "sw_thermal": parts[7], "sw_power_cap": parts[8]})
    if not rows:
        return None
    loaded = [r for r in rows if r["power"] != r["power"] or r["power"] > 300.0] or rows
    reasons = []
    for key, name in (("hw_slowdown", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                      ("sw_thermal", "sw_thermal_slowdown"), ("sw_power_cap", "sw_power_cap")):
        if any(r[key].lower() == "active" for r in rows):
            reasons.append(name)
    return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
            "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
QUANT_OPS = ("quantize_1x128", "quantize_t", "quantize_128x128")  # HBM-bound quantisers: GB/s, not TFLOP/s


def describe(w):
    import workloads as wl
    if w.op == "fp8_blockwise":
        flops = 2.0 * w.M * w.N * w.K
        byts = w.M * w.K + w.N * w.K + 2 * w.M * w.N + 4 * w.M * (w.K // 128) + 4 * (w.K // 128) * (-(-w.N // 128))
        dtype = "e4m3 (fp32 accumulate)"
    elif w.op == "int_scaled_mm":
        flops = 2.0 * w.M * w.N * w.K
        byts = w.M * w.K + w.N * w.K + 4 * w.M * w.N + 4 * (w.M + w.N)
        dtype = "s8 (s32 accumulate)"
    elif w.op == "fp8_rowwise":
        flops = 2.0 * w.M * w.N * w.K
        out_es = 1 if w.extra.get("out") == "e4m3" else 2
        byts = w.M * w.K + w.N * w.K + out_es * w.M * w.N + 4 * (w.M + 2 * w.N)  # scales and bias
        dtype = "e4m3 (fp32 accumulate)"
    elif w.op == "quantize_1x128":
        flops = 0.0  # no tensor work: the metric is bytes moved
        byts = 2 * w.M * w.K + w.M * w.K + 4 * w.M * (-(-w.K // 128))  # bf16 in, e4m3 codes + fp32 scales out
        dtype = "bf16 -> e4m3 (fp32 group scales)"
    elif w.op == "quantize_t":
        flops = 0.0
        rb, cb = -(-w.M // 128), -(-w.K // 128)
        nscales = w.K * rb if w.extra["group"] == "128x1" else rb * cb
        byts = 2 * w.M * w.K + w.M * w.K + 4 * nscales  # bf16 x [M, K] in, transposed codes + fp32 scales out
        dtype = f"bf16 -> e4m3, transposed ({w.extra['group']} groups, fp32 scales)"
    elif w.op == "quantize_128x128":
        flops = 0.0
        byts = 2 * w.M * w.K + w.M * w.K + 4 * (-(-w.M // 128)) * (-(-w.K // 128))  # bf16 in, codes + block scales
        dtype = "bf16 -> e4m3 (128x128 blocks, fp32 scales)"
    else:
        flops = 2.0 * w.M * w.G * w.N * w.K
        kb, nb = w.K // 128, -(-w.N // 128)
        byts = w.M * w.G * w.K + w.G * w.N * w.K + 2 * w.M * w.G * w.N + w.M * w.G * kb + w.G * nb * kb
        dtype = "e4m3 (fp32 accumulate)"
    return flops, float(byts), dtype


def copies_for(byts: float) -> int:
    """Independent input sets rotated per step so that consecutive steps never find their inputs in L2."""
    return max(1, math.ceil(3 * L2_BYTES / byts)) if byts < 3 * L2_BYTES else 1


def workload_config(w, world: int, byts: float) -> dict:
    """The `config` object of the JSON line; both arms print the same one for the same workload."""
    quant = w.op in QUANT_OPS
    copies = copies_for(byts)
    return {"workload": w.name, "op": w.op, "M": w.M, "N": w.N, "K": w.K, "G": w.G,
            "out_dtype": "float32" if w.op == "int_scaled_mm" else
            ("e4m3" if quant or w.extra.get("out") == "e4m3" else "bfloat16"),
            **({"scale_result": w.extra["scale_result"]} if "scale_result" in w.extra else {}),
            "l2": (f"inputs larger than L2 ({byts / 1e6:.0f} MB per step)" if copies == 1 else
                   f"{copies} rotating input copies ({copies * byts / 1e6:.0f} MB) to defeat L2"),
            "parallelism": f"replicas x{world}"}


def rowwise_out(w, device):
    """(output dtype, scale_result tensor or None) of an fp8_rowwise workload."""
    import torch
    if w.extra.get("out") == "e4m3":
        return torch.float8_e4m3fn, torch.tensor([w.extra["scale_result"]], dtype=torch.float32, device=device)
    return torch.bfloat16, None


def build_step(w, device, copies):
    """Device-resident inputs (`copies` independent sets, rotated per step) and the step closure."""
    import torch

    import int8_gemm_b200 as bs
    import workloads as wl

    d = wl.workload_inputs(w)
    sets = []
    for _ in range(copies):
        if w.op == "fp8_blockwise":
            A, B = d["A"].to(device), d["B_t"].to(device).t()
            sa, sb = d["scale_a"].to(device), d["scale_b"].to(device)
            out = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=device)
            sets.append(lambda A=A, B=B, sa=sa, sb=sb, out=out: bs.bs_gemm_fp8_blockwise(A, B, sa, sb, out=out))
        elif w.op == "int_scaled_mm":
            A, B = d["A"].to(device), d["B_t"].to(device).t()
            sa, sb = d["s_a"].to(device), d["s_b"].to(device)
            out = torch.empty(w.M, w.N, dtype=torch.float32, device=device)
            sets.append(lambda A=A, B=B, sa=sa, sb=sb, out=out: bs.int_scaled_mm(A, B, sa, sb, out=out))
        elif w.op == "fp8_rowwise":
            A, B = d["A"].to(device), d["B_t"].to(device).t()
            sa, sb, bias = d["scale_a"].to(device), d["scale_b"].to(device), d["bias"].to(device)
            odt, sr = rowwise_out(w, device)
            out = torch.empty(w.M, w.N, dtype=odt, device=device)
            sets.append(lambda A=A, B=B, sa=sa, sb=sb, bias=bias, out=out, odt=odt, sr=sr:
                        bs.bs_gemm_fp8_rowwise(A, B, sa, sb, bias, out_dtype=odt, out=out, scale_result=sr))
        elif w.op == "quantize_1x128":
            x = d["x"].to(device)
            q = torch.empty(w.M, w.K, dtype=torch.uint8, device=device)
            sc = torch.empty(w.M, -(-w.K // 128), dtype=torch.float32, device=device)
            sets.append(lambda x=x, q=q, sc=sc: bs.quantize_fp8_1x128(x, "f32", q=q, scale=sc))
        elif w.op == "quantize_t":
            x = d["x"].to(device)
            q, sc = bs.quantize_fp8_t(x, w.extra["group"], "f32")  # allocates the outputs once
            sets.append(lambda x=x, q=q, sc=sc: bs.quantize_fp8_t(x, w.extra["group"], "f32", q_t=q, scale=sc))
        elif w.op == "quantize_128x128":
            x = d["x"].to(device)
            q, sc = bs.bs_quantize_fp8_128x128(x, "f32")  # allocates the outputs once
            sets.append(lambda x=x, q=q, sc=sc: bs.bs_quantize_fp8_128x128(x, "f32", q=q, scale=sc))
        else:
            x, wt = d["x"].to(device), d["w"].to(device)
            xs, ws = d["x_scale"].to(device), d["w_scale"].to(device)
            out = torch.empty(w.M, w.G, w.N, dtype=torch.bfloat16, device=device)
            sets.append(lambda x=x, wt=wt, xs=xs, ws=ws, out=out: bs.bmm_a8w8_blockscale(x, wt, xs, ws, out=out))
    return d, sets


def e2e_runner(w, d, device, stream):
    """End-to-end steps through the public API: each step copies its inputs from pinned host memory to the
    device, runs the GEMM and copies the result back to pinned host memory.  Consecutive steps are pipelined
    over three streams with two buffer slots (inputs of step i+1 and the result of step i-1 move while step i
    computes), as a serving loop would; every step still moves all its bytes."""
    import torch

    import int8_gemm_b200 as bs

    pin = {k: v.contiguous().pin_memory() for k, v in d.items() if v is not None}
    s_res = None
    if w.op == "fp8_rowwise":
        out_shape, (out_dtype, s_res) = (w.M, w.N), rowwise_out(w, device)
    elif w.op == "fp8_blockwise":
        out_shape, out_dtype = (w.M, w.N), torch.bfloat16
    elif w.op == "int_scaled_mm":
        out_shape, out_dtype = (w.M, w.N), torch.float32
    else:
        out_shape, out_dtype = (w.M, w.G, w.N), torch.bfloat16
    host_out = [torch.empty(out_shape, dtype=out_dtype).pin_memory() for _ in range(2)]
    dev_in = [{k: torch.empty_like(v, device=device) for k, v in pin.items()} for _ in range(2)]
    dev_out = [torch.empty(out_shape, dtype=out_dtype, device=device) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in_done", "comp_done", "out_done")}
    used = [False, False]

    def compute(x, out):
        if w.op == "fp8_blockwise":
            bs.bs_gemm_fp8_blockwise(x["A"], x["B_t"].t(), x["scale_a"], x["scale_b"], out=out)
        elif w.op == "int_scaled_mm":
            bs.int_scaled_mm(x["A"], x["B_t"].t(), x["s_a"], x["s_b"], out_dtype=torch.float32, out=out)
        elif w.op == "fp8_rowwise":
            bs.bs_gemm_fp8_rowwise(x["A"], x["B_t"].t(), x["scale_a"], x["scale_b"], x.get("bias"),
                                   out_dtype=out_dtype, out=out, scale_result=s_res)
        else:
            bs.bmm_a8w8_blockscale(x["x"], x["w"], x["x_scale"], x["w_scale"], out=out)

    def run(steps):
        for i in range(steps):
            k = i % 2
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(ev["comp_done"][k])  # the step two back has consumed this input slot
                for name, v in pin.items():
                    dev_in[k][name].copy_(v, non_blocking=True)
                ev["in_done"][k].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(ev["in_done"][k])
                if used[k]:
                    stream.wait_event(ev["out_done"][k])  # its result slot has been read back
                compute(dev_in[k], dev_out[k])
                ev["comp_done"][k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp_done"][k])
                host_out[k].copy_(dev_out[k], non_blocking=True)
                ev["out_done"][k].record(s_out)
            used[k] = True
        return s_out

    run.first_stream = s_in
    return run, h2d, d2h


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def result(self):
        if self.file is None:
            return None
        try:
            with open(self.file.name) as f:
                txt = f.read()
            os.unlink(self.file.name)
        except OSError:
            return None
        return parse_clock_csv(txt)


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; never tuned)
# ---------------------------------------------------------------------------
def oracle_rows_run(w, d, rows):
    import oracle
    if w.op == "fp8_blockwise":
        oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"], rows=rows)
    elif w.op == "int_scaled_mm":
        oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], d["s_b"], rows=rows)
    elif w.op == "fp8_rowwise":
        y, _ = oracle.fp8_rowwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"], d["bias"], rows=rows)
        if w.extra.get("out") == "e4m3":
            oracle.e4m3_encode(w.extra["scale_result"] * y)
    elif w.op == "quantize_1x128":
        oracle.quantize_1x128(d["x"][rows], 0)
    elif w.op == "quantize_t":
        oracle.quantize_t(d["x"][rows], 0 if w.extra["group"] == "128x1" else 1, 0)
    elif w.op == "quantize_128x128":
        oracle.quantize_128x128(d["x"][rows], 0)
    else:
        oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"], rows=rows)


def sample_unit(w, threads: int) -> int:
    """Rows of the smallest oracle sample: one per host thread, and for the transposed quantiser whole
    128-row groups, so the sample quantises complete groups."""
    n = max(1, min(w.M, threads))
    if w.op in ("quantize_t", "quantize_128x128"):
        n = min(w.M, -(-n // 128) * 128)
    return n


def cpu_oracle_baseline(w, d, budget_s: float = 20.0):
    """Times the oracle on a bounded row sample sized to about `budget_s` seconds."""
    import oracle
    threads = oracle.num_threads()
    quant = w.op in QUANT_OPS
    flops_per_row = describe(w)[1 if quant else 0] / w.M  # bytes per row for the quantiser
    n = sample_unit(w, threads)
    t0 = time.perf_counter()
    oracle_rows_run(w, d, list(range(n)))
    dt = time.perf_counter() - t0
    rows = max(n, min(w.M, int(n * budget_s / max(dt, 1e-3) / n) * n))
    t0 = time.perf_counter()
    oracle_rows_run(w, d, list(range(rows)))
    dt = time.perf_counter() - t0
    return {"value": flops_per_row * rows / dt / (1e9 if quant else 1e12), "unit": "GB/s" if quant else "TFLOP/s",
            "cores": threads, "kind": "oracle",
            "sample": f"{rows} of {w.M} {'input' if quant else 'output'} rows of {w.name} (all columns), "
                      f"fp64 oracle, {dt:.1f} s"}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-baseline-s", type=float, default=20.0,
                    help="seconds of host-core work the cpu_baseline row sample is sized to")
    ap.add_argument("--shape", default=None,
                    help="ad-hoc problem 'M,N,K' (or 'M,G,N,K' for --op bmm) instead of a named workload")
    ap.add_argument("--op", default="fp8", choices=["fp8", "int8", "bmm"], help="operation for --shape")
    ap.add_argument("--path", default="auto", choices=["auto", "wide", "skinny", "wide1", "promote", "gemv"],
                    help="force a kernel family (wide = CTA-pair persistent, wide1 = single-CTA persistent, "
                         "promote = CTA-pair persistent with e8m0 block scales promoted on the CUDA cores)")
    ap.add_argument("--splits", type=int, default=0, choices=[0, 1, 2, 4, 8],
                    help="force the skinny kernel's split-K factor (0 = the planner's choice)")
    ap.add_argument("--stream-k", default="off", choices=["on", "off"],
                    help="off: compute every tile of the wide kernel whole (no split of the last wave)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    import workloads as wl
    if args.shape:
        dims = [int(v) for v in args.shape.split(",")]
        if args.op == "bmm":
            M, G, N, K = dims
            w = wl.Workload(f"bmm_g{G}_m{M}_n{N}_k{K}", "bmm_a8w8_blockscale", M, N, K, G=G, seed=3)
        else:
            M, N, K = dims
            op = "fp8_blockwise" if args.op == "fp8" else "int_scaled_mm"
            w = wl.Workload(f"{args.op}_{M}x{N}x{K}", op, M, N, K, seed=2 if args.op == "fp8" else 1)
    else:
        w = wl.WORKLOADS[args.workload]
    flops, byts, dtype = describe(w)

    if args.impl == "reference":
        run_reference(args, w, rank, world, flops)
        return

    import torch
    import torch.distributed as dist

    import int8_gemm_b200 as bs

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    def reduce_max(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    bs.set_path_override({"auto": 0, "wide": 1, "skinny": 2, "wide1": 3, "promote": 4, "gemv": 5}[args.path])
    bs.set_stream_k(args.stream_k == "on")
    bs.set_split_override(args.splits)
    copies = copies_for(byts)
    d, sets = build_step(w, device, copies)
    quant = w.op in QUANT_OPS
    if quant:
        plan = {"kernel": w.op, "launches": 1}
    else:
        op = {"fp8_blockwise": 1, "int_scaled_mm": 2, "bmm_a8w8_blockscale": 3, "fp8_rowwise": 4}[w.op]
        plan = bs.plan_for(op, w.M, w.G, w.N, w.K, torch.cuda.get_device_properties(device).multi_processor_count)

    for i in range(max(3, args.warmup)):
        sets[i % copies]()
    torch.cuda.synchronize()
    assert bs.device_error() == 0

    K = args.steps
    # The K steps are captured once into a CUDA graph (the library launches on the
    # caller's stream, so its kernels are recorded as graph nodes) and replayed:
    # the timed region then measures the device, not the Python call overhead.
    graph_steps = min(K, max(copies, 50))
    cap_stream = torch.cuda.Stream(device)
    cap_stream.wait_stream(torch.cuda.current_stream(device))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(graph, stream=cap_stream):
            for i in range(graph_steps):
                sets[i % copies]()
    torch.cuda.current_stream(device).wait_stream(cap_stream)
    replays = max(1, K // graph_steps)
    K = replays * graph_steps
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(replays):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    local_ms = ev[0][0].elapsed_time(ev[-1][1])
    per_launch_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    del graph
    err = bs.device_error()
    assert err == 0, f"device error word 0x{err:x}"
    step_ms, value = aggregate(local_ms / K, byts if quant else flops, world, reduce_max)
    value /= 1e9 if quant else 1e12

    # end to end through the public API with pinned host buffers
    e2e = None
    if args.e2e_steps > 0 and not quant:
        e2e_run, h2d, d2h = e2e_runner(w, d, device, stream)
        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(e2e_run.first_stream)  # every stream is idle here; the first step starts on this one
        last = e2e_run(args.e2e_steps)
        e1.record(last)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1) / args.e2e_steps)
        e2e = {"value": round(flops * world / (e2e_ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    peaks = load_peaks()
    if w.op in ("fp8_blockwise", "bmm_a8w8_blockscale", "fp8_rowwise") and flops / byts > 690 or w.op == "int_scaled_mm":
        bound, unit = "tensor", "TFLOP/s"
        peak, peak_source = tensor_peak(peaks, step_ms * K / 1e3)
        dense_peak = DENSE_TENSOR_TFLOPS
        achieved = flops / (per_launch_ms / 1e3) / 1e12
    else:
        bound, unit = "hbm", "GB/s"
        peak, peak_source = peaks["hbm_gbs"], f"{peaks.get('source')}: HBM copy"
        dense_peak = DATASHEET_HBM_GBS
        achieved = byts / (per_launch_ms / 1e3) / 1e9
    traffic = stored_traffic(w.name)

    result = {
        "metric": METRIC if w.name == DEFAULT_WORKLOAD else f"{w.name} {'GB/s' if quant else 'TFLOP/s'}",
        "value": round(value, 2),
        "unit": "GB/s" if quant else "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic (seeded N(0,1) with 1% x20 outliers, quantised per the workload recipe)",
        "config": workload_config(w, world, byts),
        "plan": plan,
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": unit,
                     "frac": round(achieved / peak, 4), "frac_basis": "of " + peak_source,
                     "traffic": traffic,
                     "kernel": f"{w.op}_kernel" if quant else
                               {1: "wide_gemm_kernel", 2: "skinny_gemm_kernel", 4: "gemv_kernel"}[plan["kernel"]],
                     "peak_source": peak_source,
                     "dense_peak": dense_peak,
                     "frac_dense_peak": round(achieved / dense_peak, 4)},
        "e2e": e2e,
        "gpu_launches": K * plan["launches"],
        "timing": f"{replays} replays of a CUDA graph holding {graph_steps} launches; CUDA events on the replay stream",
    }
    clocks = clk.result()
    if clocks:
        result["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_baseline(w, d, args.cpu_baseline_s)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(args, w, rank, world, flops):
    """The oracle on the host cores, per step a bounded row sample of the workload."""
    if rank != 0:
        return
    import oracle
    import workloads as wl
    d = wl.workload_inputs(w)
    threads = oracle.num_threads()
    rows_per_step = sample_unit(w, threads)
    sample = list(range(rows_per_step))
    for _ in range(max(1, args.warmup if args.warmup < 3 else 3)):
        oracle_rows_run(w, d, sample)
    steps = max(1, min(args.steps, 20))
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_rows_run(w, d, sample)
    dt = (time.perf_counter() - t0) / steps
    quant = w.op in QUANT_OPS
    unit = "GB/s" if quant else "TFLOP/s"
    value = (describe(w)[1] if quant else flops) / w.M * rows_per_step / dt / (1e9 if quant else 1e12)
    out = {
        "impl": "reference", "metric": METRIC if w.name == DEFAULT_WORKLOAD else f"{w.name} {unit}",
        "value": value, "unit": unit, "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle)", "data": "synthetic", "config": workload_config(w, world, describe(w)[1]),
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": f"{rows_per_step} of {w.M} {'input' if quant else 'output'} rows per step "
                                   "(all columns)"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
