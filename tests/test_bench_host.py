"""Host logic of bench.py without a GPU: clock parsing, traffic bookkeeping,
the reference (CPU oracle) arm, and the multi-rank aggregation run as two
gloo ranks on CPU (the replicas share no data; only the timing is reduced)."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_parse_clock_csv_reports_median_under_load_and_reasons():
    txt = "\n".join([
        "0, 1965, 1965, 120.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1400, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1350, 1965, 1001.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1380, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    ])
    c = bench.parse_clock_csv(txt)
    assert c["sm_mhz"] == 1380 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["samples_under_load"] == 3
    assert bench.parse_clock_csv("") is None


def test_stored_traffic_requires_current_kernel_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({
        "w_ok": {"kernel": "wide", "source_digest": bench.source_digest("wide"), "dram_bytes_per_launch": 123},
        "s_ok": {"kernel": "skinny", "source_digest": bench.source_digest("skinny"), "dram_bytes_per_launch": 7},
        "w_stale": {"kernel": "wide", "source_digest": "0" * 16, "dram_bytes_per_launch": 456},
        "w_nokernel": {"source_digest": bench.source_digest("wide"), "dram_bytes_per_launch": 9}}))
    csrc = tmp_path / "int8_gemm_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in os.listdir(os.path.join(ROOT, "int8_gemm_b200", "csrc")):
        (csrc / name).write_bytes(open(os.path.join(ROOT, "int8_gemm_b200", "csrc", name), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.stored_traffic("w_ok") == 123 and bench.stored_traffic("s_ok") == 7
    assert bench.stored_traffic("w_stale") is None and bench.stored_traffic("w_nokernel") is None
    assert bench.stored_traffic("absent") is None
    # a change to a quantiser leaves both GEMM figures valid; a change to the
    # skinny kernel's own unit leaves the wide kernel's figure valid, not the reverse
    (csrc / "kernels_quantize.cu").write_bytes(b"// changed\n" + (csrc / "kernels_quantize.cu").read_bytes())
    assert bench.stored_traffic("w_ok") == 123 and bench.stored_traffic("s_ok") == 7
    (csrc / "kernels_skinny.cu").write_bytes(b"// changed\n" + (csrc / "kernels_skinny.cu").read_bytes())
    assert bench.stored_traffic("w_ok") == 123 and bench.stored_traffic("s_ok") is None
    (csrc / "wide_kernel.cuh").write_bytes(b"// changed\n" + (csrc / "wide_kernel.cuh").read_bytes())
    assert bench.stored_traffic("w_ok") is None


def test_peaks_fall_back_when_file_missing(tmp_path):
    p = bench.load_peaks(str(tmp_path / "none.json"))
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [2.0, 3.0][rank]

    def reduce_max(v):
        t = torch.tensor([v], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    t, value = bench.aggregate(local_ms, 1e12, world, reduce_max)
    q.put((rank, t, value))
    dist.barrier()
    dist.destroy_process_group()


def test_tensor_peak_burst_for_short_sustained_for_long_timed_regions():
    peaks = {"bf16_tflops": 1642.1, "bf16_tflops_sustained": 1397.0, "source": "measured"}
    p, src = bench.tensor_peak(peaks, 0.05)
    assert p == 1642.1 * 2 and "burst" in src
    p, src = bench.tensor_peak(peaks, 1.5)
    assert p == 1397.0 * 2 and "sustained" in src
    p, src = bench.tensor_peak({"bf16_tflops": 1590.0, "source": "fallback"}, 1.5)
    assert p == 1590.0 * 2 and "burst" in src


def test_aggregate_two_gloo_ranks_uses_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [3.0, 3.0]
    assert res[0][2] == res[1][2] == pytest.approx(2e12 / 3e-3)


def test_reference_arm_prints_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "fp8_tiny_256x256x512", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # the same `config` object the GPU arm prints for this workload (one process, world size 1)
    import workloads as wl
    w = wl.WORKLOADS["fp8_tiny_256x256x512"]
    assert line["config"] == bench.workload_config(w, 1, bench.describe(w)[1])
    assert set(line["config"]) >= {"workload", "op", "M", "N", "K", "G", "out_dtype", "l2", "parallelism"}


def test_algorithmic_work_of_every_workload():
    # the roofline's algorithmic FLOPs and bytes: operands read once, results written once
    import workloads as wl
    for name, w in wl.WORKLOADS.items():
        flops, byts, _ = bench.describe(w)
        kb, nb = -(-w.K // 128), -(-w.N // 128)
        if w.op == "fp8_blockwise":
            want_f = 2 * w.M * w.N * w.K
            want_b = w.M * w.K + w.N * w.K + 2 * w.M * w.N + 4 * w.M * kb + 4 * kb * nb
        elif w.op == "int_scaled_mm":
            want_f = 2 * w.M * w.N * w.K
            want_b = w.M * w.K + w.N * w.K + 4 * w.M * w.N + 4 * (w.M + w.N)
        elif w.op == "fp8_rowwise":
            out_es = 1 if w.extra.get("out") == "e4m3" else 2
            want_f = 2 * w.M * w.N * w.K
            want_b = w.M * w.K + w.N * w.K + out_es * w.M * w.N + 4 * w.M + 8 * w.N
        elif w.op == "quantize_1x128":
            want_f, want_b = 0, 3 * w.M * w.K + 4 * w.M * kb
        elif w.op == "quantize_t":
            rb = -(-w.M // 128)
            scales = w.K * rb if w.extra["group"] == "128x1" else rb * kb
            want_f, want_b = 0, 3 * w.M * w.K + 4 * scales
        elif w.op == "quantize_128x128":
            want_f, want_b = 0, 3 * w.M * w.K + 4 * (-(-w.M // 128)) * kb
        else:
            want_f = 2 * w.M * w.G * w.N * w.K
            want_b = w.M * w.G * w.K + w.G * w.N * w.K + 2 * w.M * w.G * w.N + w.M * w.G * kb + w.G * nb * kb
        assert (flops, byts) == (want_f, want_b), name
    # the e4m3 result halves the output bytes of the same GEMM
    bf = bench.describe(wl.WORKLOADS["fp8_rowwise_16640x5120x8192"])[1]
    e4 = bench.describe(wl.WORKLOADS["fp8_rowwise_e4m3out_16640x5120x8192"])[1]
    assert bf - e4 == 16640 * 5120


def test_reference_arm_of_a_quantiser_workload():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "quant_t_128x1_16640x5120_bf16", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"


def test_kernel_source_lists_cover_every_local_include():
    # a stored ncu traffic figure is tied to a digest of its kernel's sources:
    # every header a kernel's translation unit includes must be part of it
    import re
    csrc = os.path.join(ROOT, "int8_gemm_b200", "csrc")

    def local_includes(name, seen):
        if name in seen:
            return seen
        seen.add(name)
        for inc in re.findall(r'^#include "([^"]+)"', open(os.path.join(csrc, name)).read(), flags=re.M):
            if os.path.exists(os.path.join(csrc, inc)):
                local_includes(inc, seen)
        return seen

    for kernel, files in bench.KERNEL_SOURCES.items():
        units = [f for f in files if f.endswith(".cu")]
        assert len(units) == 1, kernel
        assert local_includes(units[0], set()) <= set(files), kernel
