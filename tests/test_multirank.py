"""Host logic of the benchmark on CPU: max-over-ranks timing with two gloo
ranks (the same reduction bench.py runs over NCCL), throughput aggregation,
clock-sample summary and peak / traffic bookkeeping."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    elapsed = 100.0 + 50.0 * rank           # rank 1 is the slow one
    t = torch.tensor([elapsed], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    agg = bench.aggregate_times([float(t.item())], world, 10.0)
    out[rank] = (float(t.item()), agg["value"])
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        assert res[r][0] == 150.0
        # 10 units per rank, 2 ranks, 150 ms -> 133.33 units/s
        assert res[r][1] == pytest.approx(20.0 / 0.150)


def test_aggregate_takes_slowest_rank():
    agg = bench.aggregate_times([10.0, 12.0, 11.0], 3, 5.0)
    assert agg["ms"] == 12.0
    assert agg["value"] == pytest.approx(15.0 / 0.012)


def test_clock_summary_flags_reasons():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.max_mhz = True, 1965
    s.samples = [(0.5, 1000, 0), (1.0, 1900, 0x4), (1.5, 1950, 0),
                 (2.0, 1940, 0x40)]
    s.window = (0.9, 1.6)
    out = s.summary()
    assert out["sm_mhz"] == 1925.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples_in_timed_region"] == 2


def test_peaks_and_bytes():
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    assert bench.workload_bytes("qwen2.5-0.5b-int4-decode") == 203476992
    assert bench.workload_flops("qwen2.5-0.5b-int4-decode") == 2 * 357826560


def test_traffic_needs_matching_digest(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    csrc = tmp_path / "quantized_matmul_02_b200" / "csrc"
    os.makedirs(csrc)
    (csrc / "bc_gemv.cu").write_text("a")
    (csrc / "bc_gemv_stream.cu").write_text("c")
    (csrc / "bc_internal.cuh").write_text("b")
    d = bench.kernel_source_digest()
    f = tmp_path / "profiles" / "traffic_w.txt"
    f.write_text(f"source_digest: {d}\ndram_bytes_per_launch: 123\n")
    assert bench.recorded_traffic("w") == 123
    (csrc / "bc_gemv_stream.cu").write_text("changed")
    assert bench.recorded_traffic("w") is None


def test_decode_kernel_choice_and_launch_counts():
    """The bench's claim of kernels per step mirrors the library's dispatch:
    the streaming kernel for M <= 4 (168 matrices per launch), the tcgen05
    decode kernel plus its pre-pass for M = 5..16 (packed, or runtime below
    16 bits), the tensor-core GEMM for prefill (80 matrices per launch)."""
    assert bench.decode_kernel("qwen2.5-0.5b-int4-decode") == "stream"
    assert bench.decode_kernel("qwen3-8b-int4-decode-m16") == "tc"
    assert bench.decode_kernel("qwen3-8b-rtn3-decode-m16") == "tc"
    assert bench.launches_per_step("qwen2.5-0.5b-int4-decode", 168) == 1
    assert bench.launches_per_step("qwen3-8b-int4-decode", 252) == 2
    assert bench.launches_per_step("qwen3-8b-int4-decode-m16", 252) == 4
    assert bench.launches_per_step("qwen2.5-0.5b-int4-prefill-m2048", 168) == 3


def test_traffic_digest_covers_the_tcgen05_header(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    csrc = tmp_path / "quantized_matmul_02_b200" / "csrc"
    os.makedirs(csrc)
    for f in ("bc_gemv.cu", "bc_gemv_stream.cu", "bc_internal.cuh", "bc_tc.cuh"):
        (csrc / f).write_text(f)
    d = bench.kernel_source_digest()
    (tmp_path / "profiles" / "traffic_w.txt").write_text(
        f"source_digest: {d}\ndram_bytes_per_launch: 7\n")
    assert bench.recorded_traffic("w") == 7
    (csrc / "bc_tc.cuh").write_text("changed")
    assert bench.recorded_traffic("w") is None


def test_cpu_baseline_repeats_until_target():
    """The CPU baseline runs the oracle on prepared matrices until its time
    target, and says how many products over how many matrices it timed."""
    r = bench.cpu_baseline_sample("single-1024-rtn3-decode", target_s=0.2)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0
    assert r["cores"] >= 1
    assert "over 1 of the 1 matrices" in r["sample"]
    products = int(r["sample"].split(" matrix products")[0])
    assert products >= 2          # one matrix, run again until the target
