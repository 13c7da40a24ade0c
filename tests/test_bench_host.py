"""Host-side logic of bench.py (no GPU): rank reduction over gloo with two
ranks, per-rank seeding, algorithmic work and roofline arithmetic."""
import hashlib
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_mixture_experts_gating_b200.workloads import WORKLOADS


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    secs = [0.25, 0.75][rank]
    t, n = bench.combine_ranks(secs, 1000 * (rank + 1), dist)
    out[rank] = (t, n)
    dist.barrier()
    dist.destroy_process_group()


def test_combine_ranks_takes_max_time_and_sums_tokens_over_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1] == (0.75, 3000.0)


def test_combine_ranks_single_process_is_identity():
    assert bench.combine_ranks(0.5, 123, None) == (0.5, 123)


def test_rank_seeds_differ_and_rank0_keeps_the_workload_seed():
    seeds = {bench.rank_seed(1235, r) for r in range(8)}
    assert len(seeds) == 8 and bench.rank_seed(1235, 0) == 1235


def test_layer_work_mixtral_prefill_matches_the_closed_form():
    w = WORKLOADS["mixtral_prefill"]
    work = bench.layer_work(w, [2048] * 8)
    S = 16384
    assert work["gemm1"]["flops"] == 2 * S * 4096 * 14336 * 2
    assert work["gemm2"]["flops"] == 2 * S * 14336 * 4096
    # 6 * d * d_ff * T * k for the experts (5.77 TFLOP) plus the router
    assert abs(work["flops_layer"] - (6 * 4096 * 14336 * 16384 + 2 * 8192 * 8 * 4096)) < 1
    assert work["bytes_layer"] == 3 * 8 * 4096 * 14336 * 2 + 2 * 8192 * 4096 * 2 + 8 * 4096 * 4
    # per projection: its weights plus x (first) or y (second); no sorted or hidden rows
    assert work["gemm1"]["bytes"] == 2 * 8 * 4096 * 14336 * 2 + 8192 * 4096 * 2
    assert work["gemm2"]["bytes"] == 8 * 4096 * 14336 * 2 + 8192 * 4096 * 2


def test_layer_work_switch_counts_only_experts_with_kept_rows():
    w = WORKLOADS["switch_k1"]
    kept = [160] * 25 + [0] * 7 + [100] * 32
    work = bench.layer_work(w, kept)
    assert work["active_experts"] == 57 and work["S"] == 25 * 160 + 32 * 100
    assert work["gemm2"]["bytes"] == 57 * 768 * 3072 * 2 + 8192 * 768 * 2
    assert work["gemm1"]["flops"] == 2.0 * work["S"] * 768 * 3072


def test_layer_work_counts_four_bit_weights_as_codes_plus_scales():
    w = WORKLOADS["mixtral_decode_t1"]
    work = bench.layer_work(w, [1, 1, 0, 0, 0, 0, 0, 0], "int4")
    per = 4096 * 14336 * (0.5 + 2 / 128)
    assert work["active_experts"] == 2
    assert work["gemm1"]["bytes"] == 2 * 2 * per + 4096 * 2
    assert work["gemm2"]["bytes"] == 2 * per + 4096 * 2
    assert work["gemm1"]["flops"] == bench.layer_work(w, [1, 1, 0, 0, 0, 0, 0, 0])["gemm1"]["flops"]


def test_kernel_roofline_picks_the_binding_resource():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    r = bench.kernel_roofline(flops=1e12, nbytes=1e9, seconds=1e-3, peaks=peaks)
    assert r["bound"] == "tensor" and r["achieved"] == 1000.0 and abs(r["frac"] - 1000 / 1500) < 1e-4
    r = bench.kernel_roofline(flops=1e9, nbytes=3e9, seconds=1e-3, peaks=peaks)
    assert r["bound"] == "hbm" and r["achieved"] == 3000.0 and r["frac"] == 0.5
    assert r["frac_nominal"] == round(3000.0 / bench.NOMINAL_PEAKS["hbm_gbs"], 4)


def test_traffic_is_null_without_a_matching_profile(tmp_path, monkeypatch):
    assert bench.profiled_traffic("gemm1", "no_such_workload") is None


def test_backward_work_closed_forms():
    """Backward FLOPs: 5 (ReLU) or 8 (SwiGLU) d x d_ff contractions per kept
    row plus the router's three T x E x d; bytes: active experts' weights read,
    every expert's fp32 gradients written, x and dy read, dx and dW_r written."""
    sw = WORKLOADS["switch_k1"]
    f, b = bench.backward_work(sw, 4104, 8192, 57)
    assert f == 2.0 * 4104 * 768 * 3072 * 5 + 3 * 2.0 * 8192 * 64 * 768
    per = 2 * 768 * 3072
    assert b == 57 * per * 2 + 64 * per * 4 + 2 * 8192 * 768 * 2 + 8192 * 768 * 4 + 64 * 768 * 4
    mx = WORKLOADS["mixtral_prefill"]
    f, b = bench.backward_work(mx, 16384, 8192, 8)
    assert f == 2.0 * 16384 * 4096 * 14336 * 8 + 3 * 2.0 * 8192 * 8 * 4096
    per = 3 * 4096 * 14336
    assert b == 8 * per * 2 + 8 * per * 4 + 2 * 8192 * 4096 * 2 + 8192 * 4096 * 4 + 8 * 4096 * 4


def test_profiled_traffic_is_reported_only_while_its_sources_are_unchanged(tmp_path, monkeypatch):
    """A committed ncu summary names the sources it was taken from and their
    sha256; the bench reports its DRAM bytes only while they still match."""
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel source\n")
    (tmp_path / "profiles").mkdir()
    prof = tmp_path / "profiles" / "gemm2_someload.txt"
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    prof.write_text(f"dram_bytes_per_launch: 1234\nsource_files: kernel.cu\nsource_sha256: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("gemm2", "someload") == 1234.0
    # the 4-bit line of the same workload reads its own summary only
    assert bench.profiled_traffic("gemm2", "someload", "int4") is None
    (tmp_path / "profiles" / "gemm2_someload_int4.txt").write_text(
        f"dram_bytes_per_launch: 99\nsource_files: kernel.cu\nsource_sha256: {sha}\n")
    assert bench.profiled_traffic("gemm2", "someload", "int4") == 99.0
    src.write_text("// kernel source, changed\n")
    assert bench.profiled_traffic("gemm2", "someload") is None
    assert bench.profiled_traffic("gemm2", "someload", "int4") is None
