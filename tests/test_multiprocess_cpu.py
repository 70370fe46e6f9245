"""The multi-rank plumbing of bench.py, on the CPU with two gloo ranks: replicas
report the slowest rank's time, the whole-job value counts every replica, and
the reference arm runs on rank 0 only (the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        out[rank] = bench.max_over_ranks(local_ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    port = free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork: earlier tests started threads
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1] == 5.0


def test_replica_value_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.replica_value(1e12, 1, 10.0)
    two = bench.replica_value(1e12, 2, 10.0)
    assert one == pytest.approx(100.0) and two == pytest.approx(200.0)


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "1", "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def test_decode_reference_arm_under_torchrun_prints_once():
    """bench.py --workload decode_8k --impl reference: rank 0 times the decode oracle and
    prints one line (GB/s of cache processed); rank 1 exits without work."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "decode_8k"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["config"]["cache_len"] == 8192 and rec["e2e"]["d2h_bytes_per_step"] == 0


def test_prologue_reference_arm_under_torchrun_prints_once():
    """bench.py --workload prologue_wide_d128 --impl reference: rank 0 times the prologue
    oracle (forward and backward for Q and K of a sample of heads) and prints one line."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload",
           "prologue_wide_d128"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["config"]["T"] == 2048 and rec["e2e"]["h2d_bytes_per_step"] == 0


def test_profile_phase_samples_never_follow_a_synchronize():
    """The per-kernel events sit in steps the host has run ahead of (never the first step of
    the phase), and there are enough of them to average."""
    sys.path.insert(0, ROOT)
    import bench
    idx = bench.sampled_indices(bench.PROFILE_STEPS)
    assert 0 not in idx and len(idx) >= 10
    assert bench.sampled_steps(bench.PROFILE_STEPS) == len(idx)
    assert all(b - a == bench.EVENT_EVERY for a, b in zip(idx, idx[1:]))


def test_kernel_sum_check_flags_mismatch():
    sys.path.insert(0, ROOT)
    import bench
    ratio, warn = bench.kernel_sum_check([0.1, 0.02, 0.15, 0.1], 0.372)
    assert abs(ratio - 0.37 / 0.372) < 1e-12 and warn is None
    ratio, warn = bench.kernel_sum_check([0.1477, 0.0205, 0.1481, 0.1105], 0.3721)
    assert ratio > 1.03 and "not trusted" in warn


def test_recorded_traffic_only_for_matching_sources(tmp_path):
    """A traffic record is used only while the kernel sources hash to the recorded value."""
    sys.path.insert(0, ROOT)
    import bench
    good = tmp_path / "good.md"
    good.write_text(f"source_hash: {bench.kernel_source_hash(bench.PROLOGUE_KERNEL_FILES)}\n\n"
                    "| kernel | workload | bytes per launch |\n|---|---|---|\n"
                    "| rope_qknorm_bwd | prologue_wide_d128 | 1.5e+08 |\n")
    stale = tmp_path / "stale.md"
    stale.write_text(good.read_text().replace("source_hash: ", "source_hash: 0"))
    args = ("rope_qknorm_bwd", "prologue_wide_d128")
    assert bench.recorded_traffic(*args, str(good), bench.PROLOGUE_KERNEL_FILES) == 1.5e8
    assert bench.recorded_traffic(*args, str(stale), bench.PROLOGUE_KERNEL_FILES) is None
    assert bench.recorded_traffic("rope_qknorm_fwd", "prologue_wide_d128", str(good),
                                  bench.PROLOGUE_KERNEL_FILES) is None
