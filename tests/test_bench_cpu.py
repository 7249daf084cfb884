"""CPU tests of the benchmark's host logic: the max-over-ranks timing with two
gloo ranks, and the reference arm (the CPU oracle) in one process and under
torchrun with two ranks (rank 0 alone prints one JSON line)."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    results[rank] = bench.max_over_ranks(10.0 + 5.0 * rank)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(2, port, results), nprocs=2, join=True)
        assert dict(results) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"}


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_reference_arm_single_process():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                          "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600, check=True).stdout
    lines = _json_lines(out)
    assert len(lines) == 1
    line = lines[0]
    assert REQUIRED <= set(line)
    assert line["impl"] == "reference" and line["higher_is_better"] is False and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_two_ranks_under_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference", "--gpus", "2",
           "--workload", "tiny", "--steps", "2", "--warmup", "0"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, check=True).stdout
    lines = _json_lines(out)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_oracle_baseline_on_two_host_cores():
    """The all-cores CPU baseline: two spawned single-threaded oracle processes,
    each timing whole layers of its own copy of the inputs."""
    sys.path.insert(0, ROOT)
    import bench
    from latency_decode_b200 import datagen as dg
    us, reps = bench.time_oracle_all_cores(dg.WORKLOADS["tiny"], 0.3, 2)
    assert us > 0 and reps >= 2
    assert 1 <= bench.host_cores() <= 16


def test_recorded_traffic_matches_the_current_source_only(tmp_path, monkeypatch):
    """The bench's ncu traffic record: used while the recorded source digest
    matches the file, ignored once it does not (the kernel changed since the
    capture), and absent for an unknown kernel or workload."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.recorded_traffic("gemm_e4m3_kernel<1>", "no_such_workload") is None
    # a copy of the tree layout whose record carries a stale digest
    (tmp_path / "profiles").mkdir()
    (tmp_path / "src.cu").write_text("// kernel source\n")
    (tmp_path / "profiles" / "k.md").write_text(
        "traffic-record: kernel=k workload=w bytes_per_launch=123 source=src.cu sha256_16=0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k", "w") is None
    import hashlib
    digest = hashlib.sha256(b"// kernel source\n").hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        f"traffic-record: kernel=k workload=w bytes_per_launch=123 source=src.cu sha256_16={digest}\n")
    assert bench.recorded_traffic("k", "w") == 123
