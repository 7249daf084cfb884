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


def test_oracle_baseline_on_two_host_threads():
    """The all-cores CPU baseline: one layer at a time, its output columns and
    query heads spread over two host threads."""
    sys.path.insert(0, ROOT)
    import bench
    from latency_decode_b200 import datagen as dg
    wl = dg.WORKLOADS["tiny"]
    us, reps, secs = bench.time_oracle_threads(wl, bench.oracle_layer_inputs(wl), 0.3, 2)
    assert us > 0 and reps >= 1 and secs > 0
    assert 1 <= bench.host_cores() <= 16


@pytest.mark.parametrize("name", ["tiny", "verify4_small"])
def test_sliced_oracle_layer_equals_the_whole_oracle_layer(name):
    """Spreading a layer's output columns and query heads over threads changes
    nothing: every slice is the oracle's own function on part of the weights
    (or one head), so the outputs are identical bit for bit."""
    import dataclasses
    from concurrent.futures import ThreadPoolExecutor
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from latency_decode_b200 import datagen as dg
    if name == "tiny":
        wl = dg.WORKLOADS["tiny"]
    else:  # several query tokens, causal, grouped heads, at a size the oracle runs in seconds
        wl = dataclasses.replace(dg.WORKLOADS["verify4"], name=name, K=256, N2=1024, Hq=8, Hkv=2, d=64, L=300,
                                 Lcap=320)
    inp = bench.oracle_layer_inputs(wl)
    whole = bench.oracle_layer(wl, inp)
    with ThreadPoolExecutor(max_workers=3) as pool:
        sliced = bench.oracle_layer_sliced(wl, inp, bench.sliced_oracle_inputs(wl, inp, fc13_cols=96), pool)
    for a, b in zip(whole, sliced):
        assert a.shape == b.shape and np.array_equal(a, b)


def test_replay_plan_runs_exactly_n_steps_in_multi_step_graphs():
    """The bench replays CUDA graphs of `period` chained steps and one graph of
    the remainder: exactly n steps, and no single-step graphs unless n itself
    is 1 or leaves a remainder of 1."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.replay_plan(20, 24) == [20]        # fewer steps than the period: one graph of all of them
    assert bench.replay_plan(24, 24) == [24]
    assert bench.replay_plan(2000, 24) == [24] * 83 + [8]
    assert bench.replay_plan(48, 24) == [24, 24]
    assert bench.replay_plan(1, 24) == [1]
    assert bench.replay_plan(0, 24) == []
    for n in range(1, 200):
        for period in (1, 2, 3, 8, 24):
            plan = bench.replay_plan(n, period)
            assert sum(plan) == n and all(1 <= L <= period for L in plan)
            assert all(L == period for L in plan[:-1])


def test_graph_replayer_captures_each_length_once_and_replays_in_order():
    """GraphReplayer against a stand-in capture: the graph of length L holds
    fn(0..L-1) (each starts again at replica 0), one capture per distinct
    length, and run(n) executes exactly n steps."""
    sys.path.insert(0, ROOT)
    import bench
    log, captures = [], []

    class FakeGraph:
        def __init__(self, idxs):
            self.idxs = list(idxs)

        def replay(self):
            log.extend(self.idxs)

    def capture(fn, idxs):
        captures.append(len(idxs))
        return FakeGraph(idxs)

    rp = bench.GraphReplayer(lambda i: None, 6, capture).prepare(20)
    assert sorted(captures) == [2, 6]
    rp.run(20)
    assert log == list(range(6)) * 3 + [0, 1]
    assert rp.lengths(20) == [6, 2]
    rp.run(20)
    assert sorted(captures) == [2, 6]  # nothing captured again
    del log[:]
    rp.warm(20)  # the untimed replay ahead of a timed run: the plan's first graph, once
    assert log == list(range(6))
    del log[:]
    rp.warm(2)
    assert log == [0, 1]


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
