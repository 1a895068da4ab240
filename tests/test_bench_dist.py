"""CPU: the benchmark's multi-rank plumbing, run as two gloo ranks.

With N GPUs every rank runs an independent replica of the decode; the only
cross-rank steps are the timing reductions (max of the device times, sum of
the bytes) and barriers around the timed region.  These run here on the CPU
with the gloo backend, world size 2.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    assert bench.dist_env() == (rank, rank, world)
    bench.dist_init(world, "gloo")
    bench.barrier()
    # per-rank device times and byte counts: the slowest rank's time, the total bytes
    t_max = bench.reduce_over_ranks(10.0 + rank, "max")
    b_sum = bench.reduce_over_ranks(1000.0 * (rank + 1), "sum")
    bench.barrier()
    results[rank] = (t_max, b_sum)
    dist.destroy_process_group()


def test_two_rank_reductions():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(results) == {0: (11.0, 3000.0), 1: (11.0, 3000.0)}


def test_single_rank_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(3.5, "max") == 3.5
    assert bench.reduce_over_ranks(2.0, "sum") == 2.0


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    from workloads import make_inputs
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"gpus": 2, "steps": 1, "warmup": 3, "reference_seqs": 1})()
    bench.run_reference(args, make_inputs("tiny"))
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_workload_config_of_the_gpu_arm(monkeypatch, capsys):
    # the driver compares the two arms' configs: the reference line must carry the
    # same workload description (and data note) the GPU arm builds with describe()
    sys.path.insert(0, ROOT)
    import json
    import bench
    from workloads import make_inputs
    monkeypatch.setenv("RANK", "0")
    inp = make_inputs("tiny")
    args = type("A", (), {"gpus": 1, "steps": 1, "warmup": 3, "reference_seqs": 2,
                          "partition": 0})()
    bench.run_reference(args, inp)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.describe(inp, 0, 1)
    assert line["data"] == bench.DATA
    assert "split" not in line["config"] and "num_ranges" not in line["config"]


@pytest.mark.parametrize("workload", ["tiny", "llama"])
def test_kv_bytes_per_step(workload):
    sys.path.insert(0, ROOT)
    import bench
    from workloads import make_inputs
    inp = make_inputs(workload)
    if workload == "tiny":
        assert bench.kv_bytes_per_step(inp) == (38 + 101) * 1 * 2 * 64 * 4 == 71168
    else:
        # 32 x 4096 tokens x 8 kv heads x (K + V) x 128 x 2 bytes = 512 MiB
        assert bench.kv_bytes_per_step(inp) == 536870912
