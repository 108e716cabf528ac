"""The N > 1 plumbing of bench.py on CPU: two gloo ranks.

The decode path shards as independent replicas (every rank runs its own
batch on its own GPU, no collective on the data path); the process group only
carries the start/stop barriers and the max over ranks of the timings.  These
tests run that plumbing with world size 2 on the host, and the reference arm
end to end under torchrun, where rank 0 alone runs and prints.
"""
import json
import os
import socket
import subprocess
import sys
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    args = types.SimpleNamespace(impl="ours")
    w, r, local = bench.dist_setup(args, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank's own step time; the job's step time is the slowest rank's
    ms = bench.reduce_max(1.0 + 2.5 * rank, w, torch.device("cpu"))
    value = bench.job_throughput(w, 1_000_000_000, ms)
    bench.barrier(w)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms": ms, "value": value}, f)
    torch.distributed.destroy_process_group()


def test_barrier_and_max_over_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # both ranks see the max (rank 1's 3.5 ms) and the whole-job throughput
    # counts both replicas' bytes over that time
    for g in got:
        assert g["ms"] == 3.5
        assert g["value"] == pytest.approx(2 * 1e9 / 3.5e-3 / 1e9)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        w, r, local = bench.dist_setup(types.SimpleNamespace(impl="ours"))
        assert (w, r, local) == (1, 0, 0)
        assert not torch.distributed.is_initialized()
        assert bench.reduce_max(2.0, 1, torch.device("cpu")) == 2.0
        bench.barrier(1)
    finally:
        os.environ.update(env)


@pytest.mark.parametrize("workload,metric", [("gqa_bf16", "paged decode attention KV GB/s"),
                                             ("block_copy", "block copy GB/s")])
def test_reference_arm_under_torchrun_two_ranks(workload, metric):
    """`bench.py --impl reference` launched as an N = 2 run is launched:
    rank 0 alone times the oracle and prints one JSON line; rank 1 exits 0
    without output."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "3", "--ref-budget", "0.05", "--workload", workload]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["metric"] == metric and d["config"]["workload"] == workload
