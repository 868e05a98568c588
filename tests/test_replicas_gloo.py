"""Multi-process (world size 2, gloo, CPU) checks of the benchmark's replica
plumbing: the path shards into independent replicas with no data-path
collective, so the only cross-rank steps are the timing barrier and the
max-over-ranks reduction of the timed duration."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    barrier = bench.make_barrier(w, torch.device("cpu"))
    barrier()
    local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    t_max = bench.max_over_ranks(local_ms, w, torch.device("cpu"))
    barrier()
    out[rank] = (t_max, bench.replica_value(1e12, 4, w, t_max))
    torch.distributed.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0                      # max over ranks, seen by every rank
    # 2 ranks x 4 steps x 1e12 FLOP in 15 ms
    assert res[0][1] == pytest.approx(2 * 4 * 1e12 / 15e-3 / 1e12)


def test_replica_value_single_rank():
    assert bench.replica_value(2e12, 10, 1, 20.0) == pytest.approx(1000.0)


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    class A:
        workload, steps, warmup, gpus = "tiny", 1, 0, 2
    assert bench.run_reference(A, world=2, rank=1) is None


@pytest.mark.parametrize("workload", ["tiny", "ffn", "moe_tokens"])
def test_reference_arm_line_on_rank_zero(workload):
    # the reference arm is the CPU oracle on a bounded sample of the workload;
    # its line carries the contract's keys and a cpu_baseline describing itself
    class A:
        steps, warmup, gpus = 2, 1, 1
        x_fmt, weight_scales = "e4m3", "channel"
    A.workload = workload
    line = bench.run_reference(A, world=1, rank=0)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith(bench.workload_spec(workload)[0][:10])
