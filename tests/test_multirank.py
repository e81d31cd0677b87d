"""The N > 1 host path of the benchmark on the CPU with the gloo backend (world size
2): each rank draws its own replica (independent heads, so no data-path collective),
the job time is the maximum over ranks, and the throughput counts the work of all
ranks. The attention itself runs on GPUs only; here each rank's step is timed as a
plain sleep of a rank-dependent length."""
import os
import socket
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from io_aware_attention_flashattention_b200.inputs import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = WORKLOADS["oracle_f32_n256_d64"]
        q, _, _, _ = make_inputs(1, 1, 8, 64, torch.float32, bench.replica_seed(w, rank))
        gathered = [torch.empty_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        t0 = time.perf_counter()
        time.sleep(0.05 * (rank + 1))  # rank 1 is the slow one
        local_ms = (time.perf_counter() - t0) * 1e3
        job_ms = bench.max_over_ranks(local_ms, world)
        out[rank] = (local_ms, job_ms, bool(torch.equal(gathered[0], gathered[1])),
                     bench.job_throughput(1e12, world, 10, job_ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    local0, job0, same0, thr0 = res[0]
    local1, job1, same1, thr1 = res[1]
    assert not same0 and not same1, "ranks must draw different replicas"
    assert job0 == job1 == pytest.approx(max(local0, local1))
    assert job0 >= local0 and job1 >= 99.0
    # 2 ranks x 10 steps x 1 TFLOP in the slowest rank's time
    assert thr0 == pytest.approx(2 * 10 * 1.0 / (job0 * 1e-3))


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(2e12, 1, 5, 1000.0) == pytest.approx(10.0)
    w = WORKLOADS["long_b1h8_n16384_d128"]
    assert bench.replica_seed(w, 0) == w.seed and bench.replica_seed(w, 3) != w.seed
