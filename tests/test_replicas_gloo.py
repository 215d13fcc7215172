"""The benchmark's multi-GPU mode on CPU: two gloo ranks run the replica
plumbing (seeds, the timed region with its barriers, max over ranks, the
whole-job rate) that bench.py runs over NCCL on the GPUs."""
import json
import os
import socket
import time

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_bidirectional_linear_b200 import replicas, workloads

WORLD = 2


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        seed = replicas.replica_seed(5, rank)
        # This rank's replica input: the same workload shape, its own draw.
        wl = workloads.WORKLOADS["tiny"]
        x = workloads.make_inputs(wl, seed=seed)
        # Rank 1 is the slower one; both must report its time.
        sleep_s = 0.05 * (rank + 1)
        ms = replicas.timed(lambda: time.sleep(sleep_s), replicas.CpuTimer(), dist)
        rate = replicas.aggregate_rate(WORLD, wl.batch * wl.tokens, 4, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"seed": seed, "ms": ms, "rate": rate,
                       "q_sum": float(x["q"].double().sum())}, f)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("replicas")
    mp.start_processes(rank_main, args=(free_port(), str(out)), nprocs=WORLD,
                       start_method="spawn", join=True)
    return [json.load(open(out / f"rank{r}.json")) for r in range(WORLD)]


def test_every_rank_reports_the_slowest_time(results):
    ms = [r["ms"] for r in results]
    assert ms[0] == ms[1]
    assert ms[0] >= 100.0          # rank 1 slept 0.1 s inside the region


def test_replicas_draw_their_own_inputs(results):
    assert results[0]["seed"] != results[1]["seed"]
    assert results[0]["q_sum"] != results[1]["q_sum"]


def test_whole_job_rate_counts_every_rank(results):
    wl = workloads.WORKLOADS["tiny"]
    r = results[0]
    assert r["rate"] == pytest.approx(WORLD * wl.batch * wl.tokens * 4 / (r["ms"] / 1e3))
    assert results[1]["rate"] == r["rate"]


def test_single_process_needs_no_group():
    assert replicas.max_over_ranks(3.5, None) == 3.5
    ms = replicas.timed(lambda: time.sleep(0.01), replicas.CpuTimer())
    assert ms >= 10.0
