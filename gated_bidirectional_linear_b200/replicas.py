"""Host side of the benchmark's multi-GPU mode: independent replicas.

The operator has no data-path exchange: heads, batch elements and calls are
independent, so N GPUs run N replicas of the workload, one per rank, each on
its own seeded inputs.  Only the measurement needs the process group: every
rank enters and leaves the timed region together (a barrier and a device
synchronisation on each side), and the reported time is the maximum over
ranks.  The functions take the process group module (torch.distributed, or
None for one process) and work with any backend: NCCL on the GPUs, gloo in
the CPU tests.
"""
import time

import torch


def replica_seed(base_seed, rank):
    """Seed of rank `rank`'s inputs: each replica works on its own data."""
    return base_seed + rank


def max_over_ranks(value, dist, device="cpu"):
    """The maximum of a per-rank float over all ranks (the value itself for
    one process).  `device` holds the reduction tensor: the GPU for NCCL."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class CpuTimer:
    """Wall-clock timer with the interface of a device timer (for tests)."""

    def start(self):
        self.t0 = time.perf_counter()

    def stop(self):
        self.t1 = time.perf_counter()

    def elapsed_ms(self):
        return (self.t1 - self.t0) * 1e3


class CudaTimer:
    """CUDA events recorded on the stream the timed work is launched on."""

    def __init__(self, stream):
        self.stream = stream
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def start(self):
        self.e0.record(self.stream)

    def stop(self):
        self.e1.record(self.stream)

    def elapsed_ms(self):
        return self.e0.elapsed_time(self.e1)


def timed(run, timer, dist=None, sync=None, device="cpu"):
    """Runs `run()` once inside the timed region and returns its duration in
    ms, the maximum over ranks: barrier, sync, start, run, stop, sync,
    barrier.  `sync` waits for the device (torch.cuda.synchronize)."""
    if dist is not None:
        dist.barrier()
    if sync is not None:
        sync()
    timer.start()
    run()
    timer.stop()
    if sync is not None:
        sync()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(timer.elapsed_ms(), dist, device)


def aggregate_rate(world, units_per_step, steps, ms):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank does one replica's work)."""
    return world * units_per_step * steps / (ms / 1e3)
