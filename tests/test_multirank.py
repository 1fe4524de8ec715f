"""Multi-rank host logic of the benchmark on CPU (world size 2, gloo).

On the GPU pool each rank runs its own batch of the workload on its own GPU
with no collective on the data path (weak scaling); the job's step time is
the maximum over ranks.  This checks that plumbing without a GPU: distinct
per-rank inputs, the max reduction, and the whole-job throughput.
"""

import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    from synth import WORKLOADS, make_shape_inputs
    r, wsize, local = bench.dist_setup(world, backend="gloo")
    assert (r, wsize, local) == (rank, world, rank)
    w = WORKLOADS["mha_causal_fwdbwd"]
    seed = bench.rank_seed(w, r)
    x = make_shape_inputs(1, 2, 2, 16, 16, 64, seed=seed)
    local_ms = 10.0 + 5.0 * r  # rank 1 is slower
    ms = bench.max_over_ranks(local_ms, wsize, device="cpu")
    value = bench.job_throughput(wsize, 1e12, ms)
    t = torch.tensor([float(x["q"].astype("int64").sum())])
    gathered = [torch.zeros(1) for _ in range(wsize)]
    dist.all_gather(gathered, t)
    out[r] = (ms, value, [float(g.item()) for g in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_host_logic():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms, value, sums = out[r]
        assert ms == 15.0                      # max over ranks
        assert abs(value - 2 * 1e12 / 15e-3 / 1e12) < 1e-9
        assert sums[0] != sums[1]              # each rank drew its own batch
