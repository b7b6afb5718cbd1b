"""World-size-2 checks of the benchmark's multi-rank plumbing on CPU (gloo).

Each rank runs its own batch (seed + rank, weak scaling) and the elapsed time
reported is the maximum over ranks; the work is the sum over ranks.  No
collective touches the attention data path.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "BENCH_DIST_BACKEND": "gloo", "CUDA_VISIBLE_DEVICES": ""})
    import bench
    from variable_length_flash_varlen_b200 import workloads
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    t_max = bench.max_over_ranks(1.0 + rank, w)
    total = bench.sum_over_ranks(10.0 * (rank + 1), w)
    bench.barrier(w)
    wl = workloads.named("mha_noncausal", seed=workloads.WORKLOAD_SEEDS["mha_noncausal"] + rank)
    out[rank] = (t_max, total, tuple(wl.lengths_q))
    import torch.distributed as dist
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_max_time_sum_work_distinct_batches():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=100)
        assert p.exitcode == 0
    (t0, s0, l0), (t1, s1, l1) = out[0], out[1]
    assert t0 == t1 == 2.0          # max over ranks
    assert s0 == s1 == 30.0         # work summed over ranks
    assert l0 != l1                 # each rank draws its own batch
