"""The multi-rank plumbing of bench.py on CPU with the gloo backend (2 ranks):
every rank draws its own replica of the workload (weak scaling), and the
reported time is the max over ranks, the aggregate bandwidth the sum.  No GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    from query_adaptive_chunk_b200 import synth
    try:
        w_env, r_env, l_env = bench.dist_env()
        assert (w_env, r_env, l_env) == (world, rank, rank)
        bench.dist_init(world, "gloo")
        w = bench.rank_workload(synth.TOPK_32K.scaled(B=1, T=2048), rank)
        inp = synth.make_decode_inputs(w, device="cpu")
        qsum = float(inp["q"].float().sum())
        # distinct replicas per rank
        allq = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allq, torch.tensor([qsum], dtype=torch.float64))
        mx = bench.dist_max(10.0 + rank, world, "cpu")
        sm = bench.dist_sum(1.5 * (rank + 1), world, "cpu")
        q.put((rank, [float(x) for x in allq], mx, sm, w.seed))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_replicas_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, qs0, mx0, sm0, seed0), (_, qs1, mx1, sm1, seed1) = res
    assert qs0 == qs1 and qs0[0] != qs0[1]  # each rank drew its own replica
    assert seed0 != seed1
    assert mx0 == mx1 == 11.0  # max over ranks
    assert sm0 == sm1 == 1.5 + 3.0  # aggregate
