"""The N > 1 path of bench.py on CPU: two gloo ranks, each a replica.

Every rank builds its own plan from the same tables (the plan is a pure host
function, so all ranks get identical work lists) and reports a time; the job
value takes the slowest rank's time and all ranks' bytes (weak scaling).
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from serving_attention_paged_b200 import workloads as W
        w = W.WORKLOADS[3]()
        q, items, ci, mi = oracle.plan(w.kv_indptr, w.last_page_len, page_size=16,
                                       num_kv_heads=8, num_sms=148, ctas_per_sm=3)
        digest = torch.tensor([int(items.sum()), len(items), int(ci[-1])], dtype=torch.int64)
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms, "cpu")
        value = bench.aggregate_gbs(world, w.kv_bytes(), ms * 1e-3)
        out[rank] = (ms, value, all(torch.equal(g, gathered[0]) for g in gathered))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    from serving_attention_paged_b200 import workloads as W
    nbytes = W.WORKLOADS[3]().kv_bytes()
    for rank in range(world):
        ms, value, same_plan = res[rank]
        assert same_plan
        assert ms == 15.0  # max over ranks
        assert abs(value - world * nbytes / 15e-3 / 1e9) < 1e-9
