"""Multi-rank host logic on CPU (gloo, world size 2): each rank routes its own
BH units with the random draws keyed by the global unit index, so the ranks
together reproduce one joint run exactly; the step time reported is the
slowest rank's and the counts are summed over the ranks.  Uses the oracle as
the router (no GPU)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(w, world, layers):
    g = torch.Generator().manual_seed(1234)
    return [(torch.randn((w.bh * world, w.n, w.d), generator=g).numpy().astype(np.float32),
             torch.randn((w.bh * world, w.n, w.d), generator=g).numpy().astype(np.float32))
            for _ in range(layers)]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import rr_workloads as W
        w = W.PR1.with_(bh=2, n=40, d=8, k=4, m=3, r=3, anchor_interval=3)
        off = bench.shard_offset(rank, w)
        p = oracle.Params(nq=w.n, nk=w.n, d=w.d, k=w.k, m=w.m, r=w.r, causal=True, seed=77)
        rt = oracle.Router(p, bh=w.bh, anchor_interval=w.anchor_interval, bh_offset=off)
        for l, (q, k) in enumerate(_inputs(w, world, 4)):
            rt.step(l, q[off:off + w.bh], k[off:off + w.bh], recall=False)
        mine = np.stack([led.ids for led in rt.ledgers])
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        slowest = bench.max_over_ranks(10.0 + rank, world)
        totals = bench.sum_over_ranks([1.0 + rank, 100.0 * rank], world)
        if rank == 0:
            out.put((np.concatenate(parts), slowest, totals))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_joint_run_and_report_the_slowest():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for pr in procs:
        pr.start()
    joint_ids, slowest, totals = out.get(timeout=120)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    import oracle
    import rr_workloads as W
    w = W.PR1.with_(bh=2, n=40, d=8, k=4, m=3, r=3, anchor_interval=3)
    p = oracle.Params(nq=w.n, nk=w.n, d=w.d, k=w.k, m=w.m, r=w.r, causal=True, seed=77)
    rt = oracle.Router(p, bh=w.bh * world, anchor_interval=w.anchor_interval)
    for l, (q, k) in enumerate(_inputs(w, world, 4)):
        rt.step(l, q, k, recall=False)
    assert np.array_equal(joint_ids, np.stack([led.ids for led in rt.ledgers]))
    assert slowest == 11.0
    assert totals == [3.0, 100.0]
