"""The N > 1 benchmark path on CPU: two gloo ranks.

Each rank runs its own batch (weak scaling, replicated experts, no collective
on the data path); the step time is the max over ranks and the token count the
sum.  This checks that host logic without a GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        w = synth.WORKLOADS["switch_base"].scaled(T=64, d_model=64, d_ff=64, E=16)
        inp = synth.layer_inputs(w, x_seed_offset=rank)
        t_ms = 10.0 + 5.0 * rank  # a slower rank 1
        mx = bench.max_over_ranks(t_ms, world, device="cpu")
        tok = bench.sum_over_ranks(float(w.T), world, device="cpu")
        xs = [torch.empty_like(inp["x"]) for _ in range(world)]
        dist.all_gather(xs, inp["x"])
        w1 = [torch.empty_like(inp["W1"]) for _ in range(world)]
        dist.all_gather(w1, inp["W1"])
        q.put((rank, mx, tok, bool(torch.equal(xs[0], xs[1])), bool(torch.equal(w1[0], w1[1]))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, tok, same_x, same_w in res:
        assert mx == 15.0          # max over ranks
        assert tok == 128.0        # tokens of all ranks
        assert not same_x          # each rank has its own batch
        assert same_w              # experts are replicated


def _ep_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_mixture_experts_fwd_b200.ep import exchange_counts, rank_barrier
        E = 12
        kept_cnt = (torch.arange(E, dtype=torch.int32) * (rank + 1)) % 7
        out = torch.full((world, E), -1, dtype=torch.int32)
        cnt_all = exchange_counts(kept_cnt, world, out=out)
        token = torch.zeros(1, dtype=torch.int32)
        rank_barrier(token)
        # the host-ordered form (gloo groups, ranks sharing a GPU): CPU all-gather
        out_h = torch.full((world, E), -1, dtype=torch.int32)
        cnt_h = exchange_counts(kept_cnt, world, out=out_h, host=True)
        rank_barrier(token, host=True)
        q.put((rank, cnt_all.data_ptr() == out.data_ptr(), cnt_all.tolist(), int(token.item()),
               cnt_h.tolist(), cnt_h.data_ptr() == out_h.data_ptr()))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_count_exchange_gloo():
    """The expert-parallel host plumbing on two gloo ranks: every rank gets
    every rank's kept counts in rank order (in the caller's buffer), and the
    barrier's token stays zero."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [[(e * (r + 1)) % 7 for e in range(12)] for r in range(world)]
    for rank, in_place, cnt_all, token, cnt_h, in_place_h in res:
        assert in_place and in_place_h
        assert cnt_all == want and cnt_h == want
        assert token == 0
