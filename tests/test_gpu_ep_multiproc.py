"""Expert parallelism across processes: two ranks, each its own process on the
same GPU, in a gloo group.

What this covers that the one-process tests cannot: the receive buffers are
mapped between processes with CUDA IPC handles (``map_peer_buffers``), so the
dispatch kernel's stores and the combine kernel's loads go through another
process's mapping, and the system-scope fence after the dispatch copy is seen
from another process.  The steps are ordered from the host
(``ExpertParallelLayer(sync="host")``: each barrier is a device synchronise
plus a gloo barrier, counts travel as CPU tensors), so no kernel ever waits on
the other process.  Each rank's output is checked against the oracle's
single-device layer on that rank's batch (the Switch notes, sec. 2 opening:
the experts' weights on different devices, each rank routing its own batch).
"""
import os
import socket
import traceback

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

CASES = {
    # name: (T, d, f, E, k, capacity_factor, mode, G, expert)
    "top2": (600, 128, 256, 8, 2, 1.25, "topk", 1, "relu"),
    "top1_pairs": (2200, 64, 128, 4, 1, 1.0, "topk", 1, "relu"),  # world * C = 1100: SM pairs
    "rre": (900, 128, 256, 8, 1, 1.5, "rre", 2, "relu"),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, name, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        try:
            import oracle
            import sparse_mixture_experts_fwd_b200 as moe
            import synth
            from sparse_mixture_experts_fwd_b200.ep import ExpertParallelLayer

            T, d, f, E, k, cf, mode, G, expert = CASES[name]
            w = synth.Workload(name, T=T, d_model=d, d_ff=f, E=E, k=k, capacity_factor=cf,
                               dtype="bf16", mode=mode, num_groups=G, expert=expert, seed=7)
            inp = synth.layer_inputs(w, x_seed_offset=rank)  # each rank its own batch
            C = moe.capacity(T, E, cf)
            cfg = moe.make_config(T, d, f, E, k, C, dtype=torch.bfloat16, mode=mode,
                                  num_groups=G, seed=w.seed, expert=expert)
            dev = torch.device("cuda", 0)
            El = E // world
            layer = ExpertParallelLayer(cfg, sync="host")
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            x = inp["x"].to(dev)
            W1 = inp["W1"][rank * El:(rank + 1) * El].contiguous().to(dev)
            W2 = inp["W2"][rank * El:(rank + 1) * El].contiguous().to(dev)
            kw = dict(Wr=None if inp["Wr"] is None else inp["Wr"].to(dev),
                      bias=None if inp["bias"] is None else inp["bias"].to(dev),
                      domain_id=None if inp["domain"] is None else inp["domain"].to(dev))
            ys = []
            for _ in range(2):  # two steps: the buffers are reused across steps
                ys.append(layer.forward(x, W1, W2, status=status, **kw).clone())
                torch.cuda.synchronize()
                dist.barrier()
            ref = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=E, k=k, C=C,
                                       Wr=inp["Wr"], bias=inp["bias"], domain=inp["domain"],
                                       G=G, seed=w.seed, kind=expert)
            errs = []
            for y in ys:
                g, r = y.cpu().double(), ref["y"].double()
                bad = (g - r).abs() > 2e-2 + 1e-2 * r.abs()
                errs.append((int(bad.sum()), float((g - r).abs().max())))
            q.put((rank, int(status.item()), errs, None))
            del layer
            torch.cuda.synchronize()
            dist.barrier()
        finally:
            dist.destroy_process_group()
    except Exception:  # report to the parent instead of hanging it
        q.put((rank, -1, [], traceback.format_exc()))


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_parallel_two_processes(cuda_device, name):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
    for rank, status, errs, tb in sorted(res):
        assert tb is None, f"rank {rank}:\n{tb}"
        assert status == 0, f"rank {rank}: device status {status}"
        for step, (n_bad, max_err) in enumerate(errs):
            assert n_bad == 0, f"rank {rank} step {step}: {n_bad} outputs out of tolerance " \
                               f"(max |dy| {max_err:.3e})"
    for p in procs:
        assert p.exitcode == 0
