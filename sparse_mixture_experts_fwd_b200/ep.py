"""Expert parallelism over the GPUs of one node: the process-group plumbing.

One process per GPU.  Each rank holds E / world experts (the sparse layer's
distinct weights placed on different devices, Switch notes sec. 2, opening
paragraph) and routes its own batch.  The library's kernels move the rows:
``moe_ep_dispatch`` stores each kept row into its home rank's receive buffer
through the peer mapping (NVLink stores) and ``moe_ep_combine`` loads the
expert outputs back the same way.  This module supplies what those kernels
need from ``torch.distributed``:

* every rank's receive buffers mapped into this process (CUDA IPC handles
  exchanged once over the process group);
* the per-step all-gather of the kept counts (``cnt_all``);
* the barriers that order dispatch -> expert FFN -> combine across ranks
  (a one-word all-reduce; on NCCL it is ordered on the current stream, so
  the host never waits).

``sync="host"`` orders the steps from the host instead, for process groups
whose backend cannot order work on a CUDA stream (gloo): each barrier is a
``torch.cuda.synchronize()`` followed by a group barrier, and the kept counts
travel as CPU tensors.  No kernel then ever waits for another process, which
also lets several ranks share one GPU.

Each rank's output equals the single-device layer on that rank's batch: the
capacity C applies per batch and expert e's buffer on its home rank holds the
world * C rows its senders may keep.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (ROUTE_TOPK, _act_dtype, assign_workspace_size, ep_combine,
               ep_dispatch, ep_ffn_config, expert_ffn, ffn_workspace_size, router, topk_assign)


def exchange_counts(kept_cnt: torch.Tensor, world: int, group=None, out=None,
                    host: bool = False) -> torch.Tensor:
    """cnt_all [world, E]: row q = rank q's kept counts (an all-gather).

    ``host``: gather CPU copies (after the counts are final) and copy the
    result into ``out`` (or a new tensor on the counts' device)."""
    E = kept_cnt.numel()
    if host:
        parts = [torch.empty(E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(parts, kept_cnt.detach().to("cpu", torch.int32).view(-1), group=group)
        full = torch.stack(parts)
        if out is None:
            return full.to(kept_cnt.device)
        out.view(world, E).copy_(full)
        return out.view(world, E)
    flat = out.view(-1) if out is not None else torch.empty(world * E, dtype=torch.int32,
                                                            device=kept_cnt.device)
    dist.all_gather_into_tensor(flat, kept_cnt.contiguous().view(-1), group=group)
    return flat.view(world, E)


def rank_barrier(token: torch.Tensor, group=None, host: bool = False) -> None:
    """Every rank's work enqueued before this call completes before any
    rank's work enqueued after it (``token``: a zero word, kept zero).
    ``host``: wait for this process's GPU work, then meet the other ranks."""
    if host:
        if torch.cuda.is_initialized():  # a process that never used CUDA has nothing to wait for
            torch.cuda.synchronize()
        dist.barrier(group=group)
        return
    dist.all_reduce(token, group=group)


def map_peer_buffers(buf: torch.Tensor, group=None):
    """Device addresses of every rank's ``buf`` in this process, rank order,
    and the opened storages that keep the mappings alive."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if world == 1:
        return [buf.data_ptr()], []
    share = buf.untyped_storage()._share_cuda_()
    entry = (share, buf.storage_offset() * buf.element_size())
    entries = [None] * world
    dist.all_gather_object(entries, entry, group=group)
    addrs, keep = [], []
    for q, (sh, off) in enumerate(entries):
        if q == rank:
            addrs.append(buf.data_ptr())
            continue
        st = torch.UntypedStorage._new_shared_cuda(*sh)
        keep.append(st)
        addrs.append(st.data_ptr() + off)
    return addrs, keep


class ExpertParallelLayer:
    """One MoE layer with its experts split over the ranks of ``group``.

    ``cfg`` describes the whole layer on one rank's batch (global E, the
    rank's T and capacity C); ``forward`` takes this rank's expert shards
    W1 [E/world, f (2f for GEGLU), d] and W2 [E/world, d, f]."""

    def __init__(self, cfg, group=None, device=None, sync: str = "stream"):
        if sync not in ("stream", "host"):
            raise ValueError('sync must be "stream" or "host"')
        self.host_sync = sync == "host"
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.cfg = cfg
        self.ffn_cfg = ep_ffn_config(cfg, self.world)
        dev = (torch.device("cuda", torch.cuda.current_device()) if device is None
               else torch.device(device))
        dt = _act_dtype(cfg)
        El, PC, d, f = self.ffn_cfg.E, self.ffn_cfg.capacity, cfg.d_model, cfg.d_ff
        self.xe = torch.empty(El, PC, d, dtype=dt, device=dev)
        self.ye = torch.empty(El, PC, d, dtype=dt, device=dev)
        self.H = torch.empty(El, PC, f, dtype=dt, device=dev)
        self.ffn_ws = torch.empty(max(256, ffn_workspace_size(self.ffn_cfg)), dtype=torch.uint8,
                                  device=dev)
        self.assign_ws = torch.empty(max(256, assign_workspace_size(cfg)), dtype=torch.uint8,
                                     device=dev)
        self.logits = (torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)
                       if cfg.mode == ROUTE_TOPK else None)
        T, k, E, C = cfg.T, cfg.k, cfg.E, cfg.capacity
        self.route = {
            "expert_idx": torch.empty(T, k, dtype=torch.int32, device=dev),
            "gate": torch.empty(T, k, dtype=torch.float32, device=dev),
            "slot": torch.empty(T, k, dtype=torch.int32, device=dev),
            "kept": torch.empty(T, k, dtype=torch.uint8, device=dev),
            "tok_of_row": torch.empty(max(1, E * C), dtype=torch.int32, device=dev),
            "arrivals": torch.empty(E, dtype=torch.int32, device=dev),
            "kept_cnt": torch.empty(E, dtype=torch.int32, device=dev),
            "n_dropped": torch.empty(1, dtype=torch.int32, device=dev),
        }
        self.cnt_all = torch.empty(self.world, cfg.E, dtype=torch.int32, device=dev)
        self.local_cnt = torch.empty(El, dtype=torch.int32, device=dev)
        self.token = torch.zeros(1, dtype=torch.int32, device=dev)
        self.xe_peers, self._xe_keep = map_peer_buffers(self.xe, group)
        self.ye_peers, self._ye_keep = map_peer_buffers(self.ye, group)

    def forward(self, x, W1_local, W2_local, *, Wr=None, bias=None, domain_id=None, y=None,
                status=None):
        cfg, rank, world, g = self.cfg, self.rank, self.world, self.group
        if cfg.mode == ROUTE_TOPK:
            router(cfg, x, Wr, bias, logits=self.logits, status=status)
        r = topk_assign(cfg, logits=self.logits, domain_id=domain_id, out=self.route,
                        workspace=self.assign_ws, status=status)
        hs = self.host_sync
        exchange_counts(r["kept_cnt"], world, g, out=self.cnt_all, host=hs)
        ep_dispatch(cfg, rank, world, x, r["expert_idx"], r["slot"], r["kept"], self.cnt_all,
                    self.xe_peers, local_cnt=self.local_cnt, status=status)
        rank_barrier(self.token, g, host=hs)  # every rank's rows have landed
        expert_ffn(self.ffn_cfg, self.xe, W1_local, W2_local, self.local_cnt, H=self.H, ye=self.ye,
                   workspace=self.ffn_ws, status=status)
        rank_barrier(self.token, g, host=hs)  # every rank's expert outputs are written
        y = ep_combine(cfg, rank, world, self.ye_peers, r["expert_idx"], r["gate"], r["slot"],
                       r["kept"], self.cnt_all, y=y, status=status)
        return y

    __call__ = forward


__all__ = ["exchange_counts", "rank_barrier", "map_peer_buffers", "ExpertParallelLayer"]
