"""Helpers shared by the GPU parity tests: oracle references per workload,
tolerance checks and the margin rule for end-to-end routing."""
from __future__ import annotations

import functools
import os

import torch

import oracle
import synth

# Output tolerance for bf16 activations: |gpu - ref| <= ATOL + RTOL * |ref| per element.
ATOL, RTOL = 2e-2, 1e-2
# fp32 gates and the SparseClip norm: relative 1e-5.
GATE_RTOL = 1e-5
# End-to-end routing may differ only where adjacent sorted top-(k+1) logits are this close.
MARGIN = 1e-5


def assert_close(gpu, ref, atol=ATOL, rtol=RTOL, what="output"):
    g = gpu.detach().cpu().double()
    r = ref.detach().cpu().double()
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = (g - r).abs()
    bound = atol + rtol * r.abs()
    bad = err > bound
    if bool(bad.any()):
        i = int(torch.nonzero(bad.flatten())[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.numel()} elements out of "
                             f"tolerance; first at flat index {i}: gpu={g.flatten()[i].item()} "
                             f"ref={r.flatten()[i].item()}; max err {err.max().item():.3e}")
    return float(err.max()) if err.numel() else 0.0


def margin_exempt(logits: torch.Tensor, k: int) -> torch.Tensor:
    """Tokens whose sorted top-(k+1) fp32 oracle logits have an adjacent gap < MARGIN."""
    top = torch.topk(logits.double(), min(k + 1, logits.shape[1]), dim=1).values
    if top.shape[1] < 2:
        return torch.zeros(logits.shape[0], dtype=torch.bool)
    gaps = top[:, :-1] - top[:, 1:]
    return (gaps < MARGIN).any(dim=1)


def threads():
    return max(1, os.cpu_count() or 1)


@functools.lru_cache(maxsize=1)
def workload_case(name: str, T: int | None = None):
    """CPU inputs of a workload (optionally with fewer tokens) and the oracle's
    routing reference (router logits, gates, expert choice, slot assignment)."""
    w = synth.WORKLOADS[name]
    if T is not None:
        w = w.scaled(T=T)
    inp = synth.layer_inputs(w)
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    ref = {"C": C}
    if w.mode == "topk":
        ref["logits"] = oracle.router(inp["x"], inp["Wr"], inp["bias"], nthreads=threads())
        ref["expert_idx"], ref["gate"] = oracle.gate_topk(ref["logits"], w.k)
    else:
        ref["expert_idx"], ref["gate"] = oracle.route_rre(inp["domain"], w.E, w.num_groups, w.seed)
    ref.update(oracle.assign(ref["expert_idx"], w.E, C))
    return w, inp, ref


def to_dev(t, dev):
    return None if t is None else t.to(dev)
