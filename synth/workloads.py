"""The five layer workloads and their input recipe.

Shapes and value distributions follow the workload list this library is
measured on (a tiny fp32 Switch layer, a Switch-Base-shaped layer, an X-MoE
top-2 layer with a SparseClip norm, a PanGu-Sigma RRE layer and a large skewed
Switch layer).  Readings of the recipe's notation:

* ``W_r ~ N(0, 1/d_model)`` is a variance: std = 1/sqrt(d_model), so logits
  are roughly N(0, 1).
* expert weights ``~ N(0, 0.02)`` and gradients ``~ N(0, 1e-3)`` are stds.
* the skewed layer's 16 hot experts are experts 0..15; their +2.0 enters as a
  per-expert fp32 bias added to the router logits.
* RRE domain ids come from their own stream (tag ``domain``), independent of
  the routing hash.

Each tensor is its own generator stream (``TAGS``); the value at flat index i
of a tensor is draw #i of that stream, so a slice can be generated alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

from .gen import normal, uniform_int

TAGS = {
    "x": 1,
    "Wr": 2,
    "W1": 3,
    "W2": 4,
    "domain": 5,
    "g_dense": 6,
    "g_sparse": 7,  # segment s uses tag 7 + 16 * (s + 1)
}


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int
    capacity_factor: float
    dtype: str  # "f32" or "bf16": activations and weights
    mode: str = "topk"  # "topk" (softmax gate + top-k) or "rre"
    expert: str = "relu"  # "relu" FFN (W1 [E, f, d]) or "geglu" (W1 [E, 2f, d])
    num_groups: int = 1
    hot_experts: int = 0
    hot_bias: float = 0.0
    seed: int = 0
    x_std: float = 1.0
    expert_std: float = 0.02
    # SparseClip gradient set that rides with this workload (0 = none)
    clip_dense: int = 0
    clip_sparse_segments: int = 0
    clip_sparse_len: int = 0
    clip_std: float = 1e-3

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def router_std(self) -> float:
        return 1.0 / math.sqrt(self.d_model)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_switch": Workload("tiny_switch", T=256, d_model=64, d_ff=256, E=8, k=1,
                            capacity_factor=1.0, dtype="f32"),
    "switch_base": Workload("switch_base", T=8192, d_model=768, d_ff=3072, E=128, k=1,
                            capacity_factor=1.25, dtype="bf16"),
    "xmoe_top2": Workload("xmoe_top2", T=16384, d_model=1024, d_ff=4096, E=64, k=2,
                          capacity_factor=2.0, dtype="bf16", clip_dense=50_000_000,
                          clip_sparse_segments=64, clip_sparse_len=8_388_608),
    "pangu_rre": Workload("pangu_rre", T=32768, d_model=2560, d_ff=10240, E=64, k=1,
                          capacity_factor=1.25, dtype="bf16", mode="rre", num_groups=8),
    "skewed_switch": Workload("skewed_switch", T=65536, d_model=1024, d_ff=4096, E=256, k=1,
                              capacity_factor=1.0, dtype="bf16", hot_experts=16, hot_bias=2.0),
}


def layer_inputs(w: Workload, *, weights: bool = True, x_seed_offset: int = 0,
                 threads: int | None = None) -> dict:
    """CPU tensors for one layer call.

    Returns ``x [T,d]``, ``Wr [E,d]`` (None for RRE), ``bias [E] f32`` (None
    unless the workload has hot experts), ``domain [T] int32`` (RRE only) and,
    if ``weights``, ``W1 [E,f,d]`` and ``W2 [E,d,f]`` (both K-major).
    ``x_seed_offset`` shifts the seed of ``x`` only (one batch per rank).
    """
    dt = w.torch_dtype
    out = {
        "x": normal(w.seed + x_seed_offset, TAGS["x"], (w.T, w.d_model), w.x_std, dt,
                    threads=threads),
        "Wr": None,
        "bias": None,
        "domain": None,
    }
    if w.mode == "topk":
        out["Wr"] = normal(w.seed, TAGS["Wr"], (w.E, w.d_model), w.router_std, dt, threads=threads)
        if w.hot_experts:
            b = torch.zeros(w.E, dtype=torch.float32)
            b[: w.hot_experts] = w.hot_bias
            out["bias"] = b
    else:
        out["domain"] = uniform_int(w.seed + x_seed_offset, TAGS["domain"], w.T, w.num_groups,
                                    threads=threads)
    if weights:
        rows = 2 * w.d_ff if w.expert == "geglu" else w.d_ff  # GEGLU: gate, linear rows
        out["W1"] = normal(w.seed, TAGS["W1"], (w.E, rows, w.d_model), w.expert_std, dt,
                           threads=threads)
        out["W2"] = normal(w.seed, TAGS["W2"], (w.E, w.d_model, w.d_ff), w.expert_std, dt,
                           threads=threads)
    return out


def expert_weights(w: Workload, e: int, threads: int | None = None):
    """W1[e] and W2[e] alone, generated from their offsets in the full streams."""
    rows = 2 * w.d_ff if w.expert == "geglu" else w.d_ff
    n1, n2 = rows * w.d_model, w.d_ff * w.d_model
    W1 = normal(w.seed, TAGS["W1"], (rows, w.d_model), w.expert_std, w.torch_dtype,
                first=e * n1, threads=threads)
    W2 = normal(w.seed, TAGS["W2"], (w.d_model, w.d_ff), w.expert_std, w.torch_dtype,
                first=e * n2, threads=threads)
    return W1, W2


def sparseclip_inputs(w: Workload, *, dense: int | None = None, segments: int | None = None,
                      seg_len: int | None = None, threads: int | None = None):
    """fp32 gradient tensors: one dense tensor and ``segments`` expert tensors."""
    nd = w.clip_dense if dense is None else dense
    ns = w.clip_sparse_segments if segments is None else segments
    ls = w.clip_sparse_len if seg_len is None else seg_len
    g_dense = [normal(w.seed, TAGS["g_dense"], (nd,), w.clip_std, torch.float32, threads=threads)]
    g_sparse = [normal(w.seed, TAGS["g_sparse"] + 16 * (s + 1), (ls,), w.clip_std, torch.float32,
                       threads=threads) for s in range(ns)]
    return g_dense, g_sparse
