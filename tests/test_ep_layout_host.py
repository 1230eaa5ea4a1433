"""The expert-parallel contract on CPU, with the oracle standing in for every kernel.

The C header defines where each kept row of each rank lands on its home rank:
expert e lives on rank h = e / (E/world) in block e - h*E/world of a
[E/world, world*C, d] buffer, rank q's rows of e at offset
off_q(e) = sum over q' < q of rank q''s kept count of e, in slot order.  This
packs every rank's oracle dispatch that way, runs the oracle's expert FFN on
each home rank's packed block (capacity world*C, counts summed over ranks),
reads each rank's expert outputs back through the same offsets and combines
them with the oracle.  Because the expert network acts row by row, every
rank's output must equal the oracle's single-device layer on that rank's
batch bit for bit: the claim the expert-parallel path rests on.
"""
import pytest
import torch

import oracle
import synth


def _pack_unpack_layer(w, world):
    E, k = w.E, w.k
    El = E // world
    full = synth.layer_inputs(w)
    C = oracle.capacity(w.T, E, w.capacity_factor)
    ranks = []
    for q in range(world):
        inp = synth.layer_inputs(w, weights=False, x_seed_offset=q)
        ref = oracle.layer_forward(inp["x"], full["W1"], full["W2"], E=E, k=k, C=C, Wr=full["Wr"],
                                   bias=full["bias"], domain=inp["domain"], G=w.num_groups,
                                   seed=w.seed, kind=w.expert)
        ranks.append(ref)
    cnt = torch.stack([r["kept_cnt"] for r in ranks]).long()          # [world, E]
    off = torch.cumsum(cnt, 0) - cnt                                   # off[q, e]
    PC, d = world * C, w.d_model
    # pack: home rank h, block el, rows off[q, e] .. off[q, e] + cnt[q, e] - 1
    xe_home = [torch.zeros(El, PC, d, dtype=w.torch_dtype) for _ in range(world)]
    for q, r in enumerate(ranks):
        for e in range(E):
            h, el, n = e // El, e % El, int(cnt[q, e])
            o = int(off[q, e])
            xe_home[h][el, o:o + n] = r["xe"][e, :n]
    # each home rank runs its experts over everything it received
    ye_home = []
    for h in range(world):
        local = cnt[:, h * El:(h + 1) * El].sum(0).to(torch.int32)
        W1 = full["W1"][h * El:(h + 1) * El].contiguous()
        W2 = full["W2"][h * El:(h + 1) * El].contiguous()
        ye_home.append(oracle.expert_ffn(xe_home[h], W1, W2, local, kind=w.expert))
    # unpack each rank's rows to its own [E, C, d] view and combine
    outs = []
    for q, r in enumerate(ranks):
        ye = torch.zeros(E, C, d, dtype=w.torch_dtype)
        for e in range(E):
            h, el, n = e // El, e % El, int(cnt[q, e])
            o = int(off[q, e])
            ye[e, :n] = ye_home[h][el, o:o + n]
        outs.append(oracle.combine(ye, r["expert_idx"], r["gate"], r["slot"], r["kept"], w.T))
    return ranks, outs, cnt, PC


CASES = [
    ("top1", 2, dict(T=300, d_model=64, d_ff=64, E=8, k=1, capacity_factor=1.0)),
    ("top2", 4, dict(T=200, d_model=32, d_ff=64, E=16, k=2, capacity_factor=1.25)),
    ("rre", 2, dict(T=256, d_model=32, d_ff=32, E=8, k=1, capacity_factor=1.0, mode="rre",
                    num_groups=2)),
    ("geglu_top2", 2, dict(T=160, d_model=64, d_ff=32, E=4, k=2, capacity_factor=1.0,
                           expert="geglu", expert_std=0.1)),
    ("fp32_one_expert_per_rank", 4, dict(T=128, d_model=16, d_ff=32, E=4, k=1,
                                         capacity_factor=1.5, dtype="f32")),
    ("hot_expert", 2, dict(T=200, d_model=32, d_ff=32, E=8, k=1, capacity_factor=1.0,
                           hot_experts=1, hot_bias=100.0)),
]


@pytest.mark.parametrize("name,world,kw", CASES, ids=[c[0] for c in CASES])
def test_packed_expert_parallel_layer_equals_single_device(name, world, kw):
    base = dict(dtype="bf16", mode="topk", num_groups=1, seed=4)
    base.update(kw)
    w = synth.Workload(name, **base)
    ranks, outs, cnt, PC = _pack_unpack_layer(w, world)
    El = w.E // world
    for q, (r, y) in enumerate(zip(ranks, outs)):
        a, b = (y.view(torch.int16), r["y"].view(torch.int16)) if w.dtype == "bf16" else (y, r["y"])
        assert torch.equal(a, b), f"rank {q}"
    # every home block holds at most world * C rows, and the counts add up
    for h in range(world):
        assert int(cnt[:, h * El:(h + 1) * El].sum(0).max()) <= PC
    assert int(cnt.sum()) == sum(int(r["kept"].sum()) for r in ranks)
