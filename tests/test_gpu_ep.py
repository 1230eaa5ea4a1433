"""Expert parallelism: the EP dispatch / expert FFN / EP combine path against the oracle.

Each test runs every rank of an expert-parallel group on ONE GPU: the ranks'
buffers are separate allocations on the device and each rank's "peer table"
lists them all, so the kernels store and load through the same addressing
they use over NVLink.  The steps run in the order the cross-rank barriers
impose (all dispatches, then all expert FFNs, then all combines), so no
kernel ever waits on another.  The count exchange (an all-gather between
ranks) is a stack of the ranks' kept counts here.

Bar:
  * each rank's output equals the oracle's single-device layer on that rank's
    batch with all E experts (the capacity applies per batch), within the
    layer tolerance; routing bit-exact;
  * receive buffers bit-exact against the packed layout: expert e's block on
    its home rank holds rank 0's kept rows, then rank 1's, ..., each in slot
    order, as the oracle's per-rank dispatch lays them out;
  * the per-expert row counts equal the sum of the ranks' kept counts.
"""
import datetime
import os
import socket

import pytest
import torch

import oracle
import synth
from parity_util import assert_close, margin_exempt, threads, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe(cuda_device):
    import sparse_mixture_experts_fwd_b200 as m
    return m


# name, world, T (per rank), d, f, E, k, capacity factor, mode, G, dtype, expert
CASES = [
    ("top1_w2", 2, 600, 128, 256, 16, 1, 1.0, "topk", 1, "bf16", "relu"),
    ("top2_w4", 4, 500, 128, 128, 16, 2, 1.0, "topk", 1, "bf16", "relu"),
    # world * C = 4 * 62 = 248 rows per expert: the two-launch grouped FFN
    ("top1_w4_grouped", 4, 1000, 64, 128, 16, 1, 1.0, "topk", 1, "bf16", "relu"),
    # world * C = 8 * 75 = 600 rows per expert: the SM-pair FFN
    ("top1_w8_pairs", 8, 600, 64, 128, 8, 1, 1.0, "topk", 1, "bf16", "relu"),
    ("rre_w2", 2, 800, 64, 128, 16, 1, 1.25, "rre", 4, "bf16", "relu"),
    ("fp32_top2_w2", 2, 300, 32, 48, 8, 2, 1.5, "topk", 1, "f32", "relu"),
    ("geglu_top2_w2", 2, 400, 128, 128, 8, 2, 2.0, "topk", 1, "bf16", "geglu"),
    ("one_expert_per_rank", 4, 300, 64, 64, 4, 1, 1.0, "topk", 1, "bf16", "relu"),
    ("hot_expert_w2", 2, 700, 64, 128, 16, 1, 1.0, "topk", 1, "bf16", "relu"),
]


def _workload(case):
    name, world, T, d, f, E, k, cf, mode, G, dtype, expert = case
    hot = 100.0 if name.startswith("hot") else 0.0
    return synth.Workload(name, T=T, d_model=d, d_ff=f, E=E, k=k, capacity_factor=cf, dtype=dtype,
                          mode=mode, num_groups=G, hot_experts=1 if hot else 0, hot_bias=hot,
                          seed=11, expert=expert, expert_std=0.1 if expert == "geglu" else 0.02)


def _emulated_group(moe, w, world, dev):
    """Run every rank's EP layer step on one device; returns per-rank dicts."""
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    cfg = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, C, dtype=w.torch_dtype, mode=w.mode,
                          num_groups=w.num_groups, seed=w.seed, expert=w.expert)
    fcfg = moe.ep_ffn_config(cfg, world)
    El, PC = fcfg.E, fcfg.capacity
    assert El == w.E // world and PC == world * C
    full = synth.layer_inputs(w)  # router and the full expert set (shared by all ranks)
    ranks = []
    for q in range(world):
        inp = synth.layer_inputs(w, weights=False, x_seed_offset=q)
        r = {"inp": inp, "st": torch.zeros(1, dtype=torch.int32, device=dev)}
        r["x"] = inp["x"].to(dev)
        if w.mode == "topk":
            logits = moe.router(cfg, r["x"], full["Wr"].to(dev), to_dev(full["bias"], dev),
                                status=r["st"])
            r["route"] = moe.topk_assign(cfg, logits=logits, status=r["st"])
        else:
            r["route"] = moe.topk_assign(cfg, domain_id=inp["domain"].to(dev), status=r["st"])
        r["W1"] = full["W1"][q * El:(q + 1) * El].contiguous().to(dev)
        r["W2"] = full["W2"][q * El:(q + 1) * El].contiguous().to(dev)
        # receive buffers filled with a sentinel so rows no rank sends stay recognisable
        r["xe"] = torch.full((El, PC, w.d_model), 7.0, dtype=w.torch_dtype, device=dev)
        r["ye"] = torch.full((El, PC, w.d_model), 7.0, dtype=w.torch_dtype, device=dev)
        r["H"] = torch.empty(El, PC, w.d_ff, dtype=w.torch_dtype, device=dev)
        ranks.append(r)
    # the all-gather of the kept counts
    cnt_all = torch.stack([r["route"]["kept_cnt"] for r in ranks]).contiguous()
    xe_peers = [r["xe"] for r in ranks]
    ye_peers = [r["ye"] for r in ranks]
    for q, r in enumerate(ranks):
        ro = r["route"]
        r["local_cnt"] = moe.ep_dispatch(cfg, q, world, r["x"], ro["expert_idx"], ro["slot"],
                                         ro["kept"], cnt_all, xe_peers, status=r["st"])
    for r in ranks:  # barrier: every rank's rows have landed
        moe.expert_ffn(fcfg, r["xe"], r["W1"], r["W2"], r["local_cnt"], H=r["H"], ye=r["ye"],
                       status=r["st"])
    for q, r in enumerate(ranks):  # barrier: every expert output is written
        ro = r["route"]
        r["y"] = moe.ep_combine(cfg, q, world, ye_peers, ro["expert_idx"], ro["gate"], ro["slot"],
                                ro["kept"], cnt_all, status=r["st"])
    torch.cuda.synchronize()
    return cfg, C, full, ranks, cnt_all


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_ep_emulated_group(moe, cuda_device, case):
    name, world = case[0], case[1]
    w = _workload(case)
    cfg, C, full, ranks, cnt_all = _emulated_group(moe, w, world, cuda_device)
    El = w.E // world
    tol = dict(atol=1e-5, rtol=1e-5) if w.dtype == "f32" else {}
    refs = []
    for q, r in enumerate(ranks):
        assert int(r["st"].item()) == 0, (q, int(r["st"].item()))
        inp = r["inp"]
        ref = oracle.layer_forward(inp["x"], full["W1"], full["W2"], E=w.E, k=w.k, C=C,
                                   Wr=full["Wr"], bias=full["bias"], domain=inp["domain"],
                                   G=w.num_groups, seed=w.seed, nthreads=threads(), kind=w.expert)
        refs.append(ref)
        ro = {k_: v.cpu() for k_, v in r["route"].items()}
        if w.mode == "topk":
            differs = (ro["expert_idx"] != ref["expert_idx"]).any(1)
            assert not bool((differs & ~margin_exempt(ref["logits"], w.k)).any())
            assert not bool(differs.any()), "these cases are expected to route identically"
        for key in ("expert_idx", "slot", "kept", "kept_cnt"):
            assert torch.equal(ro[key], ref[key]), (q, key)
        assert_close(r["y"].cpu(), ref["y"], what=f"y of rank {q}", **tol)
        none_kept = ref["kept"].sum(1) == 0
        assert bool((r["y"].cpu()[none_kept] == 0).all())
    # counts and the packed receive layout
    cnt = cnt_all.cpu()
    for h in range(world):
        xe_h = ranks[h]["xe"].cpu()
        local = ranks[h]["local_cnt"].cpu()
        for el in range(El):
            e = h * El + el
            assert int(local[el]) == int(cnt[:, e].sum()), (h, el)
            off = 0
            for q in range(world):
                n = int(cnt[q, e])
                got = xe_h[el, off:off + n]
                want = refs[q]["xe"][e, :n]
                if w.dtype == "bf16":
                    got, want = got.view(torch.int16), want.view(torch.int16)
                assert torch.equal(got, want), (h, el, q)
                off += n
            # rows past the senders' total stay untouched (sentinel)
            assert bool((xe_h[el, off:].double() == 7.0).all()), (h, el)


def test_ep_world_one_matches_single_device_steps(moe, cuda_device):
    """world = 1: the EP dispatch and combine place and read every row where
    moe_dispatch and moe_combine do, so the outputs agree bit for bit."""
    w = _workload(("w1", 1, 700, 128, 256, 16, 2, 1.0, "topk", 1, "bf16", "relu"))
    cfg, C, full, ranks, cnt_all = _emulated_group(moe, w, 1, cuda_device)
    r = ranks[0]
    ro = r["route"]
    xe = moe.dispatch(cfg, r["x"], ro["expert_idx"], ro["slot"], ro["kept"])
    _, ye = moe.expert_ffn(cfg, xe, r["W1"], r["W2"], ro["kept_cnt"])
    y = moe.combine(cfg, ye, ro["expert_idx"], ro["gate"], ro["slot"], ro["kept"])
    torch.cuda.synchronize()
    assert torch.equal(r["local_cnt"].cpu(), ro["kept_cnt"].cpu())
    for e in range(w.E):
        n = int(ro["kept_cnt"][e])
        assert torch.equal(r["xe"][e, :n].view(torch.int16), xe[e, :n].view(torch.int16)), e
    assert torch.equal(r["y"].view(torch.int16), y.view(torch.int16))


def test_ep_bad_counts_reported(moe, cuda_device):
    """Counts that do not match the assignment (a sender's rows would pass the
    end of the expert's block) are skipped and flagged, not written."""
    dev = cuda_device
    world, T, d, E, C = 2, 64, 64, 4, 40
    cfg = moe.make_config(T, d, 64, E, 1, C)
    x = torch.ones(T, d, dtype=torch.bfloat16, device=dev)
    idx = torch.zeros(T, 1, dtype=torch.int32, device=dev)        # every token -> expert 0
    slot = torch.arange(T, dtype=torch.int32, device=dev).view(T, 1)
    kept = (slot < C).to(torch.uint8)
    # rank 1 claims rank 0 kept 70 rows of expert 0: rank 1's rows start at 70 > 2C - 40
    cnt_all = torch.tensor([[70, 0, 0, 0], [C, 0, 0, 0]], dtype=torch.int32, device=dev)
    El, PC = E // world, world * C
    xe = [torch.zeros(El, PC, d, dtype=torch.bfloat16, device=dev) for _ in range(world)]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.ep_dispatch(cfg, 1, world, x, idx, slot, kept, cnt_all, xe, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.STATUS_BAD_COUNTS
    # rows 70..79 of expert 0's block were written, the 30 past its end skipped
    assert int((xe[0][0].float().sum(1) > 0).sum()) == PC - 70
    st.zero_()
    y = moe.ep_combine(cfg, 1, world, xe, idx, torch.ones(T, 1, device=dev), slot, kept, cnt_all,
                       status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.STATUS_BAD_COUNTS
    assert bool((y[:10].float() == 1).all()) and bool((y[10:].float() == 0).all())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_layer_nccl_single_rank(moe, cuda_device):
    """ExpertParallelLayer on a one-rank NCCL group: the count all-gather, the
    barriers and the peer table run through torch.distributed on the GPU."""
    import torch.distributed as dist
    from sparse_mixture_experts_fwd_b200.ep import ExpertParallelLayer
    w = _workload(("nccl1", 1, 900, 128, 256, 32, 2, 1.0, "topk", 1, "bf16", "relu"))
    dev = cuda_device
    inp = synth.layer_inputs(w)
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    cfg = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, C)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        layer = ExpertParallelLayer(cfg)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        x = inp["x"].to(dev)
        W1, W2, Wr = inp["W1"].to(dev), inp["W2"].to(dev), inp["Wr"].to(dev)
        y1 = layer(x, W1, W2, Wr=Wr, status=st).clone()
        y2 = layer(x, W1, W2, Wr=Wr, status=st)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert int(st.item()) == 0
    ref = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=w.E, k=w.k, C=C, Wr=inp["Wr"],
                               bias=inp["bias"], nthreads=threads())
    assert_close(y1.cpu(), ref["y"], what="y")
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
