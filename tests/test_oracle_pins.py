"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test ties one oracle function to something independent of its code:
a hand-worked fixture under tests/golden/ (closed forms of the Switch notes'
eq. (1)-(3) and of the TorchScale SparseClip norm), a library routine on a
special case (numpy float64 matmul, torch's bf16 rounding, numpy sorting and
norms), brute-force enumeration on tiny inputs, or an invariant the pages fix
(gates sum to 1, each expert holds at most C tokens, ...).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore")


# ---------------------------------------------------------------------------
# routing: eq. (1) gate, top-k, eq. (3) capacity, drop rule
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fixture", ["top1_example.txt", "top2_example.txt"])
def test_hand_worked_routing(oracle_lib, fixture):
    g = read_golden(fixture)
    T, E, k, C = (int(g[key][0][0]) for key in ("T", "E", "k", "C"))
    logits = torch.tensor([[float(v) for v in row] for row in g["logits"]], dtype=torch.float32)
    assert logits.shape == (T, E)
    idx, gate = oracle.gate_topk(logits, k)
    a = oracle.assign(idx, E, C)
    exp = g["expect"]
    for i, (e, s, kept, p) in enumerate(exp):
        t, j = divmod(i, k)
        assert idx[t, j].item() == int(e)
        assert a["slot"][t, j].item() == int(s)
        assert a["kept"][t, j].item() == int(kept)
        assert gate[t, j].item() == pytest.approx(float(p), rel=1e-7)
    assert a["arrivals"].tolist() == [int(v) for v in g["arrivals"][0]]
    assert a["kept_cnt"].tolist() == [int(v) for v in g["kept_cnt"][0]]
    assert a["n_dropped"] == int(g["n_dropped"][0][0])


def test_capacity_closed_form(oracle_lib):
    g = read_golden("capacity_closed_form.txt")
    for name, rows in g.items():
        T, E, cf, C = rows[0]
        assert oracle.capacity(int(T), int(E), float(cf)) == int(C), name
        w = synth.WORKLOADS[name]
        assert (w.T, w.E, w.capacity_factor) == (int(T), int(E), float(cf))
    # non-integral case: the floor reading
    assert oracle.capacity(10, 3, 1.0) == 3
    assert oracle.capacity(7, 2, 1.25) == 4


def test_gate_is_softmax_and_sums_to_one(oracle_lib):
    gen = torch.Generator().manual_seed(1)
    logits = (torch.randn(200, 13, generator=gen, dtype=torch.float64) * 3).float()
    idx, gate, ps = oracle.gate_topk(logits, 2, with_prob_sum=True)
    ref = torch.softmax(logits.double(), dim=1)  # library softmax in float64
    np.testing.assert_allclose(ps.numpy(), 1.0, rtol=0, atol=1e-12)
    sel = ref.gather(1, idx.long())
    np.testing.assert_allclose(gate.double().numpy(), sel.numpy(), rtol=1e-7)
    assert bool((gate[:, 0] > 1.0 / 13).all()) and bool((gate[:, 0] <= 1.0).all())
    assert bool((gate.sum(1) <= 1.0 + 1e-7).all())
    assert bool((gate[:, 0] >= gate[:, 1]).all())


def test_topk_matches_library_sort_with_ties(oracle_lib):
    gen = torch.Generator().manual_seed(2)
    # small integer logits force many ties
    logits = torch.randint(-2, 3, (500, 7), generator=gen).float()
    for k in (1, 2):
        idx, _ = oracle.gate_topk(logits, k)
        for t in range(logits.shape[0]):
            h = logits[t].numpy()
            order = np.lexsort((np.arange(h.size), -h))  # value desc, index asc
            assert idx[t].tolist() == order[:k].tolist()


def _definitional_slots(choices, E):
    """slot of (t, j) = number of earlier assignments (token order) to the same expert."""
    slots = []
    seen = []
    for t, row in enumerate(choices):
        for j, e in enumerate(row):
            slots.append(sum(1 for (tt, jj, ee) in seen if ee == e))
            seen.append((t, j, e))
    return slots


@pytest.mark.parametrize("k,T,E", [(1, 6, 3), (2, 5, 3)])
def test_assign_brute_force(oracle_lib, k, T, E):
    per_token = [c for c in itertools.permutations(range(E), k)]
    for pattern in itertools.product(per_token, repeat=T):
        idx = torch.tensor(pattern, dtype=torch.int32).view(T, k)
        ref_slots = _definitional_slots(pattern, E)
        for C in range(0, T + 1):
            a = oracle.assign(idx, E, C)
            assert a["slot"].flatten().tolist() == ref_slots
            assert a["kept"].flatten().tolist() == [int(s < C) for s in ref_slots]
            arr = [sum(1 for row in pattern for e in row if e == x) for x in range(E)]
            assert a["arrivals"].tolist() == arr
            assert a["kept_cnt"].tolist() == [min(v, C) for v in arr]
            assert a["n_dropped"] == sum(max(0, v - C) for v in arr)
        # cheaper on the remaining capacities: keep the loop bounded
        if T * k > 10:
            break


def test_assign_invariants_random(oracle_lib):
    gen = torch.Generator().manual_seed(3)
    T, E, k, C = 3000, 17, 2, 300
    logits = torch.randn(T, E, generator=gen)
    logits[:, 3] += 1.5  # a hot expert so some overflow happens
    idx, _ = oracle.gate_topk(logits, k)
    a = oracle.assign(idx, E, C)
    kc, arr = a["kept_cnt"], a["arrivals"]
    assert int(kc.max()) <= C
    assert int(a["kept"].sum()) + a["n_dropped"] == T * k
    assert a["n_dropped"] > 0
    for e in range(E):
        assert int(kc[e]) == min(int(arr[e]), C)
        mask = (idx == e) & (a["kept"] == 1)
        assert sorted(a["slot"][mask].tolist()) == list(range(int(kc[e])))
        rows = a["tok_of_row"][e * C: e * C + int(kc[e])]
        assert bool((rows[1:] > rows[:-1]).all())            # increasing token order
        assert bool((a["tok_of_row"][e * C + int(kc[e]): (e + 1) * C] == -1).all())
        # the kept tokens are exactly the first C arrivals
        toks = [t for t in range(T) if e in idx[t].tolist()]
        assert rows.tolist() == toks[:C]


# ---------------------------------------------------------------------------
# RRE: splitmix64, groups
# ---------------------------------------------------------------------------

def test_splitmix64_published_values(oracle_lib):
    g = read_golden("splitmix64_seed0.txt")
    for t, hexval in g["out"]:
        assert oracle.splitmix64(0, int(t)) == int(hexval, 16)
    assert [oracle.splitmix64(0, t) % 8 for t in range(8)] == [int(v) for v in g["mod8"][0]]


def test_rre_groups_and_uniformity(oracle_lib):
    T, E, G = 200_000, 64, 8
    domain = synth.uniform_int(0, synth.TAGS["domain"], T, G)
    idx, gate = oracle.route_rre(domain, E, G, seed=0)
    per = E // G
    assert bool((idx[:, 0] // per == domain).all())
    assert bool((gate == 1.0).all())
    counts = torch.bincount(idx[:, 0].long() - domain.long() * per, minlength=per).double()
    expected = T / per
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 24.3  # chi^2 with 7 dof, p = 0.001
    # the in-group index is splitmix64(seed, t) mod per
    for t in (0, 1, 2, 12345, T - 1):
        assert int(idx[t, 0]) == int(domain[t]) * per + oracle.splitmix64(0, t) % per
    # another seed gives another assignment
    idx2, _ = oracle.route_rre(domain, E, G, seed=7)
    assert float((idx2 != idx).float().mean()) > 0.8


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_torch(oracle_lib):
    gen = torch.Generator().manual_seed(4)
    vals = torch.cat([
        torch.randn(4000, generator=gen) * 10.0 ** torch.randint(-30, 30, (4000,), generator=gen),
        torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 2 ** -130, 3e-39,
                      -2 ** -133, 1.00390625, 65504.0, 0.0]),
    ]).float()
    ref = vals.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.round_bf16_bits(float(v)) for v in vals], dtype=np.uint16)
    assert (got == ref).all()


# ---------------------------------------------------------------------------
# router and expert FFN against numpy float64 matmul
# ---------------------------------------------------------------------------

def test_router_matches_float64_matmul(oracle_lib):
    x = synth.normal(5, 1, (37, 96), 1.0, torch.float32)
    Wr = synth.normal(5, 2, (11, 96), 0.1, torch.float32)
    bias = torch.linspace(-1, 1, 11, dtype=torch.float32)
    got = oracle.router(x, Wr, bias)
    ref = (x.double().numpy() @ Wr.double().numpy().T + bias.double().numpy()).astype(np.float32)
    np.testing.assert_array_max_ulp(got.numpy(), ref, maxulp=1)
    xb = x.to(torch.bfloat16)
    Wb = Wr.to(torch.bfloat16)
    got_b = oracle.router(xb, Wb, None)
    ref_b = (xb.double().numpy() @ Wb.double().numpy().T).astype(np.float32)
    np.testing.assert_array_max_ulp(got_b.numpy(), ref_b, maxulp=1)


def test_expert_ffn_fp32_matches_numpy(oracle_lib):
    d, f, E, C = 48, 80, 3, 5
    xe = synth.normal(6, 1, (E, C, d), 1.0, torch.float32)
    W1 = synth.normal(6, 3, (E, f, d), 0.1, torch.float32)
    W2 = synth.normal(6, 4, (E, d, f), 0.1, torch.float32)
    kept = torch.tensor([5, 0, 3], dtype=torch.int32)
    ye, H = oracle.expert_ffn(xe, W1, W2, kept, with_H=True)
    for e in range(E):
        n = int(kept[e])
        a = xe[e, :n].double().numpy() @ W1[e].double().numpy().T
        Hr = np.maximum(a, 0).astype(np.float32)
        o = Hr.astype(np.float64) @ W2[e].double().numpy().T
        np.testing.assert_array_max_ulp(H[e, :n].numpy(), Hr, maxulp=1)
        np.testing.assert_allclose(ye[e, :n].numpy(), o.astype(np.float32), rtol=1e-6, atol=1e-7)
        assert bool((ye[e, n:] == 0).all())  # rows past kept_cnt untouched


def test_expert_ffn_bf16_matches_numpy(oracle_lib):
    d, f = 64, 128
    x = synth.normal(7, 1, (d,), 1.0, torch.bfloat16)
    W1 = synth.normal(7, 3, (f, d), 0.05, torch.bfloat16)
    W2 = synth.normal(7, 4, (d, f), 0.05, torch.bfloat16)
    out, H = oracle.expert_row(x, W1, W2, with_H=True)
    a = W1.double().numpy() @ x.double().numpy()
    Hr = torch.from_numpy(np.maximum(a, 0)).float().to(torch.bfloat16)
    # H within one bf16 ulp of torch's rounding of the float64 result
    diff = (H.view(torch.int16).int() - Hr.view(torch.int16).int()).abs()
    assert int(diff.max()) <= 1
    o = W2.double().numpy() @ H.double().numpy()
    ref = torch.from_numpy(o).float().to(torch.bfloat16)
    diff = (out.view(torch.int16).int() - ref.view(torch.int16).int()).abs()
    assert int(diff.max()) <= 1


# ---------------------------------------------------------------------------
# dispatch / combine: identity experts reproduce the gate (eq. (2), k = 1)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("k", [1, 2])
def test_identity_experts_reproduce_gate(oracle_lib, k):
    T, d, E = 40, 16, 4
    C = oracle.capacity(T, E, 1.0 if k == 1 else 1.5)
    x = synth.normal(8, 1, (T, d), 1.0, torch.float32).abs() + 0.1
    eye = torch.eye(d, dtype=torch.float32)
    W1 = eye.expand(E, d, d).contiguous()
    W2 = eye.expand(E, d, d).contiguous()
    Wr = synth.normal(8, 2, (E, d), 1.0, torch.float32)
    r = oracle.layer_forward(x, W1, W2, E=E, k=k, C=C, Wr=Wr)
    assert r["n_dropped"] > 0
    expect = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            if r["kept"][t, j]:
                expect[t] += float(r["gate"][t, j]) * x[t].double()
    np.testing.assert_allclose(r["y"].double().numpy(), expect.numpy(), rtol=1e-6, atol=0)
    dropped_all = (r["kept"].sum(1) == 0)
    assert bool((r["y"][dropped_all] == 0).all())
    # dispatch put every kept token's row in its expert slot
    for t in range(T):
        for j in range(k):
            if r["kept"][t, j]:
                e, s = int(r["expert_idx"][t, j]), int(r["slot"][t, j])
                assert torch.equal(r["xe"][e, s], x[t])


def test_layer_forward_is_composition_of_steps(oracle_lib):
    w = synth.WORKLOADS["tiny_switch"]
    inp = synth.layer_inputs(w)
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    r = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=w.E, k=w.k, C=C, Wr=inp["Wr"])
    logits = oracle.router(inp["x"], inp["Wr"])
    idx, gate = oracle.gate_topk(logits, w.k)
    a = oracle.assign(idx, w.E, C)
    xe = oracle.dispatch(inp["x"], a["tok_of_row"], a["kept_cnt"], w.E, C)
    ye = oracle.expert_ffn(xe, inp["W1"], inp["W2"], a["kept_cnt"])
    y = oracle.combine(ye, idx, gate, a["slot"], a["kept"], w.T)
    assert torch.equal(r["logits"], logits) and torch.equal(r["expert_idx"], idx)
    assert torch.equal(r["y"], y)
    # per-token row formulation agrees with the per-expert batch formulation
    for t in range(0, w.T, 17):
        if a["kept"][t, 0]:
            e = int(idx[t, 0])
            row = oracle.expert_row(inp["x"][t], inp["W1"][e], inp["W2"][e])
            assert torch.equal(row, ye[e, int(a["slot"][t, 0])])
    # closed-form load facts for this workload
    assert C == 32 and int(a["kept_cnt"].max()) <= 32
    assert int(a["kept"].sum()) + a["n_dropped"] == w.T


def test_token_forward_matches_layer(oracle_lib):
    w = synth.WORKLOADS["xmoe_top2"].scaled(T=300, d_model=128, d_ff=256, E=8)
    inp = synth.layer_inputs(w)
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    r = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=w.E, k=2, C=C, Wr=inp["Wr"])
    partly = [t for t in range(w.T) if int(r["kept"][t].sum()) == 1]
    assert partly, "expected a token with one of two choices dropped"
    for t in list(range(0, w.T, 23)) + partly[:5]:
        y = oracle.token_forward(inp["x"][t], inp["W1"], inp["W2"], r["expert_idx"][t],
                                 r["gate"][t], r["kept"][t])
        assert torch.equal(y, r["y"][t])


def test_rre_layer_has_unit_gates(oracle_lib):
    w = synth.WORKLOADS["pangu_rre"].scaled(T=512, d_model=64, d_ff=128)
    inp = synth.layer_inputs(w)
    C = oracle.capacity(w.T, w.E, w.capacity_factor)
    r = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=w.E, k=1, C=C,
                             domain=inp["domain"], G=w.num_groups, seed=w.seed)
    assert C == 10
    assert bool((r["gate"] == 1.0).all())
    t = int(torch.nonzero(r["kept"][:, 0])[0, 0])
    e, s = int(r["expert_idx"][t, 0]), int(r["slot"][t, 0])
    assert torch.equal(r["y"][t], r["ye"][e, s])  # unweighted gate: y = E_i(x)


# ---------------------------------------------------------------------------
# SparseClip
# ---------------------------------------------------------------------------

def test_sparseclip_hand_example(oracle_lib):
    g = read_golden("sparseclip_example.txt")
    E = int(g["E"][0][0])
    gd = torch.tensor([float(v) for v in g["g_dense"][0]])
    gs = torch.tensor([float(v) for v in g["g_sparse"][0]])
    assert oracle.sparseclip_norm([gd], [gs], E) == pytest.approx(float(g["norm"][0][0]), rel=1e-15)


def test_sparseclip_special_cases(oracle_lib):
    gd = [synth.normal(9, 6, (10007,), 1e-3, torch.float32), synth.normal(9, 8, (33,), 1.0, torch.float32)]
    gs = [synth.normal(9, 7 + 16 * s, (5003,), 1e-3, torch.float32) for s in range(3)]
    allg = np.concatenate([t.double().numpy() for t in gd + gs])
    # E = 1: kappa = 1, the plain global L2 norm
    assert oracle.sparseclip_norm(gd, gs, 1) == pytest.approx(float(np.linalg.norm(allg)), rel=1e-12)
    # no sparse gradient: the dense norm
    dn = float(np.linalg.norm(np.concatenate([t.double().numpy() for t in gd])))
    assert oracle.sparseclip_norm(gd, [torch.zeros(10)], 64) == pytest.approx(dn, rel=1e-12)
    # E = 64: kappa^2 = 1/64 exactly
    sn = float(np.linalg.norm(np.concatenate([t.double().numpy() for t in gs])))
    assert oracle.sparseclip_norm(gd, gs, 64) == pytest.approx(math.sqrt(dn ** 2 + sn ** 2 / 64), rel=1e-12)


# ---------------------------------------------------------------------------
# Switch load-balancing loss (eqs. 4-6) and routing entropy
# ---------------------------------------------------------------------------

def test_aux_loss_hand_examples(oracle_lib):
    g = read_golden("aux_loss_example.txt")
    alpha = float(g["alpha"][0][0])
    for case in ("caseA", "caseB"):
        lg = torch.tensor([[float(v) * math.log(3.0) for v in row] for row in g[case + "_l3"]],
                          dtype=torch.float32)
        loss, ent, f, P = oracle.aux_loss(lg, alpha)
        # ln 3 is rounded to fp32 in the logits: |rel err| ~ 1e-7
        assert loss == pytest.approx(float(g[case + "_loss"][0][0]), rel=1e-6)
        assert ent == pytest.approx(float(g[case + "_entropy"][0][0]), rel=1e-6)
        assert f.tolist() == [float(v) for v in g[case + "_f"][0]]
        assert P.tolist() == pytest.approx([float(v) for v in g[case + "_P"][0]], rel=1e-6)


@pytest.mark.parametrize("E", [1, 3, 8, 64, 256])
def test_aux_loss_closed_forms(oracle_lib, E):
    alpha = 1e-2
    # equal logits: p uniform (P_i = 1/E, entropy ln E); every argmax is expert 0
    # (tie -> lower index), so f = e_0 and the loss is alpha * E * (1/E) = alpha
    loss, ent, f, P = oracle.aux_loss(torch.zeros(7, E), alpha)
    assert loss == pytest.approx(alpha, rel=1e-12)
    assert ent == pytest.approx(math.log(E), abs=1e-12)
    assert f[0] == 1.0 and float(f.sum()) == 1.0
    assert torch.allclose(P, torch.full((E,), 1.0 / E, dtype=torch.float64), rtol=1e-12)
    # a balanced assignment (token t peaks at expert t mod E, n tokens per expert):
    # f_i = P_i = 1/E by symmetry, so the loss is alpha (the minimum the notes
    # describe); each token's entropy is ln(e^L + E - 1) - L e^L / (e^L + E - 1)
    L, n = 3.0, 5
    lg = torch.zeros(n * E, E)
    lg[torch.arange(n * E), torch.arange(n * E) % E] = L
    loss, ent, f, P = oracle.aux_loss(lg, alpha)
    z = math.exp(L) + E - 1
    assert loss == pytest.approx(alpha, rel=1e-12)
    assert ent == pytest.approx(math.log(z) - L * math.exp(L) / z, rel=1e-12, abs=1e-15)
    assert torch.allclose(f, torch.full((E,), 1.0 / E, dtype=torch.float64), rtol=1e-12)
    assert torch.allclose(P, torch.full((E,), 1.0 / E, dtype=torch.float64), rtol=1e-12)


def test_aux_loss_against_library_softmax(oracle_lib):
    # an independent statement of eqs. (4)-(6) with library routines
    T, E, alpha = 513, 40, 1e-2
    lg = synth.normal(5, 2, (T, E), 1.5, torch.float32)
    loss, ent, f, P = oracle.aux_loss(lg, alpha)
    p = torch.softmax(lg.double(), dim=1)
    P_ref = p.mean(0)
    f_ref = torch.bincount(lg.argmax(1), minlength=E).double() / T  # continuous draws: no ties
    assert torch.allclose(P, P_ref, rtol=1e-12, atol=0)
    assert torch.equal(f, f_ref)
    assert loss == pytest.approx(alpha * E * float((f_ref * P_ref).sum()), rel=1e-12)
    assert ent == pytest.approx(float(-(p * p.log()).sum(1).mean()), rel=1e-12)


def test_sparseclip_clip_hand_example(oracle_lib):
    g = read_golden("sparseclip_example.txt")
    E = int(g["E"][0][0])
    gd = torch.tensor([float(v) for v in g["g_dense"][0]])
    gs = torch.tensor([float(v) for v in g["g_sparse"][0]])
    d0, s0 = gd.clone(), gs.clone()
    coef, norm = oracle.sparseclip_clip([gd], [gs], E, float(g["max_norm"][0][0]))
    assert coef == pytest.approx(float(g["coef"][0][0]), rel=1e-15)
    assert norm == pytest.approx(float(g["norm"][0][0]), rel=1e-15)
    r = 1 / math.sqrt(2.0)
    assert gd.tolist() == [float(torch.tensor(v * r, dtype=torch.float32)) for v in d0.tolist()]
    assert gs.tolist() == [float(torch.tensor(v * r, dtype=torch.float32)) for v in s0.tolist()]
    # after clipping the reweighted norm is max_norm (up to the fp32 rounding of the values)
    assert oracle.sparseclip_norm([gd], [gs], E) == pytest.approx(5.0, rel=1e-7)


def test_sparseclip_clip_special_cases(oracle_lib):
    gd = [synth.normal(11, 6, (1001,), 1e-3, torch.float32)]
    gs = [synth.normal(11, 7 + 16 * s, (503,), 1e-3, torch.float32) for s in range(4)]
    norm = oracle.sparseclip_norm(gd, gs, 4)
    # a threshold above the norm leaves every value untouched, bit for bit
    before = [t.clone() for t in gd + gs]
    coef, _ = oracle.sparseclip_clip(gd, gs, 4, 2 * norm)
    assert coef == 1.0 and all(torch.equal(a, b) for a, b in zip(before, gd + gs))
    # below it: every tensor scaled by the same max_norm / norm, the new norm is max_norm
    coef, n2 = oracle.sparseclip_clip(gd, gs, 4, norm / 3)
    assert n2 == pytest.approx(norm, rel=1e-15) and coef == pytest.approx(1 / 3, rel=1e-12)
    for a, b in zip(before, gd + gs):
        assert torch.allclose(b.double(), a.double() / 3, rtol=2 ** -23, atol=0)
    assert oracle.sparseclip_norm(gd, gs, 4) == pytest.approx(norm / 3, rel=1e-6)
    # E = 1 (kappa = 1): the same coefficient as the library's clip-by-global-norm
    # (which adds 1e-6 to the norm)
    t = [synth.normal(12, 6, (777,), 1.0, torch.float32), synth.normal(12, 8, (333,), 1.0, torch.float32)]
    lib_t = [x.clone().requires_grad_(True) for x in t]
    for x in lib_t:
        x.grad = x.detach().clone()
    torch.nn.utils.clip_grad_norm_(lib_t, max_norm=1.0)
    oracle.sparseclip_clip([t[0]], [t[1]], 1, 1.0)
    for a, x in zip(t, lib_t):
        assert torch.allclose(a, x.grad, rtol=1e-5, atol=0)


# ---------------------------------------------------------------------------
# GEGLU expert (GLU in the feed-forward layer)
# ---------------------------------------------------------------------------

def _gelu(a):
    return 0.5 * a * (1.0 + math.erf(a / math.sqrt(2.0)))


def test_geglu_row_closed_form(oracle_lib):
    # x = e_0 and one-hot weights make each pre-activation a chosen number, so
    # H_i = GELU(g_i) * l_i by hand (GELU(1) = Phi(1) = 0.8413447460685429...)
    d, f = 8, 4
    g = [1.0, -1.0, 2.5, 0.0]
    lin = [2.0, 3.0, -0.5, 7.0]
    x = torch.zeros(d, dtype=torch.float32)
    x[0] = 1.0
    W1 = torch.zeros(2 * f, d, dtype=torch.float32)
    for i in range(f):
        W1[2 * i, 0] = g[i]
        W1[2 * i + 1, 0] = lin[i]
    W2 = torch.zeros(d, f, dtype=torch.float32)
    for i in range(f):
        W2[i, i] = 1.0  # out_i = H_i
    out, H = oracle.expert_row(x, W1, W2, with_H=True, kind="geglu")
    want = [_gelu(a) * b for a, b in zip(g, lin)]
    assert _gelu(1.0) == pytest.approx(0.8413447460685429, rel=1e-15)
    assert H.tolist() == [float(torch.tensor(v, dtype=torch.float32)) for v in want]
    assert out[:f].tolist() == H.tolist() and float(out[f:].abs().sum()) == 0.0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_geglu_against_library_gelu(oracle_lib, dtype):
    # an independent statement: torch's exact GELU on float64 products
    d, f = 64, 96
    x = synth.normal(8, 1, (d,), 1.0, dtype)
    W1 = synth.normal(8, 3, (2 * f, d), 0.1, dtype)
    W2 = synth.normal(8, 4, (d, f), 0.1, dtype)
    out, H = oracle.expert_row(x, W1, W2, with_H=True, kind="geglu")
    a = W1.double() @ x.double()
    h_ref = torch.nn.functional.gelu(a[0::2], approximate="none") * a[1::2]
    h_ref = h_ref.to(dtype)  # one rounding to the activation type
    assert torch.equal(H, h_ref) or torch.allclose(H.double(), h_ref.double(), rtol=2 ** -7, atol=0)
    o_ref = (W2.double() @ H.double()).to(dtype)
    assert torch.allclose(out.double(), o_ref.double(), rtol=2 ** -7, atol=1e-30)


def test_geglu_ffn_and_token_forward_agree(oracle_lib):
    # the per-expert batch, the per-token path and the row function give the same rows
    E, C, d, f = 3, 5, 64, 64
    xe = synth.normal(9, 1, (E, C, d), 1.0, torch.bfloat16)
    W1 = synth.normal(9, 3, (E, 2 * f, d), 0.05, torch.bfloat16)
    W2 = synth.normal(9, 4, (E, d, f), 0.05, torch.bfloat16)
    kept = torch.tensor([5, 0, 3], dtype=torch.int32)
    ye = oracle.expert_ffn(xe, W1, W2, kept, kind="geglu")
    for e in range(E):
        for r in range(int(kept[e])):
            row = oracle.expert_row(xe[e, r], W1[e], W2[e], kind="geglu")
            assert torch.equal(ye[e, r], row)
            y = oracle.token_forward(xe[e, r], W1, W2, torch.tensor([e], dtype=torch.int32),
                                     torch.tensor([1.0]), torch.tensor([1], dtype=torch.uint8),
                                     kind="geglu")
            assert torch.equal(y, row)
