"""The bounds-checked build (libmoe_b200_checked.so, moe_bounds_checked() == 1).

Run in a child process that loads the checked library
(MOE_B200_CHECK_BOUNDS=1).  The child refuses to go on unless the loaded
library reports that it checks bounds, so out-of-range indices are only ever
given to kernels that test them before touching a row.  It plants expert
indices and slots outside [0, E) x [0, C) among valid choices and checks that
moe_dispatch and moe_combine skip exactly those choices, report
MOE_STATUS_BAD_INDEX, leave canary rows around xe untouched and otherwise
produce the oracle's result; then a whole small layer through the checked
build matches the oracle like the default build.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = f"ROOT = {ROOT!r}\n" + textwrap.dedent(r"""
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, ROOT + "/tests")
    import torch
    import sparse_mixture_experts_fwd_b200 as moe
    if moe.lib.moe_bounds_checked() != 1:
        print("NOT_CHECKED", moe.LIB_PATH)
        sys.exit(3)
    import oracle
    import synth
    from parity_util import assert_close

    dev = torch.device("cuda", 0)
    T, d, E, k, C = 40, 128, 8, 2, 16
    x = synth.normal(5, 1, (T, d), 1.0, torch.bfloat16)
    g = torch.Generator().manual_seed(3)
    ei = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    a = oracle.assign(ei, E, C)
    slot, kept = a["slot"].clone(), a["kept"].clone()
    gate = torch.rand(T, k, generator=g, dtype=torch.float32)
    # planted: expert index past E, a negative expert, a slot past C, a negative slot
    bad = [(3, 0, "e", E), (5, 1, "e", -1), (7, 0, "s", C), (9, 1, "s", -2)]
    for t, j, what, v in bad:
        (ei if what == "e" else slot)[t, j] = v
        kept[t, j] = 1
    good = kept.clone()
    for t, j, _, _ in bad:
        good[t, j] = 0
    cfg = moe.make_config(T, d, 64, E, k, C, dtype=torch.bfloat16)

    # dispatch into xe with canary rows on both sides
    P = 4
    canary = -7.0
    big = torch.full((E * C + 2 * P, d), canary, dtype=torch.bfloat16, device=dev)
    xe = big[P:P + E * C].view(E, C, d)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.dispatch(cfg, x.to(dev), ei.to(dev), slot.to(dev), kept.to(dev), xe=xe, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.STATUS_BAD_INDEX, int(st.item())
    bigc = big.cpu()
    assert bool((bigc[:P] == canary).all()) and bool((bigc[P + E * C:] == canary).all())
    want = torch.full((E, C, d), canary, dtype=torch.bfloat16)
    for t in range(T):
        for j in range(k):
            if good[t, j]:
                want[ei[t, j], slot[t, j]] = x[t]
    assert torch.equal(xe.cpu().view(torch.int16), want.view(torch.int16)), "dispatch rows"

    # combine: the skipped choices contribute nothing
    ye = synth.normal(6, 2, (E, C, d), 1.0, torch.bfloat16)
    st.zero_()
    y = moe.combine(cfg, ye.to(dev), ei.to(dev), gate.to(dev), slot.to(dev), kept.to(dev),
                    status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.STATUS_BAD_INDEX, int(st.item())
    ei_ok = torch.where(good.bool(), ei, torch.zeros_like(ei))
    sl_ok = torch.where(good.bool(), slot, torch.zeros_like(slot))
    ref = oracle.combine(ye, ei_ok, gate, sl_ok, good, T)
    assert_close(y.cpu(), ref, what="combine")

    # a whole layer through the checked build: in range, no status, oracle's result
    w = synth.Workload("checked", T=700, d_model=128, d_ff=256, E=16, k=2, capacity_factor=1.0,
                       dtype="bf16", seed=9)
    inp = synth.layer_inputs(w)
    Cl = oracle.capacity(w.T, w.E, w.capacity_factor)
    cl = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, Cl, dtype=torch.bfloat16)
    st.zero_()
    yl = moe.layer_forward(cl, inp["x"].to(dev), inp["W1"].to(dev), inp["W2"].to(dev),
                           Wr=inp["Wr"].to(dev), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, int(st.item())
    r = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=w.E, k=w.k, C=Cl, Wr=inp["Wr"])
    assert_close(yl.cpu(), r["y"], what="layer (checked build)")
    print("CHECKED_OK")
""")


def test_checked_build_skips_and_reports_bad_indices(cuda_device):
    env = dict(os.environ, MOE_B200_CHECK_BOUNDS="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0 and "CHECKED_OK" in r.stdout, out[-4000:]
