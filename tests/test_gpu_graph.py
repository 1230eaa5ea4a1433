"""The layer forward captured into a CUDA graph.

``moe_layer_forward`` launches its kernels on the caller's stream with no host
synchronisation and no allocation, so a whole layer step can be captured once
(``torch.cuda.graph``, global capture mode: any call that is unsafe during
capture fails it) and replayed.  On each kernel path the replay must give the
eager call's y bit for bit, follow new contents of the captured input buffer,
and match the oracle's layer within the stated tolerance.
"""
import pytest
import torch

import oracle
import synth
from parity_util import assert_close, threads, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # name, T, d, f, E, k, cf, mode, G, dtype
    ("top2_two_launch", 1200, 128, 128, 8, 2, 2.0, "topk", 1, "bf16"),       # C = 600 > 128, d < 2048
    ("top1_fused_persistent", 1000, 128, 256, 16, 1, 1.0, "topk", 1, "bf16"),  # C = 63: one launch
    ("rre_pair_fused", 4400, 2048, 256, 8, 1, 1.0, "rre", 2, "bf16"),          # C = 550, d = 2048
    ("top2_fp32", 400, 32, 48, 8, 2, 1.5, "topk", 1, "f32"),
]


@pytest.fixture(scope="module")
def moe(cuda_device):
    import sparse_mixture_experts_fwd_b200 as m
    return m


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_layer_forward_graph_replay(moe, cuda_device, case):
    name, T, d, f, E, k, cf_, mode, G, dtype = case
    dev = cuda_device
    w = synth.Workload(name, T=T, d_model=d, d_ff=f, E=E, k=k, capacity_factor=cf_, dtype=dtype,
                       mode=mode, num_groups=G, seed=3)
    inp = synth.layer_inputs(w)
    C = moe.capacity(T, E, cf_)
    cfg = moe.make_config(T, d, f, E, k, C, dtype=w.torch_dtype, mode=mode, num_groups=G,
                          seed=w.seed)
    x = inp["x"].to(dev)
    W1, W2 = inp["W1"].to(dev), inp["W2"].to(dev)
    Wr, bias, dom = to_dev(inp["Wr"], dev), to_dev(inp["bias"], dev), to_dev(inp["domain"], dev)
    ws = torch.empty(moe.workspace_size(cfg), dtype=torch.uint8, device=dev)
    y = torch.empty(T, d, dtype=w.torch_dtype, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(device=dev)

    def call():
        moe.layer_forward(cfg, x, W1, W2, Wr=Wr, bias=bias, domain_id=dom, y=y, workspace=ws,
                          status=st, stream=torch.cuda.current_stream())

    with torch.cuda.stream(s):
        call()  # first call: the library's per-device caches and function attributes
    torch.cuda.synchronize()
    y_eager = y.clone()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="global"):
        call()
    y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(_bits(y), _bits(y_eager)), "replay differs from the eager call"

    # the oracle on the same inputs
    r = oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=E, k=k, C=C, Wr=inp["Wr"],
                             bias=inp["bias"], domain=inp["domain"], G=G, seed=w.seed,
                             nthreads=threads())
    tol = dict(atol=1e-5, rtol=1e-5) if dtype == "f32" else {}
    assert_close(y.cpu(), r["y"], what="y (graph replay)", **tol)

    # new contents in the captured x: the replay reads them
    x.copy_(synth.layer_inputs(w, weights=False, x_seed_offset=7)["x"].to(dev))
    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    y_eager2 = y.clone()
    assert not torch.equal(_bits(y_eager2), _bits(y_eager))
    y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(_bits(y), _bits(y_eager2)), "replay did not follow the new x"
    del g
