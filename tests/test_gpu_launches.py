"""The kernels one moe_layer_forward call launches, counted by the CUDA profiler.

bench.py reports ``gpu_launches`` from ``bench.kernel_launches``; this checks
that count against the kernels CUPTI sees for one call, in every regime the
library selects kernels by (dtype, routing mode, k, capacity band).
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

# (workload, overrides): each lands in a different kernel selection
REGIMES = [
    ("tiny_switch", {}),                                                # fp32 path
    ("switch_base", {"T": 2048}),                                       # top-1, C = 20
    ("xmoe_top2", {"T": 4096, "d_model": 256, "d_ff": 512}),            # top-2, C = 128
    ("xmoe_top2", {"T": 8192, "d_model": 256, "d_ff": 512}),            # C = 256
    ("pangu_rre", {"T": 26215, "d_model": 256, "d_ff": 512}),           # RRE, C = 512
    ("pangu_rre", {"T": 32768, "d_model": 256, "d_ff": 512}),           # C = 640
]


def _kernel_names(prof):
    names = []
    for ev in prof.events():
        if ev.device_type != torch.autograd.DeviceType.CUDA:
            continue
        n = ev.name
        if n.lower().startswith(("memcpy", "memset")):
            continue
        names.append(n)
    return names


@pytest.mark.parametrize("name,over", REGIMES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(REGIMES)])
def test_layer_launch_count(cuda_device, name, over):
    import bench
    import sparse_mixture_experts_fwd_b200 as moe
    w = synth.WORKLOADS[name].scaled(**over)
    C = moe.capacity(w.T, w.E, w.capacity_factor)
    inp = synth.layer_inputs(w)
    dev = cuda_device
    D = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    cfg = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, C, dtype=w.torch_dtype, mode=w.mode,
                          num_groups=w.num_groups, seed=w.seed)
    ws = torch.empty(moe.workspace_size(cfg), dtype=torch.uint8, device=dev)
    y = torch.empty(w.T, w.d_model, dtype=w.torch_dtype, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        moe.layer_forward(cfg, D["x"], D["W1"], D["W2"], Wr=D["Wr"], bias=D["bias"],
                          domain_id=D["domain"], y=y, workspace=ws, status=st)

    call()
    torch.cuda.synchronize()
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        call()
        torch.cuda.synchronize()
    assert int(st.item()) == 0
    names = _kernel_names(prof)
    assert names, "the profiler recorded no kernels"
    assert len(names) == bench.kernel_launches(w, C), names
