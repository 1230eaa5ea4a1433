"""sparseclip_norm_noalloc: the SparseClip norm for callers that cannot
allocate device memory (a runtime that hands all of HBM to its own pool at
start-up, or code that must not call the CUDA allocator where it runs).

The entry point keeps its partial sums in a fixed array inside the library
instead of a caller workspace.  This test calls it through the C ABI twice in
a row, on different gradients, and checks each result against the
workspace-taking sparseclip_norm on the same inputs and against the CPU
oracle's norm; the device's free memory is the same before and after the
second call.  It lives in its own file
that pytest collects last and passes alone in a fresh process as well as
after the other tests.
"""
import ctypes

import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

RTOL = 1e-5  # the tolerance the other SparseClip tests use


def _arrays(ts):
    ptrs = (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])
    lens = (ctypes.c_int64 * max(1, len(ts)))(*[t.numel() for t in ts])
    return ptrs, lens


def _noalloc(moe, dense, sparse, E, out):
    dp, dl = _arrays(dense)
    sp, sl = _arrays(sparse)
    vp = ctypes.c_void_p
    return moe.lib.sparseclip_norm_noalloc(ctypes.cast(dp, vp), ctypes.cast(dl, vp), len(dense),
                                           ctypes.cast(sp, vp), ctypes.cast(sl, vp), len(sparse),
                                           E, out.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)


def _grads(seed, dev, n_sparse, dense_lens):
    dense = [synth.normal(seed, 6 + 16 * i, (n,), 1e-3, torch.float32).to(dev)
             for i, n in enumerate(dense_lens)]
    sparse = [synth.normal(seed, 7 + 16 * (s + 1), (1021 + 13 * s,), 1e-3, torch.float32).to(dev)
              for s in range(n_sparse)]
    return dense, sparse


def test_noalloc_matches_workspace_entry_point(cuda_device):
    import sparse_mixture_experts_fwd_b200 as moe
    dev = cuda_device
    cases = [
        (_grads(1, dev, 300, [1_000_003, 5, 4096]), 64),  # several launches, ragged tails
        (_grads(2, dev, 64, [777_777]), 8),               # second call, other data and E
    ]
    for i, ((dense, sparse), E) in enumerate(cases):
        ref = moe.sparseclip_norm(dense, sparse, E)
        out = torch.full((3,), float("nan"), dtype=torch.float64, device=dev)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info(dev)[0]
        assert _noalloc(moe, dense, sparse, E, out) == 0, moe.lib.moe_last_error()
        torch.cuda.synchronize()
        if i > 0:  # (the first call may load the kernels' module)
            assert torch.cuda.mem_get_info(dev)[0] == free_before, "the call allocated device memory"
        got, want = out.cpu(), ref.cpu()
        assert bool(((got - want).abs() <= RTOL * want.abs()).all()), (got, want)
        norm = oracle.sparseclip_norm([t.cpu() for t in dense], [t.cpu() for t in sparse], E)
        assert abs(float(got[0]) - norm) <= RTOL * norm, (float(got[0]), norm)


def test_noalloc_rejects_too_many_tensors(cuda_device):
    import sparse_mixture_experts_fwd_b200 as moe
    dev = cuda_device
    t = torch.ones(4, dtype=torch.float32, device=dev)
    out = torch.zeros(3, dtype=torch.float64, device=dev)
    rc = _noalloc(moe, [t] * 600, [t] * 600, 4, out)
    assert rc == -2  # MOE_ERR_UNSUPPORTED: limit is 1024 tensors per call
    assert "1024" in moe.lib.moe_last_error().decode()
