"""Failure path on the GPU: a bounded wait that can never be met ends the
whole grid within about one wait limit and reports MOE_STATUS_TIMEOUT; the
context stays usable and the next call is correct.

The wait that runs out is the fused expert FFN's GEMM-2 dependency wait
(the tiles of an expert's second GEMM wait until its first GEMM has stored
every slice of H).  The test starts the kernel from a counter state that no
tile can complete: the workspace is zeroed by the test (flag
MOE_FFN_WORKSPACE_ZEROED) and expert 0's counter starts at -1, one short of
the total its GEMM-1 tiles add, so expert 0's GEMM-2 tiles wait until the
limit.  Nothing faults, traps or spins
without a bound: the limit is set to a few milliseconds for this call only.
"""
import time

import pytest
import torch

import oracle
import synth
from parity_util import assert_close, threads

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000  # 5 ms


@pytest.fixture(scope="module")
def moe(cuda_device):
    import sparse_mixture_experts_fwd_b200 as m
    return m


# C <= 128: the single-CTA persistent kernel (one counter per expert);
# C >= 512, d >= 2048: the one-launch SM-pair kernel (one counter per chunk of
# at most 256 rows of an expert; expert 0's first chunk is word 1 as well)
FFN_CASES = {
    "single_cta": (12, 100, 128, 512, [100, 37, 0, 64, 99, 1, 100, 50, 80, 100, 3, 70]),
    "sm_pairs": (4, 600, 2048, 256, [600, 300, 17, 512]),
}


def _ffn_case(name):
    E, C, d, f, kept_list = FFN_CASES[name]
    kept = torch.tensor(kept_list, dtype=torch.int32)
    xe = synth.normal(31, 1, (E, C, d), 1.0, torch.bfloat16)
    W1 = synth.normal(31, 3, (E, f, d), 0.02, torch.bfloat16)
    W2 = synth.normal(31, 4, (E, d, f), 0.02, torch.bfloat16)
    return E, C, d, f, kept, xe, W1, W2


def _wait_event(ev, seconds):
    deadline = time.monotonic() + seconds
    while not ev.query():
        if time.monotonic() > deadline:
            return False
        time.sleep(0.002)
    return True


@pytest.mark.parametrize("kernel", sorted(FFN_CASES))
def test_unmet_wait_ends_grid_with_timeout_status(moe, cuda_device, kernel):
    dev = cuda_device
    E, C, d, f, kept, xe, W1, W2 = _ffn_case(kernel)
    cfg = moe.make_config(1, d, f, E, 1, C, dtype=torch.bfloat16)
    xe_d, W1_d, W2_d, kept_d = xe.to(dev), W1.to(dev), W2.to(dev), kept.to(dev)
    H = torch.empty(E, C, f, dtype=torch.bfloat16, device=dev)
    ye = torch.empty(E, C, d, dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(max(256, moe.ffn_workspace_size(cfg)), dtype=torch.uint8, device=dev)
    # expert 0's (first chunk's) counter starts one short: it ends at its total - 1
    ws.view(torch.int32)[1] = -1
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    assert moe.wait_limit_ns() == 1_000_000_000
    moe.set_wait_limit_ns(LIMIT_NS)
    try:
        assert moe.wait_limit_ns() == LIMIT_NS
        start.record()
        moe.expert_ffn(cfg, xe_d, W1_d, W2_d, kept_d, H=H, ye=ye, workspace=ws, status=status,
                       flags=moe.FFN_WORKSPACE_ZEROED)
        end.record()
    finally:
        moe.set_wait_limit_ns(0)  # later launches get the default 1 s again
    assert moe.wait_limit_ns() == 1_000_000_000
    # the host never blocks on the device here: it polls, and gives up after 10 s
    assert _wait_event(end, 10.0), "the call did not end within 10 s"
    ms = start.elapsed_time(end)
    words = ws.view(torch.int32)[:1 + E].cpu().tolist()
    assert int(status.item()) & moe.STATUS_TIMEOUT, \
        f"status {int(status.item())} after {ms:.2f} ms; counters {words}"
    # every thread block gave up within a few limits (one per block would be ~150 x 5 ms)
    assert ms < 200.0, f"the grid took {ms:.1f} ms to give up"

    # the context is still usable: the same call from a zeroed workspace is correct
    status.zero_()
    H2 = torch.full((E, C, f), float("nan"), dtype=torch.bfloat16, device=dev)
    ye2 = torch.full((E, C, d), float("nan"), dtype=torch.bfloat16, device=dev)
    moe.expert_ffn(cfg, xe_d, W1_d, W2_d, kept_d, H=H2, ye=ye2, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ye_ref = oracle.expert_ffn(xe, W1, W2, kept, nthreads=threads())
    ye2 = ye2.cpu()
    for e in range(E):
        n = int(kept[e])
        assert_close(ye2[e, :n], ye_ref[e, :n], what=f"ye[{e}] after the timed-out call")


@pytest.mark.parametrize("kernel", sorted(FFN_CASES))
def test_status_timeout_bit_gives_up_at_once(moe, cuda_device, kernel):
    """A call that starts with the timeout bit already set in its status word
    gives up its waits at once (the word is the call's give-up signal) and
    still ends cleanly."""
    dev = cuda_device
    E, C, d, f, kept, xe, W1, W2 = _ffn_case(kernel)
    cfg = moe.make_config(1, d, f, E, 1, C, dtype=torch.bfloat16)
    status = torch.full((1,), moe.STATUS_TIMEOUT, dtype=torch.int32, device=dev)
    end = torch.cuda.Event()
    moe.expert_ffn(cfg, xe.to(dev), W1.to(dev), W2.to(dev), kept.to(dev), status=status)
    end.record()
    assert _wait_event(end, 10.0), "the call did not end within 10 s"
    assert int(status.item()) == moe.STATUS_TIMEOUT
