"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, and its host-side queries and argument validation
behave as documented (a rejected call returns before any CUDA call)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**\s*((?:moe|sparseclip)_\w+)\s*\(",
                                 src, flags=re.M)))


@pytest.fixture(scope="module")
def moe():
    import sparse_mixture_experts_fwd_b200 as m
    return m


def test_every_declared_symbol_is_exported(moe):
    names = declared_functions()
    assert len(names) >= 18, names
    raw = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in moe_b200.h but not exported"
    assert set(names) == set(moe.SIGNATURES), "binding signatures out of sync with the header"


def test_struct_layout(moe):
    assert moe.lib.moe_abi_version() == 3
    assert moe.lib.moe_config_size() == 56 == ctypes.sizeof(moe.MoEConfig)
    assert moe.lib.moe_workspace_map_size() == ctypes.sizeof(moe.WorkspaceMap)


def test_capacity_eq3(moe):
    # Switch notes sec. 2.2 eq. (3) at the five workloads, and the floor reading
    assert [moe.capacity(T, E, cf) for T, E, cf in
            [(256, 8, 1.0), (8192, 128, 1.25), (16384, 64, 2.0), (32768, 64, 1.25),
             (65536, 256, 1.0)]] == [32, 80, 512, 640, 256]
    assert moe.capacity(10, 3, 1.0) == 3
    assert moe.capacity(10, 0, 1.0) == -1
    assert moe.capacity(-1, 2, 1.0) == -1


def cfg(moe, **kw):
    base = dict(T=8192, d_model=768, d_ff=3072, E=128, k=1, capacity_=80)
    base.update(kw)
    import torch
    dtype = base.pop("dtype", torch.bfloat16)
    dtype = torch.float32 if dtype == "f32" else dtype
    return moe.make_config(base.pop("T"), base.pop("d_model"), base.pop("d_ff"), base.pop("E"),
                           base.pop("k"), base.pop("capacity_"), dtype=dtype, **base)


@pytest.mark.parametrize("kw,code", [
    (dict(E=0), -1), (dict(E=512), -2), (dict(k=3), -2), (dict(k=2, E=1), -1),
    (dict(capacity_=-1), -1), (dict(d_model=100), -2), (dict(d_ff=96), -2),
    (dict(mode="rre", k=2, num_groups=8), -1), (dict(mode="rre", num_groups=3), -1),
    (dict(T=-5), -1), (dict(expert="geglu", dtype="f32"), -2),
    (dict(T=2 ** 30, k=2), -2),  # T * k = 2^31 choices: counts and slots are 32-bit
])
def test_config_rejections(moe, kw, code):
    c = cfg(moe, **kw)
    assert moe.lib.moe_config_check(ctypes.byref(c)) == code
    assert moe.lib.moe_last_error().decode() != ""
    assert moe.lib.moe_workspace_size(ctypes.byref(c)) == 0


def test_config_accepts_workloads(moe):
    import torch
    import synth
    for w in synth.WORKLOADS.values():
        C = moe.capacity(w.T, w.E, w.capacity_factor)
        c = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, C, dtype=w.torch_dtype, mode=w.mode,
                            num_groups=w.num_groups, seed=w.seed)
        assert moe.lib.moe_config_check(ctypes.byref(c)) == 0, w.name
        m = moe.workspace_layout(c)
        es = 2 if w.dtype == "bf16" else 4
        offs = [m.logits, m.expert_idx, m.gate, m.slot, m.kept, m.tok_of_row, m.arrivals,
                m.kept_cnt, m.n_dropped, m.scratch, m.ffn_sync, m.xe, m.H, m.ye, m.total]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert m.total - m.ye >= w.E * C * w.d_model * es
        assert m.ye - m.H >= w.E * C * w.d_ff * es


def test_calls_rejected_on_host(moe):
    import torch  # noqa: F401
    c = cfg(moe)
    p = ctypes.c_void_p(4096)  # aligned dummy, never dereferenced: validation fails first
    # null x
    assert moe.lib.moe_router(ctypes.byref(c), None, p, None, p, None, None) == -1
    # misaligned logits
    assert moe.lib.moe_router(ctypes.byref(c), p, p, None, ctypes.c_void_p(4100), None, None) == -3
    # workspace too small
    assert moe.lib.moe_layer_forward(ctypes.byref(c), p, p, None, None, p, p, p, p, 10, None, None,
                                     None) == -4
    # topk_assign without its gate output
    assert moe.lib.moe_topk_assign(ctypes.byref(c), p, None, p, None, p, p, p, p, p, p, None, 0,
                                   None, None) == -1
    # the assignment takes no scratch: the size is 0 and a null workspace passes validation
    assert moe.lib.moe_assign_workspace_size(ctypes.byref(c)) == 0
    # invalid config reaches no launch
    bad = cfg(moe, k=3)
    assert moe.lib.moe_expert_ffn(ctypes.byref(bad), p, p, p, p, p, p, p, 4096, None, None) == -2
    # bf16 expert FFN without its tile-counter workspace
    assert moe.lib.moe_expert_ffn(ctypes.byref(c), p, p, p, p, p, p, None, 0, None, None) == -4
    assert moe.lib.moe_ffn_workspace_size(ctypes.byref(c)) == 768  # 4 * (1 + 128) -> 256-aligned
    assert moe.lib.moe_dispatch(None, p, p, p, p, p, None, None) == -1
    # sparseclip
    assert moe.lib.sparseclip_norm(None, None, 0, None, None, 0, 0, p, p, 1 << 20, None) == -1
    assert moe.lib.sparseclip_workspace_size(1, 64) == 1024 * 2 * 8
    assert moe.lib.sparseclip_workspace_size(-1, 0) == 0
    # aux loss: RRE has no learned gate, out is required and 8-byte aligned,
    # the workspace must be moe_aux_workspace_size bytes
    ws = moe.lib.moe_aux_workspace_size(ctypes.byref(c))
    assert ws > 0 and ws % 256 == 0
    rre = cfg(moe, mode="rre", num_groups=4)
    assert moe.lib.moe_aux_loss(ctypes.byref(rre), p, 0.01, p, None, None, p, 1 << 30, None) == -2
    assert moe.lib.moe_aux_loss(ctypes.byref(c), p, 0.01, None, None, None, p, ws, None) == -1
    assert moe.lib.moe_aux_loss(ctypes.byref(c), p, 0.01, ctypes.c_void_p(4100), None, None, p, ws,
                                None) == -3
    assert moe.lib.moe_aux_loss(ctypes.byref(c), p, 0.01, p, None, None, p, ws - 1, None) == -4


def test_expert_parallel_host_checks(moe):
    """moe_ep_ffn_config derives the per-rank FFN config; the EP calls reject
    bad rank/world, world not dividing E and unaligned or missing peer
    pointers before any launch."""
    c = cfg(moe)  # E = 128
    out = moe.MoEConfig()
    for world in (1, 2, 4, 8):
        assert moe.lib.moe_ep_ffn_config(ctypes.byref(c), world, ctypes.byref(out)) == 0
        assert (out.E, out.capacity) == (c.E // world, world * c.capacity)
        assert (out.T, out.d_model, out.d_ff, out.dtype, out.expert) == \
            (c.T, c.d_model, c.d_ff, c.dtype, c.expert)
        assert (out.k, out.mode, out.num_groups) == (1, 0, 1)
    for world in (0, 9, -1):
        assert moe.lib.moe_ep_ffn_config(ctypes.byref(c), world, ctypes.byref(out)) == -1
    c3 = cfg(moe, E=6)
    assert moe.lib.moe_ep_ffn_config(ctypes.byref(c3), 4, ctypes.byref(out)) == -1
    assert moe.lib.moe_ep_ffn_config(ctypes.byref(c), 2, None) == -1
    # RRE layers keep their routing fields on the caller's side only
    rre = cfg(moe, mode="rre", num_groups=4)
    assert moe.lib.moe_ep_ffn_config(ctypes.byref(rre), 8, ctypes.byref(out)) == 0
    assert (out.E, out.mode, out.num_groups) == (16, 0, 1)

    p = ctypes.c_void_p(4096)
    peers = (ctypes.c_void_p * 2)(4096, 8192)
    bad_peers = (ctypes.c_void_p * 2)(4096, 8200)
    null_peer = (ctypes.c_void_p * 2)(4096, None)
    disp = moe.lib.moe_ep_dispatch
    assert disp(ctypes.byref(c), 2, 2, p, p, p, p, p, peers, p, None, None) == -1   # rank >= world
    assert disp(ctypes.byref(c), 0, 9, p, p, p, p, p, peers, p, None, None) == -1   # world > 8
    assert disp(ctypes.byref(c3), 0, 4, p, p, p, p, p, peers, p, None, None) == -1  # 4 does not divide 6
    assert disp(ctypes.byref(c), 0, 2, p, p, p, p, p, bad_peers, p, None, None) == -3
    assert disp(ctypes.byref(c), 0, 2, p, p, p, p, p, null_peer, p, None, None) == -1
    assert disp(ctypes.byref(c), 0, 2, p, p, p, p, p, None, p, None, None) == -1
    assert disp(ctypes.byref(c), 0, 2, p, p, p, p, None, peers, p, None, None) == -1  # cnt_all
    comb = moe.lib.moe_ep_combine
    assert comb(ctypes.byref(c), 0, 2, peers, p, p, p, p, p, None, None, None) == -1   # y null
    assert comb(ctypes.byref(c), 0, 2, bad_peers, p, p, p, p, p, p, None, None) == -3
    assert comb(ctypes.byref(c), 3, 2, peers, p, p, p, p, p, p, None, None) == -1


def test_expert_parallel_binding_host_side(moe):
    """The Python side of the EP calls: the peer table, the per-rank FFN config
    and the refusal of CPU tensors, all before any CUDA call."""
    import torch
    t = moe._peer_table([4096, 8192], 2, "xe_peers")
    assert list(t) == [4096, 8192]
    assert moe._peer_table(None, 2, "xe_peers") is None
    with pytest.raises(ValueError, match="needs 2 entries"):
        moe._peer_table([4096], 2, "xe_peers")
    c = cfg(moe, T=4, d_model=64, d_ff=64, E=4, capacity_=2)
    f = moe.ep_ffn_config(c, 2)
    assert (f.E, f.capacity, f.T, f.d_model) == (2, 4, 4, 64)
    with pytest.raises(moe.MoEError, match="does not divide"):
        moe.ep_ffn_config(c, 3)
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    idx = torch.zeros(4, 1, dtype=torch.int32)
    cnt = torch.zeros(2, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        moe.ep_dispatch(c, 0, 2, x, idx, idx, idx.to(torch.uint8), cnt, [4096, 8192],
                        local_cnt=torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        moe.ep_combine(c, 0, 2, [4096, 8192], idx, torch.ones(4, 1), idx, idx.to(torch.uint8),
                       cnt, y=x)


def test_library_refuses_cpu_tensors(moe):
    import torch
    c = cfg(moe, T=4, d_model=64, d_ff=64, E=16, capacity_=1)
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        moe.router(c, x, torch.zeros(16, 64, dtype=torch.bfloat16),
                   logits=torch.zeros(4, 16))


def _expected_check(T, d, f, E, k, C, mode, G, dtype, expert):
    """The validity rules of moe_config as the C header documents them, restated."""
    I32 = 2 ** 31 - 1
    if T < 0 or T > I32 or E < 1:
        return -1
    if E > 256 or k not in (1, 2):
        return -2
    if k > E or C < 0:
        return -1
    if mode == 1 and (k != 1 or G < 1 or E % G):
        return -1
    if expert == 1 and dtype != 0:
        return -2
    if d < 1 or f < 1:
        return -1
    if (dtype == 0 and (d % 64 or f % 64)) or (dtype == 1 and (d % 4 or f % 4)):
        return -2
    if E * C > I32 or E * f * 2 > I32 or E * d > I32:
        return -2
    if T * k > I32:
        return -2
    return 0


def test_config_check_property(moe):
    """moe_config_check agrees with the documented rules on random configs, and
    every accepted config gets an ordered, 256-byte aligned workspace layout."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    @hyp.settings(max_examples=400, deadline=None, derandomize=True)
    @hyp.given(T=st.integers(-3, 3 * 2 ** 20), d=st.sampled_from([0, 4, 32, 64, 100, 128, 768]),
               f=st.sampled_from([0, 4, 48, 64, 96, 256, 3072]), E=st.integers(-1, 300),
               k=st.integers(0, 3), C=st.integers(-2, 5000), mode=st.integers(0, 1),
               G=st.integers(0, 9), dtype=st.integers(0, 1), expert=st.integers(0, 1))
    def check(T, d, f, E, k, C, mode, G, dtype, expert):
        c = moe.MoEConfig(T=T, d_model=d, d_ff=f, E=E, k=k, capacity=C, mode=mode, num_groups=G,
                          dtype=dtype, expert=expert, reserved=0, seed=1)
        want = _expected_check(T, d, f, E, k, C, mode, G, dtype, expert)
        assert moe.lib.moe_config_check(ctypes.byref(c)) == want
        if want != 0:
            assert moe.lib.moe_workspace_size(ctypes.byref(c)) == 0
            return
        m = moe.workspace_layout(c)
        es = 2 if dtype == 0 else 4
        offs = [m.logits, m.expert_idx, m.gate, m.slot, m.kept, m.tok_of_row, m.arrivals,
                m.kept_cnt, m.n_dropped, m.scratch, m.ffn_sync, m.xe, m.H, m.ye, m.total]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert m.expert_idx - m.logits >= (T * E * 4 if (mode == 0 and dtype == 1) else 0)
        assert m.gate - m.expert_idx >= T * k * 4 and m.kept_cnt - m.arrivals >= E * 4
        assert m.tok_of_row - m.kept >= T * k and m.arrivals - m.tok_of_row >= E * C * 4
        assert m.H - m.xe >= E * C * d * es and m.ye - m.H >= E * C * f * es
        assert m.total - m.ye >= E * C * d * es
        assert moe.lib.moe_workspace_size(ctypes.byref(c)) == m.total

    check()
