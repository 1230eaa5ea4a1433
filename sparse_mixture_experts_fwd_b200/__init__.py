"""Sparse Mixture-of-Experts layer forward for NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libmoe_b200.so`` (declared in ``include/moe_b200.h``).
Functions take CUDA torch tensors and marshal their device pointers, sizes and
the current CUDA stream into the C ABI; every step of the layer runs in the
library's CUDA kernels.  PyTorch only provides device memory and streams.

There is no CPU path: importing this package fails loudly if the library is
missing, and every call requires CUDA tensors.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_CHECK_BOUNDS=1: load the bounds-checked build (moe_bounds_checked)
CHECK_BOUNDS = os.environ.get("MOE_B200_CHECK_BOUNDS", "0") == "1"
LIB_PATH = os.path.join(_PKG, "libmoe_b200_checked.so" if CHECK_BOUNDS else "libmoe_b200.so")

MOE_OK = 0
ERRORS = {-1: "MOE_ERR_INVALID_ARGUMENT", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_ALIGNMENT",
          -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA"}
DTYPE_BF16, DTYPE_F32 = 0, 1
ROUTE_TOPK, ROUTE_RRE = 0, 1
STATUS_TIMEOUT, STATUS_BAD_DOMAIN, STATUS_BAD_COUNTS, STATUS_BAD_INDEX = 1, 2, 4, 8
FFN_WORKSPACE_ZEROED = 1

# every entry point the header declares, with its ctypes signature
_i32, _i64, _u64, _sz, _vp, _dbl = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                    ctypes.c_size_t, ctypes.c_void_p, ctypes.c_double)


class MoEConfig(ctypes.Structure):
    """Mirror of ``moe_config`` (56 bytes)."""
    _fields_ = [("T", _i64), ("d_model", _i32), ("d_ff", _i32), ("E", _i32), ("k", _i32),
                ("capacity", _i32), ("mode", _i32), ("num_groups", _i32), ("dtype", _i32),
                ("expert", _i32), ("reserved", _i32), ("seed", _u64)]


class WorkspaceMap(ctypes.Structure):
    """Mirror of ``moe_workspace_map``."""
    _fields_ = [(n, _sz) for n in ("logits", "expert_idx", "gate", "slot", "kept", "tok_of_row",
                                   "arrivals", "kept_cnt", "n_dropped", "scratch", "ffn_sync", "xe",
                                   "H", "ye",
                                   "total")]


_PCFG = ctypes.POINTER(MoEConfig)
_PVP = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "moe_abi_version": ([], _i32),
    "moe_config_size": ([], _sz),
    "moe_workspace_map_size": ([], _sz),
    "moe_error_string": ([_i32], ctypes.c_char_p),
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_capacity": ([_i64, _i32, _dbl], _i32),
    "moe_config_check": ([_PCFG], _i32),
    "moe_assign_workspace_size": ([_PCFG], _sz),
    "moe_workspace_layout": ([_PCFG, ctypes.POINTER(WorkspaceMap)], _i32),
    "moe_workspace_size": ([_PCFG], _sz),
    "sparseclip_workspace_size": ([_i32, _i32], _sz),
    "moe_router": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "moe_topk_assign": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                         _vp], _i32),
    "moe_dispatch": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "moe_ffn_workspace_size": ([_PCFG], _sz),
    "moe_expert_ffn": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp], _i32),
    "moe_expert_ffn_ex": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, ctypes.c_uint32, _vp,
                           _vp], _i32),
    "moe_set_wait_limit_ns": ([_u64], None),
    "moe_wait_limit_ns": ([], _u64),
    "moe_combine": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "moe_bounds_checked": ([], _i32),
    "moe_layer_forward": ([_PCFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp],
                          _i32),
    "moe_aux_workspace_size": ([_PCFG], _sz),
    "moe_aux_loss": ([_PCFG, _vp, _dbl, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "sparseclip_norm": ([_vp, _vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _sz, _vp], _i32),
    "sparseclip_norm_noalloc": ([_vp, _vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp], _i32),
    "sparseclip_clip": ([_vp, _vp, _i32, _vp, _vp, _i32, _i32, _dbl, _vp, _vp, _sz, _vp], _i32),
    "moe_ep_ffn_config": ([_PCFG, _i32, _PCFG], _i32),
    "moe_ep_dispatch": ([_PCFG, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _PVP, _vp, _vp, _vp], _i32),
    "moe_ep_combine": ([_PCFG, _i32, _i32, _PVP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
}


def _load_library():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python sparse_mixture_experts_fwd_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    assert lib.moe_config_size() == ctypes.sizeof(MoEConfig), "moe_config layout mismatch"
    assert lib.moe_workspace_map_size() == ctypes.sizeof(WorkspaceMap), "workspace map mismatch"
    return lib


lib = _load_library()


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        detail = lib.moe_last_error().decode()
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({detail})")
        self.code = code


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoEError(code, where)


def _dtype_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return DTYPE_BF16
    if dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"unsupported activation dtype {dtype}")


def _ptr(t, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def capacity(T: int, E: int, capacity_factor: float) -> int:
    """Eq. (3): floor(T / E * capacity_factor)."""
    return int(lib.moe_capacity(T, E, capacity_factor))


EXPERTS = {"relu": 0, "geglu": 1}


def make_config(T, d_model, d_ff, E, k, capacity_, *, dtype=torch.bfloat16, mode="topk",
                num_groups=1, seed=0, expert="relu") -> MoEConfig:
    """expert: "relu" (W1 [E, f, d]) or "geglu" (W1 [E, 2f, d], bf16 only)."""
    return MoEConfig(T=T, d_model=d_model, d_ff=d_ff, E=E, k=k, capacity=capacity_,
                     mode=ROUTE_TOPK if mode == "topk" else ROUTE_RRE, num_groups=num_groups,
                     dtype=_dtype_code(dtype), expert=EXPERTS[expert], reserved=0, seed=seed)


def config_check(cfg: MoEConfig):
    _check(lib.moe_config_check(ctypes.byref(cfg)), "moe_config_check")


def workspace_layout(cfg: MoEConfig) -> WorkspaceMap:
    m = WorkspaceMap()
    _check(lib.moe_workspace_layout(ctypes.byref(cfg), ctypes.byref(m)), "moe_workspace_layout")
    return m


def workspace_size(cfg: MoEConfig) -> int:
    return int(workspace_layout(cfg).total)


def assign_workspace_size(cfg: MoEConfig) -> int:
    config_check(cfg)
    return int(lib.moe_assign_workspace_size(ctypes.byref(cfg)))


def _act_dtype(cfg):
    return torch.bfloat16 if cfg.dtype == DTYPE_BF16 else torch.float32


def router(cfg, x, Wr, bias=None, logits=None, status=None, stream=None):
    if logits is None:
        logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=x.device)
    _check(lib.moe_router(ctypes.byref(cfg), _ptr(x, "x"), _ptr(Wr, "Wr"), _ptr(bias, "bias"),
                          _ptr(logits, "logits"), _ptr(status, "status"), _stream(stream)),
           "moe_router")
    return logits


def aux_workspace_size(cfg: MoEConfig) -> int:
    return int(lib.moe_aux_workspace_size(ctypes.byref(cfg)))


def aux_loss(cfg, logits, alpha=1e-2, workspace=None, stream=None):
    """Switch load-balancing loss and routing entropy from fp32 logits [T, E].

    Returns device float64 tensors: out [2] (loss, entropy), f [E], P [E]."""
    dev = logits.device
    out = torch.empty(2, dtype=torch.float64, device=dev)
    f = torch.empty(cfg.E, dtype=torch.float64, device=dev)
    P = torch.empty(cfg.E, dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.empty(max(256, aux_workspace_size(cfg)), dtype=torch.uint8, device=dev)
    _check(lib.moe_aux_loss(ctypes.byref(cfg), _ptr(logits, "logits"), float(alpha),
                            _ptr(out, "out"), _ptr(f, "f"), _ptr(P, "P"), _ptr(workspace, "workspace"),
                            workspace.numel(), _stream(stream)), "moe_aux_loss")
    return out, f, P


def topk_assign(cfg, logits=None, domain_id=None, out=None, workspace=None, status=None,
                stream=None):
    """Returns a dict: expert_idx, gate, slot, kept, tok_of_row, arrivals, kept_cnt, n_dropped."""
    dev = (logits if logits is not None else domain_id).device
    T, k, E, C = cfg.T, cfg.k, cfg.E, cfg.capacity
    o = out or {}
    o.setdefault("expert_idx", torch.empty(T, k, dtype=torch.int32, device=dev))
    o.setdefault("gate", torch.empty(T, k, dtype=torch.float32, device=dev))
    o.setdefault("slot", torch.empty(T, k, dtype=torch.int32, device=dev))
    o.setdefault("kept", torch.empty(T, k, dtype=torch.uint8, device=dev))
    o.setdefault("tok_of_row", torch.empty(max(1, E * C), dtype=torch.int32, device=dev))
    o.setdefault("arrivals", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("kept_cnt", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("n_dropped", torch.empty(1, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = torch.empty(max(256, assign_workspace_size(cfg)), dtype=torch.uint8, device=dev)
    _check(lib.moe_topk_assign(
        ctypes.byref(cfg), _ptr(logits, "logits"), _ptr(domain_id, "domain_id"),
        _ptr(o["expert_idx"], "expert_idx"), _ptr(o["gate"], "gate"), _ptr(o["slot"], "slot"),
        _ptr(o["kept"], "kept"), _ptr(o["tok_of_row"], "tok_of_row"),
        _ptr(o["arrivals"], "arrivals"), _ptr(o["kept_cnt"], "kept_cnt"),
        _ptr(o["n_dropped"], "n_dropped"), _ptr(workspace, "workspace"), workspace.numel(),
        _ptr(status, "status"), _stream(stream)), "moe_topk_assign")
    return o


def dispatch(cfg, x, expert_idx, slot, kept, xe=None, status=None, stream=None):
    if xe is None:
        xe = torch.empty(cfg.E, cfg.capacity, cfg.d_model, dtype=x.dtype, device=x.device)
    _check(lib.moe_dispatch(ctypes.byref(cfg), _ptr(x, "x"), _ptr(expert_idx, "expert_idx"),
                            _ptr(slot, "slot"), _ptr(kept, "kept"), _ptr(xe, "xe"),
                            _ptr(status, "status"), _stream(stream)), "moe_dispatch")
    return xe


def ffn_workspace_size(cfg: MoEConfig) -> int:
    config_check(cfg)
    return int(lib.moe_ffn_workspace_size(ctypes.byref(cfg)))


def set_wait_limit_ns(ns: int):
    """Limit of every bounded wait in the library's kernels (0 = the 1 s default)."""
    lib.moe_set_wait_limit_ns(int(ns))


def wait_limit_ns() -> int:
    return int(lib.moe_wait_limit_ns())


def expert_ffn(cfg, xe, W1, W2, kept_cnt, H=None, ye=None, workspace=None, status=None,
               stream=None, flags=0):
    """flags: FFN_WORKSPACE_ZEROED = the caller zeroed ``workspace`` on the stream already."""
    if H is None:
        H = torch.empty(cfg.E, cfg.capacity, cfg.d_ff, dtype=xe.dtype, device=xe.device)
    if ye is None:
        ye = torch.empty(cfg.E, cfg.capacity, cfg.d_model, dtype=xe.dtype, device=xe.device)
    if workspace is None:
        workspace = torch.empty(max(256, ffn_workspace_size(cfg)), dtype=torch.uint8,
                                device=xe.device)
    _check(lib.moe_expert_ffn_ex(ctypes.byref(cfg), _ptr(xe, "xe"), _ptr(W1, "W1"),
                                 _ptr(W2, "W2"), _ptr(kept_cnt, "kept_cnt"), _ptr(H, "H"),
                                 _ptr(ye, "ye"), _ptr(workspace, "workspace"), workspace.numel(),
                                 int(flags), _ptr(status, "status"), _stream(stream)),
           "moe_expert_ffn_ex")
    return H, ye


def combine(cfg, ye, expert_idx, gate, slot, kept, y=None, status=None, stream=None):
    if y is None:
        y = torch.empty(cfg.T, cfg.d_model, dtype=ye.dtype, device=ye.device)
    _check(lib.moe_combine(ctypes.byref(cfg), _ptr(ye, "ye"), _ptr(expert_idx, "expert_idx"),
                           _ptr(gate, "gate"), _ptr(slot, "slot"), _ptr(kept, "kept"),
                           _ptr(y, "y"), _ptr(status, "status"), _stream(stream)), "moe_combine")
    return y


def ep_ffn_config(cfg: MoEConfig, world: int) -> MoEConfig:
    """The expert-FFN config of one of ``world`` expert-parallel ranks:
    E / world experts, capacity world * C."""
    out = MoEConfig()
    _check(lib.moe_ep_ffn_config(ctypes.byref(cfg), int(world), ctypes.byref(out)),
           "moe_ep_ffn_config")
    return out


def _peer_table(peers, world, name):
    """Host array of ``world`` device addresses from tensors or ints (mapped peer pointers)."""
    if peers is None:
        return None
    if len(peers) != world:
        raise ValueError(f"{name} needs {world} entries, got {len(peers)}")
    addr = []
    for q, p in enumerate(peers):
        if isinstance(p, torch.Tensor):
            addr.append(_ptr(p, f"{name}[{q}]"))
        else:
            addr.append(int(p))
    return (ctypes.c_void_p * world)(*addr)


def ep_dispatch(cfg, rank, world, x, expert_idx, slot, kept, cnt_all, xe_peers, local_cnt=None,
                status=None, stream=None):
    """Expert-parallel dispatch: this rank's kept rows into their home ranks'
    receive buffers ``xe_peers`` (tensors or mapped device addresses, rank
    order).  Returns ``local_cnt`` [E / world], the rows each local expert
    receives from all ranks."""
    if local_cnt is None:
        local_cnt = torch.empty(cfg.E // world, dtype=torch.int32, device=cnt_all.device)
    _check(lib.moe_ep_dispatch(ctypes.byref(cfg), int(rank), int(world), _ptr(x, "x"),
                               _ptr(expert_idx, "expert_idx"), _ptr(slot, "slot"),
                               _ptr(kept, "kept"), _ptr(cnt_all, "cnt_all"),
                               _peer_table(xe_peers, world, "xe_peers"),
                               _ptr(local_cnt, "local_cnt"), _ptr(status, "status"),
                               _stream(stream)), "moe_ep_dispatch")
    return local_cnt


def ep_combine(cfg, rank, world, ye_peers, expert_idx, gate, slot, kept, cnt_all, y=None,
               status=None, stream=None):
    """Expert-parallel combine: y [T, d] from the home ranks' expert outputs
    ``ye_peers`` (tensors or mapped device addresses, rank order)."""
    if y is None:
        dt = torch.bfloat16 if cfg.dtype == DTYPE_BF16 else torch.float32
        y = torch.empty(cfg.T, cfg.d_model, dtype=dt, device=cnt_all.device)
    _check(lib.moe_ep_combine(ctypes.byref(cfg), int(rank), int(world),
                              _peer_table(ye_peers, world, "ye_peers"),
                              _ptr(expert_idx, "expert_idx"), _ptr(gate, "gate"),
                              _ptr(slot, "slot"), _ptr(kept, "kept"), _ptr(cnt_all, "cnt_all"),
                              _ptr(y, "y"), _ptr(status, "status"), _stream(stream)),
           "moe_ep_combine")
    return y


STAGES = ("router", "route_assign", "dispatch", "expert_ffn", "combine")


def layer_forward(cfg, x, W1, W2, *, Wr=None, bias=None, domain_id=None, y=None, workspace=None,
                  status=None, stream=None, stage_events=None):
    """The whole layer on the current stream.  Returns y; ``workspace`` keeps the intermediates.

    ``stage_events``: optional 6 ``torch.cuda.Event`` recorded before and after the
    stages named in ``STAGES`` (a profiling hook)."""
    if y is None:
        y = torch.empty(cfg.T, cfg.d_model, dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(cfg), dtype=torch.uint8, device=x.device)
    ev = None
    if stage_events is not None:
        if len(stage_events) != 6:
            raise ValueError("stage_events needs 6 events")
        s = stream if stream is not None else torch.cuda.current_stream()
        for e in stage_events:
            if e is not None and not e.cuda_event:
                e.record(s)  # torch creates its events lazily; the library re-records them
        ev = (ctypes.c_void_p * 6)(*[e.cuda_event if e is not None else None for e in stage_events])
    _check(lib.moe_layer_forward(ctypes.byref(cfg), _ptr(x, "x"), _ptr(Wr, "Wr"), _ptr(bias, "bias"),
                                 _ptr(domain_id, "domain_id"), _ptr(W1, "W1"), _ptr(W2, "W2"),
                                 _ptr(y, "y"), _ptr(workspace, "workspace"), workspace.numel(),
                                 _ptr(status, "status"),
                                 None if ev is None else ctypes.cast(ev, _vp), _stream(stream)),
           "moe_layer_forward")
    return y


def workspace_views(cfg, workspace) -> dict:
    """Tensor views of the intermediates moe_layer_forward leaves in its workspace."""
    m = workspace_layout(cfg)
    T, k, E, C, d, f = cfg.T, cfg.k, cfg.E, cfg.capacity, cfg.d_model, cfg.d_ff
    act = _act_dtype(cfg)
    es = 2 if act == torch.bfloat16 else 4

    def view(off, n, dtype, shape, itemsize):
        return workspace[off: off + n * itemsize].view(dtype).view(*shape)

    v = dict(
        expert_idx=view(m.expert_idx, T * k, torch.int32, (T, k), 4),
        gate=view(m.gate, T * k, torch.float32, (T, k), 4),
        slot=view(m.slot, T * k, torch.int32, (T, k), 4),
        kept=view(m.kept, T * k, torch.uint8, (T, k), 1),
        tok_of_row=view(m.tok_of_row, E * C, torch.int32, (E * C,), 4),
        arrivals=view(m.arrivals, E, torch.int32, (E,), 4),
        kept_cnt=view(m.kept_cnt, E, torch.int32, (E,), 4),
        n_dropped=view(m.n_dropped, 1, torch.int32, (1,), 4),
        xe=view(m.xe, E * C * d, act, (E, C, d), es),
        H=view(m.H, E * C * f, act, (E, C, f), es),
        ye=view(m.ye, E * C * d, act, (E, C, d), es),
    )
    if cfg.mode == ROUTE_TOPK and cfg.dtype == DTYPE_F32:  # bf16 layers keep no logits
        v["logits"] = view(m.logits, T * E, torch.float32, (T, E), 4)
    return v


def sparseclip_workspace_size(n_dense: int, n_sparse: int) -> int:
    return int(lib.sparseclip_workspace_size(n_dense, n_sparse))


def sparseclip_norm(dense, sparse, num_experts, out=None, workspace=None, stream=None):
    """SparseClip norm of lists of fp32 CUDA tensors; returns device double[3]
    = (norm, sum of squares dense, sum of squares expert)."""
    dense, sparse = list(dense), list(sparse)
    dev = (dense + sparse)[0].device
    if out is None:
        out = torch.empty(3, dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.empty(max(16, sparseclip_workspace_size(len(dense), len(sparse))),
                                dtype=torch.uint8, device=dev)

    def arrays(ts, name):
        ptrs = (ctypes.c_void_p * max(1, len(ts)))(*[_ptr(t, name) for t in ts])
        lens = (ctypes.c_int64 * max(1, len(ts)))(*[t.numel() for t in ts])
        return ptrs, lens

    for t in dense + sparse:
        if t.dtype != torch.float32:
            raise TypeError("SparseClip gradients must be fp32")
    dp, dl = arrays(dense, "dense")
    sp, sl = arrays(sparse, "sparse")
    _check(lib.sparseclip_norm(ctypes.cast(dp, _vp), ctypes.cast(dl, _vp), len(dense),
                               ctypes.cast(sp, _vp), ctypes.cast(sl, _vp), len(sparse),
                               num_experts, _ptr(out, "out"), _ptr(workspace, "workspace"),
                               workspace.numel(), _stream(stream)), "sparseclip_norm")
    return out


def sparseclip_clip(dense, sparse, num_experts, max_norm, out=None, workspace=None, stream=None):
    """SparseClip clipping of lists of fp32 CUDA tensors, in place; returns
    device double[4] = (norm before clipping, sum of squares dense, sum of
    squares expert, coef applied)."""
    dense, sparse = list(dense), list(sparse)
    dev = (dense + sparse)[0].device
    if out is None:
        out = torch.empty(4, dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.empty(max(16, sparseclip_workspace_size(len(dense), len(sparse))),
                                dtype=torch.uint8, device=dev)

    def arrays(ts, name):
        ptrs = (ctypes.c_void_p * max(1, len(ts)))(*[_ptr(t, name) for t in ts])
        lens = (ctypes.c_int64 * max(1, len(ts)))(*[t.numel() for t in ts])
        return ptrs, lens

    for t in dense + sparse:
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("SparseClip gradients must be contiguous fp32")
    dp, dl = arrays(dense, "dense")
    sp, sl = arrays(sparse, "sparse")
    _check(lib.sparseclip_clip(ctypes.cast(dp, _vp), ctypes.cast(dl, _vp), len(dense),
                               ctypes.cast(sp, _vp), ctypes.cast(sl, _vp), len(sparse),
                               num_experts, float(max_norm), _ptr(out, "out"),
                               _ptr(workspace, "workspace"), workspace.numel(), _stream(stream)),
           "sparseclip_clip")
    return out
