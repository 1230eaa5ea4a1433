"""ORACLE — test infrastructure only.

ctypes binding of ``moe_oracle.cpp``, the plain fp64 CPU statement of the
sparse MoE layer forward and of the SparseClip norm.  Only ``tests/``,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package; the CUDA library never calls it and shares no code with it.

All array arguments are CPU torch tensors; activation tensors are bf16 or
fp32 (their raw bits are handed over unchanged).

``MOE_ORACLE_LIB`` (environment): load that library instead of building
``libmoe_oracle.so`` — the mutation test points the pin suite at copies of
the oracle with one planted mistake each.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

DT_BF16, DT_F32 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (no CUDA) into ``oracle/libmoe_oracle.so``."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC",
                               "-pthread", _SRC, "-o", _SO])
    return _SO


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(os.environ.get("MOE_ORACLE_LIB") or build())
    i64, i32, u64, dbl, vp = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_double,
                              ctypes.c_void_p)
    sig = {
        "oracle_splitmix64": ([u64, u64], u64),
        "oracle_round_bf16": ([dbl], ctypes.c_uint16),
        "oracle_capacity": ([i64, i32, dbl], i32),
        "oracle_router": ([i64, i32, i32, i32, vp, vp, vp, vp, i32], None),
        "oracle_gate_topk": ([i64, i32, i32, vp, vp, vp, vp], None),
        "oracle_route_rre": ([i64, i32, i32, u64, vp, vp, vp], None),
        "oracle_assign": ([i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp], None),
        "oracle_dispatch": ([i64, i32, i32, i32, i32, vp, vp, vp, vp], None),
        "oracle_expert_row": ([i32, i32, i32, vp, vp, vp, vp, vp], None),
        "oracle_expert_row_geglu": ([i32, i32, i32, vp, vp, vp, vp, vp], None),
        "oracle_expert_ffn": ([i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, i32], None),
        "oracle_combine": ([i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp], None),
        "oracle_token_forward": ([i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, i32], None),
        "oracle_layer_forward": ([i64, i32, i32, i32, i32, i32, i32, i32, i32, u64] + [vp] * 19
                                 + [i32, i32], None),
        "oracle_sparseclip_norm": ([vp, vp, i32, vp, vp, i32, i32], dbl),
        "oracle_aux_loss": ([i64, i32, vp, dbl, vp, vp, vp], None),
        "oracle_sparseclip_clip": ([vp, vp, i32, vp, vp, i32, i32, dbl, vp], dbl),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def threads() -> int:
    return max(1, os.cpu_count() or 1)


def _p(t):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous CPU tensors"
    return t.data_ptr()


def _dt(t) -> int:
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_F32
    raise TypeError(f"activation dtype {t.dtype} not supported by the oracle")


def splitmix64(seed: int, t: int) -> int:
    return int(_load().oracle_splitmix64(seed, t))


def round_bf16_bits(v: float) -> int:
    return int(_load().oracle_round_bf16(v))


def capacity(T: int, E: int, capacity_factor: float) -> int:
    return int(_load().oracle_capacity(T, E, capacity_factor))


def router(x, Wr, bias=None, nthreads=None):
    T, d = x.shape
    E = Wr.shape[0]
    logits = torch.empty(T, E, dtype=torch.float32)
    _load().oracle_router(T, d, E, _dt(x), _p(x), _p(Wr), _p(bias), _p(logits),
                          nthreads or threads())
    return logits


def gate_topk(logits, k, with_prob_sum=False):
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32)
    gate = torch.empty(T, k, dtype=torch.float32)
    ps = torch.empty(T, dtype=torch.float64) if with_prob_sum else None
    _load().oracle_gate_topk(T, E, k, _p(logits), _p(idx), _p(gate), _p(ps))
    return (idx, gate, ps) if with_prob_sum else (idx, gate)


def route_rre(domain, E, G, seed):
    T = domain.shape[0]
    idx = torch.empty(T, 1, dtype=torch.int32)
    gate = torch.empty(T, 1, dtype=torch.float32)
    _load().oracle_route_rre(T, E, G, seed, _p(domain), _p(idx), _p(gate))
    return idx, gate


def assign(expert_idx, E, C):
    T, k = expert_idx.shape
    slot = torch.empty(T, k, dtype=torch.int32)
    kept = torch.empty(T, k, dtype=torch.uint8)
    tok_of_row = torch.empty(E * C, dtype=torch.int32)
    arrivals = torch.empty(E, dtype=torch.int32)
    kept_cnt = torch.empty(E, dtype=torch.int32)
    nd = torch.zeros(1, dtype=torch.int64)
    _load().oracle_assign(T, E, k, C, _p(expert_idx.contiguous()), _p(slot), _p(kept),
                          _p(tok_of_row), _p(arrivals), _p(kept_cnt), _p(nd))
    return dict(slot=slot, kept=kept, tok_of_row=tok_of_row, arrivals=arrivals,
                kept_cnt=kept_cnt, n_dropped=int(nd.item()))


def dispatch(x, tok_of_row, kept_cnt, E, C):
    T, d = x.shape
    xe = torch.zeros(E * C, d, dtype=x.dtype)
    _load().oracle_dispatch(T, d, E, C, _dt(x), _p(x), _p(tok_of_row), _p(kept_cnt), _p(xe))
    return xe.view(E, C, d)


KINDS = {"relu": 0, "geglu": 1}


def expert_row(x_row, W1_e, W2_e, with_H=False, kind="relu"):
    """One token through one expert; kind "geglu" takes W1_e [2f, d] (gate, linear rows)."""
    d = W1_e.shape[1]
    f = W2_e.shape[1]
    out = torch.empty(d, dtype=x_row.dtype)
    H = torch.empty(f, dtype=x_row.dtype) if with_H else None
    fn = _load().oracle_expert_row_geglu if kind == "geglu" else _load().oracle_expert_row
    fn(d, f, _dt(x_row), _p(x_row.contiguous()), _p(W1_e), _p(W2_e), _p(out), _p(H))
    return (out, H) if with_H else out


def expert_ffn(xe, W1, W2, kept_cnt, with_H=False, nthreads=None, kind="relu"):
    E, C, d = xe.shape
    f = W2.shape[2]
    ye = torch.zeros(E, C, d, dtype=xe.dtype)
    H = torch.zeros(E, C, f, dtype=xe.dtype) if with_H else None
    _load().oracle_expert_ffn(d, f, E, C, _dt(xe), _p(xe), _p(W1), _p(W2), _p(kept_cnt), _p(H),
                              _p(ye), nthreads or threads(), KINDS[kind])
    return (ye, H) if with_H else ye


def combine(ye, expert_idx, gate, slot, kept, T):
    E, C, d = ye.shape
    k = expert_idx.shape[1]
    y = torch.empty(T, d, dtype=ye.dtype)
    _load().oracle_combine(T, d, k, C, _dt(ye), _p(ye), _p(expert_idx), _p(gate), _p(slot),
                           _p(kept), _p(y))
    return y


def token_forward(x_row, W1, W2, expert_idx_row, gate_row, kept_row, kind="relu"):
    """Layer output of one token (eq. (2) for a single x) from full W1 [E,f,d] ([E,2f,d]
    for GEGLU), W2 [E,d,f]."""
    E, d, f = W2.shape
    k = expert_idx_row.numel()
    y = torch.empty(d, dtype=x_row.dtype)
    _load().oracle_token_forward(d, f, k, _dt(x_row), _p(x_row.contiguous()), _p(W1), _p(W2),
                                 _p(expert_idx_row.contiguous()), _p(gate_row.contiguous()),
                                 _p(kept_row.contiguous()), _p(y), KINDS[kind])
    return y


def layer_forward(x, W1, W2, *, E, k, C, Wr=None, bias=None, domain=None, G=1, seed=0,
                  with_H=False, nthreads=None, kind="relu"):
    """Every step of the layer; returns a dict of all intermediate results."""
    T, d = x.shape
    f = W2.shape[2]
    mode = 0 if domain is None else 1
    dt = x.dtype
    r = dict(
        logits=torch.zeros(T, E, dtype=torch.float32),
        expert_idx=torch.empty(T, k, dtype=torch.int32),
        gate=torch.empty(T, k, dtype=torch.float32),
        slot=torch.empty(T, k, dtype=torch.int32),
        kept=torch.empty(T, k, dtype=torch.uint8),
        tok_of_row=torch.empty(E * C, dtype=torch.int32),
        arrivals=torch.empty(E, dtype=torch.int32),
        kept_cnt=torch.empty(E, dtype=torch.int32),
        xe=torch.zeros(E, C, d, dtype=dt),
        H=torch.zeros(E, C, f, dtype=dt) if with_H else None,
        ye=torch.zeros(E, C, d, dtype=dt),
        y=torch.empty(T, d, dtype=dt),
    )
    nd = torch.zeros(1, dtype=torch.int64)
    _load().oracle_layer_forward(
        T, d, f, E, k, C, _dt(x), mode, G, seed, _p(x), _p(Wr), _p(bias), _p(domain), _p(W1),
        _p(W2), _p(r["logits"]), _p(r["expert_idx"]), _p(r["gate"]), _p(r["slot"]), _p(r["kept"]),
        _p(r["tok_of_row"]), _p(r["arrivals"]), _p(r["kept_cnt"]), _p(nd), _p(r["xe"]),
        _p(r["H"]), _p(r["ye"]), _p(r["y"]), nthreads or threads(), KINDS[kind])
    r["n_dropped"] = int(nd.item())
    return r


def sparseclip_norm(dense, sparse, E):
    """dense, sparse: lists of contiguous fp32 CPU tensors."""
    def arr(ts):
        ptrs = (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])
        lens = (ctypes.c_int64 * max(1, len(ts)))(*[t.numel() for t in ts])
        return ptrs, lens
    for t in list(dense) + list(sparse):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.device.type == "cpu"
    dp, dl = arr(dense)
    sp, sl = arr(sparse)
    return float(_load().oracle_sparseclip_norm(ctypes.cast(dp, ctypes.c_void_p),
                                                ctypes.cast(dl, ctypes.c_void_p), len(dense),
                                                ctypes.cast(sp, ctypes.c_void_p),
                                                ctypes.cast(sl, ctypes.c_void_p), len(sparse), E))


def aux_loss(logits, alpha=1e-2):
    """Switch load-balancing loss (eqs. 4-6) and mean routing entropy from fp32
    logits [T, E]: returns (loss, entropy, f [E], P [E]) in double."""
    assert logits.dtype == torch.float32 and logits.is_contiguous()
    T, E = logits.shape
    out = torch.zeros(2, dtype=torch.float64)
    f = torch.zeros(E, dtype=torch.float64)
    P = torch.zeros(E, dtype=torch.float64)
    _load().oracle_aux_loss(T, E, _p(logits), float(alpha), _p(out), _p(f), _p(P))
    return float(out[0]), float(out[1]), f, P


def sparseclip_clip(dense, sparse, E, max_norm):
    """Clip lists of contiguous fp32 CPU tensors in place; returns (coef, norm)."""
    def arr(ts):
        ptrs = (ctypes.c_void_p * max(1, len(ts)))(*[t.data_ptr() for t in ts])
        lens = (ctypes.c_int64 * max(1, len(ts)))(*[t.numel() for t in ts])
        return ptrs, lens
    for t in list(dense) + list(sparse):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.device.type == "cpu"
    dp, dl = arr(dense)
    sp, sl = arr(sparse)
    norm = ctypes.c_double(0.0)
    coef = _load().oracle_sparseclip_clip(ctypes.cast(dp, ctypes.c_void_p),
                                          ctypes.cast(dl, ctypes.c_void_p), len(dense),
                                          ctypes.cast(sp, ctypes.c_void_p),
                                          ctypes.cast(sl, ctypes.c_void_p), len(sparse), E,
                                          float(max_norm), ctypes.byref(norm))
    return float(coef), float(norm.value)
