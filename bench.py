"""Benchmark of the sparse MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the whole layer (router, gate/top-k or RRE, slot
assignment, dispatch, expert FFN, combine) over one batch of T synthetic
tokens.  The device-timed loop calls ``moe_layer_forward`` (the product entry
point) with its stage-event hook, so the step time and each stage's time come
from one run on the launching stream.  ``e2e`` times ``moe_layer_forward``
with the batch copied from pinned host memory and the output copied back
inside the timed region.

Multi-GPU (torchrun): every rank runs its own batch with replicated experts
(weak scaling, no collective on the data path); timing is the max over ranks.
``--impl reference`` times the CPU oracle instead, on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
# DRAM bytes (read + write) of the expert-FFN stage per layer step, from one ncu
# capture of the kernels as shipped (the profile named beside each number).
# A workload without a capture of its current kernels reports null.
FFN_TRAFFIC = {
    "switch_base": (1242.470e6 + 28.536e6, "profiles/ffn_tc_switch_base.md"),
    "xmoe_top2": (604.202e6 + 228.670e6 + 825.849e6 + 56.016e6, "profiles/gemm_pair_xmoe_top2.md"),
    "skewed_switch": (2218.970e6 + 73.474e6 + 2434.246e6 + 17.644e6,
                      "profiles/gemm_tc_ffn_skewed_switch.md"),
    # captured on 8 experts (same capacity and per-expert load), scaled by 64 / 8
    "pangu_rre": ((1194.575e6 + 103.069e6) * 8, "profiles/ffn_pair_pangu_rre.md"),
}
METRIC = "MoE-layer tokens/sec (1 B200); expert-FFN TFLOP/s; dispatch+combine GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="pangu_rre", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling captures: the workload cut to this many experts with the "
                         "same tokens per expert (T scaled by E'/E, same capacity)")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--expert", default="relu", choices=["relu", "geglu"],
                    help="expert network (the workloads are defined with the ReLU FFN)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loop runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
             "power.limit")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        return summarize_clock_lines(self.lines)


def summarize_clock_lines(lines):
    """Median SM clock and board power, the max clock and power limit, and every
    throttle reason seen active, from ClockSampler.QUERY lines."""
    sm, pw, mx, lim, reasons = [], [], None, None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        try:
            pw.append(float(parts[3]))
        except ValueError:
            pass
        if len(parts) > 9:
            try:
                lim = float(parts[9])
            except ValueError:
                pass
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": len(sm),
            "power_w": statistics.median(pw) if pw else None, "power_limit_w": lim}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline object)
# ---------------------------------------------------------------------------

def oracle_step_fn(w, T_s, threads=None):
    """A closure running the oracle's whole layer on the first T_s tokens of the workload."""
    import oracle
    ws = w.scaled(T=T_s)
    inp = synth.layer_inputs(ws)
    C = oracle.capacity(ws.T, ws.E, ws.capacity_factor)
    nth = threads or os.cpu_count() or 1

    def step():
        oracle.layer_forward(inp["x"], inp["W1"], inp["W2"], E=ws.E, k=ws.k, C=C, Wr=inp["Wr"],
                             bias=inp["bias"], domain=inp["domain"], G=ws.num_groups, seed=ws.seed,
                             nthreads=nth, kind=ws.expert)
    return step, nth


def size_oracle_sample(w, seconds):
    """Pick a token count whose oracle step takes about `seconds`."""
    T_s = min(w.T, max(64, int(4 * w.E / w.capacity_factor) + 1))  # capacity >= 4 in the probe
    step, _ = oracle_step_fn(w, T_s)
    t0 = time.perf_counter()
    step()
    dt = max(1e-3, time.perf_counter() - t0)
    return int(max(32, min(w.T, T_s * seconds / dt)))


def cpu_baseline(w, seconds):
    T_s = size_oracle_sample(w, seconds / 2)
    step, nth = oracle_step_fn(w, T_s)
    t0 = time.perf_counter()
    step()
    dt = time.perf_counter() - t0
    # the same oracle on one thread, on a sample sized from the multithreaded
    # rate for about a quarter of `seconds`
    T_1 = max(16, min(T_s, int(T_s / max(dt, 1e-6) / nth * seconds / 4)))
    step1, _ = oracle_step_fn(w, T_1, threads=1)
    t1 = time.perf_counter()
    step1()
    dt1 = time.perf_counter() - t1
    return {"value": T_s / dt, "unit": "tokens/s", "cores": nth, "kind": "oracle",
            "sample": f"whole layer on the first {T_s} of {w.T} tokens (capacity from eq. 3 at "
                      f"T={T_s}), fp64 CPU oracle, {nth} threads, one timed pass of {dt:.2f} s",
            "value_1thread": T_1 / dt1,
            "sample_1thread": f"whole layer on the first {T_1} tokens (capacity from eq. 3 at "
                              f"T={T_1}), 1 thread, {dt1:.2f} s"}


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    T_s = size_oracle_sample(w, 1.0)
    step, nth = oracle_step_fn(w, T_s)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = T_s * args.steps / dt
    out = {"impl": "reference", "metric": METRIC, "value": value,
           "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff,
                      "E": w.E, "k": w.k, "capacity_factor": w.capacity_factor,
                      "routing": w.mode, "tokens_per_step_sampled": T_s},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nth, "kind": "oracle",
                            "sample": f"whole layer on the first {T_s} of {w.T} tokens per step"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# the B200 arm
# ---------------------------------------------------------------------------

def kernel_launches(w, C):
    """Kernels ``moe_layer_forward`` launches per step (T > 0), stage by stage."""
    bf16 = w.dtype == "bf16"
    if w.mode == "rre":
        route = 2                       # RRE choice, slot assignment
    elif bf16:
        route = 2                       # router GEMM with gate/top-k epilogue, slot assignment
    else:
        route = 3                       # fp32 router, gate/top-k, slot assignment
    # bf16: one persistent kernel for both GEMMs when C <= 128 (single CTAs) or
    # C >= 512 with d_model >= 2048 (SM pairs); two grouped launches otherwise;
    # fp32: two FMA GEMMs
    ffn = 1 if (bf16 and (C <= 128 or (C >= 512 and w.d_model >= 2048))) else 2
    combine = 0 if (bf16 and w.k == 1) else 1   # top-1 bf16: inside the FFN's GEMM 2
    return route + 1 + ffn + combine


def stage_work(w, C, es, n_kept, tok_any):
    """Algorithmic bytes and flops of each stage of one layer step.

    Bytes count each tensor the stage must read or write once (activations,
    weights, routing arrays); H, the FFN's hidden activations, is
    implementation traffic and is not counted.
    """
    T, d, f, E, k = w.T, w.d_model, w.d_ff, w.E, w.k
    fused_combine = w.k == 1 and w.dtype == "bf16"
    st = {}
    assign_out = 5 * T * k + 4 * E * C + 8 * E   # slot, kept, row -> token map, counts
    if w.mode == "rre":
        st["router"] = (0, 0.0)
        # domain ids in, expert index and gate out, then the assignment
        st["route_assign"] = (4 * T + 8 * T * k + assign_out, 0.0)
    elif w.dtype == "bf16":
        # logits stay in TMEM: x, W_r (and bias) in, expert index and gate out
        st["router"] = (T * d * es + E * d * es + (4 * E if w.hot_experts else 0) + 8 * T * k,
                        2.0 * T * d * E)
        st["route_assign"] = (4 * T * k + assign_out, 0.0)
    else:
        st["router"] = (T * d * es + E * d * es + 4 * T * E, 2.0 * T * d * E)
        st["route_assign"] = (4 * T * E + 8 * T * k + assign_out, 0.0)
    disp = (tok_any + n_kept) * d * es + 9 * T * k
    if fused_combine:
        disp += (T - tok_any) * d * es                    # dropped tokens' output rows zeroed
    st["dispatch"] = (disp, 0.0)
    glu = w.expert == "geglu"  # W1 has 2f rows: 3 weight matrices' worth, 6 d f flops per row
    st["expert_ffn"] = ((3 if glu else 2) * E * d * f * es + 2 * n_kept * d * es,
                        (6.0 if glu else 4.0) * n_kept * d * f)
    st["combine"] = (0 if fused_combine else (n_kept + T) * d * es + 9 * T * k, 0.0)
    return st


def stage_roofline(st, stage_ms, peaks):
    """Per stage: time at the roofline (the slower of bytes at HBM and flops at
    the sustained bf16 peak) over the measured stage time."""
    out = {}
    for n, (b, fl) in st.items():
        ms = stage_ms[n]
        t_roof = max(b / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops_sustained"] * 1e12))
        out[n] = {"ms": round(ms, 5), "bytes": b, "flops": fl,
                  "bound": "tensor" if fl / (peaks["bf16_tflops_sustained"] * 1e12) >
                  b / (peaks["hbm_gbs"] * 1e9) else "hbm",
                  "gbs": round(b / (ms / 1e3) / 1e9, 1) if ms > 0 else None,
                  "frac": round(t_roof / (ms / 1e3), 3) if ms > 0 and (b or fl) else None}
    return out


def run_b200(args, w, world, rank, local):
    import sparse_mixture_experts_fwd_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    es = 2 if w.dtype == "bf16" else 4
    C = moe.capacity(w.T, w.E, w.capacity_factor)
    cfg = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, C, dtype=w.torch_dtype, mode=w.mode,
                          num_groups=w.num_groups, seed=w.seed, expert=w.expert)
    inp = synth.layer_inputs(w, x_seed_offset=rank)
    W1, W2 = inp["W1"].to(dev), inp["W2"].to(dev)
    Wr = None if inp["Wr"] is None else inp["Wr"].to(dev)
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    x_bytes = w.T * w.d_model * es
    n_rot = max(2, -(-2 * L2_BYTES // x_bytes))  # rotate batches: > 2x L2 of distinct x
    xs = [inp["x"].to(dev)]
    doms = [None if inp["domain"] is None else inp["domain"].to(dev)]
    gen_extra = synth.layer_inputs
    for r in range(1, n_rot):
        extra = gen_extra(w, weights=False, x_seed_offset=rank + 1000 * r)
        xs.append(extra["x"].to(dev))
        doms.append(None if extra["domain"] is None else extra["domain"].to(dev))
    ws = torch.empty(moe.workspace_size(cfg), dtype=torch.uint8, device=dev)
    v = moe.workspace_views(cfg, ws)
    y = torch.empty(w.T, w.d_model, dtype=w.torch_dtype, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    asg = {k: v[k] for k in ("expert_idx", "kept", "kept_cnt", "n_dropped")}
    stage_names = list(moe.STAGES)

    def step(i, evs=None):
        # one pass of the whole layer through the product entry point; the
        # library records `evs` (6 events) between its stages on `stream`
        moe.layer_forward(cfg, xs[i % n_rot], W1, W2, Wr=Wr, bias=bias,
                          domain_id=doms[i % n_rot], y=y, workspace=ws, status=status,
                          stream=stream, stage_events=evs)

    launches_per_step = kernel_launches(w, C)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for row in evs:  # create the events outside the timed region (torch creates lazily)
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    with ClockSampler(gpu_id) as clk:
        # untimed pre-roll so the clock samples cover at least 1.5 s under this load
        t_end = time.perf_counter() + 1.5
        i = 0
        with torch.cuda.stream(stream):
            while time.perf_counter() < t_end:
                step(i)
                i += 1
                if i % 32 == 0:
                    stream.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        # (A) the timed region: exactly K steps, events only at its two ends
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                step(args.warmup + i)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        # (B) K more steps with the library's stage events (each event record
        # serialises the stream, so these steps are slightly slower): the
        # per-stage split and the expert-FFN time of the roofline
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                step(args.warmup + args.steps + i, evs[i])
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    total_ms = t0.elapsed_time(t1)
    stage_ms = {n: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps
                for j, n in enumerate(stage_names)}
    total_ms_max = max_over_ranks(total_ms, world)

    # routing statistics of the last step (same every step up to x)
    kept_cnt = asg["kept_cnt"].cpu()
    n_kept = int(kept_cnt.sum())
    n_dropped = int(asg["n_dropped"].item())
    tok_any = int((asg["kept"].cpu().sum(1) > 0).sum())

    # algorithmic work of every stage; the expert FFN is the dominant one
    st = stage_work(w, C, es, n_kept, tok_any)
    stages = stage_roofline(st, stage_ms, peaks)
    ffn_bytes, ffn_flops = st["expert_ffn"]
    ffn_s = stage_ms["expert_ffn"] / 1e3
    # top-1 bf16 layers combine inside the expert FFN (its GEMM-2 epilogue writes
    # gate * row to y); the dispatch kernel then also zeroes the dropped tokens' rows
    fused_combine = w.k == 1 and w.dtype == "bf16"
    disp_bytes, comb_bytes = st["dispatch"][0], st["combine"][0]
    dc_s = (stage_ms["dispatch"] + (0.0 if fused_combine else stage_ms["combine"])) / 1e3
    # the FFN runs inside a long step: the sustained bf16 figure is its tensor peak
    if stages["expert_ffn"]["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": ffn_bytes / ffn_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": ffn_flops / ffn_s / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = FFN_TRAFFIC.get(w.name) if w.expert == "relu" else None
    roof["traffic"] = tr[0] if tr else None
    roof["traffic_unit"] = "bytes per expert-FFN stage (ncu dram__bytes_read + write)"
    roof["traffic_source"] = tr[1] if tr else None
    roof["algorithmic_bytes"] = ffn_bytes
    roof["kernel"] = ("expert FFN: " + (
        "grouped_gemm_f32_kernel x2" if w.dtype == "f32" else
        "ffn_tc_kernel x1 (both GEMMs fused)" if C <= 128 else
        "gemm_tc_kernel x2 (H = ReLU(xe W1^T), ye = H W2^T)" if C < 512 else
        "ffn_pair_kernel x1 on SM pairs (both GEMMs fused, tokens on the MMA's N side)"
        if w.d_model >= 2048 else
        "gemm_pair_kernel x2 on SM pairs (H = ReLU(xe W1^T), ye = H W2^T)"))
    roof["peak_source"] = peaks["source"]
    roof["algorithmic_per_launch"] = (f"{ffn_bytes / 1e9:.4f} GB" if roof["bound"] == "hbm"
                                      else f"{ffn_flops / 1e12:.4f} TFLOP")

    # ---- Switch load-balancing loss + routing entropy (top-k layers) ----
    # From the fp32 logits of this batch (moe_router); K back-to-back calls of
    # the C entry point timed with events on the stream.  Each call reads the
    # T x E logits once (two launches).
    aux = None
    if w.mode == "topk":
        import ctypes
        logits = moe.router(cfg, xs[0], Wr, bias, stream=stream)
        aux_ws = torch.empty(max(256, moe.aux_workspace_size(cfg)), dtype=torch.uint8, device=dev)
        aux_out = torch.empty(2, dtype=torch.float64, device=dev)
        aux_args = (ctypes.byref(cfg), ctypes.c_void_p(logits.data_ptr()), 1e-2,
                    ctypes.c_void_p(aux_out.data_ptr()), None, None,
                    ctypes.c_void_p(aux_ws.data_ptr()), aux_ws.numel(),
                    ctypes.c_void_p(stream.cuda_stream))
        for _ in range(3):
            assert moe.lib.moe_aux_loss(*aux_args) == 0
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            moe.lib.moe_aux_loss(*aux_args)
        a1.record(stream)
        torch.cuda.synchronize()
        aux_ms = a0.elapsed_time(a1) / args.steps
        aux_bytes = w.T * w.E * 4
        aux = {"ms": aux_ms, "bytes": aux_bytes, "gbs": aux_bytes / (aux_ms / 1e3) / 1e9,
               "frac_hbm": aux_bytes / (peaks["hbm_gbs"] * 1e9) / (aux_ms / 1e3),
               "loss": float(aux_out[0]), "entropy": float(aux_out[1]), "alpha": 1e-2,
               "note": "moe_aux_loss on this batch's fp32 router logits, back-to-back calls"}

    # ---- SparseClip norm and clipping step (workloads that carry gradients) ----
    # The norm reads every gradient once; the clip reads them for the norm and
    # then reads and writes them (coef ~ 1/2 on every call, so the write path
    # runs each time).  Gradients total 2.35 GB for the X-MoE workload.
    sclip = None
    if w.clip_dense and rank == 0:
        gd, gs = synth.sparseclip_inputs(w)
        gd = [t.to(dev) for t in gd]
        gs = [t.to(dev) for t in gs]
        n_el = sum(t.numel() for t in gd + gs)
        sc_ws = torch.empty(max(16, moe.sparseclip_workspace_size(len(gd), len(gs))),
                            dtype=torch.uint8, device=dev)
        sc_out = torch.empty(4, dtype=torch.float64, device=dev)
        for _ in range(3):
            moe.sparseclip_norm(gd, gs, w.E, out=sc_out, workspace=sc_ws, stream=stream)
        torch.cuda.synchronize()
        norm0 = float(sc_out[0])
        reps = min(args.steps, 20)
        c0, c1, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        c0.record(stream)
        for _ in range(reps):
            moe.sparseclip_norm(gd, gs, w.E, out=sc_out, workspace=sc_ws, stream=stream)
        c1.record(stream)
        for i in range(reps):
            moe.sparseclip_clip(gd, gs, w.E, norm0 * 0.5 ** (i + 1), out=sc_out, workspace=sc_ws,
                                stream=stream)
        c2.record(stream)
        torch.cuda.synchronize()
        norm_ms = c0.elapsed_time(c1) / reps
        clip_ms = c1.elapsed_time(c2) / reps
        nb, cb = 4 * n_el, 12 * n_el
        sclip = {"elements": n_el, "norm_ms": norm_ms, "norm_bytes": nb,
                 "norm_gbs": nb / (norm_ms / 1e3) / 1e9,
                 "norm_frac_hbm": nb / (peaks["hbm_gbs"] * 1e9) / (norm_ms / 1e3),
                 "clip_ms": clip_ms, "clip_bytes": cb, "clip_gbs": cb / (clip_ms / 1e3) / 1e9,
                 "clip_frac_hbm": cb / (peaks["hbm_gbs"] * 1e9) / (clip_ms / 1e3),
                 "coef_last": float(sc_out[3]),
                 "note": "sparseclip_norm, and sparseclip_clip (norm + in-place scale by ~1/2), "
                         "back-to-back calls on the workload's fp32 gradients"}
        del gd, gs
        torch.cuda.empty_cache()

    # ---- expert parallelism: two ranks emulated on this GPU ----
    # Both ranks' receive buffers live on this device and each rank's peer
    # table lists both, so the EP kernels issue the stores and loads they would
    # send over NVLink, here against HBM.  Rank 0 routes this batch, rank 1
    # the next rotated batch; the steps run in the order the cross-rank
    # barriers impose (both dispatches, both expert FFNs, both combines).
    ep = None
    if world == 1 and w.E % 2 == 0:
        P = 2
        fcfg = moe.ep_ffn_config(cfg, P)
        El, PC = fcfg.E, fcfg.capacity
        rk = []
        for q in range(P):
            xq, dq = xs[q % n_rot], doms[q % n_rot]
            if w.mode == "topk":
                ro = moe.topk_assign(cfg, logits=moe.router(cfg, xq, Wr, bias, stream=stream),
                                     stream=stream)
            else:
                ro = moe.topk_assign(cfg, domain_id=dq, stream=stream)
            rk.append({"x": xq, "ro": ro,
                       "xe": torch.empty(El, PC, w.d_model, dtype=w.torch_dtype, device=dev),
                       "ye": torch.empty(El, PC, w.d_model, dtype=w.torch_dtype, device=dev),
                       "H": torch.empty(El, PC, w.d_ff, dtype=w.torch_dtype, device=dev),
                       "lc": torch.empty(El, dtype=torch.int32, device=dev),
                       "y": torch.empty_like(y),
                       "W1": W1[q * El:(q + 1) * El], "W2": W2[q * El:(q + 1) * El],
                       "ws": torch.empty(max(256, moe.ffn_workspace_size(fcfg)),
                                         dtype=torch.uint8, device=dev)})
        with torch.cuda.stream(stream):
            cnt_all = torch.stack([r["ro"]["kept_cnt"] for r in rk]).contiguous()
        xe_peers = [r["xe"] for r in rk]
        ye_peers = [r["ye"] for r in rk]
        ep_status = torch.zeros(1, dtype=torch.int32, device=dev)

        def ep_step(evs):
            evs[0].record(stream)
            for q, r in enumerate(rk):
                ro = r["ro"]
                moe.ep_dispatch(cfg, q, P, r["x"], ro["expert_idx"], ro["slot"], ro["kept"],
                                cnt_all, xe_peers, local_cnt=r["lc"], status=ep_status,
                                stream=stream)
            evs[1].record(stream)
            for r in rk:
                moe.expert_ffn(fcfg, r["xe"], r["W1"], r["W2"], r["lc"], H=r["H"], ye=r["ye"],
                               workspace=r["ws"], status=ep_status, stream=stream)
            evs[2].record(stream)
            for q, r in enumerate(rk):
                ro = r["ro"]
                moe.ep_combine(cfg, q, P, ye_peers, ro["expert_idx"], ro["gate"], ro["slot"],
                               ro["kept"], cnt_all, y=r["y"], status=ep_status, stream=stream)
            evs[3].record(stream)

        ep_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
                  for _ in range(max(args.steps, args.warmup))]
        for i in range(args.warmup):
            ep_step(ep_evs[i])
        torch.cuda.synchronize()
        for i in range(args.steps):
            ep_step(ep_evs[i])
        torch.cuda.synchronize()
        assert int(ep_status.item()) == 0, "expert-parallel step reported a device status"
        t_d = sum(e[0].elapsed_time(e[1]) for e in ep_evs[:args.steps]) / args.steps
        t_f = sum(e[1].elapsed_time(e[2]) for e in ep_evs[:args.steps]) / args.steps
        t_c = sum(e[2].elapsed_time(e[3]) for e in ep_evs[:args.steps]) / args.steps
        row = w.d_model * es
        n_sent = sum(int(r["ro"]["kept"].sum()) for r in rk)
        n_src = sum(int((r["ro"]["kept"].sum(1) > 0).sum()) for r in rk)
        d_bytes = (n_src + n_sent) * row
        c_bytes = (n_sent + P * w.T) * row
        hbm = peaks["hbm_gbs"] * 1e9
        ep = {"world": P, "tokens_per_step": P * w.T, "ffn_capacity": PC,
              "dispatch_ms": t_d, "dispatch_bytes": d_bytes,
              "dispatch_frac_hbm": d_bytes / hbm / (t_d / 1e3),
              "expert_ffn_ms": t_f, "combine_ms": t_c, "combine_bytes": c_bytes,
              "combine_frac_hbm": c_bytes / hbm / (t_c / 1e3),
              "step_ms": t_d + t_f + t_c,
              "tokens_per_s": P * w.T / ((t_d + t_f + t_c) / 1e3),
              "note": "moe_ep_dispatch / moe_expert_ffn / moe_ep_combine for two ranks emulated "
                      "on one GPU (peer stores and loads hit HBM, not NVLink); events between "
                      "the three steps, routing outside the timed region"}
        del rk, xe_peers, ye_peers
        torch.cuda.empty_cache()

    # ---- e2e through moe_layer_forward with host buffers ----
    # Every step copies its batch from pinned host memory and its output back.
    # The copies run on two copy streams, double-buffered, so step i's
    # host->device copy and step i-1's device->host copy overlap step i's
    # layer on the compute stream (PCIe is full duplex).
    nbuf = 2
    xh = [torch.empty_like(xs[r], device="cpu").pin_memory() for r in range(min(n_rot, 4))]
    for r in range(len(xh)):
        xh[r].copy_(xs[r].cpu())
    dh = None
    if w.mode == "rre":
        dh = [doms[r].cpu().pin_memory() for r in range(len(xh))]
    yh = torch.empty(w.T, w.d_model, dtype=w.torch_dtype).pin_memory()
    xd = [torch.empty_like(xs[0]) for _ in range(nbuf)]
    yd = [torch.empty_like(y) for _ in range(nbuf)]
    dd = None if dh is None else [torch.empty_like(doms[0]) for _ in range(nbuf)]
    h2d = x_bytes + (w.T * 4 if dh is not None else 0)
    d2h = x_bytes
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event() for _ in range(nbuf)]
    comp_done = [torch.cuda.Event() for _ in range(nbuf)]
    out_done = [torch.cuda.Event() for _ in range(nbuf)]
    used = [False] * nbuf

    def e2e_step(i):
        b = i % nbuf
        if used[b]:
            s_in.wait_event(comp_done[b])      # the layer that read xd[b] is done
            stream.wait_event(out_done[b])     # the copy that read yd[b] is done
        with torch.cuda.stream(s_in):
            xd[b].copy_(xh[i % len(xh)], non_blocking=True)
            if dd is not None:
                dd[b].copy_(dh[i % len(dh)], non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        moe.layer_forward(cfg, xd[b], W1, W2, Wr=Wr, bias=bias,
                          domain_id=None if dd is None else dd[b], y=yd[b], workspace=ws,
                          status=status, stream=stream)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            yh.copy_(yd[b], non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    tokens_all = sum_over_ranks(float(w.T * args.steps), world)
    value = tokens_all / (total_ms_max / 1e3)
    e2e_value = tokens_all / (e2e_ms / 1e3)

    if rank != 0:
        return
    clocks = clk.summary()
    out = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff, "E": w.E,
                   "k": w.k, "capacity_factor": w.capacity_factor, "capacity": C,
                   "expert": w.expert,
                   "routing": w.mode, "tokens_per_rank_per_step": w.T,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"x rotated over {n_rot} batches ({n_rot * x_bytes / 2**20:.0f} MiB) and "
                         f"expert weights {2 * w.E * w.d_model * w.d_ff * es / 2**30:.2f} GiB, "
                         "both larger than the 126 MB L2"},
        "roofline": roof,
        "stages_ms": {k: round(v_, 5) for k, v_ in stage_ms.items()},
        "stages": stages,
        "stages_note": "stage times from events the library records between its stages "
                       "(each record serialises the stream); frac = roofline time / stage time",
        "expert_ffn_tflops": ffn_flops / ffn_s / 1e12,
        "dispatch_combine_gbs": (disp_bytes + comb_bytes) / dc_s / 1e9,
        "dispatch_combine_scope": ("dispatch only: the top-1 combine (the y scatter) runs inside "
                                   "the expert FFN's GEMM-2 epilogue and is timed with expert_ffn"
                                   if fused_combine else "dispatch and combine kernels"),
        "combine": "fused into the expert FFN's GEMM-2 epilogue" if fused_combine else "kernel",
        "aux_loss": aux,
        "sparseclip": sclip,
        "expert_parallel": ep,
        "routing": {"n_kept": n_kept, "n_dropped": n_dropped,
                    "drop_rate": n_dropped / (w.T * w.k)},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": "moe_layer_forward, copies double-buffered on two copy streams"},
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.experts:
        if args.experts <= 0 or w.E % args.experts or args.experts % max(1, w.num_groups):
            raise SystemExit("--experts must divide E and be a multiple of the group count")
        w = w.scaled(name=f"{w.name}_E{args.experts}", E=args.experts,
                     T=w.T * args.experts // w.E)
    if args.expert != "relu":
        w = w.scaled(expert=args.expert)
    world, rank, local = (1, 0, 0)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_b200(args, w, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
