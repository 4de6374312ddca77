"""Benchmark of the LatentMoE layer on B200: tokens/s of one layer forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference]

A step is one moe_forward over one batch of T synthetic tokens (router, routing
bookkeeping, latent projection, routed experts, combine, fc2 and the shared
expert).  Default workload: the Ultra-shape decode layer, bf16, T=64 (the line's
value); on one GPU the other workloads of the metric -- Ultra prefill bf16
T=8192, Ultra decode W4A16 T=256, skewed prefill W4A4 T=16384 -- follow on the
same weights and are reported under "workloads", each with its own roofline,
stage times, clocks and end-to-end figure.  With N>1
(torchrun) every rank runs its own replica on its own tokens (weak scaling, no
collective on the data path); value = all ranks' tokens / max-over-ranks time.
`--impl reference` times the CPU oracle on the host cores instead.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import atexit
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LatentMoE layer tokens/s at Ultra shape (T=64 decode, T=8192 prefill); % roofline"
UNIT = "tokens/s"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="ultra_decode_bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", action="store_true",
                    help="time the block around the layer: out = x + layer(RMSNorm(x))")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--workloads", default="auto",
                    help="extra workloads timed after --config and reported under "
                         "'workloads': all, none, a comma list, or auto (all for the "
                         "default Ultra decode on one GPU, none otherwise)")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampler over the timed region (SM clock, throttle reasons)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        atexit.register(self.__exit__)       # no sampler outlives the process
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc and self.proc.poll() is None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    from latentmoe_expert_routing_b200 import dist as D
    return D.env_ranks()


def _expert_bytes(cfg, n_touched):
    """Bytes of one expert matrix per touched expert actually streamed: dense
    bf16/fp32, or NVFP4 (4-bit codes + one E4M3 scale per 16 = 0.5625 B)."""
    if cfg.expert_fmt != "dense":
        return n_touched * cfg.F * cfg.L * 9 // 16
    es = 4 if cfg.dtype == "fp32" else 2
    return n_touched * cfg.F * cfg.L * es


def _oracle_sample(cfg, W, x, n_tok, min_s=0.0, norm=None):
    """Time the oracle, as it stands, on the first n_tok token rows: one forward,
    or repeated forwards until min_s seconds (at most 12)."""
    import numpy as np
    from oracle import moe_oracle as O
    rows = x[:n_tok]
    f = lambda t: t.detach().float().cpu().numpy()
    xs, g, b = f(rows), f(W["w_gate"]), f(W["gate_bias"])
    dense = [f(W[n]) for n in ("w_fc1", "w_fc2", "w_shared_up", "w_shared_down")]
    rows = xs
    if norm is not None:                        # the block routes its normalised rows
        y = O.rmsnorm_spec(xs, f(norm[0]), norm[1])
        rows = O.round_fp64_to_bf16(y) if cfg.dtype == "bf16" else y.astype(np.float32)
    l = O.router_logits(rows, g)
    _, _, idx, _ = O.route(l, b, cfg.k, cfg.rsf, cfg.n_group, cfg.topk_group)
    need = sorted(set(idx.reshape(-1).tolist()))
    up = {e: f(W["w_up"][e]) for e in need}       # fp32 copies; fp64 inside the call
    dn = {e: f(W["w_down"][e]) for e in need}
    reps, dt = 0, 0.0
    kw = dict(k=cfg.k, rsf=cfg.rsf, expert_fmt=cfg.expert_fmt, n_group=cfg.n_group,
              topk_group=cfg.topk_group)
    while reps < 12 and (reps == 0 or dt < min_s):
        t0 = time.perf_counter()
        if norm is None:
            O.forward(xs, g, b, *dense, lambda e: up[e].astype(np.float64),
                      lambda e: dn[e].astype(np.float64), **kw)
        else:                                   # the block: (norm weight, eps)
            O.block_forward(xs, f(norm[0]), norm[1], g, b, *dense,
                            lambda e: up[e].astype(np.float64),
                            lambda e: dn[e].astype(np.float64), dtype=cfg.dtype, **kw)
        dt += time.perf_counter() - t0
        reps += 1
    return reps * n_tok / dt, dt, reps


def _measured_traffic(cfg, n_touched):
    """DRAM bytes per grouped-GEMM launch from the committed ncu capture of the
    decode-sized kernel (bf16 experts: umma_gemm_kernel; NVFP4 experts:
    umma_wq_kernel), scaled by touched experts; None when the kernel's sources
    changed since the capture or the workload is not one the capture covers."""
    import hashlib
    name = "umma_gemm_traffic.json" if cfg.expert_fmt == "dense" else "umma_wq_traffic.json"
    p = os.path.join(ROOT, "profiles", name)
    if cfg.dtype != "bf16" or not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256()
    for f in d["source_files"]:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != d["source_sha256"]:
        return None
    return d["dram_bytes_per_touched_expert"] * n_touched


def _graph_kernel_nodes(graph):
    """Kernel nodes of a captured CUDA graph (its cudaGraph_t kept): the
    library's launches per step.  None when the runtime cannot be queried."""
    import ctypes
    try:
        rt = ctypes.CDLL("libcudart.so.12")
    except OSError:
        return None
    g = ctypes.c_void_p(graph.raw_cuda_graph())
    n = ctypes.c_size_t(0)
    if rt.cudaGraphGetNodes(g, None, ctypes.byref(n)) != 0:
        return None
    nodes = (ctypes.c_void_p * n.value)()
    if rt.cudaGraphGetNodes(g, nodes, ctypes.byref(n)) != 0:
        return None
    kinds = [ctypes.c_int(-1) for _ in range(n.value)]
    for i in range(n.value):
        if rt.cudaGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(kinds[i])) != 0:
            return None
    return sum(1 for k in kinds if k.value == 0)        # cudaGraphNodeTypeKernel


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _gen_device():
    import torch
    return "cuda" if torch.cuda.is_available() else "cpu"


def _workload_config(a, cfg, world, n_touched):
    """The workload as both arms name it: shape, format, launch and L2 note."""
    from latentmoe_expert_routing_b200 import inputs as I
    return {"workload": cfg.name, "T": cfg.T, "d_model": cfg.D, "d_latent": cfg.L,
            "experts": cfg.E, "top_k": cfg.k, "d_ff": cfg.F,
            "d_ff_shared": cfg.Fs, "expert_fmt": cfg.expert_fmt,
            "bias": cfg.bias_kind, "outlier_rows": len(I.outlier_rows(cfg)),
            "parallelism": f"replicas{world}",
            "cuda_graph": not a.no_graph,
            "block": bool(a.block),
            "l2": "no flush: each step streams the touched experts' weights "
                  f"({2 * _expert_bytes(cfg, n_touched) / 1e9:.1f} GB) > 126 MB L2"}


def _oracle_touched(cfg, W, x, norm=None):
    """Experts that the oracle's router sends at least one of the T rows to."""
    import numpy as np
    from oracle import moe_oracle as O
    f = lambda t: t.detach().float().cpu().numpy()
    rows = f(x)
    if norm is not None:
        y = O.rmsnorm_spec(rows, f(norm[0]), norm[1])
        rows = O.round_fp64_to_bf16(y) if cfg.dtype == "bf16" else y.astype(np.float32)
    l = O.router_logits(rows, f(W["w_gate"]))
    _, _, idx, _ = O.route(l, f(W["gate_bias"]), cfg.k, cfg.rsf, cfg.n_group, cfg.topk_group)
    return len(set(idx.reshape(-1).tolist()))


def run_reference(a):
    rank, world, _ = _dist()
    if rank != 0:
        return 0
    import torch
    from latentmoe_expert_routing_b200 import inputs as I
    cfg = I.CONFIGS[a.config]
    dev = _gen_device()
    W = _weights(cfg, dev)
    x = I.hidden(cfg, dev, T=cfg.T, start_row=0)
    norm = (I.norm_weight(cfg, dev), 1e-5) if a.block else None
    n_tok = cfg.T if cfg.T * cfg.D <= 64 * 256 else 2
    for _ in range(a.warmup):
        _oracle_sample(cfg, W, x, n_tok, norm=norm)
    times = [_oracle_sample(cfg, W, x, n_tok, norm=norm)[1] for _ in range(a.steps)]
    value = n_tok * a.steps / sum(times)
    sample = (f"first {n_tok} of {cfg.T} tokens per step, fp64 numpy oracle"
              + (" (block)" if a.block else ""))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": 1, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": 1e3 * sum(times) / a.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _workload_config(a, cfg, world, _oracle_touched(cfg, W, x, norm)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))
    return 0


def _weights(cfg, dev):
    from latentmoe_expert_routing_b200 import inputs as I
    import torch
    dt = torch.float32 if cfg.dtype == "fp32" else torch.bfloat16
    up = torch.empty(cfg.E, cfg.F, cfg.L, dtype=dt, device=dev)
    down = torch.empty(cfg.E, cfg.L, cfg.F, dtype=dt, device=dev)
    I.w_up_into(cfg, up)
    I.w_down_into(cfg, down)
    return dict(w_gate=I.w_gate(cfg, dev), gate_bias=I.gate_bias(cfg, dev),
                w_fc1=I.w_fc1(cfg, dev), w_fc2=I.w_fc2(cfg, dev),
                w_shared_up=I.w_shared_up(cfg, dev),
                w_shared_down=I.w_shared_down(cfg, dev), w_up=up, w_down=down)


def _layer_roofline(cfg, T, ms, hbm, tf, tf_sus, src, n_touched):
    """The whole layer against its own bound: HBM bytes of the touched experts
    and the dense weights at decode sizes; at prefill sizes the layer's FLOPs
    against the tensor peak (W4A4: expert FLOPs at the FP4 rate, the rest at
    bf16, ideal time = their sum)."""
    fl = {"gate": 2 * cfg.D * cfg.E, "fc1": 2 * cfg.D * cfg.L, "fc2": 2 * cfg.L * cfg.D,
          "shared": 4 * cfg.D * cfg.Fs}
    dense_fl = T * sum(fl.values())
    expert_fl = T * cfg.k * 4 * cfg.L * cfg.F
    if T * cfg.k / cfg.E < 64:
        es = 4 if cfg.dtype == "fp32" else 2
        dense_b = (cfg.E * cfg.D + 2 * cfg.D * cfg.L + 2 * cfg.D * cfg.Fs) * es
        b = 2 * _expert_bytes(cfg, n_touched) + dense_b
        return {"bound": "hbm", "bytes": b, "achieved": b / (ms * 1e-3) / 1e9, "peak": hbm,
                "unit": "GB/s", "frac": b / (ms * 1e-3) / 1e9 / hbm, "peak_source": src}
    peak = tf_sus or tf
    w4a4 = cfg.expert_fmt == "w4a4"
    ideal = dense_fl / (peak * 1e12) + expert_fl / (peak * (4.0 if w4a4 else 1.0) * 1e12)
    tot = dense_fl + expert_fl
    return {"bound": "tensor", "flops": tot, "achieved": tot / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "ideal_ms": ideal * 1e3, "frac": ideal / (ms * 1e-3),
            "peak_source": (f"{src} sustained bf16" +
                            (" (experts at x4, the nominal fp4/bf16 ratio)" if w4a4 else ""))}


def _measure(a, cfg, W, rank, world, local, cpu_leg):
    """Time one workload on this rank's replica; returns its line fields."""
    import torch
    from latentmoe_expert_routing_b200 import binding as B
    from latentmoe_expert_routing_b200 import dist as D
    from latentmoe_expert_routing_b200 import inputs as I
    from latentmoe_expert_routing_b200 import layer as LY
    lay = LY.layer_for(cfg, W, out_dtype=cfg.dtype)
    x = I.hidden(cfg, "cuda", T=cfg.T, start_row=0) if rank == 0 else \
        I.hidden(cfg.replace(seed=rank), "cuda")
    T = cfg.T
    tdt = x.dtype
    out = torch.empty(T, cfg.D, dtype=tdt, device="cuda")
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, cfg.k, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()

    g = I.norm_weight(cfg, "cuda")
    eps = 1e-5

    def step():
        if a.block:
            lay.block(x, g, eps, out, idx, wts)
        else:
            lay(x, out, idx, wts)

    barrier = D.barrier

    clk = Clocks(local).__enter__()          # sampling from warm-up on: GPU under load
    for _ in range(max(a.warmup, 3)):
        step()
    lay.sync()
    eager_step = step
    graph = None
    if not a.no_graph:
        # the whole forward (every library launch) captured once, replayed per step
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph):
            step()
        graph.instantiate()
        graph.replay()
        torch.cuda.synchronize()
        step = graph.replay
    launches = _graph_kernel_nodes(graph) if graph is not None else None
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(a.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    clk.__exit__()
    barrier()
    lay.sync()
    ms_max = D.max_over_ranks(e0.elapsed_time(e1) / a.steps, "cuda")

    step = eager_step
    # per-stage durations (CUDA events recorded by the library on this stream)
    B.moe_profile_enable(lay.handle, 1)
    stages = []
    for _ in range(5):
        step()
        stages.append(B.moe_profile_read(lay.handle))
    B.moe_profile_enable(lay.handle, 0)
    stage_ms = {k: statistics.median(s[k] for s in stages) for k in stages[0]}
    counts, _, _, _ = lay.routing(T)
    n_touched = int((counts > 0).sum().item())
    max_vio = float(counts.max().item()) / (T * cfg.k / cfg.E)
    lay.router_stats()
    step()
    exact_per_token = lay.router_stats() / T

    # end to end through the host entry point: pinned H2D of x, D2H of out
    # (the block has no host entry: its device call between explicit copies)
    xh = x.cpu().pin_memory()
    oh = torch.empty(T, cfg.D, dtype=tdt).pin_memory()

    def host_step():
        if a.block:
            x.copy_(xh, non_blocking=True)
            lay.block(x, g, eps, out, idx, wts)
            oh.copy_(out, non_blocking=True)
            st.synchronize()
        else:
            lay.forward_host(xh, oh)

    for _ in range(2):
        host_step()
    barrier()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(st)
    for _ in range(a.steps):
        host_step()
    h1.record(st)
    torch.cuda.synchronize()
    e2e_ms = D.max_over_ranks(h0.elapsed_time(h1) / a.steps, "cuda")

    cpu = None
    if cpu_leg:
        n_tok = min(T, 2 if cfg.D >= 4096 else T)
        v, dt, reps = _oracle_sample(cfg, W, x, n_tok, min_s=10.0,   # ~10 s of CPU work
                                     norm=(g, eps) if a.block else None)
        cpu = {"value": v, "unit": UNIT, "cores": _cores(), "kind": "oracle",
               "sample": f"first {n_tok} of {T} tokens, {reps} fp64 numpy oracle forwards "
                         f"({dt:.1f} s)"}

    hbm, tf, tf_sus, src = _peaks()
    # dominant kernel: the grouped expert GEMMs streaming the touched experts'
    # weights (up and down, one launch each); algorithmic bytes per launch =
    # touched experts x one [F, L] matrix + the activations it reads and writes
    es = 4 if cfg.dtype == "fp32" else 2
    P = T * cfg.k
    b_up = _expert_bytes(cfg, n_touched) + P * cfg.L * es + P * cfg.F * es
    b_dn = _expert_bytes(cfg, n_touched) + P * cfg.F * es + P * cfg.L * 4
    t_launch = (stage_ms["expert_up"] + stage_ms["expert_down"]) / 2
    achieved = (b_up + b_dn) / 2 / (t_launch * 1e-3) / 1e9
    prefill = P / cfg.E > 64                 # 128- / 256-token tiles
    fp4_mma = prefill and cfg.expert_fmt == "w4a4" and cfg.L % 256 == 0 and cfg.F % 256 == 0
    if cfg.dtype != "bf16":
        kname = "grouped_rows_kernel (expert up, expert down)"
    elif fp4_mma and P >= 256 * cfg.E:
        kname = ("umma_mxf4_pair_kernel (SM-pair block-scaled FP4, grouped expert up, "
                 "expert down)")
    elif fp4_mma:
        kname = "umma_mxf4_kernel (block-scaled FP4, grouped expert up, expert down)"
    elif cfg.expert_fmt != "dense":
        kname = "umma_wq_kernel (NVFP4 records, grouped expert up, expert down)"
    elif prefill and cfg.L % 256 == 0 and cfg.F % 256 == 0:
        kname = "umma_pair_kernel (two-SM, grouped expert up, expert down)"
    else:
        kname = "umma_gemm_kernel (grouped expert up, expert down)"
    if P / cfg.E >= 64:
        # prefill-sized: tensor-core bound; flops per launch = 2 * P * L * F.
        # The block-scaled FP4 MMA's peak: measured sustained bf16 x 4 (the
        # nominal dense FP4 / bf16 ratio, 9 / 2.25 PFLOP/s).
        fl = 2.0 * P * cfg.L * cfg.F
        peak = (tf_sus or tf) * (4.0 if fp4_mma else 1.0)
        roof = {"kernel": kname, "bound": "tensor", "achieved": fl / (t_launch * 1e-3) / 1e12,
                "peak": peak, "unit": "TFLOP/s",
                "frac": fl / (t_launch * 1e-3) / 1e12 / peak, "traffic": None,
                "peak_source": (f"{src} sustained bf16 x 4 (nominal fp4/bf16)" if fp4_mma
                                else f"{src} (sustained bf16)"),
                "flops_per_launch": fl}
    else:
        roof = {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": hbm,
                "unit": "GB/s", "frac": achieved / hbm,
                "traffic": _measured_traffic(cfg, n_touched),
                "peak_source": src, "bytes_per_launch": (b_up + b_dn) / 2}
    res = {
        "value": D.job_throughput(T, world, ms_max * 1e-3), "ms_per_step": ms_max,
        "dtype": cfg.dtype if cfg.expert_fmt == "dense" else f"{cfg.dtype}+nvfp4-{cfg.expert_fmt}",
        "config": _workload_config(a, cfg, world, n_touched),
        "roofline": roof,
        "layer_roofline": _layer_roofline(cfg, T, ms_max, hbm, tf, tf_sus, src, n_touched),
        "stages_ms": stage_ms,
        "experts_touched": n_touched,
        "max_load_over_mean": max_vio,
        "router_exact_logits_per_token": exact_per_token,
        "expert_weight_gbs": 2 * _expert_bytes(cfg, n_touched) /
                             ((stage_ms["expert_up"] + stage_ms["expert_down"]) * 1e-3) / 1e9,
        "layer_hbm_frac": (2 * _expert_bytes(cfg, n_touched) / (ms_max * 1e-3) / 1e9) / hbm,
        "clocks": clk.summary(),
        # library kernels in the timed region: the captured step's kernel
        # nodes (every one a launch of this library) times the steps
        "gpu_launches": None if launches is None else launches * a.steps,
        "e2e": {"value": D.job_throughput(T, world, e2e_ms * 1e-3), "unit": UNIT,
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": T * cfg.D * es,
                "d2h_bytes_per_step": T * cfg.D * es},
        "cpu_baseline": cpu,
    }
    del graph
    lay.close()
    del lay
    return res


# the other workloads of the headline metric, timed after the headline one on
# the same weights (Ultra shape, bf16 dense weights; NVFP4 layers quantise them),
# and the decode batch under the other reading of its router-bias spread
EXTRA_WORKLOADS = ["ultra_prefill_bf16", "ultra_decode_w4a16", "skewed_prefill_w4a4",
                   "ultra_decode_bf16_bias_sd001"]


def run_ours(a):
    import torch
    from latentmoe_expert_routing_b200 import dist as D
    rank, world, local = _dist()
    torch.cuda.set_device(local)
    D.init("nccl", 300, torch.device("cuda", local))
    from latentmoe_expert_routing_b200 import inputs as I
    cfg = I.CONFIGS[a.config]
    W = _weights(cfg, "cuda")
    head = _measure(a, cfg, W, rank, world, local,
                    cpu_leg=rank == 0 and world == 1 and not a.no_cpu_baseline)
    extras = {}
    names = EXTRA_WORKLOADS if a.workloads == "all" else \
        [] if a.workloads == "none" else a.workloads.split(",")
    if a.workloads == "auto":
        names = EXTRA_WORKLOADS if (world == 1 and cfg.name == "ultra_decode_bf16") else []
    for name in names:
        c = I.CONFIGS[name]
        same = all(getattr(c, f) == getattr(cfg, f) for f in ("D", "L", "E", "F", "Fs", "dtype"))
        Wc = dict(W) if same else _weights(c, "cuda")
        if c.bias_kind != cfg.bias_kind:
            Wc["gate_bias"] = I.gate_bias(c, "cuda")
        torch.cuda.empty_cache()
        try:
            extras[name] = _measure(a, c, Wc, rank, world, local, cpu_leg=False)
        except Exception as ex:          # one workload's failure keeps the others' lines
            if world > 1:                # ranks must not part ways between collectives
                raise
            extras[name] = {"error": f"{type(ex).__name__}: {ex}"[:300]}
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
                "steps": a.steps, "warmup": max(a.warmup, 3),
                "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
        line.update({k: v for k, v in head.items() if k not in ("value", "ms_per_step")})
        if extras:
            line["workloads"] = extras
        print(json.dumps(line))
    D.finish()
    return 0


def main():
    a = _args()
    if a.impl == "reference":
        return run_reference(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
