"""Benchmark of the MoE SwiGLU forward layer (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole layer (route, dispatch, expert GEMMs, shared
expert, combine) over one batch of synthetic tokens of the workload, inputs
resident in HBM.  `value` = tokens processed by all ranks / max-over-ranks
device time.  Under torchrun each rank runs its own batch with replicated
weights (data parallel, no collective on the data path): weak scaling.

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only; other ranks exit at once).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE fwd tokens/s (T=4096,D=4096,E=8,top-2,bf16); % of tensor/HBM roofline"
DEFAULT_WORKLOAD = "mixtral_bf16"


def describe(p) -> str:
    s = f"{p.name}: T={p.T} D={p.D} F={p.F} E={p.E} top-{p.k} act={p.act} experts={p.wdtype} gate={p.gate}"
    if p.capacity_factor:
        s += f" cf={p.capacity_factor}"
    if p.clamp:
        s += f" clamp={p.clamp}"
    if p.Fs:
        s += f" shared_F={p.Fs}"
    return s


def layer_flops(p, rows: int) -> float:
    """Algorithmic FLOPs of one layer pass: router 2TDE, experts 6 rows D F, shared 6 T D Fs."""
    return 2.0 * p.T * p.D * p.E + 6.0 * rows * p.D * p.F + 6.0 * p.T * p.D * p.Fs


def layer_bytes(p) -> float:
    """Algorithmic bytes: every weight once, x in, out back."""
    a = 4 if p.act == "f32" else 2
    we = {"f32": 4.0, "bf16": 2.0, "nvfp4": 0.5 + 1.0 / 16}[p.wdtype]
    return (3.0 * p.E * p.F * p.D * we + p.E * p.D * a + 3.0 * p.Fs * p.D * a + 2.0 * p.T * p.D * a)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


# the sources each recorded traffic figure depends on (a change to any of them voids the record)
TRAFFIC_SOURCES = {
    "gate_up_mixtral_bf16": ("gemm_tc.cu", "tc_ptx.cuh", "tma_host.h", "common.cuh"),
    "gate_up_sqrt_fp4": ("gemm_fp4.cu", "tc_ptx.cuh", "tma_host.h", "common.cuh"),
}


def gemm_sources_sha(files=TRAFFIC_SOURCES["gate_up_mixtral_bf16"]) -> str:
    h = hashlib.sha256()
    for n in files:
        p = os.path.join(ROOT, "mixture_experts_layer_sqrt_b200", "csrc", n)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key: str, path: str = os.path.join(ROOT, "profiles", "traffic.txt")):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel's sources are unchanged since."""
    if not os.path.exists(path) or kernel_key not in TRAFFIC_SOURCES:
        return None
    want = gemm_sources_sha(TRAFFIC_SOURCES[kernel_key])
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_key and parts[1] == want:
            return float(parts[2])
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled while the timed region runs.

    Reads NVML every 5 ms from a host thread (a 20-step Mixtral region lasts
    ~50 ms, shorter than nvidia-smi's sampling loop); falls back to an
    `nvidia-smi -lms 200` loop when NVML is unavailable.  Read-only."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_id: str, period_s: float = 0.005):
        self.proc = None
        self.thread = None
        self.samples = []
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(gpu_id)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop_evt = threading.Event()

            def loop():
                while not self.stop_evt.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except Exception:
                        pass
                    self.stop_evt.wait(period_s)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            sm = [float(c) for c, _ in self.samples]
            reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS if r & bit})
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml, 5 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi, 200 ms"}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_pass(p, arrays, n_tokens: int, seed: int):
    """One bounded pass of the float64 oracle, in two timed parts:
    route + dispatch of every token (capacity needs them all), then the expert
    FFN + combine of n_tokens sampled tokens (each touched expert's weights
    decoded once, then its rows multiplied).  Returns (route_dispatch_s, ffn_s,
    rows kept after capacity)."""
    import oracle.moe_oracle as O
    L = O.StoredLayer(arrays, p.act, p.wdtype)
    t0 = time.perf_counter()
    x = L.x()
    logits = O.router_logits(x, L.w_router())
    idx, w, _ = O.route(logits, p.k, p.gate, arrays.get("bias"), arrays.get("bias_vl"), arrays.get("image_mask"))
    C = O.expert_capacity(p.T, p.k, p.E, p.capacity_factor)
    d = O.dispatch(idx, p.E, C)
    t1 = time.perf_counter()
    toks = np.random.default_rng(seed).choice(p.T, size=min(n_tokens, p.T), replace=False)
    O.moe_forward(x, logits, idx, w, L.expert, p.E, C, p.clamp, "preact", L.shared(), tokens=toks)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, int(d["offsets"][-1])


def extrapolate_ffn(samples):
    """Fit ffn_s = fixed + per_token * n over (n, ffn_s) samples of two or more
    sizes (least squares).  The fixed part is the weight decoding, paid once
    per touched expert whatever the sample size; per_token is the marginal
    matmul cost.  Falls back to a line through the origin (the largest
    sample's rate) when the fit is not increasing."""
    n = np.array([s[0] for s in samples], dtype=np.float64)
    t = np.array([s[1] for s in samples], dtype=np.float64)
    if len(set(n.tolist())) >= 2:
        b, a = np.polyfit(n, t, 1)
        if b > 0 and a >= 0:
            return float(a), float(b)
    i = int(np.argmax(n))
    return 0.0, float(t[i] / n[i])


def cpu_core_counts():
    """(nproc: the host's usable cores, threads: the BLAS threads the oracle's matmuls use)."""
    try:
        nproc = len(os.sched_getaffinity(0))
    except AttributeError:
        nproc = os.cpu_count() or 1
    return nproc, blas_threads()


def oracle_summary(p, rd_s: float, samples, kind_note: str):
    """The oracle's whole-layer rate for all T tokens, extrapolated from the
    timed samples: T / (route_dispatch_s + fixed + per_token * T)."""
    fixed, per_tok = extrapolate_ffn(samples)
    layer_s = rd_s + fixed + per_tok * p.T
    nproc, threads = cpu_core_counts()
    sizes = sorted({int(n) for n, _ in samples})
    return {"value": p.T / layer_s, "unit": "tokens/s", "cores": threads, "nproc": nproc, "threads": threads,
            "kind": "oracle", "extrapolated": True, "route_dispatch_s": rd_s,
            "ffn_s_per_token": per_tok, "ffn_fixed_s": fixed, "layer_s": layer_s,
            "ffn_samples": [[int(n), float(t)] for n, t in samples],
            "sample": (f"float64 numpy oracle ({kind_note}): route + dispatch of all {p.T} tokens timed alone; "
                       f"expert FFN + combine timed on seeded samples of {sizes} tokens, fitted as fixed "
                       f"(weight decoding) + per-token cost and extrapolated to {p.T} tokens")}


# ------------------------------------------------------------ ranks (host)

def rank_problem(p, rank: int):
    """The token batch of one data-parallel rank: same weights, its own tokens
    (rank 0 keeps the workload's seed; rank r draws x from seed + 1000 r)."""
    return p if rank == 0 else p.with_(seed=p.seed + 1000 * rank)


def rank_arrays(p, rank: int, synth):
    arrays = synth.generate(p)
    if rank > 0:
        arrays["x"] = synth.generate(rank_problem(p, rank), experts=False)["x"]
    return arrays


def max_over_ranks(value: float, dist, device) -> float:
    """The job's time is the slowest rank's (an all-reduce MAX; identity on one rank)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Tokens per second of the whole job: every rank processes its own batch each step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def emit(res, rank: int):
    """Rank 0 prints the one JSON line; the other ranks print nothing."""
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


# --------------------------------------------------------------------- ours

def run_ours(args, p, rank, world, local_rank):
    import torch
    from mixture_experts_layer_sqrt_b200 import binding as B, synth, workload as WL
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    arrays = rank_arrays(p, rank, synth)  # each rank its own tokens, same weights
    cfg = WL.config_of(p)
    wt = WL.device_weights(p, arrays, dev)
    w = B.make_weights(wt)
    x = WL.to_torch(arrays["x"], dev)
    mask = WL.to_torch(arrays.get("image_mask"), dev)
    T, k, D = p.T, p.k, p.D
    out = torch.empty((T, D), dtype=torch.float32, device=dev)
    ws_f = B.workspace(B.workspace_size(cfg, T), dev)
    stream = torch.cuda.current_stream(dev)

    # one step = one moe_forward call (the product's own entry point); with
    # events it records them on the stream at the stage boundaries:
    # 0 | route | 1 | dispatch maps | 2 | gather | 3 | gate/up | 4 | down | 5 | shared | 6 | combine | 7
    def step(ev=None):
        if ev is None:
            B.forward(cfg, x, w, ws_f, mask, out)
        else:
            B.forward_profiled(cfg, x, w, ws_f, ev, mask, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    B.check_device_status(ws_f)
    counts = torch.empty(p.E, dtype=torch.int32, device=dev)
    B.forward(cfg, x, w, ws_f, mask, out, expert_counts_out=counts)
    cap = cfg.expert_capacity
    counts_h = counts.cpu().numpy()
    lb = load_balance(counts_h, T, k, cap)
    rows = lb["kept"]

    dist = None
    if world > 1:
        import torch.distributed as dist
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid)) if rank == 0 else None
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = B.launch_count()
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    g_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(B.STAGE_EVENTS)] for _ in range(args.steps)]
    for e in step_ev + [ev for evs in g_ev for ev in evs]:  # create every CUDA event before timing
        e.record(stream)
    torch.cuda.synchronize()
    step_ev[0].record(stream)
    for i in range(args.steps):
        step(g_ev[i])
        step_ev[i + 1].record(stream)
    torch.cuda.synchronize()
    n_launch = B.launch_count() - n0
    if dist:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = step_ev[0].elapsed_time(step_ev[-1])
    per_step = [step_ev[i].elapsed_time(step_ev[i + 1]) for i in range(args.steps)]
    names = STAGES
    stage_ms = {n: sum(e[i].elapsed_time(e[i + 1]) for e in g_ev) / args.steps for i, n in enumerate(names)}
    gemm_ms = stage_ms["gate_up"]
    B.check_device_status(ws_f)
    ms = max_over_ranks(total_ms, dist, dev) / args.steps
    value = whole_job_value(world, T, ms)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, B, WL, cfg, wt, arrays, T, D, dev, stream, dist)
    if rank != 0:
        return None
    res = report(args, p, world, rows, value, ms, per_step, gemm_ms, e2e, n_launch, clocks)
    res["stage_ms"] = stage_ms
    res["permute_combine"] = permute_combine(p, rows, stage_ms, load_peaks())
    res["load_balance"] = lb
    return res


def shared_expert_alone(B, p, x, wt, clamp_mode="preact"):
    """The always-on shared expert by itself (staged gate/up and down calls, one group)."""
    sc = B.make_config(E=1, k=1, D=p.D, F=p.Fs, clamp=p.clamp, clamp_mode=clamp_mode, act=p.act, expert=p.act)
    hs = B.expert_gate_up(sc, x, None, wt["sh_gate"], wt["sh_up"])
    return B.expert_down(sc, hs, None, wt["sh_down"])


def run_sweep(args, p, ks):
    """Per-token time of the whole layer at several top-k values on one shape
    ("5A · MoE fine-grained" sec. 4, Profiling: time per token at top-k 1, 2,
    4, and the shared expert added once at each).  For each k: moe_forward
    timed with CUDA events over args.steps steps, the load-balance diagnostic
    of its routing, and, with a shared expert, the largest deviation of
    out(shared) - out(shared weights zeroed) from the shared expert alone,
    relative to the shared expert's largest magnitude."""
    import torch
    from mixture_experts_layer_sqrt_b200 import binding as B, synth, workload as WL
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    arrays = synth.generate(p)
    wt = WL.device_weights(p, arrays, dev)
    w = B.make_weights(wt)
    x = WL.to_torch(arrays["x"], dev)
    mask = WL.to_torch(arrays.get("image_mask"), dev)
    stream = torch.cuda.current_stream(dev)
    rows = []
    for k in ks:
        q = p.with_(k=k)
        cfg = WL.config_of(q)
        ws = B.workspace(B.workspace_size(cfg, q.T), dev)
        out = torch.empty((q.T, q.D), dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            B.forward(cfg, x, w, ws, mask, out)
        counts = torch.empty(q.E, dtype=torch.int32, device=dev)
        B.forward(cfg, x, w, ws, mask, out, expert_counts_out=counts)
        torch.cuda.synchronize()
        lb = load_balance(counts.cpu().numpy(), q.T, k, cfg.expert_capacity)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            B.forward(cfg, x, w, ws, mask, out)
        e1.record(stream)
        torch.cuda.synchronize()
        B.check_device_status(ws)
        ms = e0.elapsed_time(e1) / args.steps
        row = {"k": k, "ms_per_step": ms, "us_per_token": ms * 1e3 / q.T, "tokens_per_s": q.T / (ms / 1e3),
               "layer_flops": layer_flops(q, lb["kept"]), "load_balance": lb}
        if q.Fs:
            zero = dict(wt, sh_gate=torch.zeros_like(wt["sh_gate"]), sh_up=torch.zeros_like(wt["sh_up"]),
                        sh_down=torch.zeros_like(wt["sh_down"]))
            out0 = B.forward(cfg, x, B.make_weights(zero), ws, mask)
            sh = shared_expert_alone(B, q, x, wt)
            torch.cuda.synchronize()
            row["shared_added_once_rel_err"] = float((out - out0 - sh).abs().max() / sh.abs().max())
        rows.append(row)
    return {"metric": "MoE fwd per-token time vs top-k", "unit": "us/token", "higher_is_better": False,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "dtype": "f32" if p.act == "f32" else "bf16",
            "data": "synthetic", "config": {"workload": describe(p), "top_k": list(ks)}, "sweep": rows}


def run_e2e(args, B, WL, cfg, wt, arrays, T, D, dev, stream, dist):
    """The same metric through the public API: every step uploads its tokens
    from pinned host memory and downloads its output to pinned host memory;
    MoELayer.forward_host_batches overlaps those copies with the compute of
    the neighbouring steps."""
    import torch
    world = dist.get_world_size() if dist else 1
    layer = B.MoELayer(cfg, wt, T, dev)
    x_h = WL.to_torch(arrays["x"], "cpu", pin=True)
    m_h = WL.to_torch(arrays.get("image_mask"), "cpu", pin=True)
    out_h = [torch.empty((T, D), dtype=torch.float32).pin_memory() for _ in range(2)]
    xs = [x_h] * args.steps
    outs = [out_h[i % 2] for i in range(args.steps)]
    masks = [m_h] * args.steps if m_h is not None else None
    layer.forward_host_batches(xs[:max(2, args.warmup)], outs[:max(2, args.warmup)],
                               masks[:max(2, args.warmup)] if masks else None)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    layer.forward_host_batches(xs, outs, masks)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    B.check_device_status(layer.ws)
    return {"value": whole_job_value(world, T, e2e_ms / args.steps), "unit": "tokens/s",
            "h2d_bytes_per_step": int(x_h.numel() * x_h.element_size() + (m_h.numel() if m_h is not None else 0)),
            "d2h_bytes_per_step": int(out_h[0].numel() * out_h[0].element_size()),
            "copies": "overlapped with compute on separate streams (forward_host_batches)"}


def load_balance(counts, T: int, k: int, capacity: int = 0):
    """Routing diagnostics from the per-expert assignment counts (before capacity):
    the load-balance measure E * sum_e (count_e / (T k))^2 of the ops-transformer
    MoE walkthrough (坑二: 1 when every expert gets T k / E assignments, E when
    one expert gets them all), the kept rows after capacity and the drops."""
    c = np.asarray(counts, dtype=np.int64)
    E = len(c)
    ratio = c / float(max(T * k, 1))
    kept = int(np.minimum(c, capacity).sum()) if capacity else int(c.sum())
    return {"loss": float(E * np.sum(ratio ** 2)), "kept": kept, "drops": int(T * k - kept),
            "max_count": int(c.max()) if E else 0, "min_count": int(c.min()) if E else 0}


# the stage intervals moe_forward_profiled brackets with its events
STAGES = ["route", "dispatch_maps", "gather", "gate_up", "down", "shared", "combine"]


def permute_combine(p, rows: int, stage_ms, peaks):
    """Achieved HBM bandwidth of the two data-movement stages, from their
    algorithmic bytes and their stage event times:
      gather   reads each kept row's x row and writes it to x_perm: 2 rows D a
               (+ a 4-byte row scale per row for the f16 rows of NVFP4 layers)
      combine  reads every kept row of fp32 y_perm (and the fp32 shared-expert
               row of every token) and writes the fp32 output row of every token"""
    a = 4 if p.act == "f32" else 2
    g_bytes = 2.0 * rows * p.D * a + (4.0 * rows if p.wdtype == "nvfp4" else 0.0)
    out = {}
    for name, b in (("gather", g_bytes), ("combine", 4.0 * rows * p.D + 4.0 * p.T * p.D * (2 if p.Fs else 1))):
        ms = stage_ms[name]
        gbs = b / (ms / 1e3) / 1e9 if ms > 0 else None
        out[name] = {"bytes": b, "ms": ms, "gbs": gbs, "frac": gbs / peaks["hbm"] if gbs else None}
    out["peak_gbs"] = peaks["hbm"]
    out["peak_kind"] = f"hbm_gbs of {peaks['src']}"
    return out


# fp32 layers run on the CUDA cores: 148 SMs x 128 fp32 lanes x 2 FLOP per FMA at the 1965 MHz maximum clock
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def gate_up_kernel(p, peaks):
    """The gate/up launch the roofline object describes: (name, bound, peak, sustained peak, peak note)."""
    if p.act == "f32":
        return ("grouped_gemm_simt<gate/up> (fp32 CUDA-core FMA)", "alu", FP32_ALU_TFLOPS, FP32_ALU_TFLOPS,
                "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz (nominal unit counts and clock)")
    name = ("tc_fp4_gemm<gate/up> (packed NVFP4 weights expanded on chip, f16 MMA)" if p.wdtype == "nvfp4"
            else "tc_grouped_gemm<gate/up> (grouped gate/up GEMM + SwiGLU epilogue)")
    return (name, "tensor", peaks["bf16"], peaks["bf16_sustained"], f"bf16_tflops (burst) of {peaks['src']}")


def workload_config(p, world: int, rows: int):
    """The `config` object of both arms' JSON lines."""
    return {"workload": describe(p), "tokens_per_gpu": p.T, "rows_after_capacity": rows, "out_dtype": "f32",
            "parallelism": f"dp{world} (independent token batches, replicated weights)",
            "l2": "inputs larger than L2: expert weights %.2f GB streamed every step" % (layer_bytes(p) / 1e9)}


def report(args, p, world, rows, value, ms, per_step, gemm_ms, e2e, n_launch, clocks):
    peaks = load_peaks()
    flops = layer_flops(p, rows)
    gemm1_flops = 4.0 * rows * p.D * p.F     # gate and up projections of every kept row
    # burst peak (the conservative denominator); the sustained figure is
    # reported beside it for a GPU that settles under its power cap
    peak_t = peaks["bf16"]
    achieved = gemm1_flops / (gemm_ms / 1e3) / 1e12
    kernel, bound, peak_k, peak_sus, peak_kind = gate_up_kernel(p, peaks)
    ideal_ms = max(flops / (peak_t * 1e12), layer_bytes(p) / (peaks["hbm"] * 1e9)) * 1e3
    ideal_sus_ms = max(flops / (peaks["bf16_sustained"] * 1e12), layer_bytes(p) / (peaks["hbm"] * 1e9)) * 1e3
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if p.act == "f32" else "bf16", "data": "synthetic",
        "config": workload_config(p, world, rows),
        "latency_ms": {"p50": float(np.percentile(per_step, 50)), "p95": float(np.percentile(per_step, 95)),
                       "p99": float(np.percentile(per_step, 99))},
        "layer_roofline": {"ideal_ms": ideal_ms, "frac": ideal_ms / ms, "frac_vs_sustained": ideal_sus_ms / ms,
                           "flops": flops, "bytes": layer_bytes(p),
                           "peak": f"bf16 {peak_t} TFLOP/s burst ({peaks['bf16_sustained']} sustained), "
                                   f"HBM {peaks['hbm']} GB/s, of {peaks['src']}"},
        "roofline": {"kernel": kernel,
                     "bound": bound,
                     "achieved": achieved, "peak": peak_k, "unit": "TFLOP/s", "frac": achieved / peak_k,
                     "frac_vs_sustained": achieved / peak_sus,
                     "peak_kind": peak_kind,
                     "flops_per_launch": gemm1_flops, "ms_per_launch": gemm_ms,
                     "traffic": profiled_traffic("gate_up_" + p.name)},
        "e2e": e2e,
        "gpu_launches": int(n_launch),
        "gpu_launches_per_step": n_launch / args.steps,
        "clocks": clocks,
    }
    return res


def cpu_baseline_leg(p, sizes=(64, 256)):
    """The oracle as it stands on a bounded sample of the bench workload
    (about 10-30 s of CPU work), reported beside the GPU number."""
    from mixture_experts_layer_sqrt_b200 import synth
    arrays = synth.generate(p)
    samples, rd = [], []
    for i, n in enumerate(sizes):
        r, f, _ = oracle_pass(p, arrays, n, seed=1 + i)
        rd.append(r)
        samples.append((n, f))
    return oracle_summary(p, float(np.mean(rd)), samples, "cpu_baseline")


def run_reference(args, p):
    """The reference arm: the float64 oracle on the host cores, each step a
    bounded sample of the workload (route + dispatch of all T tokens, FFN +
    combine of a few sampled tokens; steps alternate two sample sizes).  The
    line's value is the oracle's whole-layer rate for all T tokens,
    extrapolated from those steps."""
    from mixture_experts_layer_sqrt_b200 import synth
    arrays = synth.generate(p)
    sizes = (16, 96)
    for i in range(args.warmup):
        oracle_pass(p, arrays, sizes[0], seed=100 + i)
    samples, rd, step_s, rows = [], [], [], 0
    for i in range(args.steps):
        n = sizes[i % 2]
        t0 = time.perf_counter()
        r, f, rows = oracle_pass(p, arrays, n, seed=i)
        step_s.append(time.perf_counter() - t0)
        rd.append(r)
        samples.append((n, f))
    cb = oracle_summary(p, float(np.mean(rd)), samples, "--impl reference")
    value = cb["value"]
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["layer_s"] * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(p, 1, rows),
            "sample_ms_per_step": 1e3 * float(np.mean(step_s)),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep-k", default="", metavar="K1,K2,...",
                    help="time the layer at each top-k on the workload's shape instead of the bench step")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (e.g. T=1024, E=2) for a smaller profiling case")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from mixture_experts_layer_sqrt_b200 import synth
    p = synth.PROBLEMS[args.workload]
    if args.set:
        kw = {}
        for item in args.set:
            key, val = item.split("=", 1)
            cur = getattr(p, key)
            kw[key] = type(cur)(val)
        p = p.with_(name=p.name + "[" + ",".join(args.set) + "]", **kw)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":  # the oracle on the host cores: rank 0 only
        if rank == 0:
            emit(run_reference(args, p), rank)
        return

    from mixture_experts_layer_sqrt_b200 import build
    build.build()
    import torch
    if args.sweep_k:
        emit(run_sweep(args, p, [int(v) for v in args.sweep_k.split(",")]), rank)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        # short enough to end a job whose ranks wait on one another for good; long
        # enough for every rank to generate its inputs (GBs of weights) on a shared host
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, p, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_leg(p)
        emit(res, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
