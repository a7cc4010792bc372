"""Benchmark: batch-1 sparse FFN decode on B200 through the C ABI.

One step = one decode token through the whole FFN stack (predictor, gather of
active rows/columns, reduction, residual + RMSNorm between layers) of the
Llama-2-7B-shaped ReGLU workload (32 layers, d 4096, F 11008, fp16, predictor
rank 1024, ~90 % sparse).  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--config NAME] [--active FRACTION] [--layers L] [--sweep]

--impl reference times the fp64 CPU oracle on the host cores instead (the
reference arm of this benchmark), each step a bounded sample of the same work.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from activation_sparse_decode_threshold_b200 import synth  # noqa: E402

METRIC = "decode tok/s (FFN stack, batch 1) and achieved HBM GB/s on touched bytes vs peak"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SRC = os.path.join(ROOT, "activation_sparse_decode_threshold_b200", "csrc", "pi_decode_kernel.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_dram_traffic.txt")
PB = {"f32": 4, "f16": 2, "bf16": 2, "i8row": 1}


def wrow_bytes(cfg) -> float:
    if cfg.wdtype == "int4g32":
        return cfg.d / 2 + cfg.d / 16
    return cfg.d * PB[cfg.wdtype]


def algorithmic_bytes(cfg, stats: np.ndarray) -> float:
    """Touched bytes of one token given per-layer stats rows {|A|, |A_h|, e0, e1}:
    predictor (V, U, c) of every used expert, gate(+up) rows of predicted-active
    neurons, down columns of neurons with h != 0, index + h of each active
    neuron, and the router for MoE."""
    pb = PB[cfg.pdtype]
    per_expert = pb * cfg.rank * (cfg.d + cfg.F) + 4 * cfg.F
    if cfg.pdtype == "i8row":
        per_expert += 4 * (cfg.rank + cfg.F)      # one fp32 scale per row of U and of V
    rows_in = 2 if cfg.gated else 1
    w = wrow_bytes(cfg)
    tot = 0.0
    for a, ah, _, _ in stats:
        tot += cfg.top_k * per_expert + rows_in * a * w + ah * w + 8 * a
        if cfg.n_experts > 1:
            tot += cfg.n_experts * cfg.d * 2
    return tot


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def code_hash(src: str) -> str:
    """sha256/16 of C/C++ source with its comments and blank space removed,
    so that editing a comment keeps recorded counters valid while any change
    of code voids them."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()[:16]


def kernel_hash() -> str:
    with open(KERNEL_SRC, encoding="utf-8") as f:
        return code_hash(f.read())


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source and this workload; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    kv = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_sha256_16") != kernel_hash() or kv.get("workload") != workload:
        return None
    try:
        return float(kv["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                try:
                    rows.append((float(f[1]), float(f[2]), f[5:9]))
                except ValueError:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for _, _, flags in rows:
            for n, v in zip(names, flags):
                if v.lower().startswith("active"):
                    seen.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": sorted(seen), "samples": len(rows)}


def build_handle(cfg, B, device: int, active):
    h = B.pi_ffn_create(cfg.n_layers, cfg.d, cfg.F, cfg.rank, act=cfg.act, w_dtype=cfg.wdtype,
                        pred_dtype=cfg.pdtype, n_experts=cfg.n_experts, top_k=cfg.top_k,
                        device=device)
    for l in range(cfg.n_layers):
        lw = synth.make_layer(cfg, l, "cuda", active)
        B.pi_ffn_load_layer(h, l, lw.experts, lw.router,
                            np.stack([e.freq for e in lw.experts]).astype(np.float32))
        del lw
    torch.cuda.empty_cache()
    return h


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def oracle_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_sample_layers(cfg, n_layers: int, active):
    import oracle
    out = []
    for l in range(n_layers):
        lw = synth.make_layer(cfg, l, "cuda" if torch.cuda.is_available() else "cpu", active)
        n = synth.to_numpy
        ex = [oracle.Expert(act=cfg.act, wdtype=cfg.wdtype, pdtype=cfg.pdtype, w_gate=n(e.w_gate),
                            w_up=n(e.w_up), w_down=n(e.w_down), c=n(e.c), U=n(e.U), V=n(e.V),
                            s_gate=n(e.s_gate), s_up=n(e.s_up), s_down=n(e.s_down),
                            sU=n(e.sU), sV=n(e.sV))
              for e in lw.experts]
        out.append((ex, None if lw.router is None else n(lw.router)))
        del lw
    return out


def oracle_token_layer(layers, cfg, t: int, l: int) -> float:
    """Seconds for the oracle to run token t through sample layer l."""
    import oracle
    ex, router = layers[l % len(layers)]
    r = synth.token_input(cfg, t).double().numpy()
    t0 = time.perf_counter()
    oracle.decode_layer(r, ex, router)
    return time.perf_counter() - t0


def cpu_baseline(cfg, active, budget_s: float = 15.0, n_layers: int = 2):
    layers = oracle_sample_layers(cfg, n_layers, active)
    oracle_token_layer(layers, cfg, 0, 0)                 # page in, build
    secs, n, t = 0.0, 0, 0
    while secs < budget_s and n < 64:
        secs += oracle_token_layer(layers, cfg, t, n)
        n += 1
        t += 1
    per_token = secs / n * cfg.n_layers
    return {"value": 1.0 / per_token, "unit": "tok/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} token-layers ({n_layers} distinct layers of {cfg.n_layers}), "
                      f"fp64 oracle, time scaled by {cfg.n_layers} layers per token",
            "projected_from": f"{n} token-layers timed, scaled to {cfg.n_layers}-layer tokens"}


def run_reference(args, cfg, active, rank: int, world: int):
    if rank != 0:
        return 0
    layers = oracle_sample_layers(cfg, 2, active)
    for s in range(args.warmup):
        oracle_token_layer(layers, cfg, s, s)
    secs = 0.0
    for s in range(args.steps):
        secs += oracle_token_layer(layers, cfg, args.warmup + s, s)
    per_token = secs / args.steps * cfg.n_layers
    value = 1.0 / per_token
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_token * 1e3,
        "projected_from": f"{args.steps} token-layers timed ({secs:.2f} s of oracle time), "
                          f"each scaled by {cfg.n_layers} layers: ms_per_step is a projection",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(cfg, active, None),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"each step = one token through one of 2 sampled layers, "
                                   f"time scaled by {cfg.n_layers} layers"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (identity when not distributed)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, fp16 same rate)"
    return 1590.0, "fallback 1.59 PFLOP/s"


def run_prefill(args, cfg, rank: int, world: int) -> int:
    """Dense prefill of the workload's prompt (T tokens) through the stack on the
    tcgen05 path: one step = the whole prompt through every layer."""
    from activation_sparse_decode_threshold_b200 import binding as B
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    T = cfg.prefill_tokens or 512
    h = build_handle(cfg, B, local, None)
    L = cfg.n_layers
    R = synth.prefill_input(cfg, T, "cuda")
    r = torch.empty_like(R)
    for _ in range(args.warmup):
        r.copy_(R)
        B.pi_dense_ffn_prefill(h, 0, L, T, r)
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for s in range(args.steps):
            r.copy_(R)                      # the copy sits outside the events
            ev[s][0].record(stream)
            B.pi_dense_ffn_prefill(h, 0, L, T, r)
            ev[s][1].record(stream)
        torch.cuda.synchronize()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(ms)
    B.pi_ffn_destroy(h)
    if rank != 0:
        return 0
    flop = 2.0 * T * cfg.top_k * cfg.d * cfg.F * (3 if cfg.gated else 2) * L
    tflops = flop / (total_ms / args.steps / 1e3) / 1e12
    peak, kind = measured_tensor_peak()
    print(json.dumps({
        "metric": "dense prefill TFLOP/s (tcgen05 path)", "value": tflops, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 MMA, f32 accumulate", "data": "synthetic",
        "config": dict(workload_config(cfg, None, None), workload=f"{cfg.name}-prefill{T}", tokens=T),
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None, "peak_source": kind,
                     "flop_per_step": flop},
        "gpu_launches": 5 * L * args.steps,
        "clocks": clk.summary(),
    }), flush=True)
    return 0


def workload_config(cfg, active, measured_active):
    return {"workload": cfg.name, "layers": cfg.n_layers, "d_model": cfg.d, "d_ff": cfg.F,
            "rank": cfg.rank, "act": cfg.act, "weights": cfg.wdtype, "predictor": cfg.pdtype,
            "experts": cfg.n_experts, "top_k": cfg.top_k, "batch": 1, "tokens_per_step": 1,
            "target_active": active if active is not None else cfg.mean_active,
            "measured_active": measured_active,
            "l2": "inputs larger than L2: each token streams >1 GB of weights; no flush needed",
            "parallelism": "replicas (one independent stack per GPU)"}


# ---------------------------------------------------------------------------
# Further workloads, each on its own handle (reported beside the headline)
# ---------------------------------------------------------------------------
def decode_rate(cfg, B, local: int, active, steps: int, warmup: int, h=None) -> dict:
    """Decode tok/s and achieved GB/s of one workload: `steps` tokens timed with
    CUDA events after `warmup`, inputs resident, clocks sampled meanwhile."""
    own = h is None
    if own:
        h = build_handle(cfg, B, local, active)
    L = cfg.n_layers
    inputs = synth.token_inputs(cfg, steps + warmup, "cuda", 1000)
    resid = inputs.clone()
    stats = torch.zeros((steps + warmup, L, 4), device="cuda", dtype=torch.int32)
    for s in range(warmup):
        B.pi_sparse_ffn_decode(h, 0, L, resid[s], None, stats[s])
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.2)
        for s in range(steps):
            ev[s][0].record(stream)
            B.pi_sparse_ffn_decode(h, 0, L, resid[warmup + s], None, stats[warmup + s])
            ev[s][1].record(stream)
        torch.cuda.synchronize()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    if own:
        B.pi_ffn_destroy(h)
    ms = [a.elapsed_time(b) for a, b in ev]
    st = stats[warmup:].cpu().numpy()
    avg_bytes = float(np.mean([algorithmic_bytes(cfg, st[s]) for s in range(steps)]))
    mean_s = float(np.mean(ms)) / 1e3
    peak, kind = measured_peaks()
    gbs = avg_bytes / mean_s / 1e9
    return {"tok_s": 1.0 / mean_s, "ms_per_token": mean_s * 1e3, "achieved_gbs": gbs,
            "roofline_frac": gbs / peak, "peak_gbs": peak, "peak_source": kind,
            "algorithmic_bytes_per_token": avg_bytes,
            "measured_active": float(st[:, :, 0].mean() / (cfg.F * cfg.top_k)),
            "nonzero_h_fraction": float(st[:, :, 1].mean() / (cfg.F * cfg.top_k)),
            "tokens_timed": steps, "warmup": warmup, "clocks": clk.summary()}


def prefill_rate(cfg, B, local: int, h, steps: int = 3, warmup: int = 2) -> dict:
    """Dense prefill of the workload's prompt through every layer (tcgen05)."""
    T = cfg.prefill_tokens or 512
    L = cfg.n_layers
    R = synth.prefill_input(cfg, T, "cuda")
    r = torch.empty_like(R)
    for _ in range(warmup):
        r.copy_(R)
        B.pi_dense_ffn_prefill(h, 0, L, T, r)
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for s in range(steps):
            r.copy_(R)
            ev[s][0].record(stream)
            B.pi_dense_ffn_prefill(h, 0, L, T, r)
            ev[s][1].record(stream)
        torch.cuda.synchronize()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    flop = 2.0 * T * cfg.top_k * cfg.d * cfg.F * (3 if cfg.gated else 2) * L
    peak, kind = measured_tensor_peak()
    tf = flop / (ms / 1e3) / 1e12
    return {"tokens": T, "ms_per_prompt": ms, "tflops": tf, "roofline_frac": tf / peak,
            "peak_tflops": peak, "peak_source": kind, "prompts_timed": steps, "clocks": clk.summary()}


def batch_rate(cfg, B, local: int, h, nb: int, steps: int = 8, warmup: int = 3) -> dict:
    """Small-batch decode: `nb` tokens per step through pi_sparse_ffn_decode_batch,
    `steps` steps timed with CUDA events after `warmup`, inputs resident."""
    L = cfg.n_layers
    R = synth.token_inputs(cfg, nb * (steps + warmup), "cuda", 2000)
    stats = torch.zeros((steps + warmup, L, 4), device="cuda", dtype=torch.int32)
    bufs = [R[i * nb:(i + 1) * nb].clone() for i in range(steps + warmup)]
    for i in range(warmup):
        B.pi_sparse_ffn_decode_batch(h, 0, L, bufs[i], None, stats[i])
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(warmup, warmup + steps):
            B.pi_sparse_ffn_decode_batch(h, 0, L, bufs[i], None, stats[i])
        e1.record(stream)
        torch.cuda.synchronize()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    ms = e0.elapsed_time(e1) / steps
    st = stats[warmup:].cpu().numpy()
    # touched bytes per step: predictor once per launch group, the union's gate/up
    # rows, the down rows of union neurons with some h != 0, index + mask entries
    pb = PB[cfg.pdtype]
    groups = -(-nb // (4 if cfg.wdtype == "bf16" else 8))
    w = wrow_bytes(cfg)
    per_layer = [groups * (pb * cfg.rank * (cfg.d + cfg.F) + 4 * cfg.F) + (2 if cfg.gated else 1) * u * w
                 + uh * w + 8 * u for s_ in st for (u, _, uh, _) in s_]
    byts = float(np.sum(per_layer)) / steps
    peak, kind = measured_peaks()
    return {"tokens_per_step": nb, "tok_s": nb / (ms / 1e3), "ms_per_step": ms,
            "achieved_gbs": byts / (ms / 1e3) / 1e9, "roofline_frac": byts / (ms / 1e3) / 1e9 / peak,
            "peak_source": kind, "union_per_layer": float(st[:, :, 0].mean()),
            "predicted_per_layer_summed_over_tokens": float(st[:, :, 1].mean()),
            "launch_groups": groups, "steps_timed": steps, "clocks": clk.summary()}


def tp_rate(cfg, B, local: int, h, steps: int = 32, warmup: int = 4) -> dict:
    """The tensor-parallel layer sequence on one rank holding every neuron: per
    layer pi_sparse_ffn_decode_partial, (the all-reduce of y, an identity on
    one rank) and pi_residual_add -- the fused decode's work in 2 L launches."""
    L = cfg.n_layers
    R = synth.token_inputs(cfg, steps + warmup, "cuda", 3000)
    y = torch.empty(cfg.d, device="cuda")

    def token(r):
        for l in range(L):
            B.pi_sparse_ffn_decode_partial(h, l, r, y)
            B.pi_residual_add(h, r, y)
    for i in range(warmup):
        token(R[i])
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(warmup, warmup + steps):
        token(R[i])
    e1.record(stream)
    torch.cuda.synchronize()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    ms = e0.elapsed_time(e1) / steps
    return {"tok_s": 1e3 / ms, "ms_per_token": ms, "launches_per_token": 2 * L, "ranks": 1,
            "note": "per-layer launches of the sharded path with one rank; the all-reduce is an identity"}


def run_extras(B, local: int, steps: int) -> dict:
    """The other workloads of the method's measurement plan, each on its own
    handle: the mistral7b sparsity sweep, falcon40b, mixtral47b decode and the
    512-token dense prefill of the mixtral47b shape, small-batch decode of
    mistral7b, and the llama7b and mixtral47b shapes with the 8-bit per-row
    predictor.  (Small-batch decode of llama7b runs on the headline's handle.)"""
    out = {}
    m = synth.CONFIGS["mistral7b"]
    for a in m.sweep:
        if a == m.mean_active:
            h = build_handle(m, B, local, None)
            try:
                out[f"mistral7b@active{a}"] = decode_rate(m, B, local, None, steps, 8, h)
                out["mistral7b-batch4"] = batch_rate(m, B, local, h, 4)
                out["mistral7b-batch8"] = batch_rate(m, B, local, h, 8)
            finally:
                torch.cuda.synchronize()
                B.pi_ffn_destroy(h)
        else:
            out[f"mistral7b@active{a}"] = decode_rate(m, B, local, a, steps, 8)
        torch.cuda.empty_cache()
    out["falcon40b"] = decode_rate(synth.CONFIGS["falcon40b"], B, local, None, max(16, steps // 2), 8)
    torch.cuda.empty_cache()
    mx = synth.CONFIGS["mixtral47b"]
    h = build_handle(mx, B, local, None)
    try:
        out["mixtral47b"] = decode_rate(mx, B, local, None, steps, 8, h)
        out["mixtral47b-prefill512"] = prefill_rate(mx, B, local, h)
    finally:
        torch.cuda.synchronize()
        B.pi_ffn_destroy(h)
    torch.cuda.empty_cache()
    for name in ("llama7b-i8pred", "mixtral47b-i8pred"):
        out[name] = decode_rate(synth.CONFIGS[name], B, local, None, steps, 8)
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama7b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--active", type=float, default=None, help="target active fraction (bias shift)")
    ap.add_argument("--layers", type=int, default=None, help="override layer count (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads (sweep, falcon40b, mixtral47b, prefill)")
    ap.add_argument("--prefill", action="store_true",
                    help="time the dense tensor-core prefill of the workload's prompt instead of decode")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = synth.CONFIGS[args.config]
    if args.layers:
        cfg = synth.small(cfg, n_layers=args.layers)
    active = args.active

    if args.impl == "reference":
        return run_reference(args, cfg, active, rank, world)
    if args.prefill:
        return run_prefill(args, cfg, rank, world)

    from activation_sparse_decode_threshold_b200 import binding as B
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    h = build_handle(cfg, B, local, active)
    K, W, L = args.steps, args.warmup, cfg.n_layers
    first = rank * (K + W)
    inputs = synth.token_inputs(cfg, K + W, "cuda", first)
    resid = torch.empty((K + W, cfg.d), device="cuda")
    resid.copy_(inputs)
    stats = torch.zeros((K + W, L, 4), device="cuda", dtype=torch.int32)
    stream = torch.cuda.current_stream()

    for s in range(W):
        B.pi_sparse_ffn_decode(h, 0, L, resid[s], None, stats[s])
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.25)
        t_start.record(stream)
        for s in range(K):
            ev[s][0].record(stream)
            B.pi_sparse_ffn_decode(h, 0, L, resid[W + s], None, stats[W + s])
            ev[s][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    if B.pi_sync(h) != B.PI_OK:
        raise RuntimeError(B.pi_last_error())
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, "cuda")
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    value = job_throughput(K, world, total_ms)

    st = stats[W:].cpu().numpy()
    bytes_per_token = [algorithmic_bytes(cfg, st[s]) for s in range(K)]
    avg_bytes = float(np.mean(bytes_per_token))
    avg_launch_s = float(np.mean(launch_ms)) / 1e3
    achieved = avg_bytes / avg_launch_s / 1e9
    peak, peak_kind = measured_peaks()
    measured_active = float(st[:, :, 0].mean() / (cfg.F * cfg.top_k))
    nonzero_frac = float(st[:, :, 1].mean() / (cfg.F * cfg.top_k))

    e2e = None
    if not args.no_e2e:
        hin = torch.empty((K, cfg.d), dtype=torch.float32).pin_memory()
        hout = torch.empty((K, cfg.d), dtype=torch.float32).pin_memory()
        hin.copy_(inputs[W:].cpu())
        for s in range(3):
            B.pi_sparse_ffn_decode_host(h, 0, L, hin[s], hout[s])
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(K):
            B.pi_sparse_ffn_decode_host(h, 0, L, hin[s], hout[s])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
        e2e = {"value": job_throughput(K, world, e2e_ms), "unit": "tok/s",
               "h2d_bytes_per_step": 4 * cfg.d, "d2h_bytes_per_step": 4 * cfg.d}

    extra = None
    if world == 1 and not args.no_extra and not args.layers and args.config == "llama7b" and active is None:
        extra = {f"llama7b-batch{nb}": batch_rate(cfg, B, local, h, nb) for nb in (4, 8, 16)}
        extra["llama7b-tp1-per-layer"] = tp_rate(cfg, B, local, h)
    torch.cuda.synchronize()
    B.pi_ffn_destroy(h)
    torch.cuda.empty_cache()
    if extra is not None:
        extra.update(run_extras(B, local, 64))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0


    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, active)

    wl = cfg.name if active is None else f"{cfg.name}@active{active}"
    traffic = recorded_traffic(wl)
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.wdtype if cfg.wdtype != "int4g32" else "int4",
        "data": "synthetic (seeded random weights of the workload's shape, Gaussian token inputs)",
        "config": dict(workload_config(cfg, active, measured_active), workload=wl,
                       nonzero_h_fraction=nonzero_frac, accumulate="f32"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": avg_bytes,
                     "avg_launch_ms": avg_launch_s * 1e3, "kernel": "decode_kernel"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": K,
        "clocks": clk.summary(),
        "extra": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
