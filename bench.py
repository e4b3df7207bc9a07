"""Benchmark: decode tokens/s of the activation-sparse FFN stack at batch 1 on B200.

A step is one decode token through every layer of the stack: predictor, bitmask,
compaction into the block-local active lists, gather-GEMV with ReLU/ReGLU, scatter-axpy
down projection and the stack glue, all in one persistent kernel launch
(pi_decode_stack).  Inputs are seeded synthetic power-law layers generated on the device
(no datasets or trained weights exist here); every step gets a fresh token x0 ~ N(0, I).

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

With N > 1 (torchrun) every rank runs an independent replica of the stack on its own GPU:
batch-1 decode of one stack does not shard without a collective per layer that costs
more than the layer itself, so the job's throughput is the sum over replicas.
The reference arm (--impl reference) times the CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import pi_synth as S  # noqa: E402

METRIC = "decode tokens/s of sparse FFN stack at batch 1; active-bytes HBM GB/s vs peak"
WORKLOADS = {"llama2_7b": S.LLAMA2_7B, "falcon40b": S.FALCON_40B, "llama2_70b_q4": S.LLAMA2_70B_Q4,
             "opt175b": S.OPT_175B, "ffn512_cal": S.FFN512_CAL, "ffn512_lit": S.FFN512_LIT,
             "llama2_7b_adaptive": S.LLAMA2_7B_ADAPTIVE}
CSRC = os.path.join(ROOT, "activation_sparse_decode_bitmask_b200", "csrc")
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


# ------------------------------------------------------------------ helpers
def p_bytes(wl):
    return 4 if wl.p_dtype == "f32" else 2


def bytes_per_neuron(wl):
    n_mat = 3 if wl.act == "reglu" else 2
    s = {"f32": 4.0, "f16": 2.0, "q4_0": 18.0 / 32.0}[wl.w_dtype]
    return n_mat * wl.d_model * s


def predictor_bytes(wl):
    """P1 + P2 + thresholds per layer (read densely every step)."""
    return wl.d_model * wl.rank * p_bytes(wl) + wl.rank * wl.d_ff * p_bytes(wl) + 4 * wl.d_ff


def stack_predictor_bytes(wl):
    """Predictor bytes of one step through the whole stack (layers may differ in rank)."""
    return sum(predictor_bytes(wl.at_layer(l)) for l in range(wl.n_layers))


FUSED_SOURCES = ("pi_fused.cu", "pi_rowmath.cuh", "pi_ptx.cuh")


def source_hash():
    """Hash of the fused kernel's source files: a recorded ncu traffic figure applies only
    to the kernel it was captured from."""
    h = hashlib.sha256()
    for name in FUSED_SOURCES:
        with open(os.path.join(CSRC, name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profiled_traffic(workload, n_layers, batch):
    """DRAM bytes per launch (read + write) from a committed ncu capture of this exact
    kernel source.  Captures run a shorter stack of the same layers; the record holds
    bytes per layer, scaled here by the stack depth of the timed launch."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as fh:
        d = json.load(fh)
    rec = d.get(f"{workload}/B{batch}")
    if not rec or rec.get("source_hash") != source_hash():
        return None
    return int(rec["dram_bytes_per_layer"] * n_layers)


class ClockSampler:
    """NVML clock and throttle-reason samples while the timed region runs."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, index, period_s=0.01):
        self.samples, self.reasons = [], 0
        self.stop_ev = threading.Event()
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, b in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_min_mhz": float(min(self.samples)),
                "sm_max_mhz": float(self.max_mhz), "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, batch: int, ms_max: float) -> float:
    """Tokens per second of the whole job: every rank decodes `steps` steps of `batch`
    tokens on its own replica; the time is the slowest rank's."""
    return world * steps * batch / (ms_max / 1e3)


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle timing
def _oracle_layers(wl, n, device):
    from oracle import cpp as OC
    return [OC.Layer(S.make_layer(wl, l, device).to_numpy(), wl.act) for l in range(n)]


def _time_layer_steps(fn, budget_s, min_steps=2):
    """Mean seconds of fn(k) over as many calls as fit the budget (at least min_steps)."""
    times, k = [], 0
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        fn(k)
        times.append(time.perf_counter() - t0)
        k += 1
        if time.perf_counter() - t_start > budget_s and k >= min_steps:
            break
    return float(np.mean(times)), k


def oracle_tokens_per_s(wl, budget_s=15.0, batch=1, device="cuda"):
    """Time the C++ oracle's decode of one token, layer by layer, on the host cores: a
    bounded sample of layer-steps cycling through the first layers, scaled to the stack.
    Three legs share the budget: the sparse oracle on every core (the reported value), the
    sparse oracle on one core, and the dense FFN (every neuron, no predictor) on every core."""
    from oracle import cpp as OC
    OC.build()
    n_layers_sample = min(2, wl.n_layers)
    layers = _oracle_layers(wl, n_layers_sample, device)
    xs = S.make_inputs(wl.with_(x_dtype="f32"), 64 * batch, "cpu", stream_id=99).double().numpy()
    xb = lambda k: xs[(k % 64) * batch:(k % 64 + 1) * batch]
    all_cores = OC.max_threads()
    try:
        OC.set_threads(all_cores)
        sparse, k_sp = _time_layer_steps(lambda k: layers[k % n_layers_sample].layer_step(xb(k), wl.x_dtype),
                                         0.45 * budget_s)
        dense, k_de = _time_layer_steps(lambda k: layers[k % n_layers_sample].dense_ffn(xb(k)), 0.25 * budget_s, 1)
        OC.set_threads(1)
        single, k_1 = _time_layer_steps(lambda k: layers[k % n_layers_sample].layer_step(xb(k), wl.x_dtype),
                                        0.3 * budget_s, 1)
    finally:
        OC.set_threads(all_cores)
    L = wl.n_layers
    out = {"value": batch / (sparse * L), "cores": all_cores,
           "single_core_value": round(batch / (single * L), 6),
           "dense_value": round(batch / (dense * L), 6),
           "sample": (f"C++ oracle (fp64 loops), batch {batch}, layers 0..{n_layers_sample - 1} of {wl.name}, "
                      f"scaled to {L} layers: sparse layer-step {sparse * 1e3:.1f} ms on {all_cores} cores "
                      f"({k_sp} steps), {single * 1e3:.1f} ms on 1 core ({k_1} steps); dense FFN "
                      f"{dense * 1e3:.1f} ms on {all_cores} cores ({k_de} steps)")}
    return out


# ------------------------------------------------------------------ our arm
def build_stack(pi, wl, reorder=True):
    layers = []
    for l in range(wl.n_layers):
        wll = wl.at_layer(l)
        desc = pi.make_desc(wll.d_model, wll.d_ff, wll.rank, wll.act, wll.w_dtype, wll.x_dtype, wll.p_dtype)
        L = S.make_layer(wl, l, "cuda")
        g = pi.load_layer(desc, L.tensors())
        if reorder:
            pi.reorder_hot_prefix(g, L.freq)
        layers.append(g)
        del L
        torch.cuda.empty_cache()
    return layers


def run_ours(args, world, rank, local):
    import activation_sparse_decode_bitmask_b200 as pi
    wl = WORKLOADS[args.workload]
    if args.layers:
        wl = wl.with_(n_layers=args.layers)
    B = args.batch
    torch.cuda.set_device(local)
    t_gen = time.perf_counter()
    layers = build_stack(pi, wl, reorder=not args.no_reorder)
    torch.cuda.synchronize()
    t_gen = time.perf_counter() - t_gen
    r_max = max(wl.at_layer(l).rank for l in range(wl.n_layers))
    ws = pi.Workspace(wl.d_model, wl.d_ff, r_max, max(B, 1), wl.n_layers)
    K, W = args.steps, args.warmup
    xs = S.make_inputs(wl, (W + K + wl.prompt_len) * B, "cuda", stream_id=1000 + rank)
    xs = xs.view(W + K + wl.prompt_len, B, wl.d_model)
    # untimed prompt vectors (the workload's input length), then warm-up steps
    for p in range(wl.prompt_len):
        pi.decode_stack(layers, xs[p], B, ws)
    for w in range(W):
        pi.decode_stack(layers, xs[wl.prompt_len + w], B, ws)
    st = ws.status()
    if st != 0:
        raise RuntimeError(f"warm-up failed: {pi.status_str(st)}")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    base = wl.prompt_len + W
    dist_barrier(world)
    torch.cuda.synchronize()
    # the end-to-end leg runs the first timed steps' inputs again: copy them to pinned host
    # memory now, since the stack overwrites its input with its output
    Ke = min(K, args.e2e_steps)
    xh = xs[base:base + Ke].cpu().pin_memory()
    act0 = ws.active_total()
    n0 = pi.kernel_launches()
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("timed")
        e0.record(stream)
        for k in range(K):
            pi.decode_stack(layers, xs[base + k], B, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    dist_barrier(world)
    st = ws.status()
    if st != 0:
        raise RuntimeError(f"timed run failed: {pi.status_str(st)}")
    act1 = ws.active_total()
    launches = pi.kernel_launches() - n0
    ms_local = e0.elapsed_time(e1)
    ms = dist_max(ms_local, world)
    ms_step = ms / K
    value = whole_job_rate(world, K, B, ms)
    active_per_step = (act1 - act0) / K                     # summed over layers
    pred_bytes = stack_predictor_bytes(wl)
    algo_bytes = pred_bytes + active_per_step * bytes_per_neuron(wl)
    achieved = algo_bytes / (ms_local / K / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    traffic = profiled_traffic(wl.name, wl.n_layers, B)

    # end to end through the host-buffer entry point: H2D x, the stack, D2H x, sync.  The
    # call returns only after the stream is synchronised, so a host clock brackets it.
    xo = torch.empty_like(xh[0]).pin_memory()
    for k in range(min(3, Ke)):
        pi.decode_stack_host(layers, xh[k], xo, B, ws)
    dist_barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk_e2e:
        h0 = time.perf_counter()
        for k in range(Ke):
            pi.decode_stack_host(layers, xh[k], xo, B, ws)
        h1 = time.perf_counter()
    e2e_ms = dist_max((h1 - h0) * 1e3, world)
    xbytes = B * wl.d_model * (4 if wl.x_dtype == "f32" else 2)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "q4_0" if wl.w_dtype == "q4_0" else wl.w_dtype, "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.n_layers, "d_model": wl.d_model, "d_ff": wl.d_ff,
                   "rank": wl.rank, "act": wl.act, "batch": B, "weights": wl.w_dtype,
                   "mean_firing_p": wl.mean_p, "hot_reorder": not args.no_reorder,
                   "avg_active_per_layer": round(active_per_step / wl.n_layers, 1),
                   "us_per_layer": round(ms_step * 1e3 / wl.n_layers, 3),
                   "algorithmic_bytes_per_step": int(algo_bytes),
                   "predictor_bytes_per_step": int(pred_bytes),
                   "predictor_bytes_per_step_at_uniform_rank": int(wl.n_layers * predictor_bytes(wl)),
                   "layer_ranks": sorted({wl.at_layer(l).rank for l in range(wl.n_layers)}),
                   "l2": f"no flush: per-step working set {algo_bytes / 1e9:.2f} GB > 126 MB L2",
                   "parallelism": f"replicas x{world}", "setup_s": round(t_gen, 1)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": ("pi::fused_kernel (one launch per step)" if launches == K else
                                f"whole step: {launches // K} launches of the batched kernels per step"),
                     "peak_source": peak_kind},
        "e2e": {"value": round(world * Ke * B / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": xbytes, "d2h_bytes_per_step": xbytes, "steps": Ke,
                "timing": "host wall clock around the calls (each call synchronises)",
                "clocks": clk_e2e.summary()},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_tokens_per_s(wl, budget_s=args.cpu_budget, batch=B)
        out["cpu_baseline"] = {"value": round(cb["value"], 6), "unit": "tokens/s", "cores": cb["cores"],
                               "kind": "oracle", "sample": cb["sample"],
                               "single_core_value": cb["single_core_value"], "dense_value": cb["dense_value"]}
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The oracle arm: the C++ oracle decodes K tokens through the whole stack on the host
    cores (every layer: predictor, compaction, sparse FFN, glue), timed on the host clock.
    K is capped so that the timed steps fit the CPU budget."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    if args.layers:
        wl = wl.with_(n_layers=args.layers)
    B = args.batch
    from oracle import cpp as OC
    OC.build()
    cores = OC.max_threads()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    layers = _oracle_layers(wl, wl.n_layers, dev)
    xs = S.make_inputs(wl.with_(x_dtype="f32"), 64 * B, "cpu", stream_id=99).double().numpy()
    xb = lambda k: xs[(k % 64) * B:(k % 64 + 1) * B]

    def step(k):
        OC.decode_stack(xb(k), layers, wl.x_dtype)

    t0 = time.perf_counter()
    step(0)
    est = time.perf_counter() - t0
    W = min(args.warmup, 3)
    K = max(1, min(args.steps, int(args.cpu_budget / max(est, 1e-6))))
    for k in range(1, W):
        step(k)
    t0 = time.perf_counter()
    for k in range(K):
        step(W + k)
    el = time.perf_counter() - t0
    tok_s = K * B / el
    sample = (f"{K} decode steps of the C++ oracle through all {wl.n_layers} layers of {wl.name} "
              f"(batch {B}) on {cores} cores, {el:.2f} s on the host clock")
    out = {"impl": "reference", "metric": METRIC, "value": round(tok_s, 6), "unit": "tokens/s", "n_gpus": world,
           "steps": K, "warmup": W, "ms_per_step": round(el / K * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": wl.name, "layers": wl.n_layers, "d_model": wl.d_model, "d_ff": wl.d_ff,
                      "rank": wl.rank, "act": wl.act, "batch": B, "weights": wl.w_dtype},
           "cpu_baseline": {"value": round(tok_s, 6), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(tok_s, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama2_7b")
    ap.add_argument("--layers", type=int, default=0, help="override the stack depth (measurement only)")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--e2e-steps", type=int, default=256)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-reorder", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
