#!/usr/bin/env python
"""Benchmark of the fused MoE FFN forward (ffn_norm -> router top-k -> FP8 SwiGLU experts ->
combine + shared expert) through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C4] [--impl ours|reference]

One step = one moe_forward over one batch of synthetic tokens (seeded generator, inputs resident
in HBM).  Default workload: the full DeepSeek-V3.2 MoE shape at a prefill batch (T=16384,
d=7168, moe_inter=2048, 256 experts, top-8, one shared expert, FP8 e4m3 weights with float32
128x128 block scales).  With N > 1 (torchrun) every rank runs an independent replica on its own
GPU -- the layer has no exchange step when tokens are data-parallel -- and ``value`` is the
tokens of all ranks divided by the slowest rank's time.

Rank 0 prints one JSON line with the throughput, the dominant kernel's roofline fraction
(timed live with CUDA events around it), the end-to-end number through host buffers, the
oracle's CPU throughput on a bounded token sample, and the SM clocks seen during timing.
``--impl reference`` times the CPU oracle itself on the same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "MoE-layer tokens/s at DeepSeek-V3.2 shape; % of HBM or FP8 tensor-core roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_traffic.json")
KERNEL_SOURCES = ("gemm.cu", "ptx.cuh", "internal.h", "api.cu")


def kernel_sources_hash() -> str:
    """Hash of the sources that decide the grouped GEMM's memory traffic."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_ffn_norm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (read + write) from the committed ncu capture, or None when the capture
    is missing or was taken on different kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_sources_sha256_16") != kernel_sources_hash():
        return None
    return rec.get("workloads", {}).get(workload, {}).get(kernel)


def c5_alpha():
    with open(os.path.join(ROOT, "tests", "golden", "c5_alpha.json")) as f:
        return json.load(f)["alpha"]


def make_inputs(shape, device):
    return synthetic.generate(shape, device=device, alpha=c5_alpha() if shape.zipf_bias else None)


# ------------------------------------------------------------------------------------------------
# algorithmic work
# ------------------------------------------------------------------------------------------------
def work(shape, counts, act8=True):
    """FLOPs and bytes of one step and of the grouped GEMM up (the dominant kernel)."""
    T, d, I, E, k, Is = shape.T, shape.d, shape.I, shape.E, shape.k, shape.Is
    wb = 1 if shape.wtype == "fp8" else 2
    ab = 1 if (wb == 1 and act8) else 2
    touched = int((np.asarray(counts) > 0).sum())
    scl = lambda r, c: (r // 128) * (c // 128) * 4 if wb == 1 else 0
    expert_bytes = 3 * d * I * wb + 2 * scl(I, d) + scl(d, I)
    shared_bytes = 3 * d * Is * wb + 2 * scl(Is, d) + scl(d, Is)
    step_bytes = touched * expert_bytes + shared_bytes + E * d * 2 + 4 * T * d * 2
    step_flops = T * shape.flops_per_token()
    up_flops = 2 * d * 2 * I * T * k + 2 * d * 2 * Is * T
    up_bytes = touched * (2 * d * I * wb + 2 * scl(I, d)) + 2 * d * Is * wb + 2 * scl(Is, d) + \
        (T * k + T) * d * ab + (T * k * I + T * Is) * ab
    return dict(touched=touched, step_bytes=step_bytes, step_flops=step_flops, up_flops=up_flops, up_bytes=up_bytes)


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU oracle timing
# ------------------------------------------------------------------------------------------------
def oracle_throughput(shape, inputs, budget_s=20.0, max_tokens=1024, seed=0, act8=True, gpu_out=None):
    """Tokens/s of the oracle on a bounded seeded sample of the workload's tokens (all host cores).
    With the GPU's output of the same step (bf16 bits, [T, d]) the sampled tokens are also compared:
    max |err| / RMS of the oracle output and the fraction of bit-identical elements."""
    import oracle
    o = oracle.Oracle(shape, inputs, act_fp8=act8 and shape.wtype == "fp8")
    cores = oracle.default_threads()
    rng = np.random.default_rng(seed)
    n0 = min(shape.T, cores)
    t0 = time.perf_counter()
    o.forward(rng.choice(shape.T, n0, replace=False))
    dt0 = time.perf_counter() - t0
    n = int(min(max_tokens, shape.T, max(n0, budget_s / max(dt0, 1e-6) * n0)))
    toks = rng.choice(shape.T, n, replace=False)
    t1 = time.perf_counter()
    ref = o.forward(toks)
    dt = time.perf_counter() - t1
    res = {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{n} of the workload's {shape.T} tokens (seeded), full layer per token, {dt:.1f} s"}
    if gpu_out is not None:
        g = oracle.bf16_bits_to_f64(gpu_out[toks])
        r = oracle.bf16_bits_to_f64(ref["out"])
        rms = float(np.sqrt(np.mean(r ** 2)))
        res["parity"] = {"tokens": int(n), "max_err_over_rms": float(np.abs(g - r).max() / rms),
                         "bitexact_frac": float(np.mean(gpu_out[toks] == ref["out"])), "bound": 2e-2}
    return res


# ------------------------------------------------------------------------------------------------
def run_reference(args, shape, rank):
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inputs = make_inputs(shape, dev)
    import oracle
    o = oracle.Oracle(shape, inputs, act_fp8=args.act == "fp8" and shape.wtype == "fp8")
    cores = oracle.default_threads()
    n = min(shape.T, max(1, cores))
    rng = np.random.default_rng(1)
    for _ in range(args.warmup):
        o.forward(rng.choice(shape.T, n, replace=False))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.forward(rng.choice(shape.T, n, replace=False))
    dt = time.perf_counter() - t0
    v = n * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(shape, args.act == "fp8"),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} seeded tokens of {shape.T} per step, full layer per token"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(values, world, device="cpu"):
    """Every rank's timings -> the slowest rank's, on every rank (one MAX all-reduce; no-op alone)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_rate(tokens_per_rank, world, ms_per_step):
    """Tokens/s of the whole job: all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


def config_block(shape, act8=True):
    desc = synthetic.DESCRIPTIONS.get(shape.name, "reduced case of " + shape.name.split("-")[0] + " (profiling only)")
    return {"workload": f"{shape.name}: {desc}", "tokens": shape.T, "dim": shape.d,
            "moe_inter": shape.I, "experts": shape.E, "top_k": shape.k, "shared_inter": shape.Is,
            "weights": "e4m3 + fp32 128x128 block scales" if shape.wtype == "fp8" else "bf16",
            "activations": ("e4m3 1x128 groups into the expert GEMMs" if act8 else
                            "bf16 (e4m3 weight tiles widened to bf16 on chip)") if shape.wtype == "fp8" else "bf16",
            "parallelism": "replicas (token data parallel, no collective)",
            "l2": "inputs larger than L2 (expert weights stream from HBM every step)"}


def run_ours(args, shape, rank, world, device):
    import mixture_experts_ffn_norm_b200 as moe
    torch.cuda.set_device(device)
    inputs = make_inputs(shape, device)
    cfg = moe.Config.from_shape(shape)
    act8 = args.act == "fp8" and shape.wtype == "fp8"
    if shape.wtype == "fp8" and not act8:
        cfg = dataclasses.replace(cfg, amode=moe.MOE_ACT_BF16)
    layer = moe.MoELayer(cfg, {n: v for n, v in inputs.items() if n not in ("x", "residual")}, device=device)
    x, r = inputs["x"], inputs["residual"]
    out = torch.empty_like(x)
    ro = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    nev = 8
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record(stream)          # creates the underlying CUDA event before it is handed to the library
    for _ in range(W):
        layer.forward(x, r, out, ro)
    torch.cuda.synchronize()
    st = moe.moe_get_status(layer.workspace)
    if st != moe.MOE_OK:
        raise RuntimeError(moe.status_string(st))
    counts = torch.zeros(shape.E, dtype=torch.int32, device=device)
    near_tie = torch.zeros(shape.T, dtype=torch.uint8, device=device)
    if shape.E > 0:                       # a dense block has no routing
        moe.moe_debug_routing(cfg, layer.workspace, counts=counts, near_tie=near_tie)
    counts = counts.cpu().numpy()
    near_ties = int(near_tie.sum().item())

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nvtx = torch.cuda.nvtx            # named ranges for a timeline profiler (no-ops otherwise)
    nvtx.range_push(f"moe_forward x{K} (timed)")
    start.record(stream)
    for i in range(K):
        layer.forward(x, r, out, ro, events=ev[i])
    end.record(stream)
    nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end) / K
    stage = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(nev - 1)] for i in range(K)])
    st = moe.moe_get_status(layer.workspace)
    if st != moe.MOE_OK:
        raise RuntimeError(moe.status_string(st))

    # end to end through host buffers: every step copies its inputs from pinned host memory and its
    # results (out and the new residual) back.  Three streams pipeline step i+1's upload, step i's
    # forward and step i-1's download on double-buffered device tensors, ordered by events.
    xh, rh = x.cpu().pin_memory(), r.cpu().pin_memory()
    oh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    roh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    rd = [torch.empty_like(x) for _ in range(2)]
    od = [torch.empty_like(x) for _ in range(2)]
    rod = [torch.empty_like(x) for _ in range(2)]
    s_up, s_dn = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    up_done, fw_done, dn_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e_ in up_done + fw_done + dn_done:
        e_.record(stream)

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_up):
                s_up.wait_event(fw_done[b])                 # step i-2 no longer reads xd[b], rd[b]
                xd[b].copy_(xh, non_blocking=True)
                rd[b].copy_(rh, non_blocking=True)
                up_done[b].record(s_up)
            stream.wait_event(up_done[b])
            stream.wait_event(dn_done[b])                   # step i-2's results left od[b], rod[b]
            layer.forward(xd[b], rd[b], od[b], rod[b], stream=stream)
            fw_done[b].record(stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(fw_done[b])
                oh[b].copy_(od[b], non_blocking=True)
                roh[b].copy_(rod[b], non_blocking=True)
                dn_done[b].record(s_dn)
        stream.wait_stream(s_up)
        stream.wait_stream(s_dn)

    ke = max(3, min(K, 20))
    e2e_steps(4)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nvtx.range_push(f"moe_forward from host buffers x{ke} (e2e)")
    e0.record(stream)
    s_up.wait_event(e0)
    s_dn.wait_event(e0)
    e2e_steps(ke)
    e1.record(stream)
    nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / ke
    if not torch.equal(oh[(ke - 1) & 1], out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    # optional: the same forward captured once into a CUDA graph and replayed (one graph launch per step)
    graph_ms = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.graph(graph, stream=side):
            layer.forward(x, r, out, ro)
        for _ in range(W):
            graph.replay()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(K):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        graph_ms = g0.elapsed_time(g1) / K
        del graph
        if moe.moe_get_status(layer.workspace) != moe.MOE_OK:
            raise RuntimeError("graph replay failed")

    # optional: the same layer through moe_forward_next_norm (the next block's attn_norm fused into
    # the combine; the update itself is not written)
    nn_ms = None
    if args.next_norm and shape.E > 0:
        t_ = layer.t
        g_next = (1.0 + synthetic.normal(shape.seed, "next_norm_w", (shape.d,), 0.1, device=device).float()).contiguous()
        xn_next, r_next = torch.empty_like(x), torch.empty_like(x)
        call = lambda: moe.moe_forward_next_norm(cfg, x, r, t_["norm_w"], t_["gate_w"], t_.get("gate_bias"),
                                                 layer.wstruct, g_next, None, xn_next, r_next, layer.workspace)
        for _ in range(W):
            call()
        torch.cuda.synchronize()
        barrier()
        n0, n1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0.record(stream)
        for _ in range(K):
            call()
        n1.record(stream)
        torch.cuda.synchronize()
        barrier()
        nn_ms = n0.elapsed_time(n1) / K
        if moe.moe_get_status(layer.workspace) != moe.MOE_OK:
            raise RuntimeError("moe_forward_next_norm failed")

    ms, e2e_ms, nn_ms, graph_ms = max_over_ranks(
        [ms, e2e_ms, -1.0 if nn_ms is None else nn_ms, -1.0 if graph_ms is None else graph_ms], world, device)
    if rank != 0:
        return

    P, src = peaks()
    wk = work(shape, counts, act8)
    fp8 = act8             # FP8 tensor-core arithmetic
    tensor_peak = (2.0 if fp8 else 1.0) * P["bf16_tflops_sustained"]
    up_ms = float(stage[:, 4].mean())
    t_flop = wk["up_flops"] / (tensor_peak * 1e12) * 1e3
    t_byte = wk["up_bytes"] / (P["hbm_gbs"] * 1e9) * 1e3
    if t_flop >= t_byte:
        roof = {"bound": "tensor", "achieved": wk["up_flops"] / (up_ms * 1e-3) / 1e12, "peak": tensor_peak,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": wk["up_bytes"] / (up_ms * 1e-3) / 1e9, "peak": P["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(shape.name, "gemm_up") if act8 or shape.wtype != "fp8" else None
    roof["algorithmic_bytes"] = wk["up_bytes"]
    roof["kernel"] = ("gemm_kernel up (w1|w3 + SwiGLU + FP8 quant of h)" if act8 else
                      "gemm_kernel up (w1|w3 + SwiGLU, bf16 operands)")
    roof["peak_source"] = (f"{src} MEASURED_PEAKS.json: " +
                           ("2 x bf16_tflops_sustained (fp8 dense = 2 x bf16)" if roof["bound"] == "tensor" and fp8 else
                            "bf16_tflops_sustained" if roof["bound"] == "tensor" else "hbm_gbs"))
    roof["ms_per_launch"] = up_ms
    value = whole_job_rate(shape.T, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic (seeded counter-based generator)",
        "config": config_block(shape, act8),
        "roofline": roof,
        "step_roofline": {"tflops": wk["step_flops"] / (ms * 1e-3) / 1e12,
                          "tflops_frac_of_peak": wk["step_flops"] / (ms * 1e-3) / 1e12 / tensor_peak,
                          "gbs": wk["step_bytes"] / (ms * 1e-3) / 1e9,
                          "gbs_frac_of_hbm": wk["step_bytes"] / (ms * 1e-3) / 1e9 / P["hbm_gbs"],
                          "touched_experts": wk["touched"]},
        "stage_ms": {n: float(stage[:, j].mean()) for j, n in enumerate(
            ["norm", "gate_gemm", "topk", "route", "gemm_up", "gemm_down", "combine"])},
        "e2e": {"value": whole_job_rate(shape.T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": 2 * x.numel() * 2,
                "d2h_bytes_per_step": 2 * x.numel() * 2, "ms_per_step": e2e_ms,
                "how": "moe_forward on host buffers: per step H2D of x and residual, D2H of out and the new "
                       "residual (pinned), uploads / forwards / downloads pipelined on three streams"},
        "gpu_launches": moe.launches_per_forward(cfg) * K,
        "near_tie_tokens": near_ties,   # tokens whose top-k was re-decided in float64
        "clocks": clk,
    }
    if graph_ms is not None and graph_ms > 0:
        line["cuda_graph"] = {"ms_per_step": graph_ms, "tokens_per_s": whole_job_rate(shape.T, world, graph_ms),
                              "how": "the forward captured once with torch.cuda.graph and replayed; one graph launch "
                                     "per step instead of the per-kernel launches"}
    if nn_ms is not None and nn_ms > 0:
        line["next_norm_fused"] = {
            "ms_per_step": nn_ms, "tokens_per_s": whole_job_rate(shape.T, world, nn_ms),
            "plain_ms_per_step": ms,
            "how": "moe_forward_next_norm: the same layer with the next block's attn_norm in the combine; "
                   "the update is not written (saves its write and the separate norm's read of it, "
                   f"{2 * x.numel() * 2 / 1e6:.0f} MB per step)"}
    if world == 1 and not args.no_cpu_baseline:
        gbits = out.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        line["cpu_baseline"] = oracle_throughput(shape, inputs, budget_s=args.cpu_budget, act8=act8, gpu_out=gbits)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="C4", choices=sorted(synthetic.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--tokens", type=int, default=0, help="override T (smaller cases for profiling)")
    ap.add_argument("--experts", type=int, default=0, help="override E (smaller cases for profiling)")
    ap.add_argument("--graph", action="store_true", help="also time the forward replayed from a CUDA graph")
    ap.add_argument("--next-norm", action="store_true",
                    help="also time moe_forward_next_norm (the next block's attn_norm fused into the combine)")
    ap.add_argument("--act", default="fp8", choices=["fp8", "bf16"],
                    help="activations of the FP8-weight workloads: 1x128 FP8 (default) or bf16")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    shape = synthetic.CONFIGS[args.config]
    if args.tokens or args.experts:
        shape = dataclasses.replace(shape, name=shape.name + "-reduced", T=args.tokens or shape.T,
                                    E=args.experts or shape.E, zipf_bias=False)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, shape, rank)
        return
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    try:
        run_ours(args, shape, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
