"""Benchmark of the rotated W4G128 linear layer on B200.

A step is one pass of the whole hot path (activation scaling, K Givens
layers, int4 dequant and the contraction, all inside paro_linear) through
every W4G128 projection of LAYERS distinct Llama-3-8B-shaped decoder layers
(fused QKV 4096->6144, O 4096->4096, fused gate+up 4096->28672,
down 14336->4096; K = 8 rotation layers, 64 pairs per group) for one decode
batch of TOKENS synthetic tokens. LAYERS copies make each step's weights
(4 x 113 MB) larger than the 126 MB L2, so no step reads weights from L2.

value = algorithmic HBM bytes of all ranks / max-over-ranks device time:
per projection 0.5195 B per weight (int4 q + fp16 s + int4 z per 128), the
fp16 activations read and outputs written, and the rotation parameters
(per pair one fp32 cos/sin pair and two channel bytes, plus 1/alpha).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--tokens T] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "ParoQuant W4G128 linear: decode HBM GB/s, prefill TFLOP/s, % of roofline"
# decoder-layer linears (QKV and gate+up fused), by model shape
MODELS = {
    "llama3-8b": [("qkv", 4096, 6144), ("o", 4096, 4096), ("gate_up", 4096, 28672), ("down", 14336, 4096)],
    "qwen3-4b": [("qkv", 2560, 6144), ("o", 4096, 2560), ("gate_up", 2560, 19456), ("down", 9728, 2560)],
    "qwen3-14b": [("qkv", 5120, 7168), ("o", 5120, 5120), ("gate_up", 5120, 34816), ("down", 17408, 5120)],
}
PROJ = MODELS["llama3-8b"]
K_LAYERS = 8
GROUP = 128          # channels per quantisation (and rotation) group; --group changes it


def weight_bytes(n_in, n_out, group=None):
    g = group or GROUP
    return n_in * n_out // 2 + (n_out * n_in // g) * 2 + (n_out * n_in // g) // 2


def rot_param_bytes(n_in, K=K_LAYERS, P=None):
    P = P or GROUP // 2
    return K * (n_in // GROUP) * P * (8 + 2) + 4 * n_in


def linear(B, rot, x, qw, sp, zp, n_out, Y=None, ws=None):
    """The layer call: paro_linear for group 128, paro_linear_ex otherwise."""
    if GROUP == 128:
        return B.paro_linear(rot, x, qw, sp, zp, n_out, Y=Y, ws=ws)
    return B.paro_linear_ex(rot, x, qw, sp, zp, n_out, group=GROUP, Y=Y, ws=ws)


def call_bytes(T, n_in, n_out):
    return weight_bytes(n_in, n_out) + 2 * T * n_in + 2 * T * n_out + rot_param_bytes(n_in)


# DRAM bytes (read + write) per decode-kernel launch, mean over the four
# projections (qkv 13.24 MB, o 8.89 MB, gate+up 61.18 MB, down 31.00 MB), from
# one ncu capture at 16 tokens of the decode kernel built from the gemv.cu
# whose SHA-256 prefix is GEMV_TRAFFIC_SOURCE; reported only while gemv.cu is
# that file (any change to it nulls the figure until it is captured again).
GEMV_TRAFFIC_PER_LAUNCH_T16 = (13244928 + 8886016 + 61185280 + 31004928) / 4
GEMV_TRAFFIC_SOURCE = "4c0f8d3a1a030105"


def gemv_source_sha() -> str:
    import hashlib
    with open(os.path.join(ROOT, "rotated_w4_linear_b200", "csrc", "gemv.cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def gemv_traffic(tokens: int, model: str):
    """The captured DRAM traffic per decode launch, if it belongs to this
    workload and to the current kernel source; else None."""
    if tokens != 16 or model != "llama3-8b" or GROUP != 128 or gemv_source_sha() != GEMV_TRAFFIC_SOURCE:
        return None
    return GEMV_TRAFFIC_PER_LAUNCH_T16


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for ln in f:
                    p = [x.strip() for x in ln.split(",")]
                    if len(p) >= 9 and p[1].replace(".", "").isdigit():
                        rows.append(p)
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------------------- ranks
def max_over_ranks(dist, values, device=None):
    """Every rank passes its own device times; every rank gets the maximum of
    each over all ranks (the slowest rank defines the step)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def decode_line(args, world, elapsed, e2e_elapsed, kern_s, step_bytes, gemv_bytes, n_calls,
                hbm_peak, peak_kind, h2d, d2h, per_proj, n_launch, clocks):
    """The JSON line of the decode workload. Times are max-over-ranks seconds
    for args.steps steps; every rank moved step_bytes per step."""
    value = step_bytes * args.steps * world / elapsed / 1e9
    achieved = gemv_bytes * args.steps / kern_s / 1e9
    return {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 (int4 weights, fp32 accumulate)",
        "data": f"synthetic (seeded {args.model}-shaped layers; weights quantised on the GPU from T W)",
        "config": config(args),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": gemv_traffic(args.tokens, args.model),
                     "kernel": "gemv_kernel (int4 decode; timed on unrotated inputs, the branch that "
                               "reads X in natural order)",
                     "us_per_launch": 1e6 * kern_s / (args.steps * n_calls),
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "e2e": {"value": step_bytes * args.steps * world / e2e_elapsed / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "decode_kernel_per_projection": per_proj,
        "gpu_launches": n_launch,
        "clocks": clocks,
    }


def emit(line, rank):
    """Rank 0 prints the one JSON line; the other ranks print nothing."""
    if rank == 0:
        print(json.dumps(line), flush=True)
        return True
    return False


# --------------------------------------------------------------------------- oracle baseline
def cpu_baseline(tokens: int, budget_s: float = 12.0, torch=None, B=None):
    """The CPU fp64 oracle as it stands, on a bounded sample: whole projections
    of one layer (every output row), one after another until ~budget_s.
    With torch and the binding given, the four projections of that layer
    also run through paro_linear on the GPU and are compared with the
    oracle's outputs: the literal max |dY| beside the 1e-2 bar and the format
    floor (the ideal fp16 pipeline's own max error), and the Frobenius error.
    Returns (cpu_baseline, parity or None)."""
    from oracle import paro_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = 1
    done_bytes, t_total, n_calls, names = 0, 0.0, 0, []
    par = {"max_abs_dY": 0.0, "format_floor": 0.0, "rel_fro": 0.0, "max_abs_Y": 0.0}
    for i, (name, n_in, n_out) in enumerate(PROJ * 16):
        seed = synth.layer_seed(2, i % len(PROJ))
        pairs, theta, alpha = synth.rotation_params(n_in, K_LAYERS, seed, pairs_per_group=GROUP // 2, group=GROUP)
        q, s, z = synth.w4_codes(n_out, n_in, seed, group=GROUP)
        x = synth.activations(tokens, n_in, seed)
        t0 = time.perf_counter()
        y_ref = O.linear(x, pairs, theta, alpha, q, s, z, group=GROUP)
        t_total += time.perf_counter() - t0
        done_bytes += call_bytes(tokens, n_in, n_out)
        n_calls += 1
        names.append(name)
        if B is not None and i < len(PROJ):
            rot = B.paro_rot_create(pairs, theta, alpha, group=GROUP)
            qw, sp, zp = B.paro_pack_weights(torch.from_numpy(q), torch.from_numpy(s), torch.from_numpy(z),
                                             group=GROUP)
            y = linear(B, rot, torch.from_numpy(x).cuda(), qw, sp, zp, n_out).cpu().numpy().astype(np.float64)
            rot.close()
            floor = O.linear_fp16_pipeline(x, pairs, theta, alpha, q, s, z, group=GROUP).astype(np.float64)
            rel, mx = O.output_errors(y, y_ref)
            par["max_abs_dY"] = max(par["max_abs_dY"], mx)
            par["rel_fro"] = max(par["rel_fro"], rel)
            par["format_floor"] = max(par["format_floor"], float(np.max(np.abs(floor - y_ref))))
            par["max_abs_Y"] = max(par["max_abs_Y"], float(np.max(np.abs(y_ref))))
        if t_total > budget_s:
            break
    base = {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{n_calls} projection calls ({'+'.join(names)}) of one layer, every output row, "
                      f"{tokens} tokens, fp64 numpy ({t_total:.1f} s)"}
    if B is None:
        return base, None
    par.update({"bar_abs": 1e-2, "bar_rel": 2e-3,
                "sample": f"the four projections of one {'-'.join(n for n, _, _ in PROJ)} layer at {tokens} tokens, "
                          "every output, GPU paro_linear against the fp64 oracle (max over the four)"})
    return base, par


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    step_bytes = sum(call_bytes(args.tokens, i, o) for _, i, o in PROJ)
    from oracle import paro_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = 1
    # one step of the reference arm: the four projections of one layer with
    # 1/16 of their output rows (a bounded sample of the GPU arm's step)
    inputs = []
    for i, (name, n_in, n_out) in enumerate(PROJ):
        seed = synth.layer_seed(2, i)
        pairs, theta, alpha = synth.rotation_params(n_in, K_LAYERS, seed, pairs_per_group=GROUP // 2, group=GROUP)
        q, s_, z = synth.w4_codes(n_out // 16, n_in, seed, group=GROUP)
        x = synth.activations(args.tokens, n_in, seed)
        inputs.append((x, pairs, theta, alpha, q, s_, z))
    times = []
    for k in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for inp in inputs:
            O.linear(*inp, group=GROUP)
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    sample_bytes = sum(call_bytes(args.tokens, i, o // 16) for _, i, o in PROJ)
    v = sample_bytes * len(times) / sum(times) / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config(args),
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": int(cores), "kind": "oracle",
                             "sample": "each step: the four projections of one layer with 1/16 of the output "
                                       f"rows, {args.tokens} tokens (step bytes {sample_bytes} of {step_bytes})"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config(args):
    shapes = ", ".join(f"{n} {i}x{o}" for n, i, o in PROJ)
    return {"workload": f"{getattr(args, 'model', 'llama3-8b')} decoder-layer W4G{GROUP} linears ({shapes}), "
                        f"decode {args.tokens} tokens, K={K_LAYERS} rotation layers x {GROUP // 2} pairs/group",
            "tokens": args.tokens, "layers_per_step": args.layers, "rotation_layers": K_LAYERS,
            "group": GROUP, "l2": f"inputs larger than L2: {args.layers} distinct layers per step",
            "parallelism": f"replicas x{args.gpus}"}


# --------------------------------------------------------------------------- rotation alone
def rotate_result(torch, B, local, T, K, P, steps, warmup, n_in=4096):
    """paro_rotate on X [T][n_in] (fp16 in, fp16 out), distinct inputs per
    call so that each pass moves more than L2, replayed from a CUDA graph.
    Algorithmic bytes: X read + X' written + the rotation parameters
    (per pair an fp32 cos/sin pair and two channel bytes, plus 1/alpha)."""
    torch.cuda.set_device(local)
    P = GROUP // 2 if P is None else P
    pairs, theta, alpha = synth.rotation_params(n_in, K, synth.layer_seed(1, K), pairs_per_group=P, group=GROUP)
    rot = B.paro_rot_create(pairs, theta, alpha, group=GROUP)
    copies = min(64, max(1, (512 << 20) // (4 * T * n_in)))   # > L2 for T >= 256
    xs = [torch.from_numpy(synth.activations(T, n_in, synth.layer_seed(1, c))).cuda() for c in range(copies)]
    ys = [torch.empty_like(x) for x in xs]
    stream = torch.cuda.current_stream()
    # one pass over the copies captured in a CUDA graph: small batches are
    # timed without the host's per-call launch cost
    for x, y in zip(xs, ys):
        B.paro_rotate(rot, x, y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for x, y in zip(xs, ys):
            B.paro_rotate(rot, x, y)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    per = e0.elapsed_time(e1) / 1e3 / (steps * len(xs))
    del g
    rot.close()
    nbytes = 4 * T * n_in + K * (n_in // GROUP) * P * 10 + 4 * n_in
    hbm_peak, _, kind = peaks()
    if GROUP == 256:
        kern = "rotate_tc256_kernel (tensor cores, 256-channel groups)"
    else:
        kern = "rotate_tc_kernel (tensor cores)" if T > 16 else "rotate_quad_kernel (Givens)"
    return {"workload": f"paro_rotate tokens={T} hidden={n_in} K={K} group={GROUP} pairs/group={P}",
            "us_per_call": per * 1e6, "GB/s": nbytes / per / 1e9,
            "roofline": {"bound": "hbm", "achieved": nbytes / per / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": nbytes / per / 1e9 / hbm_peak, "traffic": None, "kernel": kern,
                         "bytes_per_call": nbytes, "peak_source": f"{kind} hbm_gbs"},
            "copies": copies, "l2": "inputs larger than L2 (distinct copies per pass)" if 4 * T * n_in * copies > 126e6
            else "inputs smaller than L2", "clocks": clk.summary(), "fault_code": B.paro_fault_status(clear=True)}


def bench_rotate(args, torch, B, local):
    print(json.dumps(rotate_result(torch, B, local, args.tokens, args.rot_k, args.rot_pairs, args.steps,
                                   args.warmup)), flush=True)
    return 0


# --------------------------------------------------------------------------- prefill
def prefill_result(torch, B, local, T, steps, warmup, model):
    """One decoder layer's projections (`model` shapes) at T tokens: rotation +
    tensor-core GEMM per projection, replayed as a CUDA graph. Reports the
    layer's FLOP rate (2 T in out per projection; the time includes the
    rotation launches) against the measured dense 16-bit tensor peak, the
    rotation overhead against the same GEMMs on unrotated inputs (theta = 0,
    alpha = 1: no rotation launch), and the rotations alone."""
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    calls = []
    for i, (name, n_in, n_out) in enumerate(MODELS[model]):
        seed = synth.layer_seed(3, i)
        pairs, theta, alpha = synth.rotation_params(n_in, K_LAYERS, seed, pairs_per_group=GROUP // 2, group=GROUP)
        rot = B.paro_rot_create(pairs, theta, alpha, group=GROUP)
        w = torch.from_numpy(synth.weight(n_out, n_in, seed)).to(dev)
        qw, sp, zp = B.paro_pack_weights(*B.paro_quantize_weights(rot, w), group=GROUP)
        del w
        x = torch.from_numpy(synth.activations(T, n_in, seed)).to(dev)
        calls.append(dict(rot=rot, n_in=n_in, n_out=n_out, qw=qw, sp=sp, zp=zp, x=x,
                          y=torch.empty((T, n_out), dtype=torch.float16, device=dev),
                          ws=B.workspace(T, n_in, n_out, dev)))

    def step(rotate=True):
        for p in calls:
            linear(B, p["rot"] if rotate else None, p["x"], p["qw"], p["sp"], p["zp"], p["n_out"], Y=p["y"],
                   ws=p["ws"])

    def rotations():
        for p in calls:
            B.paro_rotate(p["rot"], p["x"], p["ws"][: p["x"].numel() * 2].view(torch.float16).view(p["x"].shape))

    step(); step(False); rotations()
    torch.cuda.synchronize()
    graphs = {}
    for key, fn in (("rotated", lambda: step(True)), ("unrotated", lambda: step(False)), ("rotation", rotations)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graphs[key] = g
    for _ in range(warmup):
        for g in graphs.values():
            g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = {}
    with ClockSampler(local) as clk:
        for key, g in graphs.items():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            times[key] = e0.elapsed_time(e1) / 1e3 / steps
    flops = sum(2.0 * T * p["n_in"] * p["n_out"] for p in calls)
    _, _, kind = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tc_peak = float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        tc_peak = 1400.0
    tf = flops / times["rotated"] / 1e12
    shapes = ", ".join(f"{n} {i}x{o}" for n, i, o in MODELS[model])
    res = {"workload": f"prefill {model} decoder-layer projections ({shapes}), {T} tokens, K={K_LAYERS}",
           "ms_per_layer": 1e3 * times["rotated"], "ms_per_layer_unrotated": 1e3 * times["unrotated"],
           "ms_rotation_alone": 1e3 * times["rotation"],
           "TFLOP/s": tf, "TFLOP/s_unrotated_control": flops / times["unrotated"] / 1e12,
           "rotation_overhead": times["rotated"] / times["unrotated"] - 1.0,
           "rotation_share": times["rotation"] / times["rotated"],
           "roofline": {"bound": "tensor", "achieved": tf, "peak": tc_peak, "unit": "TFLOP/s",
                        "frac": tf / tc_peak, "traffic": None,
                        "kernel": "gemm_w4_kernel (tcgen05), timed with its rotation launches (the whole layer)",
                        "flops_per_layer": flops,
                        "peak_source": f"{kind} bf16_tflops_sustained (fp16 and bf16 share the dense tensor rate)"},
           "note": "the unrotated control reads X from HBM; the rotated layer's GEMM reads X' that the rotation "
                   "just wrote, partly from L2, so the overhead can come out below zero",
           "l2": "inputs larger than L2", "clocks": clk.summary(),
           "fault_code": B.paro_fault_status(clear=True)}
    del graphs
    for p in calls:
        p["rot"].close()
    return res


def bench_prefill(args, torch, B, local):
    print(json.dumps(prefill_result(torch, B, local, args.tokens, args.steps, args.warmup, args.model)), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--tokens", type=int, default=16)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--impl", default="paro", choices=["paro", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the rotation and prefill figures that the decode line carries by default")
    ap.add_argument("--workload", default="decode", choices=["decode", "rotate", "prefill"],
                    help="decode: the headline step; rotate: paro_rotate alone (hidden 4096); "
                         "prefill: one layer's projections at --tokens (tensor-core GEMM)")
    ap.add_argument("--model", default="llama3-8b", choices=sorted(MODELS),
                    help="decoder-layer shapes (the headline line is llama3-8b)")
    ap.add_argument("--group", type=int, default=128, choices=[64, 128, 256],
                    help="channels per quantisation and rotation group (the headline is 128)")
    ap.add_argument("--rot-k", type=int, default=8)
    ap.add_argument("--rot-pairs", type=int, default=None)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    global PROJ, GROUP
    PROJ = MODELS[args.model]
    GROUP = args.group

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    from rotated_w4_linear_b200 import binding as B

    if args.workload == "rotate":
        return bench_rotate(args, torch, B, local)
    if args.workload == "prefill":
        return bench_prefill(args, torch, B, local)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    T = args.tokens
    dev = torch.device("cuda", local)
    # ---- setup (untimed): per layer copy and projection, rotation + RTN on the GPU
    layers = []
    for l in range(args.layers):
        projs = []
        for i, (name, n_in, n_out) in enumerate(PROJ):
            seed = synth.layer_seed(2, 100 * (rank * args.layers + l) + i)
            pairs, theta, alpha = synth.rotation_params(n_in, K_LAYERS, seed, pairs_per_group=GROUP // 2,
                                                        group=GROUP)
            rot = B.paro_rot_create(pairs, theta, alpha, group=GROUP)
            w = torch.from_numpy(synth.weight(n_out, n_in, seed)).to(dev)
            q, s, z = B.paro_quantize_weights(rot, w)
            qw, sp, zp = B.paro_pack_weights(q, s, z, group=GROUP)
            del w, q, s, z
            x = torch.from_numpy(synth.activations(T, n_in, seed)).to(dev)
            y = torch.empty((T, n_out), dtype=torch.float16, device=dev)
            ws = B.workspace(T, n_in, n_out, dev)
            projs.append(dict(name=name, n_in=n_in, n_out=n_out, rot=rot, qw=qw, sp=sp, zp=zp, x=x, y=y, ws=ws))
        layers.append(projs)
    torch.cuda.synchronize()
    calls = [p for projs in layers for p in projs]
    step_bytes = sum(call_bytes(T, p["n_in"], p["n_out"]) for p in calls)
    stream = torch.cuda.current_stream()

    def step(rotate=True):
        for p in calls:
            linear(B, p["rot"] if rotate else None, p["x"], p["qw"], p["sp"], p["zp"], p["n_out"], Y=p["y"],
                   ws=p["ws"])

    # The step is captured once into a CUDA graph (a decode engine replays its
    # step the same way); replays remove the host's per-call launch cost from
    # the device timing. The e2e number below goes through the per-call API.
    step()
    torch.cuda.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    # the decode kernel alone (no rotation launch), for its own roofline
    g_gemv = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_gemv):
        step(rotate=False)
    for _ in range(args.warmup):
        g_step.replay()
        g_gemv.replay()
    torch.cuda.synchronize()

    # ---- timed region: device time of K steps
    hbm_peak, _, peak_kind = peaks()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = vis.split(",")[local].strip() if vis else str(local)
    with ClockSampler(smi_index) as clk:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k_start, k_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for k in range(args.steps):
            g_step.replay()
        t_end.record(stream)
        # the decode kernel's launches alone, same inputs, same number of steps
        k_start.record(stream)
        for k in range(args.steps):
            g_gemv.replay()
        k_end.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    elapsed = t_start.elapsed_time(t_end) / 1e3
    kern_s = k_start.elapsed_time(k_end) / 1e3
    clocks = clk.summary()

    # per projection: the decode kernel alone, and rotation + decode kernel,
    # one graph per projection shape
    per_proj = {}
    for i, (name, n_in, n_out) in enumerate(PROJ):
        sel = [p for p in calls if p["name"] == name]
        res = {}
        for rotate in (False, True):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for p in sel:
                    linear(B, p["rot"] if rotate else None, p["x"], p["qw"], p["sp"], p["zp"], p["n_out"],
                           Y=p["y"], ws=p["ws"])
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            res[rotate] = e0.elapsed_time(e1) * 1e3 / (args.steps * len(sel))
            del g
        nb = weight_bytes(n_in, n_out) + 2 * T * (n_in + n_out)
        per_proj[name] = {"us": round(res[False], 2), "GB/s": round(nb / res[False] / 1e3, 1),
                          "us_with_rotation": round(res[True], 2)}
    n_launch = args.steps * len(calls) * 2          # rotation + decode kernel per projection
    gemv_bytes = sum(weight_bytes(p["n_in"], p["n_out"]) + 2 * T * (p["n_in"] + p["n_out"]) for p in calls)

    # ---- e2e: every step's X comes from pinned host memory and its Y goes
    # back to host memory, through the per-call public API. A serving loop
    # overlaps the transfers with compute: one host->device copy of all of a
    # step's inputs and one device->host copy of all its outputs, each on its
    # own copy stream (the link is full duplex), double-buffered against the
    # compute stream.
    x_sizes = [p["x"].numel() for p in calls]
    y_sizes = [p["y"].numel() for p in calls]
    xh = torch.empty(sum(x_sizes), dtype=torch.float16).pin_memory()
    yh = torch.empty(sum(y_sizes), dtype=torch.float16).pin_memory()
    xh.copy_(torch.cat([p["x"].reshape(-1).cpu() for p in calls]))
    h2d, d2h = xh.numel() * 2, yh.numel() * 2
    sets = []
    for _ in range(2):                              # double-buffered device inputs/outputs
        xd = torch.empty(sum(x_sizes), dtype=torch.float16, device=dev)
        yd = torch.empty(sum(y_sizes), dtype=torch.float16, device=dev)
        xs_, ys_, ox, oy = [], [], 0, 0
        for p, nx, ny in zip(calls, x_sizes, y_sizes):
            xs_.append(xd[ox:ox + nx].view_as(p["x"]))
            ys_.append(yd[oy:oy + ny].view_as(p["y"]))
            ox += nx
            oy += ny
        sets.append(dict(xd=xd, yd=yd, xs=xs_, ys=ys_, ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(),
                         ev_out=torch.cuda.Event(), used=False))
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    # the public per-call API of a decode loop: one prepared layer per
    # projection (weights and workspace checked once, X and Y per call)
    for p in calls:
        p["layer"] = B.ParoLinear(p["rot"], p["qw"], p["sp"], p["zp"], p["n_in"], p["n_out"], group=GROUP)
        p["layer"]._workspace(T)

    def e2e_step(k):
        st = sets[k & 1]
        with torch.cuda.stream(h2d_stream):        # inputs: one copy, after the set was last read
            if st["used"]:
                h2d_stream.wait_event(st["ev_done"])
            st["xd"].copy_(xh, non_blocking=True)
            st["ev_in"].record(h2d_stream)
        stream.wait_event(st["ev_in"])
        if st["used"]:
            stream.wait_event(st["ev_out"])         # the set's previous outputs are on the host
        for p, x_, y_ in zip(calls, st["xs"], st["ys"]):
            p["layer"](x_, Y=y_)
        st["ev_done"].record(stream)
        with torch.cuda.stream(d2h_stream):        # outputs: one copy
            d2h_stream.wait_event(st["ev_done"])
            yh.copy_(st["yd"], non_blocking=True)
            st["ev_out"].record(d2h_stream)
        st["used"] = True

    for k in range(3):
        e2e_step(k)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)                       # the first input copy is inside the timed region
    for k in range(args.steps):
        e2e_step(k)
    e1.record(d2h_stream)                           # after the last step's outputs reached the host
    torch.cuda.synchronize()
    e2e_elapsed = e0.elapsed_time(e1) / 1e3

    elapsed, e2e_elapsed, kern_s = max_over_ranks(dist, [elapsed, e2e_elapsed, kern_s], dev)
    line = decode_line(args, world, elapsed, e2e_elapsed, kern_s, step_bytes, gemv_bytes, len(calls),
                       hbm_peak, peak_kind, h2d, d2h, per_proj, n_launch, clocks)
    # a bounded wait that ran out would void the numbers: the fault word must read 0
    line["fault_code"] = B.paro_fault_status(clear=True)
    del g_step, g_gemv
    for projs in layers:
        for p in projs:
            p["rot"].close()
    del layers, calls, sets
    torch.cuda.empty_cache()
    # the other two kernels of the path, in the same run: the rotation alone
    # (paro_rotate on [8192 x 4096], K = 8) and one prefill layer at 8192
    # tokens (tensor-core GEMM, with the rotation overhead); every rank runs
    # them on its own GPU, rank 0 reports its figures
    if not args.no_extra:
        xs = min(args.steps, 20)
        line["rotate"] = rotate_result(torch, B, local, 8192, K_LAYERS, None, xs, 3)
        line["prefill"] = prefill_result(torch, B, local, 8192, xs, 3, args.model)
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], line["parity"] = cpu_baseline(T, torch=torch, B=B)
    emit(line, rank)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
