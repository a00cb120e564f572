"""Benchmark of the QUADS rollout MoE layer hot path on B200.

One step = one forward of the large MoE layer (T=16384 tokens, H=4096,
I=1536, E=128 experts, top-8 routing with per-expert logit skew, RAC k=128
per GEMM): routing, NVFP4 quantization of X with residual scores, top-k
channel selection and RAC residuals, RAC weight gather, the grouped W4A4+RAC
gate/up GEMM with SwiGLU, quantization of h, gather, the grouped W4A4+RAC down
GEMM with router-weighted combine.  Weights are NVFP4 before timing (the
rollout engine holds quantized weights).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs an independent replica on its own batch (weak scaling, no collective on
the data path); time is the max over ranks.

Prints one JSON line (rank 0).  value = whole-job algorithmic TFLOP/s of the
layer (FP4 + RAC FLOPs of both GEMMs, padding not counted) over the device
time of the K timed steps.  The reference arm (--impl reference) times the CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "moe_t16384_e128"
METRIC = "W4A4+RAC grouped MoE GEMM TFLOPS and % FP4 peak; quantize GB/s and % HBM"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_PER_BF16 = 4.0          # nominal dense FP4 : BF16 tensor-core ratio (9 : 2.25 PFLOP/s)
NOMINAL_FP4_TFLOPS = 9000.0  # B200 dense FP4, datasheet (context)
QUANT_BYTES_PER_ELEM = 2.5625   # 2 B bf16 read + 0.5 B codes + 1/16 B scale written

# DRAM traffic of k_moe_gemm per launch (dram__bytes_read.sum + dram__bytes_write.sum,
# averaged over the gate/up and down launches of one step) from a one-pass ncu
# capture of this benchmark's two timed steps (the ncu command is kept with the
# profile summaries), valid only for the kernel code it was taken on: sha256 of
# gemm.cu + ptx.cuh + common.cuh with comments removed and whitespace collapsed
# (a comment edit leaves the kernel, and the figure, as is).
GEMM_TRAFFIC = {"bytes_per_launch": 2510646592, "sources_sha256": "73032c09631fc5ff9bc6af674e64f9246b28a629c20ce14fc86c1cf4f7b93e08"}


def _code_only(src: str) -> str:
    """C/C++ source without comments, whitespace runs collapsed (string literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"' or c == "'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c.isspace():
            if out and out[-1] != " ":
                out.append(" ")                  # a run of whitespace -> one space
            i += 1
        else:
            out.append(c)
            i += 1
    return "".join(out)


def gemm_traffic():
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm.cu", "ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "quantization_nvfp4_quantize_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    ok = GEMM_TRAFFIC["sources_sha256"] == h.hexdigest()
    return GEMM_TRAFFIC["bytes_per_launch"] if ok else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w4a16", action="store_true", help="skip the trainer-side W4A16 line of the default run")
    ap.add_argument("--no-formats", action="store_true", help="skip the W4A4 / W8A8 / BF16 grouped-GEMM table")
    ap.add_argument("--no-sweep", action="store_true", help="skip the layer-error sweep over RAC channels and outliers")
    ap.add_argument("--no-variants", action="store_true", help="skip the per-variant RAC step times")
    return ap.parse_args()


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sus=1400.0, source="fallback")


def tensor_peak(p, clk, per_bf16=1.0):
    """Tensor-core peak for a kernel timed inside the run: the burst bf16
    figure (a cuBLAS GEMM timed alone at full clock) times the dtype's nominal
    ratio to bf16, scaled by the median SM clock sampled during the timed
    region over its maximum (a clock-bound pipe).  Returns (peak, source)."""
    base = p["bf16"] * per_bf16
    if clk and clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        f = min(1.0, float(clk["sm_mhz"]) / float(clk["sm_max_mhz"]))
        return base * f, (f"{p['source']} bf16 burst x{per_bf16:g} x sampled SM clock "
                          f"{clk['sm_mhz']:.0f}/{clk['sm_max_mhz']:.0f} MHz")
    return base, f"{p['source']} bf16 burst x{per_bf16:g} (no clock samples)"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}.csv")
        self.gpu = gpu_index
        if enabled:
            try:
                self.f = open(self.path, "w")
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                             stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [s.strip() for s in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx = float(p[2])
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.remove(self.path)
        if not sm:
            return None
        loaded = [s for s in sm if s > 300] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    from quantization_nvfp4_quantize_b200 import workloads as wl, api
    from quantization_nvfp4_quantize_b200.moe import MoELayerW4A4
    if wl.CONFIGS[args.workload].w4a16:
        return run_ours_w4a16(args)

    ws, rank = init_dist("nccl" if torch.cuda.is_available() else "gloo")
    _, _, local = dist_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = wl.CONFIGS[args.workload]
    seed = args.seed + rank                      # independent replica per rank
    x = wl.activations(cfg, seed, device=dev)
    logits = wl.router_logits(cfg, seed, device=dev)
    w13, w2 = wl.weights(cfg, seed, device=dev)
    layer = MoELayerW4A4(w13, w2, cfg.tokens, cfg.topk, cfg.rac_k)
    del w13, w2
    torch.cuda.empty_cache()
    fl = wl.flops(cfg)
    step_flops = fl["fp4"] + fl["rac"]
    stream = torch.cuda.current_stream(dev)

    # per-kernel timing hooks around the two GEMMs and the two quantize calls
    ev = {"gemm": [], "quant": []}
    orig_gemm, orig_quant = api.grouped_gemm, api.quantize

    def timed(kind, fn):
        def wrap(*a, **k):
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            out = fn(*a, **k)
            e.record(stream)
            ev[kind].append((s, e, a, k))
            return out
        return wrap

    for _ in range(args.warmup):
        layer.forward(x, logits)
    torch.cuda.synchronize()
    barrier()

    api.grouped_gemm, api.quantize = timed("gemm", orig_gemm), timed("quant", orig_quant)
    import quantization_nvfp4_quantize_b200.moe as moe_mod
    moe_mod.api = api
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    if clocks.proc is not None:
        time.sleep(0.5)                 # let the sampler start before the timed region
    torch.cuda.synchronize()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        layer.forward(x, logits)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    api.grouped_gemm, api.quantize = orig_gemm, orig_quant
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, dev)

    gemm_ms = sum(s.elapsed_time(e) for s, e, _, _ in ev["gemm"])
    quant_ms = sum(s.elapsed_time(e) for s, e, _, _ in ev["quant"])
    n_gemm = len(ev["gemm"])
    # algorithmic work per step
    M = cfg.tokens * cfg.topk
    quant_elems = cfg.tokens * cfg.hidden + M * cfg.inter
    p = peaks()
    fp4_peak, peak_source = tensor_peak(p, clk, FP4_PER_BF16)
    gemm_fp4_tflops = fl["fp4"] * args.steps / (gemm_ms * 1e-3) / 1e12
    gemm_all_tflops = step_flops * args.steps / (gemm_ms * 1e-3) / 1e12
    quant_gbs = quant_elems * QUANT_BYTES_PER_ELEM * args.steps / (quant_ms * 1e-3) / 1e9

    # end to end through the public API with host buffers
    e2e = run_e2e(layer, x, logits, args, dev)
    # the streaming quantize kernel alone (tensor scale given: no amax pass, no
    # selection or residual), on the layer's own X and h
    qk = time_quantize_kernel(layer, x, args.steps, dev)
    # per step: route 3, X quantize 5 (amax, quantize, score reduce, select, residual),
    # gather 1, GEMM 1, h quantize 4 (its amax comes from the GEMM epilogue), gather 1, GEMM 1
    n_launch_per_step = 16
    out = {
        "metric": METRIC,
        "value": round(step_flops * args.steps * ws / (ms_max * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e2m1+e4m3 (fp32 accum), bf16 RAC", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: T={cfg.tokens} H={cfg.hidden} I={cfg.inter} E={cfg.experts} "
                               f"top-{cfg.topk} RAC k={cfg.rac_k}",
                   "l2": "inputs larger than L2 (NVFP4 weights 1.36 GB)", "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "tensor", "kernel": "k_moe_gemm",
                     "achieved": round(gemm_fp4_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_fp4_tflops / fp4_peak, 4), "traffic": gemm_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": peak_source + f" (nominal FP4:BF16 {FP4_PER_BF16:g})",
                     "frac_nominal_fp4": round(gemm_fp4_tflops / NOMINAL_FP4_TFLOPS, 4),
                     "achieved_incl_rac": round(gemm_all_tflops, 1),
                     "gemm_ms_per_step": round(gemm_ms / args.steps, 4), "launches_per_step": n_gemm // args.steps},
        "quantize": {"gbs": round(quant_gbs, 1), "peak_gbs": p["hbm"], "frac": round(quant_gbs / p["hbm"], 4),
                     "ms_per_step": round(quant_ms / args.steps, 4),
                     "bytes_per_elem": QUANT_BYTES_PER_ELEM, "elems_per_step": quant_elems,
                     "scope": "whole nvfp4_quantize calls (amax, quantize, score reduce, select, RAC residual)",
                     "kernel": qk},
        "e2e": e2e,
        "gpu_launches": n_launch_per_step * args.steps,
        "clocks": clk,
    }
    if not args.no_w4a16:
        # the trainer-side path (weight QDQ + W4A16 grouped GEMMs) on its own
        # workload, in the same run
        del layer, x, logits
        torch.cuda.empty_cache()
        w = run_ours_w4a16(args, workload="qat_w4a16_e128", emit=False)
        out["w4a16"] = {k: w[k] for k in ("metric", "value", "unit", "ms_per_step", "roofline", "qdq", "e2e")}
        out["w4a16"]["config"] = w["config"]["workload"]
        out["gpu_launches"] += w["gpu_launches"]
    if not args.no_formats:
        # the same grouped expert GEMMs on the same layer in other formats:
        # the pages quote native NVFP4 GEMMs at ~2x FP8 and ~4x BF16
        if "layer" in locals():
            del layer
        torch.cuda.empty_cache()
        out["gemm_formats"] = run_formats(args, dev)
        out["gpu_launches"] += out["gemm_formats"].pop("_launches")
    if not args.no_variants:
        # cost side of RAC: whole layer steps of the same workload without RAC
        # and with each RAC variant
        if "layer" in locals():
            del layer
        torch.cuda.empty_cache()
        out["rac_variants"] = run_rac_variants(args, dev)
        out["gpu_launches"] += out["rac_variants"].pop("_launches")
    if not args.no_sweep:
        # accuracy side of RAC: the error it leaves on one dense layer, by
        # compensated channel share and outlier strength (untimed)
        torch.cuda.empty_cache()
        out["error_sweep"] = run_error_sweep(args, dev)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, seed=args.seed, n_experts=64)
    if rank == 0:
        print(json.dumps(out), flush=True)
    return out


def run_rac_variants(args, dev):
    """Layer step time of the large layer without RAC and with each RAC
    variant (same inputs and routing), CUDA events around whole steps."""
    import torch
    from quantization_nvfp4_quantize_b200 import workloads as wl
    from quantization_nvfp4_quantize_b200 import moe as moe_mod
    cfg = wl.CONFIGS[WORKLOAD]
    x = wl.activations(cfg, args.seed, device=dev)
    logits = wl.router_logits(cfg, args.seed, device=dev)
    w13, w2 = wl.weights(cfg, args.seed, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 5))
    H, I = cfg.hidden, cfg.inter
    variants = (
        ("no_rac", dict(rac_k=0), 10),
        ("rac_k128", dict(rac_k=cfg.rac_k), 16),
        ("rac_50pct", dict(rac_k=moe_mod.rac_channels(50, H), rac_k_h=moe_mod.rac_channels(50, I)), 16),
        ("rac_second_pass", dict(rac_k=cfg.rac_k, rac_mode="nvfp4"), 20),
        ("rac_per_expert", dict(rac_k=cfg.rac_k, rac_scope="expert"), 17),
    )
    res, launches = {}, 0
    for name, kw, n_launch in variants:
        layer = moe_mod.MoELayerW4A4(w13, w2, cfg.tokens, cfg.topk, **kw)
        for _ in range(2):
            layer.forward(x, logits)
        torch.cuda.synchronize()
        s_ = torch.cuda.Event(enable_timing=True)
        e_ = torch.cuda.Event(enable_timing=True)
        s_.record(stream)
        for _ in range(steps):
            layer.forward(x, logits)
        e_.record(stream)
        torch.cuda.synchronize()
        res[name] = {"ms_per_step": round(s_.elapsed_time(e_) / steps, 4)}
        launches += n_launch * steps
        del layer
        torch.cuda.empty_cache()
    base = res["no_rac"]["ms_per_step"]
    for name in res:
        res[name]["overhead_vs_no_rac"] = round(res[name]["ms_per_step"] / base - 1, 4)
    res["k"] = {"rac_k128": [cfg.rac_k, cfg.rac_k], "rac_50pct": [moe_mod.rac_channels(50, H), moe_mod.rac_channels(50, I)]}
    res["note"] = "whole layer steps of the bench workload (X side, h side), CUDA events around the steps"
    res["_launches"] = launches
    return res


def run_error_sweep(args, dev):
    """err(k) = ||Y_RAC(k) - X What^T||_F / ||X What^T||_F of one dense layer
    for RAC on k% of the input channels (bf16 residual and the NVFP4 second
    pass) and outlier channels of growing strength."""
    from quantization_nvfp4_quantize_b200 import workloads as wl
    from quantization_nvfp4_quantize_b200.sweep import LayerErrorProbe, rac_channels
    sw = wl.SWEEP
    T, K, N = sw["tokens"], sw["channels"], sw["out"]
    ks = [rac_channels(p_, K) for p_ in sw["percents"]]
    probe = LayerErrorProbe(wl.dense_weight(N, K, args.seed, device=dev), T)
    res = {"metric": "||Y_RAC(k) - X What^T||_F / ||X What^T||_F",
           "workload": f"dense T={T} K={K} N={N}; X N(0,1) with {int(round(sw['outlier_frac'] * K))} channels "
                       "x alpha; W N(0,0.02) in NVFP4",
           "percents": list(sw["percents"]), "k": ks, "bf16_residual": {}, "nvfp4_second_pass": {}}
    for a in sw["alphas"]:
        x = wl.outlier_activations(T, K, a, args.seed, frac=sw["outlier_frac"], device=dev)
        res["bf16_residual"][f"alpha_{a:g}"] = [float(f"{e:.4g}") for e in probe.errors(x, ks, "bf16")]
        res["nvfp4_second_pass"][f"alpha_{a:g}"] = [float(f"{e:.4g}") for e in probe.errors(x, ks, "nvfp4")]
    return res


def run_formats(args, dev):
    """Grouped-GEMM time of the large layer (gate/up + down, same routing and
    shapes) for NVFP4 W4A4 with and without RAC, per-tensor E4M3 W8A8 and BF16
    (the trainer-side GEMM on NVFP4 fake-quantized weights), each timed with
    CUDA events around its two GEMM launches over a few layer steps."""
    import torch
    from quantization_nvfp4_quantize_b200 import workloads as wl, api
    from quantization_nvfp4_quantize_b200 import moe as moe_mod
    cfg = wl.CONFIGS[WORKLOAD]
    fl = wl.flops(cfg)
    x = wl.activations(cfg, args.seed, device=dev)
    logits = wl.router_logits(cfg, args.seed, device=dev)
    w13, w2 = wl.weights(cfg, args.seed, device=dev)
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 5))
    res, launches = {}, 0

    def timed_gemms(layer, names):
        ev = []
        saved = {n: getattr(api, n) for n in names}

        def wrap(fn):
            def w(*a, **k):
                s_ = torch.cuda.Event(enable_timing=True)
                e_ = torch.cuda.Event(enable_timing=True)
                s_.record(stream)
                o = fn(*a, **k)
                e_.record(stream)
                ev.append((s_, e_))
                return o
            return w
        for _ in range(2):
            layer.forward(x, logits)
        torch.cuda.synchronize()
        for n in names:
            setattr(api, n, wrap(saved[n]))
        try:
            for _ in range(steps):
                layer.forward(x, logits)
            torch.cuda.synchronize()
        finally:
            for n in names:
                setattr(api, n, saved[n])
        return sum(a.elapsed_time(b) for a, b in ev) / steps

    for name, make, names, n_launch in (
            ("w4a4_rac", lambda: moe_mod.MoELayerW4A4(w13, w2, cfg.tokens, cfg.topk, cfg.rac_k), ["grouped_gemm"], 16),
            ("w4a4", lambda: moe_mod.MoELayerW4A4(w13, w2, cfg.tokens, cfg.topk, 0), ["grouped_gemm"], 10),
            ("w8a8", lambda: moe_mod.MoELayerW8A8(w13, w2, cfg.tokens, cfg.topk), ["w8a8_grouped_gemm"], 8),
            ("bf16", lambda: moe_mod.MoELayerW4A16(w13, w2, cfg.tokens, cfg.topk), ["bf16_grouped_gemm"], 6)):
        layer = make()
        ms = timed_gemms(layer, names)
        res[name] = {"gemm_ms_per_step": round(ms, 4), "tflops": round(fl["fp4"] / (ms * 1e-3) / 1e12, 1)}
        launches += n_launch * (steps + 2)
        del layer
        torch.cuda.empty_cache()
    res["w4a4_over_w8a8"] = round(res["w8a8"]["gemm_ms_per_step"] / res["w4a4"]["gemm_ms_per_step"], 3)
    res["w4a4_over_bf16"] = round(res["bf16"]["gemm_ms_per_step"] / res["w4a4"]["gemm_ms_per_step"], 3)
    res["rac_overhead"] = round(res["w4a4_rac"]["gemm_ms_per_step"] / res["w4a4"]["gemm_ms_per_step"] - 1, 4)
    res["flops"] = "2*M*N*K of both expert GEMMs (no RAC), the same for every format"
    res["_launches"] = launches
    return res


def time_quantize_kernel(layer, x_in, steps, dev):
    """k_quantize (+ its score reduction) alone on the layer's X (written to
    its k_r routed rows) and h, with the tensor scales the step computed:
    algorithmic bytes 2 B read + 0.5625 B written per element, and the bytes
    the X pass moves with its routed copies."""
    import torch
    from quantization_nvfp4_quantize_b200 import api
    r = layer.routing
    stream = torch.cuda.current_stream(dev)
    E, H, I, T, kr = layer.E, layer.H, layer.I, layer.T, layer.k_r

    def xq():
        api.quantize(x_in, rac_k=0, s_t=layer.xq.s_t, dst_rows=r.dst_row, fanout=kr, m_out=layer.m_pad,
                     want_score=True, out=layer.xq, workspace=layer.ws_x)

    def hq():
        api.quantize(layer.h, rac_k=0, s_t=layer.hq.s_t, m_out=layer.m_pad, m_valid=r.offsets[E:],
                     want_score=True, out=layer.hq, workspace=layer.ws_h)

    for _ in range(2):
        xq(); hq()
    n = max(3, steps)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        ev[i][0].record(stream); xq(); ev[i][1].record(stream)
        ev[i][2].record(stream); hq(); ev[i][3].record(stream)
    torch.cuda.synchronize()
    x_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / n
    h_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / n
    h_rows = int(r.offsets[E].item())
    x_el, h_el = T * H, h_rows * I
    p = peaks()
    gbs = lambda b, ms: b / (ms * 1e-3) / 1e9
    x_alg, h_alg = x_el * QUANT_BYTES_PER_ELEM, h_el * QUANT_BYTES_PER_ELEM
    x_moved = x_el * (2.0 + kr * 0.5625)
    tot = gbs(x_alg + h_alg, x_ms + h_ms)
    return {"gbs": round(tot, 1), "frac": round(tot / p["hbm"], 4), "ms_per_step": round(x_ms + h_ms, 4),
            "x_pass": {"us": round(x_ms * 1e3, 1), "gbs": round(gbs(x_alg, x_ms), 1),
                       "gbs_moved_incl_routed_copies": round(gbs(x_moved, x_ms), 1), "elems": x_el},
            "h_pass": {"us": round(h_ms * 1e3, 1), "gbs": round(gbs(h_alg, h_ms), 1), "elems": h_el},
            "bytes_per_elem": QUANT_BYTES_PER_ELEM,
            "scope": "k_quantize with scores and the score reduction; tensor scale given"}


METRIC_W4A16 = "W4A16 BF16 grouped MoE GEMM TFLOPS and % BF16 peak; weight QDQ GB/s and % HBM"
QDQ_BYTES_PER_ELEM = 4.0    # 2 B bf16 weight read + 2 B bf16 fake-quantized weight written


def run_ours_w4a16(args, workload=None, emit=True):
    """Trainer-side step (asymmetric QAT): NVFP4 fake quantization of every
    expert weight (they change every optimizer step), then the W4A16 layer
    forward: routing, routed-row gather of X, BF16 grouped gate/up GEMM with
    SwiGLU, BF16 grouped down GEMM with router-weighted combine."""
    import torch
    from quantization_nvfp4_quantize_b200 import workloads as wl, api
    from quantization_nvfp4_quantize_b200.moe import MoELayerW4A16

    ws, rank = init_dist("nccl" if torch.cuda.is_available() else "gloo")
    _, _, local = dist_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = wl.CONFIGS[workload or args.workload]
    seed = args.seed + rank
    x = wl.activations(cfg, seed, device=dev)
    logits = wl.router_logits(cfg, seed, device=dev)
    w13, w2 = wl.weights(cfg, seed, device=dev)
    layer = MoELayerW4A16(w13, w2, cfg.tokens, cfg.topk)
    fl = wl.flops(cfg)
    step_flops = fl["fp4"]                        # the same two products, in BF16
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.set_weights(w13, w2)
        return layer.forward(x, logits)

    ev = {"gemm": [], "qdq": []}
    orig_gemm = api.bf16_grouped_gemm
    orig_qdq = layer.set_weights

    def timed(kind, fn):
        def wrap(*a, **k):
            s_ = torch.cuda.Event(enable_timing=True)
            e_ = torch.cuda.Event(enable_timing=True)
            s_.record(stream)
            out = fn(*a, **k)
            e_.record(stream)
            ev[kind].append((s_, e_))
            return out
        return wrap

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    api.bf16_grouped_gemm = timed("gemm", orig_gemm)
    layer.set_weights = timed("qdq", orig_qdq)
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    if clocks.proc is not None:
        time.sleep(0.5)
    torch.cuda.synchronize()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    api.bf16_grouped_gemm = orig_gemm
    layer.set_weights = orig_qdq
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, dev)
    gemm_ms = sum(s_.elapsed_time(e_) for s_, e_ in ev["gemm"])
    qdq_ms = sum(s_.elapsed_time(e_) for s_, e_ in ev["qdq"])
    p = peaks()
    bf16_peak, peak_source = tensor_peak(p, clk, 1.0)
    gemm_tflops = step_flops * args.steps / (gemm_ms * 1e-3) / 1e12
    w_elems = w13.numel() + w2.numel()
    qdq_gbs = w_elems * QDQ_BYTES_PER_ELEM * args.steps / (qdq_ms * 1e-3) / 1e9

    # end to end through the public API: X and logits from pinned host memory, Y back
    xh, lh = x.cpu().pin_memory(), logits.cpu().pin_memory()
    yh = torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory()
    xd, ld_ = torch.empty_like(x), torch.empty_like(logits)
    e_steps = max(1, args.steps // 2)

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        ld_.copy_(lh, non_blocking=True)
        layer.set_weights(w13, w2)
        yh.copy_(layer.forward(xd, ld_), non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    s_ = torch.cuda.Event(enable_timing=True)
    e_ = torch.cuda.Event(enable_timing=True)
    s_.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e_.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(s_.elapsed_time(e_), dev)
    out = {
        "metric": METRIC_W4A16,
        "value": round(step_flops * args.steps * ws / (ms_max * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 (fp32 accum), NVFP4 fake-quantized weights", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: T={cfg.tokens} H={cfg.hidden} I={cfg.inter} E={cfg.experts} "
                               f"top-{cfg.topk}, weight QDQ every step",
                   "l2": "inputs larger than L2 (bf16 weights 1.2 GB)", "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "tensor", "kernel": "k_moe_gemm (BF16 stages)",
                     "achieved": round(gemm_tflops, 1), "peak": round(bf16_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / bf16_peak, 4), "traffic": None,
                     "peak_source": peak_source,
                     "gemm_ms_per_step": round(gemm_ms / args.steps, 4), "launches_per_step": 2},
        "qdq": {"gbs": round(qdq_gbs, 1), "peak_gbs": p["hbm"], "frac": round(qdq_gbs / p["hbm"], 4),
                "ms_per_step": round(qdq_ms / args.steps, 4), "bytes_per_elem": QDQ_BYTES_PER_ELEM,
                "elems_per_step": w_elems},
        "e2e": {"value": round(step_flops * e_steps * ws / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": xh.numel() * xh.element_size() + lh.numel() * lh.element_size(),
                "d2h_bytes_per_step": yh.numel() * yh.element_size()},
        # per step: 2 x (amax + quantize) for the weights, route (3), gather, 2 GEMMs
        "gpu_launches": 10 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and emit:
        print(json.dumps(out), flush=True)
    return out


def run_e2e(layer, x, logits, args, dev):
    """Same metric through the public API with host buffers: every step copies
    its X and router logits from pinned host memory to the device and reads
    its Y back into pinned host memory.  Steps are pipelined the way a serving
    loop would run them: inputs of step i+1 travel host->device on one copy
    stream and Y of step i-1 device->host on another (PCIe is full duplex)
    while step i computes; Y is staged device-to-device so the next step can
    reuse the layer's output buffer.  Two buffers per direction; events order
    every reuse."""
    import torch
    steps = max(2, args.steps // 2)
    xh = [x.cpu().pin_memory() for _ in range(2)]
    lh = [logits.cpu().pin_memory() for _ in range(2)]
    yh = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    ld = [torch.empty_like(logits) for _ in range(2)]
    ys = [torch.empty_like(layer.y) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()

    def run(n, start):
        in_ready = [ev(), ev()]      # inputs of buffer b landed
        in_free = [None, None]       # the step that read buffer b has finished
        out_ready = [ev(), ev()]     # ys[b] holds a finished Y
        out_free = [None, None]      # the read-back of ys[b] has finished
        s_in.wait_event(start)       # no copy starts before the timed region
        s_out.wait_event(start)
        with torch.cuda.stream(s_in):
            xd[0].copy_(xh[0], non_blocking=True)
            ld[0].copy_(lh[0], non_blocking=True)
            in_ready[0].record(s_in)
        for i in range(n):
            b = i & 1
            if i + 1 < n:            # prefetch the next step's inputs
                nb = (i + 1) & 1
                with torch.cuda.stream(s_in):
                    if in_free[nb] is not None:
                        s_in.wait_event(in_free[nb])
                    xd[nb].copy_(xh[nb], non_blocking=True)
                    ld[nb].copy_(lh[nb], non_blocking=True)
                    in_ready[nb].record(s_in)
            comp.wait_event(in_ready[b])
            y = layer.forward(xd[b], ld[b])
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            ys[b].copy_(y, non_blocking=True)
            in_free[b] = ev()
            in_free[b].record(comp)
            out_ready[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[b])
                yh[b].copy_(ys[b], non_blocking=True)
                out_free[b] = ev()
                out_free[b].record(s_out)
        for f in out_free:           # the end event follows every read-back
            if f is not None:
                comp.wait_event(f)

    w = torch.cuda.Event()
    w.record(comp)
    run(2, w)                        # warm-up
    torch.cuda.synchronize()
    barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(comp)
    run(steps, s)
    e.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), dev)
    from quantization_nvfp4_quantize_b200 import workloads as wl
    cfg = wl.CONFIGS[args.workload]
    fl = wl.flops(cfg)
    ws = dist_env()[0]
    return {"value": round((fl["fp4"] + fl["rac"]) * steps * ws / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": xh[0].numel() * xh[0].element_size() + lh[0].numel() * lh[0].element_size(),
            "d2h_bytes_per_step": yh[0].numel() * yh[0].element_size(),
            "pipelined": "H2D of step i+1 and D2H of step i-1 overlap step i (two copy streams)"}


# --------------------------------------------------------------- CPU oracle

def cpu_baseline(cfg, seed=0, n_experts=8):
    """The oracle, as it stands, on a bounded sample of the workload: every
    routed row of the first `n_experts` experts (their tokens' X rows are
    quantized, scored and selected, then both W4A4+RAC products, SwiGLU and
    the h quantization run on those rows).  Weight quantization is done
    before timing, as on the GPU.  Returns TFLOP/s of the sample."""
    import numpy as np
    import torch
    import oracle
    from quantization_nvfp4_quantize_b200 import workloads as wl

    x = wl.activations(cfg, seed)
    logits = wl.router_logits(cfg, seed)
    xn = x.view(torch.int16).numpy().view(np.uint16)
    idx, gate = oracle.route(logits.numpy(), cfg.topk)
    g = torch.Generator().manual_seed(1234)
    E_s = n_experts
    w13 = [(torch.randn(2 * cfg.inter, cfg.hidden, generator=g) * 0.02).to(torch.bfloat16) for _ in range(E_s)]
    w2 = [(torch.randn(cfg.hidden, cfg.inter, generator=g) * 0.02).to(torch.bfloat16) for _ in range(E_s)]
    w13q = [oracle.quantize(w.view(torch.int16).numpy().view(np.uint16)).xhat for w in w13]
    w2q = [oracle.quantize(w.view(torch.int16).numpy().view(np.uint16)).xhat for w in w2]
    rows = [(t, j) for e in range(E_s) for t, j in zip(*np.nonzero(idx == e))]
    toks = np.array(sorted({t for t, _ in rows}))
    k = cfg.rac_k
    t0 = time.perf_counter()
    qx = oracle.quantize(xn[toks])
    S_x = oracle.select_topk(oracle.channel_score(qx.resid), k)
    rho_x = oracle.rac_residual(qx.resid, qx.s_t, S_x)
    pos = {t: i for i, t in enumerate(toks)}
    h = []
    for e in range(E_s):
        tt = np.array([pos[t] for t, j in rows if idx[t, j] == e], dtype=np.int64)
        y = oracle.w4a4_rac_matmul(qx.xhat[tt], qx.s_t, rho_x[tt], S_x, w13q[e])
        h.append(oracle.f32_to_bf16(oracle.swiglu(y, cfg.inter).astype(np.float32)))
    hb = np.concatenate(h)
    qh = oracle.quantize(hb)
    S_h = oracle.select_topk(oracle.channel_score(qh.resid), k)
    rho_h = oracle.rac_residual(qh.resid, qh.s_t, S_h)
    start = 0
    for e in range(E_s):
        n = h[e].shape[0]
        oracle.w4a4_rac_matmul(qh.xhat[start:start + n], qh.s_t, rho_h[start:start + n], S_h, w2q[e])
        start += n
    dt = time.perf_counter() - t0
    M = len(rows)
    flops = 2.0 * M * (2 * cfg.inter * cfg.hidden + cfg.hidden * cfg.inter) + \
        2.0 * M * (2 * cfg.inter + cfg.hidden) * k
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"all {M} routed rows of experts 0..{E_s - 1} ({len(toks)} tokens) of {cfg.name}; "
                      f"weights of those experts quantized before timing"}


def run_reference(args):
    """--impl reference: the oracle as it stands on the host cores, each step a
    bounded sample (the routed rows of 2 experts) of the same workload."""
    ws, rank = init_dist("gloo")
    if rank != 0:
        return None
    from quantization_nvfp4_quantize_b200 import workloads as wl
    cfg = wl.CONFIGS[args.workload]
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(cfg, seed=args.seed, n_experts=2)
        if i >= args.warmup:
            vals.append(r)
    tot_s = sum(v["seconds"] for v in vals)
    value = statistics.mean(v["value"] for v in vals)
    out = {"impl": "reference", "metric": METRIC,
           "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / max(1, len(vals)), 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
           "data": "synthetic",
           "config": {"workload": f"{cfg.name}: T={cfg.tokens} H={cfg.hidden} I={cfg.inter} E={cfg.experts} "
                                  f"top-{cfg.topk} RAC k={cfg.rac_k}"},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": vals[0]["cores"],
                            "kind": "oracle", "sample": vals[0]["sample"]},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return out


def main():
    args = parse()
    try:
        if args.impl == "reference":
            run_reference(args)
        else:
            run_ours(args)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
