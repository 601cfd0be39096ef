"""Benchmark of the routed low-bit MoE layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME|all] [--impl ours|reference]

One step = one full layer forward (routing, permutation, grouped SwiGLU
expert FFN over packed weights, combine) over one batch of synthetic input
resident in HBM.  The default workload is the decode layer (T=1 token,
d_model=4096, 256 routed experts, top-8, d_ff=2048, affine 4-bit group-64
experts plus an 8-bit shared expert).  Inputs larger than L2 between
steps: where a step reads under 8x L2 of weights (decode, mixed), 4 copies
of the layer (equal values, distinct buffers, GBs in all) are cycled, so a
step reads weights last touched 3 steps earlier, behind hundreds of MB of
other copies' traffic, as the layers of a model do, and the same kernel ran
just before it; the same steps are also timed on ONE copy with L2 flushed
before each step by READING a 512 MiB buffer (outside the events; a read
leaves no dirty lines) and reported as "l2_flushed" in the same line.
Workloads that read many times L2 per step (hash, prefill) take one copy
flushed before each step (--layers overrides).  The reported step time is
the median over the timed steps (min, mean and p90 beside it).  --config all
prints one line per layer configuration (tiny, hash, mixed, prefill, then
the decode line last).

With N > 1 (launched by torchrun) every rank runs an independent replica of
the layer on its own GPU ("replicas only": the layer has no exchange step on
one node in this build); the value is the sum of all ranks' tokens over the
slowest rank's device time.

--impl reference times the fp64 CPU oracle (test infrastructure, run as it
stands) on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("MoE-layer tokens/s at 1 B200; achieved HBM GB/s (decode) / tensor TFLOPS (prefill) vs peak")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="decode", help="workload name, or 'all' (one line each, decode last)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffn-path", default="auto", choices=["auto", "gemv", "tc"],
                    help="expert-FFN implementation: library default, weight-streaming GEMV, tensor-core GEMM")
    ap.add_argument("--cpu-budget", type=float, default=25.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--layers", type=int, default=0,
                    help="copies of the layer cycled between timed steps (1: one copy, L2 flushed before each step; "
                         "0: 4 copies when a step reads under 8x L2 of weights, else 1)")
    ap.add_argument("--override", action="append", default=[],
                    help="key=value change to the workload (profiling small cases), e.g. E=16")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), \
            d.get("bf16_tflops_sustained", d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


NOMINAL_HBM_GBS = 8000.0       # B200 HBM3e, the figure the layer's bandwidth target is set against
NOMINAL_F16_TFLOPS = 2250.0    # B200 dense fp16/bf16 tensor rate


def roofline_entry(dom, dom_ms, work, kflops, tensor_path, peak, traffic):
    """The binding roofline of the dominant kernel `dom` (median launch time
    `dom_ms`): tensor FLOPs or HBM bytes, whichever it is closer to (small
    batches on the tensor-core path stream weights far below the machine
    balance point).  `peak` = (hbm GB/s, bf16 burst TFLOP/s, bf16 sustained
    TFLOP/s, "measured"|"fallback").  The tensor denominator is the burst
    rate: the kernel runs for about a millisecond inside a few-millisecond
    step, not in a seconds-long loop; the sustained fraction is reported
    beside it."""
    hbm, bf16, bf16_sus, peak_kind = peak
    sec = dom_ms * 1e-3
    tflops_dom = kflops.get(dom, 0.0) / sec / 1e12 if tensor_path else 0.0
    gbs_dom = work.get(dom, 0) / sec / 1e9
    if tensor_path and dom in kflops and tflops_dom / bf16 >= gbs_dom / hbm:
        # fp16 x fp16 -> fp32 tcgen05 MMAs: the nominal fp16 and bf16 dense rates are equal,
        # so the measured bf16 cuBLAS rate is the denominator
        return {"bound": "tensor", "kernel": dom, "achieved": tflops_dom, "peak": bf16, "unit": "TFLOP/s",
                "frac": tflops_dom / bf16, "traffic": traffic,
                "peak_kind": f"{peak_kind} bf16_tflops burst (cuBLAS; fp16 nominal = bf16 nominal)",
                "frac_of_sustained_peak": tflops_dom / bf16_sus, "sustained_peak": bf16_sus,
                "frac_of_nominal": tflops_dom / NOMINAL_F16_TFLOPS,
                "nominal_peak": NOMINAL_F16_TFLOPS, "algorithmic_flops_per_launch": kflops[dom],
                "algorithmic_bytes_per_launch": work.get(dom, 0), "hbm_frac": gbs_dom / hbm}
    out = {"bound": "hbm", "kernel": dom, "achieved": gbs_dom, "peak": hbm, "unit": "GB/s",
           "frac": gbs_dom / hbm, "traffic": traffic, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
           "frac_of_nominal": gbs_dom / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS,
           "algorithmic_bytes_per_launch": work.get(dom, 0)}
    if tensor_path and dom in kflops:
        out["tensor_frac"] = tflops_dom / bf16
    return out


def src_hash(files=None):
    """Hash of the kernel sources (the listed csrc files, else all of them):
    a stored ncu traffic figure only applies while its kernel is unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_moe_route_b200", "csrc")
    paths = [os.path.join(csrc, f) for f in files] if files else glob.glob(os.path.join(csrc, "*"))
    for p in sorted(paths):
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def workload_desc(cfg):
    f13, f2 = cfg["w13"], cfg["w2"]
    fmt = lambda t: f"{t[0]}{t[1]}g{t[2]}" if t[0] == "affine" else "mxfp4g32"  # noqa: E731
    d = {"workload": cfg["name"], "T": cfg["T"], "d_model": cfg["d"], "n_experts": cfg["E"], "top_k": cfg["k"],
         "d_ff": cfg["f"], "routing": cfg["routing"], "w1_w3": fmt(f13), "w2": fmt(f2)}
    if cfg.get("shared"):
        d["shared_expert"] = f"{fmt(cfg['shared'])} d_ff={cfg['f_shared']}"
    return d


# ---------------------------------------------------------------- algorithmic bytes / flops
def kernel_work(inp, ids, tensor_path=False):
    """Algorithmic bytes of each kernel label the library can report for one
    forward (and the flops).  The expert-FFN entries depend on the path: the
    weight-streaming GEMV runs the shared expert inside the routed launches
    and keeps h in fp32; the tensor-core path runs it as its own launches
    (the *_shared labels) and keeps token rows and h in fp16.

    Returns (work, flops, distinct routed experts, weight bytes, kflops)."""
    import numpy as np
    c = inp.cfg
    T, d, E, k, f = c["T"], c["d"], c["E"], c["k"], c["f"]
    ids = np.asarray(ids)
    active = np.unique(ids)
    n_act = len(active)
    b13 = inp.w1.packed_bytes_per_expert() + inp.w3.packed_bytes_per_expert()
    b2 = inp.w2.packed_bytes_per_expert()
    sh13 = sh2 = 0
    Tk = T * k
    Ts = T if inp.shared is not None else 0
    if inp.shared is not None:
        sh13 = inp.shared[0].packed_bytes_per_expert() + inp.shared[1].packed_bytes_per_expert()
        sh2 = inp.shared[2].packed_bytes_per_expert()
    fs = c.get("f_shared", 0) if inp.shared is not None else 0
    work = {}
    perm = Tk * 4 * 3 + (E + 1) * 4               # ids in, sorted rows + inverse out, offsets
    if c["routing"] == "hash":
        rows = len(np.unique(ids))
        work["route_hash"] = T * d * 2 + T * 4 + Tk * 4 + rows * d * 4 + Tk * 8
        work["route_hash_permute"] = work["route_hash"] + perm
    else:
        work["router_logits"] = E * d * 4 + T * d * 2 + T * E * 4
        work["topk"] = T * E * 4 + E * 4 + Tk * 8
        work["route_topk_permute"] = E * d * 4 + T * d * 2 + E * 4 + Tk * 8 + perm
    n_chunks = (Tk + 1023) // 1024                 # multi-CTA permutation: per-chunk expert counts
    work["permute_count"] = Tk * 4 + n_chunks * E * 4
    work["permute_scan"] = 2 * n_chunks * E * 4 + (E + 1) * 4
    work["permute"] = perm
    if tensor_path:
        work["gather_f16"] = T * d * 2 + (Tk + Ts) * d * 2 + Tk * 4
        work["tile_plan"] = (E + 1) * 4 + ((Tk + 127) // 128 + E) * 16
        work["ffn_w13_swiglu"] = n_act * b13 + Tk * d * 2 + Tk * f * 2
        work["ffn_w2"] = n_act * b2 + Tk * f * 2 + Tk * d * 4
        work["ffn_w13_swiglu_shared"] = sh13 + Ts * d * 2 + Ts * fs * 2
        work["ffn_w2_shared"] = sh2 + Ts * fs * 2 + Ts * d * 4
    else:
        P = Tk + Ts
        work["ffn_w13_swiglu"] = n_act * b13 + sh13 + T * d * 2 + P * max(f, fs) * 4
        work["ffn_w2"] = n_act * b2 + sh2 + P * max(f, fs) * 4 + P * d * 4
    work["combine"] = (Tk + Ts) * d * 4 + T * d * 2 + Tk * 8
    # the fused small-batch launch: every weight byte once, the router's
    # rows (all of them, or the table's experts in hash mode), x in, out back
    rw_bytes = inp.router_w.element_size() if getattr(inp, "router_w", None) is not None else 4
    router = (len(np.unique(ids)) if c["routing"] == "hash" else E) * d * rw_bytes
    work["decode_fused"] = n_act * (b13 + b2) + sh13 + sh2 + router + 2 * T * d * 2
    flops = 2.0 * T * k * 3 * d * f + (2.0 * T * 3 * d * fs if fs else 0.0)
    kflops = {"ffn_w13_swiglu": 2.0 * T * k * 2 * d * f, "ffn_w2": 2.0 * T * k * d * f,
              "ffn_w13_swiglu_shared": 2.0 * T * 2 * d * fs, "ffn_w2_shared": 2.0 * T * d * fs}
    return work, flops, n_act, (n_act * (b13 + b2) + sh13 + sh2), kflops


def layer_copies(requested, step_weight_bytes, l2_bytes):
    """Copies of the layer cycled between timed steps: the requested number,
    or (0) four when a step reads under 8x L2 of weights, else one (flushed)."""
    if requested > 0:
        return requested
    return 4 if step_weight_bytes < 8 * l2_bytes else 1


def layer_tensors(inp):
    """Every device tensor of one layer's inputs (for its size)."""
    ts = [inp.x, inp.router_w, inp.router_b, inp.token_ids, inp.tid2eid]
    for m in [inp.w1, inp.w3, inp.w2] + list(inp.shared or ()):
        ts += [m.q, m.scales, m.biases]
    return [t for t in ts if t is not None]


def layer_bytes(work, labels):
    """Algorithmic bytes of one forward: the kernels that actually ran."""
    return sum(work.get(lab, 0) for lab in labels)


def step_stats(ms):
    """Median (the reported step), min, mean and p90 of the timed steps."""
    srt = sorted(ms)
    return {"median": statistics.median(srt), "min": srt[0], "mean": statistics.mean(srt),
            "p90": srt[min(len(srt) - 1, int(0.9 * len(srt)))]}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-i", self.gpu_id, "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle timing
def oracle_sample_time(inp, budget_s: float, max_pairs=None, start_pair: int = 0):
    """Time the oracle on a bounded sample; returns (seconds per token, sample description, pairs, blas threads).

    Routing runs for every token; the expert FFN then runs for consecutive
    (token, slot) pairs starting at ``start_pair`` until the time budget (or
    max_pairs) is spent.  The per-token time is extrapolated from the pairs
    done: k routed slots plus the shared expert make one token.
    """
    import oracle
    c = inp.cfg
    T, d, k = c["T"], c["d"], c["k"]
    x = inp.x.float().cpu().numpy()
    t0 = time.perf_counter()
    if c["routing"] == "hash":
        ids, w = oracle.route_hash(x, inp.router_w.float().cpu().numpy(), inp.token_ids.cpu().numpy(),
                                   inp.tid2eid.cpu().numpy())
    else:
        ids, w, _, _ = oracle.route_learned(x, inp.router_w.float().cpu().numpy(), inp.router_b.cpu().numpy(), k)
    oracle.permute(ids, c["E"])
    t_route = time.perf_counter() - t0
    ppt = k + (1 if inp.shared is not None else 0)
    mats = {"w1": inp.w1, "w3": inp.w3, "w2": inp.w2}
    shared = dict(zip(("w1", "w3", "w2"), inp.shared)) if inp.shared is not None else None
    done, t_ffn, pair = 0, 0.0, start_pair % (T * ppt)
    while True:
        tok, j = divmod(pair, ppt)
        t1 = time.perf_counter()
        src, e = (mats, int(ids[tok, j])) if j < k else (shared, 0)
        n_in = {"w1": d, "w3": d, "w2": src["w1"].n_out}
        W = {n: oracle.dequant(m.fmt, m.bits, m.group, n_in[n], *m.expert_numpy(e)) for n, m in src.items()}
        oracle.swiglu_ffn(W["w1"], W["w3"], W["w2"], x[tok:tok + 1])
        t_ffn += time.perf_counter() - t1
        done += 1
        pair = (pair + 1) % (T * ppt)
        if t_ffn >= budget_s or (max_pairs and done >= max_pairs):
            break
    per_token = t_ffn / done * ppt + t_route / T
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        blas = 1
    desc = (f"routing for all {T} tokens ({t_route:.2f}s) + {done} (token, expert) FFN pairs "
            f"({t_ffn:.1f}s); per-token time = mean pair time x {ppt} + routing time / T")
    return per_token, desc, done, blas


def overrides(args):
    out = {}
    for kv in args.override:
        key, val = kv.split("=", 1)
        out[key] = int(val) if val.lstrip("-").isdigit() else val
    return out


def max_over_ranks(v, device):
    """The largest of every rank's v (the slowest rank's time); v itself on one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank, world, ms):
    """Tokens per second of the whole job: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms * 1e-3)


def reference_arm(args):
    """The oracle, as it stands, on this host's cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np  # noqa: F401
    import torch
    from synthetic import make_inputs
    dev = torch.device("cuda:0") if torch.cuda.is_available() else torch.device("cpu")
    names = CONFIG_ORDER if args.config == "all" else [args.config]
    for name in names:
        if name.startswith("mhc") or name.startswith("mxfp8"):
            reference_kernel_line(args, name, dev, 150.0 / len(names))
            continue
        inp = make_inputs(name, dev, **overrides(args))
        reference_line(args, inp, 150.0 / len(names))


def reference_kernel_line(args, name, dev, budget_total):
    """Reference-arm line of a single-kernel workload (mHC mixing, mxfp8
    rows): the oracle on a bounded sample, in the metric of our line."""
    if name.startswith("mhc"):
        from synthetic import HC_CONFIGS, make_hc_inputs
        cfg = dict(HC_CONFIGS[name], name=name)
        cfg.update(overrides(args))
        inp = make_hc_inputs(cfg, dev)
        metric = "mHC Sinkhorn-mixed tokens/s at 1 B200; achieved HBM GB/s vs peak"
        config = {"workload": name, "T": cfg["T"], "hc_mult": cfg["n"], "d": cfg["d"], "iters": cfg["iters"],
                  "eps": cfg["eps"]}
        rate = lambda b: hc_oracle_rate(inp, b)  # noqa: E731
    else:
        from synthetic import FP8_CONFIGS, make_fp8_inputs
        cfg = dict(FP8_CONFIGS[name], name=name)
        cfg.update(overrides(args))
        inp = make_fp8_inputs(cfg, dev)
        metric = "mxfp8 weight elements/s dequantised to bf16 at 1 B200; achieved HBM GB/s vs peak"
        config = {"workload": name, "rows": cfg["rows"], "n_in": cfg["n_in"]}
        rate = lambda b: fp8_oracle_rate(inp, b)  # noqa: E731
    step_budget = max(0.5, budget_total / max(1, args.steps + args.warmup))
    vals, t0 = [], time.perf_counter()
    for s in range(args.warmup + args.steps):
        cb = rate(step_budget)
        if s >= args.warmup:
            vals.append(cb["value"])
        if time.perf_counter() - t0 > budget_total:
            break
    value = statistics.mean(vals) if vals else cb["value"]
    unit = cb["unit"]
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": len(vals), "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": dict(cb, value=value,
                                 sample=f"per step: {cb['sample']}; steps capped at {budget_total:.0f}s of CPU work"),
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def reference_line(args, inp, budget_total):
    """One reference-arm line: the oracle on a bounded sample of inp's workload."""
    c = inp.cfg
    step_budget = max(0.5, budget_total / max(1, args.steps + args.warmup))
    times, pairs = [], 0
    desc = ""
    t_start = time.perf_counter()
    n_steps = 0
    for s in range(args.warmup + args.steps):
        per_tok, desc, done, blas = oracle_sample_time(inp, step_budget, max_pairs=1, start_pair=s)
        if s >= args.warmup:
            times.append(per_tok)
            pairs += done
            n_steps += 1
        if time.perf_counter() - t_start > budget_total:
            break
    per_tok = statistics.mean(times) if times else float("nan")
    value = 1.0 / per_tok
    cores = blas
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": n_steps, "warmup": args.warmup, "ms_per_step": per_tok * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(c),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {desc}; steps capped at {budget_total:.0f}s of CPU work"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
CONFIG_ORDER = ["tiny", "hash", "mixed", "prefill", "decode"]   # --config all: decode (the headline) last


def run_config(name, args, dev, world, rank):
    """Time one layer configuration; returns its JSON line (dict)."""
    import numpy as np  # noqa: F401
    import torch

    import bit_quantized_moe_route_b200 as moe
    from synthetic import make_inputs

    inp = make_inputs(name, dev, **overrides(args))
    c = inp.cfg
    T, d, k = c["T"], c["d"], c["k"]
    dims = moe.make_dims(T, d, c["f"], c["E"], k, c["routing"] == "hash",
                         c.get("vocab", 0) if c["routing"] == "hash" else 0,
                         c.get("f_shared", 0) if inp.shared is not None else 0, router_dtype=inp.router_w.dtype)
    ws = moe.alloc_workspace(dims, dev)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    ids = torch.empty(T, k, dtype=torch.int32, device=dev)
    wts = torch.empty(T, k, dtype=torch.float32, device=dev)
    # copies of the layer in distinct buffers, cycled between timed steps,
    # where a step reads few enough weight bytes that L2 could otherwise carry
    # some from one step to the next; a step reading many times L2 takes one
    # copy with L2 flushed before each step
    moe.forward(dims, inp.x, inp.token_ids, inp.router_w, inp.router_b, inp.tid2eid, inp.w1, inp.w3, inp.w2,
                inp.shared, out, ws, topk_ids_out=ids, topk_w_out=wts)
    torch.cuda.synchronize()
    step_weight_bytes = kernel_work(inp, ids.cpu().numpy(), False)[3]
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    n_layers = layer_copies(args.layers, step_weight_bytes, l2_bytes)
    layers = [inp] + [inp.clone() for _ in range(n_layers - 1)]
    # L2 flush by a read of 512 MiB (> 4x L2) into one small result
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_sum = torch.empty((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)

    def fwd(s=0):
        ly = layers[s % n_layers]
        moe.forward(dims, ly.x, ly.token_ids, ly.router_w, ly.router_b, ly.tid2eid, ly.w1, ly.w3, ly.w2,
                    ly.shared, out, ws, topk_ids_out=ids, topk_w_out=wts)

    def between_steps():
        if n_layers == 1:
            flush_l2()

    for i in range(max(3, args.warmup, n_layers)):
        between_steps()
        fwd(i)
    torch.cuda.synchronize()

    # ---- timed region: K forwards over the cycled copies (or one copy with
    # L2 flushed between them, outside the events)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if getattr(props, "uuid", None) else str(dev.index))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    for s in range(args.steps):
        between_steps()
        step_ev[s][0].record(stream)
        fwd(s)
        step_ev[s][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    st = step_stats([a.elapsed_time(b) for a, b in step_ev])
    ms_per_step = max_over_ranks(st["median"], dev)
    # ---- per-kernel durations: a second timed pass with CUDA events recorded
    # by the library between its kernels on the same stream (the events add
    # small gaps between kernels, so the step time above is taken without them)
    k_steps = min(args.steps, 200)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(16)] for _ in range(k_steps)]
    keep = []
    torch.cuda.synchronize()
    for s in range(k_steps):
        between_steps()
        keep.append(moe.set_timing_events(evs[s]))
        fwd(s)
    torch.cuda.synchronize()
    labels = moe.timing_labels()
    per_kernel = {}
    for s in range(k_steps):
        for i, lab in enumerate(labels):
            per_kernel.setdefault(lab, []).append(evs[s][i].elapsed_time(evs[s][i + 1]))
    kern_ms = {lab: statistics.median(v) for lab, v in per_kernel.items()}

    # the same steps on one copy with L2 (code included) flushed before each
    # (after the per-kernel pass, so that pass follows the same load as the
    # timed steps)
    flushed = None
    if n_layers > 1:
        for s in range(args.steps):
            flush_l2()
            step_ev[s][0].record(stream)
            fwd(0)
            step_ev[s][1].record(stream)
        torch.cuda.synchronize()
        stf = step_stats([a.elapsed_time(b) for a, b in step_ev])
        ms_flushed = max_over_ranks(stf["median"], dev)
        flushed = {"value": whole_job_rate(T, world, ms_flushed), "ms_per_step": ms_flushed, "step_ms": stf}

    # ---- end-to-end through the C ABI with host buffers (pinned), copies inside
    x_h = inp.x.cpu().pin_memory()
    tok_h = inp.token_ids.cpu().pin_memory() if inp.token_ids is not None else None
    out_h = torch.empty(T, d, dtype=torch.bfloat16).pin_memory()
    layer_args = [(ly.router_w, ly.router_b, ly.tid2eid, ly.w1, ly.w3, ly.w2, ly.shared) for ly in layers]
    for i in range(max(3, n_layers)):
        moe.forward_host(dims, x_h, tok_h, *layer_args[i % n_layers], out_h, ws)
    torch.cuda.synchronize()
    e2e_steps = max(10, min(args.steps, 200))
    e2e = []
    for s in range(e2e_steps):
        # L2 flushed before every step here: the flush keeps the GPU busy
        # while the host issues the call, so the events time the copies and
        # the kernels, as in the one-copy figure (a synchronous call on an idle
        # GPU would add the host's issue time, which varies box to box)
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        moe.forward_host(dims, x_h, tok_h, *layer_args[s % n_layers], out_h, ws)
        b.record(stream)
        b.synchronize()
        e2e.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(statistics.median(e2e), dev)
    h2d = T * d * 2 + (T * 4 if tok_h is not None else 0)
    d2h = T * d * 2
    err = moe.read_device_error(ws)

    tensor_path = "tile_plan" in labels
    work, flops, n_act, weight_bytes, kflops = kernel_work(inp, ids.cpu().numpy(), tensor_path)
    hbm, bf16, bf16_sus, peak_kind = peaks()
    dom = max(kern_ms, key=kern_ms.get)
    dom_ms = kern_ms[dom]
    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof):
        with open(prof) as fh:
            tj = json.load(fh)
        ent = tj.get(c["name"], {}).get(dom)
        if ent and ent.get("src_hash") == src_hash(ent.get("files")):
            traffic = ent.get("dram_bytes_per_launch")
    roofline = roofline_entry(dom, dom_ms, work, kflops, tensor_path, (hbm, bf16, bf16_sus, peak_kind), traffic)
    lbytes = layer_bytes(work, labels)
    value = whole_job_rate(T, world, ms_per_step)
    if n_layers > 1:
        copy_gb = sum(t.numel() * t.element_size() for t in layer_tensors(inp)) / 1e9
        l2_desc = (f"inputs larger than L2: {n_layers} copies of the layer ({copy_gb:.2f} GB each, distinct buffers) "
                   f"cycled, no flush; a step's weights were last read {n_layers - 1} steps earlier, behind "
                   f"{(n_layers - 1) * lbytes / 1e6:.0f} MB of other copies' traffic, and the same kernels ran "
                   "just before, as in a multi-layer model (one copy with L2 flushed before each step: l2_flushed)")
    else:
        l2_desc = "flushed by reading a 512 MiB buffer between timed steps (outside the events)"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16" if tensor_path else "f32", "data": "synthetic",
        "config": dict(workload_desc(c), ffn_path=args.ffn_path, l2=l2_desc,
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "step_ms": st,
        "l2_flushed": flushed,
        "roofline": roofline,
        "layer": {"bytes_per_step": lbytes, "weight_bytes": weight_bytes, "distinct_routed_experts": n_act,
                  "GBps_whole_step": lbytes / (ms_per_step * 1e-3) / 1e9,
                  "frac_whole_step": lbytes / (ms_per_step * 1e-3) / 1e9 / hbm,
                  "flops_per_step": flops, "TFLOPs_whole_step": flops / (ms_per_step * 1e-3) / 1e12,
                  "kernel_ms_median": kern_ms, "kernels": labels},
        "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "l2": "flushed before each step (kernel code evicted too)"},
        "gpu_launches": len(labels) * args.steps,
        "kernel_timing_steps": k_steps,
        "clocks": clocks,
        "device_error": err,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        budget = args.cpu_budget if name == "decode" or args.config != "all" else min(args.cpu_budget, 10.0)
        per_tok, desc, done, blas = oracle_sample_time(inp, budget)
        line["cpu_baseline"] = {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": blas, "kind": "oracle",
                                "sample": desc, "cores_available": len(os.sched_getaffinity(0))}
    del inp, layers, flush, ws
    torch.cuda.empty_cache()
    return line


def run_hc_config(name, args, dev, world, rank):
    """Time the fused mHC Sinkhorn mixing kernel on its own (one launch per
    step); HBM-bound: the n residual copies are read once and written once."""
    import torch

    import bit_quantized_moe_route_b200 as moe
    from synthetic import HC_CONFIGS, make_hc_inputs

    cfg = dict(HC_CONFIGS[name], name=name)
    cfg.update(overrides(args))
    inp = make_hc_inputs(cfg, dev)
    T, n, d = cfg["T"], cfg["n"], cfg["d"]
    out = torch.empty_like(inp.h)
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_sum = torch.empty((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moe.hc_sinkhorn_mix(inp.logits, inp.h, out, cfg["iters"], cfg["eps"])

    for _ in range(max(3, args.warmup)):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if getattr(props, "uuid", None) else str(dev.index))
    sampler.start()
    time.sleep(0.2)
    for s in range(args.steps):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        evs[s][0].record(stream)
        step()
        evs[s][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    st = step_stats([a.elapsed_time(b) for a, b in evs])
    ms = max_over_ranks(st["median"], dev)
    # e2e: host logits and copies in, mixed copies back
    L_h = inp.logits.cpu().pin_memory()
    h_h = inp.h.cpu().pin_memory()
    o_h = torch.empty_like(h_h).pin_memory()
    L_d, h_d = torch.empty_like(inp.logits), torch.empty_like(inp.h)
    e2e = []
    for s in range(max(10, min(args.steps, 50))):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        L_d.copy_(L_h, non_blocking=True)
        h_d.copy_(h_h, non_blocking=True)
        moe.hc_sinkhorn_mix(L_d, h_d, out, cfg["iters"], cfg["eps"])
        o_h.copy_(out, non_blocking=True)
        b.record(stream)
        b.synchronize()
        e2e.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(statistics.median(e2e), dev)
    hbm, bf16, bf16_sus, peak_kind = peaks()
    nbytes = T * n * d * 2 * 2 + T * n * n * 4
    roof = {"bound": "hbm", "kernel": "hc_sinkhorn_mix", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm,
            "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "traffic": None,
            "peak_kind": f"{peak_kind} hbm_gbs (copy)", "algorithmic_bytes_per_launch": nbytes,
            "frac_of_nominal": nbytes / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS}
    line = {"metric": "mHC Sinkhorn-mixed tokens/s at 1 B200; achieved HBM GB/s vs peak",
            "value": whole_job_rate(T, world, ms), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": name, "T": T, "hc_mult": n, "d": d, "iters": cfg["iters"], "eps": cfg["eps"],
                       "l2": "flushed by reading a 512 MiB buffer between timed steps (outside the events)"},
            "step_ms": st, "roofline": roof,
            "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * n * d * 2 + T * n * n * 4, "d2h_bytes_per_step": T * n * d * 2,
                    "ms_per_step": e2e_ms},
            "gpu_launches": args.steps, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = hc_oracle_rate(inp, min(args.cpu_budget, 10.0))
    del inp, flush
    torch.cuda.empty_cache()
    return line


def run_fp8_config(name, args, dev, world, rank):
    """Time the mxfp8 -> bf16 row dequantisation on its own (one launch per
    step); HBM-bound: 1 + 1/32 bytes read and 2 written per element."""
    import torch

    import bit_quantized_moe_route_b200 as moe
    from synthetic import FP8_CONFIGS, make_fp8_inputs

    cfg = dict(FP8_CONFIGS[name], name=name)
    cfg.update(overrides(args))
    inp = make_fp8_inputs(cfg, dev)
    rows, n_in = cfg["rows"], cfg["n_in"]
    out = torch.empty(rows, n_in, dtype=torch.bfloat16, device=dev)
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.int32, device=dev)
    flush_sum = torch.empty((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moe.dequant_mxfp8(inp.codes, inp.scales, out)

    for _ in range(max(3, args.warmup)):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid) if getattr(props, "uuid", None) else str(dev.index))
    sampler.start()
    time.sleep(0.2)
    for s in range(args.steps):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        evs[s][0].record(stream)
        step()
        evs[s][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    st = step_stats([a.elapsed_time(b) for a, b in evs])
    ms = max_over_ranks(st["median"], dev)
    # e2e: host codes and scales in, bf16 rows back
    c_h, s_h = inp.codes.cpu().pin_memory(), inp.scales.cpu().pin_memory()
    o_h = torch.empty(rows, n_in, dtype=torch.bfloat16).pin_memory()
    c_d, s_d = torch.empty_like(inp.codes), torch.empty_like(inp.scales)
    e2e = []
    for s in range(max(10, min(args.steps, 30))):
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        c_d.copy_(c_h, non_blocking=True)
        s_d.copy_(s_h, non_blocking=True)
        moe.dequant_mxfp8(c_d, s_d, out)
        o_h.copy_(out, non_blocking=True)
        b.record(stream)
        b.synchronize()
        e2e.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(statistics.median(e2e), dev)
    hbm, bf16, bf16_sus, peak_kind = peaks()
    n = rows * n_in
    nbytes = n + n // 32 + 2 * n
    roof = {"bound": "hbm", "kernel": "dequant_mxfp8", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm,
            "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "traffic": None,
            "peak_kind": f"{peak_kind} hbm_gbs (copy)", "algorithmic_bytes_per_launch": nbytes,
            "frac_of_nominal": nbytes / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS}
    line = {"metric": "mxfp8 weight elements/s dequantised to bf16 at 1 B200; achieved HBM GB/s vs peak",
            "value": world * n / (ms * 1e-3), "unit": "elements/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3->bf16", "data": "synthetic",
            "config": {"workload": name, "rows": rows, "n_in": n_in, "e8m0_range": [cfg["e_lo"], cfg["e_hi"]],
                       "l2": "flushed by reading a 512 MiB buffer between timed steps (outside the events)"},
            "step_ms": st, "roofline": roof,
            "e2e": {"value": world * n / (e2e_ms * 1e-3), "unit": "elements/s",
                    "h2d_bytes_per_step": n + n // 32, "d2h_bytes_per_step": 2 * n, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = fp8_oracle_rate(inp, min(args.cpu_budget, 10.0))
    del inp, flush, out
    torch.cuda.empty_cache()
    return line


def fp8_oracle_rate(inp, budget):
    """The oracle's mxfp8 decode on a bounded sample of rows (elements/s)."""
    import numpy as np
    import oracle
    sample = min(inp.cfg["rows"], 64)
    codes = np.ascontiguousarray(inp.codes[:sample].cpu().numpy())
    words = codes.view(np.uint32)
    scales = inp.scales[:sample].cpu().numpy()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.dequant_mxfp8(words, scales, inp.cfg["n_in"])
        reps += 1
        if time.perf_counter() - t0 > budget:
            break
    rate = reps * sample * inp.cfg["n_in"] / (time.perf_counter() - t0)
    return {"value": rate, "unit": "elements/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} x {sample} rows of the same workload (numpy fp64)",
            "cores_available": len(os.sched_getaffinity(0))}


def hc_oracle_rate(inp, budget):
    """The oracle's Sinkhorn mixing on a bounded sample of tokens (tokens/s)."""
    import oracle
    cfg = inp.cfg
    sample = min(cfg["T"], 256)
    L = inp.logits[:sample].cpu().double().numpy()
    h = inp.h[:sample].cpu().double().numpy()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.hc_mix(oracle.hc_sinkhorn(L, cfg["iters"], cfg["eps"]), h)
        reps += 1
        if time.perf_counter() - t0 > budget:
            break
    per_tok = (time.perf_counter() - t0) / (reps * sample)
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} x {sample} tokens of the same workload (numpy fp64)",
            "cores_available": len(os.sched_getaffinity(0))}


def ours_arm(args):
    import torch
    import torch.distributed as dist

    import bit_quantized_moe_route_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    moe.load_library()
    moe.set_ffn_path({"auto": moe.FFN_AUTO, "gemv": moe.FFN_GEMV, "tc": moe.FFN_TENSOR_CORE}[args.ffn_path])
    names = CONFIG_ORDER if args.config == "all" else [args.config]
    for name in names:
        run = run_hc_config if name.startswith("mhc") else run_fp8_config if name.startswith("mxfp8") else run_config
        line = run(name, args, dev, world, rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        ours_arm(args)


if __name__ == "__main__":
    main()
