"""Benchmark of the Fast-dLLM DualCache decoder on the LLaDA-8B shape.

One "step" = one full block-wise generation (every block-start refresh and
every DualCache block step: the whole hot path) of gen_len tokens after a
prompt, with random N(0, 0.02) bf16 weights of the LLaDA-8B shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fdllm|reference]

Prints one JSON line.  value = generated tokens/s of the whole job (all
ranks), timed with CUDA events on the decoder's stream around K generations
with the prompt already in HBM (max over ranks).  e2e = the same metric
through the host-buffer C call (prompt copied in, tokens copied out every
step).  roofline = the dominant kernel class of a separate profiled
generation (per-launch CUDA events), against MEASURED_PEAKS.json.
cpu_baseline = the float64 oracle on the host cores on a bounded sample.
Multi-GPU runs are independent replicas (one sequence per rank).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gen tokens/s (LLaDA-8B shape, DualCache, tau=0.9)"


def metric_name(wl):
    if wl.name == WORKLOAD and wl.tau == 0.9 and wl.cache_mode == "dual":
        return METRIC
    return f"gen tokens/s ({wl.name}, {wl.cache_mode}, tau={wl.tau})"
WORKLOAD = "llada8b-p256-g256"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _config(wl, n):
    big = wl.shape.n_params * wl.shape.elem_bytes > 1_000_000_000
    return {"workload": wl.name, "model_shape": wl.shape.name, "prompt_len": wl.prompt_len,
            "gen_len": wl.gen_len, "block_size": wl.block_size, "tau": wl.tau,
            "cache_mode": wl.cache_mode, "batch_per_gpu": 1, "global_batch": n,
            "weights": f"random N(0,0.02) {wl.shape.dtype}, seed {wl.shape.seed}",
            "l2": ("no flush needed: each step streams the weights (> 126 MB L2)" if big else
                   "the model fits in L2: a parity configuration, not a bandwidth measurement"),
            "parallelism": "replicas" if n > 1 else "single"}


def _dtype(wl):
    return "f32" if wl.shape.dtype == "fp32" else "bf16"


def _arithmetic(wl):
    """What the kernels compute in, beside the model dtype of `dtype`."""
    if wl.shape.dtype == "fp32":
        return "f32 on CUDA cores (f32 weights and activations)"
    return ("bf16 weights held as f16 (exact for |w| >= 2^-17); tensor-core products on f16 "
            "operands with f32 accumulation; activations, q, K/V and softmax weights stored "
            "as two f16 terms (hi + lo); f32 residual stream, norms and softmax")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = sorted(v for v in (num(r[1]) for r in rows) if v is not None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": num(rows[0][2]),
                "samples": len(rows), "reasons": reasons}


def roofline_from_profile(stats, hbm, tf_sustained, peak_kind, traffic):
    """Dominant kernel class of the generation: the block-step weight
    streamers (chain kernel launches, HBM-bound) or the full-forward GEMMs
    (tensor-bound).  achieved = algorithmic bytes (flops) of its launches /
    their summed event time."""
    groups = {"step": [s for s in stats if s["name"] == "chain.step" or
                       (s["name"].startswith("gemm.") and s["name"].endswith(".step"))],
              "full": [s for s in stats if s["name"].startswith("gemm.") and s["name"].endswith(".full")]}
    tot = {k: sum(s["total_ms"] for s in v) for k, v in groups.items()}
    total_all = sum(s["total_ms"] for s in stats) or 1.0
    key = max(tot, key=tot.get)
    g = groups[key]
    ms = tot[key]
    launches = sum(s["launches"] for s in g)
    if key == "step":
        achieved = sum(s["bytes"] for s in g) / (ms * 1e-3) / 1e9
        out = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s"}
    else:
        achieved = sum(s["flops"] for s in g) / (ms * 1e-3) / 1e12
        out = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tf_sustained,
               "unit": "TFLOP/s"}
    per_launch_bytes = sum(s["bytes"] for s in g) / max(1, launches)
    out["frac"] = round(out["achieved"] / out["peak"], 4)
    out["traffic"] = traffic.get(key)
    out["kernel"] = ("chain_kernel (DualCache block-step GEMMs + norms)" if key == "step"
                     else "gemm_tc2_kernel (full-forward GEMMs on SM pairs)")
    out["share_of_kernel_time"] = round(ms / total_all, 3)
    out["launches"] = launches
    out["algorithmic_bytes_per_launch"] = round(per_launch_bytes)
    out["peak_source"] = peak_kind
    out["classes"] = {s["name"]: {"launches": s["launches"], "ms": round(s["total_ms"], 3),
                                  "GBps": round(s["bytes"] / (s["total_ms"] * 1e-3) / 1e9, 1)
                                  if s["total_ms"] else None,
                                  "TFps": round(s["flops"] / (s["total_ms"] * 1e-3) / 1e12, 1)
                                  if s["total_ms"] else None} for s in stats}
    return out


def block_step_roofline(wl, cached_ms, hbm):
    """The DualCache block step against the HBM roofline: weight bytes + K/V
    bytes read per step (the step's algorithmic bytes) / its measured time,
    against 8 TB/s (the nominal figure the target is stated in) and against
    the measured copy bandwidth."""
    from kv_cache_decode_dualcache_b200 import synth
    sh = wl.shape
    L = wl.prompt_len + wl.gen_len
    weight_bytes = 2 * synth.step_weight_params(sh)
    kv_bytes = sh.n_layers * L * sh.n_kv_heads * sh.head_dim * 2 * 2   # K and V, bf16 values
    total = weight_bytes + kv_bytes
    t = cached_ms * 1e-3
    return {"bytes_per_step": total, "ms_per_step": round(cached_ms, 3),
            "achieved_GBps": round(total / t / 1e9, 1),
            "frac_of_8TBps": round(total / t / 8e12, 4),
            "frac_of_measured": round(total / t / (hbm * 1e9), 4),
            "note": "weights (bf16) + K,V of all L positions read once per block step"}


def generate_roofline(wl, steps_per_block, value, hbm, tf):
    """Whole-generate roofline: every executed step at the slower of its
    algorithmic bytes / HBM bandwidth and its FLOPs / tensor peak; gen_len
    over the sum is the roofline tokens/s, and the measured tokens/s is a
    fraction of it.  A block's first step (every step without a cache) is a
    full forward over all L rows; a DualCache step runs the block rows, a
    prefix-cache step rows [s, L), both over the K/V of all L positions.
    Bytes: the weights once and the K/V of all positions once per step;
    FLOPs: 2 x weights x rows (the LM head on the block rows only) plus
    4 x rows x L x H x hd per layer of attention.  Single-sequence bf16
    workloads only (None for batches and for the fp32 model)."""
    from kv_cache_decode_dualcache_b200 import synth
    if wl.batch != 1 or not steps_per_block or wl.shape.dtype == "fp32":
        return None   # the fp32 model lives in L2 and runs no tensor-core path
    sh = wl.shape
    P, G, B = wl.prompt_len, wl.gen_len, wl.block_size
    L = P + G
    es = sh.elem_bytes
    head = sh.vocab * sh.d_model
    layers = synth.step_weight_params(sh) - head
    bytes_step = es * (layers + head) + es * 2 * sh.n_layers * L * sh.n_kv_heads * sh.head_dim

    def flops(rows):
        return (2.0 * layers * rows + 2.0 * head * B
                + 4.0 * rows * L * sh.n_heads * sh.head_dim * sh.n_layers)

    def step_s(rows, bw, pk):
        return max(bytes_step / bw, flops(rows) / pk)

    peaks = {"nominal": (8e12, 2.25e15), "measured": (hbm * 1e9, tf * 1e12)}
    out = {"steps": {"full": 0, "cached": 0}, "tokens_per_s": {}, "frac": {},
           "full_step_ms": {}, "block_step_ms": {}}
    for b, n in enumerate(steps_per_block):
        out["steps"]["full"] += 1 if wl.cache_mode != "none" else n
        out["steps"]["cached"] += n - 1 if wl.cache_mode != "none" else 0
    for name, (bw, pk) in peaks.items():
        total = 0.0
        for b, n in enumerate(steps_per_block):
            s = P + b * B
            cached_rows = {"dual": B, "prefix": L - s}.get(wl.cache_mode)
            if cached_rows is None:
                total += n * step_s(L, bw, pk)
            else:
                total += step_s(L, bw, pk) + (n - 1) * step_s(cached_rows, bw, pk)
        out["tokens_per_s"][name] = round(G / total, 2)
        out["frac"][name] = round(value / (G / total), 4)
        out["full_step_ms"][name] = round(1e3 * step_s(L, bw, pk), 3)
        out["block_step_ms"][name] = round(1e3 * step_s(B, bw, pk), 3)
    out["peaks"] = {"nominal": "8 TB/s, 2.25 PFLOP/s dense bf16",
                    "measured": f"{hbm:g} GB/s copy, {tf:g} TFLOP/s sustained bf16 GEMM"}
    return out


def _traffic_record(record, source):
    """ncu DRAM bytes per launch recorded in profiles/<record> for the current
    source of the kernel (csrc/<source>), if any: null once the kernel has
    changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", record)
    try:
        rec = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
        src = open(os.path.join(ROOT, "kv_cache_decode_dualcache_b200", "csrc", source),
                   "rb").read()
        if rec.get("source_sha256") == hashlib.sha256(src).hexdigest():
            return float(rec["bytes_per_launch"])
    except Exception:
        pass
    return None


def traffic_records():
    """Per kernel class of roofline_from_profile: the recorded DRAM bytes."""
    return {"step": _traffic_record("chain_traffic.txt", "chain.cu"),
            "full": _traffic_record("gemm_tc2_traffic.txt", "gemm_tc2.cu")}


# ---------------------------------------------------------------- replicas
def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank passes its own device-timed
    milliseconds and gets the maximum (identity on one rank)."""
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, steps, gen_tokens_per_step, ms_max):
    """Whole-job throughput of independent replicas: every rank generated
    steps * gen_tokens_per_step tokens within the slowest rank's time."""
    return world * steps * gen_tokens_per_step / (ms_max * 1e-3)


def replica_prompt(shape, prompt_len, rank):
    """Rank r decodes its own sequence: the workload's prompt recipe with
    salt r (rank 0 gets the single-GPU prompt)."""
    from kv_cache_decode_dualcache_b200 import synth
    return synth.make_prompt(shape, prompt_len, salt=rank).numpy()


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(wl, weights_host, step_counts, sample_layers=4):
    """The float64 oracle, as it stands, on a bounded sample: one block-start
    full forward and one DualCache block step of a model with the first
    `sample_layers` layers, each scaled to the full depth.  Returns the
    oracle's generated tokens/s estimated with the GPU run's step counts."""
    import numpy as np
    import torch
    from kv_cache_decode_dualcache_b200 import synth
    from oracle.model import Model

    sample_layers = min(sample_layers, wl.shape.n_layers)
    shape = synth.with_layers(wl.shape, sample_layers)
    w = {k: v for k, v in weights_host.items()
         if not k.startswith("layers.") or int(k.split(".")[1]) < sample_layers}
    model = Model(shape.as_dict(), w)
    P, G, B = wl.prompt_len, wl.gen_len, wl.block_size
    L = P + G
    prompt = synth.make_prompt(wl.shape, P).numpy()
    x = np.concatenate([prompt, np.full(G, wl.shape.mask_id)])
    t0 = time.perf_counter()
    _, kv = model.forward(x, range(L), return_kv=True, head_rows=range(P, P + B))  # refresh
    t_refresh = time.perf_counter() - t0
    cur = x.copy()
    cur[P:P + B // 2] = prompt[:B // 2]
    t0 = time.perf_counter()
    model.forward(cur, range(P, P + B), cache=kv)                                  # DualCache step
    t_step = time.perf_counter() - t0
    scale = wl.shape.n_layers / sample_layers
    n_ref, n_cached = step_counts
    total = scale * (n_ref * t_refresh + n_cached * t_step)
    return {"tok_s": G / total, "t_refresh_s": t_refresh * scale, "t_step_s": t_step * scale,
            "sample_s": t_refresh + t_step, "threads": torch.get_num_threads(),
            "layers": sample_layers}


def oracle_full_generate(wl, weights_host, reps=1):
    """Small models: the float64 oracle's whole block-wise generate of the
    workload (every step, not a sample), timed on the host cores."""
    import torch
    from kv_cache_decode_dualcache_b200 import synth
    from oracle.decode import generate
    from oracle.model import Model
    model = Model(wl.shape.as_dict(), weights_host)
    prompt = synth.make_prompt(wl.shape, wl.prompt_len).numpy()
    t0 = time.perf_counter()
    for _ in range(reps):
        res = generate(model, prompt, wl.gen_len, wl.block_size, wl.tau, wl.cache_mode)
    dt = (time.perf_counter() - t0) / reps
    return {"tok_s": wl.gen_len / dt, "sample_s": dt * reps, "steps": res.steps,
            "threads": torch.get_num_threads()}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from kv_cache_decode_dualcache_b200 import synth
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if wl.shape.n_params < 50_000_000 and wl.batch == 1:
        return run_reference_whole(args, wl, {k: v.cpu() for k, v in
                                              synth.make_weights(wl.shape, device=dev).items()})
    sample_layers = min(4, wl.shape.n_layers)
    w = synth.make_weights(wl.shape, device=dev)
    w = {k: v.cpu() for k, v in w.items()
         if not k.startswith("layers.") or int(k.split(".")[1]) < sample_layers}
    # step counts of this workload's decode (8 blocks; the GPU run measured
    # 3.25 steps per block on average); the oracle runs the same schedule
    n_blocks = wl.gen_len // wl.block_size
    counts = (n_blocks, args.ref_cached_steps)
    vals = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(wl, w, counts, sample_layers)
        if i >= args.warmup:
            vals.append(r)
    v = sum(r["tok_s"] for r in vals) / len(vals)
    sample_s = [round(r["sample_s"], 3) for r in vals]
    line = {"impl": "reference", "metric": metric_name(wl), "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            # an estimate: each "step" times one bounded sample, not a whole
            # generation; ms_per_step is the measured time of one sample, the
            # estimated time of one generation is in "estimate"
            "ms_per_step": 1e3 * sum(sample_s) / len(sample_s), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "estimated": True,
            "estimate": {"ms_per_generation": 1e3 * wl.gen_len / v,
                         "measured_sample_seconds": sample_s,
                         "timed_region_seconds": round(sum(sample_s), 3),
                         "layers_run": sample_layers, "layers_model": wl.shape.n_layers,
                         "layer_scale": wl.shape.n_layers / sample_layers,
                         "refresh_steps_per_generation": counts[0],
                         "cached_steps_per_generation": counts[1],
                         "step_counts_from": "the GPU decoder's schedule on this workload "
                                             "(--ref-cached-steps; the float64 oracle cannot "
                                             "run the whole generation in minutes)"},
            "config": _config(wl, 1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["threads"],
                             "kind": "oracle",
                             "sample": f"per step: one block-start full forward and one DualCache "
                                       f"block step of the first {sample_layers} of "
                                       f"{wl.shape.n_layers} layers, scaled x"
                                       f"{wl.shape.n_layers / sample_layers:g}; "
                                       f"{counts[0]} refresh + {counts[1]} cached steps"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_whole(args, wl, w_host):
    """Reference arm of a small model: the float64 oracle runs the whole
    generate of the workload each step (no sample, no estimate)."""
    vals = []
    for i in range(args.warmup + args.steps):
        r = oracle_full_generate(wl, w_host)
        if i >= args.warmup:
            vals.append(r)
    v = sum(r["tok_s"] for r in vals) / len(vals)
    secs = sum(r["sample_s"] for r in vals)
    line = {"impl": "reference", "metric": metric_name(wl), "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "estimated": False,
            "config": _config(wl, 1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["threads"],
                             "kind": "oracle",
                             "sample": f"the whole generate of this workload per step "
                                       f"({vals[0]['steps']} denoising steps, float64 oracle)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def run_fdllm(args, wl):
    import numpy as np
    import torch
    import torch.distributed as dist
    from kv_cache_decode_dualcache_b200 import build, fdllm, synth

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()

    def barrier():
        if world > 1:
            dist.barrier()

    shape = wl.shape
    P, G, B, tau = wl.prompt_len, wl.gen_len, wl.block_size, wl.tau
    stream = torch.cuda.Stream()
    dec = fdllm.Decoder(shape, P + G, device=local, stream=stream.cuda_stream)
    w = synth.make_weights(shape, device="cuda")
    dec.load_weights(w)
    want_cpu = (not args.no_cpu_baseline) and world == 1 and rank == 0
    small = shape.n_params < 50_000_000   # the oracle runs the whole generate
    w_host = None
    if want_cpu:
        w_host = {k: v.cpu() for k, v in w.items()
                  if small or not k.startswith("layers.") or int(k.split(".")[1]) < 4}
    del w
    torch.cuda.empty_cache()
    prompt = replica_prompt(shape, P, rank)
    prompt_host = torch.from_numpy(prompt).pin_memory()
    prompt_dev = prompt_host.to(f"cuda:{local}")
    out_dev = torch.empty(G, dtype=torch.int32, device=f"cuda:{local}")
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        dec.generate_device(prompt_dev, G, B, tau, out_dev, wl.cache_mode)
    torch.cuda.synchronize()

    # ---- timed region: device-resident prompt
    sampler = ClockSampler(local) if rank == 0 else None
    dec.launch_count(reset=True)
    steps_total = 0
    barrier()
    torch.cuda.synchronize()
    # one event between generations (the call returns once its work is done)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for i in range(args.steps):
        steps_total += dec.generate_device(prompt_dev, G, B, tau, out_dev, wl.cache_mode)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = evs[0].elapsed_time(evs[-1])
    per_gen = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps))
    launches = dec.launch_count(reset=True)
    clocks = sampler.stop() if sampler else None
    ms_max = max_over_ranks(ms, world, f"cuda:{local}")
    value = job_tokens_per_s(world, args.steps, G, ms_max)
    tokens = out_dev.cpu().numpy()

    # ---- end to end: host buffers through the C call
    out_host = torch.empty(G, dtype=torch.int32).pin_memory()
    barrier()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    e2e_steps = 0
    stats = None
    for _ in range(args.steps):
        res, nsteps, stats = dec.generate(prompt_host.numpy(), G, B, tau, wl.cache_mode)
        out_host.numpy()[:] = res
        e2e_steps += nsteps
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_value = job_tokens_per_s(world, args.steps, G,
                                 max_over_ranks(e2.elapsed_time(e3), world, f"cuda:{local}"))
    steps_per_gen = e2e_steps / args.steps
    # the device-resident call and the host-buffer call run the same decode:
    # their tokens must be identical
    same_tokens = bool(np.array_equal(np.asarray(tokens), np.asarray(out_host.numpy())))
    if not same_tokens:
        print("bench: device-resident and host-buffer generates returned different tokens",
              file=sys.stderr)
    h2d = P * 4
    d2h = G * 4 + int(round(steps_per_gen)) * 20   # tokens + per-step state / error words

    # ---- roofline: one profiled generation (per-launch events)
    fdllm.fdllm_profile_enable(dec.ctx, True)
    dec.generate_device(prompt_dev, G, B, tau, out_dev, wl.cache_mode)
    prof = fdllm.fdllm_profile_read(dec.ctx)
    fdllm.fdllm_profile_enable(dec.ctx, False)
    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    roof = roofline_from_profile(prof, hbm, tf_sust, peak_kind, traffic_records())
    timing = dec.generate(prompt, G, B, tau, wl.cache_mode, timing=True)[2]

    cpu = None
    if want_cpu and small:
        cores = len(os.sched_getaffinity(0))
        torch.set_num_threads(cores)
        r = oracle_full_generate(wl, w_host)
        cpu = {"value": r["tok_s"], "unit": "tokens/s", "cores": r["threads"], "kind": "oracle",
               "sample": f"the whole generate of this workload ({r['steps']} denoising steps, "
                         f"float64 oracle, {r['sample_s']:.2f} s)"}
    elif want_cpu:
        cores = len(os.sched_getaffinity(0))
        torch.set_num_threads(cores)
        r = oracle_sample(wl, w_host, (timing.refresh_steps, timing.cached_steps))
        cpu = {"value": r["tok_s"], "unit": "tokens/s", "cores": r["threads"], "kind": "oracle",
               "sample": "one block-start full forward and one DualCache block step of the "
                         f"first {r['layers']} of {wl.shape.n_layers} layers (float64 oracle), "
                         f"scaled x{wl.shape.n_layers / r['layers']:g} and weighted by "
                         f"this run's {timing.refresh_steps} refresh + {timing.cached_steps} "
                         f"cached steps ({r['sample_s']:.1f} s of CPU work)",
               "t_refresh_s": round(r["t_refresh_s"], 3), "t_step_s": round(r["t_step_s"], 3)}

    if rank == 0:
        line = {"metric": metric_name(wl), "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": _dtype(wl), "arithmetic": _arithmetic(wl),
                "data": "synthetic",
                "config": _config(wl, world),
                "decode": {"denoising_steps_per_generation": steps_total / args.steps,
                           "ms_per_generation": {"median": round(per_gen[len(per_gen) // 2], 3),
                                                 "min": round(per_gen[0], 3),
                                                 "max": round(per_gen[-1], 3)},
                           "steps_per_block": timing.steps_per_block,
                           "refresh_ms_per_step": round(timing.refresh_ms / max(1, timing.refresh_steps), 3),
                           "cached_ms_per_step": round(timing.cached_ms / max(1, timing.cached_steps), 3),
                           "tokens_checksum": int(np.asarray(tokens, dtype=np.int64).sum()),
                           "tokens_match_host_call": same_tokens},
                "generate_roofline": generate_roofline(wl, timing.steps_per_block, value, hbm,
                                                       tf_sust),
                "block_step_roofline": (block_step_roofline(
                    wl, timing.cached_ms / timing.cached_steps, hbm)
                    if timing.cached_steps else None),   # cache off: every step is a refresh
                "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s",
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches,
                "roofline": roof,
                "clocks": clocks,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    dec.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_fdllm_batch(args, wl):
    """Variable-length batch (independent sequences, per-sequence block
    schedules, one shared weight stream per global step) through
    fdllm_generate_batch; value = generated tokens of the whole batch per
    second of device time (host prompts in, tokens out: the batched entry
    point is host-buffer only, so value and e2e time the same call)."""
    import numpy as np
    import torch
    from kv_cache_decode_dualcache_b200 import build, fdllm, synth
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    shape = wl.shape
    G, B, tau = wl.gen_len, wl.block_size, wl.tau
    lens = synth.make_batch_prompt_lengths(wl.batch)
    prompts = [synth.make_prompt(shape, n, salt=rank * 1000 + i).numpy() for i, n in enumerate(lens)]
    stream = torch.cuda.Stream()
    dec = fdllm.Decoder(shape, max(lens) + G, device=local, stream=stream.cuda_stream,
                        max_batch=wl.batch)
    w = synth.make_weights(shape, device="cuda")
    dec.load_weights(w)
    del w
    torch.cuda.empty_cache()
    for _ in range(args.warmup):
        dec.generate_batch(prompts, G, B, tau, wl.cache_mode)
    sampler = ClockSampler(local) if rank == 0 else None
    dec.launch_count(reset=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    steps = None
    for _ in range(args.steps):
        out, steps, st = dec.generate_batch(prompts, G, B, tau, wl.cache_mode)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = dec.launch_count(reset=True)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(e0.elapsed_time(e1), world, f"cuda:{local}")
    value = job_tokens_per_s(world, args.steps, wl.batch * G, ms)
    timing = dec.generate_batch(prompts, G, B, tau, wl.cache_mode, timing=True)[2]
    fdllm.fdllm_profile_enable(dec.ctx, True)
    dec.generate_batch(prompts, G, B, tau, wl.cache_mode)
    prof = fdllm.fdllm_profile_read(dec.ctx)
    fdllm.fdllm_profile_enable(dec.ctx, False)
    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    roof = roofline_from_profile(prof, hbm, tf_sust, peak_kind, traffic_records())
    if rank == 0:
        cfg = _config(wl, world)
        cfg.update({"prompt_lens": lens, "batch_per_gpu": wl.batch,
                    "global_batch": wl.batch * world,
                    "batching": f"continuous batching over {wl.batch} sequence slots: one "
                                "forward per global step over every active sequence's rows "
                                "(shared weight stream)"})
        line = {"metric": metric_name(wl), "value": round(value, 2), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "arithmetic": _arithmetic(wl), "data": "synthetic",
                "config": cfg,
                "decode": {"denoising_steps_per_generation": int(np.asarray(steps).sum()),
                           "refresh_ms_per_step": round(timing.refresh_ms / max(1, timing.refresh_steps), 3),
                           "cached_ms_per_step": round(timing.cached_ms / max(1, timing.cached_steps), 3)},
                "e2e": {"value": round(value, 2), "unit": "tokens/s",
                        "h2d_bytes_per_step": 4 * sum(lens), "d2h_bytes_per_step": 4 * wl.batch * G},
                "gpu_launches": launches, "roofline": roof, "clocks": clocks, "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    dec.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_kv_similarity(args, wl):
    """The approximate cache's premise on this workload: cosine of the K/V a
    full forward gives at the first block's start and after that block's
    first denoising step, per layer, over the positions a DualCache step
    takes from the cache (prefix and suffix); fdllm_kv_similarity on the
    GPU.  Random weights: the numbers show the diagnostic, not a trained
    model's behaviour."""
    import numpy as np
    import torch
    from kv_cache_decode_dualcache_b200 import build, fdllm, synth
    torch.cuda.set_device(0)
    build.build()
    shape = wl.shape
    P, G, B = wl.prompt_len, wl.gen_len, wl.block_size
    dec = fdllm.Decoder(shape, P + G, device=0)
    w = synth.make_weights(shape, device="cuda")
    dec.load_weights(w)
    del w
    prompt = synth.make_prompt(shape, P).numpy()
    x_a = np.concatenate([prompt, np.full(G, shape.mask_id)]).astype(np.int32)
    r = dec.step_debug(x_a, x_a, P, B, wl.tau, "dual", logits=False)
    x_b = x_a.copy()
    x_b[P:P + B][r["unmask"]] = r["tok"][r["unmask"]]
    dec.kv_similarity(x_a, x_b)  # warm-up (allocates the cache copy)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    cos = dec.kv_similarity(x_a, x_b)
    ms = (time.perf_counter() - t0) * 1e3
    reused = np.r_[0:P, P + B:P + G]
    layers = [{"layer": li,
               "k_min": round(float(cos[li, 0, reused].min()), 6),
               "k_mean": round(float(cos[li, 0, reused].mean()), 6),
               "v_min": round(float(cos[li, 1, reused].min()), 6),
               "v_mean": round(float(cos[li, 1, reused].mean()), 6)} for li in range(shape.n_layers)]
    line = {"metric": f"K/V cosine similarity, block start vs after its first step ({wl.name})",
            "unit": "cosine", "unmasked_by_the_step": int(r["unmask"].sum()),
            "positions_reused": int(reused.size), "call_ms": round(ms, 2),
            "data": "synthetic (random N(0,0.02) weights)", "layers": layers}
    print(json.dumps(line), flush=True)
    dec.close()
    return 0


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_replicas(n: int, argv, script: str = None, timeout_s: float = 3600.0) -> int:
    """Run `script argv` as n ranks of one node under torch.distributed.run
    (rendezvous on 127.0.0.1), passing their output through; returns the
    launcher's exit code.  bench.py uses it when --gpus N > 1 is given without
    a launcher around it."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           script or os.path.abspath(__file__)] + list(argv)
    try:
        return subprocess.run(cmd, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        print(f"bench.py: the {n} replica ranks did not finish within {timeout_s:.0f} s",
              file=sys.stderr)
        return 124


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fdllm", choices=["fdllm", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    help="another configuration of the same decoder (synth.WORKLOADS), "
                         "e.g. llada8b-p1024-g1024, dream7b-p512-g512")
    ap.add_argument("--tau", type=float, default=None, help="override the workload's tau")
    ap.add_argument("--cache-mode", default=None, choices=["none", "prefix", "dual"],
                    help="override the workload's cache mode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-similarity", action="store_true",
                    help="print the K/V similarity diagnostic for the workload instead")
    ap.add_argument("--ref-cached-steps", type=int, default=18,
                    help="cached steps per generation assumed by the reference arm")
    args = ap.parse_args()
    world_env = os.environ.get("WORLD_SIZE")
    if args.gpus > 1 and world_env is None:
        # no launcher around this process: start the N replica ranks here
        return launch_replicas(args.gpus, sys.argv[1:])
    if world_env is not None and int(world_env) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}", file=sys.stderr)
        return 2
    from kv_cache_decode_dualcache_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.tau is not None or args.cache_mode is not None:
        import dataclasses
        wl = dataclasses.replace(wl, tau=wl.tau if args.tau is None else args.tau,
                                 cache_mode=args.cache_mode or wl.cache_mode)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.kv_similarity:
        return run_kv_similarity(args, wl)
    if wl.batch > 1:
        return run_fdllm_batch(args, wl)
    return run_fdllm(args, wl)


if __name__ == "__main__":
    sys.exit(main())
