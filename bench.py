#!/usr/bin/env python
"""Denoise-step throughput of the AuraFlow forward on B200.

One step = one step of the 25-step, shift-1.73 sampling loop on the
1024 x 1024 workload, run through the sampler plan (af_sampler: every step's
modulations from one GEMM per 25-step run, each step a CUDA graph): the
latent [1, 4, 128, 128] is duplicated into a CFG batch of 2, the full
AuraFlowTransformer2DModel forward (patch embed, 4 joint + 32 single blocks,
pre-final, unpatchify; D = 3072, 12 x 256 heads, FFN 8192, 256 text tokens +
8 registers) runs on it, and the guidance combine + flow-match Euler update
moves the latent to the next sigma.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl af|reference]
                    [--workload 1024|1536] [--fp8] [--direct] [--no-cpu-baseline]
                    [--no-e2e] [--case single_block]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own
independent replica (weak scaling, no collective on the data path); the
elapsed time is the max over ranks.  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload.  ``--fp8`` times the 8-bit
variant (e4m3 operands for every block projection), ``--direct`` the per-step entry
point without the plan.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "denoise steps/s (full 36-block fwd, 1024², B=2) + bf16 TFLOP/s % of peak"
WORKLOADS = {
    "1024": dict(H=128, W=128, L=256, G=64,
                 name="AuraFlow denoise step at 1024x1024: latent 4x128x128, CFG batch 2, 4 joint + 32 single "
                      "blocks, D=3072 (12x256 heads), FFN 8192, 256 text + 8 register tokens, 4096 image tokens"),
    "1536": dict(H=192, W=192, L=256, G=96,
                 name="AuraFlow denoise step at 1536x1536: latent 4x192x192, CFG batch 2, 4 joint + 32 single "
                      "blocks, D=3072, 256 text + 8 register tokens, 9216 image tokens"),
}
GUIDANCE = 3.5
N_SCHED = 25
SHIFT = 1.73
NOMINAL_BF16_TFLOPS = 2250.0   # B200 dense bf16 tensor-core peak (nominal, without sparsity)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="af", choices=["af", "reference"])
    ap.add_argument("--workload", default="1024", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-1536", action="store_true", help="skip the 1536x1536 sub-record of the default line")
    ap.add_argument("--seed", type=int, default=4)
    ap.add_argument("--fp8", action="store_true",
                    help="8-bit variant: e4m3 operands for every block projection (af_weights_quantize_fp8)")
    ap.add_argument("--direct", action="store_true",
                    help="time the per-step entry point (af_denoise_step) instead of the sampler plan")
    ap.add_argument("--case", default="step", choices=["step", "single_block", "small_model"],
                    help="single_block: time one full-shape AuraFlowSingleTransformerBlock only; "
                         "small_model: a 1-block model's forward + guidance/Euler step at the workload's "
                         "shapes (every HBM-bound kernel, a few GB on the device); both are small "
                         "commands for profiler captures")
    return ap.parse_args()


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"):
            if k in m:
                p[k] = float(m[k])
        p["source"] = "measured"
    return p


def model_dims():
    D, F, heads, hd, Dj, R = 3072, 8192, 12, 256, 2048, 8
    return D, F, heads, hd, Dj, R


def step_flops(H, W, L, B=2):
    """Algorithmic FLOPs of one forward (dense matmuls + attention) at batch B."""
    D, F, heads, hd, Dj, R = model_dims()
    Ni = (H // 2) * (W // 2)
    N = R + L + Ni
    per_block = 2.0 * N * (4 * D * D + 3 * D * F) + 4.0 * N * N * D
    ada_rows = (2 * 4 + 32) * 6 * D + 2 * D
    return B * (36 * per_block + 2.0 * L * Dj * D + 2.0 * ada_rows * D + 2.0 * Ni * D * 16 * 2)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock / throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm_sorted = sorted(sm)
        return {"sm_mhz": sm_sorted[len(sm_sorted) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- CPU oracle sample

class OracleBlockSample:
    """One AuraFlowSingleTransformerBlock of the workload (B = 2, all tokens)
    in the fp64 oracle; inputs drawn once, ``run()`` times one evaluation."""

    def __init__(self, H, W, L, seed, n_rows=None):
        import oracle as O
        import synth
        self.O = O
        self.cfg = O.Config(num_mmdit_layers=0, num_single_dit_layers=1, pos_embed_max_size=(W // 2) ** 2)
        self.N = 8 + L + (H // 2) * (W // 2) if n_rows is None else n_rows
        self.pre = "single_transformer_blocks.0."
        self.w = synth.weights(seed, [s for s in O.weight_specs(self.cfg) if s[0].startswith(self.pre)])
        self.x = synth.activations(seed, "bench_x", (2, self.N, self.cfg.inner_dim))
        self.temb = synth.conditioning(seed, (2, self.cfg.inner_dim))

    def run(self):
        t0 = time.perf_counter()
        self.O.single_block(self.x, self.temb, self.w, self.pre, self.cfg)
        return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    H, W, L = wl["H"], wl["W"], wl["L"]
    small = OracleBlockSample(H, W, L, args.seed, n_rows=512)
    for _ in range(args.warmup):   # warm-up on a small token count (pages BLAS in)
        small.run()
    sample = OracleBlockSample(H, W, L, args.seed)
    N = sample.N
    times = [sample.run() for _ in range(args.steps)]
    per_block = sum(times) / len(times)
    step_s = 36 * per_block
    value = 1.0 / step_s
    cores = blas_threads()
    sample = (f"one single DiT block of the workload (B=2, {N} tokens, D=3072) in the fp64 numpy oracle per "
              f"timed unit; a denoise step is taken as 36 such blocks (joint blocks cost the same FLOPs); "
              f"{cpu_model()}")
    # what ran: args.steps single blocks of ms_per_step each; value is the
    # steps/s those blocks extrapolate to (36 blocks per denoise step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_block * 1000.0,
            "timed_unit": "one single DiT block (1/36 of a denoise step); steps and ms_per_step count blocks",
            "extrapolated_to_step": {"blocks_per_step": 36, "s_per_denoise_step": step_s, "steps_per_s": value},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl["name"], "sample": "1 of 36 blocks per timed unit"},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA arm

def make_weights(af, torch, w, seed, device):
    """Seeded synthetic weights filled on the device by the library
    (af_weights_init_random: linear weights ~N(0, 0.02^2), positions
    ~N(0, 0.1^2), registers ~N(0, 0.02^2))."""
    w.init_random(seed, 0.02)
    torch.cuda.synchronize()


def run_af(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import diffusion_transformer_denoising_auraflow_b200 as af

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    H, W, L, G = wl["H"], wl["W"], wl["L"], wl["G"]
    Ni = (H // 2) * (W // 2)
    cfg = af.Config.default(pos_embed_max_size=G * G)
    w = af.Weights(cfg, local_rank)
    make_weights(af, torch, w, args.seed, device)
    if args.fp8:
        w.quantize_fp8()
        torch.cuda.synchronize()
    s = af.Scratch(w, 2, Ni, L)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)   # graphs cannot be captured on the legacy default stream

    gen = torch.Generator(device=device)
    gen.manual_seed(args.seed * 7919 + rank)
    lat0 = torch.randn(1, 4, H, W, generator=gen, device=device)
    text = torch.randn(2, L, 2048, generator=gen, device=device).to(torch.bfloat16)
    lat = lat0.clone()
    sig = af.sigma_schedule(N_SCHED, SHIFT)
    lat_d = torch.empty_like(lat0)
    text_d = torch.empty_like(text)
    # the product path: the sampler plan (all modulations in one GEMM per
    # 25-step run, every step a CUDA graph), one plan per bound latent buffer
    plans = {} if args.direct else {id(lat): af.Sampler(w, s, lat, text, sig, GUIDANCE, use_graphs=True),
                                    id(lat_d): af.Sampler(w, s, lat_d, text_d, sig, GUIDANCE, use_graphs=True)}

    def direct_step(i, latents, text_emb):
        j = i % N_SCHED
        af.denoise_step(w, s, latents, text_emb, GUIDANCE, sig[j], sig[j + 1], stream)

    def step(i, latents, text_emb):
        if args.direct:
            return direct_step(i, latents, text_emb)
        plan, j = plans[id(latents)], i % N_SCHED
        if j == 0:
            plan.prepare(stream)    # modulation table of the whole run, timed with its first step
        plan.step(j, stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    # build the plans: capture and instantiate all N_SCHED step graphs (untimed)
    for plan_lat, plan_txt in ((lat, text), (lat_d, text_d)):
        if args.direct:
            break
        plan_lat.copy_(lat0)
        plan_txt.copy_(text)
        for i in range(N_SCHED):
            step(i, plan_lat, plan_txt)
    lat.copy_(lat0)
    # warm-up
    for i in range(args.warmup):
        step(i, lat, text)
    s.sync()

    # ---- timed region (device events on the launching stream)
    c0 = s.launch_counts()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(i, lat, text)
        e1.record(stream)
        barrier()
    elapsed = e0.elapsed_time(e1) / 1000.0
    s.sync()
    c1 = s.launch_counts()
    launches = sum(c1) - sum(c0)
    t_max = max_over_ranks(elapsed)
    value = world * args.steps / t_max
    clocks = clk.summary()

    # ---- the per-step path (no plan, no graphs): same kernels, the step's modulations by one GEMM each step
    direct = None
    if not args.direct:
        for i in range(2):
            direct_step(i, lat, text)
        barrier()
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e4.record(stream)
        for i in range(args.steps):
            direct_step(i, lat, text)
        e5.record(stream)
        barrier()
        direct = world * args.steps / max_over_ranks(e4.elapsed_time(e5) / 1000.0)

    # ---- per-kernel-class device time over a few more steps (live roofline);
    # the event profiler brackets every launch, so it runs on the per-step path
    n_prof = max(3, min(args.steps, 5))
    barrier()
    s.profile_begin()
    for i in range(n_prof):
        direct_step(i, lat, text)
    ms, nl, work = s.profile_end()
    pk = peaks()
    gemm_ms_launch = ms[0] / max(nl[0], 1)
    gemm_flops_launch = work[0] / max(nl[0], 1)
    gemm_tflops = gemm_flops_launch / (gemm_ms_launch * 1e-3) / 1e12
    attn_tflops = work[1] / (ms[1] * 1e-3) / 1e12 if ms[1] > 0 else None
    ln_gbs = work[2] / (ms[2] * 1e-3) / 1e9 if ms[2] > 0 else None
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "gemm_traffic.txt")
    if os.path.exists(tpath):
        try:
            import hashlib
            with open(tpath) as f:
                tr = dict(ln.split(":", 1) for ln in f.read().splitlines() if ln and not ln.startswith("#"))
            h = hashlib.sha1()
            for name in ("gemm.cu", "ptx.cuh", "af_internal.h"):
                with open(os.path.join(ROOT, "diffusion_transformer_denoising_auraflow_b200", "csrc", name), "rb") as f:
                    h.update(f.read())
            if tr.get("sources_sha1", "").strip() == h.hexdigest() and args.workload == "1024":  # stale once the kernel changes; captured at 1024^2
                traffic = float(tr["bytes_per_launch"])
        except (OSError, ValueError, KeyError):
            traffic = None
    peak = pk["bf16_tflops_sustained"]
    peak_note = f"{pk['source']} (sustained cuBLAS bf16)"
    if args.fp8:
        # every block projection is e4m3 (2x the bf16 rate nominally); the context embedder and the
        # plan's modulation GEMM stay bf16: weight the peak by the FLOP shares of one step
        D, F, _, _, Dj, _ = model_dims()
        Ntok = 8 + L + Ni
        blocks = 36 * 2.0 * 2 * Ntok * (4 * D * D + 3 * D * F)
        ctx = 2 * 2.0 * L * Dj * D
        f8 = blocks / (blocks + ctx)
        peak = 1.0 / (f8 / (2.0 * peak) + (1.0 - f8) / peak)
        peak_note += f"; {f8:.1%} of GEMM FLOPs e4m3 at 2x (nominal ratio), FLOP-weighted"
    roofline = {"bound": "tensor", "kernel": "gemm_tcgen05_pair (M >= 1024) / gemm_tcgen05",
                "achieved": gemm_tflops,
                "peak": peak, "unit": "TFLOP/s", "frac": gemm_tflops / peak,
                "traffic": None if args.fp8 else traffic, "peak_source": peak_note,
                "flops_per_launch": gemm_flops_launch, "ms_per_launch": gemm_ms_launch}
    step_ms_classes = [x / n_prof for x in ms]

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        lat_h = lat0.cpu().pin_memory()
        text_h = text.cpu().pin_memory()
        out_h = torch.empty_like(lat_h).pin_memory()
        for i in range(2):
            lat_d.copy_(lat_h, non_blocking=True)
            text_d.copy_(text_h, non_blocking=True)
            step(i, lat_d, text_d)
            out_h.copy_(lat_d, non_blocking=True)
        barrier()
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2.record(stream)
        for i in range(args.steps):
            lat_d.copy_(lat_h, non_blocking=True)
            text_d.copy_(text_h, non_blocking=True)
            step(i, lat_d, text_d)
            out_h.copy_(lat_d, non_blocking=True)
        e3.record(stream)
        barrier()
        t_e2e = max_over_ranks(e2.elapsed_time(e3) / 1000.0)
        e2e = {"value": world * args.steps / t_e2e, "unit": "steps/s",
               "h2d_bytes_per_step": lat_h.numel() * 4 + text_h.numel() * 2,
               "d2h_bytes_per_step": out_h.numel() * 4}
    s.sync()

    flops = step_flops(H, W, L)
    tflops = flops * value / world / 1e12
    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_max / args.steps * 1000.0, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 (block projections) + bf16" if args.fp8 else "bf16",
            "data": "synthetic (seeded random weights ~N(0,0.02^2), positions ~N(0,0.1^2); latents, text ~N(0,1))",
            "config": {"workload": wl["name"], "cfg_batch": 2, "tokens": 8 + L + Ni, "global_batch": 2 * world,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "no flush needed: each step streams 13.6 GB of weights (> 126 MB L2)"},
            "tflops": tflops, "tflops_frac_of_peak": tflops * 1e12 / (pk["bf16_tflops"] * 1e12),
            "tflops_peak_used": pk["bf16_tflops"], "peak_source": pk["source"] + " (burst cuBLAS bf16)",
            "tflops_frac_of_nominal_peak": tflops / NOMINAL_BF16_TFLOPS,
            "nominal_peak_tflops": NOMINAL_BF16_TFLOPS,
            "clocks": clocks, "gpu_launches": launches, "roofline": roofline,
            "kernel_ms_per_step": {"gemm": step_ms_classes[0], "attention": step_ms_classes[1],
                                   "ln_modulate": step_ms_classes[2], "other": step_ms_classes[3]},
            "kernel_rates": {"attention_tflops": attn_tflops, "ln_modulate_gbs": ln_gbs},
            "e2e": e2e,
            "path": ("per-step calls (af_denoise_step)" if args.direct else
                     "af_sampler: modulations of all 25 steps in one GEMM per run (timed), steps as CUDA graphs"),
            "plan_prepare": (None if args.direct else
                             f"the 25-step modulation GEMM (af_sampler_prepare) is timed at every step whose index "
                             f"is a multiple of 25: {(args.steps + N_SCHED - 1) // N_SCHED} time(s) in these "
                             f"{args.steps} steps"),
            "per_step_path_steps_per_s": direct,
        }
    for plan in plans.values():
        plan.close()
    s.close()
    w.close()
    if line is not None and world == 1 and args.workload == "1024" and not args.no_1536:
        line["workloads"] = {"1536": measure_1536(args, af, torch, device, stream, pk)}
    return line


def measure_1536(args, af, torch, device, stream, pk):
    """The 1536 x 1536 workload (latent 4 x 192 x 192, 9216 image + 264 text
    tokens, 96 x 96 position grid), timed like the main line through the
    sampler plan (graphs captured untimed first), plus the per-kernel-class
    split of one per-step-path step."""
    wl = WORKLOADS["1536"]
    H, W, L, G = wl["H"], wl["W"], wl["L"], wl["G"]
    Ni = (H // 2) * (W // 2)
    w = af.Weights(af.Config.default(pos_embed_max_size=G * G), device.index)
    make_weights(af, torch, w, args.seed, device)
    if args.fp8:
        w.quantize_fp8()
    s = af.Scratch(w, 2, Ni, L)
    gen = torch.Generator(device=device)
    gen.manual_seed(args.seed * 7919 + 1536)
    lat0 = torch.randn(1, 4, H, W, generator=gen, device=device)
    text = torch.randn(2, L, 2048, generator=gen, device=device).to(torch.bfloat16)
    lat = lat0.clone()
    sig = af.sigma_schedule(N_SCHED, SHIFT)
    plan = af.Sampler(w, s, lat, text, sig, GUIDANCE, use_graphs=True)
    plan.prepare(stream)
    for i in range(N_SCHED):       # capture every step graph (untimed)
        plan.step(i, stream)
    lat.copy_(lat0)
    steps = max(3, min(args.steps, 8))
    plan.prepare(stream)
    for i in range(2):
        plan.step(i, stream)
    s.sync(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        e0.record(stream)
        for i in range(steps):
            j = i % N_SCHED
            if j == 0:
                plan.prepare(stream)
            plan.step(j, stream)
        e1.record(stream)
        torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1000.0
    s.profile_begin()
    af.denoise_step(w, s, lat, text, GUIDANCE, sig[3], sig[4], stream)
    ms, nl, work = s.profile_end(stream)
    plan.close()
    s.close()
    w.close()
    value = steps / t
    tflops = step_flops(H, W, L) * value / 1e12
    return {"workload": wl["name"], "tokens": 8 + L + Ni, "steps": steps, "value": value, "unit": "steps/s",
            "ms_per_step": t / steps * 1000.0, "tflops": tflops,
            "tflops_frac_of_peak": tflops / pk["bf16_tflops"], "tflops_frac_of_nominal_peak": tflops / NOMINAL_BF16_TFLOPS,
            "kernel_ms_per_step": {"gemm": ms[0], "attention": ms[1], "ln_modulate": ms[2], "other": ms[3]},
            "kernel_rates": {"gemm_tflops": work[0] / (ms[0] * 1e-3) / 1e12 if ms[0] > 0 else None,
                             "attention_tflops": work[1] / (ms[1] * 1e-3) / 1e12 if ms[1] > 0 else None,
                             "ln_modulate_gbs": work[2] / (ms[2] * 1e-3) / 1e9 if ms[2] > 0 else None},
            "clocks": clk.summary(),
            "note": "same timing as the main line (sampler plan, CUDA graphs, device events, prepare timed at "
                    "step 0); kernel split from one per-step-path step under the event profiler"}


def run_single_block_case(args):
    """One AuraFlowSingleTransformerBlock at the workload's full shape (B = 2,
    8 + L + Ni tokens, D = 3072), repeated: warm-up, then --steps timed calls."""
    import torch
    import diffusion_transformer_denoising_auraflow_b200 as af
    wl = WORKLOADS[args.workload]
    H, W, L, G = wl["H"], wl["W"], wl["L"], wl["G"]
    Ni = (H // 2) * (W // 2)
    N = 8 + L + Ni
    cfg = af.Config.default(num_mmdit_layers=0, num_single_dit_layers=1, pos_embed_max_size=G * G)
    w = af.Weights(cfg, 0)
    make_weights(af, torch, w, args.seed, torch.device("cuda", 0))
    if args.fp8:
        w.quantize_fp8()
    s = af.Scratch(w, 2, Ni, L)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(args.seed)
    x = torch.randn(2, N, 3072, generator=gen, device="cuda").to(torch.bfloat16)
    temb = torch.randn(2, 3072, generator=gen, device="cuda")
    for _ in range(args.warmup):
        af.single_block(w, s, 0, x, temb)
    s.sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        af.single_block(w, s, 0, x, temb)
    e1.record()
    s.sync()
    ms = e0.elapsed_time(e1) / args.steps
    D, F = 3072, 8192
    flops = 2 * (2.0 * N * (4 * D * D + 3 * D * F) + 4.0 * N * N * D)
    print(json.dumps({"case": "single_block", "fp8": bool(args.fp8), "tokens": N, "ms_per_block": ms,
                      "tflops": flops / (ms * 1e-3) / 1e12}), flush=True)
    return 0


def run_small_model_case(args):
    """A model with one single DiT block at the workload's full shapes (CFG
    batch 2, 8 + L + Ni tokens, D = 3072): every HBM-bound kernel of the step
    (timestep MLP and modulation GEMV, patch embed, LayerNorm + modulate,
    output stage, guidance + Euler) at full size, with ~0.5 GB of weights."""
    import torch
    import diffusion_transformer_denoising_auraflow_b200 as af
    wl = WORKLOADS[args.workload]
    H, W, L, G = wl["H"], wl["W"], wl["L"], wl["G"]
    Ni = (H // 2) * (W // 2)
    cfg = af.Config.default(num_mmdit_layers=0, num_single_dit_layers=1, pos_embed_max_size=G * G)
    w = af.Weights(cfg, 0)
    make_weights(af, torch, w, args.seed, torch.device("cuda", 0))
    s = af.Scratch(w, 2, Ni, L)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(args.seed)
    lat = torch.randn(1, 4, H, W, generator=gen, device="cuda")
    text = torch.randn(2, L, 2048, generator=gen, device="cuda").to(torch.bfloat16)
    sig = af.sigma_schedule(N_SCHED, SHIFT)
    for i in range(args.warmup):
        af.denoise_step(w, s, lat, text, GUIDANCE, sig[i % N_SCHED], sig[i % N_SCHED + 1])
    s.sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        af.denoise_step(w, s, lat, text, GUIDANCE, sig[i % N_SCHED], sig[i % N_SCHED + 1])
    e1.record()
    s.sync()
    print(json.dumps({"case": "small_model", "tokens": 8 + L + Ni, "ms_per_step": e0.elapsed_time(e1) / args.steps,
                      "finite": bool(torch.isfinite(lat).all().item())}), flush=True)
    return 0


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.case == "single_block":
        return run_single_block_case(args)
    if args.case == "small_model":
        return run_small_model_case(args)
    # CPU baseline first (before any CUDA context), rank 0 at N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = WORKLOADS[args.workload]
        OracleBlockSample(wl["H"], wl["W"], wl["L"], args.seed, n_rows=512).run()   # page BLAS in
        sample = OracleBlockSample(wl["H"], wl["W"], wl["L"], args.seed)
        t, N = sample.run(), sample.N
        cpu = {"value": 1.0 / (36 * t), "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"one single DiT block of the workload (B=2, {N} tokens) in the fp64 numpy oracle, "
                         f"{t:.2f} s, scaled to a 36-block step; {cpu_model()}"}
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    line = run_af(args, rank, world, local_rank)
    if rank == 0:
        line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
