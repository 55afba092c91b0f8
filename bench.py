#!/usr/bin/env python
"""Benchmark of the fused FP8 ReLU^2 MLP block (fwd + bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload step16k]
                    [--impl ours|reference]

One step = one pass of the whole block over one batch of synthetic tokens:
fused up-projection (BF16 post + FP8 copy + partial amax), FP8
down-projection, the BF16 backward (dPre through sqrt(post), dX, dW1, dW2),
the partial-amax reduction with the delayed-scale update, and the W2 FP8
cache refresh.  Inputs are resident in HBM when the timed region starts; L2
is flushed (a 256 MiB write) between timed steps, outside the step's events.
Each timed step is one CUDA-graph replay whose event-record nodes mark the
step (on the launching stream); every fourth one also marks the dominant
kernel, whose duration the roofline object reports; a per-kernel breakdown
comes from separate untimed steps.  ``e2e`` repeats the measurement through the same public API
with the step's inputs copied in from pinned host memory and its results
(out, dX) copied back, inside the timed region.

On one GPU the default run (step16k) also runs the forward-only workload
(fwd16k, M=16384) and the training step at M=49152 (train49k) as child
processes with the same steps and warm-up, and nests their summaries in the
line's ``also`` object (``--no-also`` skips them).

Multi-GPU: one process per GPU under torchrun; ``--gpus N`` run without a
torchrun environment starts the N ranks itself (and ``--gpus N`` under a
different WORLD_SIZE is an error, so a scaling run cannot silently time one
GPU).  Every rank runs its own batch of M tokens (weak scaling): by default
the data-parallel step (partial amax all-reduced with MAX, dW1/dW2
all-reduced on a side stream beside dX), ``--replicas`` for independent
replicas; the time is the max over ranks.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only; other ranks exit 0).
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ReLU² MLP fwd+bwd tokens/s and % of FP8/BF16 roofline at d=768,h=3072"
FWD_METRIC = "ReLU² MLP fwd tokens/s and % of FP8/BF16 roofline at d=768,h=3072"
LINEAR_METRIC = "FP8 linear (attention QKV projection) fwd+bwd tokens/s and % of FP8/BF16 roofline"
CE_METRIC = "softcapped cross-entropy LM head fwd+bwd tokens/s and % of FP8/BF16 roofline at d=768,V=50304"
CE_CAP = 15.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="step16k",
                    choices=["step16k", "fwd16k", "train49k", "heavytail", "stack9", "qkv16k", "ce16k"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--eager", action="store_true", help="launch every call from the host instead of replaying a CUDA graph")
    ap.add_argument("--no-pdl", action="store_true", help="launch without programmatic dependent launch")
    ap.add_argument("--serial", action="store_true",
                    help="time the step with every kernel on one stream (default: the scale update and the "
                         "W2 cache refresh run on a second stream beside the GEMMs)")
    ap.add_argument("--fp8-up", action="store_true",
                    help="run the up-projection on e4m3 copies of x and W1 as well (x quantiser + W1 cache per step)")
    ap.add_argument("--compare-library", action="store_true",
                    help="time each GEMM of the step16k block against cuBLAS (torch.mm / torch._scaled_mm) on the "
                         "same shapes, one launch at a time with L2 flushed, and print one JSON line")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (small cases for profiling; not a bench line)")
    ap.add_argument("--bf16-head", action="store_true",
                    help="ce16k: BF16 logits instead of the e4m3 LM head")
    ap.add_argument("--shard-grads", action="store_true",
                    help="with N>1, reduce-scatter dW1/dW2 (each rank keeps h/N rows) instead of all-reducing them")
    ap.add_argument("--replicas", action="store_true",
                    help="with N>1, run independent replicas (no partial-amax / dW all-reduce)")
    ap.add_argument("--no-also", action="store_true",
                    help="step16k on one GPU: do not also run the fwd16k and train49k workloads (their summaries "
                         "go into the line's `also` object)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# peaks
# ---------------------------------------------------------------------------

# the dominant kernel of a training step is timed with events on every
# DOM_EVERY-th timed step (see run_ours)
DOM_EVERY = 4

# the B200's dense datasheet peaks: the step fractions are also reported
# against these (the measured-peak fractions are the primary ones)
SPEC_PEAKS = {"bf16_tflops": 2250.0, "fp8_tflops": 4500.0, "hbm_gbs": 8000.0}


def roofline_s(work, bf16_tf, fp8_tf, hbm_gbs, keys=None):
    """Roofline time of a step: the sum over its kernels of the slower of the
    tensor time (BF16 and FP8 FLOPs at their peaks) and the HBM time."""
    ks = list(work) if keys is None else keys
    return sum(max(work[k]["bf16"] / (bf16_tf * 1e12) + work[k]["fp8"] / (fp8_tf * 1e12),
                   work[k]["bytes"] / (hbm_gbs * 1e9)) for k in ks)


def spec_roofline(step_s, roof_fn, fwd_s=None, fwd_fn=None):
    """The step (and forward) roofline fractions against SPEC_PEAKS;
    roof_fn(bf16_tf, fp8_tf, hbm_gbs) -> seconds."""
    P = SPEC_PEAKS
    r = roof_fn(P["bf16_tflops"], P["fp8_tflops"], P["hbm_gbs"])
    out = {"roofline_ms": r * 1e3, "frac": r / step_s, "peaks": dict(P, source="B200 dense datasheet")}
    if fwd_fn is not None:
        rf = fwd_fn(P["bf16_tflops"], P["fp8_tflops"], P["hbm_gbs"])
        out.update(fwd_roofline_ms=rf * 1e3, fwd_frac=rf / fwd_s)
    return out


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def measure_fp8_peak(torch, bf16_peak):
    """Burst e4m3 GEMM throughput (8192^3, torch._scaled_mm) for the FP8
    roofline; falls back to 2x the BF16 peak (the nominal dense ratio)."""
    try:
        n = 8192
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = 1e30
        for _ in range(10):
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1) * 1e-3)
        del a, b
        return 2 * n ** 3 / best / 1e12, "measured (torch._scaled_mm e4m3 8192^3, best of 10)"
    except Exception as ex:  # pragma: no cover
        return 2 * bf16_peak, f"2x bf16 peak (nominal ratio; scaled_mm failed: {type(ex).__name__})"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polled from a thread)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = self.gpu = self.driver = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            name, drv = pynvml.nvmlDeviceGetName(self.h), pynvml.nvmlSystemGetDriverVersion()
            self.gpu = name.decode() if isinstance(name, bytes) else name
            self.driver = drv.decode() if isinstance(drv, bytes) else drv
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "gpu": self.gpu,
                "driver": self.driver}


# ---------------------------------------------------------------------------
# algorithmic work per kernel (per launch at M tokens)
# ---------------------------------------------------------------------------

def kernel_work(M, d, h):
    """FLOPs (by precision) and minimum HBM bytes of each kernel of a step."""
    F = 2 * M * d * h
    return {
        "up_fused": dict(bf16=F, fp8=0, bytes=2 * M * d + 2 * h * d + 2 * M * h + M * h),
        "down_fp8": dict(bf16=0, fp8=F, bytes=M * h + d * h + 2 * M * d),
        "bwd_dpre": dict(bf16=F, fp8=0, bytes=2 * M * d + 2 * h * d + 2 * M * h + 2 * M * h),
        "bwd_dx": dict(bf16=F, fp8=0, bytes=2 * M * h + 2 * h * d + 2 * M * d),
        "bwd_dw": dict(bf16=2 * F, fp8=0, bytes=2 * M * h + 2 * M * d + 2 * M * h + 2 * M * d + 8 * h * d),
        "amax_scale": dict(bf16=0, fp8=0, bytes=4 * (8 * -(-M // 256)) * (4 * -(-h // 256))),
        "w2_cache": dict(bf16=0, fp8=0, bytes=2 * (2 * h * d) + d * h),
    }


def src_digest():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "fp8_relu_mlp_b200", "csrc", "*"))):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def load_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    d = json.load(open(p))
    if d.get("src_digest") != src_digest():
        return {}
    return d.get("workloads", {}).get(workload, {})


# ---------------------------------------------------------------------------
# oracle on the host cores
# ---------------------------------------------------------------------------

def oracle_step_timer(W, tokens, seed=0, fp8_up=False):
    """Returns (fn running one oracle step on `tokens` tokens of the workload,
    threads used)."""
    import numpy as np
    from fp8_relu_mlp_b200 import synth
    from oracle import ref
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        threads = 1
    if W.name.startswith("ce"):
        # the LM head: logits, softcapped cross-entropy, its gradient and the
        # BF16 backward through the head (e4m3 logits from the oracle's copies)
        # The step refreshes the weight cache once per W.M tokens; a sampled
        # step of `tokens` tokens re-quantises the same share of W's rows.
        # The full e4m3 copy the logits need is built once, before timing.
        H = synth.make_head_problem(tokens, W.d, W.h, T=1, seed=seed)
        Wq, _, swi = ref.w1_cache(H["W"])
        share = max(1, (W.h * tokens) // W.M)

        def step():
            ref.w1_cache(H["W"][:share])
            xq, _ = ref.quantise_x(H["x"], np.float32(448.0 / 10.0))
            y = ref.head_logits_fp8(xq, Wq, np.float32(10.0 / 448.0), swi)
            f = ref.ce_forward(y, H["targets"], [1.0], CE_CAP)
            g = ref.ce_grad_scale(1.0, f["weight_sum"], True)
            ref.ce_backward(H["x"], H["W"], ref.ce_backward_dlogits(y, H["targets"], [1.0], CE_CAP, f["lse"], g))
            return np
        return step, threads
    if W.name.startswith("qkv"):
        P = synth.make_problem(tokens, W.d, W.h, seed=seed)
        g = synth.rng(5)
        dY = synth.to_bf16_bits(g.standard_normal((tokens, W.h), dtype=np.float32))
        st = {"s": ref.scale_state_init(W.margin, 1.0)}

        def step():
            xq, a = ref.quantise_x(P["x"], st["s"]["scale"])
            Wq, _, swi = ref.w1_cache(P["W1"])
            ref.linear_fp8(xq, Wq, st["s"]["scale_inv"], swi)
            st["s"] = ref.scale_update(st["s"], a)
            ref.linear_bwd(P["x"], P["W1"], dY)
            return np
        return step, threads
    if W.layers > 1:
        g = synth.rng(seed)
        r0 = synth.to_bf16_bits(synth.make_x(g, tokens, W.d, "normal"))
        dtop = synth.to_bf16_bits(synth.make_x(g, tokens, W.d, "normal"))
        Ps = [synth.make_problem(1, W.d, W.h, seed=l) for l in range(W.layers)]
        st = {"s": [ref.scale_state_init(W.margin, 1.0) for _ in range(W.layers)],
              "x": [ref.scale_state_init(W.margin, 1.0) for _ in range(W.layers)]}

        def step():
            layers = []
            for P in Ps:
                W2q_t, s_w, s_wi = ref.w2_cache(P["W2"])
                layers.append(dict(W1=P["W1"], W2=P["W2"], W2q_t=W2q_t, w2_scale_inv=s_wi))
                if fp8_up:
                    layers[-1]["W1q"], _, layers[-1]["w1_scale_inv"] = ref.w1_cache(P["W1"])
            scales = [(x["scale"], x["scale_inv"]) for x in st["s"]]
            if fp8_up:
                saved, _ = ref.stack_forward_fp8up(r0, layers, scales,
                                                   [(x["scale"], x["scale_inv"]) for x in st["x"]])
                st["x"] = [ref.scale_update(x, sv["x_amax"]) for x, sv in zip(st["x"], saved)]
            else:
                saved, _ = ref.stack_forward(r0, layers, scales)
            ref.stack_backward(saved, layers, dtop)
            st["s"] = [ref.scale_update(x, sv["amax"]) for x, sv in zip(st["s"], saved)]
            return np
        return step, threads
    P = synth.make_problem(tokens, W.d, W.h, seed=seed)
    st = {"s": ref.scale_state_init(W.margin, 1.0)}
    if not W.backward:
        W2q_t, _, s_wi = ref.w2_cache(P["W2"])

        def step():  # forward with the delayed scale, then the scale update
            f = ref.forward(P["x"], P["W1"], W2q_t, s_wi, st["s"]["scale"], st["s"]["scale_inv"])
            st["s"] = ref.scale_update(st["s"], f["amax"])
            return np
        return step, threads

    def step():
        W2q_t, s_w, s_wi = ref.w2_cache(P["W2"])
        f = ref.forward(P["x"], P["W1"], W2q_t, s_wi, st["s"]["scale"], st["s"]["scale_inv"])
        ref.backward(P["x"], P["W1"], P["W2"], f["post"], P["dOut"])
        st["s"] = ref.scale_update(st["s"], f["amax"])
        return np
    return step, threads


def oracle_tokens(W, kind):
    """Tokens per oracle step: about a second of host work per step."""
    if W.name.startswith("ce"):
        return 64
    if W.layers > 1:
        return 128 if kind == "baseline" else 32
    return 512 if kind == "baseline" else 256


def metric_of(W):
    if not W.backward:
        return FWD_METRIC
    if W.name.startswith("ce"):
        return CE_METRIC
    if W.name.startswith("qkv"):
        return LINEAR_METRIC
    return METRIC


def _time_steps(step, seconds, max_reps=50):
    t0 = time.perf_counter()
    reps = 0
    while True:
        step()
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= max_reps:
            return reps, el


def cpu_baseline(W, seconds, tokens=None, fp8_up=False):
    """The oracle on the host cores: all of them (the BLAS pool's threads),
    then one thread on a third of the budget."""
    tokens = tokens or oracle_tokens(W, "baseline")
    step, threads = oracle_step_timer(W, tokens, fp8_up=fp8_up)
    step()  # untimed: first-touch of the inputs and numpy's buffers
    reps, el = _time_steps(step, seconds)
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            r1, e1 = _time_steps(step, seconds / 3)
        single = {"value": tokens * r1 / e1, "unit": "tokens/s", "cores": 1, "sample": f"{r1} steps, {e1:.1f} s"}
    except Exception:  # pragma: no cover
        pass
    return {"value": tokens * reps / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "single_thread": single,
            "sample": ("each step also re-quantises its token share of the head's rows (weight cache); "
                       if W.name.startswith("ce") else "") +
                      f"{reps} oracle steps of {tokens} tokens of the {W.name} workload "
                      f"(d={W.d}, {'V' if W.name.startswith('ce') else 'h'}={W.h}, {W.layers} layer(s); "
                      f"the whole {'fwd+bwd' if W.backward else 'forward'} step), {el:.1f} s; "
                      f"tokens/s extrapolated from {tokens}-token steps to the workload's {W.M} tokens "
                      f"(the oracle's work is linear in the tokens)"}


def run_reference(a, W, world, rank):
    if rank != 0:
        return
    tokens = oracle_tokens(W, "reference")
    step, threads = oracle_step_timer(W, tokens)
    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    el = time.perf_counter() - t0
    v = tokens * a.steps / el
    sample = f"{a.steps} oracle steps of {tokens} tokens each (bounded sample of {W.name}: M={W.M}, d={W.d}, h={W.h})"
    if W.name.startswith("ce"):
        sample += (f"; each step also re-quantises {tokens}/{W.M} of the head's rows, its share of the "
                   f"once-per-step weight-cache refresh")
    line = {"metric": metric_of(W), "value": v, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": el / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (bf16/e4m3 rounding emulated)", "data": "synthetic",
            "config": config_of(W), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(W):
    return {"workload": f"{W.name}: {W.description}", "M_per_gpu": W.M, "d": W.d, "h": W.h,
            "x_dist": W.x_dist, "l2": "flushed (256 MiB write) between timed steps"}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def run_ours(a, W, world, rank, local_rank):
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)  # before the communicator binds a device
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.fp8mlp_set_programmatic_launch(not a.no_pdl)
    M, d, h = W.M, W.d, W.h
    peaks = load_peaks()
    fp8_peak, fp8_src = measure_fp8_peak(torch, peaks["bf16_tflops"])

    blk = MLPBlock(M, d, h, device=dev, margin=W.margin, fp8_up=a.fp8_up)
    P = synth.make_problem(M, d, h, seed=rank, x_dist=W.x_dist)
    blk.x.copy_(MLPBlock.bits_to_bf16(P["x"], dev))
    blk.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], dev))
    blk.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], dev))
    blk.dOut.copy_(MLPBlock.bits_to_bf16(P["dOut"], dev))
    blk.refresh_w2_cache()
    if a.fp8_up:
        blk.refresh_w1_cache()
    blk.calibrate()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = ["up_fused", "down_fp8", "bwd_dpre", "bwd_dx", "bwd_dw", "amax_scale", "w2_cache"]

    def step(ev=None):
        def mark(i):
            if ev is not None and ev[i] is not None:
                ev[i].record()  # the current stream: the capture stream while capturing
        mark(0)
        if a.fp8_up:
            blk._quantize_x()
            blk._up_fp8(0)
        else:
            A.fp8mlp_up_proj_fused(M, d, h, blk.x, blk.W1, blk.state, blk.post, blk.post_fp8, blk.partial_amax)
        mark(1)
        A.fp8mlp_down_proj_fp8(M, d, h, blk.post_fp8, blk.W2q_t, blk.w2_scale_inv, blk.state, blk.out)
        mark(2)
        A.fp8mlp_bwd_dpre(M, d, h, blk.dOut, blk.W2, blk.post, blk.dPre, A.LAUNCH_OVERLAP_PREVIOUS)
        mark(3)
        A.fp8mlp_bwd_dx(M, d, h, blk.dPre, blk.W1, blk.dX)
        mark(4)
        A.fp8mlp_bwd_dw(M, d, h, blk.x, blk.dPre, blk.post, blk.dOut, blk.dW1, blk.dW2, A.LAUNCH_OVERLAP_PREVIOUS)
        mark(5)
        blk.update_scale()
        mark(6)
        blk.refresh_w2_cache()
        if a.fp8_up:
            blk.refresh_w1_cache()
        mark(7)

    if world > 1 and not a.replicas:
        return run_dp(a, W, world, rank, local_rank, blk, flush, dist, peaks, fp8_peak, fp8_src, P)

    # one step = one CUDA-graph replay of the whole call sequence.  A first,
    # untimed pass with an event between every kernel gives the per-kernel
    # breakdown and picks the dominant kernel; the timed steps carry only four
    # events (start, around the dominant kernel, end) to keep event overhead
    # out of the measured step.
    step()
    torch.cuda.synchronize()

    side = torch.cuda.Stream(dev)

    def step_overlap(ev=None):
        # the same calls; the scale update and the W2 cache refresh on a
        # second stream beside the GEMMs (the refresh for this step's
        # down-projection moves to the start of the step)
        def mark(i):
            if ev is not None and ev[i] is not None:
                ev[i].record()
        blk.train_step_overlapped(side, mark=mark)

    def graph_of(marks, fn=step):
        evs = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(8)]
        want = set(marks)
        sub = [evs[i] if i in want else None for i in range(8)]
        g = None if a.eager else blk.capture(lambda: fn(sub))
        return g, evs

    def replay(g, evs, marks, fn=step):
        if g is not None:
            g.replay()
        else:
            fn([evs[i] if i in marks else None for i in range(8)])

    all_marks = list(range(8))
    g_all, ev_all = graph_of(all_marks)
    for _ in range(max(a.warmup, 3)):
        flush.zero_()
        replay(g_all, ev_all, all_marks)
    torch.cuda.synchronize()
    per_kernel = {n: [] for n in names}
    for _ in range(5):
        flush.zero_()
        replay(g_all, ev_all, all_marks)
        ev_all[7].synchronize()
        for k, n in enumerate(names):
            per_kernel[n].append(ev_all[k].elapsed_time(ev_all[k + 1]))
    breakdown = {n: statistics.median(v) for n, v in per_kernel.items()}
    dom_i = max(range(len(names)), key=lambda k: breakdown[names[k]])
    marks = [0, dom_i, dom_i + 1, 7]
    timed_fn = step if (a.serial or dom_i > 4) else step_overlap
    if timed_fn is step_overlap:
        step_overlap()
        torch.cuda.synchronize()
    # Two graphs of the same calls: one with events around the dominant kernel
    # and one with only the step's start and end events.  An event between
    # two kernels keeps the second from starting in the first one's last wave
    # (dW in dX's), which costs the step about 12 us, so the dominant kernel
    # is timed on every DOM_EVERY-th timed step (the first included) and the
    # other timed steps replay the graph without those two events.  Every one
    # of the K timed steps counts in `value`.
    marks_plain = [0, 7]
    n_cap0 = A.fp8mlp_kernel_launch_count()
    g_t, ev_t = graph_of(marks, timed_fn)
    kernels_per_step = A.fp8mlp_kernel_launch_count() - n_cap0 if g_t is not None else None
    g_p, ev_p = graph_of(marks_plain, timed_fn)
    for _ in range(2):
        for g_, e_, m_ in ((g_t, ev_t, marks), (g_p, ev_p, marks_plain)):
            flush.zero_()
            replay(g_, e_, m_, timed_fn)
    torch.cuda.synchronize()
    A.fp8mlp_clear_device_status()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = A.fp8mlp_kernel_launch_count()
    step_ms, dom_ms = [], []
    with ClockSampler(local_rank) as clk:
        for i in range(a.steps):
            flush.zero_()
            if i % DOM_EVERY == 0:
                replay(g_t, ev_t, marks, timed_fn)
                ev_t[7].synchronize()
                step_ms.append(ev_t[0].elapsed_time(ev_t[7]))
                dom_ms.append(ev_t[dom_i].elapsed_time(ev_t[dom_i + 1]))
            else:
                replay(g_p, ev_p, marks_plain, timed_fn)
                ev_p[7].synchronize()
                step_ms.append(ev_p[0].elapsed_time(ev_p[7]))
        torch.cuda.synchronize()
    launches = (A.fp8mlp_kernel_launch_count() - n0) if g_t is None else kernels_per_step * a.steps
    if dist:
        dist.barrier()
    status = A.fp8mlp_get_device_status()
    total_s = sum(step_ms) * 1e-3
    if dist:
        t = torch.tensor([total_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    value = M * world * a.steps / total_s

    # roofline of the dominant kernel (timed live inside the timed steps) and
    # of the whole step
    work = kernel_work(M, d, h)
    if a.fp8_up:
        F = 2 * M * d * h
        work["up_fused"] = dict(bf16=0, fp8=F, bytes=2 * M * d + M * d + M * d + h * d + 3 * M * h)
        work["w2_cache"]["bytes"] += 2 * (2 * h * d) + h * d
    avg = {n: v * 1e-3 for n, v in breakdown.items()}
    dom = names[dom_i]
    dom_s = statistics.mean(dom_ms) * 1e-3
    wd = work[dom]
    peak_dom = fp8_peak if wd["fp8"] else peaks["bf16_tflops"]
    achieved = (wd["bf16"] + wd["fp8"]) / dom_s / 1e12
    traffic = load_traffic(W.name).get(dom)
    roof_t = roofline_s(work, peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    fwd_s = avg["up_fused"] + avg["down_fp8"]

    def fwd_fn(pb, p8, bw):
        return sum(work[k]["bf16"] / (pb * 1e12) + work[k]["fp8"] / (p8 * 1e12) for k in ("up_fused", "down_fp8"))
    fwd_roof = fwd_fn(peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    spec = spec_roofline(total_s / a.steps, lambda pb, p8, bw: roofline_s(work, pb, p8, bw), fwd_s, fwd_fn)

    e2e = None
    if not a.no_e2e:
        e2e = measure_e2e(a, blk, P, torch, dev, stream, M, world, dist)
    schedule = None
    if W.spike_steps and rank == 0:
        schedule = spike_schedule(W, blk, P, torch, dev)

    line = None
    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+e4m3 (fp32 accumulate)",
            "data": "synthetic (seeded; shapes of the 768-dim GPT-2-small / nanochat MLP)",
            "config": dict(config_of(W), parallelism=f"dp{world} replicas" if world > 1 else "single GPU",
                           up_projection="e4m3 (x quantiser + W1 cache in the step)" if a.fp8_up else "bf16"),
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_dom,
                         "unit": "TFLOP/s", "frac": achieved / peak_dom, "traffic": traffic,
                         "peak_source": (fp8_src if wd["fp8"] else
                                         f"bf16_tflops burst of {peaks['source']} peaks"),
                         "timed_launches": len(dom_ms),
                         "timing": f"CUDA events around the kernel on every {DOM_EVERY}th timed step (the first "
                                   f"included); the other timed steps replay the same calls without those two "
                                   f"events, which would keep the kernel from starting in the previous one's "
                                   f"last wave"},
            "step_roofline": {"roofline_ms": roof_t * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof_t / (total_s / a.steps),
                              "fwd_ms": fwd_s * 1e3, "fwd_roofline_ms": fwd_roof * 1e3,
                              "fwd_frac": fwd_roof / fwd_s, "fwd_tokens_per_s": M / fwd_s,
                              "peaks": {"bf16_tflops": peaks["bf16_tflops"], "fp8_tflops": fp8_peak,
                                        "hbm_gbs": peaks["hbm_gbs"]}, "spec": spec},
            "kernels_ms": breakdown,
            "kernels_ms_note": "median of 5 untimed steps with an event between every kernel",
            "clocks": clocks, "gpu_launches": int(launches), "device_status": status,
            "launch_mode": ("eager" if g_t is None else "cuda_graph") + ("" if a.no_pdl else " + programmatic dependent launch")
                           + ("" if timed_fn is step else " + scale update and W2 cache on a second stream"),
        }
        if e2e:
            line["e2e"] = e2e
        if schedule:
            line["spike_schedule"] = schedule
        if not a.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(W, a.cpu_seconds)
        if (W.name == "step16k" and world == 1 and not a.no_also and not a.fp8_up and not a.serial
                and not a.eager and not a.no_pdl):
            line["also"] = also_workloads(a)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return line


def spike_schedule(W, blk, P, torch, dev):
    """Run the workload's step schedule (x doubled at the spike steps) and
    report, per step, the delayed scale used, the amax measured and the
    fraction of FP8 codes that saturated at +-448."""
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200.block import MLPBlock
    x0 = MLPBlock.bits_to_bf16(P["x"], dev)
    A.fp8mlp_scale_state_init(blk.state, W.margin, 1.0)
    blk.x.copy_(x0)
    blk.calibrate()
    steps = []
    for t in range(W.steps):
        blk.x.copy_(x0 * W.spike_factor if t in W.spike_steps else x0)
        s_used = blk.read_state()["scale"]
        blk.train_step()
        st = blk.read_state()
        sat = float(((blk.post_fp8 & 0x7F) == 0x7E).float().mean())
        steps.append({"step": t, "scale": s_used, "amax": st["amax_prev"], "saturated_frac": sat})
    return {"spike_steps": list(W.spike_steps), "x_factor": W.spike_factor, "steps": steps}


def run_dp(a, W, world, rank, local_rank, blk, flush, dist, peaks, fp8_peak, fp8_src, P=None):
    """Data-parallel training step on N ranks: each rank its own M tokens; the
    partial amax is all-reduced (MAX) and dW1/dW2 all-reduced (mean) over
    NCCL on a side stream that overlaps the dX GEMM (fp8_relu_mlp_b200.dp).
    Steps are issued eagerly; the time is the max over ranks."""
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200.dp import DataParallelStep
    M, d, h = W.M, W.d, W.h
    stepper = DataParallelStep(blk, shard_grads=a.shard_grads)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(max(a.warmup, 3)):
        flush.zero_()
        stepper()
    torch.cuda.synchronize()
    A.fp8mlp_clear_device_status()
    dist.barrier()
    torch.cuda.synchronize()
    step_ms, dom_ms = [], []
    n0 = A.fp8mlp_kernel_launch_count()
    with ClockSampler(local_rank) as clk:
        for _ in range(a.steps):
            flush.zero_()
            stepper(mark=lambda i: ev[i].record())
            ev[3].synchronize()
            step_ms.append(ev[0].elapsed_time(ev[3]))
            dom_ms.append(ev[1].elapsed_time(ev[2]))
    launches = A.fp8mlp_kernel_launch_count() - n0
    dist.barrier()
    status = A.fp8mlp_get_device_status()
    total_s = sum(step_ms) * 1e-3
    t = torch.tensor([total_s], device=blk.device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_s = float(t.item())
    value = M * world * a.steps / total_s
    work = kernel_work(M, d, h)
    dom_s = statistics.mean(dom_ms) * 1e-3
    achieved = work["bwd_dw"]["bf16"] / dom_s / 1e12
    e2e = None
    if not a.no_e2e and P is not None:
        e2e = measure_e2e(a, blk, P, torch, blk.device, None, M, world, dist, step_fn=stepper)
    roof_t = roofline_s(work, peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    spec = spec_roofline(total_s / a.steps, lambda pb, p8, bw: roofline_s(work, pb, p8, bw))
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+e4m3 (fp32 accumulate)",
            "data": "synthetic (seeded; shapes of the 768-dim GPT-2-small / nanochat MLP)",
            "config": dict(config_of(W), parallelism=f"dp{world}: NCCL all-reduce of partial amax (MAX) "
                                                     f"and {'reduce-scatter' if a.shard_grads else 'all-reduce'} "
                                                     f"of dW1/dW2 (mean), overlapped with dX"),
            "roofline": {"bound": "tensor", "kernel": "bwd_dw", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": load_traffic(W.name).get("bwd_dw"),
                         "peak_source": f"bf16_tflops burst of {peaks['source']} peaks"},
            "step_roofline": {"roofline_ms": roof_t * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof_t / (total_s / a.steps), "spec": spec},
            "clocks": clk.summary(), "gpu_launches": int(launches), "device_status": status,
            "launch_mode": "eager",
        }
        if e2e:
            line["e2e"] = e2e
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return None


def run_fwd(a, W, world, rank, local_rank):
    """The forward alone (inference with delayed scaling): per step the fused
    BF16 up-projection (post, its e4m3 copy, partial amax), the e4m3
    down-projection and the scale update for the next step; one CUDA graph
    per step.  The weights do not change, so the W2 cache is refreshed once."""
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)  # before the communicator binds a device
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.fp8mlp_set_programmatic_launch(not a.no_pdl)
    M, d, h = W.M, W.d, W.h
    peaks = load_peaks()
    fp8_peak, fp8_src = measure_fp8_peak(torch, peaks["bf16_tflops"])
    blk = MLPBlock(M, d, h, device=dev, margin=W.margin, with_backward=False)
    P = synth.make_problem(M, d, h, seed=rank, x_dist=W.x_dist)
    for k in ("x", "W1", "W2"):
        getattr(blk, k).copy_(MLPBlock.bits_to_bf16(P[k], dev))
    blk.refresh_w2_cache()
    blk.calibrate()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    npa = blk.partial_amax.numel()

    def step(ev=None, bufs=None, marks=(0, 1, 2, 3)):
        def mark(i):
            if ev is not None and i in marks:
                ev[i].record()
        xb, ob = bufs if bufs is not None else (blk.x, blk.out)
        mark(0)
        A.fp8mlp_up_proj_fused(M, d, h, xb, blk.W1, blk.state, blk.post, blk.post_fp8, blk.partial_amax)
        mark(1)
        A.fp8mlp_down_proj_fp8(M, d, h, blk.post_fp8, blk.W2q_t, blk.w2_scale_inv, blk.state, ob)
        mark(2)
        A.fp8mlp_amax_reduce_update_scale(blk.partial_amax, npa, blk.state)
        mark(3)

    step()
    torch.cuda.synchronize()
    # as in the training step: the events between the kernels (which time
    # the up-projection, the dominant kernel, and the down-projection) are in
    # every DOM_EVERY-th timed step; the others replay the same calls with
    # only the start and end events, so that each kernel may start while the
    # previous one finishes
    ev = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(4)]
    ev_p = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(4)]
    n_cap0 = A.fp8mlp_kernel_launch_count()
    graph = graph_p = None
    if not a.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(ev)
        graph_p = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_p):
            step(ev_p, marks=(0, 3))
    kps = (A.fp8mlp_kernel_launch_count() - n_cap0) // 2 if graph is not None else 3

    def run(timed=True):
        if timed:
            graph.replay() if graph is not None else step(ev)
        else:
            graph_p.replay() if graph_p is not None else step(ev_p, marks=(0, 3))

    for _ in range(max(a.warmup, 3)):
        for t_ in (True, False):
            flush.zero_()
            run(t_)
    torch.cuda.synchronize()
    A.fp8mlp_clear_device_status()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, up_ms, down_ms = [], [], []
    with ClockSampler(local_rank) as clk:
        for i in range(a.steps):
            flush.zero_()
            if i % DOM_EVERY == 0:
                run(True)
                ev[3].synchronize()
                step_ms.append(ev[0].elapsed_time(ev[3]))
                up_ms.append(ev[0].elapsed_time(ev[1]))
                down_ms.append(ev[1].elapsed_time(ev[2]))
            else:
                run(False)
                ev_p[3].synchronize()
                step_ms.append(ev_p[0].elapsed_time(ev_p[3]))
    status = A.fp8mlp_get_device_status()
    total_s = sum(step_ms) * 1e-3
    if dist:
        t = torch.tensor([total_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    work = kernel_work(M, d, h)
    up_s = statistics.mean(up_ms) * 1e-3
    achieved = work["up_fused"]["bf16"] / up_s / 1e12
    fwd_keys = ("up_fused", "down_fp8", "amax_scale")
    roof = roofline_s(work, peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"], fwd_keys)
    spec = spec_roofline(total_s / a.steps, lambda pb, p8, bw: roofline_s(work, pb, p8, bw, fwd_keys))
    e2e = None
    if not a.no_e2e:
        # x in from pinned host memory and out back, every step; copies
        # overlapped with the neighbouring steps (two device buffer sets)
        from fp8_relu_mlp_b200.hostio import HostPipeline
        xh = blk.x.cpu().pin_memory()
        oh = torch.empty_like(blk.out, device="cpu").pin_memory()
        sets = [(blk.x, blk.out), (blk.x.clone(), torch.empty_like(blk.out))]
        pipe = HostPipeline(lambda k: step(bufs=sets[k]), [[sb[0]] for sb in sets], [[sb[1]] for sb in sets],
                            device=dev, graph=not a.eager)
        pipe.run([xh], [oh], max(a.warmup, 3))
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        timer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        pipe.run([xh], [oh], a.steps, timer)
        timer[1].synchronize()
        te = timer[0].elapsed_time(timer[1]) * 1e-3
        if dist:
            tt = torch.tensor([te], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            te = float(tt.item())
        e2e = {"value": M * world * a.steps / te, "unit": "tokens/s",
               "h2d_bytes_per_step": int(2 * xh.numel()), "d2h_bytes_per_step": int(2 * oh.numel()),
               "overlap": "copies on two streams beside the compute, double-buffered device sets",
               "copy_bound": {"value": copy_bound(torch, dev, [xh], [oh], M * world), "unit": "tokens/s",
                              "note": "the same pinned copies alone, both directions at once (this rank's link)"}}
    if rank == 0:
        line = {
            "metric": FWD_METRIC,
            "value": M * world * a.steps / total_s, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup,
            "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 up-projection, e4m3 down-projection (fp32 accumulate)",
            "data": "synthetic (seeded; shapes of the 768-dim GPT-2-small / nanochat MLP)",
            "config": dict(config_of(W), parallelism=f"dp{world} replicas" if world > 1 else "single GPU"),
            "roofline": {"bound": "tensor", "kernel": "up_fused", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "timed_launches": len(up_ms),
                         "timing": f"CUDA events around the kernel on every {DOM_EVERY}th timed step (the first "
                                   f"included); the other timed steps replay the same calls without them",
                         "traffic": load_traffic(W.name).get("up_fused"),
                         "peak_source": "bf16_tflops burst of measured peaks"},
            "step_roofline": {"roofline_ms": roof * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof / (total_s / a.steps), "peaks": {**peaks, "fp8_tflops": fp8_peak},
                              "spec": spec},
            "kernels_ms": {"up_fused": statistics.median(up_ms), "down_fp8": statistics.median(down_ms)},
            "clocks": clk.summary(), "gpu_launches": int(kps * a.steps), "device_status": status,
            "launch_mode": "eager" if graph is None else "cuda_graph",
        }
        if e2e is not None:
            line["e2e"] = e2e
        if not a.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(W, a.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_linear(a, W, world, rank, local_rank):
    """The FP8 linear layer on the same kernels (attention QKV projection
    shape): per step the x quantiser, the e4m3 GEMM with its dequantising
    epilogue, the x-scale update, the weight-cache refresh and the BF16
    backward (dX, dW); one CUDA graph per step."""
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)  # before the communicator binds a device
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.fp8mlp_set_programmatic_launch(not a.no_pdl)
    M, K, N = W.M, W.d, W.h
    peaks = load_peaks()
    fp8_peak, fp8_src = measure_fp8_peak(torch, peaks["bf16_tflops"])
    P = synth.make_problem(M, K, N, seed=rank)
    bf, u8 = torch.bfloat16, torch.uint8
    x = MLPBlock.bits_to_bf16(P["x"], dev)
    Wt = MLPBlock.bits_to_bf16(P["W1"], dev)
    g = synth.rng(5)
    dY = MLPBlock.bits_to_bf16(synth.to_bf16_bits(g.standard_normal((M, N), dtype=np.float32)), dev)
    st = torch.zeros(8, device=dev)
    A.fp8mlp_scale_state_init(st, W.margin, 1.0)
    xq = torch.empty(M, K, dtype=u8, device=dev)
    npx = A.fp8mlp_x_partial_amax_count(M, K)
    pax = torch.empty(npx, device=dev)
    Wq = torch.empty(N, K, dtype=u8, device=dev)
    winv = torch.ones(4, device=dev)
    ws = torch.empty(A.fp8mlp_workspace_size(0, K, N), dtype=u8, device=dev)
    y = torch.empty(M, N, dtype=bf, device=dev)
    dX = torch.empty(M, K, dtype=bf, device=dev)
    dW = torch.empty(N, K, dtype=torch.float32, device=dev)
    wsl = torch.empty(max(16, A.fp8mlp_linear_bwd_workspace_size(M, K, N)), dtype=u8, device=dev)
    flush = torch.empty(256 << 20, dtype=u8, device=dev)
    A.fp8mlp_weight_fp8_cache_refresh(N, K, Wt, Wq, winv, ws)
    A.fp8mlp_quantize_x(M, K, x, st, xq, pax)
    A.fp8mlp_amax_reduce_update_scale(pax, npx, st)

    def step(ev=None, bufs=None, marks=(0, 1, 2, 3)):
        def mark(i):
            if ev is not None and i in marks:
                ev[i].record()
        xb, dYb, yb, dXb = bufs if bufs is not None else (x, dY, y, dX)
        mark(0)
        A.fp8mlp_quantize_x(M, K, xb, st, xq, pax)
        mark(1)
        A.fp8mlp_linear_fwd_fp8(M, K, N, xq, Wq, winv, st, yb)
        mark(2)
        A.fp8mlp_amax_reduce_update_scale(pax, npx, st)
        A.fp8mlp_linear_bwd(M, K, N, xb, Wt, dYb, dXb, dW, workspace=wsl)
        A.fp8mlp_weight_fp8_cache_refresh(N, K, Wt, Wq, winv, ws)
        mark(3)

    step()
    torch.cuda.synchronize()
    # the events around the forward GEMM (the dominant kernel) in every
    # DOM_EVERY-th timed step; the others replay the same calls with only the
    # start and end events (see run_ours)
    ev = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(4)]
    ev_p = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(4)]
    n_cap0 = A.fp8mlp_kernel_launch_count()
    graph = graph_p = None
    if not a.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(ev)
        graph_p = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_p):
            step(ev_p, marks=(0, 3))
        kps = (A.fp8mlp_kernel_launch_count() - n_cap0) // 2
    else:
        kps = A.fp8mlp_kernel_launch_count() - n_cap0

    def run(timed=True):
        if timed:
            graph.replay() if graph is not None else step(ev)
        else:
            graph_p.replay() if graph_p is not None else step(ev_p, marks=(0, 3))

    for _ in range(max(a.warmup, 3)):
        for t_ in (True, False):
            flush.zero_()
            run(t_)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, fwd_ms = [], []
    with ClockSampler(local_rank) as clk:
        for i in range(a.steps):
            flush.zero_()
            if i % DOM_EVERY == 0:
                run(True)
                ev[3].synchronize()
                step_ms.append(ev[0].elapsed_time(ev[3]))
                fwd_ms.append(ev[1].elapsed_time(ev[2]))
            else:
                run(False)
                ev_p[3].synchronize()
                step_ms.append(ev_p[0].elapsed_time(ev_p[3]))
    total_s = sum(step_ms) * 1e-3
    if dist:
        t = torch.tensor([total_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    F = 2 * M * K * N
    fwd_s = statistics.mean(fwd_ms) * 1e-3
    achieved = F / fwd_s / 1e12
    def roof_fn(pb, p8, bw):
        return F / (p8 * 1e12) + 2 * F / (pb * 1e12) + (2 * M * K + M * K) / (bw * 1e9)
    roof = roof_fn(peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    spec = spec_roofline(total_s / a.steps, roof_fn)
    e2e = None
    if not a.no_e2e:
        # x and the upstream gradient dY in from pinned host memory, y and dX
        # back, every step; copies overlapped with the neighbouring steps
        from fp8_relu_mlp_b200.hostio import HostPipeline
        xh, dyh = x.cpu().pin_memory(), dY.cpu().pin_memory()
        yh, dxh = torch.empty_like(y, device="cpu").pin_memory(), torch.empty_like(dX, device="cpu").pin_memory()
        sets = [(x, dY, y, dX), (x.clone(), dY.clone(), torch.empty_like(y), torch.empty_like(dX))]
        pipe = HostPipeline(lambda k: step(bufs=sets[k]), [[sb[0], sb[1]] for sb in sets],
                            [[sb[2], sb[3]] for sb in sets], device=dev, graph=not a.eager)
        pipe.run([xh, dyh], [yh, dxh], max(a.warmup, 3))
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        timer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        pipe.run([xh, dyh], [yh, dxh], a.steps, timer)
        timer[1].synchronize()
        te = timer[0].elapsed_time(timer[1]) * 1e-3
        if dist:
            tt = torch.tensor([te], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            te = float(tt.item())
        e2e = {"value": M * world * a.steps / te, "unit": "tokens/s",
               "h2d_bytes_per_step": int(2 * (xh.numel() + dyh.numel())),
               "d2h_bytes_per_step": int(2 * (yh.numel() + dxh.numel())),
               "overlap": "copies on two streams beside the compute, double-buffered device sets"}
    if rank == 0:
        line = {
            "metric": LINEAR_METRIC,
            "value": M * world * a.steps / total_s, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup,
            "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 forward, bf16 backward (fp32 accumulate)", "data": "synthetic",
            "config": dict(config_of(W), K=K, N=N, parallelism=f"dp{world} replicas" if world > 1 else "single GPU"),
            "roofline": {"bound": "tensor", "kernel": "linear_fwd_fp8", "achieved": achieved, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp8_peak,
                         "traffic": load_traffic(W.name).get("linear_fwd_fp8"), "peak_source": fp8_src,
                         "timed_launches": len(fwd_ms),
                         "timing": f"CUDA events around the kernel on every {DOM_EVERY}th timed step (the first "
                                   f"included); the other timed steps replay the same calls without them"},
            "step_roofline": {"roofline_ms": roof * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof / (total_s / a.steps), "spec": spec},
            "clocks": clk.summary(), "gpu_launches": int(kps * a.steps),
            "launch_mode": "eager" if graph is None else "cuda_graph",
        }
        if e2e:
            line["e2e"] = e2e
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_compare_library(a, W):
    """Each GEMM of the block next to cuBLAS on the same shapes and output
    types (torch.mm; torch._scaled_mm for the e4m3 down-projection): a
    reference for what a library GEMM with a plain store epilogue reaches at
    these sizes.  One launch at a time, L2 flushed before each, median of 11."""
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock
    dev = torch.device("cuda", 0)
    M, d, h = W.M, W.d, W.h
    blk = MLPBlock(M, d, h, device=dev, margin=W.margin)
    P = synth.make_problem(M, d, h, seed=0)
    for k in ("x", "W1", "W2", "dOut"):
        getattr(blk, k).copy_(MLPBlock.bits_to_bf16(P[k], dev))
    blk.refresh_w2_cache()
    blk.calibrate()
    blk.forward()
    blk.backward()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    one = torch.ones((), device=dev)
    W2q = blk.W2q_t  # [d, h] e4m3, K-major: the second operand of q . W2q^T
    ops = [
        ("up_fused (post, e4m3 copy, partial amax)", 1,
         lambda: A.fp8mlp_up_proj_fused(M, d, h, blk.x, blk.W1, blk.state, blk.post, blk.post_fp8,
                                        blk.partial_amax)),
        ("cuBLAS x . W1^T -> bf16 [M,h]", 1, lambda: torch.mm(blk.x, blk.W1.t())),
        ("down_fp8 (e4m3, scaled epilogue)", 1,
         lambda: A.fp8mlp_down_proj_fp8(M, d, h, blk.post_fp8, blk.W2q_t, blk.w2_scale_inv, blk.state, blk.out)),
        ("cuBLAS e4m3 q . W2q^T -> bf16 [M,d] (torch._scaled_mm)", 1,
         lambda: torch._scaled_mm(blk.post_fp8.view(torch.float8_e4m3fn), W2q.view(torch.float8_e4m3fn).t(),
                                  scale_a=one, scale_b=one, out_dtype=torch.bfloat16)),
        ("bwd_dpre (dPost GEMM + 2 sqrt(post) epilogue)", 1,
         lambda: A.fp8mlp_bwd_dpre(M, d, h, blk.dOut, blk.W2, blk.post, blk.dPre)),
        ("cuBLAS dOut . W2^T -> bf16 [M,h]", 1, lambda: torch.mm(blk.dOut, blk.W2.t())),
        ("bwd_dx", 1, lambda: A.fp8mlp_bwd_dx(M, d, h, blk.dPre, blk.W1, blk.dX)),
        ("cuBLAS dPre . W1 -> bf16 [M,d]", 1, lambda: torch.mm(blk.dPre, blk.W1)),
        ("bwd_dw (dW1 and dW2, fp32, one launch)", 2,
         lambda: A.fp8mlp_bwd_dw(M, d, h, blk.x, blk.dPre, blk.post, blk.dOut, blk.dW1, blk.dW2)),
        ("cuBLAS dPre^T . x -> fp32 [h,d] (dW1 only)", 1,
         lambda: torch.mm(blk.dPre.t(), blk.x, out_dtype=torch.float32)),
    ]
    F = 2 * M * d * h
    res = []
    for name, nF, f in ops:
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        ts = []
        for _ in range(11):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        us = float(np.median(ts)) * 1e3
        res.append({"gemm": name, "us": round(us, 1), "tflops": round(nF * F / us / 1e6, 1)})
    print(json.dumps({"compare_library": res, "config": config_of(W), "clocks_note": "single launches, L2 flushed",
                      "torch": torch.__version__}), flush=True)


def ce_work(M, d, V, fp8):
    """FLOPs (by precision) and minimum HBM bytes of each call of a head step."""
    F = 2 * M * d * V
    e = 1 if fp8 else 2
    nparts = 4 * -(-V // 256)  # partial sums per row: one per epilogue warp's 64 columns of a tile
    w = {
        "ce_fwd": dict(bf16=0 if fp8 else F, fp8=F if fp8 else 0,
                       bytes=e * M * d + e * V * d + 2 * 4 * nparts * M + 12 * M),
        "ce_bwd_dlogits": dict(bf16=0 if fp8 else F, fp8=F if fp8 else 0,
                               bytes=e * M * d + e * V * d + 8 * M + 2 * M * V),
        "dx": dict(bf16=F, fp8=0, bytes=2 * M * V + 2 * V * d + 2 * M * d),
        "dw": dict(bf16=F, fp8=0, bytes=2 * M * V + 2 * M * d + 4 * V * d),
    }
    if fp8:
        w["quantize_x"] = dict(bf16=0, fp8=0, bytes=3 * M * d)
        w["w_cache"] = dict(bf16=0, fp8=0, bytes=2 * (2 * V * d) + V * d)
    return w


def run_ce(a, W, world, rank, local_rank):
    """The softcapped cross-entropy LM head: per step (e4m3 head) the x
    quantiser, the fused head GEMM + cross-entropy, the x-scale update, the
    dlogits GEMM, dX and dW through the BF16 head, the weight-cache refresh;
    (BF16 head) the fused GEMM, dlogits, dX, dW.  Every rank runs its own
    tokens (weak scaling, no collective).  One CUDA graph per step."""
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)  # before the communicator binds a device
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.fp8mlp_set_programmatic_launch(not a.no_pdl)
    fp8 = not a.bf16_head
    M, d, V = W.M, W.d, W.h
    peaks = load_peaks()
    fp8_peak, fp8_src = measure_fp8_peak(torch, peaks["bf16_tflops"])
    H = synth.make_head_problem(M, d, V, T=1, seed=rank)
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    x = MLPBlock.bits_to_bf16(H["x"], dev)
    Wt = MLPBlock.bits_to_bf16(H["W"], dev)
    tg = torch.from_numpy(H["targets"]).to(dev)
    lse = torch.empty(M, device=dev)
    loss = torch.zeros(3, device=dev)
    ws = torch.empty(A.fp8mlp_ce_workspace_size(M, V, 1), dtype=u8, device=dev)
    dl = torch.empty(M, V, dtype=bf, device=dev)
    dX = torch.empty(M, d, dtype=bf, device=dev)
    dW = torch.empty(V, d, dtype=f32, device=dev)
    st = torch.zeros(8, device=dev)
    A.fp8mlp_scale_state_init(st, W.margin, 1.0)
    xq = torch.empty(M, d, dtype=u8, device=dev)
    npx = A.fp8mlp_x_partial_amax_count(M, d)
    pax = torch.empty(npx, device=dev)
    Wq = torch.empty(V, d, dtype=u8, device=dev)
    winv = torch.ones(4, device=dev)
    wsw = torch.empty(A.fp8mlp_workspace_size(0, d, V), dtype=u8, device=dev)
    flush = torch.empty(256 << 20, dtype=u8, device=dev)
    if fp8:
        # the delayed x-scale needs one step of history
        A.fp8mlp_weight_fp8_cache_refresh(V, d, Wt, Wq, winv, wsw)
        A.fp8mlp_quantize_x(M, d, x, st, xq, pax)
        A.fp8mlp_amax_reduce_update_scale(pax, npx, st)

    def make_calls(x, tg, dX, loss):
        """The step's calls on one set of input / result buffers."""
        calls = []
        if fp8:
            calls.append(("quantize_x", lambda: A.fp8mlp_quantize_x(M, d, x, st, xq, pax)))
            calls.append(("ce_fwd", lambda: A.fp8mlp_ce_fwd_fp8(M, d, V, 1, xq, st, Wq, winv, tg, None, CE_CAP, lse,
                                                                None, loss, ws)))
            calls.append(("ce_bwd_dlogits", lambda: A.fp8mlp_ce_bwd_dlogits_fp8(M, d, V, 1, xq, st, Wq, winv, tg,
                                                                                None, CE_CAP, lse, loss, None,
                                                                                A.CE_MEAN, dl)))
            calls.append(("x_scale", lambda: A.fp8mlp_amax_reduce_update_scale(pax, npx, st)))
        else:
            calls.append(("ce_fwd", lambda: A.fp8mlp_ce_fwd(M, d, V, 1, x, Wt, tg, None, CE_CAP, lse, None, loss,
                                                            ws)))
            calls.append(("ce_bwd_dlogits", lambda: A.fp8mlp_ce_bwd_dlogits(M, d, V, 1, x, Wt, tg, None, CE_CAP,
                                                                            lse, loss, None, A.CE_MEAN, dl)))
        # dX = dlogits . W is the same contraction as the MLP's dX = dPre . W1
        calls.append(("dx", lambda: A.fp8mlp_bwd_dx(M, d, V, dl, Wt, dX)))
        # dW does not depend on dX: it may start while the dX GEMM drains
        calls.append(("dw", lambda: A.fp8mlp_linear_bwd(M, d, V, x, Wt, dl, None, dW, A.LAUNCH_OVERLAP_PREVIOUS)))
        if fp8:
            calls.append(("w_cache", lambda: A.fp8mlp_weight_fp8_cache_refresh(V, d, Wt, Wq, winv, wsw)))
        return calls

    calls = make_calls(x, tg, dX, loss)
    names = [n for n, _ in calls]
    n_ev = len(calls) + 1

    def step(ev=None, marks=None):
        for i, (_, f) in enumerate(calls):
            if ev is not None and (marks is None or i in marks):
                ev[i].record()
            f()
        if ev is not None:
            ev[n_ev - 1].record()

    def graph_of(marks):
        ev = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(n_ev)]
        if a.eager:
            return None, ev
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(ev, marks)
        return g, ev

    def replay(g, ev, marks):
        if g is not None:
            g.replay()
        else:
            step(ev, marks)

    step()
    torch.cuda.synchronize()
    # untimed breakdown: an event between every call
    g_b, ev_b = graph_of(None)
    per = {n: [] for n in names}
    for _ in range(5):
        flush.zero_()
        replay(g_b, ev_b, None)
        ev_b[-1].synchronize()
        for i, n in enumerate(names):
            per[n].append(ev_b[i].elapsed_time(ev_b[i + 1]))
    breakdown = {n: statistics.median(v) for n, v in per.items()}
    dom_i = max(range(len(names)), key=lambda k: breakdown[names[k]])
    marks = {0, dom_i, dom_i + 1}
    n_cap0 = A.fp8mlp_kernel_launch_count()
    g_t, ev_t = graph_of(marks)
    kernels_per_step = A.fp8mlp_kernel_launch_count() - n_cap0
    for _ in range(max(a.warmup, 3)):
        flush.zero_()
        replay(g_t, ev_t, marks)
    torch.cuda.synchronize()
    A.fp8mlp_clear_device_status()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = A.fp8mlp_kernel_launch_count()
    step_ms, dom_ms = [], []
    with ClockSampler(local_rank) as clk:
        for _ in range(a.steps):
            flush.zero_()
            replay(g_t, ev_t, marks)
            ev_t[-1].synchronize()
            step_ms.append(ev_t[0].elapsed_time(ev_t[-1]))
            dom_ms.append(ev_t[dom_i].elapsed_time(ev_t[dom_i + 1]))
        torch.cuda.synchronize()
    launches = (A.fp8mlp_kernel_launch_count() - n0) if g_t is None else kernels_per_step * a.steps
    status = A.fp8mlp_get_device_status()
    total_s = sum(step_ms) * 1e-3
    if dist:
        t = torch.tensor([total_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    work = ce_work(M, d, V, fp8)
    dom = names[dom_i]
    wd = work.get(dom, dict(bf16=0, fp8=0, bytes=0))
    dom_s = statistics.mean(dom_ms) * 1e-3
    if wd["bf16"] or wd["fp8"]:
        peak_dom = fp8_peak if wd["fp8"] else peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "kernel": dom, "achieved": (wd["bf16"] + wd["fp8"]) / dom_s / 1e12,
                    "peak": peak_dom, "unit": "TFLOP/s", "traffic": load_traffic(W.name).get(dom),
                    "peak_source": fp8_src if wd["fp8"] else f"bf16_tflops burst of {peaks['source']} peaks"}
    else:
        roofline = {"bound": "hbm", "kernel": dom, "achieved": wd["bytes"] / dom_s / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "traffic": load_traffic(W.name).get(dom),
                    "peak_source": f"hbm_gbs of {peaks['source']} peaks"}
    roofline["frac"] = roofline["achieved"] / roofline["peak"]
    roof_t = roofline_s(work, peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    fwd_s = breakdown["ce_fwd"] * 1e-3
    wf = work["ce_fwd"]

    def fwd_fn(pb, p8, bw):
        return wf["bf16"] / (pb * 1e12) + wf["fp8"] / (p8 * 1e12)
    fwd_roof = fwd_fn(peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    spec = spec_roofline(total_s / a.steps, lambda pb, p8, bw: roofline_s(work, pb, p8, bw), fwd_s, fwd_fn)

    e2e = None
    if not a.no_e2e:
        # the same step through the public API with host buffers: x and the
        # targets come in from pinned host memory, the loss and dX go back,
        # every step; the copies overlap the neighbouring steps' compute
        # (two buffer sets, hostio.HostPipeline)
        from fp8_relu_mlp_b200.hostio import HostPipeline
        xh = torch.from_numpy(H["x"].view(np.int16)).view(bf).pin_memory()
        th = torch.from_numpy(H["targets"]).pin_memory()
        lh = torch.empty(3, dtype=f32).pin_memory()
        dxh = torch.empty(M, d, dtype=bf).pin_memory()
        sets = [dict(x=x, tg=tg, dX=dX, loss=loss),
                dict(x=x.clone(), tg=tg.clone(), dX=torch.empty_like(dX), loss=torch.zeros_like(loss))]
        set_calls = [make_calls(**sb) for sb in sets]

        def set_step(k):
            for _, f in set_calls[k]:
                f()

        pipe = HostPipeline(set_step, [[sb["x"], sb["tg"]] for sb in sets], [[sb["loss"], sb["dX"]] for sb in sets],
                            device=dev, graph=not a.eager)
        pipe.run([xh, th], [lh, dxh], max(a.warmup, 3))
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        timer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        pipe.run([xh, th], [lh, dxh], a.steps, timer)
        timer[1].synchronize()
        te = timer[0].elapsed_time(timer[1]) * 1e-3
        if dist:
            tt = torch.tensor([te], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            te = float(tt.item())
        e2e = {"value": M * world * a.steps / te, "unit": "tokens/s",
               "h2d_bytes_per_step": int(xh.numel() * 2 + th.numel() * 4),
               "d2h_bytes_per_step": int(lh.numel() * 4 + dxh.numel() * 2),
               "overlap": "copies on two streams beside the compute, double-buffered device sets"}
    if rank == 0:
        line = {
            "metric": CE_METRIC, "value": M * world * a.steps / total_s, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("e4m3 head forward" if fp8 else "bf16 head forward") + ", bf16 backward (fp32 accumulate)",
            "data": "synthetic (seeded; GPT-2 vocabulary padded to 50304, d=768)",
            "config": dict(config_of(W), V=V, softcap=CE_CAP, targets_per_token=1, reduction="mean",
                           head="e4m3 (x quantiser + weight cache in the step)" if fp8 else "bf16",
                           parallelism=f"dp{world} replicas" if world > 1 else "single GPU"),
            "roofline": roofline,
            "step_roofline": {"roofline_ms": roof_t * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof_t / (total_s / a.steps), "fwd_ms": fwd_s * 1e3,
                              "fwd_roofline_ms": fwd_roof * 1e3, "fwd_frac": fwd_roof / fwd_s,
                              "peaks": {"bf16_tflops": peaks["bf16_tflops"], "fp8_tflops": fp8_peak,
                                        "hbm_gbs": peaks["hbm_gbs"]}, "spec": spec},
            "kernels_ms": breakdown,
            "kernels_ms_note": "median of 5 untimed steps with an event between every call; ce_fwd includes "
                               "its two small reduction kernels",
            "clocks": clk.summary(), "gpu_launches": int(launches), "device_status": status,
            "launch_mode": ("eager" if g_t is None else "cuda_graph") + ("" if a.no_pdl else " + programmatic dependent launch"),
        }
        if e2e:
            line["e2e"] = e2e
        if not a.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(W, a.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_stack(a, W, world, rank, local_rank):
    """The 9-layer stack workload: per step, forward through every layer
    (RMSNorm, block, residual), backward through every layer, the scale
    updates and the W2 cache refreshes, replayed as one CUDA graph."""
    import numpy as np
    import torch
    from fp8_relu_mlp_b200 import _abi as A
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock, MLPStack

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)  # before the communicator binds a device
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.fp8mlp_set_programmatic_launch(not a.no_pdl)
    L, M, d, h = W.layers, W.M, W.d, W.h
    peaks = load_peaks()
    fp8_peak, fp8_src = measure_fp8_peak(torch, peaks["bf16_tflops"])
    S = MLPStack(L, M, d, h, device=dev, margin=W.margin, fp8_up=a.fp8_up)
    g = synth.rng(1000 + rank)
    r0 = synth.to_bf16_bits(synth.make_x(g, M, d, "normal"))
    dtop = synth.to_bf16_bits(synth.make_x(g, M, d, "normal"))
    for l, b in enumerate(S.blocks):
        P = synth.make_problem(1, d, h, seed=100 * rank + l)
        b.W1.copy_(MLPBlock.bits_to_bf16(P["W1"], dev))
        b.W2.copy_(MLPBlock.bits_to_bf16(P["W2"], dev))
    S.r[0].copy_(MLPBlock.bits_to_bf16(r0, dev))
    io = {"dtop": MLPBlock.bits_to_bf16(dtop, dev)}  # dL/dr_L of the step (an input, like r_0)
    S.refresh_w2_caches()
    S.calibrate()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    last = S.blocks[L - 1]

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record()
        mark(0)
        S.forward()
        S.dr.copy_(io["dtop"])
        # backward of the top layer, with its dW launch marked
        A.fp8mlp_bwd_dpre(M, d, h, S.dr, last.W2, last.post, last.dPre)
        A.fp8mlp_bwd_dx(M, d, h, last.dPre, last.W1, last.dX)
        mark(1)
        A.fp8mlp_bwd_dw(M, d, h, last.x, last.dPre, last.post, S.dr, last.dW1, last.dW2)
        mark(2)
        A.fp8mlp_rmsnorm_bwd(M, d, S.r[L - 1], S.rstd[L - 1], last.dX, S.dr, S.dr)
        for l in range(L - 2, -1, -1):
            b = S.blocks[l]
            A.fp8mlp_mlp_bwd(M, d, h, b.x, b.W1, b.W2, b.post, S.dr, b.dPre, b.dX, b.dW1, b.dW2)
            A.fp8mlp_rmsnorm_bwd(M, d, S.r[l], S.rstd[l], b.dX, S.dr, S.dr)
        S.update_scales()
        S.refresh_w2_caches()
        mark(3)

    step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True, external=not a.eager) for _ in range(4)]
    n_cap0 = A.fp8mlp_kernel_launch_count()
    graph = None if a.eager else S.blocks[0].capture(lambda: step(ev))
    kernels_per_step = A.fp8mlp_kernel_launch_count() - n_cap0

    def run():
        if graph is not None:
            graph.replay()
        else:
            step(ev)

    for _ in range(max(a.warmup, 3)):
        flush.zero_()
        run()
    torch.cuda.synchronize()
    A.fp8mlp_clear_device_status()
    if dist:
        dist.barrier()
    step_ms, dom_ms = [], []
    n0 = A.fp8mlp_kernel_launch_count()
    with ClockSampler(local_rank) as clk:
        for _ in range(a.steps):
            flush.zero_()
            run()
            ev[3].synchronize()
            step_ms.append(ev[0].elapsed_time(ev[3]))
            dom_ms.append(ev[1].elapsed_time(ev[2]))
    launches = kernels_per_step * a.steps if graph is not None else A.fp8mlp_kernel_launch_count() - n0
    status = A.fp8mlp_get_device_status()
    total_s = sum(step_ms) * 1e-3
    if dist:
        t = torch.tensor([total_s], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    value = M * world * a.steps / total_s
    work = kernel_work(M, d, h)
    # per layer: the five GEMMs and the small kernels, plus RMSNorm fwd (read r,
    # write x), residual add (read r, out; write r'), RMSNorm bwd (read r, dX,
    # dr; write dr) and the dr copy
    norm_bytes = (2 + 3 + 4) * 2 * M * d
    if a.fp8_up:
        # e4m3 up-projection (x and W1 copies); the RMSNorm also writes x's
        # copy; the W1 cache is refreshed every step
        F = 2 * M * d * h
        work["up_fused"] = dict(bf16=0, fp8=F, bytes=M * d + h * d + 3 * M * h)
        work["w2_cache"]["bytes"] += 2 * (2 * h * d) + h * d
        norm_bytes += M * d
    def roof_fn(pb, p8, bw):
        return L * (roofline_s(work, pb, p8, bw) + norm_bytes / (bw * 1e9)) + 4 * M * d / (bw * 1e9)
    roof_t = roof_fn(peaks["bf16_tflops"], fp8_peak, peaks["hbm_gbs"])
    dom_s = statistics.mean(dom_ms) * 1e-3
    achieved = work["bwd_dw"]["bf16"] / dom_s / 1e12
    # a step of tens of milliseconds runs under the power cap: the kernel is
    # compared with the sustained BF16 figure
    peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    e2e = None
    if not a.no_e2e:
        # r_0 and dL/dr_L in from pinned host memory, r_L and dL/dr_0 back,
        # every step; copies overlapped with the neighbouring steps
        # (hostio.HostPipeline over two sets of those four buffers)
        from fp8_relu_mlp_b200.hostio import HostPipeline
        r0h = torch.from_numpy(r0.view(np.int16)).view(torch.bfloat16).pin_memory()
        dth = torch.from_numpy(dtop.view(np.int16)).view(torch.bfloat16).pin_memory()
        rLh = torch.empty(M, d, dtype=torch.bfloat16).pin_memory()
        dr0h = torch.empty(M, d, dtype=torch.bfloat16).pin_memory()
        sets = [dict(r0=S.r[0], dtop=io["dtop"], rL=S.r[L], dr=S.dr)]
        sets.append({k: v.clone() for k, v in sets[0].items()})

        def set_step(k):
            S.r[0], io["dtop"], S.r[L], S.dr = sets[k]["r0"], sets[k]["dtop"], sets[k]["rL"], sets[k]["dr"]
            step()

        pipe = HostPipeline(set_step, [[sb["r0"], sb["dtop"]] for sb in sets], [[sb["rL"], sb["dr"]] for sb in sets],
                            device=dev, graph=not a.eager)
        S.r[0], io["dtop"], S.r[L], S.dr = sets[0]["r0"], sets[0]["dtop"], sets[0]["rL"], sets[0]["dr"]
        pipe.run([r0h, dth], [rLh, dr0h], 2)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        timer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        pipe.run([r0h, dth], [rLh, dr0h], a.steps, timer)
        timer[1].synchronize()
        t2 = timer[0].elapsed_time(timer[1]) * 1e-3
        if dist:
            tt = torch.tensor([t2], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            t2 = float(tt.item())
        e2e = {"value": M * world * a.steps / t2, "unit": "tokens/s", "h2d_bytes_per_step": 4 * M * d,
               "d2h_bytes_per_step": 4 * M * d,
               "overlap": "copies on two streams beside the compute, double-buffered device sets"}
    if rank == 0:
        traffic = load_traffic(W.name).get("bwd_dw")
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": total_s / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+e4m3 (fp32 accumulate)",
            "data": "synthetic (seeded; 9-layer 768-dim ReLU^2 stack of the nanochat runs)",
            "config": dict(config_of(W), layers=L, parallelism=f"dp{world} replicas" if world > 1 else "single GPU",
                           up_projection="e4m3 (x quantised in the RMSNorm kernel, W1 cache in the step)"
                           if a.fp8_up else "bf16"),
            "roofline": {"bound": "tensor", "kernel": "bwd_dw (top layer)", "achieved": achieved,
                         "peak": peak_sus, "unit": "TFLOP/s", "frac": achieved / peak_sus,
                         "traffic": traffic,
                         "peak_source": f"bf16_tflops_sustained of {peaks['source']} peaks (long step, power cap)"},
            "step_roofline": {"roofline_ms": roof_t * 1e3, "measured_ms": total_s / a.steps * 1e3,
                              "frac": roof_t / (total_s / a.steps),
                              "peaks": {"bf16_tflops": peaks["bf16_tflops"], "fp8_tflops": fp8_peak,
                                        "hbm_gbs": peaks["hbm_gbs"]},
                              "spec": spec_roofline(total_s / a.steps, roof_fn)},
            "clocks": clk.summary(), "gpu_launches": int(launches), "device_status": status,
            "launch_mode": "eager" if graph is None else "cuda_graph",
        }
        if e2e:
            line["e2e"] = e2e
        if not a.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(W, a.cpu_seconds, fp8_up=a.fp8_up)
        print(json.dumps(line), flush=True)
    if dist:
        del graph
        dist.barrier()
        dist.destroy_process_group()


def copy_bound(torch, dev, host_in, host_out, tokens, reps=5):
    """Tokens/s if a step were nothing but its copies: the same pinned host
    tensors copied in (host to device) and out (device to host) at once on
    two streams, as the pipelined end-to-end step overlaps them."""
    din = [torch.empty_like(h, device=dev) for h in host_in]
    dout = [torch.empty_like(h, device=dev) for h in host_out]
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)

    def once():
        with torch.cuda.stream(s1):
            for h, d in zip(host_in, din):
                d.copy_(h, non_blocking=True)
        with torch.cuda.stream(s2):
            for h, d in zip(host_out, dout):
                h.copy_(d, non_blocking=True)

    s1.wait_stream(cur)
    s2.wait_stream(cur)
    once()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    s1.wait_stream(cur)
    s2.wait_stream(cur)
    for _ in range(reps):
        once()
    cur.wait_stream(s1)
    cur.wait_stream(s2)
    e1.record(cur)
    e1.synchronize()
    return tokens * reps / (e0.elapsed_time(e1) * 1e-3)


def measure_e2e(a, blk, P, torch, dev, stream, M, world, dist, step_fn=None):
    """Same step through the public API with host buffers: every step's
    inputs (x, dOut) come from pinned host memory and its results (out, dX)
    go back to pinned host memory inside the timed region.  The copies run
    on their own streams, overlapped with the neighbouring steps' compute
    (``hostio.block_pipeline``: two device buffer sets, one CUDA graph each;
    ``step_fn``, the data-parallel step, is launched eagerly)."""
    import numpy as np
    from fp8_relu_mlp_b200.hostio import block_pipeline
    xh = torch.from_numpy(P["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    gh = torch.from_numpy(P["dOut"].view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty_like(blk.out, device="cpu").pin_memory()
    dxh = torch.empty_like(blk.dX, device="cpu").pin_memory()
    side = torch.cuda.Stream(dev)
    pipe = block_pipeline(blk, side, graph=not a.eager and step_fn is None, step_fn=step_fn)
    pipe.run([xh, gh], [oh, dxh], max(a.warmup, 3))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    timer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    pipe.run([xh, gh], [oh, dxh], a.steps, timer)
    timer[1].synchronize()
    t = timer[0].elapsed_time(timer[1]) * 1e-3
    if dist:
        tt = torch.tensor([t], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t = float(tt.item())
    cb = copy_bound(torch, dev, [xh, gh], [oh, dxh], M * world)
    return {"value": M * world * a.steps / t, "unit": "tokens/s",
            "h2d_bytes_per_step": int(xh.numel() * 2 + gh.numel() * 2),
            "d2h_bytes_per_step": int(oh.numel() * 2 + dxh.numel() * 2),
            "overlap": "copies on two streams beside the compute, double-buffered device sets",
            "copy_bound": {"value": cb, "unit": "tokens/s",
                           "note": "the same pinned copies alone, both directions at once (this rank's link)"}}


def also_workloads(a):
    """The other two MLP workloads of the benchmark suite, each run as a
    child process of this command on the same GPU with the same steps and
    warm-up (the forward alone at M=16384; the training step at M=49152),
    summarised for the default line's `also` object."""
    import subprocess
    out = {}
    for wl in ("fwd16k", "train49k"):
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", wl, "--steps", str(a.steps), "--warmup",
               str(a.warmup), "--no-cpu-baseline", "--no-also"] + (["--no-e2e"] if a.no_e2e else [])
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
            lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
            if r.returncode != 0 or not lines:
                out[wl] = {"error": f"exit {r.returncode}: {r.stderr.strip()[-300:]}"}
                continue
            d = json.loads(lines[-1])
            sr = d.get("step_roofline", {})
            out[wl] = {"metric": d["metric"], "value": d["value"], "unit": d["unit"], "ms_per_step": d["ms_per_step"],
                       "steps": d["steps"], "warmup": d["warmup"], "config": d["config"]["workload"],
                       "step_roofline_frac": sr.get("frac"), "step_roofline_frac_spec": sr.get("spec", {}).get("frac"),
                       "roofline": d.get("roofline"), "e2e": (d.get("e2e") or {}).get("value"),
                       "clocks": d.get("clocks"), "gpu_launches": d.get("gpu_launches"),
                       "device_status": d.get("device_status")}
        except Exception as ex:  # pragma: no cover
            out[wl] = {"error": f"{type(ex).__name__}: {ex}"}
    return out


def relaunch(n):
    """--gpus N > 1 outside a torchrun environment: start N ranks of this same
    command, one process per GPU on this node, rendezvous on 127.0.0.1, and
    return the exit status of the launcher (non-zero if any rank failed)."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def main():
    a = parse()
    from fp8_relu_mlp_b200 import synth
    W = synth.WORKLOADS[a.workload]
    if a.tokens:
        # a smaller case of the same workload (ncu captures); the committed
        # traffic figures are per full-size launch, so they are not looked up
        import dataclasses
        W = dataclasses.replace(W, M=a.tokens, name=f"{W.name}@{a.tokens}")
    if "WORLD_SIZE" not in os.environ and a.gpus > 1:
        return relaunch(a.gpus)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != a.gpus:
        print(f"bench.py: --gpus {a.gpus} but WORLD_SIZE={world}: launch one rank per GPU "
              f"(torchrun --nproc-per-node {a.gpus}), or run without WORLD_SIZE set and bench.py starts them",
              file=sys.stderr, flush=True)
        return 2
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, W, world, rank)
        return 0
    if a.compare_library:
        if rank == 0:
            run_compare_library(a, W)
        return 0
    if not W.backward:
        run_fwd(a, W, world, rank, local_rank)
    elif W.name.startswith("qkv"):
        run_linear(a, W, world, rank, local_rank)
    elif W.name.startswith("ce"):
        run_ce(a, W, world, rank, local_rank)
    elif W.layers > 1:
        run_stack(a, W, world, rank, local_rank)
    else:
        run_ours(a, W, world, rank, local_rank)
    return 0


if __name__ == "__main__":
    sys.exit(main())
