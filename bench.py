"""Benchmark of the NF4 / double-quant / QLoRA-linear hot path on B200.

One step = one pass of the whole path over the LLaMA-7B-shaped layer set
(q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008; 2048 tokens, r=64,
alpha=16): for every matrix, quantize + double-quantize the bf16 weight,
dequantize it to bf16, QLoRA forward (Y, T) and backward (dX, dA, dB).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` = fwd+bwd algorithmic TFLOP/s of the
whole step (quantize and dequantize time included in the denominator),
summed over ranks.  The step's working set (~1.3 GB) is far larger than the
126 MB L2, so no flush is needed between steps.

`components` (one GPU) time each kernel family on its own, with CUDA events,
inputs out of L2 (rotation over buffer sets larger than twice the L2, or an L2
flush before each call), medians:
  quantize / dequant   the 7 weights of the 7B set, GB/s
  fwd / bwd            the step's qlora_linear calls, TFLOP/s
  decode               28672x8192 and 8192x28672 at M in {1,4,16}, GB/s
  llama70b             whole-model (80 layers) quantize and dequantize GB/s;
                       fwd+bwd TFLOP/s at 512 tokens on the 7 layer shapes
  robust               4095x11007 at 4096 tokens, r=8: quantize, dequantize,
                       fwd, bwd
  merge                LoRA merge (r=64) of the 7 weights, GB/s
  f16                  the FP16 compute type: fwd+bwd on q, gate, down
  variants             quantize / dequantize GB/s of the storage variants
N > 1 runs data-parallel replicas (weak scaling: 2048 tokens per rank); the
step's one exchange is an NCCL all-reduce of every matrix's dA and dB, held
in one flat bucket.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_nf4_quantized_12_b200 import workloads  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ algorithmic work
def quant_bytes(N, K):
    numel = N * K
    nb = (numel + 63) // 64
    return 2 * numel + (numel + 1) // 2 + nb + 4 * ((nb + 255) // 256)


def fwd_flops(M, N, K, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


def bwd_flops(M, N, K, r):
    return 2 * M * N * K + 4 * M * N * r + 4 * M * K * r


# ncu dram__bytes_read.sum + dram__bytes_write.sum of the forward fused GEMM on the
# 4096x4096 weight at 2048 tokens (profiles/nf4_gemm_4096x4096_2048tok.md), mean
# of two launches, taken on the kernel as built
GEMM_FWD_Q_DRAM_BYTES = (26550784 + 0 + 26549504 + 0) // 2
GEMM_FWD_Q_DRAM_CASE = ("nf4_gemm_kernel<0,0>, 4096x4096 weight, 2048 tokens, r=64: ncu dram__bytes_read.sum + "
                        "dram__bytes_write.sum per launch, mean of two launches (algorithmic reads 26.47 MB; the "
                        "16.8 MB output stays in L2 within the capture)")


def decode_bytes(M, N, K, r):
    numel = N * K
    nb = (numel + 63) // 64
    return (numel + 1) // 2 + nb + 4 * ((nb + 255) // 256) + 2 * M * K + 2 * M * N + 2 * r * (K + N)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ our arm
class Step:
    """All buffers of one step over the 7B layer set, resident on the GPU."""

    def __init__(self, device, wl, host_copy=False, world=1):
        from bit_nf4_quantized_12_b200 import binding, dp
        self.b = binding
        self.dp = dp
        self.wl = wl
        self.dev = device
        self.world = world
        self.mats = []
        M, r = wl.tokens, wl.r
        # dA, dB of all 7 matrices live in one flat bucket: with N ranks the
        # step ends with one all-reduce of it (data-parallel replicas)
        self.bucket = dp.GradBucket.for_layers([(K, N, r) for _, N, K in wl.mats], device)
        for idx, (name, N, K) in enumerate(wl.mats):
            seed = workloads.matrix_seed(wl.name, 0, idx)
            d = dict(name=name, N=N, K=K)
            d["W"] = workloads.weight(N, K, wl.w_std, seed=seed, device=device)
            d.update(workloads.layer_inputs(M, N, K, r, seed=seed, device=device))
            d["qw"] = binding.empty_quantized(N, K, device)
            d["Wd"] = torch.empty(N, K, dtype=torch.bfloat16, device=device)
            d["Y"] = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            d["T"] = torch.empty(M, r, dtype=torch.bfloat16, device=device)
            d["dX"] = torch.empty(M, K, dtype=torch.bfloat16, device=device)
            d["dA"], d["dB"] = self.bucket.views[idx]
            d["ws"] = binding.workspace(M, N, K, r, device)
            if host_copy:
                d["host"] = {k: d[k].cpu().pin_memory() for k in ("W", "X", "dY", "A", "B")}
                d["host_out"] = {k: torch.empty(d[k].shape, dtype=d[k].dtype).pin_memory()
                                 for k in ("Y", "dX", "dA", "dB")}
            self.mats.append(d)
        self.launches_per_step = 7 * (1 + 1 + 2 + 4)

    def run(self, events=None):
        b, wl = self.b, self.wl
        for d in self.mats:
            if events is not None:
                events["q"][0].append(_ev())
            b.quantize(d["W"], out=d["qw"])
            if events is not None:
                events["q"][1].append(_ev())
                events["dq"][0].append(_ev())
            b.dequant(d["qw"], out=d["Wd"])
            if events is not None:
                events["dq"][1].append(_ev())
                events["fwd"][0].append(_ev())
            b.linear_fwd(d["X"], d["qw"], d["A"], d["B"], wl.s, ws=d["ws"], Y=d["Y"], T=d["T"])
            if events is not None:
                events["fwd"][1].append(_ev())
                events["bwd"][0].append(_ev())
            b.linear_bwd(d["dY"], d["X"], d["qw"], d["A"], d["B"], wl.s, T=d["T"], ws=d["ws"], dX=d["dX"],
                         dA=d["dA"], dB=d["dB"])
            if events is not None:
                events["bwd"][1].append(_ev())
        if self.world > 1:   # the one exchange step: global dA, dB over the replicas' tokens
            self.dp.allreduce_lora_grads([self.bucket.flat])

    def run_e2e(self):
        """Same step through the public API with host buffers: H2D inputs,
        compute, D2H of the step's results (Y, dX, dA, dB)."""
        for d in self.mats:
            for k, h in d["host"].items():
                d[k].copy_(h, non_blocking=True)
        self.run()
        for d in self.mats:
            for k, h in d["host_out"].items():
                h.copy_(d[k], non_blocking=True)

    def e2e_bytes(self):
        h2d = sum(t.numel() * t.element_size() for d in self.mats for t in d["host"].values())
        d2h = sum(t.numel() * t.element_size() for d in self.mats for t in d["host_out"].values())
        return h2d, d2h


def _ev():
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def _pair_ms(starts, ends):
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def decode_component(device, peaks):
    """Decode (the forward with 1-16 tokens: the dequant-fused decode kernel,
    r=16) on 28672x8192 and 8192x28672 at M in {1,4,16}: each call timed
    alone with CUDA events, L2 flushed before it, median of 10."""
    from bit_nf4_quantized_12_b200 import binding
    wl = workloads.WORKLOADS["decode"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    res = {}
    for (name, N, K) in wl.mats:
        W = workloads.weight(N, K, wl.w_std, seed=0, device=device)
        qw = binding.quantize(W)
        del W
        for M in wl.decode_m:
            io = workloads.layer_inputs(M, N, K, wl.r, seed=1, device=device)
            ws = binding.workspace(M, N, K, wl.r, device)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            T = torch.empty(M, wl.r, dtype=torch.bfloat16, device=device)
            times = []
            for it in range(13):
                flush.zero_()
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                _gpu_ahead()
                s.record()
                binding.linear_fwd(io["X"], qw, io["A"], io["B"], wl.s, ws=ws, Y=Y, T=T)
                e.record()
                torch.cuda.synchronize()
                if it >= 3:
                    times.append(s.elapsed_time(e))
            ms = statistics.median(times)
            gbs = decode_bytes(M, N, K, wl.r) / (ms * 1e-3) / 1e9
            res[f"{N}x{K}_m{M}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                     "frac": round(gbs / peaks["hbm_gbs"], 3)}
        del qw
    return res


def _gpu_ahead():
    """Queue ~0.1 ms of GPU spinning before a timed call, so that the host has
    enqueued the whole call (binding, argument checks, launches) before the
    GPU reaches its start event: the events then bracket GPU time only, not
    the host's launch overhead."""
    torch.cuda._sleep(200_000)


def _median_ms(fn, reps, flush=None, warm=3):
    """Median CUDA-event time of fn() over reps calls (after warm calls),
    with flush() (untimed) before each call when given."""
    times = []
    for it in range(warm + reps):
        if flush is not None:
            flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _gpu_ahead()
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        if it >= warm:
            times.append(s.elapsed_time(e))
    return statistics.median(times)


def bandwidth_component(step, peaks, rounds=50):
    """Quantize, dequantize and LoRA merge (r=64) of the 7 LLaMA-7B-shaped
    weights, each call timed alone with CUDA events.  The calls rotate over the 7 weights (404 MB
    of bf16 W, 101 MB of NF4 storage, 404 MB of bf16 output: well over twice
    the 126 MB L2), so every call starts with its inputs out of L2.  Median of
    `rounds` calls per weight; GB/s = algorithmic bytes / sum of medians."""
    b = step.b
    out = {}
    for kind in ("quantize", "dequant", "merge"):
        per = {i: [] for i in range(len(step.mats))}
        for it in range(3 + rounds):
            for i, d in enumerate(step.mats):
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                _gpu_ahead()
                s.record()
                if kind == "quantize":
                    b.quantize(d["W"], out=d["qw"])
                elif kind == "dequant":
                    b.dequant(d["qw"], out=d["Wd"])
                else:
                    b.lora_merge(d["qw"], d["A"], d["B"], step.wl.s, out=d["Wd"])
                e.record()
                per[i].append((s, e))
            torch.cuda.synchronize()
        med = [statistics.median([s.elapsed_time(e) for s, e in per[i][3:]]) for i in per]
        nbytes = sum(quant_bytes(d["N"], d["K"]) for d in step.mats)
        if kind == "merge":   # plus the LoRA factors, read once
            nbytes += sum(2 * step.wl.r * (d["N"] + d["K"]) for d in step.mats)
        gbs = nbytes / (sum(med) * 1e-3) / 1e9
        out[kind] = {"GB/s": gbs, "frac": gbs / peaks["hbm_gbs"], "us_per_weight_set": sum(med) * 1e3,
                     "timing": f"median of {rounds} calls per weight, calls rotating over the 7 weights "
                               f"(inputs out of L2)"}
    return out


def llama70b_component(device, peaks, layers=80, reps=20):
    """The LLaMA-70B-shaped configuration: every one of the 80 layers' 7
    weights is generated from its own seed, quantized (only the NF4 storage is
    kept: 35.3 GB resident), then dequantized once to bf16; each call is timed
    alone with L2 flushed before it.  Then qlora_linear fwd+bwd at 512 tokens
    (batch 1 x seq 512), r=64, alpha=16 on the 7 shapes of layer 0."""
    from bit_nf4_quantized_12_b200 import binding
    wl = workloads.WORKLOADS["llama70b"]
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    flush = flush_buf.zero_
    stored = []
    q_ms = 0.0
    nbytes = 0
    for layer in range(layers):
        for idx, (name, N, K) in enumerate(wl.mats):
            W = workloads.weight(N, K, wl.w_std, seed=workloads.matrix_seed("llama70b", layer, idx), device=device)
            qw = binding.empty_quantized(N, K, device)
            flush()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            _gpu_ahead()
            s.record()
            binding.quantize(W, out=qw)
            e.record()
            torch.cuda.synchronize()
            q_ms += s.elapsed_time(e)
            nbytes += quant_bytes(N, K)
            stored.append((layer, idx, qw))
            del W
    scratch = torch.empty(max(N * K for _, N, K in wl.mats), dtype=torch.bfloat16, device=device)
    dq_ms = 0.0
    for layer, idx, qw in stored:
        out = scratch[: qw.rows * qw.cols].view(qw.rows, qw.cols)
        flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _gpu_ahead()
        s.record()
        binding.dequant(qw, out=out)
        e.record()
        torch.cuda.synchronize()
        dq_ms += s.elapsed_time(e)
    res = {"weights": int(sum(q.rows * q.cols for _, _, q in stored)),
           "nf4_storage_GB": sum(q.packed.numel() + q.c1q.numel() + 4 * q.c2.numel() for _, _, q in stored) / 1e9,
           "quantize": {"GB/s": nbytes / (q_ms * 1e-3) / 1e9, "ms": q_ms},
           "dequant": {"GB/s": nbytes / (dq_ms * 1e-3) / 1e9, "ms": dq_ms}}
    for k in ("quantize", "dequant"):
        res[k]["frac"] = res[k]["GB/s"] / peaks["hbm_gbs"]
    del scratch
    # fwd + bwd at 512 tokens on layer 0's weights
    M, r, s_ = wl.tokens, wl.r, wl.s
    per = {}
    tf_f = tf_b = ms_f = ms_b = 0.0
    for layer, idx, qw in stored[: len(wl.mats)]:
        name, N, K = wl.mats[idx]
        io = workloads.layer_inputs(M, N, K, r, seed=workloads.matrix_seed("llama70b", 0, idx), device=device)
        ws = binding.workspace(M, N, K, r, device)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        T = torch.empty(M, r, dtype=torch.bfloat16, device=device)
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=device)
        dA = torch.empty(K, r, dtype=torch.float32, device=device)
        dB = torch.empty(r, N, dtype=torch.float32, device=device)
        f = _median_ms(lambda: binding.linear_fwd(io["X"], qw, io["A"], io["B"], s_, ws=ws, Y=Y, T=T), reps, flush)
        bb = _median_ms(lambda: binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s_, T=T, ws=ws, dX=dX,
                                                   dA=dA, dB=dB), reps, flush)
        per[f"{name} {N}x{K}"] = {"fwd_us": round(f * 1e3, 1), "bwd_us": round(bb * 1e3, 1),
                                  "fwd_TFLOP/s": round(fwd_flops(M, N, K, r) / (f * 1e-3) / 1e12, 1),
                                  "bwd_TFLOP/s": round(bwd_flops(M, N, K, r) / (bb * 1e-3) / 1e12, 1)}
        tf_f += fwd_flops(M, N, K, r)
        tf_b += bwd_flops(M, N, K, r)
        ms_f += f
        ms_b += bb
    fwd_t = tf_f / (ms_f * 1e-3) / 1e12
    bwd_t = tf_b / (ms_b * 1e-3) / 1e12
    both = (tf_f + tf_b) / ((ms_f + ms_b) * 1e-3) / 1e12
    res["linear_512_tokens"] = {
        "fwd": {"TFLOP/s": fwd_t, "frac": fwd_t / peaks["bf16_tflops_sustained"],
                "frac_burst": fwd_t / peaks["bf16_tflops"]},
        "bwd": {"TFLOP/s": bwd_t, "frac": bwd_t / peaks["bf16_tflops_sustained"],
                "frac_burst": bwd_t / peaks["bf16_tflops"]},
        "fwd+bwd": {"TFLOP/s": both, "frac": both / peaks["bf16_tflops_sustained"],
                    "frac_burst": both / peaks["bf16_tflops"]},
        "per_matrix": per, "timing": f"median of {reps} calls each, L2 flushed before every call"}
    del stored
    return res


def f16_component(device, peaks, reps=10):
    """The FP16 compute type: qlora_linear fwd+bwd on three 7B-shaped weights
    (q 4096x4096, gate 11008x4096, down 4096x11008) at 2048 tokens, r=64, with
    X, A, B, dY in fp16; each call timed alone, L2 flushed before it."""
    from bit_nf4_quantized_12_b200 import binding
    wl = workloads.WORKLOADS["llama7b"]
    M, r, s_ = wl.tokens, wl.r, wl.s
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device).zero_
    fl = ms = 0.0
    per = {}
    for idx in (0, 4, 6):
        name, N, K = wl.mats[idx]
        seed = workloads.matrix_seed("llama7b", 0, idx)
        qw = binding.quantize(workloads.weight(N, K, wl.w_std, seed=seed, device=device))
        io = {k: v.to(torch.float16) for k, v in workloads.layer_inputs(M, N, K, r, seed=seed, device=device).items()}
        ws = binding.workspace(M, N, K, r, device)
        Y = torch.empty(M, N, dtype=torch.float16, device=device)
        T = torch.empty(M, r, dtype=torch.float16, device=device)
        f = _median_ms(lambda: binding.linear_fwd(io["X"], qw, io["A"], io["B"], s_, ws=ws, Y=Y, T=T), reps, flush)
        b = _median_ms(lambda: binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s_, T=T, ws=ws), reps, flush)
        w = fwd_flops(M, N, K, r) + bwd_flops(M, N, K, r)
        per[f"{name} {N}x{K}"] = round(w / ((f + b) * 1e-3) / 1e12, 1)
        fl += w
        ms += f + b
    t = fl / (ms * 1e-3) / 1e12
    return {"fwd+bwd": {"TFLOP/s": t, "frac": t / peaks["bf16_tflops_sustained"]}, "per_matrix_TFLOP/s": per,
            "peak_note": "fp16 and bf16 share one dense tensor-core rate; the bf16 measured peak is used"}


def variants_component(device, peaks, reps=20):
    """Quantize and dequantize of the 11008x4096 weight in each storage
    format variant (uniform INT4 table; FP32 scale1; uint8 scale1), each call
    timed alone with L2 flushed before it."""
    from bit_nf4_quantized_12_b200 import binding
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device).zero_
    N, K = 11008, 4096
    W = workloads.weight(N, K, 0.02, seed=4, device=device)
    Wd = torch.empty_like(W)
    res = {}
    for qt, dq, name in ((binding.QUANT_NF4, binding.DQ_E4M3, "nf4+fp8/fp32 (the method)"),
                         (binding.QUANT_INT4, binding.DQ_E4M3, "int4+fp8/fp32"),
                         (binding.QUANT_NF4, binding.DQ_NONE, "nf4+fp32 scale1"),
                         (binding.QUANT_NF4, binding.DQ_U8, "nf4+uint8/fp32")):
        qw = binding.empty_quantized(N, K, device, qt, dq)
        q = _median_ms(lambda: binding.quantize(W, out=qw), reps, flush)
        d = _median_ms(lambda: binding.dequant(qw, out=Wd), reps, flush)
        nbytes = 2 * N * K + qw.packed.numel() + qw.c1q.numel() * qw.c1q.element_size() + 4 * qw.c2.numel()
        res[name] = {"quantize_GB/s": round(nbytes / (q * 1e-3) / 1e9, 1),
                     "dequant_GB/s": round(nbytes / (d * 1e-3) / 1e9, 1),
                     "quantize_frac": round(nbytes / (q * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                     "dequant_frac": round(nbytes / (d * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
    return res


def robust_component(device, peaks, reps=5):
    """The robustness configuration: W 4095x11007 (ragged final block and
    group; Student-t(3) with 0.1% outliers x20), qlora_linear fwd+bwd at 4096
    tokens, r=8, alpha=32; plus quantize / dequantize of that weight."""
    from bit_nf4_quantized_12_b200 import binding
    wl = workloads.WORKLOADS["robust"]
    _, N, K = wl.mats[0]
    M, r, s_ = wl.tokens, wl.r, wl.s
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    flush = flush_buf.zero_
    W = workloads.weight(N, K, wl.w_std, seed=0, device=device, kind=wl.w_kind)
    io = workloads.layer_inputs(M, N, K, r, seed=0, device=device)
    qw = binding.quantize(W)
    Wd = torch.empty_like(W)
    qm = _median_ms(lambda: binding.quantize(W, out=qw), 20, flush)
    dm = _median_ms(lambda: binding.dequant(qw, out=Wd), 20, flush)
    ws = binding.workspace(M, N, K, r, device)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    T = torch.empty(M, r, dtype=torch.bfloat16, device=device)
    f = _median_ms(lambda: binding.linear_fwd(io["X"], qw, io["A"], io["B"], s_, ws=ws, Y=Y, T=T), reps, flush, 1)
    bb = _median_ms(lambda: binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s_, T=T, ws=ws), reps,
                    flush, 1)
    plan = binding.plan(M, N, K, r)
    path = {binding.PATH_FUSED: "fused tensor-core", binding.PATH_DECODE: "decode",
            binding.PATH_GENERIC: "generic CUDA-core"}[plan["path"]]
    qb = quant_bytes(N, K)
    ft = fwd_flops(M, N, K, r) / (f * 1e-3) / 1e12
    bt = bwd_flops(M, N, K, r) / (bb * 1e-3) / 1e12
    return {"path": path,
            "quantize": {"GB/s": qb / (qm * 1e-3) / 1e9, "frac": qb / (qm * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "dequant": {"GB/s": qb / (dm * 1e-3) / 1e9, "frac": qb / (dm * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "fwd": {"TFLOP/s": ft, "frac": ft / peaks["bf16_tflops_sustained"], "us": f * 1e3},
            "bwd": {"TFLOP/s": bt, "frac": bt / peaks["bf16_tflops_sustained"], "us": bb * 1e3}}


# ------------------------------------------------------------------ oracle arm
def oracle_sample_step(wl, frac_rows, seed=0):
    """The oracle over a row sample of every matrix of the step: quantize and
    dequantize the sampled W rows (group-aligned), forward for those output
    features, backward restricted to them.  Returns (flops done, seconds)."""
    import oracle
    M, r, s = wl.tokens, wl.r, wl.s
    flops = 0.0
    secs = 0.0
    for idx, (name, N, K) in enumerate(wl.mats):
        mseed = workloads.matrix_seed(wl.name, 0, idx)
        n_rows = max(16, int(N * frac_rows) // 16 * 16)
        n0 = (seed * 7919 + idx * 104729) % (N - n_rows + 1)
        W = workloads.weight(N, K, wl.w_std, seed=mseed)
        io = workloads.layer_inputs(M, N, K, r, seed=mseed)
        Wb = workloads.bits(W[n0:n0 + n_rows])
        X, A = workloads.bits(io["X"]), workloads.bits(io["A"])
        Bs = workloads.bits(io["B"][:, n0:n0 + n_rows].contiguous())
        dYs = workloads.bits(io["dY"][:, n0:n0 + n_rows].contiguous())
        t0 = time.perf_counter()
        packed, c1q, c2, _ = oracle.quantize(Wb)
        Wd = oracle.dequant(packed, c1q, c2, Wb.size).reshape(n_rows, K)
        Y, T = oracle.qlora_fwd(X, Wd, A, Bs, s)
        oracle.qlora_bwd(dYs, X, Wd, A, Bs, s, T)
        secs += time.perf_counter() - t0
        flops += fwd_flops(M, n_rows, K, r) + bwd_flops(M, n_rows, K, r)
    return flops, secs


def blas_threads():
    """Threads numpy's BLAS uses (the oracle's matmuls); the C quantize and
    dequantize loops are single-threaded."""
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_baseline(wl, frac, seed=0):
    """The oracle's sampled step on one host core and on all of them (BLAS
    threads; the C loops run on one core either way)."""
    from threadpoolctl import threadpool_limits
    out = {}
    with threadpool_limits(limits=1, user_api="blas"):
        f1, s1 = oracle_sample_step(wl, frac, seed)
    fa, sa = oracle_sample_step(wl, frac, seed)
    out["all"] = {"value": fa / sa / 1e12, "cores": blas_threads(), "secs": sa}
    out["one"] = {"value": f1 / s1 / 1e12, "cores": 1, "secs": s1}
    return out


def max_over_ranks(ms, pg, device):
    """The slowest rank's time: the job is done when every replica is."""
    if pg is None:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, step_flops, steps, ms):
    """Aggregate TFLOP/s of `world` replicas that each ran `steps` steps in `ms`."""
    return world * step_flops * steps / (ms * 1e-3) / 1e12


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    frac = 1.0 / 256
    for _ in range(args.warmup):
        oracle_sample_step(wl, frac)
    flops, secs = 0.0, 0.0
    for k in range(args.steps):
        f, s_ = oracle_sample_step(wl, frac, seed=k + 1)
        flops += f
        secs += s_
    value = flops / secs / 1e12
    sample = (f"oracle (plain C quantize/dequant + float64 numpy GEMM) on 1/256 of the output features of each of "
              f"the 7 matrices per step (group-aligned row slice), all {wl.tokens} tokens")
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(wl, 1),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


METRIC = "NF4 dequant/quant GB/s and qlora_linear TFLOP/s, % of B200 roofline"


def config_dict(wl, n):
    return {"workload": "llama7b_layer_set: q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008; "
                        "quantize+dq, dequant, qlora fwd+bwd at 2048 tokens, r=64, alpha=16",
            "global_batch": wl.tokens * n, "seq_len": 512, "rank": wl.r, "alpha": wl.alpha,
            "parallelism": f"dp{n}: tokens split across replicas, one NCCL all-reduce of the dA/dB bucket per step"
                           if n > 1 else "single",
            "l2": "step working set ~1.3 GB > 126 MB L2; no flush between steps"}


def kernel_case(case, n):
    """n launches of one call on the 7B q matrix (4096x4096, 2048 tokens, r=64),
    or on the 28672x8192 decode weight at M=16 ("decode") or M=1 ("gemv": the
    same decode kernel with one token); "merge" merges the r=64 adapter into
    the 4096x4096 weight;
    quantize and dequant run on the 28672x8192 weight, whose 470 MB of bf16
    exceed the L2: a small case for ncu."""
    from bit_nf4_quantized_12_b200 import binding
    dev = torch.device("cuda", 0)
    wl = workloads.WORKLOADS["llama7b"]
    M, r, s = wl.tokens, wl.r, wl.s
    N, K = 4096, 4096
    if case in ("decode", "gemv"):
        M, r, s, N, K = (16 if case == "decode" else 1), 16, 1.0, 28672, 8192
    if case in ("quantize", "dequant"):
        M, r, s, N, K = 16, 16, 1.0, 28672, 8192
    if case in ("robust_fwd", "robust_bwd"):   # ragged K and N: the fused GEMM's ragged mode
        M, r, s, N, K = 4096, 8, 4.0, 4095, 11007
    W = workloads.weight(N, K, 0.02, seed=0, device=dev)
    io = workloads.layer_inputs(M, N, K, r, seed=0, device=dev)
    qw = binding.quantize(W)
    Wd = torch.empty_like(W)
    ws = binding.workspace(M, N, K, r, dev)
    Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], s, ws=ws)
    for _ in range(n):
        if case == "quantize":
            binding.quantize(W, out=qw)
        elif case == "dequant":
            binding.dequant(qw, out=Wd)
        elif case == "merge":
            binding.lora_merge(qw, io["A"], io["B"], s, out=Wd)
        elif case in ("fwd", "decode", "gemv", "robust_fwd"):
            binding.linear_fwd(io["X"], qw, io["A"], io["B"], s, ws=ws, Y=Y, T=T)
        else:
            binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s, T=T, ws=ws)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--kernel-case", default=None, choices=["quantize", "dequant", "fwd", "bwd", "decode", "gemv", "merge", "robust_fwd",
                                                         "robust_bwd"],
                    help="run a few launches of one call on one 7B-shaped matrix (for ncu), print nothing")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = workloads.WORKLOADS["llama7b"]

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    if args.kernel_case:
        kernel_case(args.kernel_case, args.steps)
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    peaks, peak_kind = load_peaks()

    step = Step(device, wl, host_copy=True, world=world)
    step_launches = step.launches_per_step
    # warm-up: at least W steps and at least ~1.5 s of load, with the clock
    # sampler already running so that its samples cover the loaded GPU
    clocks = ClockSampler(local)
    clocks.start()
    t_w = time.perf_counter()
    nw = 0
    while nw < max(3, args.warmup) or time.perf_counter() - t_w < 1.5:
        step.run()
        nw += 1
        if nw % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    # ---- timed region: K device-resident steps
    ev = {k: ([], []) for k in ("q", "dq", "fwd", "bwd")}
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t0 = _ev()
    for _ in range(args.steps):
        step.run(events=ev)
    t1 = _ev()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), pg, device)

    M, r = wl.tokens, wl.r
    step_flops = sum(fwd_flops(M, N, K, r) + bwd_flops(M, N, K, r) for _, N, K in wl.mats)
    value = whole_job_tflops(world, step_flops, args.steps, ms)

    comp = {}
    qb = sum(quant_bytes(N, K) for _, N, K in wl.mats) * args.steps
    q_ms = sum(_pair_ms(*ev["q"]))
    dq_ms = sum(_pair_ms(*ev["dq"]))
    f_ms = sum(_pair_ms(*ev["fwd"]))
    b_ms = sum(_pair_ms(*ev["bwd"]))
    fl_f = sum(fwd_flops(M, N, K, r) for _, N, K in wl.mats) * args.steps
    fl_b = sum(bwd_flops(M, N, K, r) for _, N, K in wl.mats) * args.steps
    comp["quantize"] = {"GB/s": qb / (q_ms * 1e-3) / 1e9, "ms_per_step": q_ms / args.steps}
    comp["dequant"] = {"GB/s": qb / (dq_ms * 1e-3) / 1e9, "ms_per_step": dq_ms / args.steps}
    comp["fwd"] = {"TFLOP/s": fl_f / (f_ms * 1e-3) / 1e12, "ms_per_step": f_ms / args.steps}
    comp["bwd"] = {"TFLOP/s": fl_b / (b_ms * 1e-3) / 1e12, "ms_per_step": b_ms / args.steps}
    for k in ("quantize", "dequant"):
        comp[k]["frac"] = comp[k]["GB/s"] / peaks["hbm_gbs"]
    for k in ("fwd", "bwd"):
        comp[k]["frac"] = comp[k]["TFLOP/s"] / peaks["bf16_tflops_sustained"]
        comp[k]["frac_burst"] = comp[k]["TFLOP/s"] / peaks["bf16_tflops"]

    # dominant work: the qlora_linear calls (forward + backward)
    gemm_tflops = (fl_f + fl_b) / ((f_ms + b_ms) * 1e-3) / 1e12
    roofline = {"kernel": "qlora_linear_fwd+bwd calls (nf4_gemm_kernel + skinny_gemm_kernel)",
                "bound": "tensor", "achieved": gemm_tflops, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": gemm_tflops / peaks["bf16_tflops_sustained"],
                "frac_burst": gemm_tflops / peaks["bf16_tflops"],
                "peak_kind": f"{peak_kind} bf16_tflops_sustained",
                # DRAM read+write of one forward launch of the fused GEMM from the
                # ncu capture of the kernel as built (see traffic_case)
                "traffic": GEMM_FWD_Q_DRAM_BYTES,
                "traffic_case": GEMM_FWD_Q_DRAM_CASE}

    # ---- end to end through the public API with host buffers
    h2d, d2h = step.e2e_bytes()
    for _ in range(2):
        step.run_e2e()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e0 = _ev()
    for _ in range(args.steps):
        step.run_e2e()
    e1 = _ev()
    torch.cuda.synchronize()
    ems = max_over_ranks(e0.elapsed_time(e1), pg, device)
    e2e_value = whole_job_tflops(world, step_flops, args.steps, ems)

    if not args.no_components and rank == 0 and world == 1:
        bw = bandwidth_component(step, peaks)
        comp["quantize"].update({"step_GB/s": comp["quantize"].pop("GB/s"), "step_frac": comp["quantize"].pop("frac")})
        comp["dequant"].update({"step_GB/s": comp["dequant"].pop("GB/s"), "step_frac": comp["dequant"].pop("frac")})
        comp["quantize"].update(bw["quantize"])
        comp["dequant"].update(bw["dequant"])
        comp["merge"] = bw["merge"]
        del step
        torch.cuda.empty_cache()
        comp["decode"] = decode_component(device, peaks)
        torch.cuda.empty_cache()
        comp["llama70b"] = llama70b_component(device, peaks)
        torch.cuda.empty_cache()
        comp["robust"] = robust_component(device, peaks)
        torch.cuda.empty_cache()
        comp["f16"] = f16_component(device, peaks)
        comp["variants"] = variants_component(device, peaks)

    cpu = None
    if rank == 0 and world == 1:
        ob = oracle_baseline(wl, 1.0 / 256)
        sample = ("oracle on 1/256 of the output features of each of the 7 matrices (quantize+dequant of those "
                  "rows, fwd+bwd restricted to them), all 2048 tokens")
        cpu = {"value": ob["all"]["value"], "unit": "TFLOP/s", "cores": ob["all"]["cores"], "kind": "oracle",
               "sample": sample + "; C quantize/dequant loops single-threaded, numpy BLAS on all cores",
               "single_core": {"value": ob["one"]["value"], "unit": "TFLOP/s", "cores": 1}}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_dict(wl, world), "roofline": roofline, "components": comp,
                "cpu_baseline": cpu, "clocks": clk,
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": step_launches * args.steps,
                "peaks": {"kind": peak_kind, "hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                          "bf16_tflops_sustained": peaks["bf16_tflops_sustained"]}}
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
