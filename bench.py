"""Throughput benchmark of the M²RNN layer recurrence on B200.

One "step" is one pass of the whole hot path over one batch of synthetic
input: the forward scan (writing checkpoints) followed by the backward
(BPTT with recompute) for training workloads, the forward alone for forward
workloads.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own shard of the
global batch (weak scaling; same W, rank-seeded data).  The only exchange is
the all-reduce of dW (the gradient of the shared per-head W is a sum over the
global batch) in training workloads.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores on a bounded sample of the same workload (whole (b, h) pairs at full
length), because the pages describe no runnable reference implementation.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from non_linear_matrix_persistent_b200 import WORKLOADS, make_inputs  # noqa: E402
from non_linear_matrix_persistent_b200.inputs import make_shard_inputs  # noqa: E402

METRIC = "M2RNN layer fwd(+bwd) tokens/s on 1 B200; tensor-pipe % and HBM GB/s via ncu"
DEFAULT_WORKLOAD = "layer410m_train"
L2_FLUSH_BYTES = 256 << 20
NUM_SMS = 148
SFU_PER_SM_PER_CLK = 16      # special-function (exp / reciprocal / tanh) results per SM per clock
# SFU operations the kernels spend per tanh: the accurate tanh is 1 - 2/(1 + e^{2x})
# (one exp and one reciprocal), the fast-tanh inference mode one tanh.approx.
# This is an implementation cost; the roofline fraction counts the method's
# work, one tanh per state element and step.
SFU_OPS_PER_TANH = {"accurate": 2, "fast": 1}
# Forward-only workloads timed beside the training step (each its own CUDA-event
# timing, L2 flushed between steps).
FORWARD_CONFIGS = ("tiny_fp32", "layer410m_fwd", "long_b1_fwd", "layer7b_moe_fwd")
# Training workloads (forward with checkpoints + backward) timed beside the main one.
TRAINING_CONFIGS = ("layer7b_moe_train",)
CSRC = os.path.join(ROOT, "non_linear_matrix_persistent_b200", "csrc")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu, self.period = gpu_index, period_ms
        self.proc = self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", str(self.period)],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)   # let the first sample land before the timed region
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": sorted(reasons), "samples": len(rows)}


def per_step_counts(w):
    """Algorithmic work per (b, h, t) of each kernel: tanh count, tensor FLOP
    (one GEMM forward, three backward) and compulsory HBM bytes (bf16 inputs,
    fp32 outputs and gradients, the fp32 checkpoint amortised over C steps)."""
    K, V, C = w.K, w.V, w.ckpt_stride
    fwd = {"tanh": K * V, "flop": 2.0 * K * V * V,
           "bytes": (2 * K + V) * 2 + 4 + 4 * V + (4.0 * K * V / C if w.backward else 0.0)}
    bwd = {"tanh": K * V, "flop": 3 * 2.0 * K * V * V,
           "bytes": (2 * K + 2 * V) * 2 + 4 + (2 * K + V) * 4 + 4 + 4.0 * K * V / C}
    return fwd, bwd


def forward_kernel(w):
    """(kernel name, source file) of the forward that runs for workload w, by
    the library's dispatch rule: the fp32 debug mode has its own kernel;
    64-column states with B·H·K/8 <= 148 rows-of-8 run the row kernel (one
    warp per state row); everything else the tcgen05 kernel."""
    if w.mode != "bf16":
        return "m2rnn_fwd_fp32_kernel", "debug_fp32.cu"
    if w.V == 64 and w.K % 8 == 0 and w.B * w.H * (w.K // 8) <= NUM_SMS:
        return "m2rnn_fwd_rows_kernel", "fwd_rows.cu"
    return "m2rnn_fwd_tc_kernel", "fwd_tc.cu"


def backward_kernel(w):
    """(kernel name, source file) of the tensor-core backward for workload w:
    the extended-operand kernel for V = 64 with K >= 32 and a checkpoint
    stride that its tensor-memory scratch holds (16 steps at K = 32, 8 at
    K = 64 and 128), the general-shape kernel otherwise."""
    if w.V == 64 and w.K in (32, 64, 128) and w.ckpt_stride <= (16 if w.K == 32 else 8):
        return "m2rnn_bwd_tc_kernel", "bwd_tc.cu"
    return "m2rnn_bwd_tcg_kernel", "bwd_tcg.cu"


def profile_name(kernel, workload):
    """profiles/ summary of one kernel on one workload: m2rnn_fwd_tc_kernel on
    layer410m_train is m2rnn_fwd_tc_layer410m_train.md."""
    return "%s_%s.md" % (kernel[:-len("_kernel")], workload)


def launches_per_step(w) -> int:
    """Kernels of this library that one step launches: the forward scan, plus
    the sum of the row slices' partial readouts when the forward splits rows
    (its workspace then holds the partials), plus the backward and its dW
    reduction for a training workload."""
    from non_linear_matrix_persistent_b200 import _lib
    d = _lib.Dims(w.B, w.H, w.T, w.K, w.V, _lib.MODE_BF16_TC if w.mode == "bf16" else _lib.MODE_FP32_DEBUG,
                  w.ckpt_stride, 0, 0)
    sliced = _lib.lib().m2rnn_workspace_size(d, 0) > 256
    return 1 + (1 if sliced else 0) + (2 if w.backward else 0)


def kernel_digest(src: bytes) -> str:
    """Fingerprint of a kernel build: its source code (comments and blank space
    removed, so that editing a comment keeps a profile valid) and the nvcc flags
    it is built with."""
    from non_linear_matrix_persistent_b200.build import NVCC_FLAGS
    text = src.decode("utf-8")
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    code = " ".join(text.split())
    flags = " ".join(f for f in NVCC_FLAGS if not f.startswith("-I"))
    return hashlib.sha256((code + "\n" + flags).encode()).hexdigest()[:16]


# Device-code headers the kernel files include; a profile is tied to them as
# well (kernels.h holds only host-side declarations).
KERNEL_HEADERS = ("common.cuh", "ptx.cuh", "tc_common.cuh")


def kernel_source(kernel_file: str) -> bytes:
    """The kernel file followed by the shared headers it is compiled with."""
    parts = [open(os.path.join(CSRC, kernel_file), "rb").read()]
    for h in KERNEL_HEADERS:
        path = os.path.join(CSRC, h)
        if os.path.exists(path):
            parts.append(open(path, "rb").read())
    return b"\n".join(parts)


def measured_traffic(kernel_file: str, profile_md: str):
    """DRAM bytes per launch recorded in a profiles/ summary, when that summary
    was taken from the current kernel build (kernel_digest of the kernel file
    and its headers); else None."""
    try:
        src = kernel_source(kernel_file)
        text = open(os.path.join(ROOT, "profiles", profile_md)).read()
    except OSError:
        return None
    digest = kernel_digest(src)
    m = re.search(r"build fingerprint of %s: `([0-9a-f]+)`" % re.escape(kernel_file), text)
    t = re.search(r"DRAM traffic per launch: ([0-9.]+) bytes", text)
    if m and t and m.group(1) == digest:
        return float(t.group(1))
    return None


def _sample_pairs(w, cores):
    """One distinct (b, h) pair per host thread (the oracle runs one pair per
    thread), at most all of them: pair i of the sample is number
    (i · s) mod B·H for a stride s coprime to B·H, spread over the batch and
    heads."""
    import math
    pairs_total = w.B * w.H
    npairs = max(1, min(pairs_total, cores))
    s = 37
    while math.gcd(s, pairs_total) != 1:
        s += 1
    return [divmod((i * s) % pairs_total, w.H) for i in range(npairs)]


def _oracle_sample(w, pairs, cores):
    from oracle import oracle
    x = make_inputs(w)

    def sel(n):
        return torch.stack([x[n][b, h] for b, h in pairs])[None]
    W = torch.stack([x["W"][h] for _, h in pairs])
    H0 = None if x["H0"] is None else sel("H0")
    args = (sel("k"), sel("v"), sel("q"), sel("f"), W, H0)

    def run():
        if w.backward:
            oracle.backward(*args, sel("dY"), nthreads=cores)
        else:
            oracle.forward(*args, nthreads=cores)
    return run


FMA_PER_SM_PER_CLK = 128     # fp32 fused multiply-adds per SM per clock (CUDA cores)


def kernel_entry(ms_mean, cnt, units, T, peaks, peak_kind, sm_max, sm_mhz, tanh_kind="accurate", traffic=None,
                 pipe="tensor"):
    """Roofline figures of one kernel from its mean CUDA-event time.

    The bound is the special-function unit: the method evaluates one tanh per
    state element and step (K·V per (b, h, t)), and the derived peak is
    148 SMs x 16 results per SM per clock x the maximum SM clock.  The SFU
    operations the implementation spends per tanh are reported apart
    (`sfu_ops`); the tensor-pipe and HBM fractions of the same launch go beside
    them.  `units` is the (b, h, t) steps one launch processes.  `pipe` names
    where the transition product runs: "tensor" (tcgen05 or mma.sync, against
    the measured bf16 peak) or "fma" (CUDA-core FFMA, against the derived fp32
    peak 148 SMs x 128 FMA x 2 FLOP x the maximum SM clock)."""
    s = ms_mean / 1e3
    tanh_rate = cnt["tanh"] * units / s / 1e9
    sfu_peak = NUM_SMS * SFU_PER_SM_PER_CLK * sm_max * 1e6 / 1e9
    per = SFU_OPS_PER_TANH[tanh_kind]
    e = {
        "ms": ms_mean,
        "bound": "alu", "unit": "Gtanh/s", "achieved": tanh_rate, "peak": sfu_peak, "frac": tanh_rate / sfu_peak,
        "peak_source": "derived: %d SMs x %d SFU results/clk x %.0f MHz (one tanh per state element and step)" % (
            NUM_SMS, SFU_PER_SM_PER_CLK, sm_max),
        "sfu_ops": {"per_tanh": per, "achieved_gops": per * tanh_rate, "frac": per * tanh_rate / sfu_peak},
        "traffic": traffic,
        "algorithmic_per_step": cnt,
        "units_per_launch": units,
        "hbm": {"achieved_gbs": cnt["bytes"] * units / s / 1e9, "peak_gbs": peaks["hbm_gbs"],
                "frac": cnt["bytes"] * units / s / 1e9 / peaks["hbm_gbs"], "peak_kind": peak_kind},
        "cycles_per_recurrence_step": s * sm_mhz * 1e6 / T,
    }
    if cnt.get("flop"):
        tf = cnt["flop"] * units / s / 1e12
        if pipe == "tensor":
            e["tensor"] = {"achieved_tflops": tf, "peak_tflops": peaks["bf16_tflops"],
                           "frac": tf / peaks["bf16_tflops"], "peak_kind": peak_kind}
        else:
            fpk = NUM_SMS * FMA_PER_SM_PER_CLK * 2 * sm_max * 1e6 / 1e12
            e["fma"] = {"achieved_tflops": tf, "peak_tflops": fpk, "frac": tf / fpk, "peak_kind": "derived"}
    return e


def kernel_pipe(kernel):
    """Where a kernel's transition product runs (see kernel_entry)."""
    return "fma" if kernel in ("m2rnn_fwd_rows_kernel", "m2rnn_fwd_fp32_kernel") else "tensor"


def time_forward_config(name, steps, warmup, dev, flush, peaks, peak_kind, sm_max, sm_mhz):
    """One forward-only workload: the default forward (and, for bf16 inputs,
    the fast-tanh inference forward) timed per step with CUDA events on the
    launching stream, L2 flushed between steps."""
    from non_linear_matrix_persistent_b200 import api
    w = WORKLOADS[name]
    x = make_inputs(w, device=str(dev))
    B, H, T, K, V = w.B, w.H, w.T, w.K, w.V
    out = {"y": torch.empty(B, H, T, V, device=dev), "HT": torch.empty(B, H, K, V, device=dev)}
    stream = torch.cuda.current_stream(dev)
    variants = [("accurate", False)] + ([("fast", True)] if w.mode == "bf16" else [])
    res = {"B": B, "H": H, "T": T, "K": K, "V": V, "mode": w.mode, "tokens": B * T}
    for kind, fast in variants:
        def run():
            api.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], out=out, fast_tanh=fast)
        for _ in range(warmup):
            run()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            run()
            b.record(stream)
        torch.cuda.synchronize()
        if api.device_status(dev) != 0:
            raise RuntimeError("device-side wait ran out in the %s forward" % name)
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        cnt, _ = per_step_counts(w)
        kname, ksrc = forward_kernel(w)
        traffic = measured_traffic(ksrc, profile_name(kname, name)) if kind == "accurate" else None
        e = kernel_entry(ms, cnt, B * H * T, T, peaks, peak_kind, sm_max, sm_mhz, kind, traffic, kernel_pipe(kname))
        e["kernel"] = kname
        e["tokens_per_s"] = B * T / (ms / 1e3)
        e["steps"] = steps
        res["forward" if kind == "accurate" else "forward_fast_tanh"] = e
    del x, out
    return res


def time_training_config(name, steps, warmup, dev, flush, peaks, peak_kind, sm_max, sm_mhz):
    """One training workload: the forward with checkpoints and the backward,
    each timed per step with CUDA events on the launching stream, L2 flushed
    between steps."""
    from non_linear_matrix_persistent_b200 import api
    w = WORKLOADS[name]
    x = make_inputs(w, device=str(dev))
    B, H, T, K, V, C = w.B, w.H, w.T, w.K, w.V, w.ckpt_stride
    out = {"y": torch.empty(B, H, T, V, device=dev), "HT": torch.empty(B, H, K, V, device=dev),
           "ckpt": torch.empty(B, H, (T + C - 1) // C, K, V, device=dev)}
    gout = {}
    stream = torch.cuda.current_stream(dev)

    def run(ev=None):
        if ev is not None:
            ev[0].record(stream)
        api.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], ckpt_stride=C, want_ckpt=True, out=out)
        if ev is not None:
            ev[1].record(stream)
        gout.update(api.backward(x["k"], x["v"], x["q"], x["f"], x["W"], out["ckpt"], x["dY"], ckpt_stride=C,
                                 out=gout))
        if ev is not None:
            ev[2].record(stream)
    for _ in range(warmup):
        run()
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    torch.cuda.synchronize()
    for ev in evs:
        flush.zero_()
        run(ev)
    torch.cuda.synchronize()
    if api.device_status(dev) != 0:
        raise RuntimeError("device-side wait ran out in the %s step" % name)
    fwd = statistics.mean(a.elapsed_time(b) for a, b, c in evs)
    bwd = statistics.mean(b.elapsed_time(c) for a, b, c in evs)
    cf, cb = per_step_counts(w)
    units = B * H * T
    res = {"B": B, "H": H, "T": T, "K": K, "V": V, "ckpt_stride": C, "tokens": B * T, "steps": steps,
           "ms_per_step": fwd + bwd, "tokens_per_s": B * T / ((fwd + bwd) / 1e3),
           "forward": kernel_entry(fwd, cf, units, T, peaks, peak_kind, sm_max, sm_mhz,
                                   pipe=kernel_pipe(forward_kernel(w)[0])),
           "backward": kernel_entry(bwd, cb, units, T, peaks, peak_kind, sm_max, sm_mhz)}
    for part, (kname, ksrc) in (("forward", forward_kernel(w)), ("backward", backward_kernel(w))):
        res[part]["kernel"] = kname
        res[part]["traffic"] = measured_traffic(ksrc, profile_name(kname, name))
    del x, out, gout
    return res


def bench_config(w, world):
    """The workload description both arms print (same keys, same values)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "K": w.K, "V": w.V, "ckpt_stride": w.ckpt_stride,
            "global_batch": w.B * world, "seq_len": w.T, "parallelism": "dp%d" % world,
            "l2": "flushed between timed steps (256 MB write)"}


def run_reference(args, w):
    """fp64 CPU oracle on a bounded sample of (b, h) pairs at full length."""
    from oracle import oracle
    pairs = _sample_pairs(w, oracle.default_threads())
    cores = len(pairs)   # threads that run
    run = _oracle_sample(w, pairs, cores)
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        run()
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    tok = w.B * w.T * len(pairs) / (w.B * w.H)
    value = tok * len(times) / sum(times)
    sample = "%d of %d (b,h) pairs at full T=%d, %s" % (len(pairs), w.B * w.H, w.T,
                                                         "fwd+bwd" if w.backward else "fwd")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline(w):
    from oracle import oracle
    pairs = _sample_pairs(w, oracle.default_threads())
    cores = len(pairs)   # threads that run
    run = _oracle_sample(w, pairs, cores)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    tok = w.B * w.T * len(pairs) / (w.B * w.H)
    return {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d (b,h) pairs at full T=%d, %s, one run" % (
                len(pairs), w.B * w.H, w.T, "fwd+bwd" if w.backward else "fwd")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the main workload (no forward-only configs)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller cases of the same kernels for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from non_linear_matrix_persistent_b200 import parallel
    rank, world = parallel.world_from_env()
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.batch > 0:
        w = w.with_(B=args.batch)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        parallel.init("nccl", timeout_s=120)

    from non_linear_matrix_persistent_b200 import api
    x_host = make_shard_inputs(w, rank)
    x = {n: (None if t is None else t.to(dev)) for n, t in x_host.items()}
    C = w.ckpt_stride
    B, H, T, K, V = w.B, w.H, w.T, w.K, w.V
    outs = {"y": torch.empty(B, H, T, V, device=dev), "HT": torch.empty(B, H, K, V, device=dev),
            "ckpt": torch.empty(B, H, (T + C - 1) // C, K, V, device=dev)}
    gouts = {}
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        api.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], ckpt_stride=C, want_ckpt=w.backward, out=outs)
        if ev is not None:
            ev[1].record(stream)
        if w.backward:
            g = api.backward(x["k"], x["v"], x["q"], x["f"], x["W"], outs["ckpt"], x["dY"], ckpt_stride=C, out=gouts)
            gouts.update(g)
            parallel.allreduce_dW(g["dW"])
        if ev is not None:
            ev[2].record(stream)

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if api.device_status(dev) != 0:
        raise RuntimeError("device-side wait ran out during warm-up")

    # kernel timing: per-step CUDA events on the launching stream, L2 flushed between steps
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
    step_ms = [a.elapsed_time(c) for a, b, c in evs]
    fwd_ms = [a.elapsed_time(b) for a, b, c in evs]
    bwd_ms = [b.elapsed_time(c) for a, b, c in evs]
    total_ms = parallel.max_over_ranks(sum(step_ms), dev)
    if api.device_status(dev) != 0:
        raise RuntimeError("device-side wait ran out during the timed region")
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T * world
    value = tokens_per_step / (ms_per_step / 1e3)

    # End to end through the public API from host memory.  Every step copies
    # its inputs from pinned host memory, runs the forward (and backward), and
    # reads its results back (y and, for training, all six gradients).  Steps
    # are pipelined as a streaming training or serving loop runs them: three
    # streams (inputs in, compute, results out) and two device buffer sets, so
    # that step i's compute overlaps step i+1's input copy and step i-1's
    # result copy.  The timed region spans the first input copy to the last
    # result copy.
    pinned = {n: t.pin_memory() for n, t in x_host.items() if t is not None}
    res_names = ["y"] + (["dk", "dv", "dq", "df", "dW", "dH0"] if w.backward else [])
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    nbuf = 2
    dbuf = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in pinned.items()} for _ in range(nbuf)]
    fbuf = [{"y": torch.empty(B, H, T, V, device=dev), "HT": torch.empty(B, H, K, V, device=dev),
             "ckpt": torch.empty(B, H, (T + C - 1) // C, K, V, device=dev)} for _ in range(nbuf)]
    gshape = {"dk": (B, H, T, K), "dv": (B, H, T, V), "dq": (B, H, T, K), "df": (B, H, T), "dW": (H, V, V),
              "dH0": (B, H, K, V)}
    gbuf = [{n: torch.empty(s, device=dev) for n, s in gshape.items()} for _ in range(nbuf)]
    hbuf = [{n: torch.empty((fbuf[0]["y"] if n == "y" else gbuf[0][n]).shape, pin_memory=True) for n in res_names}
            for _ in range(nbuf)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in hbuf[0].values())

    def e2e_run(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_comp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(s_in)
        for i in range(nsteps):
            b = i % nbuf
            with torch.cuda.stream(s_in):
                if i >= nbuf:
                    s_in.wait_event(ev_comp[i - nbuf])   # the compute that read this buffer set is done
                for n, t in pinned.items():
                    dbuf[b][n].copy_(t, non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[i])
                if i >= nbuf:
                    s_comp.wait_event(ev_out[i - nbuf])  # its results were read back
                xd = dbuf[b]
                api.forward(xd["k"], xd["v"], xd["q"], xd["f"], xd["W"], xd.get("H0"), ckpt_stride=C,
                            want_ckpt=w.backward, out=fbuf[b])
                if w.backward:
                    api.backward(xd["k"], xd["v"], xd["q"], xd["f"], xd["W"], fbuf[b]["ckpt"], xd["dY"],
                                 ckpt_stride=C, out=gbuf[b])
                    parallel.allreduce_dW(gbuf[b]["dW"])
                ev_comp[i].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                for n in res_names:
                    hbuf[b][n].copy_(fbuf[b]["y"] if n == "y" else gbuf[b][n], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(args.warmup)
    if world > 1:
        dist.barrier()
    e2e_total = parallel.max_over_ranks(e2e_run(args.steps), dev)
    e2e_value = tokens_per_step / (e2e_total / args.steps / 1e3)
    with torch.cuda.stream(s_comp):   # the end-to-end steps used that stream's workspace
        if api.device_status(dev) != 0:
            raise RuntimeError("device-side wait ran out during the end-to-end steps")

    peaks, peak_kind = _peaks()
    clocks = clk.summary()
    sm_mhz = clocks.get("sm_mhz") or float(peaks.get("sm_max_mhz", 1965.0))
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    cf, cb = per_step_counts(w)
    units = B * H * T   # (b, h, t) steps per launch on this rank
    kernels = {}
    for (name, src), ms_list, cnt, bwd in ((forward_kernel(w), fwd_ms, cf, False),
                                          (backward_kernel(w), bwd_ms, cb, True)):
        if bwd and not w.backward:
            continue
        kernels[name] = kernel_entry(statistics.mean(ms_list), cnt, units, T, peaks, peak_kind, sm_max, sm_mhz,
                                     "accurate", measured_traffic(src, profile_name(name, w.name)),
                                     kernel_pipe(name))
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    roofline = dict(kernel=dom, **{k: v for k, v in kernels[dom].items()})
    roofline["kernels"] = kernels

    # Forward-only workloads on the same clock (rank 0 of a single-GPU run).
    forward_configs = None
    if world == 1 and not args.no_extra:
        fsteps = max(3, min(args.steps, 10))
        forward_configs = {}
        for name in FORWARD_CONFIGS:
            forward_configs[name] = time_forward_config(name, fsteps, args.warmup, dev, flush, peaks, peak_kind,
                                                        sm_max, sm_mhz)
        training_configs = {}
        for name in TRAINING_CONFIGS:
            training_configs[name] = time_training_config(name, max(3, min(args.steps, 5)), args.warmup, dev,
                                                          flush, peaks, peak_kind, sm_max, sm_mhz)
    launches = args.steps * launches_per_step(w)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(w, world),
            "clocks": clocks, "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_total / args.steps,
                    "how": "pinned host inputs -> device -> fwd+bwd -> all results to pinned host, every step; "
                           "3 streams, 2 buffer sets (step i compute overlaps i+1 copy-in and i-1 copy-out)"},
            "roofline": roofline}
    if forward_configs is not None:
        line["forward_configs"] = forward_configs
        line["training_configs"] = training_configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
