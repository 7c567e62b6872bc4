"""Throughput benchmark of the M²RNN layer recurrence on B200.

One "step" is one pass of the whole hot path over one batch of synthetic
input: the forward scan (writing checkpoints) followed by the backward
(BPTT with recompute) for training workloads, the forward alone for forward
workloads.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own shard of the
global batch (weak scaling; the ranks' inputs differ by seed).  The only
exchange is the all-reduce of dW (the gradient of the shared per-head W is a
sum over the global batch) in training workloads.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores on a bounded sample of the same workload (whole (b, h) pairs at full
length), because there is no runnable reference implementation.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from non_linear_matrix_persistent_b200 import WORKLOADS, make_inputs  # noqa: E402

METRIC = "M2RNN layer fwd(+bwd) tokens/s on 1 B200"
DEFAULT_WORKLOAD = "layer410m_train"
L2_FLUSH_BYTES = 256 << 20
MUFU_PER_SM_PER_CLK = 16      # tanh.approx results per SM per clock (4 per SM sub-partition)
NUM_SMS = 148


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
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
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def algorithmic_counts(w):
    """Per-launch algorithmic work of the forward scan (the dominant kernel)."""
    steps = w.B * w.H * w.T
    return {
        "tanh": steps * w.K * w.V,                          # one tanh per state element per step
        "gemm_flop": 2.0 * steps * w.K * w.V * w.V,          # H_{t-1}W
        "hbm_bytes": steps * ((2 * w.K + w.V) * 2 + 4 + 4 * w.V),  # k,q,v (bf16), f, y (fp32)
    }


def run_reference(args, w):
    """fp64 CPU oracle on a bounded sample of (b, h) pairs at full length."""
    from oracle import oracle
    cores = oracle.default_threads()
    pairs_total = w.B * w.H
    # sample size: enough pairs to keep every core busy, bounded by the work budget
    per_pair_flop = 2.0 * w.T * w.K * w.V * w.V * (4.0 if w.backward else 1.0)
    budget = float(os.environ.get("M2RNN_REF_FLOP_BUDGET", 2.0e10))
    npairs = int(max(1, min(pairs_total, cores, budget // per_pair_flop)))
    x = make_inputs(w)
    pairs = [(i % w.B, (i * 7) % w.H) for i in range(npairs)]

    def sel(n):
        return torch.stack([x[n][b, h] for b, h in pairs])[None]
    k, v, q, f = sel("k"), sel("v"), sel("q"), sel("f")
    W = torch.stack([x["W"][h] for _, h in pairs])
    H0 = None if x["H0"] is None else sel("H0")
    dY = sel("dY") if w.backward else None
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if w.backward:
            oracle.backward(k, v, q, f, W, H0, dY, nthreads=cores)
        else:
            oracle.forward(k, v, q, f, W, H0, nthreads=cores)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    tok = w.B * w.T * npairs / pairs_total
    value = tok * len(times) / sum(times)
    sample = "%d of %d (b,h) pairs at full T=%d, %s" % (npairs, pairs_total, w.T,
                                                         "fwd+bwd" if w.backward else "fwd")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "K": w.K, "V": w.V},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline(w):
    from oracle import oracle
    cores = oracle.default_threads()
    pairs_total = w.B * w.H
    per_pair_flop = 2.0 * w.T * w.K * w.V * w.V * (4.0 if w.backward else 1.0)
    npairs = int(max(1, min(pairs_total, cores, 2.0e10 // per_pair_flop)))
    x = make_inputs(w)
    pairs = [(i % w.B, (i * 7) % w.H) for i in range(npairs)]

    def sel(n):
        return torch.stack([x[n][b, h] for b, h in pairs])[None]
    W = torch.stack([x["W"][h] for _, h in pairs])
    H0 = None if x["H0"] is None else sel("H0")
    t0 = time.perf_counter()
    if w.backward:
        oracle.backward(sel("k"), sel("v"), sel("q"), sel("f"), W, H0, sel("dY"), nthreads=cores)
    else:
        oracle.forward(sel("k"), sel("v"), sel("q"), sel("f"), W, H0, nthreads=cores)
    dt = time.perf_counter() - t0
    tok = w.B * w.T * npairs / pairs_total
    return {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d (b,h) pairs at full T=%d, %s, one run" % (
                npairs, pairs_total, w.T, "fwd+bwd" if w.backward else "fwd")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    from non_linear_matrix_persistent_b200 import api
    wr = w.with_(seed=w.seed + rank)
    x_host = make_inputs(wr)
    x = {n: (None if t is None else t.to(dev)) for n, t in x_host.items()}
    C = 16
    B, H, T, K, V = w.B, w.H, w.T, w.K, w.V
    outs = {"y": torch.empty(B, H, T, V, device=dev), "HT": torch.empty(B, H, K, V, device=dev),
            "ckpt": torch.empty(B, H, (T + C - 1) // C, K, V, device=dev)}
    gouts = {}
    stream = torch.cuda.current_stream(dev)

    def step():
        y, HT, ck = api.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], ckpt_stride=C,
                                want_ckpt=w.backward, out=outs)
        if w.backward:
            g = api.backward(x["k"], x["v"], x["q"], x["f"], x["W"], ck, x["dY"], ckpt_stride=C, out=gouts)
            gouts.update(g)
            if dist is not None:
                dist.all_reduce(g["dW"])
        return y

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if api.device_status(dev) != 0:
        raise RuntimeError("device-side wait ran out during warm-up")

    # kernel-only timing: per-step CUDA events on the launching stream, L2 flushed between steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    fwd_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            fwd_ev[i][0].record(stream)
            api.forward(x["k"], x["v"], x["q"], x["f"], x["W"], x["H0"], ckpt_stride=C, want_ckpt=w.backward,
                        out=outs)
            fwd_ev[i][1].record(stream)
            if w.backward:
                g = api.backward(x["k"], x["v"], x["q"], x["f"], x["W"], outs["ckpt"], x["dY"], ckpt_stride=C,
                                 out=gouts)
                gouts.update(g)
                if dist is not None:
                    dist.all_reduce(g["dW"])
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    fwd_ms = [a.elapsed_time(b) for a, b in fwd_ev]
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    if api.device_status(dev) != 0:
        raise RuntimeError("device-side wait ran out during the timed region")
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T * world
    value = tokens_per_step / (ms_per_step / 1e3)

    # end-to-end through the public API with host buffers: pinned H2D of the
    # step's inputs, the step, D2H of its results
    pinned = {n: (None if t is None else t.pin_memory()) for n, t in x_host.items()}
    res_names = ["y"] + (["dk", "dv", "dq", "df", "dW", "dH0"] if w.backward else [])
    h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
    host_out = {}
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        xd = {n: (None if t is None else t.to(dev, non_blocking=True)) for n, t in pinned.items()}
        y, _, ck = api.forward(xd["k"], xd["v"], xd["q"], xd["f"], xd["W"], xd["H0"], ckpt_stride=C,
                               want_ckpt=w.backward)
        res = {"y": y}
        if w.backward:
            res.update(api.backward(xd["k"], xd["v"], xd["q"], xd["f"], xd["W"], ck, xd["dY"], ckpt_stride=C))
            if dist is not None:
                dist.all_reduce(res["dW"])
        for n in res_names:
            if n not in host_out:
                host_out[n] = torch.empty(res[n].shape, dtype=res[n].dtype, pin_memory=True)
            host_out[n].copy_(res[n], non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    e2e_total = sum(e2e_ms)
    if dist is not None:
        t = torch.tensor([e2e_total], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total = float(t.item())
    e2e_value = tokens_per_step / (e2e_total / args.steps / 1e3)

    peaks, peak_kind = _peaks()
    clocks = clk.summary()
    cnt = algorithmic_counts(w)
    fwd_avg_s = sum(fwd_ms) / len(fwd_ms) / 1e3
    sm_mhz_peak = float(peaks.get("sm_max_mhz", 1965.0))
    mufu_peak = NUM_SMS * MUFU_PER_SM_PER_CLK * sm_mhz_peak * 1e6 / 1e9   # Gtanh/s
    achieved_tanh = cnt["tanh"] / fwd_avg_s / 1e9
    roofline = {"kernel": "m2rnn_fwd_tc_kernel", "bound": "alu", "unit": "Gtanh/s",
                "achieved": achieved_tanh, "peak": mufu_peak, "frac": achieved_tanh / mufu_peak,
                "peak_source": "derived: %d SMs x %d MUFU tanh/clk x %.0f MHz" % (NUM_SMS, MUFU_PER_SM_PER_CLK,
                                                                                  sm_mhz_peak),
                "traffic": None,
                "tensor": {"achieved_tflops": cnt["gemm_flop"] / fwd_avg_s / 1e12,
                           "peak_tflops": peaks["bf16_tflops"],
                           "frac": cnt["gemm_flop"] / fwd_avg_s / 1e12 / peaks["bf16_tflops"],
                           "peak_kind": peak_kind},
                "hbm": {"achieved_gbs": cnt["hbm_bytes"] / fwd_avg_s / 1e9, "peak_gbs": peaks["hbm_gbs"],
                        "frac": cnt["hbm_bytes"] / fwd_avg_s / 1e9 / peaks["hbm_gbs"], "peak_kind": peak_kind},
                "fwd_ms": fwd_avg_s * 1e3,
                "cycles_per_step": fwd_avg_s * sm_mhz_peak * 1e6 / T}
    launches = args.steps * (1 + (2 if w.backward else 0))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "T": T, "K": K, "V": V, "ckpt_stride": C,
                       "global_batch": B * world, "seq_len": T, "parallelism": "dp%d" % world,
                       "l2": "flushed between timed steps (256 MB write)"},
            "clocks": clocks, "gpu_launches": launches,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "roofline": roofline}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
