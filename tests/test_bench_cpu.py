"""Host logic of bench.py (no GPU): algorithmic unit counts, the build
fingerprint that ties a profiles/ summary to the kernel source it was taken
from, and the parsing of the clock samples."""
import os

import pytest

import bench
from non_linear_matrix_persistent_b200 import WORKLOADS


def test_per_step_counts_training_workload():
    fwd, bwd = bench.per_step_counts(WORKLOADS["layer410m_train"])
    K = V = 64
    assert fwd["flop"] == 2 * K * V * V and bwd["flop"] == 3 * 2 * K * V * V
    assert fwd["tanh"] == bwd["tanh"] == K * V
    assert WORKLOADS["layer410m_train"].ckpt_stride == 8
    # forward: k, q, v bf16 in, f in, y fp32 out, the fp32 checkpoint every 8 steps
    assert fwd["bytes"] == (2 * K + V) * 2 + 4 + 4 * V + 4 * K * V / 8 == 2692
    # backward: k, q, v, dy bf16 and f in, dk, dq, dv, df fp32 out, one checkpoint read per 8 steps
    assert bwd["bytes"] == (2 * K + 2 * V) * 2 + 4 + (2 * K + V) * 4 + 4 + 4 * K * V / 8 == 3336
    f_only, _ = bench.per_step_counts(WORKLOADS["layer410m_fwd"])
    assert f_only["bytes"] == 2692 - 4 * K * V / 8   # no checkpoints without a backward
    _, bwd7 = bench.per_step_counts(WORKLOADS["layer7b_moe_train"])
    assert bwd7["bytes"] == (4 * 128) * 2 + 4 + (3 * 128) * 4 + 4 + 4 * 128 * 128 / 8


def test_kernel_digest_ignores_comments_only():
    src = b"__global__ void k(float* p) {\n  p[0] = 1.f;  // one\n}\n"
    same = b"/* header */\n__global__ void k(float* p)\n{\n\n  p[0] = 1.f;\n}\n// end\n"
    other = b"__global__ void k(float* p) {\n  p[0] = 2.f;  // one\n}\n"
    assert bench.kernel_digest(src) == bench.kernel_digest(same)
    assert bench.kernel_digest(src) != bench.kernel_digest(other)


def test_measured_traffic_only_for_the_profiled_build(tmp_path, monkeypatch):
    csrc, prof = tmp_path / "csrc", tmp_path / "profiles"
    csrc.mkdir()
    prof.mkdir()
    src = b"__global__ void k() {}\n"
    (csrc / "k.cu").write_bytes(src)
    text = "build fingerprint of k.cu: `%s` (...)\n\nDRAM traffic per launch: 1234 bytes (...)\n"
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (prof / "k.md").write_text(text % bench.kernel_digest(src))
    assert bench.measured_traffic("k.cu", "k.md") == 1234.0
    (prof / "k.md").write_text(text % ("0" * 16))
    assert bench.measured_traffic("k.cu", "k.md") is None
    assert bench.measured_traffic("k.cu", "missing.md") is None


def test_clock_summary_parses_samples_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 820.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")
    s = bench.ClockSampler(0)
    s.proc, s.path = object(), str(path)   # as if nvidia-smi had written the file
    out = s.summary()
    assert out["sm_mhz"] == 1950.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
    assert not os.path.exists(path)
    assert bench.ClockSampler(0).summary()["reasons"] == ["unsampled"]


@pytest.mark.parametrize("world", [1, 4])
def test_bench_config_names_the_workload(world):
    w = WORKLOADS["layer410m_train"]
    c = bench.bench_config(w, world)
    assert c["workload"] == "layer410m_train" and c["global_batch"] == 8 * world
    assert c["parallelism"] == "dp%d" % world and "l2" in c


@pytest.mark.parametrize("name", sorted(WORKLOADS))
@pytest.mark.parametrize("cores", [1, 3, 16, 500])
def test_cpu_sample_is_one_distinct_pair_per_thread(name, cores):
    w = WORKLOADS[name]
    pairs = bench._sample_pairs(w, cores)
    assert len(pairs) == min(cores, w.B * w.H)
    assert len(set(pairs)) == len(pairs)
    assert all(0 <= b < w.B and 0 <= h < w.H for b, h in pairs)


def test_launches_per_step():
    from non_linear_matrix_persistent_b200 import build
    build.build()   # the workspace query needs the library (it launches nothing)
    # training: forward, backward, dW reduction; 128 pairs fill the GPU, so rows are not split
    assert bench.launches_per_step(WORKLOADS["layer410m_train"]) == 3
    assert bench.launches_per_step(WORKLOADS["layer410m_fwd"]) == 1
    # 16 pairs: the forward splits rows and sums the slices' readouts in a second kernel
    assert bench.launches_per_step(WORKLOADS["long_b1_fwd"]) == 2
    assert bench.launches_per_step(WORKLOADS["tiny_fp32"]) == 1


def test_roofline_fraction_counts_one_tanh_per_element():
    """frac is the method's tanh rate (K·V per (b, h, t)) over the derived SFU
    peak; the implementation's SFU operations per tanh are reported apart."""
    w = WORKLOADS["layer410m_train"]
    fwd, _ = bench.per_step_counts(w)
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}
    units = w.B * w.H * w.T
    ms = 2.0
    e = bench.kernel_entry(ms, fwd, units, w.T, peaks, "measured", 1965.0, 1965.0, "accurate")
    tanh_rate = 64 * 64 * units / (ms / 1e3) / 1e9
    peak = 148 * 16 * 1965.0 / 1e3
    assert e["unit"] == "Gtanh/s" and abs(e["achieved"] - tanh_rate) < 1e-9 * tanh_rate
    assert abs(e["peak"] - peak) < 1e-9 and abs(e["frac"] - tanh_rate / peak) < 1e-12
    assert e["sfu_ops"]["per_tanh"] == 2 and abs(e["sfu_ops"]["frac"] - 2 * e["frac"]) < 1e-12
    fast = bench.kernel_entry(ms, fwd, units, w.T, peaks, "measured", 1965.0, 1965.0, "fast")
    assert fast["frac"] == e["frac"] and fast["sfu_ops"]["per_tanh"] == 1
    assert abs(e["tensor"]["achieved_tflops"] - 2 * 64 ** 3 * units / 2e-3 / 1e12) < 1e-6
    assert abs(e["cycles_per_recurrence_step"] - 2e-3 * 1965e6 / w.T) < 1e-6
    # a CUDA-core kernel reports its product against the derived fp32 FMA peak instead
    c = bench.kernel_entry(ms, fwd, units, w.T, peaks, "measured", 1965.0, 1965.0, pipe="fma")
    assert "tensor" not in c and c["fma"]["peak_tflops"] == 148 * 128 * 2 * 1965.0 / 1e6
    assert bench.kernel_pipe("m2rnn_fwd_rows_kernel") == "fma" and bench.kernel_pipe("m2rnn_bwd_tc_kernel") == "tensor"


def test_kernel_digest_covers_the_shared_headers(tmp_path, monkeypatch):
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    (csrc / "k.cu").write_bytes(b"__global__ void k() {}\n")
    (csrc / "ptx.cuh").write_bytes(b"#define A 1\n")
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    d1 = bench.kernel_digest(bench.kernel_source("k.cu"))
    (csrc / "ptx.cuh").write_bytes(b"#define A 2\n")
    assert bench.kernel_digest(bench.kernel_source("k.cu")) != d1


@pytest.mark.parametrize("B,H,K,V", [(1, 16, 64, 64), (2, 16, 64, 64), (8, 16, 64, 64), (2, 3, 64, 64),
                                     (1, 16, 128, 64), (1, 4, 16, 64), (2, 3, 64, 32), (4, 32, 128, 128)])
def test_forward_kernel_rule_matches_the_library(B, H, K, V):
    """bench.forward_kernel mirrors the library's dispatch; the library shows
    its choice in the forward workspace: the row kernel keeps K/8 partial
    readouts per pair, the tensor-core kernel at most K/16."""
    from non_linear_matrix_persistent_b200 import _lib, build
    build.build()
    T = 5
    w = WORKLOADS["layer410m_fwd"].with_(B=B, H=H, K=K, V=V, T=T)
    ws = _lib.lib().m2rnn_workspace_size(_lib.Dims(B, H, T, K, V, 0, 16, 0, 0), 0)
    rows = ws == 256 + (K // 8) * B * H * T * V * 4
    assert (bench.forward_kernel(w)[0] == "m2rnn_fwd_rows_kernel") == rows
    assert bench.profile_name(bench.forward_kernel(w)[0], "x") in ("m2rnn_fwd_rows_x.md", "m2rnn_fwd_tc_x.md")


def test_backward_kernel_rule():
    w = WORKLOADS["layer410m_train"]
    assert bench.backward_kernel(w) == ("m2rnn_bwd_tc_kernel", "bwd_tc.cu")
    assert bench.backward_kernel(WORKLOADS["layer7b_moe_train"]) == ("m2rnn_bwd_tcg_kernel", "bwd_tcg.cu")
    assert bench.backward_kernel(w.with_(K=16)) == ("m2rnn_bwd_tcg_kernel", "bwd_tcg.cu")
    # the extended-operand kernel's scratch holds 8 steps at K = 64, 128 and 16 at K = 32
    assert bench.backward_kernel(w.with_(ckpt_stride=16)) == ("m2rnn_bwd_tcg_kernel", "bwd_tcg.cu")
    assert bench.backward_kernel(w.with_(K=128)) == ("m2rnn_bwd_tc_kernel", "bwd_tc.cu")
    assert bench.backward_kernel(w.with_(K=32, ckpt_stride=16)) == ("m2rnn_bwd_tc_kernel", "bwd_tc.cu")
