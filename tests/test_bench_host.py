"""Host logic of bench.py that needs no GPU: a DRAM-traffic figure recorded
from an ncu capture is used only while the kernel's source file and the device
headers beside it are unchanged."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_recorded_traffic_goes_stale_with_kernel_or_header(tmp_path, monkeypatch):
    csrc = tmp_path / "test_sequence_layers_layer_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel v1")
    (csrc / "a.cuh").write_text("header v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha("k.cu")
    (tmp_path / "profiles" / "k_kernel__w.md").write_text(
        f"traffic: kernel=k_kernel workload=w bytes_per_launch=1234 source_sha={sha}\n")

    def current():
        return bench.recorded_traffic("k_kernel", "w", bench.source_sha("k.cu"))

    assert current() == 1234.0
    assert bench.recorded_traffic("k_kernel", "other_workload", sha) is None
    (csrc / "a.cuh").write_text("header v2")  # a device header changed
    assert current() is None
    (csrc / "a.cuh").write_text("header v1")
    assert current() == 1234.0
    (csrc / "k.cu").write_text("kernel v2")  # the kernel itself changed
    assert current() is None


def test_workload_accounting():
    """Bytes and FLOPs per token that the roofline divides by, from the
    shapes: Z costs 4 bytes an element, 2 with a bf16 Z; the large-chunk
    read-out moves Q in and Z out; the backward does 20 d^2 FLOPs a token."""
    from test_sequence_layers_layer_b200 import synth
    lin = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
    d = lin.d
    fp32_z = bench.algo_bytes_per_token(lin)
    assert fp32_z == 3 * d * 2 + 4 + 4 * d + 2 * 4 * d * d / lin.T
    assert bench.algo_bytes_per_token(lin, 2) == fp32_z - 2 * d
    ch = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"]
    plan = {p[0]: p for p in bench.kernel_plan(ch)}
    plan16 = {p[0]: p for p in bench.kernel_plan(ch, 2)}
    kv_eta_w = 2 * ch.d * 2 + 4 + 8 * ch.d * ch.d / ch.T  # K, V, eta in; W0 in, W_out out
    assert plan["chunk_fwd_kernel"][3] == kv_eta_w + ch.d * 2 + 4 * ch.d  # Q in, Z out
    assert plan16["chunk_fwd_kernel"][3] == kv_eta_w + ch.d * 2 + 2 * ch.d
    assert plan["chunk_fwd_kernel"][4] == 6 * ch.d ** 2 + 2 * ch.d ** 3 / ch.b
    assert bench.bwd_flops_per_token(64) == 20 * 64 * 64
    assert bench.bwd_bytes_per_token(lin) == 3 * d * 2 + 4 * d + 4 + 3 * 4 * d + 4


def test_latency_floor_accounting():
    """One dependent step = scan time / (waves * ceil(T/b)): one CTA per
    sequence, one CTA per SM."""
    from test_sequence_layers_layer_b200 import synth
    lin = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
    f = bench.latency_floor(lin, bench.kernel_plan(lin), [0.256])
    assert f["dependent_steps"] == 128 and f["waves"] == 1 and f["concurrent_sequences"] == 96
    assert abs(f["us_per_minibatch_step"] - 2.0) < 1e-12
    big = lin.scaled(B=32, T=2047)  # 384 sequences: 3 waves; 128 steps with a partial last one
    f = bench.latency_floor(big, bench.kernel_plan(big), [3.0])
    assert f["waves"] == 3 and f["dependent_steps"] == 128
    ch = synth.WORKLOADS["chunk_d128_c2048_b4h8_t32768"]
    f = bench.latency_floor(ch, bench.kernel_plan(ch), [0.032])
    assert f["kernel"] == "chunk_fwd_kernel" and f["dependent_steps"] == 16
    assert abs(f["us_per_minibatch_step"] - 2.0) < 1e-12 and "upper bound" in f["note"]
    mlp = synth.WORKLOADS["mlp_ln_d64_dh256_b4h12_t8192"]
    f = bench.latency_floor(mlp, bench.kernel_plan(mlp), [1.0])
    assert f["concurrent_sequences"] == 48 and f["waves"] == 1
    assert isinstance(bench.cpu_model(), str)


def test_segments_option_is_checked_before_any_gpu_work():
    import subprocess
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload",
            "chunk_d128_c2048_b4h8_t32768"]
    r = subprocess.run(base + ["--segments", "3"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "does not split" in r.stderr
    r = subprocess.run(base[:2] + ["--workload", "linear_ln_d64_b8h12_t2048", "--segments", "2"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "large-chunk" in r.stderr


def test_mlp_backward_flop_count():
    """24 products of 2 d dh FLOPs per token (checkpoint forward 5, recompute
    5, token backward 11, end-of-mini-batch weight terms 3)."""
    assert bench.mlp_bwd_flops_per_token(64, 256) == 24 * 2 * 64 * 256


def test_bench_parity_on_the_oracle_sample():
    """The bench's parity figure compares the sampled sequences only, per
    output, as max |gpu - ref| / max |ref|."""
    import numpy as np
    import torch
    from test_sequence_layers_layer_b200 import synth
    wl = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"].scaled(B=2, H=2, T=8)
    r = np.random.default_rng(0)
    Zr = r.standard_normal((2, 2, 8, 64))
    Wr = r.standard_normal((2, 2, 64, 64))
    Zg, Wg = Zr.copy(), Wr.copy()
    Zg[0, 1, 3, 5] += 1e-3 * np.abs(Zr).max()      # sequence 1 is sampled
    Wg[1, 1, 0, 0] += 0.5                           # sequence 3 is not
    outs = (torch.from_numpy(Zg).float(), torch.from_numpy(Wg).float())
    p = bench.bench_parity(wl, outs, {"seqs": [0, 1], "ref": (Zr, Wr)})
    assert p["sequences"] == 2 and p["of"] == 4 and p["tolerance"] == 2e-3
    assert abs(p["z_max_rel_err"] - 1e-3) < 1e-5
    assert p["w_out_max_rel_err"] < 1e-6
    mlp = synth.WORKLOADS["mlp_ln_d64_dh256_b4h12_t8192"]
    assert "note" in bench.bench_parity(mlp, None, None)
