#!/usr/bin/env python
"""Benchmark of the TTT-layer forward pass on B200 (libttt.so through its C ABI).

Default workload: large-chunk TTT with a linear fast weight, d = 128, chunk
2048, apply-then-update, eta = 1/2048, B = 4, H = 8, T = 32768, bf16 Q/K/V
(1,048,576 tokens per step): the largest single-GPU workload. `--workload`
selects the others (TTT-Linear + LN at d = 64, the long-context TTT-Linear,
TTT-MLP, the fp32 d = 16 case).
A step is one library call over one batch of seeded synthetic inputs that
are already resident in HBM; between timed steps a 256 MiB buffer is written
to flush the 126 MB L2. Steps are timed with CUDA events on the launching
stream; with several GPUs (one process each, torchrun) every rank runs its
own batch (different seed; weak scaling, no collective on the data path) and
the slowest rank's time is reported.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from test_sequence_layers_layer_b200 import synth  # noqa: E402

DEFAULT_WORKLOAD = "chunk_d128_c2048_b4h8_t32768"
METRIC = "TTT-layer fwd tokens/sec at 1 B200; % of dense bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- workload math

def weight_bytes(wl) -> int:
    return 4 * (2 * wl.d * wl.dh if wl.kind == "mlp" else wl.d * wl.d)


def algo_bytes_per_token(wl, zb: int = 4) -> float:
    """Interface bytes a token must move: Q, K, V in, eta in, Z out (zb bytes an
    element: 4 for fp32, 2 for bf16), plus the fast weight read once and
    written once per sequence, spread over T."""
    e = 2 if wl.dtype == "bf16" else 4
    return 3 * wl.d * e + 4 + zb * wl.d + 2 * weight_bytes(wl) / wl.T


def algo_flops_per_token(wl) -> float:
    """Dense-contraction FLOPs per token of the method (dual form): for the
    linear weight, K W, Q W and K^T G (2 d^2 each) plus the causal b x b terms;
    for the MLP, seven 2 d dh products plus the causal terms; for large
    chunks, Q W, K W and K^T G."""
    d, b = wl.d, wl.b
    if wl.kind == "linear":
        return 6 * d * d + 2 * (b + 1) * d
    if wl.kind == "mlp":
        return 14 * d * wl.dh + 10 * (b + 1) * d
    return 6 * d * d


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_plan(wl, zb: int = 4, tcgen05_mlp: bool = False):
    """Kernels one library call launches, in launch order:
    (name, source file, arithmetic type, algorithmic bytes/token, FLOPs/token)."""
    e = 2 if wl.dtype == "bf16" else 4
    d = wl.d
    if wl.kind == "chunk" and wl.dtype == "bf16" and d == 128 and wl.b % 128 == 0:
        # One launch: K, V and eta in, A_c | B_c = K^T [eta K | eta V]; the
        # scan W_{c+1} = W_c - A_c W_c + B_c (d^3 per chunk; W0 in, W_out
        # out); Q in, Z = Q W_c out.
        return [("chunk_fwd_kernel", "ttt_chunk_tc.cu", "bf16",
                 3 * d * e + 4 + zb * d + 8 * d * d / wl.T, 6 * d * d + 2 * d ** 3 / wl.b)]
    if wl.kind == "linear" and wl.dtype == "bf16" and d == 64 and wl.b == 16:
        return [("linear_ln_scan_kernel", "ttt_linear_tc.cu", "bf16", algo_bytes_per_token(wl, zb),
                 algo_flops_per_token(wl))]
    if wl.kind == "mlp" and wl.dtype == "bf16" and d == 64 and wl.dh == 256 and wl.b == 16:
        if tcgen05_mlp:
            return [("mlp_umma_scan_kernel", "ttt_mlp_umma.cu", "bf16",
                     algo_bytes_per_token(wl, zb), algo_flops_per_token(wl))]
        return [("mlp_ln_scan_kernel", "ttt_mlp_tc.cu", "bf16", algo_bytes_per_token(wl, zb),
                 algo_flops_per_token(wl))]
    name = {"linear": "linear_simt_kernel", "mlp": "mlp_simt_kernel",
            "chunk": "chunk_simt_kernel"}[wl.kind]
    return [(name, "ttt_simt.cu", "f32", algo_bytes_per_token(wl, zb), algo_flops_per_token(wl))]


def source_sha(fname: str) -> str:
    """Hash of a kernel's source file together with the device headers (.cuh)
    beside it, so that a recorded ncu figure goes stale when either changes."""
    csrc = os.path.join(ROOT, "test_sequence_layers_layer_b200", "csrc")
    h = hashlib.sha256()
    for path in [os.path.join(csrc, fname)] + sorted(glob.glob(os.path.join(csrc, "*.cuh"))):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, sha: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/, valid
    only while the kernel's source is unchanged (same sha)."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    pat = re.compile(r"traffic: kernel=(\S+) workload=(\S+) bytes_per_launch=([0-9.e+]+) "
                     r"source_sha=(\S+)")
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        for line in open(os.path.join(pdir, fn)):
            m = pat.search(line)
            if m and m.group(1) == kernel and m.group(2) == workload and m.group(4) == sha:
                return float(m.group(3))
    return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running
    (reads only; changes no setting)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        reasons = sorted({name for _, _, rs in inside for bit, name in self.REASONS.items()
                          if rs & bit})
        return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside)}


# ----------------------------------------------------------------------------- GPU arm

def device_tensors(inp, dev):
    import torch

    def qkv(vals, bits):
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(vals).to(dev)

    x = dict(Q=qkv(inp.Q, inp.Q_bits), K=qkv(inp.K, inp.K_bits), V=qkv(inp.V, inp.V_bits),
             eta=torch.from_numpy(inp.eta).to(dev), W1=torch.from_numpy(inp.W1).to(dev),
             gamma=torch.from_numpy(inp.gamma).to(dev), beta=torch.from_numpy(inp.beta).to(dev),
             W2=torch.from_numpy(inp.W2).to(dev) if inp.W2 is not None else None)
    return x


def make_caller(wl, x, stream, z_bf16=False, tcgen05_mlp=False):
    """Returns (call, outputs) where call() enqueues one library call on `stream`."""
    import torch
    import test_sequence_layers_layer_b200 as ttt
    B, H, T, d = wl.B, wl.H, wl.T, wl.d
    dev = x["Q"].device
    dt = ttt.TTT_BF16 if wl.dtype == "bf16" else ttt.TTT_FP32
    Z = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32, device=dev)
    zf = ttt.TTT_F_Z_BF16 if z_bf16 else 0
    sp = stream.cuda_stream
    if wl.kind == "linear":
        Wo = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        flags = (ttt.TTT_F_LN if wl.ln else 0) | zf

        def call(x=x):
            ttt.ttt_linear_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                               Z, Wo, B, H, T, d, wl.b, dt, flags, sp)
        return call, (Z, Wo)
    if wl.kind == "mlp":
        W1o = torch.empty((B, H, d, wl.dh), dtype=torch.float32, device=dev)
        W2o = torch.empty((B, H, wl.dh, d), dtype=torch.float32, device=dev)

        fn = ttt.ttt_diag_mlp_fwd_tcgen05 if tcgen05_mlp else ttt.ttt_mlp_fwd

        def call(x=x):
            fn(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"], x["beta"], Z, W1o,
               W2o, B, H, T, d, wl.dh, wl.b, dt, ttt.TTT_F_LN | zf, sp)
        return call, (Z, W1o, W2o)
    Wo = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    need = ttt.ttt_chunk_workspace_bytes(B, H, T, d, wl.b)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)

    def call(x=x):
        ttt.ttt_chunk_fwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], Z, Wo, B, H, T, d, wl.b,
                          dt, zf, ws, need, sp)
    return call, (Z, Wo)


def rank_workload(wl, rank):
    """Weak scaling: every rank runs the whole workload on its own seeded
    inputs (its own independent sequences); no data moves between ranks."""
    return wl.scaled(seed=wl.seed + rank)


def reduce_across_ranks(total_ms, e2e_ms, launches, world, device):
    """Job-level figures from per-rank ones: the slowest rank's device time
    (MAX) and the launches of all ranks (SUM). Every rank takes both
    collectives in the same order."""
    if world <= 1:
        return total_ms, e2e_ms, launches
    import torch
    import torch.distributed as dist
    t = torch.tensor([total_ms, e2e_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    lc = torch.tensor([launches], dtype=torch.float64, device=device)
    dist.all_reduce(lc)
    return float(t[0]), float(t[1]), int(lc[0])


def aggregate(wl, world, steps, total_ms):
    """(tokens per step over all ranks, ms per step, whole-job tokens/s)."""
    tokens = wl.tokens * world
    return tokens, total_ms / steps, tokens * steps / (total_ms / 1e3)


SM_COUNT = 148


def latency_floor(wl, plan, kern_ms_per_call):
    """The sequential chain's cost: each sequence scans ceil(T/b) dependent
    mini-batch (or chunk) steps, one CTA (a 2-CTA cluster for the warp-level
    MMA TTT-MLP scan) per sequence, one CTA per SM. With w waves of
    sequences per launch the scan kernel's time divided by w * ceil(T/b) is
    the time of one dependent step. Returns a dict for the bench line."""
    idx = next((i for i, p in enumerate(plan) if "scan" in p[0]), len(plan) - 1)
    ctas = 2 if plan[idx][0] == "mlp_ln_scan_kernel" else 1
    nseq = wl.B * wl.H
    concurrent = min(nseq, SM_COUNT // ctas)
    waves = -(-nseq // concurrent)
    steps = -(-wl.T // wl.b)
    out = {"us_per_minibatch_step": kern_ms_per_call[idx] * 1e3 / (waves * steps),
           "dependent_steps": steps, "concurrent_sequences": concurrent, "waves": waves,
           "kernel": plan[idx][0]}
    if plan[idx][0] == "chunk_fwd_kernel":
        out["note"] = ("the scan shares its launch with the Gram products and the read-out: an "
                       "upper bound on one chunk step")
    return out


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def gpu_arm(args, wl, rank, world, keep=None):
    import torch
    import torch.distributed as dist
    import test_sequence_layers_layer_b200 as ttt

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    ttt.lib()
    peaks, peaks_src = load_peaks()
    inp = synth.make_inputs(rank_workload(wl, rank))
    x = device_tensors(inp, dev)
    stream = torch.cuda.Stream(dev)
    zb = 2 if args.z_bf16 else 4
    call, outs = make_caller(wl, x, stream, args.z_bf16, args.mlp_kernel == "tcgen05")
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[dev.index])

    plan = kernel_plan(wl, zb, args.mlp_kernel == "tcgen05")
    multi = len(plan) > 1
    sampler = ClockSampler(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            call()
        stream.synchronize()
        if ttt.ttt_device_status(stream.cuda_stream) != 0:
            raise RuntimeError("device status error after warm-up")
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        kern_tot = [0.0] * len(plan)
        if multi and (args.steps > 512 or args.steps * (len(plan) + 1) > 2048):
            raise SystemExit("--steps: at most 512 calls / 2048 kernel events are timed per run")
        if multi:
            # the library records events between its own launches on `stream`
            ttt.ttt_diag_kernel_timing(True)
        barrier()
        torch.cuda.synchronize()
        n0 = ttt.ttt_launch_count()
        t0 = time.perf_counter()
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            call()
            ends[k].record(stream)
        torch.cuda.synchronize()
        t1 = time.perf_counter()
        launches = ttt.ttt_launch_count() - n0
        if keep is not None:
            keep["outs"] = outs  # the last timed call's outputs, for the parity check
        if multi:
            # summed over the timed calls; read once, after the loop, so the
            # host never waits on the device inside it
            kern_tot = ttt.ttt_diag_kernel_times(len(plan))
            ttt.ttt_diag_kernel_timing(False)
            if len(kern_tot) != len(plan):
                raise RuntimeError(f"expected {len(plan)} kernels per call, got {len(kern_tot)}")
        barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    if not multi:
        kern_tot = [total_ms]

    # e2e through the C ABI with host buffers: pinned host -> device inputs,
    # the call, device -> pinned host outputs, every step.
    host_in = {k: v.cpu().pin_memory() for k, v in x.items() if v is not None}
    dev_in = {k: torch.empty_like(v) for k, v in x.items() if v is not None}
    call_e2e, outs_e2e = make_caller(wl, dev_in, stream, args.z_bf16, args.mlp_kernel == "tcgen05")
    host_out = [o.cpu().pin_memory() for o in outs_e2e if o is not None]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(o.numel() * o.element_size() for o in host_out)
    e2e_steps = max(3, min(args.steps, 10))
    slices = args.e2e_slices if args.e2e_slices is not None else 4
    sliced = slices > 0 and wl.kind in ("linear", "chunk")
    with torch.cuda.stream(stream):
        def e2e_step():
            for k, v in host_in.items():
                dev_in[k].copy_(v, non_blocking=True)
            call_e2e()
            for h, o in zip(host_out, [o for o in outs_e2e if o is not None]):
                h.copy_(o, non_blocking=True)
        if sliced:
            from test_sequence_layers_layer_b200 import hostio

            host_pair = (host_out[0], host_out[1])

            def e2e_step():  # noqa: F811  (copies overlapped across batch slices)
                if wl.kind == "chunk":
                    hostio.chunk_fwd_host(host_in["Q"], host_in["K"], host_in["V"], host_in["eta"],
                                          host_in["W1"], chunk=wl.b, slices=slices,
                                          z_bf16=args.z_bf16, out=host_pair)
                else:
                    hostio.linear_fwd_host(host_in["Q"], host_in["K"], host_in["V"], host_in["eta"],
                                           host_in["W1"], host_in.get("gamma"), host_in.get("beta"),
                                           b=wl.b, ln=wl.ln, slices=slices,
                                           z_bf16=args.z_bf16, out=host_pair)
        e2e_step()
        stream.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    sampler.stop()
    if ttt.ttt_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error in the timed region")

    total_ms, e2e_ms, launches = reduce_across_ranks(total_ms, e2e_ms, launches, world, dev)
    tokens, ms_per_step, value = aggregate(wl, world, args.steps, total_ms)
    # The dominant kernel: largest share of the timed device time. Its average
    # launch duration comes from CUDA events on the launching stream (the
    # step's own events when the call is one kernel).
    dom = max(range(len(plan)), key=lambda i: kern_tot[i])
    kname, ksrc, kdtype, kbytes, kflops = plan[dom]
    kern_ms = kern_tot[dom] / args.steps
    ai = kflops / kbytes
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if ai > ridge else "hbm"
    if bound == "hbm":
        per_launch = kbytes * wl.tokens
        achieved = per_launch / (kern_ms / 1e3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        per_launch = kflops * wl.tokens
        achieved = per_launch / (kern_ms / 1e3) / 1e12
        peak, unit = peaks["bf16_tflops"], "TFLOP/s"
    tflops = algo_flops_per_token(wl) * wl.tokens / (ms_per_step / 1e3) / 1e12
    sha = source_sha(ksrc)
    wname = (wl.name + ("_zbf16" if args.z_bf16 else "")
             + ("_tcgen05" if args.mlp_kernel == "tcgen05" and wl.kind == "mlp" else ""))
    traffic = recorded_traffic(kname, wname, sha)
    clocks = sampler.summary(t0, t1)
    kernels = [{"name": p[0], "ms_per_launch": kern_tot[i] / args.steps,
                "share": kern_tot[i] / max(sum(kern_tot), 1e-12)} for i, p in enumerate(plan)]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": kdtype,
        "data": "synthetic (seeded SplitMix64 normals; bf16-rounded Q/K/V)",
        "config": {"workload": wname, "B": wl.B, "H": wl.H, "T": wl.T, "d": wl.d,
                   "mini_batch": wl.b, "layer_norm": wl.ln, "qkv_dtype": wl.dtype,
                   "z_dtype": "bf16" if args.z_bf16 else "fp32",
                   "tokens_per_step_per_gpu": wl.tokens, "l2": "flushed between steps (256 MiB write)",
                   "parallelism": f"replicas x{world} (independent sequences)"},
        "pct_of_bf16_tensor_peak": 100.0 * tflops / peaks["bf16_tflops"],
        "pct_of_bf16_tensor_peak_sustained": 100.0 * tflops / peaks["bf16_tflops_sustained"],
        "algorithmic_tflops": tflops,
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                     "kernel": kname, "peak_source": peaks_src,
                     "algorithmic_per_launch": per_launch, "kernel_ms": kern_ms},
        "kernels": kernels,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copies": f"overlapped over {slices} slices of the (batch, head) grid (hostio)" if sliced
                else "in series with the call"},
        "gpu_launches": launches,
        "clocks": clocks,
        "step_ms_min_median": [min(step_ms), statistics.median(step_ms)],
        "latency_floor": latency_floor(wl, plan, [t / args.steps for t in kern_tot]),
    }
    return line


# ----------------------------------------------------------------------------- CPU (oracle) arm

def oracle_inputs(wl):
    """The workload's seeded inputs as float64 arrays, the oracle's input form."""
    inp = synth.make_inputs(wl)
    return {k: (np.asarray(getattr(inp, k), dtype=np.float64) if getattr(inp, k) is not None else None)
            for k in ("Q", "K", "V", "eta", "W1", "W2", "gamma", "beta")}


def oracle_sample(wl, budget_s: float, keep=None, f64=None):
    """Time the oracle on whole sequences of the workload, threaded over the
    host cores, growing the sample until about budget_s of work or the whole
    workload. Returns (tokens/s, cores, description); with `keep` (a dict),
    also leaves there the sampled sequences ("seqs") and the oracle's outputs
    of the last, largest sample ("ref"). `f64`: the inputs from
    oracle_inputs(wl), made here if not given (not part of the timing)."""
    import oracle

    if f64 is None:
        f64 = oracle_inputs(wl)
    cores = oracle.num_threads()
    nseq_total = wl.B * wl.H

    def run(seqs):
        t0 = time.perf_counter()
        if wl.kind == "linear":
            out = oracle.linear_primal(f64["Q"], f64["K"], f64["V"], f64["eta"], f64["W1"],
                                       f64["gamma"], f64["beta"], b=wl.b, ln=wl.ln, seqs=seqs,
                                       with_w=True)
        elif wl.kind == "mlp":
            out = oracle.mlp_primal(f64["Q"], f64["K"], f64["V"], f64["eta"], f64["W1"], f64["W2"],
                                    f64["gamma"], f64["beta"], b=wl.b, seqs=seqs)
        else:
            out = oracle.chunk_primal(f64["Q"], f64["K"], f64["V"], f64["eta"], f64["W1"],
                                      chunk=wl.b, seqs=seqs)
        el = time.perf_counter() - t0
        if keep is not None:
            keep["seqs"], keep["ref"] = list(seqs), out
        return el

    n = min(cores, nseq_total)
    dt = run(list(range(n)))
    while dt < budget_s / 4 and n < nseq_total:
        n = min(nseq_total, max(n * 2, int(n * budget_s / max(dt, 1e-3) / 2)))
        dt = run(list(range(n)))
    tok = n * wl.T
    desc = f"{n} of {nseq_total} sequences, full length T={wl.T} ({tok} tokens), {cores} threads"
    return tok / dt, cores, desc


def bench_parity(wl, outs, sample, z_bf16=False):
    """Max relative error (max |gpu - oracle| / max |oracle|, per output) of
    the timed call's outputs on the sequences the CPU-baseline leg ran through
    the oracle. `outs` are the call's output tensors ([B, H, ...]); `sample`
    holds "seqs" and "ref" from oracle_sample. Not computed for the TTT-MLP
    workload, whose exact recurrence is chaotic on some sequences (the
    parity tests compare it where it is conditioned)."""
    if wl.kind == "mlp":
        return {"note": "not computed for TTT-MLP: chaotic sequences (see the parity tests)"}
    seqs = sample["seqs"]
    S = wl.B * wl.H
    res = {"sequences": len(seqs), "of": S,
           "tolerance": 2e-3 if wl.dtype == "bf16" else 1e-5,
           "z_dtype": "bf16" if z_bf16 else "fp32"}
    for name, g, r in zip(("z", "w_out"), outs, sample["ref"]):
        gs = np.asarray(g.float().reshape(S, -1).cpu().numpy(), dtype=np.float64)[seqs]
        rs = np.asarray(r, dtype=np.float64).reshape(S, -1)[seqs]
        res[name + "_max_rel_err"] = float(np.abs(gs - rs).max() / max(np.abs(rs).max(), 1e-30))
    return res


def reference_arm(args, wl):
    vals = []
    cores, desc = None, None
    per_step_budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    f64 = oracle_inputs(wl)  # once: every step times the oracle on the same inputs
    for k in range(args.warmup + args.steps):
        v, cores, desc = oracle_sample(wl, per_step_budget, f64=f64)
        if k >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wl.tokens / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded SplitMix64 normals; bf16-rounded Q/K/V)",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T, "d": wl.d,
                   "mini_batch": wl.b},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main

def decode_arm(args, wl):
    """Single-token decode (b = 1 streaming): `--decode N` runs N one-token
    calls per sequence with the state updated in place, as a CUDA graph when
    capture works (else plain launches), and reports the time per step."""
    import torch
    import test_sequence_layers_layer_b200 as ttt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.decode
    dwl = wl.scaled(T=n, b=1)
    inp = synth.make_inputs(dwl)
    x = device_tensors(inp, dev)
    dt = ttt.TTT_BF16 if dwl.dtype == "bf16" else ttt.TTT_FP32
    flags = (ttt.TTT_F_LN if dwl.ln else 0) | ttt.TTT_F_W0_PER_SEQ
    toks = [{k: x[k][:, :, i:i + 1].contiguous() for k in ("Q", "K", "V", "eta")} for i in range(n)]
    state = x["W1"].unsqueeze(0).repeat(dwl.B, 1, 1, 1)
    W0 = state.clone()
    z = torch.empty((dwl.B, dwl.H, 1, dwl.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def steps():
        for t in toks:
            ttt.ttt_linear_fwd(t["Q"], t["K"], t["V"], t["eta"], state, x["gamma"], x["beta"], z,
                               state, dwl.B, dwl.H, 1, dwl.d, 1, dt, flags, stream.cuda_stream)

    if dwl.kind == "mlp":  # TTT-MLP: both layers' state per sequence, updated in place
        state2 = x["W2"].unsqueeze(0).repeat(dwl.B, 1, 1, 1)
        W0_2 = state2.clone()

        def steps():  # noqa: F811
            for t in toks:
                ttt.ttt_mlp_fwd(t["Q"], t["K"], t["V"], t["eta"], state, state2, x["gamma"],
                                x["beta"], z, state, state2, dwl.B, dwl.H, 1, dwl.d, dwl.dh, 1, dt,
                                ttt.TTT_F_LN | ttt.TTT_F_W0_PER_SEQ, stream.cuda_stream)

    if args.decode_one_call:  # all n tokens in one call, the weight on chip across them
        qkv = {k: x[k].contiguous() for k in ("Q", "K", "V", "eta")}
        zn = torch.empty((dwl.B, dwl.H, n, dwl.d), dtype=torch.float32, device=dev)

        def steps():  # noqa: F811
            if dwl.kind == "mlp":
                ttt.ttt_mlp_decode_tokens(qkv["Q"], qkv["K"], qkv["V"], qkv["eta"], state, state2,
                                          x["gamma"], x["beta"], zn, dwl.B, dwl.H, n, dwl.d,
                                          dwl.dh, dt, ttt.TTT_F_LN, stream.cuda_stream)
            else:
                ttt.ttt_linear_decode_tokens(qkv["Q"], qkv["K"], qkv["V"], qkv["eta"], state,
                                             x["gamma"], x["beta"], zn, dwl.B, dwl.H, n, dwl.d,
                                             dt, ttt.TTT_F_LN if dwl.ln else 0,
                                             stream.cuda_stream)
    elif args.decode_kernel and dwl.kind == "mlp":  # the one-token TTT-MLP kernel
        def steps():  # noqa: F811
            for t in toks:
                ttt.ttt_mlp_decode(t["Q"], t["K"], t["V"], t["eta"], state, state2, x["gamma"],
                                   x["beta"], z, dwl.B, dwl.H, dwl.d, dwl.dh, dt, ttt.TTT_F_LN,
                                   stream.cuda_stream)
    elif args.decode_kernel:  # the one-token kernel (W in registers); same buffers
        def steps():  # noqa: F811
            for t in toks:
                ttt.ttt_linear_decode(t["Q"], t["K"], t["V"], t["eta"], state, x["gamma"],
                                      x["beta"], z, dwl.B, dwl.H, dwl.d, dt,
                                      ttt.TTT_F_LN if dwl.ln else 0, stream.cuda_stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            steps()
        stream.synchronize()
        graph = None
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                steps()
            graph = g
        except Exception:
            graph = None
        state.copy_(W0)
        if dwl.kind == "mlp":
            state2.copy_(W0_2)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(1, args.steps)
        e0.record(stream)
        for _ in range(reps):
            if graph is not None:
                graph.replay()
            else:
                steps()
        e1.record(stream)
        stream.synchronize()
    if ttt.ttt_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error in the decode loop")
    us = e0.elapsed_time(e1) * 1e3 / (reps * n)
    return {
        "metric": ("TTT-MLP" if dwl.kind == "mlp" else "TTT-Linear")
                  + " single-token decode step (b = 1, state updated in place)",
        "value": us, "unit": "us/step", "higher_is_better": False,
        "tokens_per_s": dwl.B * dwl.H / (us * 1e-6),
        "n_gpus": 1, "steps": reps * n, "warmup": args.warmup, "dtype": dwl.dtype,
        "data": "synthetic (seeded SplitMix64 normals; bf16-rounded Q/K/V)",
        "config": {"workload": wl.name + "_decode", "B": dwl.B, "H": dwl.H, "d": dwl.d,
                   "layer_norm": dwl.ln, "tokens_per_step": dwl.B * dwl.H,
                   "cuda_graph": graph is not None,
                   "entry_point": ((("ttt_mlp_decode_tokens" if dwl.kind == "mlp"
                                     else "ttt_linear_decode_tokens") + f" ({n} tokens, one call)")
                                   if args.decode_one_call else
                                   ("ttt_mlp_decode" if dwl.kind == "mlp" else "ttt_linear_decode")
                                   if args.decode_kernel else
                                   ("ttt_mlp_fwd" if dwl.kind == "mlp" else "ttt_linear_fwd")
                                   + " (T = 1, b = 1)")},
    }


def segmented_arm(args, wl):
    """`--segments N` (large-chunk workloads): the forward split into N
    segments of whole chunks per sequence on one GPU
    (seqpar.chunk_fwd_segmented: segment maps, their fold, the segments'
    forwards). L2 flushed between steps. Reports tokens/s of the whole call
    and the device time of each of its three stages."""
    import torch
    import test_sequence_layers_layer_b200 as ttt
    from test_sequence_layers_layer_b200 import seqpar

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nseg = args.segments
    B, H, T, d, C = wl.B, wl.H, wl.T, wl.d, wl.b
    x = device_tensors(synth.make_inputs(wl), dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    Ts = T // nseg
    view = {k: x[k].view(B, H * nseg, Ts, d) for k in ("Q", "K", "V")}
    view["eta"] = x["eta"].view(B, H * nseg, Ts)

    def call():
        return seqpar.chunk_fwd_segmented(x["Q"], x["K"], x["V"], x["eta"], x["W1"], chunk=C,
                                          nseg=nseg, z_bf16=args.z_bf16, stream=stream)

    def stages(ev):
        ev[0].record(stream)
        M, N = ttt.chunk_map(view["K"], view["V"], view["eta"], chunk=C, stream=stream)
        ev[1].record(stream)
        W_in = torch.empty_like(M)
        W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        ttt.affine_prefix(M, N, x["W1"], W_in, W_out, S=B * H, H=H, nseg=nseg,
                          seq_stride=nseg * d * d, seg_stride=d * d, stream=stream)
        ev[2].record(stream)
        ttt.chunk_fwd(view["Q"], view["K"], view["V"], view["eta"], W_in, chunk=C,
                      w0_per_seq=True, stream=stream, want_w=False, z_bf16=args.z_bf16)
        ev[3].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            call()
        stream.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        n0 = ttt.ttt_launch_count()
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            call()
            ends[k].record(stream)
        stream.synchronize()
        launches = ttt.ttt_launch_count() - n0
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for k in range(args.steps):
            flush.zero_()
            stages(evs[k])
        stream.synchronize()
    if ttt.ttt_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error in the segmented loop")
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    stage_ms = [sum(ev[i].elapsed_time(ev[i + 1]) for ev in evs) / args.steps for i in range(3)]
    return {
        "metric": "large-chunk TTT forward, sequence split into segments, tokens/s at 1 B200",
        "value": wl.tokens / (ms / 1e3), "unit": "tokens/s", "higher_is_better": True,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "dtype": wl.dtype, "data": "synthetic (seeded SplitMix64 normals; bf16-rounded Q/K/V)",
        "config": {"workload": f"{wl.name}_seg{nseg}", "B": B, "H": H, "T": T, "d": d,
                   "chunk": C, "segments": nseg, "z_dtype": "bf16" if args.z_bf16 else "fp32",
                   "l2": "flushed between steps (256 MiB write)"},
        "stages_ms": {"segment_maps": stage_ms[0], "fold": stage_ms[1],
                      "segment_forwards": stage_ms[2]},
        "dependent_steps": {"fold": nseg - 1, "chunk_scan": T // (nseg * C)},
        "gpu_launches": launches,
    }


# fp32 FMA lanes of a B200 (148 SMs x 128 lanes, 2 FLOP per FMA) at the SM clock:
# the peak of a kernel bound by plain fp32 arithmetic on CUDA cores.
FP32_LANES = 148 * 128


def mlp_bwd_flops_per_token(d: int, dh: int) -> float:
    """Algorithmic FLOPs of the TTT-MLP backward per token, counting its d x dh
    products (2 d dh FLOPs each): the checkpoint forward (k W1, a W2, Gx W2^T
    and the two weight updates: 5), the key side and read-out recomputed in the
    reverse pass (5), the token's read-out backward and second-order term
    (dxq W2^T, dhq W1^T, the two rank-one Phi updates, k Phi1, a Phi2, dga W2,
    dx W2^T, Phi2 Gx, Phi1 Gh, dh W1^T: 11) and the end-of-mini-batch weight
    terms (3): 24 products. The O(b (d + dh)) dual sums are left out."""
    return 48.0 * d * dh


def bwd_flops_per_token(d: int) -> float:
    """Algorithmic FLOPs of the TTT-Linear backward per token: the forward
    re-run (k W, and the K^T G update: 4 d^2) and the reverse step (k W and q W,
    dzpre W^T, G Om^T, k Om, dx W^T, and the two weight-gradient outer products:
    16 d^2); the O(b d) causal terms are left out."""
    return 20.0 * d * d


def chunk_bwd_flops_per_token(d: int, chunk: int) -> float:
    """Large-chunk backward: the three per-chunk Gram products (A_c, B_c,
    Q^T dZ: 6 d^2), the two affine scans (2 d^3 each per chunk, spread over
    the chunk's tokens) and the five per-token products (R, P, dQ and the two
    terms of dK: 10 d^2)."""
    return 16.0 * d * d + 4.0 * d ** 3 / chunk


def bwd_bytes_per_token(wl) -> float:
    """Algorithmic HBM bytes per token: Q, K, V in once, dZ and eta in, dQ, dK,
    dV and deta out (the W_m checkpoints are the kernel's choice, not counted)."""
    e = 2 if wl.dtype == "bf16" else 4
    return 3 * wl.d * e + 4 * wl.d + 4 + 3 * 4 * wl.d + 4


def backward_arm(args, wl):
    """Backward pass (`--backward`): ttt_linear_bwd, ttt_chunk_bwd or
    ttt_mlp_bwd on the workload's inputs with a seeded dZ, all resident in
    HBM, L2 flushed between steps."""
    import torch
    import test_sequence_layers_layer_b200 as ttt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ttt.lib()
    inp = synth.make_inputs(wl)
    x = device_tensors(inp, dev)
    rng = np.random.default_rng(wl.seed + 101)
    dZ = torch.from_numpy(rng.standard_normal((wl.B, wl.H, wl.T, wl.d)).astype(np.float32)).to(dev)
    chunk, mlp = wl.kind == "chunk", wl.kind == "mlp"
    if mlp:
        need = ttt.ttt_mlp_bwd_workspace_bytes(wl.B, wl.H, wl.T, wl.d, wl.dh, wl.b)
    else:
        need = (ttt.ttt_chunk_bwd_workspace_bytes if chunk else ttt.ttt_linear_bwd_workspace_bytes)(
            wl.B, wl.H, wl.T, wl.d, wl.b)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = [torch.empty((wl.B, wl.H, wl.T, wl.d), **f32) for _ in range(3)]
    geta = torch.empty((wl.B, wl.H, wl.T), **f32)
    gW0 = torch.empty(tuple(x["W1"].shape), **f32)
    gW2 = torch.empty(tuple(x["W2"].shape), **f32) if mlp else None
    gg, gb = torch.empty((wl.H, wl.d), **f32), torch.empty((wl.H, wl.d), **f32)
    dt = ttt.TTT_BF16 if wl.dtype == "bf16" else ttt.TTT_FP32
    flags = ttt.TTT_F_LN if wl.ln else 0
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def call():
        if mlp:
            ttt.ttt_mlp_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["W2"], x["gamma"],
                            x["beta"], dZ, None, None, *g, geta, gW0, gW2, gg, gb, wl.B, wl.H,
                            wl.T, wl.d, wl.dh, wl.b, dt, ttt.TTT_F_LN, ws, need,
                            stream.cuda_stream)
        elif chunk:
            ttt.ttt_chunk_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], dZ, None, *g, geta, gW0,
                              wl.B, wl.H, wl.T, wl.d, wl.b, dt, 0, ws, need, stream.cuda_stream)
        else:
            ttt.ttt_linear_bwd(x["Q"], x["K"], x["V"], x["eta"], x["W1"], x["gamma"], x["beta"],
                               dZ, None, *g, geta, gW0, gg, gb, wl.B, wl.H, wl.T, wl.d, wl.b, dt,
                               flags, ws, need, stream.cuda_stream)

    sampler = ClockSampler(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            call()
        stream.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ttt.ttt_diag_kernel_timing(True)
        n0 = ttt.ttt_launch_count()
        t0 = time.perf_counter()
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            call()
            ends[k].record(stream)
        torch.cuda.synchronize()
        t1 = time.perf_counter()
        launches = ttt.ttt_launch_count() - n0
        kern = ttt.ttt_diag_kernel_times(8)
        ttt.ttt_diag_kernel_timing(False)
    sampler.stop()
    if ttt.ttt_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device status error in the timed region")
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms = sum(step_ms) / args.steps
    # the large-chunk FLOP count covers all its kernels, so it is divided by
    # their summed time
    kern_ms = (sum(kern) if chunk else kern[0]) / args.steps
    tc_gram = chunk and wl.d == 128 and wl.dtype == "bf16" and wl.b % 32 == 0
    tc_tok = tc_gram and wl.b % 128 == 0
    chunk_names = (["cb_gram_tc_kernel", "cb_scan_tc_kernel"] if tc_gram
                   else ["cb_gram_kernel", "cb_scan_kernel"])
    chunk_names = (chunk_names
                   + (["cb_tok_tc_kernel<RP>", "cb_tok_tc_kernel<DK>", "cb_tok_tc_kernel<DQ>"]
                      if tc_tok else ["cb_tok_kernel"]) + ["cb_sum_over_batch_kernel (dW0)"])
    knames = (chunk_names
              if chunk else ["mlp_bwd_kernel", "mlp_bwd_sum_kernel"] if mlp
              else ["linear_bwd_kernel", "sum_over_batch_kernel (dW0)",
                    "sum_over_batch_kernel (dgamma)", "sum_over_batch_kernel (dbeta)"])
    clocks = sampler.summary(t0, t1)
    mhz = clocks.get("sm_mhz") or 1965
    peak = FP32_LANES * 2 * mhz * 1e6 / 1e12
    flop = (chunk_bwd_flops_per_token(wl.d, wl.b) if chunk
            else mlp_bwd_flops_per_token(wl.d, wl.dh) if mlp else bwd_flops_per_token(wl.d)) * wl.tokens
    achieved = flop / (kern_ms / 1e3) / 1e12
    line = {
        "metric": ("Large-chunk TTT" if chunk else "TTT-MLP" if mlp else "TTT-Linear") +
                  " backward tokens/sec at 1 B200 (outer gradients of every input)",
        "value": wl.tokens / (ms / 1e3), "unit": "tokens/s", "higher_is_better": True,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "dtype": "f32", "data": "synthetic (seeded SplitMix64 normals; bf16-rounded Q/K/V; normal dZ)",
        "config": {"workload": wl.name + "_backward", "B": wl.B, "H": wl.H, "T": wl.T, "d": wl.d,
                   "mini_batch": wl.b, "layer_norm": wl.ln, "qkv_dtype": wl.dtype,
                   "l2": "flushed between steps (256 MiB write)"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": ("all backward kernels" if chunk
                                else "mlp_bwd_kernel" if mlp else "linear_bwd_kernel"),
                     "peak_source": f"derived: {FP32_LANES} fp32 lanes x 2 FLOP x {mhz} MHz",
                     "algorithmic_per_launch": flop, "kernel_ms": kern_ms,
                     "hbm_bytes_per_token": None if mlp else bwd_bytes_per_token(wl)},
    }
    # With the products on the tensor cores the fp32 ALU roofline no longer
    # bounds the call: the unavoidable HBM traffic against the copy peak.
    if tc_tok:
        peaks, peaks_src = load_peaks()
        hb = bwd_bytes_per_token(wl) * wl.tokens
        ach = hb / (kern_ms / 1e3) / 1e9
        line_roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "all backward kernels", "peak_source": peaks_src,
                     "algorithmic_per_launch": hb, "kernel_ms": kern_ms,
                     "note": ("Gram, scans and per-token products on the tensor cores; bytes are "
                              "the inputs and gradients only (not the per-chunk workspace)"),
                     "tflops_algorithmic": achieved}
    else:
        line_roof = None
    line.update({
        "kernels": [{"name": n, "ms_per_launch": t / args.steps} for n, t in zip(knames, kern)],
        "gpu_launches": launches,
        "clocks": clocks,
        "step_ms_min_median": [min(step_ms), statistics.median(step_ms)],
    })
    if line_roof is not None:
        line["roofline"] = line_roof
    if not args.no_cpu_baseline and mlp:
        from oracle import backward as ob
        sub = wl.scaled(B=1, H=1, T=min(wl.T, 4 * wl.b))
        si = synth.make_inputs(sub)
        dz = rng.standard_normal((1, 1, sub.T, sub.d))
        t0 = time.perf_counter()
        ob.mlp_grads(si.Q, si.K, si.V, si.eta, si.W1, si.W2, si.gamma, si.beta, dz, b=sub.b)
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": sub.T / el, "unit": "tokens/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"1 sequence, T={sub.T}: float64 autograd backward"}
    if not args.no_cpu_baseline and not chunk and not mlp:
        from oracle import backward as ob
        sub = wl.scaled(B=1, H=1, T=min(wl.T, 512))
        si = synth.make_inputs(sub)
        dz = rng.standard_normal((1, 1, sub.T, sub.d))
        t0 = time.perf_counter()
        ob.linear_grads(si.Q, si.K, si.V, si.eta, si.W1, si.gamma, si.beta, dz, None, b=sub.b,
                        ln=sub.ln)
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": sub.T / el, "unit": "tokens/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"1 sequence, T={sub.T}: float64 autograd backward"}
    return line


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ttt", choices=["ttt", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--z-bf16", action="store_true",
                    help="store Z as bf16 (TTT_F_Z_BF16) instead of fp32")
    ap.add_argument("--backward", action="store_true",
                    help="time the TTT-Linear backward (linear workloads) instead")
    ap.add_argument("--decode", type=int, default=0,
                    help="time N single-token decode steps (linear workloads) instead")
    ap.add_argument("--decode-kernel", action="store_true",
                    help="with --decode: time the one-token kernel (ttt_linear_decode, "
                         "ttt_mlp_decode)")
    ap.add_argument("--decode-one-call", action="store_true",
                    help="with --decode N: all N tokens in one call with the weight on chip "
                         "(ttt_linear_decode_tokens, ttt_mlp_decode_tokens)")
    ap.add_argument("--e2e-slices", type=int, default=None,
                    help="e2e leg (linear and large-chunk workloads): overlap the host copies with "
                         "the compute over N slices of the (batch, head) grid (hostio.linear_fwd_host, "
                         "hostio.chunk_fwd_host); default 4, 0 = copies in series with one call")
    ap.add_argument("--segments", type=int, default=0,
                    help="time the large-chunk forward split into N segments per sequence")
    ap.add_argument("--mlp-kernel", default="default", choices=["default", "tcgen05"],
                    help="TTT-MLP workload: time the single-issuer tensor-core kernel "
                         "(ttt_diag_mlp_fwd_tcgen05) instead of ttt_mlp_fwd")
    ap.add_argument("--B", type=int, default=None,
                    help="override the workload's batch size (smaller profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.B:
        wl = wl.scaled(B=args.B, name=f"{wl.name}_B{args.B}")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.backward:
        if rank == 0:
            print(json.dumps(backward_arm(args, wl)), flush=True)
        return

    if args.decode:
        if wl.kind == "chunk":
            ap.error("--decode times the TTT-Linear and TTT-MLP workloads")

        if rank == 0:
            print(json.dumps(decode_arm(args, wl)), flush=True)
        return

    if args.segments:
        if wl.kind != "chunk":
            ap.error("--segments times the large-chunk workloads")
        if args.segments < 1 or wl.T % (args.segments * wl.b):
            ap.error(f"--segments {args.segments}: T = {wl.T} does not split into segments of "
                     f"whole chunks of {wl.b}")
        if rank == 0:
            print(json.dumps(segmented_arm(args, wl)), flush=True)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, wl)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        kept = {}
        line = gpu_arm(args, wl, rank, world, kept if (rank == 0 and world == 1) else None)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            sample = {}
            v, cores, desc = oracle_sample(wl, args.cpu_budget, sample)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores,
                                    "kind": "oracle", "sample": desc,
                                    "cpu_model": cpu_model()}
            try:  # a failure here must not cost the bench line
                line["parity"] = bench_parity(wl, kept["outs"], sample, args.z_bf16)
            except Exception as e:  # pragma: no cover - reported, not raised
                line["parity"] = {"error": repr(e)}
        elif rank == 0:
            line["cpu_baseline"] = None
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
