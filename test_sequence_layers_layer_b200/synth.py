"""Seeded synthetic inputs for the TTT-layer forward pass.

This module only draws numbers. It holds none of the layer's arithmetic, so
both the CUDA path and the CPU oracle can be fed from it without sharing any
computation.

Generator: a counter-based SplitMix64 stream per (seed, tensor id), the
construction of Steele, Lea and Flood ("Fast splittable pseudorandom number
generators", OOPSLA 2014) with Vigna's published finaliser constants. Element
i of a stream uses counters 2i and 2i+1; their top 53 bits become uniforms in
(0, 1) and one Box-Muller transform turns the pair into one standard normal.

Workload recipes follow the five workloads the TTT pages motivate (TTT-Linear
with and without LayerNorm, a long-context run, TTT-MLP, and large-chunk
apply-then-update); their value distributions are:
Q, K, V ~ N(0, 1)/sqrt(d); fast weights ~ N(0, 0.02^2); LayerNorm gain
1 + N(0, 0.02^2) and bias N(0, 0.02^2); per-token inner step size
eta_t = base * sigmoid(u_t)/d with u_t ~ N(0, 1) (base 1, or 0.1 for the MLP),
or a constant.
bf16 tensors are the round-to-nearest-even bf16 values of the fp32 draws.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids of the streams, fixed in this order.
TID_Q, TID_K, TID_V, TID_U, TID_W1, TID_W2, TID_GAMMA, TID_BETA = range(8)

_BLOCK = 1 << 22  # elements generated per numpy block


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser (wrapping uint64 arithmetic), in place."""
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, tid: int) -> np.uint64:
    """Starting state of the stream for tensor `tid` under `seed`."""
    with np.errstate(over="ignore"):
        base = np.array([(int(seed) << 8) | int(tid)], dtype=np.uint64)
        base += _GOLDEN
        return _mix64(base)[0]


def uniforms(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in (0, 1) for counters start .. start+count-1."""
    key = stream_key(seed, tid)
    x = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x *= _GOLDEN
        x += key
    _mix64(x)
    x >>= np.uint64(11)
    u = x.astype(np.float64)
    u += 0.5
    u *= 2.0 ** -53
    return u


def normals(seed: int, tid: int, n: int) -> np.ndarray:
    """n standard normals (float64) of stream (seed, tid)."""
    out = np.empty(n, dtype=np.float64)

    def block(lo):
        cnt = min(_BLOCK, n - lo)
        u = uniforms(seed, tid, 2 * lo, 2 * cnt)
        r = np.log(u[0::2])
        r *= -2.0
        np.sqrt(r, out=r)
        c = u[1::2] * (2.0 * math.pi)
        np.cos(c, out=c)
        np.multiply(r, c, out=out[lo:lo + cnt])

    starts = range(0, n, _BLOCK)
    if n > _BLOCK:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(block, starts))
    else:
        for lo in starts:
            block(lo)
    return out


def round_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round fp32 values to bf16, nearest-even.

    Returns (values as float32, exactly representable in bf16; raw bf16 bits
    as uint16)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    bits = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    hi = (bits >> np.uint64(16)).astype(np.uint16)
    vals = bits.astype(np.uint32).view(np.float32)
    return vals.reshape(f.shape), hi.reshape(f.shape)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, the form of f, dtype and eta recipe."""
    name: str
    kind: str           # "linear" | "mlp" | "chunk"
    B: int
    H: int
    T: int
    d: int
    b: int              # mini-batch (linear, mlp) or chunk (chunk) size
    ln: bool            # f(k) = k + LN(...) when True
    dtype: str          # "fp32" | "bf16" (dtype of Q, K, V)
    eta: str            # "const:<value>" | "sigmoid_over_d" | "sigmoid_over_d:<base>"
    dh: int = 0         # MLP hidden width
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.T

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Names state what each is and its sizes.
WORKLOADS = {
    "linear_fp32_d16": Workload("linear_fp32_d16", "linear", B=1, H=1, T=64, d=16, b=16,
                                ln=False, dtype="fp32", eta="const:0.1"),
    "linear_ln_d64_b8h12_t2048": Workload("linear_ln_d64_b8h12_t2048", "linear", B=8, H=12,
                                          T=2048, d=64, b=16, ln=True, dtype="bf16",
                                          eta="sigmoid_over_d"),
    "linear_ln_d64_b1h32_t32768": Workload("linear_ln_d64_b1h32_t32768", "linear", B=1, H=32,
                                           T=32768, d=64, b=16, ln=True, dtype="bf16",
                                           eta="sigmoid_over_d"),
    "mlp_ln_d64_dh256_b4h12_t8192": Workload("mlp_ln_d64_dh256_b4h12_t8192", "mlp", B=4, H=12,
                                             T=8192, d=64, b=16, ln=True, dtype="bf16",
                                             eta="sigmoid_over_d", dh=256),
    "chunk_d128_c2048_b4h8_t32768": Workload("chunk_d128_c2048_b4h8_t32768", "chunk", B=4, H=8,
                                             T=32768, d=128, b=2048, ln=False, dtype="bf16",
                                             eta="const:0.00048828125"),
}


@dataclasses.dataclass
class Inputs:
    """Host arrays of one workload. Q, K, V are float32 (bf16-exact when the
    workload is bf16); *_bits hold the raw bf16 bits for the device."""
    wl: Workload
    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    eta: np.ndarray
    W1: np.ndarray
    W2: np.ndarray | None
    gamma: np.ndarray
    beta: np.ndarray
    Q_bits: np.ndarray | None = None
    K_bits: np.ndarray | None = None
    V_bits: np.ndarray | None = None


def _qkv(wl: Workload, tid: int):
    n = wl.B * wl.H * wl.T * wl.d
    x = (normals(wl.seed, tid, n) / math.sqrt(wl.d)).astype(np.float32)
    x = x.reshape(wl.B, wl.H, wl.T, wl.d)
    if wl.dtype == "bf16":
        vals, bits = round_bf16(x)
        return vals, bits
    return x, None


def make_inputs(wl: Workload) -> Inputs:
    """Draw every input of workload `wl` (deterministic in wl.seed)."""
    Q, Qb = _qkv(wl, TID_Q)
    K, Kb = _qkv(wl, TID_K)
    V, Vb = _qkv(wl, TID_V)
    if wl.eta.startswith("const:"):
        eta = np.full((wl.B, wl.H, wl.T), float(wl.eta[6:]), dtype=np.float32)
    elif wl.eta == "sigmoid_over_d" or wl.eta.startswith("sigmoid_over_d:"):
        base = float(wl.eta.split(":")[1]) if ":" in wl.eta else 1.0
        u = normals(wl.seed, TID_U, wl.B * wl.H * wl.T)
        eta = (base * (1.0 / (1.0 + np.exp(-u))) / wl.d).astype(np.float32)
        eta = eta.reshape(wl.B, wl.H, wl.T)
    else:
        raise ValueError(f"unknown eta recipe {wl.eta!r}")
    if wl.kind == "mlp":
        W1 = (0.02 * normals(wl.seed, TID_W1, wl.H * wl.d * wl.dh)).astype(np.float32)
        W1 = W1.reshape(wl.H, wl.d, wl.dh)
        W2 = (0.02 * normals(wl.seed, TID_W2, wl.H * wl.dh * wl.d)).astype(np.float32)
        W2 = W2.reshape(wl.H, wl.dh, wl.d)
    else:
        W1 = (0.02 * normals(wl.seed, TID_W1, wl.H * wl.d * wl.d)).astype(np.float32)
        W1 = W1.reshape(wl.H, wl.d, wl.d)
        W2 = None
    gamma = (1.0 + 0.02 * normals(wl.seed, TID_GAMMA, wl.H * wl.d)).astype(np.float32)
    beta = (0.02 * normals(wl.seed, TID_BETA, wl.H * wl.d)).astype(np.float32)
    return Inputs(wl, Q, K, V, eta, W1, W2, gamma.reshape(wl.H, wl.d),
                  beta.reshape(wl.H, wl.d), Qb, Kb, Vb)
