"""Python binding of libttt.so, the B200 library for a Test-Time-Training (TTT)
layer: its forward passes (TTT-Linear, TTT-MLP, large chunk), the backward
passes of TTT-Linear and large-chunk TTT, and the affine-map calls behind the
sequence-parallel large-chunk forward (seqpar.py).

The functions named like the C ABI (ttt_linear_fwd, ttt_mlp_fwd,
ttt_chunk_fwd, ...) take exactly the C arguments; a pointer argument may be a
torch tensor (its data_ptr() is passed), an int address, or None. They only
marshal arguments: every step of the computation runs in the library's CUDA
kernels. linear_fwd / mlp_fwd / chunk_fwd / linear_bwd / chunk_bwd /
chunk_map / affine_prefix are conveniences that read the shapes off torch
tensors and allocate the outputs (and workspaces) with torch.

There is no fallback: if libttt.so is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libttt.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "ttt.h")

TTT_OK = 0
TTT_BF16, TTT_FP32 = 0, 1
TTT_F_LN = 1
TTT_F_W0_PER_SEQ = 2
TTT_F_Z_BF16 = 4
TTT_F_L2_KEYS = 8

_P = ctypes.c_void_p
_I = ctypes.c_int
_lib = None


class TTTError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {status}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load libttt.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libttt.so not built at {LIB_PATH}; run build.py")
        L = ctypes.CDLL(LIB_PATH)
        L.ttt_abi_version.restype = _I
        L.ttt_abi_version.argtypes = []
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_status_string.argtypes = [_I]
        L.ttt_linear_fwd.restype = _I
        L.ttt_linear_fwd.argtypes = [_P] * 9 + [_I] * 6 + [ctypes.c_uint, _P]
        L.ttt_mlp_decode.restype = _I
        L.ttt_mlp_decode.argtypes = [_P] * 9 + [_I] * 5 + [ctypes.c_uint, _P]
        L.ttt_linear_decode.restype = _I
        L.ttt_linear_decode.argtypes = [_P] * 8 + [_I] * 4 + [ctypes.c_uint, _P]
        L.ttt_linear_fwd_steps.restype = _I
        L.ttt_linear_fwd_steps.argtypes = [_P] * 9 + [_I] * 6 + [ctypes.c_uint, _P]
        L.ttt_linear_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_linear_bwd_workspace_bytes.argtypes = [_I] * 5
        L.ttt_linear_bwd.restype = _I
        L.ttt_linear_bwd.argtypes = [_P] * 16 + [_I] * 6 + [ctypes.c_uint, _P, ctypes.c_size_t, _P]
        L.ttt_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_chunk_bwd_workspace_bytes.argtypes = [_I] * 5
        L.ttt_chunk_bwd.restype = _I
        L.ttt_chunk_bwd.argtypes = [_P] * 12 + [_I] * 6 + [ctypes.c_uint, _P, ctypes.c_size_t, _P]
        L.ttt_mlp_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_mlp_bwd_workspace_bytes.argtypes = [_I] * 6
        L.ttt_mlp_bwd.restype = _I
        L.ttt_mlp_bwd.argtypes = [_P] * 19 + [_I] * 7 + [ctypes.c_uint, _P, ctypes.c_size_t, _P]
        L.ttt_mlp_fwd.restype = _I
        L.ttt_mlp_fwd.argtypes = [_P] * 11 + [_I] * 7 + [ctypes.c_uint, _P]
        L.ttt_chunk_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_chunk_workspace_bytes.argtypes = [_I] * 5
        L.ttt_chunk_fwd.restype = _I
        L.ttt_chunk_fwd.argtypes = [_P] * 7 + [_I] * 6 + [ctypes.c_uint, _P, ctypes.c_size_t, _P]
        L.ttt_chunk_fwd_noalloc.restype = _I
        L.ttt_chunk_fwd_noalloc.argtypes = [_P] * 7 + [_I] * 6 + [ctypes.c_uint, _P]
        L.ttt_chunk_map_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_chunk_map_workspace_bytes.argtypes = [_I] * 6
        L.ttt_chunk_map.restype = _I
        L.ttt_chunk_map.argtypes = [_P] * 5 + [_I] * 6 + [_P, ctypes.c_size_t, _P]
        L.ttt_linear_map_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_linear_map_workspace_bytes.argtypes = [_I] * 6
        L.ttt_linear_map.restype = _I
        L.ttt_linear_map.argtypes = [_P] * 5 + [_I] * 6 + [_P, ctypes.c_size_t, _P]
        L.ttt_affine_prefix.restype = _I
        L.ttt_affine_prefix.argtypes = ([_P] * 5 + [_I] * 4 + [ctypes.c_longlong] * 2
                                        + [ctypes.c_uint, _P])
        L.ttt_device_status.restype = _I
        L.ttt_device_status.argtypes = [_P]
        L.ttt_launch_count.restype = ctypes.c_ulonglong
        L.ttt_launch_count.argtypes = []
        L.ttt_diag_kernel_timing.restype = _I
        L.ttt_diag_kernel_timing.argtypes = [_I]
        L.ttt_diag_kernel_times.restype = _I
        L.ttt_diag_kernel_times.argtypes = [ctypes.POINTER(ctypes.c_float), _I]
        L.ttt_selftest_umma.restype = _I
        L.ttt_selftest_umma.argtypes = [_I] * 5 + [_P, _P, _P, _P]
        L.ttt_diag_gelu.restype = _I
        L.ttt_diag_gelu.argtypes = [_P, _P, _P, _I, _P]
        L.ttt_diag_wait_timeout.restype = _I
        L.ttt_diag_wait_timeout.argtypes = [ctypes.c_uint, _P]
        L.ttt_linear_decode_tokens.restype = _I
        L.ttt_linear_decode_tokens.argtypes = [_P] * 8 + [_I] * 5 + [ctypes.c_uint, _P]
        L.ttt_mlp_decode_tokens.restype = _I
        L.ttt_mlp_decode_tokens.argtypes = [_P] * 9 + [_I] * 6 + [ctypes.c_uint, _P]
        L.ttt_diag_mlp_fwd_tcgen05.restype = _I
        L.ttt_diag_mlp_fwd_tcgen05.argtypes = [_P] * 11 + [_I] * 7 + [ctypes.c_uint, _P]
        L.ttt_diag_umma_issue_cycles.restype = _I
        L.ttt_diag_umma_issue_cycles.argtypes = [_I] * 4 + [_P, _P]
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions the public headers (include/*.h) declare."""
    import glob
    names = []
    for path in sorted(glob.glob(os.path.join(os.path.dirname(HEADER_PATH), "*.h"))):
        names += re.findall(r"TTT_API\s+[\w\s\*]*?\b(ttt_\w+)\s*\(", open(path).read())
    return names


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, rc):
    if rc != TTT_OK:
        raise TTTError(fn, rc)
    return rc


def status_string(status: int) -> str:
    return lib().ttt_status_string(int(status)).decode()


def abi_version() -> int:
    return lib().ttt_abi_version()


# ----------------------------------------------------------------- C-ABI calls

def ttt_linear_fwd(Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out, B, H, T, d, b, dt, flags,
                   stream=None, check=True):
    rc = lib().ttt_linear_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(ln_gamma),
                              _ptr(ln_beta), _ptr(Z), _ptr(W_out), B, H, T, d, b, dt, flags,
                              _stream(stream))
    return _check("ttt_linear_fwd", rc) if check else rc


def ttt_mlp_decode(q, k, v, eta, W1, W2, ln_gamma, ln_beta, z, B, H, d, dh, dt, flags,
                   stream=None, check=True):
    rc = lib().ttt_mlp_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W1), _ptr(W2),
                              _ptr(ln_gamma), _ptr(ln_beta), _ptr(z), B, H, d, dh, dt, flags,
                              _stream(stream))
    return _check("ttt_mlp_decode", rc) if check else rc


def ttt_linear_decode(q, k, v, eta, W, ln_gamma, ln_beta, z, B, H, d, dt, flags, stream=None,
                      check=True):
    rc = lib().ttt_linear_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W), _ptr(ln_gamma),
                                 _ptr(ln_beta), _ptr(z), B, H, d, dt, flags, _stream(stream))
    return _check("ttt_linear_decode", rc) if check else rc


def ttt_linear_decode_tokens(q, k, v, eta, W, ln_gamma, ln_beta, z, B, H, n, d, dt, flags,
                             stream=None, check=True):
    rc = lib().ttt_linear_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W),
                                        _ptr(ln_gamma), _ptr(ln_beta), _ptr(z), B, H, n, d, dt,
                                        flags, _stream(stream))
    return _check("ttt_linear_decode_tokens", rc) if check else rc


def ttt_mlp_decode_tokens(q, k, v, eta, W1, W2, ln_gamma, ln_beta, z, B, H, n, d, dh, dt, flags,
                          stream=None, check=True):
    rc = lib().ttt_mlp_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(eta), _ptr(W1), _ptr(W2),
                                     _ptr(ln_gamma), _ptr(ln_beta), _ptr(z), B, H, n, d, dh, dt,
                                     flags, _stream(stream))
    return _check("ttt_mlp_decode_tokens", rc) if check else rc


def ttt_linear_fwd_steps(Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out, B, H, T, d, n_steps, dt,
                         flags, stream=None, check=True):
    rc = lib().ttt_linear_fwd_steps(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0),
                                    _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z), _ptr(W_out), B, H, T,
                                    d, n_steps, dt, flags, _stream(stream))
    return _check("ttt_linear_fwd_steps", rc) if check else rc


def ttt_linear_bwd_workspace_bytes(B, H, T, d, b) -> int:
    return int(lib().ttt_linear_bwd_workspace_bytes(B, H, T, d, b))


def ttt_linear_bwd(Q, K, V, eta, W0, ln_gamma, ln_beta, dZ, dW_out, dQ, dK, dV, deta, dW0, dgamma,
                   dbeta, B, H, T, d, b, dt, flags, workspace, workspace_bytes, stream=None,
                   check=True):
    rc = lib().ttt_linear_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(ln_gamma),
                              _ptr(ln_beta), _ptr(dZ), _ptr(dW_out), _ptr(dQ), _ptr(dK), _ptr(dV),
                              _ptr(deta), _ptr(dW0), _ptr(dgamma), _ptr(dbeta), B, H, T, d, b, dt,
                              flags, _ptr(workspace), workspace_bytes, _stream(stream))
    return _check("ttt_linear_bwd", rc) if check else rc


def ttt_chunk_bwd_workspace_bytes(B, H, T, d, chunk) -> int:
    return int(lib().ttt_chunk_bwd_workspace_bytes(B, H, T, d, chunk))


def ttt_chunk_bwd(Q, K, V, eta, W0, dZ, dW_out, dQ, dK, dV, deta, dW0, B, H, T, d, chunk, dt, flags,
                  workspace, workspace_bytes, stream=None, check=True):
    rc = lib().ttt_chunk_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(dZ),
                             _ptr(dW_out), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(deta), _ptr(dW0), B,
                             H, T, d, chunk, dt, flags, _ptr(workspace), workspace_bytes,
                             _stream(stream))
    return _check("ttt_chunk_bwd", rc) if check else rc


def ttt_mlp_bwd_workspace_bytes(B, H, T, d, dh, b) -> int:
    return int(lib().ttt_mlp_bwd_workspace_bytes(B, H, T, d, dh, b))


def ttt_mlp_bwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ, dW1_out, dW2_out, dQ, dK, dV,
                deta, dW1_0, dW2_0, dgamma, dbeta, B, H, T, d, dh, b, dt, flags, workspace,
                workspace_bytes, stream=None, check=True):
    rc = lib().ttt_mlp_bwd(*[_ptr(x) for x in (Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ,
                                               dW1_out, dW2_out, dQ, dK, dV, deta, dW1_0, dW2_0,
                                               dgamma, dbeta)],
                           B, H, T, d, dh, b, dt, flags, _ptr(workspace), workspace_bytes,
                           _stream(stream))
    return _check("ttt_mlp_bwd", rc) if check else rc


def ttt_mlp_fwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1_out, W2_out, B, H, T, d, dh,
                b, dt, flags, stream=None, check=True):
    rc = lib().ttt_mlp_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W1_0), _ptr(W2_0),
                           _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z), _ptr(W1_out), _ptr(W2_out),
                           B, H, T, d, dh, b, dt, flags, _stream(stream))
    return _check("ttt_mlp_fwd", rc) if check else rc


def ttt_diag_mlp_fwd_tcgen05(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1_out, W2_out, B, H,
                             T, d, dh, b, dt, flags, stream=None, check=True):
    rc = lib().ttt_diag_mlp_fwd_tcgen05(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W1_0),
                                        _ptr(W2_0), _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z),
                                        _ptr(W1_out), _ptr(W2_out), B, H, T, d, dh, b, dt, flags,
                                        _stream(stream))
    return _check("ttt_diag_mlp_fwd_tcgen05", rc) if check else rc


def ttt_diag_umma_issue_cycles(M, N, count, nacc, cycles, stream=None, check=True):
    rc = lib().ttt_diag_umma_issue_cycles(M, N, count, nacc, _ptr(cycles), _stream(stream))
    return _check("ttt_diag_umma_issue_cycles", rc) if check else rc


def ttt_chunk_workspace_bytes(B, H, T, d, chunk) -> int:
    return int(lib().ttt_chunk_workspace_bytes(B, H, T, d, chunk))


def ttt_chunk_fwd(Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, dt, flags, workspace,
                  workspace_bytes, stream=None, check=True):
    rc = lib().ttt_chunk_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(Z),
                             _ptr(W_out), B, H, T, d, chunk, dt, flags, _ptr(workspace),
                             workspace_bytes, _stream(stream))
    return _check("ttt_chunk_fwd", rc) if check else rc


def ttt_chunk_fwd_noalloc(Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, dt, flags, stream=None,
                          check=True):
    """ttt_chunk_fwd with the library's static scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/ttt.h)."""
    rc = lib().ttt_chunk_fwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _ptr(W0), _ptr(Z),
                                     _ptr(W_out), B, H, T, d, chunk, dt, flags, _stream(stream))
    return _check("ttt_chunk_fwd_noalloc", rc) if check else rc


def ttt_chunk_map_workspace_bytes(B, H, T, d, chunk, dt) -> int:
    return int(lib().ttt_chunk_map_workspace_bytes(B, H, T, d, chunk, dt))


def ttt_chunk_map(K, V, eta, M, N, B, H, T, d, chunk, dt, workspace, workspace_bytes, stream=None,
                  check=True):
    rc = lib().ttt_chunk_map(_ptr(K), _ptr(V), _ptr(eta), _ptr(M), _ptr(N), B, H, T, d, chunk, dt,
                             _ptr(workspace), workspace_bytes, _stream(stream))
    return _check("ttt_chunk_map", rc) if check else rc


def ttt_linear_map_workspace_bytes(B, H, T, d, b, dt) -> int:
    return int(lib().ttt_linear_map_workspace_bytes(B, H, T, d, b, dt))


def ttt_linear_map(K, V, eta, M, N, B, H, T, d, b, dt, workspace, workspace_bytes, stream=None,
                   check=True):
    rc = lib().ttt_linear_map(_ptr(K), _ptr(V), _ptr(eta), _ptr(M), _ptr(N), B, H, T, d, b, dt,
                              _ptr(workspace), workspace_bytes, _stream(stream))
    return _check("ttt_linear_map", rc) if check else rc


def ttt_affine_prefix(M, N, W0, W_in, W_end, S, H, nseg, d, seq_stride, seg_stride, flags,
                      stream=None, check=True):
    rc = lib().ttt_affine_prefix(_ptr(M), _ptr(N), _ptr(W0), _ptr(W_in), _ptr(W_end), S, H, nseg,
                                 d, seq_stride, seg_stride, flags, _stream(stream))
    return _check("ttt_affine_prefix", rc) if check else rc


def ttt_device_status(stream=None) -> int:
    return lib().ttt_device_status(_stream(stream))


def ttt_launch_count() -> int:
    return int(lib().ttt_launch_count())


def ttt_diag_kernel_timing(enable: bool) -> int:
    return lib().ttt_diag_kernel_timing(int(bool(enable)))


def ttt_diag_kernel_times(max_kernels: int = 8) -> list[float]:
    """Per kernel position, the summed duration (ms) over the calls recorded since
    timing was enabled (diagnostic)."""
    buf = (ctypes.c_float * max_kernels)()
    n = lib().ttt_diag_kernel_times(buf, max_kernels)
    if n < 0:
        raise TTTError("ttt_diag_kernel_times", n)
    return [buf[i] for i in range(min(n, max_kernels))]


def ttt_selftest_umma(M, N, K, a_layout, b_layout, A, B, D, stream=None, check=True):
    """Diagnostic (include/ttt_diag.h): D = A @ B through one tcgen05 MMA chain."""
    rc = lib().ttt_selftest_umma(M, N, K, a_layout, b_layout, _ptr(A), _ptr(B), _ptr(D),
                                 _stream(stream))
    return _check("ttt_selftest_umma", rc) if check else rc


def ttt_diag_wait_timeout(limit_us, stream=None, check=True):
    """Diagnostic (include/ttt_diag.h): a bounded on-chip wait that runs out."""
    rc = lib().ttt_diag_wait_timeout(limit_us, _stream(stream))
    return _check("ttt_diag_wait_timeout", rc) if check else rc


def ttt_diag_gelu(h, gelu, gelu_prime, n, stream=None, check=True):
    """Diagnostic (include/ttt_diag.h): the MLP kernel's GELU and GELU'."""
    rc = lib().ttt_diag_gelu(_ptr(h), _ptr(gelu), _ptr(gelu_prime), n, _stream(stream))
    return _check("ttt_diag_gelu", rc) if check else rc


# ----------------------------------------------------------------- conveniences

def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return TTT_BF16
    if t.dtype == torch.float32:
        return TTT_FP32
    raise TypeError(f"Q/K/V must be bf16 or fp32, got {t.dtype}")


def linear_fwd(Q, K, V, eta, W0, ln_gamma=None, ln_beta=None, *, b, ln, w0_per_seq=False,
               stream=None, want_w=True, z_bf16=False, l2_keys=False):
    """TTT-Linear forward. Q, K, V: [B,H,T,d] cuda tensors (bf16 or fp32).
    l2_keys: normalise every key to unit length (TTT_F_L2_KEYS).
    Returns (Z fp32 [B,H,T,d], W_out fp32 [B,H,d,d] or None)."""
    import torch
    B, H, T, d = Q.shape
    Z = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32, device=Q.device)
    W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=Q.device) if want_w else None
    flags = (TTT_F_LN if ln else 0) | (TTT_F_W0_PER_SEQ if w0_per_seq else 0) | \
        (TTT_F_Z_BF16 if z_bf16 else 0) | (TTT_F_L2_KEYS if l2_keys else 0)
    ttt_linear_fwd(Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out, B, H, T, d, b,
                   _dtype_code(Q), flags, stream)
    return Z, W_out


def mlp_decode(q, k, v, eta, W1, W2, ln_gamma, ln_beta, *, z=None, z_bf16=False, stream=None):
    """One TTT-MLP token per sequence, d = 64, dh = 256: q, k, v [B, H, 64], eta
    [B, H], W1 [B, H, 64, 256] and W2 [B, H, 256, 64] fp32 updated in place
    (ttt_mlp_decode). Returns z."""
    import torch
    B, H, d = q.shape
    if z is None:
        z = torch.empty((B, H, d), dtype=torch.bfloat16 if z_bf16 else torch.float32,
                        device=q.device)
    ttt_mlp_decode(q, k, v, eta, W1, W2, ln_gamma, ln_beta, z, B, H, d, W1.shape[-1],
                   _dtype_code(q), TTT_F_LN | (TTT_F_Z_BF16 if z_bf16 else 0), stream)
    return z


def linear_decode(q, k, v, eta, W, ln_gamma=None, ln_beta=None, *, ln, z=None, z_bf16=False,
                  l2_keys=False, stream=None):
    """One TTT-Linear token per sequence, d = 64: q, k, v [B, H, 64], eta [B, H],
    W [B, H, 64, 64] fp32 updated in place (ttt_linear_decode). Returns z."""
    import torch
    B, H, d = q.shape
    if z is None:
        z = torch.empty((B, H, d), dtype=torch.bfloat16 if z_bf16 else torch.float32,
                        device=q.device)
    flags = (TTT_F_LN if ln else 0) | (TTT_F_Z_BF16 if z_bf16 else 0) | \
        (TTT_F_L2_KEYS if l2_keys else 0)
    ttt_linear_decode(q, k, v, eta, W, ln_gamma, ln_beta, z, B, H, d, _dtype_code(q), flags,
                      stream)
    return z


def linear_decode_tokens(Q, K, V, eta, W, ln_gamma=None, ln_beta=None, *, ln, z_bf16=False,
                         l2_keys=False, stream=None):
    """n TTT-Linear tokens per sequence in one call, d = 64: Q, K, V [B, H, n, 64],
    eta [B, H, n], W [B, H, 64, 64] fp32 updated in place, the weight on chip
    across the tokens (ttt_linear_decode_tokens). Returns Z [B, H, n, 64]."""
    import torch
    B, H, n, d = Q.shape
    Z = torch.empty((B, H, n, d), dtype=torch.bfloat16 if z_bf16 else torch.float32,
                    device=Q.device)
    flags = (TTT_F_LN if ln else 0) | (TTT_F_Z_BF16 if z_bf16 else 0) | \
        (TTT_F_L2_KEYS if l2_keys else 0)
    ttt_linear_decode_tokens(Q, K, V, eta, W, ln_gamma, ln_beta, Z, B, H, n, d, _dtype_code(Q),
                             flags, stream)
    return Z


def mlp_decode_tokens(Q, K, V, eta, W1, W2, ln_gamma, ln_beta, *, z_bf16=False, stream=None):
    """n TTT-MLP tokens per sequence in one call, d = 64, dh = 256: Q, K, V
    [B, H, n, 64], eta [B, H, n], W1 [B, H, 64, 256] and W2 [B, H, 256, 64] fp32
    updated in place, both on chip across the tokens (ttt_mlp_decode_tokens).
    Returns Z [B, H, n, 64]."""
    import torch
    B, H, n, d = Q.shape
    Z = torch.empty((B, H, n, d), dtype=torch.bfloat16 if z_bf16 else torch.float32,
                    device=Q.device)
    ttt_mlp_decode_tokens(Q, K, V, eta, W1, W2, ln_gamma, ln_beta, Z, B, H, n, d, W1.shape[-1],
                          _dtype_code(Q), TTT_F_LN | (TTT_F_Z_BF16 if z_bf16 else 0), stream)
    return Z


def linear_fwd_steps(Q, K, V, eta, W0, ln_gamma=None, ln_beta=None, *, n_steps, ln,
                     w0_per_seq=False, stream=None, want_w=True, z_bf16=False, l2_keys=False):
    """TTT-Linear forward, online, n_steps gradient steps per token before its
    read-out (ttt_linear_fwd_steps). Returns (Z, W_out) like linear_fwd."""
    import torch
    B, H, T, d = Q.shape
    Z = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32, device=Q.device)
    W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=Q.device) if want_w else None
    flags = (TTT_F_LN if ln else 0) | (TTT_F_W0_PER_SEQ if w0_per_seq else 0) | \
        (TTT_F_Z_BF16 if z_bf16 else 0) | (TTT_F_L2_KEYS if l2_keys else 0)
    ttt_linear_fwd_steps(Q, K, V, eta, W0, ln_gamma, ln_beta, Z, W_out, B, H, T, d, n_steps,
                         _dtype_code(Q), flags, stream)
    return Z, W_out


def linear_bwd(Q, K, V, eta, W0, ln_gamma, ln_beta, dZ, dW_out=None, *, b, ln, w0_per_seq=False,
               workspace=None, stream=None):
    """TTT-Linear backward. Returns a dict of fp32 cuda tensors: Q, K, V, eta,
    W0 and (with ln) gamma, beta -- the gradients of sum(Z * dZ) +
    sum(W_out * dW_out). Allocates the workspace with torch unless one is given."""
    import torch
    B, H, T, d = Q.shape
    dev = Q.device
    f32 = dict(dtype=torch.float32, device=dev)
    need = ttt_linear_bwd_workspace_bytes(B, H, T, d, b)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    g = dict(Q=torch.empty((B, H, T, d), **f32), K=torch.empty((B, H, T, d), **f32),
             V=torch.empty((B, H, T, d), **f32), eta=torch.empty((B, H, T), **f32),
             W0=torch.empty(tuple(W0.shape), **f32))
    if ln:
        g["gamma"] = torch.empty((H, d), **f32)
        g["beta"] = torch.empty((H, d), **f32)
    flags = (TTT_F_LN if ln else 0) | (TTT_F_W0_PER_SEQ if w0_per_seq else 0)
    ttt_linear_bwd(Q, K, V, eta, W0, ln_gamma, ln_beta, dZ, dW_out, g["Q"], g["K"], g["V"],
                   g["eta"], g["W0"], g.get("gamma"), g.get("beta"), B, H, T, d, b, _dtype_code(Q),
                   flags, workspace, workspace.numel() * workspace.element_size(), stream)
    return g


def mlp_bwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ, dW1_out=None, dW2_out=None, *, b,
            w0_per_seq=False, workspace=None, stream=None):
    """TTT-MLP backward. Returns a dict of fp32 gradients with keys Q, K, V,
    eta, W1, W2, gamma, beta (W1/W2 shaped like W1_0/W2_0)."""
    import torch
    B, H, T, d = Q.shape
    dh = W1_0.shape[-1]
    f = dict(device=Q.device, dtype=torch.float32)
    g = {"Q": torch.empty((B, H, T, d), **f), "K": torch.empty((B, H, T, d), **f),
         "V": torch.empty((B, H, T, d), **f), "eta": torch.empty((B, H, T), **f),
         "W1": torch.empty(tuple(W1_0.shape), **f), "W2": torch.empty(tuple(W2_0.shape), **f),
         "gamma": torch.empty((H, d), **f), "beta": torch.empty((H, d), **f)}
    need = ttt_mlp_bwd_workspace_bytes(B, H, T, d, dh, b)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=Q.device)
    flags = TTT_F_LN | (TTT_F_W0_PER_SEQ if w0_per_seq else 0)
    ttt_mlp_bwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, dZ, dW1_out, dW2_out, g["Q"], g["K"],
                g["V"], g["eta"], g["W1"], g["W2"], g["gamma"], g["beta"], B, H, T, d, dh, b,
                _dtype_code(Q), flags, workspace, workspace.numel() * workspace.element_size(),
                stream)
    return g


def chunk_bwd(Q, K, V, eta, W0, dZ, dW_out=None, *, chunk, w0_per_seq=False, workspace=None,
              stream=None):
    """Large-chunk TTT backward. Returns a dict of fp32 cuda tensors Q, K, V,
    eta, W0: the gradients of sum(Z * dZ) + sum(W_out * dW_out)."""
    import torch
    B, H, T, d = Q.shape
    f32 = dict(dtype=torch.float32, device=Q.device)
    need = ttt_chunk_bwd_workspace_bytes(B, H, T, d, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    g = dict(Q=torch.empty((B, H, T, d), **f32), K=torch.empty((B, H, T, d), **f32),
             V=torch.empty((B, H, T, d), **f32), eta=torch.empty((B, H, T), **f32),
             W0=torch.empty(tuple(W0.shape), **f32))
    ttt_chunk_bwd(Q, K, V, eta, W0, dZ, dW_out, g["Q"], g["K"], g["V"], g["eta"], g["W0"], B, H, T,
                  d, chunk, _dtype_code(Q), TTT_F_W0_PER_SEQ if w0_per_seq else 0, workspace,
                  workspace.numel() * workspace.element_size(), stream)
    return g


def mlp_fwd(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, *, b, w0_per_seq=False, stream=None,
            want_w=True, z_bf16=False, kernel="default"):
    """TTT-MLP forward. Returns (Z, W1_out, W2_out). kernel="tcgen05" runs the
    diagnostic single-issuer tensor-core kernel (ttt_diag_mlp_fwd_tcgen05)."""
    import torch
    B, H, T, d = Q.shape
    dh = W1_0.shape[-1]
    Z = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32, device=Q.device)
    W1o = torch.empty((B, H, d, dh), dtype=torch.float32, device=Q.device) if want_w else None
    W2o = torch.empty((B, H, dh, d), dtype=torch.float32, device=Q.device) if want_w else None
    flags = TTT_F_LN | (TTT_F_W0_PER_SEQ if w0_per_seq else 0) | (TTT_F_Z_BF16 if z_bf16 else 0)
    fn = ttt_diag_mlp_fwd_tcgen05 if kernel == "tcgen05" else ttt_mlp_fwd
    fn(Q, K, V, eta, W1_0, W2_0, ln_gamma, ln_beta, Z, W1o, W2o, B, H, T, d, dh, b,
       _dtype_code(Q), flags, stream)
    return Z, W1o, W2o


def chunk_fwd(Q, K, V, eta, W0, *, chunk, w0_per_seq=False, workspace=None, stream=None,
              want_w=True, z_bf16=False):
    """Large-chunk TTT forward (apply-then-update). Allocates the workspace
    with torch unless one is given. Returns (Z, W_out)."""
    import torch
    B, H, T, d = Q.shape
    Z = torch.empty((B, H, T, d), dtype=torch.bfloat16 if z_bf16 else torch.float32, device=Q.device)
    W_out = torch.empty((B, H, d, d), dtype=torch.float32, device=Q.device) if want_w else None
    need = ttt_chunk_workspace_bytes(B, H, T, d, chunk)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    flags = (TTT_F_W0_PER_SEQ if w0_per_seq else 0) | (TTT_F_Z_BF16 if z_bf16 else 0)
    ttt_chunk_fwd(Q, K, V, eta, W0, Z, W_out, B, H, T, d, chunk, _dtype_code(Q), flags,
                  workspace, need, stream)
    return Z, W_out


def chunk_map(K, V, eta, *, chunk, workspace=None, stream=None):
    """Affine map W -> M W + N of each sequence's chunks (see ttt_chunk_map).
    Returns (M, N), each [B, H, d, d] fp32."""
    import torch
    B, H, T, d = K.shape
    M = torch.empty((B, H, d, d), dtype=torch.float32, device=K.device)
    N = torch.empty_like(M)
    dt = _dtype_code(K)
    need = ttt_chunk_map_workspace_bytes(B, H, T, d, chunk, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=K.device)
    ttt_chunk_map(K, V, eta, M, N, B, H, T, d, chunk, dt, workspace,
                  workspace.numel() * workspace.element_size(), stream)
    return M, N


def linear_map(K, V, eta, *, b, workspace=None, stream=None):
    """Affine map W -> M W + N of each sequence's mini-batches of TTT-Linear
    without LayerNorm (see ttt_linear_map). Returns (M, N), each [B, H, d, d]."""
    import torch
    B, H, T, d = K.shape
    M = torch.empty((B, H, d, d), dtype=torch.float32, device=K.device)
    N = torch.empty_like(M)
    dt = _dtype_code(K)
    need = ttt_linear_map_workspace_bytes(B, H, T, d, b, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=K.device)
    ttt_linear_map(K, V, eta, M, N, B, H, T, d, b, dt, workspace,
                   workspace.numel() * workspace.element_size(), stream)
    return M, N


def affine_prefix(M, N, W0, W_in, W_end=None, *, S, H, nseg, seq_stride, seg_stride,
                  w0_per_seq=False, stream=None):
    """Fold segment maps into starting weights (see ttt_affine_prefix); writes
    W_in and, if given, W_end."""
    d = M.shape[-1]
    ttt_affine_prefix(M, N, W0, W_in, W_end, S, H, nseg, d, seq_stride, seg_stride,
                      TTT_F_W0_PER_SEQ if w0_per_seq else 0, stream)
