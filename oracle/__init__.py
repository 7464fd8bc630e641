"""CPU oracle for NVFP4 W4A4 linear layers (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The library never does.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, FP32 quantisation steps as
the pages' format definition reads, FP64 dequantisation and GEMM).  This module
only marshals numpy arrays and composes those steps into the whole linear
layer.  See the C file's header for the readings taken where the pages are
silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

# Block size and the E2M1 value set, restated from the pages' format
# definition ("Background", item 1) for the Python-level helpers below.
BLOCK = 16


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        F = ctypes.c_float
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode_many.argtypes = [P, I, P]
        L.oracle_e4m3_encode_many.argtypes = [P, I, P]
        L.oracle_amax.argtypes = [P, I, I, I]
        L.oracle_amax.restype = F
        L.oracle_global_scale_from_amax.argtypes = [F]
        L.oracle_global_scale_from_amax.restype = F
        L.oracle_global_scale.argtypes = [P, I, I, I]
        L.oracle_global_scale.restype = F
        L.oracle_quantize.argtypes = [P, I, I, I, F, P, P]
        L.oracle_dequantize.argtypes = [P, P, I, I, F, P]
        L.oracle_sf_tiled_bytes.argtypes = [I, I]
        L.oracle_sf_tiled_bytes.restype = I
        L.oracle_sf_tiled_offset.argtypes = [I, I, I]
        L.oracle_sf_tiled_offset.restype = I
        L.oracle_sf_to_tiled.argtypes = [P, I, I, P]
        L.oracle_gemm.argtypes = [P, P, I, I, I, P]
        L.oracle_bf16_round.argtypes = [P, I, P]
        L.oracle_silu_mul_bf16.argtypes = [P, P, I, P]
        L.oracle_gdn_gates.argtypes = [P, P, I, I, I, P, P, P, P]
        L.oracle_fp8_scale_from_amax.argtypes = [ctypes.c_float]
        L.oracle_fp8_scale_from_amax.restype = ctypes.c_float
        L.oracle_fp8_quantize.argtypes = [P, I, ctypes.c_float, P]
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    """Exact FP32 view of an array-like (torch BF16/FP32 tensors included)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------- formats
def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(code)


def e2m1_encode(y) -> np.ndarray:
    """Signed E2M1 codes (sign bit = sign of y) of an FP32 array."""
    y = _f32(y).ravel()
    out = np.empty(y.size, np.uint8)
    lib().oracle_e2m1_encode_many(_ptr(y), y.size, _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes of |x| (round-to-nearest-even, saturating to 448)."""
    x = _f32(x).ravel()
    out = np.empty(x.size, np.uint8)
    lib().oracle_e4m3_encode_many(_ptr(x), x.size, _ptr(out))
    return out


# --------------------------------------------------------------------------- quantisation
def amax(x) -> np.float32:
    x = _f32(x)
    x2 = x.reshape(-1, x.shape[-1]) if x.ndim > 1 else x.reshape(1, -1)
    return np.float32(lib().oracle_amax(_ptr(x2), x2.shape[0], x2.shape[1], x2.shape[1]))


def global_scale(x) -> np.float32:
    """Per-tensor FP32 decode scale amax / 2688 (1 when that is 0)."""
    return np.float32(lib().oracle_global_scale_from_amax(float(amax(x))))


def global_scale_from_amax(a: float) -> np.float32:
    return np.float32(lib().oracle_global_scale_from_amax(float(a)))


def quantize(x, s_g):
    """Return ``(q, sf)``: packed codes ``rows x k/2`` and row-major scales ``rows x k/16``."""
    x = _f32(x)
    rows, k = x.shape
    if k % BLOCK:
        raise ValueError("k must be a multiple of 16")
    q = np.empty((rows, k // 2), np.uint8)
    sf = np.empty((rows, k // BLOCK), np.uint8)
    lib().oracle_quantize(_ptr(x), rows, k, k, float(np.float32(s_g)), _ptr(q), _ptr(sf))
    return q, sf


def dequantize(q: np.ndarray, sf: np.ndarray, s_g) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, k = q.shape[0], q.shape[1] * 2
    out = np.empty((rows, k), np.float64)
    lib().oracle_dequantize(_ptr(q), _ptr(sf), rows, k, float(np.float32(s_g)), _ptr(out))
    return out


def sf_tiled_bytes(rows: int, k: int) -> int:
    return int(lib().oracle_sf_tiled_bytes(rows, k))


def sf_tiled_offset(row: int, kb: int, k: int) -> int:
    return int(lib().oracle_sf_tiled_offset(row, kb, k))


def sf_to_tiled(sf: np.ndarray, k: int) -> np.ndarray:
    sf = np.ascontiguousarray(sf, np.uint8)
    out = np.empty(sf_tiled_bytes(sf.shape[0], k), np.uint8)
    lib().oracle_sf_to_tiled(_ptr(sf), sf.shape[0], k, _ptr(out))
    return out


def sf_from_tiled(tiled: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Row-major view of a tiled scale buffer, using the oracle's own index map."""
    tiled = np.asarray(tiled, np.uint8).ravel()
    nb = k // BLOCK
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(nb, dtype=np.int64)[None, :]
    katoms = (nb + 3) // 4
    off = ((r // 128) * katoms + b // 4) * 512 + (r % 128 % 32) * 16 + (r % 128 // 32) * 4 + b % 4
    return tiled[off]


# --------------------------------------------------------------------------- GEMM
def gemm(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """FP64 C = A_hat . W_hat^T (W is N x K)."""
    a_hat = np.ascontiguousarray(a_hat, np.float64)
    w_hat = np.ascontiguousarray(w_hat, np.float64)
    m, k = a_hat.shape
    n = w_hat.shape[0]
    c = np.empty((m, n), np.float64)
    lib().oracle_gemm(_ptr(a_hat), _ptr(w_hat), m, n, k, _ptr(c))
    return c


class QuantizedModule:
    """One separately calibrated module: its codes, row-major scales and global scale."""

    def __init__(self, w, s_g=None):
        w = _f32(w)
        self.s_g = global_scale(w) if s_g is None else np.float32(s_g)
        self.q, self.sf = quantize(w, self.s_g)
        self.n, self.k = w.shape

    def dequantize(self) -> np.ndarray:
        return dequantize(self.q, self.sf, self.s_g)


def quantize_modules(modules):
    return [QuantizedModule(w) for w in modules]


def fused_weight_hat(qmods) -> np.ndarray:
    """Dequantised fused weight: every module's rows carry its OWN global scale."""
    return np.concatenate([qm.dequantize() for qm in qmods], axis=0)


def linear(a, modules, act_scale=None, rows=None):
    """The whole W4A4 linear layer in FP64: returns ``(C64, info)``.

    ``rows`` (optional index array) restricts the output to those rows of A,
    for sizes where the full FP64 GEMM would be too slow.
    """
    a32 = _f32(a)
    s_ga = global_scale(a32) if act_scale is None else np.float32(act_scale)
    qmods = quantize_modules(modules)
    if rows is not None:
        a32 = a32[np.asarray(rows)]
    qa, sfa = quantize(a32, s_ga)
    a_hat = dequantize(qa, sfa, s_ga)
    c = gemm(a_hat, fused_weight_hat(qmods))
    return c, dict(s_ga=s_ga, qa=qa, sfa=sfa, a_hat=a_hat, qmods=qmods)


# --------------------------------------------------------------------------- BF16 / MLP glue
def bf16_round(x) -> np.ndarray:
    """Round an FP32 array to BF16, returned as uint16 bit patterns."""
    x = _f32(x).ravel()
    out = np.empty(x.size, np.uint16)
    lib().oracle_bf16_round(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def silu_mul_bf16(g_bits: np.ndarray, u_bits: np.ndarray) -> np.ndarray:
    g_bits = np.ascontiguousarray(g_bits, np.uint16).ravel()
    u_bits = np.ascontiguousarray(u_bits, np.uint16).ravel()
    out = np.empty(g_bits.size, np.uint16)
    lib().oracle_silu_mul_bf16(_ptr(g_bits), _ptr(u_bits), g_bits.size, _ptr(out))
    return out


def fp8_scale_from_amax(amax) -> np.float32:
    """Calibrated per-tensor FP8 KV-cache scale: ``amax / 448`` (1 if 0)."""
    return np.float32(lib().oracle_fp8_scale_from_amax(float(np.float32(amax))))


def fp8_quantize(x, scale) -> np.ndarray:
    """E4M3 bytes of ``x * (1 / scale)`` (FP32, RNE, saturating), same shape."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_fp8_quantize(_ptr(x), x.size, float(np.float32(scale)), _ptr(out))
    return out


def gdn_gates(a, b, A_log, dt_bias):
    """GDN gates in FP64: ``g = -exp(A_log) * softplus(a + dt_bias)`` and
    ``beta = sigmoid(b)`` for m x heads inputs ``a``, ``b`` (FP32 views)."""
    a = _f32(a)
    b = _f32(b)
    m, heads = a.shape
    if b.shape != (m, heads):
        raise ValueError("a and b must have the same shape")
    A_log = _f32(A_log).ravel()
    dt_bias = _f32(dt_bias).ravel()
    g = np.empty((m, heads), np.float64)
    beta = np.empty((m, heads), np.float64)
    lib().oracle_gdn_gates(_ptr(a), _ptr(b), m, heads, heads, _ptr(A_log), _ptr(dt_bias), _ptr(g), _ptr(beta))
    return g, beta


def num_threads() -> int:
    return int(lib().oracle_num_threads())
