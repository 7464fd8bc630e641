"""NVFP4 W4A4 linear layers for B200 (sm_100a): Python binding of libnvfp4.

Argument marshalling only.  Every step of the path (amax, block quantisation,
the block-scaled GEMM and its per-module scale epilogue) runs in the CUDA
kernels behind the C ABI declared in ``include/nvfp4.h``; PyTorch supplies
device memory and the current stream.  There is no CPU fallback: if
``libnvfp4.so`` is missing or cannot be loaded every call raises.

The raw C entry points are available under their C names
(``nvfp4_quantize_weight``, ``nvfp4_quantize_act``, ``nvfp4_gemm``, ...) on
the object returned by :func:`load`; the helpers below wrap them for torch
tensors.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

NVFP4_IN_BF16, NVFP4_IN_FP32 = 0, 1
NVFP4_OUT_BF16, NVFP4_OUT_FP32 = 0, 1
NVFP4_GEMM_AUTO, NVFP4_GEMM_FORCE_LARGE, NVFP4_GEMM_FORCE_DECODE, NVFP4_GEMM_FORCE_LARGE_PAIR = 0, 1, 2, 3
NVFP4_MAX_SEGMENTS = 16
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "ALIGNMENT", 4: "CUDA", 5: "TIMEOUT",
                6: "WORKSPACE"}
EXPORTED = ("nvfp4_sf_bytes", "nvfp4_sf_offset", "nvfp4_quant_workspace_size", "nvfp4_gemm_workspace_size",
            "nvfp4_gemm_kernel_for",
            "nvfp4_quantize_weight", "nvfp4_quantize_act", "nvfp4_silu_mul_quantize", "nvfp4_gemm",
            "nvfp4_linear_decode", "nvfp4_linear_prefill", "nvfp4_linear_prefill_workspace_size",
            "nvfp4_gemm_swiglu_quantize", "nvfp4_gemm_decode_noalloc", "nvfp4_gemm_gdn",
            "nvfp4_fp8_calibrate", "nvfp4_kv_cache_quantize_fp8",
            "nvfp4_get_last_error_string", "nvfp4_check_device_status", "nvfp4_selftest_wait_timeout",
            "nvfp4_version")
NVFP4_NOALLOC_MAX_M = 16


class NVFP4Error(RuntimeError):
    def __init__(self, call: str, status: int, detail: str):
        super().__init__(f"{call}: {STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status


class Segment(ctypes.Structure):
    _fields_ = [("col_begin", ctypes.c_int64), ("col_end", ctypes.c_int64), ("w_global_scale", ctypes.c_float)]


class GdnGates(ctypes.Structure):
    _fields_ = [("a_col", ctypes.c_int32), ("b_col", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("g", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("ldg", ctypes.c_int64)]


_lib = None


def load():
    """Load ``libnvfp4.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise NVFP4Error("load", 4, f"{LIB_PATH} is not built; run `python -m nvfp4_w4a4_quantized_07_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, SZ, U32, INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_int
    L.nvfp4_sf_bytes.argtypes = [I64, I64]
    L.nvfp4_sf_bytes.restype = SZ
    L.nvfp4_sf_offset.argtypes = [I64, I64, I64]
    L.nvfp4_sf_offset.restype = I64
    L.nvfp4_quant_workspace_size.argtypes = []
    L.nvfp4_quant_workspace_size.restype = SZ
    L.nvfp4_gemm_workspace_size.argtypes = [I64, I64, I64, U32]
    L.nvfp4_gemm_workspace_size.restype = SZ
    L.nvfp4_gemm_kernel_for.argtypes = [I64, I64, INT, U32, INT]
    L.nvfp4_gemm_kernel_for.restype = INT
    L.nvfp4_quantize_weight.argtypes = [P, INT, I64, I64, I64, I64, I64, P, P, P, P, P, SZ, P]
    L.nvfp4_quantize_weight.restype = INT
    L.nvfp4_quantize_act.argtypes = [P, INT, I64, I64, I64, P, P, P, P, P, SZ, P]
    L.nvfp4_quantize_act.restype = INT
    L.nvfp4_silu_mul_quantize.argtypes = [P, P, I64, I64, I64, P, P, P, P, P, I64, P, SZ, P]
    L.nvfp4_silu_mul_quantize.restype = INT
    L.nvfp4_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, ctypes.POINTER(Segment), INT, P, INT, I64, P, SZ, U32, P]
    L.nvfp4_gemm.restype = INT
    L.nvfp4_gemm_gdn.argtypes = [P, P, P, P, P, I64, I64, I64, ctypes.POINTER(Segment), INT, P, I64,
                                 ctypes.POINTER(GdnGates), P, SZ, U32, P]
    L.nvfp4_gemm_gdn.restype = INT
    L.nvfp4_fp8_calibrate.argtypes = [P, INT, I64, I64, I64, P, P, P]
    L.nvfp4_fp8_calibrate.restype = INT
    L.nvfp4_kv_cache_quantize_fp8.argtypes = [P, P, INT, I64, I64, I64, I64, P, I64, P, P, P, P, I64, P]
    L.nvfp4_kv_cache_quantize_fp8.restype = INT
    L.nvfp4_gemm_swiglu_quantize.argtypes = [P, P, P, P, P, I64, I64, I64, ctypes.POINTER(Segment), INT, P, P, P, P]
    L.nvfp4_gemm_swiglu_quantize.restype = INT
    L.nvfp4_linear_decode.argtypes = [P, INT, I64, I64, I64, P, P, P, P, I64, ctypes.POINTER(Segment), INT, P, INT,
                                      I64, P, SZ, P]
    L.nvfp4_linear_decode.restype = INT
    L.nvfp4_linear_prefill.argtypes = [P, INT, I64, I64, I64, P, P, P, P, P, I64, ctypes.POINTER(Segment), INT, P,
                                       INT, I64, P, SZ, P]
    L.nvfp4_linear_prefill.restype = INT
    L.nvfp4_linear_prefill_workspace_size.argtypes = [I64]
    L.nvfp4_linear_prefill_workspace_size.restype = SZ
    L.nvfp4_gemm_decode_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, ctypes.POINTER(Segment), INT, P, INT, I64,
                                            P]
    L.nvfp4_gemm_decode_noalloc.restype = INT
    L.nvfp4_get_last_error_string.argtypes = []
    L.nvfp4_get_last_error_string.restype = ctypes.c_char_p
    L.nvfp4_check_device_status.argtypes = [P]
    L.nvfp4_check_device_status.restype = INT
    L.nvfp4_selftest_wait_timeout.argtypes = [ctypes.c_longlong, P]
    L.nvfp4_selftest_wait_timeout.restype = INT
    L.nvfp4_version.argtypes = []
    L.nvfp4_version.restype = INT
    _lib = L
    return L


def _check(call: str, status: int):
    if status != 0:
        raise NVFP4Error(call, status, load().nvfp4_get_last_error_string().decode())


def _stream(device=None):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _in_dtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return NVFP4_IN_BF16
    if t.dtype == torch.float32:
        return NVFP4_IN_FP32
    raise TypeError(f"NVFP4 inputs must be bfloat16 or float32, got {t.dtype}")


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libnvfp4 operates on CUDA tensors only")


def sf_bytes(rows: int, k: int) -> int:
    return int(load().nvfp4_sf_bytes(rows, k))


def sf_offset(row: int, kblock: int, k: int) -> int:
    return int(load().nvfp4_sf_offset(row, kblock, k))


def _ws_key(device):
    """Cache key of a default workspace: the device and the stream the call
    runs on (the current stream).  Calls on one stream run in order and may
    share a workspace; calls on different streams may overlap, so each stream
    gets its own.  The workspace is allocated while that stream is current, so
    when a larger one replaces it the caching allocator hands the old memory
    out again only in that stream's order."""
    import torch
    dev = torch.device(device)
    return dev, int(torch.cuda.current_stream(dev).cuda_stream)


_quant_ws_cache = {}


def quant_workspace(device) -> "torch.Tensor":
    """A cached workspace of nvfp4_quant_workspace_size bytes for the
    dynamic-scale quantisers, one per (device, current stream).  It needs no
    initialisation (the library clears the amax word it uses on the call's
    stream), so it is allocated once and not filled."""
    import torch
    key = _ws_key(device)
    ws = _quant_ws_cache.get(key)
    if ws is None:
        ws = torch.empty(load().nvfp4_quant_workspace_size(), dtype=torch.uint8, device=key[0])
        _quant_ws_cache[key] = ws
    return ws


@dataclass
class QuantizedActivation:
    q: "torch.Tensor"       # m x k/2 uint8
    sf: "torch.Tensor"      # tiled scales, uint8
    scale: "torch.Tensor"   # 1-element float32 device tensor (s_ga)
    m: int
    k: int


@dataclass
class FusedWeight:
    q: "torch.Tensor"       # n x k/2 uint8
    sf: "torch.Tensor"      # tiled scales, uint8
    segments: list          # [(col_begin, col_end, w_global_scale)]
    n: int
    k: int


def quantize_act(a, act_scale=None, workspace=None, out: QuantizedActivation | None = None) -> QuantizedActivation:
    """On-the-fly activation quantisation (``nvfp4_quantize_act``).

    ``act_scale``: 1-element float32 CUDA tensor holding a calibrated decode
    scale (static mode) or ``None`` (dynamic: amax/2688 computed on device).
    """
    import torch
    _require_cuda(a, act_scale)
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("activations must be a 2-D tensor with unit column stride")
    m, k = a.shape
    L = load()
    if out is None:
        out = QuantizedActivation(
            q=torch.empty((m, k // 2), dtype=torch.uint8, device=a.device),
            sf=torch.empty(max(L.nvfp4_sf_bytes(m, k), 1), dtype=torch.uint8, device=a.device),
            scale=torch.empty(1, dtype=torch.float32, device=a.device), m=m, k=k)
    if act_scale is None and workspace is None:
        workspace = quant_workspace(a.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("nvfp4_quantize_act", L.nvfp4_quantize_act(
        _ptr(a), _in_dtype(a), m, k, a.stride(0), _ptr(act_scale), _ptr(out.scale), _ptr(out.q), _ptr(out.sf),
        _ptr(workspace), ws_bytes, _stream(a.device)))
    return out


def silu_mul_quantize(g, u, h_scale=None, return_h: bool = False, workspace=None,
                      out: QuantizedActivation | None = None, h_out=None):
    """MLP glue (``nvfp4_silu_mul_quantize``): h = bf16(silu(g) * u) quantised
    to NVFP4.  ``g`` and ``u`` are BF16 m x f CUDA tensors with unit column
    stride and the same row stride (e.g. the two halves of a fused gate/up
    GEMM output).  ``h_scale`` is a static 1-element FP32 device scale or
    ``None`` (dynamic).  ``h_out`` (a contiguous m x f BF16 tensor) or
    ``return_h`` also stores h.  Returns ``(QuantizedActivation, h or None)``."""
    import torch
    _require_cuda(g, u, h_scale)
    if g.dtype != torch.bfloat16 or u.dtype != torch.bfloat16:
        raise TypeError("g and u must be bfloat16")
    if g.shape != u.shape or g.dim() != 2 or g.stride() != u.stride() or g.stride(1) != 1:
        raise ValueError("g and u must be 2-D tensors of one shape and row stride, unit column stride")
    m, f = g.shape
    L = load()
    if out is None:
        out = QuantizedActivation(
            q=torch.empty((m, f // 2), dtype=torch.uint8, device=g.device),
            sf=torch.empty(max(L.nvfp4_sf_bytes(m, f), 1), dtype=torch.uint8, device=g.device),
            scale=torch.empty(1, dtype=torch.float32, device=g.device), m=m, k=f)
    h = h_out
    if h is None and return_h:
        h = torch.empty((m, f), dtype=torch.bfloat16, device=g.device)
    if h is not None and (h.shape != (m, f) or h.dtype != torch.bfloat16 or not h.is_contiguous()):
        raise ValueError("h_out must be a contiguous m x f bfloat16 tensor")
    if h_scale is None and workspace is None:
        workspace = quant_workspace(g.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("nvfp4_silu_mul_quantize", L.nvfp4_silu_mul_quantize(
        _ptr(g), _ptr(u), m, f, g.stride(0), _ptr(h_scale), _ptr(out.scale), _ptr(out.q), _ptr(out.sf),
        _ptr(h), f, _ptr(workspace), ws_bytes, _stream(g.device)))
    return out, h


def quantize_weight(modules, global_scales=None, workspace=None) -> FusedWeight:
    """Quantise separately calibrated modules into one fused weight
    (``nvfp4_quantize_weight`` once per module).  ``global_scales[i]`` (a
    Python float) fixes module i's decode scale; ``None`` computes amax/2688
    on the device (the call then synchronises to return it)."""
    import torch
    modules = list(modules)
    if not modules:
        raise ValueError("need at least one module")
    k = modules[0].shape[1]
    device = modules[0].device
    n_total = sum(w.shape[0] for w in modules)
    L = load()
    q = torch.empty((n_total, k // 2), dtype=torch.uint8, device=device)
    sf = torch.empty(max(L.nvfp4_sf_bytes(n_total, k), 1), dtype=torch.uint8, device=device)
    if workspace is None:
        workspace = quant_workspace(device)
    segs = []
    off = 0
    for i, w in enumerate(modules):
        _require_cuda(w)
        if w.dim() != 2 or w.shape[1] != k or w.stride(1) != 1:
            raise ValueError("every module must be a 2-D n_i x k tensor with unit column stride")
        n = w.shape[0]
        given = None if global_scales is None or global_scales[i] is None else ctypes.c_float(global_scales[i])
        got = ctypes.c_float(0.0)
        _check("nvfp4_quantize_weight", L.nvfp4_quantize_weight(
            _ptr(w), _in_dtype(w), n, k, w.stride(0), off, n_total,
            None if given is None else ctypes.byref(given), _ptr(q), _ptr(sf), ctypes.byref(got),
            _ptr(workspace), workspace.numel(), _stream(device)))
        segs.append((off, off + n, float(got.value)))
        off += n
    return FusedWeight(q=q, sf=sf, segments=segs, n=n_total, k=k)


def segment_array(segments):
    arr = (Segment * len(segments))()
    for i, (b, e, s) in enumerate(segments):
        arr[i].col_begin, arr[i].col_end, arr[i].w_global_scale = b, e, s
    return arr


_ws_cache = {}


def gemm_workspace(m: int, n: int, k: int, flags: int, device):
    """A cached workspace of at least nvfp4_gemm_workspace_size bytes, one per
    (device, current stream); it needs no initialisation (the decode kernel
    tags what it writes)."""
    import torch
    need = int(load().nvfp4_gemm_workspace_size(m, n, k, flags))
    if need == 0:
        return None
    key = _ws_key(device)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=key[0])
        _ws_cache[key] = ws
    return ws


def gemm(a: QuantizedActivation, w: FusedWeight, out_dtype=None, flags: int = NVFP4_GEMM_AUTO,
         segments=None, out=None, workspace=None):
    """``C = nvfp4_gemm(a, w)``: m x n output, BF16 by default.  ``segments``
    overrides the fused weight's own segment table; ``workspace`` defaults to a
    buffer cached per (device, current stream) when the chosen kernel needs
    one."""
    import torch
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if a.k != w.k:
        raise ValueError("K mismatch between activations and weight")
    segments = w.segments if segments is None else segments
    if out is None:
        out = torch.empty((a.m, w.n), dtype=out_dtype, device=a.q.device)
    odt = {torch.bfloat16: NVFP4_OUT_BF16, torch.float32: NVFP4_OUT_FP32}[out.dtype]
    arr = segment_array(segments)
    L = load()
    if workspace is None:
        workspace = gemm_workspace(a.m, w.n, w.k, flags, out.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("nvfp4_gemm", L.nvfp4_gemm(
        _ptr(a.q), _ptr(a.sf), _ptr(a.scale), _ptr(w.q), _ptr(w.sf), a.m, w.n, w.k, arr, len(segments),
        _ptr(out), odt, out.stride(0), _ptr(workspace), ws_bytes, flags, _stream(out.device)))
    return out


def gemm_gdn(a: QuantizedActivation, w: FusedWeight, a_col: int, b_col: int, A_log, dt_bias, flags: int = NVFP4_GEMM_AUTO,
             out=None, g=None, beta=None, workspace=None):
    """``nvfp4_gemm_gdn``: the fused GDN input projection (BF16 ``C``) with the
    Gated DeltaNet gates computed in its epilogue from the head-wide column
    ranges at ``a_col`` and ``b_col`` (one column per head; ``A_log`` and
    ``dt_bias`` are FP32 device vectors of the head count).  Returns
    ``(C, g, beta)``, the gates FP32 m x heads."""
    import torch
    _require_cuda(A_log, dt_bias)
    if a.k != w.k:
        raise ValueError("K mismatch between activations and weight")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32 or A_log.numel() != dt_bias.numel():
        raise ValueError("A_log and dt_bias must be FP32 vectors of one length (the head count)")
    heads = A_log.numel()
    dev = a.q.device
    if out is None:
        out = torch.empty((a.m, w.n), dtype=torch.bfloat16, device=dev)
    if g is None:
        g = torch.empty((a.m, heads), dtype=torch.float32, device=dev)
    if beta is None:
        beta = torch.empty((a.m, heads), dtype=torch.float32, device=dev)
    if g.stride(0) != beta.stride(0) or g.stride(-1) != 1 or beta.stride(-1) != 1:
        raise ValueError("g and beta must share a row stride with contiguous rows")
    A_log, dt_bias = A_log.contiguous(), dt_bias.contiguous()
    gates = GdnGates(a_col, b_col, heads, A_log.data_ptr(), dt_bias.data_ptr(), g.data_ptr(), beta.data_ptr(),
                     g.stride(0))
    arr = segment_array(w.segments)
    L = load()
    if workspace is None:
        workspace = gemm_workspace(a.m, w.n, w.k, flags, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("nvfp4_gemm_gdn", L.nvfp4_gemm_gdn(
        _ptr(a.q), _ptr(a.sf), _ptr(a.scale), _ptr(w.q), _ptr(w.sf), a.m, w.n, w.k, arr, len(w.segments),
        _ptr(out), out.stride(0), ctypes.byref(gates), _ptr(workspace), ws_bytes, flags, _stream(dev)))
    return out, g, beta


def fp8_calibrate(x, amax, scale):
    """``nvfp4_fp8_calibrate``: fold ``x`` (BF16/FP32, leading dimension =
    rows, the rest flattened into the width) into the running ``amax`` and
    write the calibrated FP8 scale ``amax / 448`` into ``scale`` (both
    1-element FP32 device tensors; start ``amax`` at 0)."""
    _require_cuda(x, amax, scale)
    x2 = x.reshape(x.shape[0], -1) if x.dim() != 2 else x
    _check("nvfp4_fp8_calibrate", load().nvfp4_fp8_calibrate(
        _ptr(x2), _in_dtype(x2), x2.shape[0], x2.shape[1], x2.stride(0), _ptr(amax), _ptr(scale),
        _stream(x.device)))
    return scale


def kv_cache_quantize_fp8(k, v, k_scale, v_scale, k_cache, v_cache, slot_mapping=None):
    """``nvfp4_kv_cache_quantize_fp8``: quantise the new tokens' K and V
    (``tokens x ...``, BF16/FP32) to E4M3 with their calibrated scales and
    store token t's row in cache row ``slot_mapping[t]`` (int64; negative =
    skip; None = slot t).  The caches are uint8 ``num_slots x ...`` tensors
    whose rows are written in place."""
    import torch
    _require_cuda(k, v, k_scale, v_scale, k_cache, v_cache, slot_mapping)
    if k.shape != v.shape or k.dtype != v.dtype:
        raise ValueError("k and v must have one shape and dtype")
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8 or k_cache.shape != v_cache.shape:
        raise ValueError("the caches must be uint8 tensors of one shape")
    if k_cache.stride(0) != v_cache.stride(0):
        raise ValueError("the caches must share a row stride")
    if slot_mapping is not None and (slot_mapping.dtype != torch.int64 or slot_mapping.numel() != k.shape[0]):
        raise ValueError("slot_mapping must be int64 with one entry per token")
    k2 = k.reshape(k.shape[0], -1)
    v2 = v.reshape(v.shape[0], -1)
    kc = k_cache.view(k_cache.shape[0], -1)     # a view: the kernel writes the caller's rows
    vc = v_cache.view(v_cache.shape[0], -1)
    if kc.shape[1] != k2.shape[1]:
        raise ValueError("cache rows and K/V rows differ in width")
    _check("nvfp4_kv_cache_quantize_fp8", load().nvfp4_kv_cache_quantize_fp8(
        _ptr(k2), _ptr(v2), _in_dtype(k2), k2.shape[0], k2.shape[1], k2.stride(0), v2.stride(0),
        _ptr(slot_mapping), kc.shape[0], _ptr(k_scale), _ptr(v_scale), _ptr(kc), _ptr(vc), kc.stride(0),
        _stream(k.device)))
    return k_cache, v_cache


def gemm_decode_noalloc(a: QuantizedActivation, w: FusedWeight, out, segments=None):
    """``nvfp4_gemm_decode_noalloc``: the decode GEMM into the caller's ``out``
    (m x n, BF16 or FP32) using the library's built-in scratch; neither this
    wrapper nor the C call allocates device memory.  m <= 16."""
    if a.k != w.k:
        raise ValueError("K mismatch between activations and weight")
    segments = w.segments if segments is None else segments
    odt = NVFP4_OUT_FP32 if out.element_size() == 4 else NVFP4_OUT_BF16
    arr = segment_array(segments)
    _check("nvfp4_gemm_decode_noalloc", load().nvfp4_gemm_decode_noalloc(
        _ptr(a.q), _ptr(a.sf), _ptr(a.scale), _ptr(w.q), _ptr(w.sf), a.m, w.n, w.k, arr, len(segments),
        _ptr(out), odt, out.stride(0), _stream(out.device)))
    return out


def gemm_swiglu_quantize(a: QuantizedActivation, w: FusedWeight, h_scale, out: QuantizedActivation | None = None):
    """``nvfp4_gemm_swiglu_quantize``: the gate/up GEMM of a gated MLP with
    h = bf16(silu(g) * u) quantised in its epilogue (static scale ``h_scale``,
    a 1-element FP32 device tensor).  ``w`` holds [gate; up] (2f rows).
    Returns h as a QuantizedActivation (m x f), ready for the down GEMM."""
    import torch
    _require_cuda(h_scale)
    if a.k != w.k or w.n % 2 != 0:
        raise ValueError("K mismatch, or the weight is not [gate; up]")
    f = w.n // 2
    L = load()
    if out is None:
        out = QuantizedActivation(
            q=torch.empty((a.m, f // 2), dtype=torch.uint8, device=a.q.device),
            sf=torch.empty(max(L.nvfp4_sf_bytes(a.m, f), 1), dtype=torch.uint8, device=a.q.device),
            scale=h_scale, m=a.m, k=f)
    arr = segment_array(w.segments)
    _check("nvfp4_gemm_swiglu_quantize", L.nvfp4_gemm_swiglu_quantize(
        _ptr(a.q), _ptr(a.sf), _ptr(a.scale), _ptr(w.q), _ptr(w.sf), a.m, f, w.k, arr, len(w.segments),
        _ptr(h_scale), _ptr(out.q), _ptr(out.sf), _stream(a.q.device)))
    return out


def linear_decode(a, w: FusedWeight, act_scale=None, out_dtype=None, out=None, workspace=None, scale_out=None):
    """``nvfp4_linear_decode``: one W4A4 layer for m <= 64 tokens in one launch
    (activation quantisation fused into the decode GEMM).  ``act_scale``: a
    1-element FP32 device scale, or ``None`` for the dynamic scale (written to
    ``scale_out`` when given).  Returns the m x n output."""
    import torch
    _require_cuda(a, act_scale)
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("activations must be a 2-D tensor with unit column stride")
    m, k = a.shape
    if k != w.k:
        raise ValueError("K mismatch between activations and weight")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((m, w.n), dtype=out_dtype, device=a.device)
    odt = {torch.bfloat16: NVFP4_OUT_BF16, torch.float32: NVFP4_OUT_FP32}[out.dtype]
    if workspace is None:
        workspace = gemm_workspace(max(m, 1), w.n, w.k, NVFP4_GEMM_FORCE_DECODE, out.device)
    arr = segment_array(w.segments)
    _check("nvfp4_linear_decode", load().nvfp4_linear_decode(
        _ptr(a), _in_dtype(a), m, k, a.stride(0), _ptr(act_scale), _ptr(scale_out), _ptr(w.q), _ptr(w.sf), w.n,
        arr, len(w.segments), _ptr(out), odt, out.stride(0), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(out.device)))
    return out


_prefill_ws_cache: dict = {}


def linear_prefill(a, w: FusedWeight, act_scale, out_dtype=None, out=None, a_out: QuantizedActivation | None = None,
                   workspace=None):
    """``nvfp4_linear_prefill``: one W4A4 layer for m > 64 tokens in one
    launch (the static-scale activation quantisation fused into the large-M
    GEMM).  ``act_scale``: 1-element FP32 device scale.  ``a_out`` receives the
    quantised activations (allocated when not given).  Returns
    ``(out, a_out)``."""
    import torch
    _require_cuda(a, act_scale)
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("activations must be a 2-D tensor with unit column stride")
    m, k = a.shape
    if k != w.k:
        raise ValueError("K mismatch between activations and weight")
    L = load()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((m, w.n), dtype=out_dtype, device=a.device)
    odt = {torch.bfloat16: NVFP4_OUT_BF16, torch.float32: NVFP4_OUT_FP32}[out.dtype]
    if a_out is None:
        a_out = QuantizedActivation(
            q=torch.empty((m, k // 2), dtype=torch.uint8, device=a.device),
            sf=torch.empty(max(L.nvfp4_sf_bytes(m, k), 1), dtype=torch.uint8, device=a.device),
            scale=act_scale, m=m, k=k)
    if workspace is None:
        # one per (device, current stream): calls that may overlap must not share it
        need = max(int(L.nvfp4_linear_prefill_workspace_size(m)), 16)
        key = _ws_key(a.device)
        ws = _prefill_ws_cache.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=a.device)   # zeroed once, as the call requires
            _prefill_ws_cache[key] = ws
        workspace = ws
    arr = segment_array(w.segments)
    _check("nvfp4_linear_prefill", L.nvfp4_linear_prefill(
        _ptr(a), _in_dtype(a), m, k, a.stride(0), _ptr(act_scale), _ptr(a_out.q), _ptr(a_out.sf), _ptr(w.q),
        _ptr(w.sf), w.n, arr, len(w.segments), _ptr(out), odt, out.stride(0), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(out.device)))
    return out, a_out


def linear(a, w: FusedWeight, act_scale=None, out_dtype=None, flags: int = NVFP4_GEMM_AUTO):
    """One W4A4 linear layer: quantise ``a`` on the fly, then the fused GEMM."""
    return gemm(quantize_act(a, act_scale), w, out_dtype=out_dtype, flags=flags)


def check_device_status(device=None):
    _check("nvfp4_check_device_status", load().nvfp4_check_device_status(_stream(device)))


def version() -> int:
    return int(load().nvfp4_version())


def gemm_kernel_for(m: int, n: int, sms: int, flags: int = NVFP4_GEMM_AUTO, with_gates: bool = False) -> int:
    """``nvfp4_gemm_kernel_for``: the NVFP4_GEMM_FORCE_* value of the kernel
    nvfp4_gemm runs for an m x n output on a device with ``sms`` SMs."""
    return int(load().nvfp4_gemm_kernel_for(m, n, sms, flags, int(bool(with_gates))))
