"""The C-ABI library: it loads, exports every symbol include/nvfp4.h declares,
its layout helpers agree with the oracle's independent index map, and argument
errors come back as status codes before any CUDA call (so these run without a
GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return nv.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("nvfp4_quantize_weight", "nvfp4_quantize_act", "nvfp4_gemm"):
        assert n in names
    assert set(names) == set(nv.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version(lib):
    assert lib.nvfp4_version() >= 100


def test_sf_layout_helpers_match_oracle_map(lib):
    for rows, k in [(1, 32), (64, 256), (129, 288), (300, 320), (12384, 5120)]:
        assert lib.nvfp4_sf_bytes(rows, k) == oracle.sf_tiled_bytes(rows, k)
    rng = np.random.default_rng(0)
    for _ in range(2000):
        k = int(rng.integers(1, 400)) * 16
        row = int(rng.integers(0, 5000))
        kb = int(rng.integers(0, k // 16))
        assert lib.nvfp4_sf_offset(row, kb, k) == oracle.sf_tiled_offset(row, kb, k)
    assert lib.nvfp4_sf_offset(0, 0, 30) == -1
    assert lib.nvfp4_sf_offset(-1, 0, 32) == -1
    assert lib.nvfp4_sf_bytes(4, 24) == 0


def _status(fn, *args):
    return fn(*args)


FAKE = ctypes.c_void_p(0x10000)          # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def test_quantize_act_argument_errors(lib):
    ws = ctypes.c_void_p(0x20000)
    st = lib.nvfp4_quantize_act(FAKE, 0, 8, 48, 48, None, FAKE, FAKE, FAKE, ws, 256, None)
    assert st == 1 and b"multiple of 32" in lib.nvfp4_get_last_error_string()
    assert lib.nvfp4_quantize_act(FAKE, 7, 8, 64, 64, FAKE, None, FAKE, FAKE, None, 0, None) == 1   # bad dtype
    assert lib.nvfp4_quantize_act(FAKE, 0, 8, 64, 32, FAKE, None, FAKE, FAKE, None, 0, None) == 1   # lda < k
    assert lib.nvfp4_quantize_act(None, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, None, 0, None) == 1   # null input
    assert lib.nvfp4_quantize_act(MISALIGNED, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, None, 0, None) == 3
    assert lib.nvfp4_quantize_act(FAKE, 0, 8, 64, 68, FAKE, None, FAKE, FAKE, None, 0, None) == 3   # row pitch
    # dynamic mode needs an output scale and a workspace
    assert lib.nvfp4_quantize_act(FAKE, 0, 8, 64, 64, None, None, FAKE, FAKE, ws, 256, None) == 1
    assert lib.nvfp4_quantize_act(FAKE, 0, 8, 64, 64, None, FAKE, FAKE, FAKE, None, 0, None) == 6
    assert lib.nvfp4_quantize_act(FAKE, 0, 8, 64, 64, None, FAKE, FAKE, FAKE, ws, 16, None) == 6
    # empty input is a no-op that needs no device
    assert lib.nvfp4_quantize_act(FAKE, 0, 0, 64, 64, FAKE, None, FAKE, FAKE, None, 0, None) == 0


def test_quantize_weight_argument_errors(lib):
    one = ctypes.c_float(1.0)
    bad = ctypes.c_float(-1.0)
    nan = ctypes.c_float(float("nan"))
    out = ctypes.c_float(0)
    f = lib.nvfp4_quantize_weight
    assert f(FAKE, 0, 16, 64, 64, 10, 20, ctypes.byref(one), FAKE, FAKE, None, None, 0, None) == 1  # rows overflow
    assert f(FAKE, 0, 16, 64, 64, -1, 20, ctypes.byref(one), FAKE, FAKE, None, None, 0, None) == 1
    assert f(FAKE, 0, 16, 64, 64, 0, 16, ctypes.byref(bad), FAKE, FAKE, None, None, 0, None) == 1
    assert f(FAKE, 0, 16, 64, 64, 0, 16, ctypes.byref(nan), FAKE, FAKE, None, None, 0, None) == 1
    assert f(FAKE, 0, 16, 64, 64, 0, 16, None, FAKE, FAKE, None, FAKE, 256, None) == 1        # no scale out
    assert f(FAKE, 0, 16, 64, 64, 0, 16, None, FAKE, FAKE, ctypes.byref(out), None, 0, None) == 6
    assert f(FAKE, 0, 16, 64, 64, 0, 16, ctypes.byref(one), MISALIGNED, FAKE, None, None, 0, None) == 3


def _segs(*triples):
    return nv.segment_array(list(triples))


def test_gemm_segment_table_errors(lib):
    g = lib.nvfp4_gemm

    def call(segs, n=64, nsegs=None):
        nsegs = len(segs) if nsegs is None else nsegs
        return g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, n, 64, segs, nsegs, FAKE, 0, n, None, 0, 0, None)

    assert call(_segs((0, 32, 1.0), (40, 64, 1.0))) == 1          # gap
    assert call(_segs((0, 48, 1.0), (32, 64, 1.0))) == 1          # overlap
    assert call(_segs((32, 64, 1.0), (0, 32, 1.0))) == 1          # unsorted
    assert call(_segs((0, 48, 1.0))) == 1                         # does not cover n
    assert call(_segs((0, 24, 1.0), (24, 64, 1.0))) == 1          # boundary not a multiple of 16
    assert call(_segs((0, 64, 0.0))) == 1                         # non-positive scale
    assert call(_segs((0, 64, float("inf")))) == 1
    assert call(_segs((0, 64, 1.0)), nsegs=0) == 1
    many = _segs(*[(16 * i, 16 * (i + 1), 1.0) for i in range(17)])
    assert call(many, n=17 * 16) == 1                             # more than 16 segments
    assert b"segment" in lib.nvfp4_get_last_error_string()


def test_gemm_shape_and_alignment_errors(lib):
    g = lib.nvfp4_gemm
    s = _segs((0, 64, 1.0))
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 48, s, 1, FAKE, 0, 64, None, 0, 0, None) == 1      # k % 32
    s40 = _segs((0, 40, 1.0))
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 40, 64, s40, 1, FAKE, 0, 40, None, 0, 0, None) == 1    # n % 16
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 32, None, 0, 0, None) == 1      # ldc < n
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 5, 64, None, 0, 0, None) == 1      # out dtype
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, None, 0, 9, None) == 1      # flags
    assert g(FAKE, FAKE, None, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, None, 0, 0, None) == 1      # null scale
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, MISALIGNED, 0, 64, None, 0, 0, None) == 3
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 68, None, 0, 0, None) == 3     # row pitch
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 65, 64, 64, s, 1, FAKE, 0, 64, None, 0, 2, None) == 2     # decode m>64
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 64, s, 1, FAKE, 0, 64, None, 0, 0, None) == 0      # empty


def test_valid_call_without_a_gpu_fails_loudly(lib):
    """With arguments that pass validation, a machine without a usable sm_100a
    GPU gets NVFP4_ERR_CUDA / UNSUPPORTED, never a silent result."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    s = _segs((0, 64, 1.0))
    st = lib.nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 200, 64, 64, s, 1, FAKE, 0, 64, None, 0, 0, None)
    assert st in (2, 4)
    assert lib.nvfp4_get_last_error_string()
    ws = ctypes.c_void_p(0x40000)
    st = lib.nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, ws, 1 << 24, 0, None)
    assert st in (2, 4)


def test_decode_gemm_requires_workspace(lib):
    s = _segs((0, 64, 1.0))
    need = lib.nvfp4_gemm_workspace_size(8, 64, 64, 0)
    assert need > 0 and lib.nvfp4_gemm_workspace_size(8, 64, 64, 1) == 0
    assert lib.nvfp4_gemm_workspace_size(300, 64, 64, 0) == 0
    assert lib.nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, None, 0, 0, None) == 6
    ws = ctypes.c_void_p(0x40000)
    assert lib.nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, ws, need - 16, 0, None) == 6
    assert lib.nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, s, 1, FAKE, 0, 64, MISALIGNED, need, 0,
                          None) == 3


def test_decode_noalloc_limits_without_a_device(lib):
    """The allocation-free decode call refuses m above its built-in scratch
    before touching a device, and m == 0 is a no-op."""
    s = _segs((0, 64, 1.0))
    f = lib.nvfp4_gemm_decode_noalloc
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 17, 64, 64, s, 1, FAKE, 0, 64, None) == 2
    msg = lib.nvfp4_get_last_error_string()
    assert b"m <= 16" in msg and b"workspace" in msg
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 64, 64, s, 1, FAKE, 0, 64, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 64, 64, s, 1, FAKE, 0, 64, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 64, s, 1, FAKE, 0, 64, None) == 0
    assert nv.NVFP4_NOALLOC_MAX_M == 16
    # the built-in scratch is exactly the decode workspace for 16 tokens
    assert lib.nvfp4_gemm_workspace_size(16, 64, 64, nv.NVFP4_GEMM_FORCE_DECODE) == 160 * 16 * 128 * 8


def test_silu_mul_quantize_argument_errors(lib):
    f = lib.nvfp4_silu_mul_quantize
    ws = ctypes.c_void_p(0x20000)
    assert f(FAKE, FAKE, 8, 48, 96, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 1     # f % 32
    assert f(FAKE, FAKE, 8, 64, 32, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 1     # ldgu < f
    assert f(None, FAKE, 8, 64, 128, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 1    # null g
    assert f(FAKE, FAKE, 8, 64, 128, FAKE, None, FAKE, FAKE, FAKE, 32, None, 0, None) == 1   # ldh < f
    assert f(FAKE, MISALIGNED, 8, 64, 128, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 3
    assert f(FAKE, FAKE, 8, 64, 68, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 3     # row pitch
    assert f(FAKE, FAKE, 8, 64, 128, None, None, FAKE, FAKE, None, 0, ws, 256, None) == 1    # dynamic: no scale out
    assert f(FAKE, FAKE, 8, 64, 128, None, FAKE, FAKE, FAKE, None, 0, None, 0, None) == 6    # dynamic: no workspace
    assert f(FAKE, FAKE, 0, 64, 128, FAKE, None, FAKE, FAKE, None, 0, None, 0, None) == 0    # empty


def test_linear_decode_argument_errors(lib):
    f = lib.nvfp4_linear_decode
    s = _segs((0, 64, 1.0))
    ws = ctypes.c_void_p(0x40000)
    need = lib.nvfp4_gemm_workspace_size(8, 64, 64, 2)
    assert f(FAKE, 0, 65, 64, 64, FAKE, None, FAKE, FAKE, 64, s, 1, FAKE, 0, 64, ws, need, None) == 2   # m > 64
    assert f(FAKE, 0, 8, 48, 48, FAKE, None, FAKE, FAKE, 64, s, 1, FAKE, 0, 64, ws, need, None) == 1    # k % 32
    assert f(FAKE, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, 40, _segs((0, 40, 1.0)), 1, FAKE, 0, 40, ws, need,
             None) == 1                                                                                  # n % 16
    assert f(FAKE, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, 64, s, 1, FAKE, 0, 64, None, 0, None) == 6     # workspace
    assert f(MISALIGNED, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, 64, s, 1, FAKE, 0, 64, ws, need, None) == 3
    assert f(FAKE, 0, 8, 64, 64, FAKE, None, FAKE, FAKE, 64, _segs((0, 48, 1.0)), 1, FAKE, 0, 64, ws, need,
             None) == 1                                                                                  # segments
    assert f(FAKE, 0, 0, 64, 64, FAKE, None, FAKE, FAKE, 64, s, 1, FAKE, 0, 64, ws, need, None) == 0     # empty


def test_gemm_swiglu_quantize_argument_errors(lib):
    f = lib.nvfp4_gemm_swiglu_quantize
    s2 = _segs((0, 128, 1.0), (128, 256, 1.0))
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 64, 64, _segs((0, 128, 1.0)), 1, FAKE, FAKE, FAKE, None) == 1  # f % 128
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 128, 48, s2, 2, FAKE, FAKE, FAKE, None) == 1                    # k % 32
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 128, 64, _segs((0, 128, 1.0)), 1, FAKE, FAKE, FAKE, None) == 1  # segs
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 128, 64, s2, 2, None, FAKE, FAKE, None) == 1                    # no scale
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 128, 64, s2, 2, FAKE, MISALIGNED, FAKE, None) == 3
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 128, 64, s2, 2, FAKE, FAKE, FAKE, None) == 0                    # empty


def test_gemm_gdn_argument_errors(lib):
    f = lib.nvfp4_gemm_gdn
    s = _segs((0, 128, 1.0))

    def call(a_col=64, b_col=96, heads=32, ldg=32, ptrs=(FAKE, FAKE, FAKE, FAKE), m=8, n=128):
        gates = nv.GdnGates(a_col, b_col, heads, *[None if p is None else p.value for p in ptrs], ldg)
        segs = s if n == 128 else _segs((0, n, 1.0))
        return f(FAKE, FAKE, FAKE, FAKE, FAKE, m, n, 64, segs, 1, FAKE, n, ctypes.byref(gates), None, 0, 1, None)

    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 128, 64, s, 1, FAKE, 128, None, None, 0, 1, None) == 1   # no gates
    assert call(heads=0) == 1
    assert call(a_col=-1) == 1
    assert call(a_col=100) == 1                          # a range past n
    assert call(b_col=97) == 1                           # b range past n
    assert call(ldg=16) == 1                             # ldg < heads
    assert call(ptrs=(FAKE, None, FAKE, FAKE)) == 1      # no dt_bias
    assert call(ptrs=(FAKE, FAKE, FAKE, ctypes.c_void_p(0x10002))) == 3
    assert call(a_col=100) == 1 and b"gemm_gdn" in lib.nvfp4_get_last_error_string()
    assert call(m=0) == 0                                # empty


def test_fp8_kv_argument_errors(lib):
    cal = lib.nvfp4_fp8_calibrate
    assert cal(FAKE, 0, 8, 24, 24, FAKE, FAKE, None) == 1          # width % 16
    assert cal(FAKE, 0, 8, 32, 16, FAKE, FAKE, None) == 1          # ld < width
    assert cal(FAKE, 0, 8, 32, 32, None, FAKE, None) == 1          # no amax
    assert cal(FAKE, 5, 8, 32, 32, FAKE, FAKE, None) == 1          # dtype
    assert cal(MISALIGNED, 0, 8, 32, 32, FAKE, FAKE, None) == 3
    kv = lib.nvfp4_kv_cache_quantize_fp8

    def call(tokens=8, width=64, ld=64, slots=FAKE, num_slots=16, cache_ld=64, k=FAKE, ks=FAKE, kc=FAKE, dt=0):
        return kv(k, FAKE, dt, tokens, width, ld, ld, slots, num_slots, ks, FAKE, kc, FAKE, cache_ld, None)

    assert call(width=40) == 1                                     # width % 16
    assert call(ld=32) == 1                                        # ld < width
    assert call(cache_ld=48) == 1                                  # cache row shorter than width
    assert call(num_slots=-1) == 1
    assert call(slots=None, tokens=20) == 1                        # identity mapping past the cache
    assert call(ks=None) == 1                                      # no scale
    assert call(dt=3) == 1
    assert call(k=MISALIGNED) == 3
    assert call(cache_ld=72) == 3                                  # cache rows not 16-byte aligned
    assert call(slots=ctypes.c_void_p(0x10004)) == 3              # slot table not 8-byte aligned
    assert call(tokens=1 << 28, width=256) == 2                    # too many units
    assert call(tokens=0) == 0 and call(tokens=0, k=None) == 0     # empty
    assert call(width=40) == 1 and b"kv_cache_quantize_fp8" in lib.nvfp4_get_last_error_string()


def test_new_bindings_refuse_host_tensors(lib):
    """The gate and KV-cache calls run on the GPU only: host tensors are
    rejected before any work (no CPU fallback)."""
    import torch
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    one = torch.ones(1, dtype=torch.float32)
    cache = torch.zeros(8, 32, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        nv.fp8_calibrate(x, torch.zeros(1), one)
    with pytest.raises(ValueError, match="CUDA"):
        nv.kv_cache_quantize_fp8(x, x, one, one, cache, cache.clone())
    with pytest.raises(ValueError, match="CUDA"):
        nv.gemm_gdn(None, None, 0, 48, torch.zeros(48), torch.zeros(48))


def test_gemm_kernel_choice(lib):
    """AUTO: decode kernel up to 64 tokens; above, the CTA-pair kernel where it
    needs no more waves of tiles than the single-CTA kernel (148 SMs)."""
    import nvfp4_w4a4_quantized_07_b200 as nv
    pick = nv.gemm_kernel_for
    D, L, P = nv.NVFP4_GEMM_FORCE_DECODE, nv.NVFP4_GEMM_FORCE_LARGE, nv.NVFP4_GEMM_FORCE_LARGE_PAIR
    assert pick(1, 5120, 148) == D and pick(64, 34816, 148) == D
    assert pick(65, 5120, 148) == L and pick(255, 5120, 148) == L
    # 8192 x 12384: 64 x 49 = 3136 tiles = 22 waves; pairs: 32 x 49 = 1568 on 74 pairs = 22 waves
    assert pick(8192, 12384, 148) == P
    assert pick(4096, 5120, 148) == P                  # 5 waves either way
    assert pick(3712, 5120, 148) == L                  # 4 waves against 5 (29 row tiles do not pair up)
    assert pick(4736, 5120, 148) == L                  # 740 tiles = 5 waves; 380 pair tiles = 6 waves
    assert pick(8192, 12384, 148, with_gates=True) == L
    assert pick(8192, 12384, 148, flags=L) == L and pick(8, 128, 148, flags=P) == P
    assert pick(-1, 16, 148) == -1 and pick(16, 16, 0) == -1 and pick(16, 16, 148, flags=9) == -1


def test_linear_prefill_argument_errors(lib):
    f = lib.nvfp4_linear_prefill
    s = _segs((0, 256, 1.0))
    ws = ctypes.c_void_p(0x40000)
    need = lib.nvfp4_linear_prefill_workspace_size(300)
    assert need == 16 * ((3 * 8 + 15) // 16) and lib.nvfp4_linear_prefill_workspace_size(-1) == 0
    args = lambda m=300, dt=0, k=256, scale=FAKE, a=FAKE, wsp=ws, wsb=need, segs=s, n=256: (
        a, dt, m, k, k, scale, FAKE, FAKE, FAKE, FAKE, n, segs, 1, FAKE, 0, n, wsp, wsb, None)
    assert f(*args(m=64)) == 2                        # m <= 64: the decode layer's job
    assert f(*args(dt=1)) == 2                        # FP32 activations: two-call path
    assert f(*args(scale=None)) == 1                  # static scale required
    assert f(*args(k=48)) == 1                        # k % 32
    assert f(*args(wsp=None, wsb=0)) == 6             # workspace
    assert f(*args(wsb=need - 16)) == 6
    assert f(*args(a=MISALIGNED)) == 3
    assert f(*args(segs=_segs((0, 128, 1.0)))) == 1   # segments do not cover n
    assert f(*args(m=0)) == 0                         # empty


def test_default_workspaces_are_per_device_and_stream(lib, monkeypatch):
    """The binding's default workspaces (dynamic-scale quantisers, decode GEMM
    partials, one-launch prefill ready words) are cached per (device, current
    stream): calls on one stream reuse one buffer, calls on another stream get
    their own, and a larger need replaces the buffer.  Host logic only: the
    current stream and the device allocations are faked."""
    import torch

    class FakeStream:
        def __init__(self, handle):
            self.cuda_stream = handle

    current = {"h": 0x1000}
    made = []
    host_empty = torch.empty

    def fake_alloc(*shape, dtype=None, device=None, **kw):
        assert torch.device(device).type == "cuda"
        t = host_empty(*shape, dtype=dtype)
        made.append(t)
        return t

    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: FakeStream(current["h"]))
    monkeypatch.setattr(torch, "empty", fake_alloc)
    monkeypatch.setattr(nv, "_quant_ws_cache", {})
    monkeypatch.setattr(nv, "_ws_cache", {})

    q1 = nv.quant_workspace("cuda:0")
    assert q1.numel() == lib.nvfp4_quant_workspace_size()
    assert nv.quant_workspace("cuda:0") is q1
    dec = nv.NVFP4_GEMM_FORCE_DECODE
    g1 = nv.gemm_workspace(16, 5120, 5120, dec, "cuda:0")
    assert g1.numel() == lib.nvfp4_gemm_workspace_size(16, 5120, 5120, dec)
    assert nv.gemm_workspace(1, 5120, 5120, dec, "cuda:0") is g1          # smaller need: same buffer
    assert nv.gemm_workspace(8192, 5120, 5120, nv.NVFP4_GEMM_AUTO, "cuda:0") is None
    current["h"] = 0x2000                                                 # another stream
    q2 = nv.quant_workspace("cuda:0")
    g2 = nv.gemm_workspace(16, 5120, 5120, dec, "cuda:0")
    assert q2 is not q1 and g2 is not g1
    g3 = nv.gemm_workspace(64, 5120, 5120, dec, "cuda:0")                 # larger need: replaced
    assert g3 is not g2 and g3.numel() == lib.nvfp4_gemm_workspace_size(64, 5120, 5120, dec)
    current["h"] = 0x1000                                                 # back on the first stream
    assert nv.quant_workspace("cuda:0") is q1 and nv.gemm_workspace(16, 5120, 5120, dec, "cuda:0") is g1
    assert nv._ws_key("cuda:0") == (torch.device("cuda:0"), 0x1000)
    assert len(made) == 5
