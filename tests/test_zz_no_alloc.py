"""The allocation-free decode GEMM (``nvfp4_gemm_decode_noalloc``), called
through the C ABI, against the workspace entry point ``nvfp4_gemm`` with
NVFP4_GEMM_FORCE_DECODE and against the oracle.

Two calls in a row on different problems, then the first problem again, so
that each call finds the built-in scratch holding the previous call's flags and
partial tiles.  The decode kernel sums partial tiles in a fixed CTA order, so
both entry points must give the same bits; each result must also meet the GEMM
tolerance against the oracle (per element 1e-3 * |A_hat row| * |W_hat row|,
relative Frobenius 2e-3).  This file is collected last and also passes on its
own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from helpers import act_from_codes, assert_gemm_close, dequant_codes, weight_from_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return nv.load()


def _problem(seed, m, widths, k):
    rng = np.random.default_rng(seed)
    n = sum(widths)
    ca = rng.integers(0, 16, (m, k)).astype(np.uint8)
    cw = rng.integers(0, 16, (n, k)).astype(np.uint8)
    sa = rng.integers(0x20, 0x48, (m, k // 16)).astype(np.uint8)
    sw = rng.integers(0x20, 0x48, (n, k // 16)).astype(np.uint8)
    s_ga = np.float32(0.75)
    segs, off = [], 0
    for i, wdt in enumerate(widths):
        segs.append((off, off + wdt, float(np.float32(0.5 + 0.37 * i))))
        off += wdt
    a = act_from_codes(ca, sa, s_ga)
    w = weight_from_codes(cw, sw, segs)
    a_hat = dequant_codes(ca, sa, s_ga)
    w_hat = np.concatenate([dequant_codes(cw[b:e], sw[b:e], np.float32(s)) for b, e, s in segs], axis=0)
    c64 = oracle.gemm(a_hat, w_hat)
    return a, w, a_hat, w_hat, c64


def _noalloc(lib, a, w, out):
    arr = nv.segment_array(w.segments)
    odt = nv.NVFP4_OUT_FP32 if out.dtype == torch.float32 else nv.NVFP4_OUT_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.nvfp4_gemm_decode_noalloc(
        ctypes.c_void_p(a.q.data_ptr()), ctypes.c_void_p(a.sf.data_ptr()), ctypes.c_void_p(a.scale.data_ptr()),
        ctypes.c_void_p(w.q.data_ptr()), ctypes.c_void_p(w.sf.data_ptr()), a.m, w.n, w.k, arr, len(w.segments),
        ctypes.c_void_p(out.data_ptr()), odt, out.stride(0), stream)
    assert st == 0, lib.nvfp4_get_last_error_string()


def test_noalloc_decode_matches_workspace_entry_point_on_consecutive_calls(lib):
    p1 = _problem(101, 16, (256, 128, 512), 1024)     # full 16 tokens, three segments
    p2 = _problem(202, 5, (2048, 1536), 2560)         # ragged token count, longer k
    out1 = torch.empty((16, p1[1].n), dtype=torch.float32, device="cuda")
    out2 = torch.empty((5, p2[1].n), dtype=torch.bfloat16, device="cuda")
    out1_again = torch.empty_like(out1)
    torch.cuda.synchronize()

    _noalloc(lib, p1[0], p1[1], out1)                 # first call: one-time set-up, then the kernel
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    _noalloc(lib, p2[0], p2[1], out2)                 # second call in a row, same stream
    _noalloc(lib, p1[0], p1[1], out1_again)           # the first problem once more
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, "the allocation-free call changed the device's free memory"
    nv.check_device_status()

    ref1 = nv.gemm(p1[0], p1[1], out_dtype=torch.float32, flags=nv.NVFP4_GEMM_FORCE_DECODE)
    ref2 = nv.gemm(p2[0], p2[1], out_dtype=torch.bfloat16, flags=nv.NVFP4_GEMM_FORCE_DECODE)
    ref2_32 = nv.gemm(p2[0], p2[1], out_dtype=torch.float32, flags=nv.NVFP4_GEMM_FORCE_DECODE)
    torch.cuda.synchronize()
    assert torch.equal(out1, ref1), "first call differs from nvfp4_gemm"
    assert torch.equal(out2, ref2), "second call differs from nvfp4_gemm"
    assert torch.equal(out1_again, ref1), "third call differs from nvfp4_gemm"
    assert_gemm_close(out1, p1[4], p1[2], p1[3], "first problem")
    assert_gemm_close(ref2_32, p2[4], p2[2], p2[3], "second problem")
    # BF16 output = round-to-nearest-even of the FP32 output
    assert torch.equal(out2, ref2_32.to(torch.bfloat16))


def test_noalloc_decode_rejects_more_tokens_than_its_scratch(lib):
    a, w, *_ = _problem(303, 17, (256,), 256)
    out = torch.zeros((17, w.n), dtype=torch.bfloat16, device="cuda")
    arr = nv.segment_array(w.segments)
    st = lib.nvfp4_gemm_decode_noalloc(
        ctypes.c_void_p(a.q.data_ptr()), ctypes.c_void_p(a.sf.data_ptr()), ctypes.c_void_p(a.scale.data_ptr()),
        ctypes.c_void_p(w.q.data_ptr()), ctypes.c_void_p(w.sf.data_ptr()), a.m, w.n, w.k, arr, 1,
        ctypes.c_void_p(out.data_ptr()), nv.NVFP4_OUT_BF16, out.stride(0),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2 and b"m <= 16" in lib.nvfp4_get_last_error_string()
    torch.cuda.synchronize()
    assert not out.any(), "a refused call wrote output"
