"""Guard bands: every entry point writes only inside the buffers it is given.

Each output is carved out of a larger device buffer filled with a sentinel
byte (4 KB on either side); after the call the sentinel must be intact before
and after every output and, for outputs with a leading dimension larger than
their width, in the gap at the end of every row.  Shapes are ragged (rows not a
multiple of the 128- or 256-row tiles, widths not a multiple of the 256-column
tiles, K with a partial k-tile) so that clipped tile edges, padding rows and
padding k-blocks meet the ends of the buffers."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic

pytestmark = pytest.mark.gpu
SENT = 0xA5
PAD = 4096
LARGE, DECODE, PAIR = nv.NVFP4_GEMM_FORCE_LARGE, nv.NVFP4_GEMM_FORCE_DECODE, nv.NVFP4_GEMM_FORCE_LARGE_PAIR


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


class Guard:
    """`nbytes` of device memory between two sentinel bands."""

    def __init__(self, nbytes):
        self.n = nbytes
        self.buf = torch.full((PAD + nbytes + PAD,), SENT, dtype=torch.uint8, device="cuda")

    def bytes(self):
        return self.buf[PAD:PAD + self.n]

    def view(self, dtype, shape):
        return self.bytes().view(dtype).view(shape)

    def check(self, what):
        b = self.buf.cpu().numpy()
        assert (b[:PAD] == SENT).all(), f"{what}: bytes written before the buffer"
        assert (b[PAD + self.n:] == SENT).all(), f"{what}: bytes written after the buffer"


class Strided(Guard):
    """A rows x cols tensor with row stride `ld` elements; the row gaps hold the sentinel too."""

    def __init__(self, rows, cols, ld, dtype):
        self.rows, self.cols, self.ld = rows, cols, ld
        self.esz = torch.tensor([], dtype=dtype).element_size()
        super().__init__(rows * ld * self.esz)
        self.full = self.view(dtype, (rows, ld))
        self.t = self.full[:, :cols]

    def check(self, what):
        super().check(what)
        rows = self.bytes().cpu().numpy().reshape(self.rows, self.ld * self.esz)
        assert (rows[:, self.cols * self.esz:] == SENT).all(), f"{what}: bytes written in the row gap"


def _act(m, k, seed, static=True):
    a = synthetic.activations(m, k, seed=seed)[0].cuda()
    scale = nv.quantize_act(a).scale.clone() if static else None
    return a, scale


def _weight(widths, k, seed):
    return nv.quantize_weight([synthetic.weights(n, k, 0.02, seed=seed + i).cuda() for i, n in enumerate(widths)])


def _guarded_act(m, k):
    gq, gsf, gsc = Guard(m * k // 2), Guard(nv.sf_bytes(m, k)), Guard(4)
    out = nv.QuantizedActivation(q=gq.view(torch.uint8, (m, k // 2)), sf=gsf.bytes(),
                                 scale=gsc.view(torch.float32, (1,)), m=m, k=k)
    return out, (gq, gsf, gsc)


@pytest.mark.parametrize("static", [True, False])
def test_quantize_act(static):
    m, k = 130, 96
    a, scale = _act(m, k, 1, static)
    out, guards = _guarded_act(m, k)
    nv.quantize_act(a, act_scale=scale, out=out)
    torch.cuda.synchronize()
    nv.check_device_status()
    for g, what in zip(guards, ("codes", "scales", "scale")):
        g.check(what)


def test_quantize_weight_rows_of_one_module():
    """Quantising the second module of a fused buffer writes only its rows of
    the codes (and, being the last module, the padding scale rows)."""
    n0, n1, k = 200, 144, 320
    L = nv.load()
    w = synthetic.weights(n1, k, 0.02, seed=3).cuda()
    gq, gsf = Guard((n0 + n1) * k // 2), Guard(nv.sf_bytes(n0 + n1, k))
    scale = ctypes.c_float(0.01)
    got = ctypes.c_float(0.0)
    ws = nv.quant_workspace(w.device)
    st = L.nvfp4_quantize_weight(w.data_ptr(), 0, n1, k, k, n0, n0 + n1, ctypes.byref(scale), gq.bytes().data_ptr(),
                                 gsf.bytes().data_ptr(), ctypes.byref(got), ws.data_ptr(), ws.numel(),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    gq.check("codes")
    gsf.check("scales")
    codes = gq.bytes().cpu().numpy().reshape(n0 + n1, k // 2)
    assert (codes[:n0] == SENT).all(), "rows of the first module were written"


@pytest.mark.parametrize("flags,m", [(LARGE, 130), (PAIR, 130), (DECODE, 5), (DECODE, 37)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm(flags, m, out_dtype):
    widths, k = (48, 208, 32, 112), 320
    n = sum(widths)
    a, scale = _act(m, k, 2)
    aq = nv.quantize_act(a, act_scale=scale)
    fw = _weight(widths, k, 10)
    c = Strided(m, n, n + 24, out_dtype)
    nv.gemm(aq, fw, out=c.t, flags=flags)
    torch.cuda.synchronize()
    nv.check_device_status()
    c.check("C")


def test_gemm_decode_noalloc():
    m, widths, k = 5, (400,), 320
    a, scale = _act(m, k, 4)
    aq = nv.quantize_act(a, act_scale=scale)
    fw = _weight(widths, k, 20)
    c = Strided(m, 400, 424, torch.bfloat16)
    nv.gemm_decode_noalloc(aq, fw, c.t)
    torch.cuda.synchronize()
    nv.check_device_status()
    c.check("C")


def test_linear_decode():
    m, k, widths = 9, 320, (48, 352)
    a, scale = _act(m, k, 5)
    fw = _weight(widths, k, 30)
    c = Strided(m, 400, 424, torch.bfloat16)
    nv.linear_decode(a, fw, act_scale=scale, out=c.t)
    torch.cuda.synchronize()
    nv.check_device_status()
    c.check("C")


def test_linear_prefill():
    m, k, widths = 1300, 320, (48, 352)
    a, scale = _act(m, k, 6)
    fw = _weight(widths, k, 40)
    c = Strided(m, 400, 424, torch.bfloat16)
    aq, guards = _guarded_act(m, k)
    nv.linear_prefill(a, fw, scale, out=c.t, a_out=aq)
    torch.cuda.synchronize()
    nv.check_device_status()
    c.check("C")
    guards[0].check("codes")
    guards[1].check("scales")


@pytest.mark.parametrize("static", [True, False])
def test_silu_mul_quantize(static):
    m, f = 130, 96
    gu = synthetic.mlp_glue_inputs(m, f).cuda()
    out, guards = _guarded_act(m, f)
    gh = Guard(m * f * 2)
    h = gh.view(torch.bfloat16, (m, f))
    h_scale = torch.tensor([0.01], dtype=torch.float32, device="cuda") if static else None
    nv.silu_mul_quantize(gu[:, :f], gu[:, f:], h_scale=h_scale, out=out, h_out=h)
    torch.cuda.synchronize()
    nv.check_device_status()
    for g, what in zip(guards + (gh,), ("codes", "scales", "scale", "h")):
        g.check(what)


def test_gemm_swiglu_quantize():
    m, f, k = 130, 128, 320
    a, scale = _act(m, k, 7)
    aq = nv.quantize_act(a, act_scale=scale)
    fw = _weight((f, f), k, 50)
    out, guards = _guarded_act(m, f)
    h_scale = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    nv.gemm_swiglu_quantize(aq, fw, h_scale, out=out)
    torch.cuda.synchronize()
    nv.check_device_status()
    guards[0].check("codes")
    guards[1].check("scales")


@pytest.mark.parametrize("flags,m", [(nv.NVFP4_GEMM_AUTO, 130), (PAIR, 130), (DECODE, 7)])
def test_gemm_gdn(flags, m):
    heads, k = 48, 320
    widths = (256, heads, heads)
    n = sum(widths)
    a, scale = _act(m, k, 8)
    aq = nv.quantize_act(a, act_scale=scale)
    fw = _weight(widths, k, 60)
    A_log, dt_bias = (t.cuda() for t in synthetic.gdn_gate_params(heads))
    c = Strided(m, n, n + 16, torch.bfloat16)
    g = Strided(m, heads, heads + 16, torch.float32)
    beta = Strided(m, heads, heads + 16, torch.float32)
    nv.gemm_gdn(aq, fw, 256, 256 + heads, A_log, dt_bias, flags=flags, out=c.t, g=g.t, beta=beta.t)
    torch.cuda.synchronize()
    nv.check_device_status()
    c.check("C")
    g.check("g")
    beta.check("beta")


def test_kv_cache_quantize_fp8():
    tokens, width, slots = 37, 1024, 80
    k_rows, v_rows = (t.cuda() for t in synthetic.kv_rows(tokens, width=width, seed=3))
    ks = torch.empty(1, dtype=torch.float32, device="cuda")
    vs = torch.empty(1, dtype=torch.float32, device="cuda")
    nv.fp8_calibrate(k_rows, torch.zeros(1, dtype=torch.float32, device="cuda"), ks)
    nv.fp8_calibrate(v_rows, torch.zeros(1, dtype=torch.float32, device="cuda"), vs)
    perm = torch.randperm(slots, generator=torch.Generator().manual_seed(1))[:tokens]
    slot_map = perm.clone()
    slot_map[::5] = -1                                 # some tokens are padding
    gk, gv = Guard(slots * width), Guard(slots * width)
    nv.kv_cache_quantize_fp8(k_rows, v_rows, ks, vs, gk.view(torch.uint8, (slots, width)),
                             gv.view(torch.uint8, (slots, width)), slot_map.cuda())
    torch.cuda.synchronize()
    nv.check_device_status()
    named = set(int(s) for s in slot_map.tolist() if s >= 0)
    for g, what in ((gk, "K cache"), (gv, "V cache")):
        g.check(what)
        rows = g.bytes().cpu().numpy().reshape(slots, width)
        untouched = [r for r in range(slots) if r not in named]
        assert (rows[untouched] == SENT).all(), f"{what}: rows not in the slot table were written"
