"""GPU parity of the Gated DeltaNet gate epilogue (``nvfp4_gemm_gdn``):

  g    = -exp(A_log) * softplus(a + dt_bias)    ("Why Gated DeltaNet Survives
  beta = sigmoid(b)                               4-Bit Quantization", page
                                                  summary, "Gated DeltaNet
                                                  Mechanics"; abstract (ii))

``C`` must be bit-identical to ``nvfp4_gemm`` with the same arguments, and
the gates must match the oracle's FP64 gates evaluated on the BF16 values of
C's a and b columns (the values the kernel reads).  Tolerance, from the FP32
arithmetic: the kernel rounds t = a + dt_bias to FP32 (relative 2^-24 of t,
which moves softplus by at most |t| 2^-24 of itself, since sigmoid <=
softplus) and evaluates exp, log1p, one add and one multiply (a few ulp), so
|g - g64| <= (|t| + 16) 2^-23 |g64|; beta takes one exp, an add and a divide:
|beta - beta64| <= 2^-20 beta64.  Both add 1e-37 absolute for results that
underflow FP32."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic

pytestmark = pytest.mark.gpu
LARGE, DECODE, AUTO = nv.NVFP4_GEMM_FORCE_LARGE, nv.NVFP4_GEMM_FORCE_DECODE, nv.NVFP4_GEMM_AUTO
PAIR = nv.NVFP4_GEMM_FORCE_LARGE_PAIR
SENTINEL = 12345.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _check_gates(c, g, beta, a_col, b_col, A_log, dt_bias):
    heads = A_log.numel()
    cf = c.float().cpu().numpy()
    a = np.ascontiguousarray(cf[:, a_col:a_col + heads])
    b = np.ascontiguousarray(cf[:, b_col:b_col + heads])
    g64, beta64 = oracle.gdn_gates(a, b, A_log.numpy(), dt_bias.numpy())
    t = np.abs(a.astype(np.float64) + dt_bias.double().numpy())
    gg = g[:, :heads].double().cpu().numpy()
    bb = beta[:, :heads].double().cpu().numpy()
    g_err = np.abs(gg - g64) - ((t + 16) * 2.0 ** -23 * np.abs(g64) + 1e-37)
    b_err = np.abs(bb - beta64) - (2.0 ** -20 * beta64 + 1e-37)
    assert g_err.max() <= 0, ("g", np.unravel_index(g_err.argmax(), g_err.shape), g_err.max())
    assert b_err.max() <= 0, ("beta", np.unravel_index(b_err.argmax(), b_err.shape), b_err.max())
    assert np.all(gg <= 0) and np.all((bb >= 0) & (bb <= 1))   # exact 0 where FP32 underflows


def _run(p, flags, a_col, b_col, heads, ldg=None, seed=9):
    fw = nv.quantize_weight([w.cuda() for w in p.modules])
    aq = nv.quantize_act(p.a.cuda())
    A_log, dt_bias = synthetic.gdn_gate_params(heads, seed)
    ldg = heads if ldg is None else ldg
    g = torch.full((p.m, ldg), SENTINEL, dtype=torch.float32, device="cuda")
    beta = torch.full((p.m, ldg), SENTINEL, dtype=torch.float32, device="cuda")
    c, g, beta = nv.gemm_gdn(aq, fw, a_col, b_col, A_log.cuda(), dt_bias.cuda(), flags=flags, g=g, beta=beta)
    plain = nv.gemm(aq, fw, out_dtype=torch.bfloat16, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(c, plain), "C differs from nvfp4_gemm"
    assert torch.all(g[:, heads:] == SENTINEL) and torch.all(beta[:, heads:] == SENTINEL)
    _check_gates(c, g, beta, a_col, b_col, A_log, dt_bias)
    return c, g, beta


@pytest.mark.parametrize("flags,m", [(LARGE, 300), (AUTO, 130), (PAIR, 300), (DECODE, 8), (DECODE, 33),
                                     (AUTO, 64), (LARGE, 5)])
def test_gdn_gates_in_proj_layout(flags, m):
    """The in-proj layout with small q/k/v modules: the a and b ranges are the
    last two 48-wide segments."""
    p = synthetic.gdn_in_proj(m=m, k=512, widths=(256, 256, 512, 512, 48, 48),
                              stds=(0.02, 0.02, 0.02, 0.02, 0.2, 0.2))
    _run(p, flags, 1536, 1584, 48, ldg=64)


@pytest.mark.parametrize("flags,m", [(LARGE, 200), (PAIR, 260), (DECODE, 17)])
def test_gdn_gates_unaligned_ranges(flags, m):
    """Ranges that start inside a 32-column chunk and cross chunk, half-tile
    and 256-column tile boundaries, with rows past the last full tile."""
    p = synthetic.gdn_in_proj(m=m, k=256, widths=(512,), stds=(0.5,))
    _run(p, flags, 40, 240, 24)


def test_gdn_gates_extreme_arguments():
    """Large-magnitude a and b (weights scaled up) reach both tails of
    softplus and sigmoid."""
    p = synthetic.gdn_in_proj(m=150, k=512, widths=(128, 64, 64), stds=(0.02, 8.0, 8.0))
    c, g, beta = _run(p, LARGE, 128, 192, 64)
    a = c[:, 128:192].float()
    assert a.abs().max().item() > 30 and c[:, 192:256].float().abs().max().item() > 30


def test_gdn_gates_fused_in_proj_8192():
    """The full fused in-proj (8192 x 5120 against [2048, 2048, 4096, 4096,
    48, 48]) in the launch configuration the benchmark times: every gate
    checked against the oracle."""
    p = synthetic.gdn_in_proj()
    _run(p, AUTO, 12288, 12336, 48)
