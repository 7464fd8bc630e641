"""GPU parity of the MLP glue h = bf16(silu(g) * u) and its NVFP4 quantisation
(``nvfp4_silu_mul_quantize``) against the oracle.

h: each element within one BF16 unit in the last place of the oracle's
(e^-x comes from two different exp implementations, CUDA's expf and the host
C library's, which may differ by an FP32 ulp or two), and at most 0.1 % of
elements off at all.  The quantised bytes, the tiled scales (with padding) and
the tensor scale must equal the oracle's on the kernel's own h bit for bit
(the quantiser's FP32 decisions are fixed by the same reading as
``nvfp4_quantize_act``: "Why Gated DeltaNet Survives 4-Bit Quantization", page
summary "Background" item 1)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import assert_gemm_close, dequant_codes, sf_rowmajor, to_np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ordered(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns mapped to integers in value order (-0 and +0 adjacent)."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def _check_h(g: torch.Tensor, u: torch.Tensor, h: torch.Tensor):
    ref = oracle.silu_mul_bf16(_bits(g), _bits(u)).reshape(h.shape)
    got = _bits(h)
    d = np.abs(_ordered(got) - _ordered(ref))
    assert d.max() <= 1, f"h off by {d.max()} BF16 ulps"
    assert (d > 0).mean() <= 1e-3, f"{(d > 0).mean():.2e} of h elements differ"


def _check_quant(h: torch.Tensor, out: nv.QuantizedActivation, s: np.float32):
    h32 = h.float().cpu().numpy()
    q_ref, sf_ref = oracle.quantize(h32, s)
    np.testing.assert_array_equal(to_np_u8(out.q), q_ref)
    np.testing.assert_array_equal(to_np_u8(out.sf), oracle.sf_to_tiled(sf_ref, h32.shape[1]))


SHAPES = [(1, 32), (3, 64), (130, 1056), (300, 2048)]


@pytest.mark.parametrize("m,f", SHAPES)
@pytest.mark.parametrize("mode", ["dynamic", "static"])
def test_silu_mul_quantize_bit_exact(m, f, mode):
    gu = synthetic.mlp_glue_inputs(m, f, seed=m + f).cuda()
    g, u = gu[:, :f], gu[:, f:]
    scale = None
    if mode == "static":
        h_ref = oracle.silu_mul_bf16(_bits(g.cpu()), _bits(u.cpu())).reshape(m, f)
        s_cal = np.float32(oracle.global_scale(oracle.bf16_bits_to_f32(h_ref)) * np.float32(1.3))
        scale = torch.tensor([s_cal], dtype=torch.float32, device="cuda")
    out, h = nv.silu_mul_quantize(g, u, h_scale=scale, return_h=True)
    torch.cuda.synchronize()
    _check_h(g, u, h)
    s = np.float32(out.scale.item())
    if mode == "dynamic":
        assert s == oracle.global_scale(h.float().cpu().numpy())
    else:
        assert s == np.float32(scale.item())
    _check_quant(h, out, s)
    # the same codes without the h copy
    out2, none = nv.silu_mul_quantize(g, u, h_scale=scale)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(out2.q, out.q) and torch.equal(out2.sf, out.sf) and torch.equal(out2.scale, out.scale)


def test_silu_mul_special_values():
    """Saturating exponentials, signed zeros and denormal gates."""
    gvals = [-200.0, -88.0, -20.0, -1e-30, -0.0, 0.0, 1e-30, 3e-39, 20.0, 88.0, 200.0, 1.0, -1.0, 0.5, -0.5, 4.0]
    uvals = [1.0, -2.0, 3.0, 1e20, -1.0, 7.0, -1e30, 1e38, 0.5, -0.25, 1e-3, 0.0, -0.0, 1e4, -1e4, 2.0]
    m, f = 4, 32
    gate = torch.tensor(gvals * 2, dtype=torch.float32).repeat(m, 1) * torch.tensor([1.0, -1.0, 3.0, 1e-3]).view(m, 1)
    up = torch.tensor(uvals * 2, dtype=torch.float32).repeat(m, 1)
    gu = torch.cat([gate, up], dim=1).to(torch.bfloat16).cuda()
    g, u = gu[:, :f], gu[:, f:]
    out, h = nv.silu_mul_quantize(g, u, return_h=True)
    torch.cuda.synchronize()
    _check_h(g, u, h)
    s = np.float32(out.scale.item())
    assert s == oracle.global_scale(h.float().cpu().numpy())
    _check_quant(h, out, s)


def test_config_long_prefill_mlp_sampled():
    """The long-prefill MLP at full size: A 32768x5120 -> fused gate/up GEMM
    (two 17408-wide modules, own scales) -> glue (dynamic scale) -> down GEMM
    5120x17408.  Each stage is checked by the oracle on the previous stage's
    GPU output: the gate/up GEMM and the down GEMM on sampled rows and
    columns within the GEMM tolerance, the glue on sampled rows bit for bit
    and its tensor scale over the whole of h."""
    p = synthetic.mlp_gate_up()
    m, k, f = p.m, p.k, synthetic.MLP_INTERMEDIATE
    dev = torch.device("cuda")
    fw1 = nv.quantize_weight([w.to(dev) for w in p.modules])
    w2 = synthetic.mlp_down_weight()
    fw2 = nv.quantize_weight([w2.to(dev)])
    a = p.a.to(dev)
    aq = nv.quantize_act(a)
    c1 = nv.gemm(aq, fw1)                                   # m x 2f BF16
    hq, h = nv.silu_mul_quantize(c1[:, :f], c1[:, f:], return_h=True)
    c2 = nv.gemm(hq, fw2, out_dtype=torch.float32)         # m x 5120
    torch.cuda.synchronize()
    nv.check_device_status()

    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, 4, replace=False)]))
    rsel = torch.from_numpy(rows).to(dev)

    # stage 1: gate/up GEMM on sampled rows x sampled columns of each module
    a32 = p.a.float().numpy()
    s_ga = oracle.global_scale(a32)
    assert np.float32(aq.scale.item()) == s_ga
    qa, sfa = oracle.quantize(a32[rows], s_ga)
    a_hat = oracle.dequantize(qa, sfa, s_ga)
    cols, w_rows = [], []
    for i, w in enumerate(p.modules):
        w32 = w.float().numpy()
        s_w = oracle.global_scale(w32)
        pick = np.unique(np.concatenate([[0, f - 1], rng.choice(f, 30, replace=False)]))
        qw, sfw = oracle.quantize(w32[pick], s_w)
        w_rows.append(oracle.dequantize(qw, sfw, s_w))
        cols.append(i * f + pick)
    w_hat = np.concatenate(w_rows)
    csel = torch.from_numpy(np.concatenate(cols)).to(dev)
    c1_s = c1[rsel][:, csel].float()
    assert_gemm_close(c1_s, oracle.gemm(a_hat, w_hat), a_hat, w_hat, "gate/up GEMM")

    # stage 2: glue on the GPU's own gate/up output
    s_h = np.float32(hq.scale.item())
    h_amax = float(h.cpu().abs().max().item())              # exact: a max of BF16 values, on the host
    assert s_h == oracle.global_scale_from_amax(np.float32(h_amax))
    g_rows, u_rows = c1[rsel, :f].cpu(), c1[rsel, f:].cpu()
    _check_h(g_rows, u_rows, h[rsel])
    h32 = h[rsel].float().cpu().numpy()
    q_ref, sf_ref = oracle.quantize(h32, s_h)
    np.testing.assert_array_equal(to_np_u8(hq.q[rsel]), q_ref)
    np.testing.assert_array_equal(sf_rowmajor(hq.sf, m, f)[rows], sf_ref)

    # stage 3: down GEMM on sampled rows x sampled columns
    h_hat = oracle.dequantize(q_ref, sf_ref, s_h)
    w2_32 = w2.float().numpy()
    s_w2 = oracle.global_scale(w2_32)
    pick = np.unique(np.concatenate([[0, k - 1], rng.choice(k, 30, replace=False)]))
    qw2, sfw2 = oracle.quantize(w2_32[pick], s_w2)
    w2_hat = oracle.dequantize(qw2, sfw2, s_w2)
    c2_s = c2[rsel][:, torch.from_numpy(pick).to(dev)]
    assert_gemm_close(c2_s, oracle.gemm(h_hat, w2_hat), h_hat, w2_hat, "down GEMM")


FUSED_CASES = [
    # (m, f, k)
    (300, 256, 512),
    (129, 1024, 1056),
    (8192, 17408, 5120),
]


@pytest.mark.parametrize("m,f,k", FUSED_CASES)
def test_swiglu_epilogue_equals_gemm_then_glue(m, f, k):
    """nvfp4_gemm_swiglu_quantize (glue in the gate/up GEMM's epilogue, static
    h scale) must give the bytes of the BF16 gate/up GEMM followed by
    nvfp4_silu_mul_quantize with the same scale."""
    a, _ = synthetic.activations(m, k, seed=m + f + k)
    gate = synthetic.weights(f, k, 0.02, seed=3).cuda()
    up = synthetic.weights(f, k, 0.05, seed=4).cuda()
    fw = nv.quantize_weight([gate, up])
    aq = nv.quantize_act(a.cuda())
    c1 = nv.gemm(aq, fw)                                              # m x 2f BF16
    calib, _ = nv.silu_mul_quantize(c1[:, :f], c1[:, f:])              # a calibration run for h's scale
    h_scale = (calib.scale * 1.1).contiguous()
    ref, h_cuda = nv.silu_mul_quantize(c1[:, :f], c1[:, f:], h_scale=h_scale, return_h=True)
    got = nv.gemm_swiglu_quantize(aq, fw, h_scale)
    torch.cuda.synchronize()
    nv.check_device_status()
    assert torch.equal(got.q, ref.q)
    assert torch.equal(got.sf, ref.sf)

    # Against the oracle, on sampled rows of the gate/up output (itself checked
    # against the oracle's FP64 GEMM elsewhere): the unfused glue's h is within
    # one BF16 ulp of oracle.silu_mul_bf16, the fused codes and scales are the
    # oracle's quantisation of that h bit for bit, and they equal the oracle's
    # quantisation of its own h except in blocks where the two exp
    # implementations put an element of h on either side of a rounding point.
    rng = np.random.default_rng(m + f)
    rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, min(m, 64), replace=False)]))
    rsel = torch.from_numpy(rows).cuda()
    s_h = np.float32(h_scale.item())
    gemm_rows = rows[:: max(1, len(rows) // 8)]
    c1_32 = nv.gemm(aq, fw, out_dtype=torch.float32)[torch.from_numpy(gemm_rows).cuda()]
    c64, info = oracle.linear(a, [gate.cpu(), up.cpu()], rows=gemm_rows)
    assert_gemm_close(c1_32, c64, info["a_hat"], oracle.fused_weight_hat(info["qmods"]), "gate/up GEMM")
    g_rows, u_rows = c1[rsel, :f].cpu(), c1[rsel, f:].cpu()
    _check_h(g_rows, u_rows, h_cuda[rsel])
    got_q, got_sf = to_np_u8(got.q[rsel]), sf_rowmajor(got.sf, m, f)[rows]
    q_cuda, sf_cuda = oracle.quantize(h_cuda[rsel].float().cpu().numpy(), s_h)
    np.testing.assert_array_equal(got_q, q_cuda)
    np.testing.assert_array_equal(got_sf, sf_cuda)
    h_ref = oracle.bf16_bits_to_f32(oracle.silu_mul_bf16(_bits(g_rows), _bits(u_rows))).reshape(len(rows), f)
    q_ref, sf_ref = oracle.quantize(h_ref, s_h)
    block_codes_differ = (got_q.reshape(len(rows), f // 16, 8) != q_ref.reshape(len(rows), f // 16, 8)).any(axis=2)
    blocks_differ = block_codes_differ | (got_sf != sf_ref)
    assert blocks_differ.mean() <= 5e-3, f"{blocks_differ.mean():.2e} of 16-element blocks differ from the oracle's"
