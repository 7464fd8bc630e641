"""GPU parity of the block-scaled FP4 GEMM and its per-module scale epilogue
against the oracle's FP64 GEMM over dequantised operands.

Tolerance (stated for the GEMM output before the BF16 cast): per element
|C - C64| <= 1e-3 * |A_hat row| * |W_hat row| and relative Frobenius error
<= 2e-3.  The fused-segment GEMM must equal the per-module GEMMs within the
same tolerance, and a single-shared-scale GEMM must fail it ("Why Gated
DeltaNet Survives 4-Bit Quantization": abstract, last sentence; news article,
"Risks and caveats")."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import (act_from_codes, assert_gemm_close, dequant_codes, gemm_check, to_np_u8,
                     weight_from_codes)

pytestmark = pytest.mark.gpu
LARGE, DECODE, AUTO = nv.NVFP4_GEMM_FORCE_LARGE, nv.NVFP4_GEMM_FORCE_DECODE, nv.NVFP4_GEMM_AUTO
PAIR = nv.NVFP4_GEMM_FORCE_LARGE_PAIR


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _w_hat_segments(codes, sf, segments):
    parts = [dequant_codes(codes[b:e], sf[b:e], np.float32(s)) for b, e, s in segments]
    return np.concatenate(parts, axis=0)


# --------------------------------------------------------------------------- constructed operands
@pytest.mark.parametrize("kind", ["unit_scales", "row_scales", "kblock_scales", "random"])
@pytest.mark.parametrize("flags", [LARGE, DECODE, PAIR])
def test_gemm_constructed_operands(kind, flags):
    """Operands built directly from codes and scale bytes isolate the data path
    (unit scales), the scale row mapping and the scale K mapping."""
    rng = np.random.default_rng({"unit_scales": 1, "row_scales": 2, "kblock_scales": 3, "random": 4}[kind])
    m = 48 if flags == DECODE else 300
    n, k = 384, 512
    ca = rng.integers(0, 16, (m, k)).astype(np.uint8)
    cw = rng.integers(0, 16, (n, k)).astype(np.uint8)
    if kind == "unit_scales":
        sa = np.full((m, k // 16), 0x38, np.uint8)
        sw = np.full((n, k // 16), 0x38, np.uint8)
    elif kind == "row_scales":
        sa = np.repeat((0x30 + np.arange(m) % 16).astype(np.uint8)[:, None], k // 16, 1)
        sw = np.repeat((0x28 + np.arange(n) % 24).astype(np.uint8)[:, None], k // 16, 1)
    elif kind == "kblock_scales":
        sa = np.repeat((0x30 + np.arange(k // 16) % 16).astype(np.uint8)[None, :], m, 0)
        sw = np.repeat((0x34 + np.arange(k // 16) % 9).astype(np.uint8)[None, :], n, 0)
    else:
        sa = rng.integers(0x20, 0x50, (m, k // 16)).astype(np.uint8)
        sw = rng.integers(0x20, 0x50, (n, k // 16)).astype(np.uint8)
    s_ga = np.float32(0.5)
    segments = [(0, 128, 1.0), (128, 336, 0.25), (336, 384, 2.0)]
    a = act_from_codes(ca, sa, s_ga)
    w = weight_from_codes(cw, sw, segments)
    c = nv.gemm(a, w, out_dtype=torch.float32, flags=flags)
    torch.cuda.synchronize()
    a_hat = dequant_codes(ca, sa, s_ga)
    w_hat = _w_hat_segments(cw, sw, segments)
    c64 = oracle.gemm(a_hat, w_hat)
    if kind == "unit_scales":
        # small dyadic values: the FP32 accumulation is exact
        np.testing.assert_array_equal(c.double().cpu().numpy(), c64)
    assert_gemm_close(c, c64, a_hat, w_hat, kind)


# --------------------------------------------------------------------------- the oracle end to end
def _run_linear(p, flags, out_dtype=torch.float32, act_scale=None):
    fw = nv.quantize_weight([w.cuda() for w in p.modules])
    aq = nv.quantize_act(p.a.cuda(), act_scale=act_scale)
    c = nv.gemm(aq, fw, out_dtype=out_dtype, flags=flags)
    torch.cuda.synchronize()
    return c, aq, fw


def _oracle_linear(p, rows=None):
    c64, info = oracle.linear(p.a, p.modules, rows=rows)
    return c64, info["a_hat"], oracle.fused_weight_hat(info["qmods"])


@pytest.mark.parametrize("flags", [AUTO, LARGE, PAIR])
def test_config_tiny_fp32_and_bf16(flags):
    """64x256 FP32 activations with one x50 column against a 128x256 FP32 weight."""
    p = synthetic.tiny()
    c32, aq, fw = _run_linear(p, flags, torch.float32)
    c16 = nv.gemm(aq, fw, out_dtype=torch.bfloat16, flags=flags)
    torch.cuda.synchronize()
    c64, a_hat, w_hat = _oracle_linear(p)
    assert_gemm_close(c32, c64, a_hat, w_hat, "tiny")
    # BF16 output = round-to-nearest-even of the same call's FP32 output
    assert torch.equal(c16.cpu(), c32.cpu().to(torch.bfloat16))


RAGGED = [
    # (m, widths, k)
    (1, (16,), 64),
    (3, (48, 208, 32, 112), 96),
    (16, (400,), 288),
    (64, (2048, 48, 48), 256),
    (127, (48, 208, 32, 112), 320),
    (128, (256,), 512),
    (129, (48, 208, 32, 112), 512),
    (300, (96, 400, 16), 1056),
]


@pytest.mark.parametrize("m,widths,k", RAGGED)
@pytest.mark.parametrize("flags", [AUTO, LARGE, PAIR])
def test_gemm_ragged_shapes_and_mid_tile_segments(m, widths, k, flags):
    a, _ = synthetic.activations(m, k, seed=m + k)
    stds = [0.02 if i % 2 == 0 else 0.2 for i in range(len(widths))]
    mods = [synthetic.weights(n, k, s, seed=1 + i) for i, (n, s) in enumerate(zip(widths, stds))]
    p = synthetic.LinearProblem("ragged", a, mods)
    c, _, _ = _run_linear(p, flags)
    c64, a_hat, w_hat = _oracle_linear(p)
    assert_gemm_close(c, c64, a_hat, w_hat, f"m={m} widths={widths} k={k}")


def test_fused_segments_equal_unfused_modules_and_shared_scale_fails():
    """The pages' fix: the fused GEMM equals the six per-module GEMMs; applying
    one shared global scale (module 0's, or the largest) fails the check."""
    p = synthetic.gdn_in_proj(m=256, k=512)
    c, aq, fw = _run_linear(p, LARGE)
    c64, a_hat, w_hat = _oracle_linear(p)
    assert_gemm_close(c, c64, a_hat, w_hat, "fused")
    # per-module GEMMs (each its own 1-segment call on its own quantised module)
    parts = []
    for w in p.modules:
        fwi = nv.quantize_weight([w.cuda()])
        parts.append(nv.gemm(aq, fwi, out_dtype=torch.float32, flags=LARGE))
    unfused = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    assert_gemm_close(unfused, c64, a_hat, w_hat, "unfused")
    assert_gemm_close(c, unfused.double().cpu().numpy(), a_hat, w_hat, "fused vs unfused")
    scales = [s for _, _, s in fw.segments]
    for shared in (scales[0], max(scales)):
        bad = nv.gemm(aq, fw, out_dtype=torch.float32, flags=LARGE, segments=[(0, fw.n, shared)])
        torch.cuda.synchronize()
        ratio, fro = gemm_check(bad, c64, a_hat, w_hat)
        assert ratio > 1.0 and fro > 2e-3, (shared, ratio, fro)


@pytest.mark.parametrize("flags", [LARGE, DECODE, PAIR])
def test_gemm_is_deterministic(flags):
    m = 40 if flags == DECODE else 300
    p = synthetic.gdn_in_proj(m=m, k=1024, widths=(512, 48, 48, 1024), stds=(0.02, 0.2, 0.2, 0.02))
    c1, aq, fw = _run_linear(p, flags, torch.bfloat16)
    c2 = nv.gemm(aq, fw, out_dtype=torch.bfloat16, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)


def test_output_leading_dimension_and_bf16_consistency():
    p = synthetic.gdn_in_proj(m=200, k=256, widths=(128, 48, 80), stds=(0.02, 0.2, 0.02))
    fw = nv.quantize_weight([w.cuda() for w in p.modules])
    aq = nv.quantize_act(p.a.cuda())
    big = torch.full((200, 512), 7.0, dtype=torch.float32, device="cuda")
    nv.gemm(aq, fw, out_dtype=torch.float32, out=big[:, :256], flags=LARGE)
    c16 = nv.gemm(aq, fw, out_dtype=torch.bfloat16, flags=LARGE)
    torch.cuda.synchronize()
    assert torch.all(big[:, 256:] == 7.0)                       # columns past n untouched
    assert torch.equal(c16.cpu(), big[:, :256].cpu().to(torch.bfloat16))
    c64, a_hat, w_hat = _oracle_linear(p)
    assert_gemm_close(big[:, :256], c64, a_hat, w_hat)


# --------------------------------------------------------------------------- full-size configurations
def _sample_rows(m, count, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, m - 129, m - 1]
    rows = np.unique(np.concatenate([np.array([r for r in fixed if 0 <= r < m]),
                                     rng.choice(m, size=min(count, m), replace=False)]))
    return rows


def test_config_prefill_4096x5120x5120_sampled_rows():
    p = synthetic.prefill()
    c, aq, fw = _run_linear(p, AUTO, torch.bfloat16)
    rows = _sample_rows(p.m, 48)
    c64, a_hat, w_hat = _oracle_linear(p, rows=rows)
    # quantised operands bit-exact in full
    a32 = p.a.float().numpy()
    s_ga = np.float32(aq.scale.item())
    q_ref, _ = oracle.quantize(a32, s_ga)
    np.testing.assert_array_equal(to_np_u8(aq.q), q_ref)
    c32 = nv.gemm(aq, fw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_gemm_close(c32[torch.from_numpy(rows).cuda()], c64, a_hat, w_hat, "prefill")
    assert torch.equal(c.cpu(), c32.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("flags", [AUTO, LARGE, PAIR])
def test_config_fused_gdn_in_proj_8192_sampled_rows(flags):
    """8192 x 5120 activations against six separately calibrated modules
    [2048, 2048, 4096, 4096, 48, 48] (N = 12384), checked against the oracle
    and the six unfused GEMMs on sampled rows; one shared global scale
    (module 0's, or the largest) must fail the same check at this size."""
    p = synthetic.gdn_in_proj()
    c32, aq, fw = _run_linear(p, flags, torch.float32)
    rows = _sample_rows(p.m, 32)
    c64, a_hat, w_hat = _oracle_linear(p, rows=rows)
    rsel = torch.from_numpy(rows).cuda()
    assert_gemm_close(c32[rsel], c64, a_hat, w_hat, "gdn in-proj")
    parts = [nv.gemm(aq, nv.quantize_weight([w.cuda()]), out_dtype=torch.float32, flags=flags)[rsel]
             for w in p.modules]
    torch.cuda.synchronize()
    unfused = torch.cat(parts, dim=1)
    assert_gemm_close(c32[rsel], unfused.double().cpu().numpy(), a_hat, w_hat, "fused vs unfused")
    scales = [s for _, _, s in fw.segments]
    for shared in (scales[0], max(scales)):
        bad = nv.gemm(aq, fw, out_dtype=torch.float32, flags=flags, segments=[(0, fw.n, shared)])[rsel]
        torch.cuda.synchronize()
        ratio, fro = gemm_check(bad, c64, a_hat, w_hat)
        assert ratio > 1.0 and fro > 2e-3, (shared, ratio, fro)


def test_config_mlp_gate_up_fused_equals_unfused_and_shared_scale_fails():
    """The long-prefill MLP's fused gate/up GEMM (32768 x 5120 against two
    separately calibrated 17408-row modules, N = 34816) against the oracle and
    its two unfused GEMMs on sampled rows; one shared global scale (either
    module's) must fail the same check."""
    p = synthetic.mlp_gate_up()
    c32, aq, fw = _run_linear(p, AUTO, torch.float32)
    rows = _sample_rows(p.m, 6)
    c64, a_hat, w_hat = _oracle_linear(p, rows=rows)
    rsel = torch.from_numpy(rows).cuda()
    assert_gemm_close(c32[rsel], c64, a_hat, w_hat, "mlp gate/up")
    parts = [nv.gemm(aq, nv.quantize_weight([w.cuda()]), out_dtype=torch.float32)[rsel] for w in p.modules]
    torch.cuda.synchronize()
    unfused = torch.cat(parts, dim=1)
    assert_gemm_close(c32[rsel], unfused.double().cpu().numpy(), a_hat, w_hat, "fused vs unfused")
    # Both modules are N(0, 0.02): their scales differ by only ~0.4 %, so a
    # shared scale stays inside the per-element bound and fails on the
    # Frobenius error alone (about 3e-3 against 2e-3).
    scales = [s for _, _, s in fw.segments]
    assert len(scales) == 2 and scales[0] != scales[1]
    for shared in scales:
        bad = nv.gemm(aq, fw, out_dtype=torch.float32, segments=[(0, fw.n, shared)])[rsel]
        torch.cuda.synchronize()
        ratio, fro = gemm_check(bad, c64, a_hat, w_hat)
        assert not (ratio <= 1.0 and fro <= 2e-3), (shared, ratio, fro)


@pytest.mark.parametrize("shape", list(synthetic.DECODE_SHAPES))
@pytest.mark.parametrize("m", synthetic.DECODE_M)
def test_config_decode_sweep(m, shape):
    p = synthetic.decode(m, shape)
    c, aq, fw = _run_linear(p, AUTO, torch.float32)
    # oracle on a sample of output columns (weight rows) of every module
    rng = np.random.default_rng(m)
    a32 = p.a.float().numpy()
    s_ga = oracle.global_scale(a32)
    qa, sfa = oracle.quantize(a32, s_ga)
    a_hat = oracle.dequantize(qa, sfa, s_ga)
    cols, w_rows = [], []
    off = 0
    for w in p.modules:
        w32 = w.float().numpy()
        s_w = oracle.global_scale(w32)
        pick = np.unique(np.concatenate([[0, w32.shape[0] - 1], rng.choice(w32.shape[0], 24, replace=False)]))
        qw, sfw = oracle.quantize(w32[pick], s_w)
        w_rows.append(oracle.dequantize(qw, sfw, s_w))
        cols.append(off + pick)
        off += w32.shape[0]
    w_hat = np.concatenate(w_rows)
    cols = np.concatenate(cols)
    c64 = oracle.gemm(a_hat, w_hat)
    assert_gemm_close(c[:, torch.from_numpy(cols).cuda()], c64, a_hat, w_hat, f"decode m={m} {shape}")
