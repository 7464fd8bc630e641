"""GPU parity of the quantisers: packed nibbles and tiled scale bytes must equal
the oracle's bit for bit ("Why Gated DeltaNet Survives 4-Bit Quantization",
page summary "Background" item 1: E2M1 values, E4M3 block scale = blockmax/6,
FP32 per-tensor scale)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import sf_rowmajor, to_np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


SHAPES = [(1, 32), (3, 64), (64, 256), (127, 288), (129, 5120), (300, 320), (1000, 1056)]


def _check_act(a: torch.Tensor, out: nv.QuantizedActivation, s_used: np.float32):
    a32 = a.float().numpy()
    m, k = a32.shape
    q_ref, sf_ref = oracle.quantize(a32, s_used)
    np.testing.assert_array_equal(to_np_u8(out.q), q_ref)
    tiled_ref = oracle.sf_to_tiled(sf_ref, k)
    got = to_np_u8(out.sf)
    assert got.size == tiled_ref.size
    np.testing.assert_array_equal(got, tiled_ref)      # includes the zero padding


@pytest.mark.parametrize("m,k", SHAPES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_act_dynamic_bit_exact(m, k, dtype):
    a, _ = synthetic.activations(m, k, seed=m * 7 + k, n_outliers=max(1, k // 1000), dtype=dtype)
    out = nv.quantize_act(a.cuda())
    torch.cuda.synchronize()
    s = np.float32(out.scale.item())
    assert s == oracle.global_scale(a.float().numpy())
    _check_act(a, out, s)


@pytest.mark.parametrize("m,k", SHAPES[:5])
def test_quantize_act_static_bit_exact(m, k):
    a, _ = synthetic.activations(m, k, seed=11 + m, dtype=torch.bfloat16)
    # a calibrated scale with headroom (static mode, the pages' calibration-only PTQ)
    s = np.float32(oracle.global_scale(a.float().numpy()) * np.float32(1.7))
    scale = torch.tensor([s], dtype=torch.float32, device="cuda")
    out = nv.quantize_act(a.cuda(), act_scale=scale)
    torch.cuda.synchronize()
    assert np.float32(out.scale.item()) == s
    _check_act(a, out, s)


def _edge_blocks():
    """FP32 rows of 16-element blocks that hit every rounding decision."""
    ties = [6.0, -3.0, 1.0, 0.3, 0.25, 0.75, -1.25, 1.75, 2.5, 3.5, 5.0, 5.5, -0.1, 0.0, 4.25, -6.0]
    neg_zero = [-0.0] * 15 + [6.0]
    zeros = [0.0] * 16
    tiny_max = [0.005, -0.001] + [0.0] * 14                      # block scale underflows to 0
    denorm = [1e-40, -2e-40, 3e-39] + [0.0] * 13
    near_mid = [6.0] + [np.nextafter(np.float32(v), np.float32(d)) for v, d in
                         [(0.25, 1), (0.25, 0), (0.75, 0), (0.75, 1), (2.5, 1), (2.5, 0), (5.0, 0), (5.0, 1),
                          (1.25, 1), (1.75, 0), (3.5, 0), (3.5, 1), (0.5, 1), (1.5, 0), (4.0, 1)]]
    big = [6.0e4, -3.0e4] + [1.0] * 14
    rows = [ties, neg_zero, zeros, tiny_max, denorm, near_mid, big, [-v for v in ties]]
    return np.array([sum(rows[i:i + 2], []) for i in range(0, len(rows), 2)], np.float32)  # 4 x 32


@pytest.mark.parametrize("s_g", [1.0, 1e-3, 0.37, 2.0 ** -20, 7.5e3])
def test_quantize_edge_blocks_bit_exact(s_g):
    """Ties to even, signed zeros, all-zero and underflowing blocks, E4M3
    saturation (a static scale far too small), denormal inputs."""
    x = np.tile(_edge_blocks(), (1, 1))
    a = torch.from_numpy(x)
    scale = torch.tensor([s_g], dtype=torch.float32, device="cuda")
    out = nv.quantize_act(a.cuda(), act_scale=scale)
    torch.cuda.synchronize()
    _check_act(a, out, np.float32(s_g))


def test_quantize_act_strided_rows():
    base, _ = synthetic.activations(40, 512, seed=5)
    a = base.cuda()[:, :256]                                      # lda = 512 > k
    out = nv.quantize_act(a)
    torch.cuda.synchronize()
    s = np.float32(out.scale.item())
    _check_act(base[:, :256].contiguous(), out, s)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_weight_fused_modules_bit_exact(dtype):
    k = 320
    widths, stds = (48, 128, 80, 16), (0.02, 0.02, 0.2, 0.05)
    mods = [synthetic.weights(n, k, s, seed=1 + i, dtype=dtype) for i, (n, s) in enumerate(zip(widths, stds))]
    fw = nv.quantize_weight([w.cuda() for w in mods])
    torch.cuda.synchronize()
    q_all, sf_all, off = [], [], 0
    for (b, e, s), w in zip(fw.segments, mods):
        w32 = w.float().numpy()
        assert np.float32(s) == oracle.global_scale(w32)
        q_ref, sf_ref = oracle.quantize(w32, np.float32(s))
        np.testing.assert_array_equal(to_np_u8(fw.q)[b:e], q_ref)
        np.testing.assert_array_equal(sf_rowmajor(fw.sf, e - b, k, b), sf_ref)
        q_all.append(q_ref)
        sf_all.append(sf_ref)
    np.testing.assert_array_equal(to_np_u8(fw.sf), oracle.sf_to_tiled(np.concatenate(sf_all), k))


def test_quantize_weight_given_scale():
    w = synthetic.weights(96, 256, 0.02, seed=3)
    s = float(np.float32(0.0001234))
    fw = nv.quantize_weight([w.cuda()], global_scales=[s])
    torch.cuda.synchronize()
    assert fw.segments[0][2] == np.float32(s)
    q_ref, sf_ref = oracle.quantize(w.float().numpy(), np.float32(s))
    np.testing.assert_array_equal(to_np_u8(fw.q), q_ref)
    np.testing.assert_array_equal(to_np_u8(fw.sf), oracle.sf_to_tiled(sf_ref, 256))


def test_quantize_full_size_prefill_activation_bit_exact():
    """The 8192 x 5120 activation of the fused in-projection, in full."""
    p = synthetic.gdn_in_proj(m=8192, widths=(16,), stds=(0.02,))
    out = nv.quantize_act(p.a.cuda())
    torch.cuda.synchronize()
    s = np.float32(out.scale.item())
    assert s == oracle.global_scale(p.a.float().numpy())
    _check_act(p.a, out, s)


def test_quantize_is_deterministic():
    a, _ = synthetic.activations(513, 2048, seed=9)
    a = a.cuda()
    o1 = nv.quantize_act(a)
    o2 = nv.quantize_act(a)
    torch.cuda.synchronize()
    assert torch.equal(o1.q, o2.q) and torch.equal(o1.sf, o2.sf) and torch.equal(o1.scale, o2.scale)


def test_bounded_wait_reports_timeout():
    """A wait that nothing ends runs out after its limit and is reported; the
    context stays usable."""
    L = nv.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    nv.check_device_status()
    assert L.nvfp4_selftest_wait_timeout(2_000_000, stream) == 0
    with pytest.raises(nv.NVFP4Error) as e:
        nv.check_device_status()
    assert e.value.status == 5
    nv.check_device_status()                                       # cleared
    x = torch.ones(4, device="cuda")
    assert x.sum().item() == 4.0
