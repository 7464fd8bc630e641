"""GPU parity of the calibrated FP8 KV cache ("Why Gated DeltaNet Survives
4-Bit Quantization": abstract; Glonce article, "How to use it"): the
calibration's running amax and scale, and every cache byte, bit-exact
against the oracle (both sides take the E4M3 rounding decision on the same
FP32 product x * (1/s))."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic

pytestmark = pytest.mark.gpu
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _calibrated(k, v):
    dev = "cuda"
    scales = []
    for x in (k, v):
        amax = torch.zeros(1, dtype=torch.float32, device=dev)
        scale = torch.empty(1, dtype=torch.float32, device=dev)
        nv.fp8_calibrate(x.to(dev), amax, scale)
        scales.append(scale)
    return scales


def _check_cache(k, v, ks, vs, kc, vc, slots, num_slots):
    """Rows named by a valid slot equal the oracle's bytes; the others hold the sentinel."""
    kc, vc = kc.cpu().numpy(), vc.cpu().numpy()
    sk, sv = np.float32(ks.item()), np.float32(vs.item())
    want_k = oracle.fp8_quantize(k.float().cpu().numpy(), sk)
    want_v = oracle.fp8_quantize(v.float().cpu().numpy(), sv)
    slots = np.arange(k.shape[0]) if slots is None else slots.cpu().numpy()
    written = np.zeros(num_slots, bool)
    for t, sl in enumerate(slots):
        if 0 <= sl < num_slots:
            np.testing.assert_array_equal(kc[sl, :want_k.shape[1]], want_k[t], err_msg=f"K token {t} slot {sl}")
            np.testing.assert_array_equal(vc[sl, :want_v.shape[1]], want_v[t], err_msg=f"V token {t} slot {sl}")
            written[sl] = True
    assert np.all(kc[~written] == SENTINEL) and np.all(vc[~written] == SENTINEL)
    assert np.all(kc[written, want_k.shape[1]:] == SENTINEL)           # bytes past the width untouched


def test_calibration_running_amax_and_scale():
    k1, _ = synthetic.kv_rows(100, seed=1)
    k2, _ = synthetic.kv_rows(60, seed=2, outlier_gain=20.0)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    scale = torch.empty(1, dtype=torch.float32, device="cuda")
    nv.fp8_calibrate(k1.cuda(), amax, scale)
    torch.cuda.synchronize()
    a1 = k1.float().abs().max().item()
    assert amax.item() == a1 and scale.item() == oracle.fp8_scale_from_amax(a1)
    nv.fp8_calibrate(k2.cuda(), amax, scale)
    torch.cuda.synchronize()
    a12 = max(a1, k2.float().abs().max().item())
    assert amax.item() == a12 and scale.item() == oracle.fp8_scale_from_amax(a12)
    zero = torch.zeros(1, dtype=torch.float32, device="cuda")
    nv.fp8_calibrate(torch.zeros(4, 32, dtype=torch.bfloat16, device="cuda"), zero, scale)
    torch.cuda.synchronize()
    assert zero.item() == 0.0 and scale.item() == 1.0


@pytest.mark.parametrize("tokens,width,dtype", [(37, 1024, torch.bfloat16), (5, 48, torch.float32),
                                                (1, 128, torch.bfloat16), (300, 512, torch.float32)])
def test_kv_quantize_scatter(tokens, width, dtype):
    """A shuffled slot table with padding (-1) and an out-of-range entry."""
    k, v = synthetic.kv_rows(tokens, width, seed=tokens)
    k, v = k.to(dtype), v.to(dtype)
    ks, vs = _calibrated(k, v)
    num_slots = 2 * tokens + 7
    rng = np.random.default_rng(tokens)
    slots = rng.permutation(num_slots)[:tokens].astype(np.int64)
    slots[rng.random(tokens) < 0.2] = -1
    if tokens > 2:
        slots[1] = num_slots + 3
    slots_t = torch.from_numpy(slots).cuda()
    kc = torch.full((num_slots, width + 32), SENTINEL, dtype=torch.uint8, device="cuda")
    vc = torch.full((num_slots, width + 32), SENTINEL, dtype=torch.uint8, device="cuda")
    nv.kv_cache_quantize_fp8(k.cuda(), v.cuda(), ks, vs, kc[:, :width], vc[:, :width], slots_t)
    torch.cuda.synchronize()
    _check_cache(k, v, ks, vs, kc, vc, slots_t, num_slots)


def test_kv_quantize_strided_rows_identity_slots_and_extreme_scales():
    """Strided K/V rows, no slot table, a scale that saturates K and one that
    sends V into the subnormals."""
    tokens, width = 64, 256
    base_k = (torch.randn(tokens, width + 64) * 50).to(torch.bfloat16).cuda()
    base_v = (torch.randn(tokens, width + 64) * 1e-3).to(torch.bfloat16).cuda()
    k, v = base_k[:, :width], base_v[:, :width]
    ks = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    vs = torch.tensor([1.0], dtype=torch.float32, device="cuda")
    kc = torch.full((tokens + 3, width), SENTINEL, dtype=torch.uint8, device="cuda")
    vc = torch.full((tokens + 3, width), SENTINEL, dtype=torch.uint8, device="cuda")
    nv.kv_cache_quantize_fp8(k, v, ks, vs, kc, vc)
    torch.cuda.synchronize()
    _check_cache(k.cpu(), v.cpu(), ks, vs, kc, vc, None, tokens + 3)
    kb = kc[:tokens].cpu().numpy()
    assert np.mean((kb & 0x7F) == 0x7E) > 0.5                         # saturated
    assert np.any((vc[:tokens].cpu().numpy() & 0x78) == 0)             # subnormal bytes


def test_kv_prefill_8192_tokens():
    """An 8192-token prefill of one layer (4 KV heads x 256), every byte."""
    k, v = synthetic.kv_rows(8192)
    ks, vs = _calibrated(k, v)
    slots = torch.randperm(8192 + 512, generator=torch.Generator().manual_seed(3))[:8192].to(torch.int64).cuda()
    kc = torch.full((8192 + 512, k.shape[1]), SENTINEL, dtype=torch.uint8, device="cuda")
    vc = torch.full((8192 + 512, k.shape[1]), SENTINEL, dtype=torch.uint8, device="cuda")
    nv.kv_cache_quantize_fp8(k.cuda(), v.cuda(), ks, vs, kc, vc, slots)
    torch.cuda.synchronize()
    _check_cache(k, v, ks, vs, kc, vc, slots, 8192 + 512)
