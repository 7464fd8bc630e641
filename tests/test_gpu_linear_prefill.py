"""nvfp4_linear_prefill: the static-scale activation quantisation fused into
the large-M GEMM (one launch).  Its quantised activations must equal
nvfp4_quantize_act's bytes and its output nvfp4_gemm's (single-CTA kernel)
bit for bit -- the fused kernel only moves where and when A is quantised and
the order in which tiles run, not the arithmetic of any element -- and one
case is checked against the oracle directly.  Shapes cover ragged rows, K and
segments, several bands of the banded tile order, a first phase that covers
every m-block (few tiles) and one that does not (many tiles)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import assert_gemm_close, to_np_u8

pytestmark = pytest.mark.gpu
LARGE = nv.NVFP4_GEMM_FORCE_LARGE


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _problem(m, widths, k, seed):
    a, _ = synthetic.activations(m, k, seed=seed)
    mods = [synthetic.weights(n, k, 0.02 * (1 + i), seed=seed + 1 + i) for i, n in enumerate(widths)]
    return a, mods


def _compare(a, mods, out_dtype):
    a_dev = a.cuda()
    fw = nv.quantize_weight([w.cuda() for w in mods])
    scale = nv.quantize_act(a_dev).scale.clone()          # calibration run: the static scale
    ref_q = nv.quantize_act(a_dev, act_scale=scale)
    ref_c = nv.gemm(ref_q, fw, out_dtype=out_dtype, flags=LARGE)
    c, aq = nv.linear_prefill(a_dev, fw, scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    nv.check_device_status()
    assert torch.equal(aq.q, ref_q.q), "codes differ from nvfp4_quantize_act"
    assert torch.equal(aq.sf, ref_q.sf), "scales differ from nvfp4_quantize_act"
    assert torch.equal(c, ref_c), "output differs from nvfp4_gemm"
    return c, aq, fw, scale


@pytest.mark.parametrize("m,widths,k", [
    (65, (256,), 256),                         # one partial m-block
    (129, (48, 208, 32, 112), 96),             # ragged K (one partial k-tile), four segments
    (300, (400,), 1056),
    (1300, (2048, 48, 48), 512),               # 11 m-blocks: two bands
    (4100, (256,), 320),                       # 33 m-blocks, 33 tiles: every m-block before the mainloop
    (3000, (4096, 4096), 1024),                # 24 m-blocks x 32 n-blocks: most m-blocks while the MMAs run
])
def test_fused_equals_two_launches(m, widths, k):
    _compare(*_problem(m, widths, k, seed=m + k), torch.bfloat16)


def test_fused_fp32_output_and_oracle():
    a, mods = _problem(300, (48, 208, 32, 112), 512, seed=5)
    c, aq, fw, scale = _compare(a, mods, torch.float32)
    c64, info = oracle.linear(a, mods, act_scale=float(scale.item()))
    np.testing.assert_array_equal(to_np_u8(aq.q), info["qa"])
    assert_gemm_close(c, c64, info["a_hat"], oracle.fused_weight_hat(info["qmods"]), "linear_prefill")


def test_config_gdn_in_proj_8192_fused():
    """The fused GDN-style in-proj (8192 x 5120 against six modules)."""
    p = synthetic.gdn_in_proj()
    _compare(p.a, p.modules, torch.bfloat16)


def test_back_to_back_calls_share_the_workspace():
    """Consecutive calls on one stream reuse the ready words (tagged per call)
    with different shapes; each result equals the call made alone."""
    probs = [_problem(m, (n,), 512, seed=i) for i, (m, n) in enumerate([(1000, 512), (257, 1024), (2048, 256)])]
    devs = []
    for a, mods in probs:
        a_dev = a.cuda()
        fw = nv.quantize_weight([w.cuda() for w in mods])
        scale = nv.quantize_act(a_dev).scale.clone()
        devs.append((a_dev, fw, scale))
    refs = []
    for a_dev, fw, scale in devs:
        c, _ = nv.linear_prefill(a_dev, fw, scale)
        torch.cuda.synchronize()
        refs.append(c.clone())
    outs = []
    torch.cuda._sleep(2_000_000)
    for rep in range(3):
        for a_dev, fw, scale in devs:
            outs.append(nv.linear_prefill(a_dev, fw, scale)[0])
    torch.cuda.synchronize()
    nv.check_device_status()
    for i, o in enumerate(outs):
        assert torch.equal(o, refs[i % len(refs)]), f"call {i}"
