"""GPU parity of the fused decode layer (``nvfp4_linear_decode``): the
activation quantisation runs inside the decode GEMM, so its output must equal,
bit for bit, ``nvfp4_quantize_act`` followed by ``nvfp4_gemm`` with
NVFP4_GEMM_FORCE_DECODE (same block arithmetic, same accumulation order), and
its dynamic scale must equal the oracle's amax/2688 ("Why Gated DeltaNet
Survives 4-Bit Quantization": W4A4 with on-the-fly activation quantisation,
abstract).  One full decode shape is also checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import assert_gemm_close

pytestmark = pytest.mark.gpu
DECODE = nv.NVFP4_GEMM_FORCE_DECODE


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _weights(widths, k, seed):
    mods = [synthetic.weights(n_i, k, 0.02 * (1 + 4 * (i % 2)), seed=seed + i).cuda() for i, n_i in enumerate(widths)]
    return nv.quantize_weight(mods)


CASES = [
    # (m, widths, k)
    (1, (256,), 256),
    (5, (48, 208, 32, 112), 288),
    (16, (1024, 512), 1024),
    (17, (400,), 320),
    (33, (256, 256), 2048),
    (64, (2048, 48, 48), 1056),
]


@pytest.mark.parametrize("m,widths,k", CASES)
@pytest.mark.parametrize("mode", ["static", "dynamic"])
@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
def test_linear_decode_equals_quantize_then_gemm(m, widths, k, mode, in_dtype):
    a, _ = synthetic.activations(m, k, seed=m * 31 + k, n_outliers=max(1, k // 1000), dtype=in_dtype)
    a = a.cuda()
    fw = _weights(widths, k, seed=11)
    scale = None
    if mode == "static":
        scale = torch.tensor([oracle.global_scale(a.float().cpu().numpy()) * np.float32(1.25)],
                             dtype=torch.float32, device="cuda")
    ref_q = nv.quantize_act(a, act_scale=scale)
    ref = nv.gemm(ref_q, fw, out_dtype=torch.float32, flags=DECODE)
    s_out = torch.zeros(1, dtype=torch.float32, device="cuda")
    got = nv.linear_decode(a, fw, act_scale=scale, out_dtype=torch.float32, scale_out=s_out)
    got16 = nv.linear_decode(a, fw, act_scale=scale)
    torch.cuda.synchronize()
    nv.check_device_status()
    assert torch.equal(got, ref)
    assert torch.equal(got16, ref.to(torch.bfloat16))
    assert torch.equal(s_out, ref_q.scale)
    if mode == "dynamic":
        assert np.float32(s_out.item()) == oracle.global_scale(a.float().cpu().numpy())


def test_linear_decode_shape_against_oracle():
    """16 tokens x the 12384 x 5120 six-module weight, sampled output columns."""
    p = synthetic.decode(16, "12384x5120")
    fw = nv.quantize_weight([w.cuda() for w in p.modules])
    c = nv.linear_decode(p.a.cuda(), fw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    a32 = p.a.float().numpy()
    s_ga = oracle.global_scale(a32)
    qa, sfa = oracle.quantize(a32, s_ga)
    a_hat = oracle.dequantize(qa, sfa, s_ga)
    cols, w_rows, off = [], [], 0
    for w in p.modules:
        w32 = w.float().numpy()
        s_w = oracle.global_scale(w32)
        pick = np.unique(np.concatenate([[0, w32.shape[0] - 1], rng.choice(w32.shape[0], 12, replace=False)]))
        qw, sfw = oracle.quantize(w32[pick], s_w)
        w_rows.append(oracle.dequantize(qw, sfw, s_w))
        cols.append(off + pick)
        off += w32.shape[0]
    w_hat = np.concatenate(w_rows)
    sel = torch.from_numpy(np.concatenate(cols)).cuda()
    assert_gemm_close(c[:, sel], oracle.gemm(a_hat, w_hat), a_hat, w_hat, "linear_decode 16 x 12384x5120")
