"""Decode GEMMs launched back to back with programmatic dependent launch.

A decode GEMM may start (and stream weights) while the previous kernel in the
stream is still running; it must not read activations or scales, or write
its output or the shared workspace, before that kernel has completed.  These
tests enqueue chains with no host synchronisation in between and compare every
result bit for bit with the same call made alone (each single call is itself
checked against the oracle in test_gpu_gemm.py):

* several decode GEMMs sharing one workspace and writing one output buffer in
  turn (a write-after-write and write-after-read chain on C and the partial
  tiles), each result copied out by the next kernel in the stream;
* a layer chain in which each GEMM's activations come from the previous GEMM's
  output through nvfp4_quantize_act (a read-after-write chain)."""
import pytest
import torch

import nvfp4_w4a4_quantized_07_b200 as nv
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic

pytestmark = pytest.mark.gpu
DECODE = nv.NVFP4_GEMM_FORCE_DECODE


@pytest.fixture(scope="module", autouse=True)
def _built():
    nvbuild.build()
    nv.load()


def _weights(widths, k, seed):
    return nv.quantize_weight([synthetic.weights(n, k, 0.02, seed=seed + i).cuda() for i, n in enumerate(widths)])


@pytest.mark.parametrize("m", [1, 16, 64])
def test_back_to_back_decode_gemms_share_output_and_workspace(m):
    k = 2048
    fws = [_weights((1024,), k, 10), _weights((512, 512, 256), k, 20), _weights((1536,), k, 30),
           _weights((256, 768), k, 40)]
    n_max = max(f.n for f in fws)
    a, _ = synthetic.activations(m, k, seed=m)
    aq = nv.quantize_act(a.cuda())
    ws = torch.empty(nv.load().nvfp4_gemm_workspace_size(m, n_max, k, DECODE), dtype=torch.uint8, device="cuda")
    # reference: each call alone, synchronised
    refs = []
    for f in fws:
        c = torch.empty((m, f.n), dtype=torch.float32, device="cuda")
        nv.gemm(aq, f, out=c, out_dtype=torch.float32, flags=DECODE, workspace=ws)
        torch.cuda.synchronize()
        refs.append(c.clone())
    # chain: the same calls three times over, one shared output buffer, each
    # result copied away by the next operation in the stream
    shared = torch.empty((m, n_max), dtype=torch.float32, device="cuda")
    got = []
    torch.cuda._sleep(2_000_000)          # let the host enqueue the whole chain
    for rep in range(3):
        for f in fws:
            nv.gemm(aq, f, out=shared[:, :f.n], out_dtype=torch.float32, flags=DECODE, workspace=ws)
            got.append(shared[:, :f.n].clone())
    torch.cuda.synchronize()
    nv.check_device_status()
    for i, g in enumerate(got):
        assert torch.equal(g, refs[i % len(fws)]), f"chained call {i} differs from the call made alone"


def test_layer_chain_through_quantize_act():
    """C of one decode GEMM, requantised, is the next GEMM's input."""
    m, k = 16, 1024
    fws = [_weights((k,), k, 50 + 10 * i) for i in range(4)]
    a, _ = synthetic.activations(m, k, seed=7)
    a = a.cuda()
    scale = torch.tensor([0.01], dtype=torch.float32, device="cuda")

    def run(sync):
        x = a
        outs = []
        for f in fws:
            q = nv.quantize_act(x, act_scale=scale)
            x = nv.gemm(q, f, out_dtype=torch.bfloat16, flags=DECODE)
            outs.append(x)
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [o.clone() for o in outs]

    ref = run(True)
    torch.cuda._sleep(2_000_000)
    got = run(False)
    nv.check_device_status()
    for i, (g, r) in enumerate(zip(got, ref)):
        assert torch.equal(g, r), f"layer {i}"


@pytest.mark.parametrize("m,n,k", [(16, 512, 17408), (64, 256, 17408), (64, 256, 40960), (5, 768, 40960)])
def test_decode_tiles_split_over_many_ctas(m, n, k):
    """Few output tiles and a long K: every tile's k-tiles are spread over
    dozens of CTAs (up to one per SM), so each participant sums a slice of
    one or no column groups and, at 64 tokens, the reduction gathers the
    partials in several chunks.  Checked against the oracle's FP64 GEMM."""
    import oracle
    from helpers import assert_gemm_close
    a, _ = synthetic.activations(m, k, seed=m + n)
    w = synthetic.weights(n, k, 0.02, seed=n)
    fw = nv.quantize_weight([w.cuda()])
    aq = nv.quantize_act(a.cuda())
    c = nv.gemm(aq, fw, out_dtype=torch.float32, flags=DECODE)
    torch.cuda.synchronize()
    nv.check_device_status()
    c64, info = oracle.linear(a, [w])
    assert_gemm_close(c, c64, info["a_hat"], oracle.fused_weight_hat(info["qmods"]), f"m={m} n={n} k={k}")
