"""The C boundary used from C: tests/c_host/linear_layer.c includes
include/nvfp4.h, links libnvfp4.so and the CUDA driver (no PyTorch, no
Python), and runs the single prefill projection (4096 x 5120 BF16 activations
with 0.1% x100 outlier channels, 5120 x 5120 weight from N(0, 0.02)) through
nvfp4_quantize_weight, nvfp4_quantize_act and nvfp4_gemm, plus invalid calls
that must be rejected with their documented status.  Its outputs are checked
here against the oracle: packed codes and scale bytes bit for bit, the GEMM on
sampled rows within the GEMM tolerance, the BF16 output as the rounding of the
FP32 output."""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_07_b200 import build as nvbuild
from nvfp4_w4a4_quantized_07_b200 import synthetic
from helpers import assert_gemm_close

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "c_host", "linear_layer.c")


def cuda_root() -> str:
    return os.path.dirname(os.path.dirname(nvbuild.nvcc()))


def compile_host_program(out_dir: str) -> str:
    """gcc, C11, warnings as errors: the header must be plain C."""
    lib = nvbuild.build()
    exe = os.path.join(out_dir, "linear_layer")
    cuda = cuda_root()
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I" + os.path.join(nvbuild.ROOT, "include"),
           "-I" + os.path.join(cuda, "include"), SOURCE, "-o", exe, "-L" + os.path.dirname(lib), "-lnvfp4",
           "-Wl,-rpath," + os.path.dirname(lib), "-L" + os.path.join(cuda, "lib64", "stubs"), "-lcuda"]
    subprocess.run(cmd, check=True)
    return exe


def test_host_program_compiles_against_the_header():
    """Runs without a GPU: the program compiles and links (driver stub)."""
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        assert os.path.exists(compile_host_program(d))


@pytest.mark.gpu
def test_prefill_layer_from_c_matches_the_oracle(tmp_path):
    exe = compile_host_program(str(tmp_path))
    p = synthetic.prefill()
    m, k, n = p.m, p.k, p.n
    p.a.contiguous().view(torch.int16).numpy().tofile(tmp_path / "a.bf16")
    p.modules[0].contiguous().view(torch.int16).numpy().tofile(tmp_path / "w.bf16")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES=os.environ.get("CUDA_VISIBLE_DEVICES", "0"))
    run = subprocess.run([exe, str(tmp_path), str(m), str(n), str(k)], capture_output=True, text=True, env=env,
                         timeout=300)
    assert run.returncode == 0, run.stderr + run.stdout
    s_ga, s_gw = np.fromfile(tmp_path / "scales.bin", dtype=np.float32)

    def read(name, dtype=np.uint8):
        return np.fromfile(tmp_path / name, dtype=dtype)

    # quantisation: scales and bytes bit-exact against the oracle
    a32 = p.a.float().numpy()
    w32 = p.modules[0].float().numpy()
    assert s_ga == oracle.global_scale(a32) and s_gw == oracle.global_scale(w32)
    qa, sfa = oracle.quantize(a32, s_ga)
    qw, sfw = oracle.quantize(w32, s_gw)
    np.testing.assert_array_equal(read("a_q.bin").reshape(m, k // 2), qa)
    np.testing.assert_array_equal(read("w_q.bin").reshape(n, k // 2), qw)
    np.testing.assert_array_equal(oracle.sf_from_tiled(read("a_sf.bin"), m, k), sfa)
    np.testing.assert_array_equal(oracle.sf_from_tiled(read("w_sf.bin"), n, k), sfw)
    # the GEMM on sampled rows
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 127, 128, m - 1], rng.choice(m, 28, replace=False)]))
    c32 = read("c32.bin", np.float32).reshape(m, n)
    c64, info = oracle.linear(p.a, p.modules, rows=rows)
    assert_gemm_close(c32[rows], c64, info["a_hat"], oracle.fused_weight_hat(info["qmods"]), "C host prefill")
    c16 = read("c16.bin", np.uint16).reshape(m, n)
    np.testing.assert_array_equal(c16, oracle.bf16_round(c32).reshape(m, n))
