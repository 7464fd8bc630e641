"""Seeded synthetic inputs shaped like a 27B hybrid layer's linear projections.

This module holds no quantization or GEMM arithmetic: it only draws random
tensors.  The same host bytes feed both the CUDA path and the CPU oracle.

Recipe (all on the host, torch CPU ``Generator``):

* activations: N(0, 1) in FP32, then a seeded set of ``round(frac * K)``
  distinct channels (columns) is multiplied by ``gain`` for every row, which
  mimics the residual-stream outlier channels the pages describe for
  Qwen3.8-27B ("Why Gated DeltaNet Survives 4-Bit Quantization", abstract,
  mechanism (i)).  The outlier columns are drawn from the same generator after
  the normals.  The FP32 tensor is then cast to the requested dtype (BF16 by
  default, round-to-nearest-even).
* weights: N(0, std) in FP32 from their own seed, cast the same way.

Module seeds: activations use ``seed``; module ``i`` of a fused weight uses
``1 + i``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import math

import torch

HIDDEN = 5120

# Output widths of the fused GDN-style input projection: q, k, v, z and the two
# 48-wide gate inputs.  Their sum (12384) is the fused N.
GDN_IN_PROJ_WIDTHS = (2048, 2048, 4096, 4096, 48, 48)
GDN_IN_PROJ_STDS = (0.02, 0.02, 0.02, 0.02, 0.2, 0.2)
MLP_INTERMEDIATE = 17408


def activations(m: int, k: int, seed: int = 0, outlier_frac: float = 0.001,
                outlier_gain: float = 100.0, n_outliers: int | None = None,
                dtype: torch.dtype = torch.bfloat16):
    """Return ``(A, outlier_columns)``; ``A`` is ``m x k`` row-major."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    a = torch.randn(m, k, generator=g, dtype=torch.float32)
    if n_outliers is None:
        n_outliers = int(round(outlier_frac * k))
    cols = torch.randperm(k, generator=g)[:n_outliers].sort().values
    if n_outliers:
        a[:, cols] *= outlier_gain
    return a.to(dtype).contiguous(), cols


def weights(n: int, k: int, std: float, seed: int, dtype: torch.dtype = torch.bfloat16):
    """``n x k`` weight (nn.Linear layout: output rows, K contiguous)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    w = torch.randn(n, k, generator=g, dtype=torch.float32) * std
    return w.to(dtype).contiguous()


@dataclass
class LinearProblem:
    """One linear layer: activations and a list of separately calibrated modules."""
    name: str
    a: torch.Tensor
    modules: list = field(default_factory=list)   # list of n_i x K weights
    outlier_cols: torch.Tensor | None = None

    @property
    def m(self) -> int:
        return self.a.shape[0]

    @property
    def k(self) -> int:
        return self.a.shape[1]

    @property
    def widths(self) -> list:
        return [w.shape[0] for w in self.modules]

    @property
    def n(self) -> int:
        return sum(self.widths)

    @property
    def flops(self) -> int:
        return 2 * self.m * self.n * self.k


def tiny() -> LinearProblem:
    """64x256 FP32 activations with one x50 column; 128x256 FP32 weight."""
    a, cols = activations(64, 256, seed=0, n_outliers=1, outlier_gain=50.0,
                          dtype=torch.float32)
    w = weights(128, 256, 0.02, seed=1, dtype=torch.float32)
    return LinearProblem("tiny 64x256 . 128x256 (fp32 in)", a, [w], cols)


def prefill(m: int = 4096, k: int = HIDDEN, n: int = HIDDEN) -> LinearProblem:
    """Single projection, one global weight scale."""
    a, cols = activations(m, k, seed=0)
    w = weights(n, k, 0.02, seed=1)
    return LinearProblem(f"prefill {m}x{k} . {n}x{k}", a, [w], cols)


def gdn_in_proj(m: int = 8192, k: int = HIDDEN, widths=GDN_IN_PROJ_WIDTHS,
                stds=GDN_IN_PROJ_STDS) -> LinearProblem:
    """Fused six-module GDN-style input projection, per-module global scales."""
    a, cols = activations(m, k, seed=0)
    mods = [weights(n_i, k, s_i, seed=1 + i) for i, (n_i, s_i) in enumerate(zip(widths, stds))]
    return LinearProblem(f"fused gdn in-proj {m}x{k} . {sum(widths)}x{k} ({len(widths)} segments)",
                         a, mods, cols)


def mlp_gate_up(m: int = 32768, k: int = HIDDEN, inter: int = MLP_INTERMEDIATE) -> LinearProblem:
    """Fused gate/up projection (two modules of ``inter`` rows)."""
    a, cols = activations(m, k, seed=0)
    mods = [weights(inter, k, 0.02, seed=1), weights(inter, k, 0.02, seed=2)]
    return LinearProblem(f"mlp gate/up {m}x{k} . {2 * inter}x{k}", a, mods, cols)


def mlp_down_weight(k: int = MLP_INTERMEDIATE, n: int = HIDDEN) -> torch.Tensor:
    return weights(n, k, 0.02, seed=3)


def gdn_gate_params(heads: int = 48, seed: int = 9):
    """Per-head parameters of a Gated DeltaNet layer's gates, drawn the usual
    way such layers are initialised: ``A_log = log(U(1, 16))`` and ``dt_bias``
    the inverse softplus of a step size log-uniform in [1e-3, 1e-1].  FP32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    A_log = torch.log(1.0 + 15.0 * torch.rand(heads, generator=g, dtype=torch.float64))
    dt = torch.exp(math.log(1e-3) + (math.log(1e-1) - math.log(1e-3)) * torch.rand(heads, generator=g,
                                                                                    dtype=torch.float64))
    dt_bias = dt + torch.log(-torch.expm1(-dt))
    return A_log.float(), dt_bias.float()


KV_HEADS, HEAD_DIM = 4, 256   # one attention layer's K/V row: 4 KV heads x 256


def kv_rows(tokens: int, width: int = KV_HEADS * HEAD_DIM, seed: int = 11, outlier_frac: float = 0.02,
            outlier_gain: float = 8.0):
    """New tokens' K and V rows (BF16, tokens x width): V ~ N(0, 1); K ~ N(0, 1)
    with a fixed ``outlier_frac`` of its channels scaled by ``outlier_gain``
    (keys carry a few large-magnitude channels)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    k = torch.randn(tokens, width, generator=g, dtype=torch.float32)
    n_out = max(1, int(round(outlier_frac * width)))
    cols = torch.randperm(width, generator=g)[:n_out]
    k[:, cols] *= outlier_gain
    v = torch.randn(tokens, width, generator=g, dtype=torch.float32)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def mlp_glue_inputs(m: int, f: int, seed: int = 5, gate_std: float = 2.0) -> torch.Tensor:
    """A fused ``[gate | up]`` BF16 tensor of shape ``m x 2f`` (gate N(0, gate_std^2),
    up N(0, 1)), the shape of a fused gate/up GEMM output."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    gate = torch.randn(m, f, generator=g, dtype=torch.float32) * gate_std
    up = torch.randn(m, f, generator=g, dtype=torch.float32)
    return torch.cat([gate, up], dim=1).to(torch.bfloat16).contiguous()


DECODE_SHAPES = {
    # name: (list of module widths, K, list of stds)
    "5120x5120": ([5120], HIDDEN, [0.02]),
    "12384x5120": (list(GDN_IN_PROJ_WIDTHS), HIDDEN, [0.02] * 6),
    "34816x5120": ([MLP_INTERMEDIATE, MLP_INTERMEDIATE], HIDDEN, [0.02, 0.02]),
    "5120x17408": ([HIDDEN], MLP_INTERMEDIATE, [0.02]),
}
DECODE_M = (1, 4, 16, 64)


def decode(m: int, shape: str) -> LinearProblem:
    widths, k, stds = DECODE_SHAPES[shape]
    a, _ = activations(m, k, seed=0, n_outliers=0)
    mods = [weights(n_i, k, s_i, seed=1 + i) for i, (n_i, s_i) in enumerate(zip(widths, stds))]
    return LinearProblem(f"decode m={m} {shape}", a, mods, None)
