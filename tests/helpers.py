"""Shared helpers for the GPU parity tests: marshalling between the oracle's
numpy view and the library's device buffers, and the tolerance check of the
GEMM parity (per element 1e-3 * |A_hat row| * |W_hat row|, relative Frobenius
2e-3, both before the BF16 cast)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import nvfp4_w4a4_quantized_07_b200 as nv

ELEM_TOL = 1e-3
FRO_TOL = 2e-3


def to_np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)


def sf_rowmajor(sf_tiled: torch.Tensor, rows: int, k: int, row_offset: int = 0) -> np.ndarray:
    """Row-major view of (part of) a tiled scale buffer via the oracle's own map."""
    full = oracle.sf_from_tiled(to_np_u8(sf_tiled), row_offset + rows, k)
    return full[row_offset:row_offset + rows]


def gemm_check(c_gpu, c64: np.ndarray, a_hat: np.ndarray, w_hat: np.ndarray):
    """Return (max element error / bound, relative Frobenius error)."""
    c = c_gpu.detach().double().cpu().numpy() if isinstance(c_gpu, torch.Tensor) else np.asarray(c_gpu, np.float64)
    rn = np.linalg.norm(a_hat, axis=1)
    wn = np.linalg.norm(w_hat, axis=1)
    bound = ELEM_TOL * rn[:, None] * wn[None, :]
    err = np.abs(c - c64)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    denom = np.linalg.norm(c64)
    fro = np.linalg.norm(c - c64) / denom if denom > 0 else np.linalg.norm(c - c64)
    return float(ratio.max()), float(fro)


def assert_gemm_close(c_gpu, c64, a_hat, w_hat, what=""):
    ratio, fro = gemm_check(c_gpu, c64, a_hat, w_hat)
    assert ratio <= 1.0 and fro <= FRO_TOL, f"{what}: max err/bound {ratio:.3g}, rel Frobenius {fro:.3g}"


def device_operands(codes: np.ndarray, sf_rm: np.ndarray, device="cuda"):
    """Pack signed E2M1 codes (rows x k) and row-major scale bytes into the
    library's buffers: packed q (low nibble = even element) and tiled scales."""
    rows, k = codes.shape
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    tiled = oracle.sf_to_tiled(sf_rm, k)
    return torch.from_numpy(q).to(device), torch.from_numpy(tiled).to(device)


def act_from_codes(codes, sf_rm, s_ga, device="cuda") -> nv.QuantizedActivation:
    q, sf = device_operands(codes, sf_rm, device)
    scale = torch.tensor([s_ga], dtype=torch.float32, device=device)
    return nv.QuantizedActivation(q=q, sf=sf, scale=scale, m=codes.shape[0], k=codes.shape[1])


def weight_from_codes(codes, sf_rm, segments, device="cuda") -> nv.FusedWeight:
    q, sf = device_operands(codes, sf_rm, device)
    return nv.FusedWeight(q=q, sf=sf, segments=segments, n=codes.shape[0], k=codes.shape[1])


def dequant_codes(codes, sf_rm, s_g):
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return oracle.dequantize(q, sf_rm, s_g)
