"""Shared helpers for the GPU parity tests (tolerances and marshalling)."""
import numpy as np
import torch

import oracle

QMV_REL = 1e-3          # qmv: relative error 1e-3 (fp32 accumulation)
QMM_REL = 2e-2          # qmm/gather: |err| <= 2e-2 * |x_row| * |w_row| / sqrt(K)


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def check_qmv(y: np.ndarray, ref: np.ndarray, absdot: np.ndarray):
    """Per element |y - ref| <= 1e-3 * sum_k |x w| and max-norm relative <= 1e-3."""
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(np.isfinite(y))
    worst = float(np.max(err / np.maximum(absdot, 1e-300)))
    assert worst <= QMV_REL, f"per-element relative error {worst:.3e}"
    rel = float(err.max() / max(np.abs(ref).max(), 1e-300))
    assert rel <= QMV_REL, f"max-norm relative error {rel:.3e}"
    return worst, rel


def check_qmm(y: np.ndarray, ref: np.ndarray, xnorm: np.ndarray, wnorm: np.ndarray, k: int):
    """max |y - ref| <= 2e-2 * ||x_m|| * ||w_n|| / sqrt(K), per element."""
    bound = QMM_REL * np.outer(xnorm, wnorm) / np.sqrt(k)
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(np.isfinite(y))
    worst = float(np.max(err / np.maximum(bound, 1e-300)))
    assert worst <= 1.0, f"error / bound = {worst:.3f}"
    return worst


def row_norms_x(x_bits: np.ndarray) -> np.ndarray:
    return np.linalg.norm(oracle.bf16_to_f32(x_bits).astype(np.float64), axis=1)


def row_norms_w(qtype: int, w: np.ndarray, k: int) -> np.ndarray:
    return np.linalg.norm(oracle.dequantize(qtype, w, k).astype(np.float64), axis=1)
