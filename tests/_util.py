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


def zero_weights_at(qtype: int, w: np.ndarray, cols) -> np.ndarray:
    """Copy of the packed rows w ([N, row_bytes] or [E, N, row_bytes]) in which
    every row holds, at the value columns `cols`, the code that decodes to an
    exact zero: the format's code offset (q8_0: code 0; q4_0: nibble 8; q6_K:
    6-bit code 32, i.e. low nibble 0 and high bits 2).  Byte positions follow
    the block layouts (q4_0: value i < 16 in the low nibble of byte i, value
    i >= 16 in the high nibble of byte i - 16; q6_K: value 128h + 32q + l in
    nibble q >> 1 of ql[64h + 32 (q & 1) + l] and bits 2q of qh[32h + l])."""
    out = np.array(w, dtype=np.uint8, copy=True)
    flat = out.reshape(-1, out.shape[-1])
    for c in cols:
        if qtype == oracle.Q8_0:
            b, i = divmod(int(c), 32)
            flat[:, 34 * b + 2 + i] = 0
        elif qtype == oracle.Q4_0:
            b, i = divmod(int(c), 32)
            o = 18 * b + 2 + (i & 15)
            flat[:, o] = (flat[:, o] & 0xF0) | 0x08 if i < 16 else (flat[:, o] & 0x0F) | 0x80
        elif qtype == oracle.Q6_K:
            b, i = divmod(int(c), 256)
            h, r = divmod(i, 128)
            q, l = divmod(r, 32)
            o = 210 * b + 64 * h + 32 * (q & 1) + l
            flat[:, o] &= np.uint8(0xFF ^ (0xF << (4 * (q >> 1))))
            oh = 210 * b + 128 + 32 * h + l
            flat[:, oh] = (flat[:, oh] & np.uint8(0xFF ^ (3 << (2 * q)))) | np.uint8(2 << (2 * q))
        else:
            raise ValueError("no zero code for this format")
    return out
