"""Seeded synthetic inputs for the GGUF block-quantized matmul path.

This module only draws random numbers and places them into the byte fields of
the wire blocks; it performs none of the decode or matmul arithmetic.  Both the
CPU oracle (``oracle/``) and the CUDA library are fed the very same bytes.

Block field positions follow the GGUF/ggml wire layout whose per-codec sizes
are printed in the mlx-kquant README (METADATA page), "Codec reference" table:
q4_K 144 B / 256 values, q5_K 176 B / 256, q6_K 210 B / 256 values, q8_0 34 B /
32 values, q4_0 18 B / 32.

Distributions (one ``numpy.random.Generator(PCG64(seed))`` stream per tensor):

* q4_K: ``qs`` uniform bytes (uniform 4-bit codes), the 12 packed scale bytes
  uniform (equivalent to independent uniform 6-bit scale/min codes in 0..63,
  the 96 bits being disjoint), ``d, dmin = fp16(|N(0,1)| * 1e-3)``.
* q6_K: ``ql``/``qh`` uniform bytes, int8 sub-scales uniform in [-64, 63],
  ``d = fp16(|N(0,1)| * 1e-3)``.
* q8_0: int8 codes uniform in [-128, 127], ``d = fp16(|N(0,1)| * 1e-3)``.
* q5_K (176 B): as q4_K for ``d, dmin``, the scale bytes and the nibbles, plus
  uniform bytes for the 32 high-bit bytes ``qh``.
* q4_0 (18 B): ``d = fp16(|N(0,1)| * 1e-3)``, uniform nibble bytes.
* activations: bf16 (round-to-nearest-even) of N(0,1), returned as uint16 bits.
"""
from __future__ import annotations

import numpy as np

Q4_0, Q8_0, Q4_K, Q5_K, Q6_K = 2, 8, 12, 13, 14
NAMES = {Q4_0: "q4_0", Q8_0: "q8_0", Q4_K: "q4_K", Q5_K: "q5_K", Q6_K: "q6_K"}
BLOCK_VALUES = {Q4_0: 32, Q8_0: 32, Q4_K: 256, Q5_K: 256, Q6_K: 256}
BLOCK_BYTES = {Q4_0: 18, Q8_0: 34, Q4_K: 144, Q5_K: 176, Q6_K: 210}

SEED_W, SEED_X, SEED_ROUTE = 0, 1, 2


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def row_bytes(qtype: int, k: int) -> int:
    if k % BLOCK_VALUES[qtype]:
        raise ValueError(f"K={k} is not a multiple of {BLOCK_VALUES[qtype]}")
    return k // BLOCK_VALUES[qtype] * BLOCK_BYTES[qtype]


def _scale_f16(g: np.random.Generator, n: int) -> np.ndarray:
    return (np.abs(g.standard_normal(n)) * 1e-3).astype(np.float16)


def weights(qtype: int, n: int, k: int, seed: int = SEED_W, experts: int = 0) -> np.ndarray:
    """Random wire bytes shaped [n, row_bytes] (or [experts, n, row_bytes])."""
    g = rng(seed)
    lead = (experts,) if experts else ()
    nblk = (experts or 1) * n * (k // BLOCK_VALUES[qtype])
    bpb = BLOCK_BYTES[qtype]
    blocks = g.integers(0, 256, size=(nblk, bpb), dtype=np.uint8)
    if qtype in (Q4_K, Q5_K):
        dd = _scale_f16(g, 2 * nblk).reshape(nblk, 2)
        blocks[:, 0:4] = dd.view(np.uint8).reshape(nblk, 4)
    elif qtype == Q6_K:
        blocks[:, 192:208] = g.integers(-64, 64, size=(nblk, 16), dtype=np.int8).view(np.uint8)
        blocks[:, 208:210] = _scale_f16(g, nblk).view(np.uint8).reshape(nblk, 2)
    elif qtype in (Q8_0, Q4_0):
        blocks[:, 0:2] = _scale_f16(g, nblk).view(np.uint8).reshape(nblk, 2)
    else:
        raise ValueError(qtype)
    return blocks.reshape(*lead, n, row_bytes(qtype, k))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def activations(m: int, k: int, seed: int = SEED_X) -> np.ndarray:
    """bf16 N(0,1) activations [m, k] as uint16 bits."""
    return f32_to_bf16_bits(rng(seed).standard_normal((m, k), dtype=np.float32))


def activations_scaled(scales, k: int, seed: int = SEED_X) -> np.ndarray:
    """bf16 activations [len(scales), k] as uint16 bits, row i drawn from
    N(0, scales[i]^2): rows of very different magnitude in one batch."""
    g = rng(seed)
    rows = [np.float32(sc) * g.standard_normal(k, dtype=np.float32) for sc in scales]
    return f32_to_bf16_bits(np.stack(rows))


def activations_outliers(m: int, k: int, small: float, big: float, per_row: int,
                         seed: int = SEED_X) -> np.ndarray:
    """bf16 activations [m, k] as uint16 bits: N(0, small^2) values with
    `per_row` entries per row replaced by +-big at seeded positions."""
    g = rng(seed)
    x = np.float32(small) * g.standard_normal((m, k), dtype=np.float32)
    for i in range(m):
        pos = g.choice(k, per_row, replace=False)
        x[i, pos] = np.float32(big) * np.where(g.random(per_row) < 0.5, -1.0, 1.0).astype(np.float32)
    return f32_to_bf16_bits(x)


def routing(tokens: int, n_experts: int, top_k: int, seed: int = SEED_ROUTE) -> np.ndarray:
    """int32 [tokens, top_k]: the first top_k entries of a seeded permutation
    of 0..n_experts-1 per token (distinct experts, uniformly at random)."""
    g = rng(seed)
    keys = g.random((tokens, n_experts))
    return np.argsort(keys, axis=1, kind="stable")[:, :top_k].astype(np.int32)


# Named workloads: the five shapes the path is specified and measured on.
WORKLOADS = {
    "c0_q4K_qmv_4096x4096": dict(kind="qmv", types=[Q4_K], m=[1], n=4096, k=4096, dequant=True),
    "c1_q8_0_q6K_qmv_14336x4096": dict(kind="qmv", types=[Q8_0, Q6_K], m=[1], n=14336, k=4096),
    "c2_q4K_qmv_4096x14336": dict(kind="qmv", types=[Q4_K], m=[1, 4, 8, 16], n=4096, k=14336),
    "c3_q4K_q6K_qmm_2048x14336x4096": dict(kind="qmm", types=[Q4_K, Q6_K], m=[2048], n=14336, k=4096),
    "c4_q4K_gather_8x14336x4096_t512_top2": dict(kind="gather", types=[Q4_K], experts=8, tokens=512,
                                                 top_k=2, n=14336, k=4096),
}
