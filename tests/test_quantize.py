"""Encoder on the GPU vs the CPU oracle: the wire bytes must be identical
(integer output whose codes are decided in fp32 by the same fixed steps on
both sides), on ragged shapes, scale extremes and a full-size tensor, and the
GPU's bytes decode back within the oracle's round-trip bound."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle

pytestmark = pytest.mark.gpu


def gpu_quantize(qtype, w):
    return kq.quantize(torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda(), qtype).cpu().numpy()


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
@pytest.mark.parametrize("rows,k", [(37, 2048), (1, 256), (5, 1280)])
def test_quantize_bytes_match_oracle(qtype, rows, k):
    g = np.random.default_rng(rows + k)
    w = (g.standard_normal((rows, k)) * g.uniform(1e-3, 5, (rows, 1))).astype(np.float32)
    assert np.array_equal(gpu_quantize(qtype, w), oracle.quantize(qtype, w))


def test_quantize_q8_0_partial_last_group():
    # 7 q8_0 blocks: the last warp group holds fewer than 8 blocks
    w = np.random.default_rng(3).standard_normal((7, 32)).astype(np.float32)
    assert np.array_equal(gpu_quantize(kq.Q8_0, w.reshape(1, -1)), oracle.quantize(kq.Q8_0, w.reshape(1, -1)))


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
def test_quantize_special_values(qtype):
    g = np.random.default_rng(5)
    w = g.standard_normal((8, 512)).astype(np.float32)
    w[0] = 0.0                                  # all-zero blocks
    w[1] = -0.0                                 # negative zeros
    w[2, :256] = 3.0                            # constant block
    w[3] = -np.abs(w[3])                        # all negative (q4_K min below zero)
    w[4] = np.abs(w[4])                         # all positive (q4_K min = 0)
    w[5, ::7] = 0.0                             # sprinkled zeros
    w[6] *= 1e-6                                # tiny scales (binary16 subnormal d)
    w[7] = np.round(w[7] * 4) / 4               # values on a coarse grid (rounding ties)
    assert np.array_equal(gpu_quantize(qtype, w), oracle.quantize(qtype, w))


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
def test_quantize_full_size_and_round_trip(qtype):
    g = np.random.default_rng(7)
    w = (g.standard_normal((4096, 4096)) * 0.02).astype(np.float32)
    q = gpu_quantize(qtype, w)
    assert np.array_equal(q, oracle.quantize(qtype, w))
    d = kq.dequantize(torch.from_numpy(q).cuda(), qtype, 4096).cpu().numpy()
    step = {kq.Q4_K: 1 / 15, kq.Q6_K: 1 / 31, kq.Q8_0: 1 / 127}[qtype]
    amax = np.abs(w).max()
    assert np.abs(d - w).max() <= amax * step     # a coarse bound; the exact ones are in the oracle pins


def test_quantize_empty_and_unsupported_codec():
    z = torch.empty(0, 256, dtype=torch.float32, device="cuda")
    assert kq.quantize(z, kq.Q4_K).shape == (0, 144)
    with pytest.raises(kq.KQError, match="unsupported"):
        kq.quantize(torch.zeros(1, 256, device="cuda"), kq.Q5_K)
