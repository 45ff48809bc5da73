"""kq_dequantize vs the CPU oracle: bit-exact (compared as fp32 bit patterns)."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import dev_u8

pytestmark = pytest.mark.gpu


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
@pytest.mark.parametrize("n,k", [(1, 256), (7, 768), (33, 4096), (130, 2304)])
def test_bit_exact(qtype, n, k):
    w = synth.weights(qtype, n, k, seed=100 + n)
    y = kq.dequantize(dev_u8(w), qtype, k).cpu().numpy()
    assert np.array_equal(bits(y), bits(oracle.dequantize(qtype, w, k)))


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
def test_random_bytes_and_zero_blocks(qtype):
    vpb, bpb = kq.block_info(qtype)
    k = 4 * 256
    raw = np.random.default_rng(7).integers(0, 256, size=(64, k // vpb * bpb), dtype=np.uint8)
    raw[5] = 0                                     # all-zero blocks: +0.0 / -0.0 signs matter
    y = kq.dequantize(dev_u8(raw), qtype, k).cpu().numpy()
    ref = oracle.dequantize(qtype, raw, k)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(y), nan)
    assert np.array_equal(bits(y)[~nan], bits(ref)[~nan])


def test_empty_is_a_no_op():
    out = torch.full((0, 256), 7.0, device="cuda")
    kq.dequantize(torch.empty(0, 144, dtype=torch.uint8, device="cuda"), kq.Q4_K, 256, out=out)
    torch.cuda.synchronize()


def test_full_size_4096x4096_q4K():
    n = k = 4096
    w = synth.weights(kq.Q4_K, n, k)
    y = kq.dequantize(dev_u8(w), kq.Q4_K, k).cpu().numpy()
    assert np.array_equal(bits(y), bits(oracle.dequantize(kq.Q4_K, w, k)))


def test_deterministic():
    w = dev_u8(synth.weights(kq.Q6_K, 64, 2048))
    a = kq.dequantize(w, kq.Q6_K, 2048)
    b = kq.dequantize(w, kq.Q6_K, 2048)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
