"""q5_K and q4_0 on the GPU vs the CPU oracle: dequantize bit-exact, the
tensor-core products (qmm, gather) within the qmm bound, and kq_qmv within
the qmv bound: the staged tensor-core decode kernel (q5_K up to M = 16,
q4_0 up to M = 2) and beyond it the exact fp32 decode-and-dot kernel."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmm, check_qmv, dev_bf16, dev_u8, row_norms_w, row_norms_x

pytestmark = pytest.mark.gpu
CODECS = [kq.Q5_K, kq.Q4_0]


@pytest.mark.parametrize("qtype", CODECS)
def test_dequantize_bit_exact(qtype):
    k = 2048
    w = synth.weights(qtype, 37, k, seed=3)
    out = kq.dequantize(dev_u8(w), qtype, k).cpu().numpy()
    assert np.array_equal(out.view(np.uint32), oracle.dequantize(qtype, w, k).view(np.uint32))
    # fully random bytes (any finite binary16 scale)
    raw = np.random.default_rng(4).integers(0, 256, size=(64, synth.row_bytes(qtype, 256)), dtype=np.uint8)
    vpb, bpb = synth.BLOCK_VALUES[qtype], synth.BLOCK_BYTES[qtype]
    blk = raw.reshape(-1, bpb)
    for off in ((0, 2) if qtype == kq.Q5_K else (0,)):
        h = blk[:, off:off + 2].copy().view(np.uint16)
        h[(h & 0x7c00) == 0x7c00] &= 0x3fff       # no inf / NaN scales
        blk[:, off:off + 2] = h.view(np.uint8)
    raw = blk.reshape(64, -1)
    out = kq.dequantize(dev_u8(raw), qtype, 256).cpu().numpy()
    assert np.array_equal(out.view(np.uint32), oracle.dequantize(qtype, raw, 256).view(np.uint32))


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m,n", [(300, 200), (2, 1000)])
def test_qmm_vs_oracle(qtype, m, n):
    k = 2048
    w = synth.weights(qtype, n, k, seed=5)
    x = synth.activations(m, k, seed=6)
    y = kq.qmm(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    check_qmm(y, oracle.matmul(qtype, w, k, x), row_norms_x(x), row_norms_w(qtype, w, k), k)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m", [1, 2, 3, 5, 16])
def test_qmv_vs_oracle(qtype, m):
    n, k = 1000, 4096
    w = synth.weights(qtype, n, k, seed=7)
    x = synth.activations(m, k, seed=8)
    y = kq.qmv(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    ref, a = oracle.matmul(qtype, w, k, x, absdot=True)
    check_qmv(y, ref, a)


@pytest.mark.parametrize("qtype", CODECS)
def test_gather_vs_oracle(qtype):
    experts, n, k = 3, 160, 1024
    ids = np.sort(np.random.default_rng(9).integers(0, experts, 300)).astype(np.uint32)
    tiles = oracle.tile_map(ids, experts)
    w = synth.weights(qtype, n, k, seed=10, experts=experts)
    x = synth.activations(len(ids), k, seed=11)
    tm = torch.tensor(np.array(tiles, dtype=np.int64).reshape(-1, 3), dtype=torch.int32).cuda()
    cnt = torch.tensor([len(tiles)], dtype=torch.int32).cuda()
    y = kq.gather_qmm(dev_bf16(x), dev_u8(w), qtype, tm, cnt).cpu().numpy()
    ref = oracle.gather_qmm(qtype, w, k, x, tiles)
    xn = row_norms_x(x)
    for e in range(experts):
        r = np.nonzero(ids == e)[0]
        check_qmm(y[r], ref[r], xn[r], row_norms_w(qtype, w[e], k), k)


def test_q4_0_qmv_needs_whole_256_value_steps():
    # q4_0 rows of 96 values: dequantize works, the decode product refuses
    w = synth.weights(kq.Q4_0, 8, 96, seed=12)
    d = kq.dequantize(dev_u8(w), kq.Q4_0, 96).cpu().numpy()
    assert np.array_equal(d.view(np.uint32), oracle.dequantize(kq.Q4_0, w, 96).view(np.uint32))
    with pytest.raises(kq.KQError, match="unsupported"):
        kq.qmv(dev_bf16(synth.activations(1, 96)), dev_u8(w), kq.Q4_0)
