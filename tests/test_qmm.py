"""kq_qmm (tcgen05) vs the fp64 CPU oracle:
max |y - ref| <= 2e-2 * ||x_row|| * ||w_row|| / sqrt(K)."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmm, dev_bf16, dev_u8, row_norms_w, row_norms_x

pytestmark = pytest.mark.gpu
CODECS = [kq.Q4_K, kq.Q6_K, kq.Q8_0]


def run_full(qtype, n, k, m, seed=0):
    w = synth.weights(qtype, n, k, seed=seed)
    x = synth.activations(m, k, seed=seed + 1)
    y = kq.qmm(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    ref = oracle.matmul(qtype, w, k, x)
    return check_qmm(y, ref, row_norms_x(x), row_norms_w(qtype, w, k), k)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m,n", [(1, 128), (16, 130), (300, 200), (512, 384)])
def test_small_shapes(qtype, m, n):
    run_full(qtype, n, 2048, m, seed=m + n)


@pytest.mark.parametrize("qtype", CODECS)
def test_k4096_ragged(qtype):
    run_full(qtype, 257, 4096, 513, seed=11)


# (m, n) with more (256-row, 128-weight-row) units than SMs, so that the last
# partial round of the grid is split: into four 64-row sub-units (m=300,
# n=10240: 160 units, some sub-units past the end of m), into two 128-row
# sub-units (m=200, n=25344: 198 units) and not at all (m=100, n=31744: 248
# units); the split depends on the SM count, all three are covered on 148 SMs
@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m,n", [(300, 10240), (200, 25344), (100, 31744)])
def test_last_round_split(qtype, m, n):
    # a q6_K row of K values is a multiple of 16 bytes only when K % 2048 == 0
    run_full(qtype, n, 2048 if qtype == kq.Q6_K else 256, m, seed=m + 7)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K])
def test_c3_full_size_sampled(qtype):
    m, n, k = 2048, 14336, 4096
    w = synth.weights(qtype, n, k)
    x = synth.activations(m, k)
    y = kq.qmm(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    g = np.random.default_rng(123)
    rows = np.sort(g.choice(m, 48, replace=False))
    cols = np.sort(g.choice(n, 48, replace=False))
    wn = row_norms_w(qtype, w, k)
    xn = row_norms_x(x)
    # all N for sampled activation rows, all M for sampled weight rows
    ref_r = oracle.matmul(qtype, w, k, x[rows])
    check_qmm(y[rows], ref_r, xn[rows], wn, k)
    ref_c = oracle.matmul(qtype, w[cols], k, x)
    check_qmm(y[:, cols], ref_c, xn, wn[cols], k)


def test_matches_qmv_at_small_m():
    n, k = 256, 4096
    w = dev_u8(synth.weights(kq.Q4_K, n, k, seed=21))
    x = dev_bf16(synth.activations(8, k, seed=22))
    a = kq.qmm(x, w, kq.Q4_K).double()
    b = kq.qmv(x, w, kq.Q4_K).double()
    wn = torch.from_numpy(row_norms_w(kq.Q4_K, synth.weights(kq.Q4_K, n, k, seed=21), k)).cuda()
    xn = x.float().norm(dim=1).double()
    assert torch.all((a - b).abs() <= 2e-2 * xn[:, None] * wn[None, :] / np.sqrt(k))


@pytest.mark.parametrize("qtype", CODECS)
def test_deterministic(qtype):
    w = dev_u8(synth.weights(qtype, 384, 2048, seed=1))
    x = dev_bf16(synth.activations(300, 2048, seed=2))
    assert torch.equal(kq.qmm(x, w, qtype), kq.qmm(x, w, qtype))


# q6_K rows that are not a 16-byte multiple (K / 256 not a multiple of 8: 210
# bytes per block) take the flat view of the weights, each row's window loaded
# on its own and decoded at its own byte offset: K = 768 (630-byte rows),
# K = 11008 (9030-byte rows), ragged M and N, several units and the last-round
# split
@pytest.mark.parametrize("m,n,k", [(70, 130, 768), (300, 257, 11008), (200, 25344, 768)])
def test_q6K_rows_not_16_byte_multiple(m, n, k):
    assert synth.row_bytes(kq.Q6_K, k) % 16 != 0
    run_full(kq.Q6_K, n, k, m, seed=k + m)


def test_q6K_k11008_large_sampled():
    m, n, k = 1024, 14336, 11008
    w = synth.weights(kq.Q6_K, n, k, seed=3)
    x = synth.activations(m, k, seed=4)
    y = kq.qmm(dev_bf16(x), dev_u8(w), kq.Q6_K).cpu().numpy()
    g = np.random.default_rng(5)
    rows = np.sort(g.choice(m, 16, replace=False))
    cols = np.sort(g.choice(n, 16, replace=False))
    wn = row_norms_w(kq.Q6_K, w, k)
    xn = row_norms_x(x)
    check_qmm(y[rows], oracle.matmul(kq.Q6_K, w, k, x[rows]), xn[rows], wn, k)
    check_qmm(y[:, cols], oracle.matmul(kq.Q6_K, w[cols], k, x), xn, wn[cols], k)
