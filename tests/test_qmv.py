"""kq_qmv vs the fp64 CPU oracle: per-element error <= 1e-3 * sum_k |x*w| and
max-norm relative error <= 1e-3, plus determinism and row independence."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmv, dev_bf16, dev_u8

pytestmark = pytest.mark.gpu
CODECS = [kq.Q4_K, kq.Q6_K, kq.Q8_0, kq.Q5_K, kq.Q4_0]


def run(qtype, n, k, m, seed=0):
    w = synth.weights(qtype, n, k, seed=seed)
    x = synth.activations(m, k, seed=seed + 1)
    y = kq.qmv(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    ref, absdot = oracle.matmul(qtype, w, k, x, absdot=True)
    return check_qmv(y, ref, absdot)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 8, 9, 16])
def test_small_shapes(qtype, m):
    # several 16-row CTAs plus a ragged tail, K spanning several stages
    run(qtype, 16 * 5 + 3, 2048 + 1024, m, seed=m)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("k", [256, 768, 4352])
def test_unaligned_rows_and_tails(qtype, k):
    # K=768 gives q6_K rows of 630 bytes (not a multiple of 16: staging fallback);
    # 4352 = 17 blocks leaves a partial stage
    run(qtype, 40, k, 1, seed=k)
    run(qtype, 40, k, 7, seed=k + 1)


def test_c0_q4K_4096x4096_m1():
    run(kq.Q4_K, 4096, 4096, 1, seed=synth.SEED_W)


@pytest.mark.parametrize("qtype", [kq.Q8_0, kq.Q6_K])
def test_c1_14336x4096_m1(qtype):
    run(qtype, 14336, 4096, 1, seed=synth.SEED_W)


@pytest.mark.parametrize("m", [1, 4, 8, 16])
def test_c2_q4K_4096x14336(m):
    run(kq.Q4_K, 4096, 14336, m, seed=synth.SEED_W)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q5_K])
@pytest.mark.parametrize("m", [7, 9, 16])
def test_q4K_long_k_many_tokens(qtype, m):
    # an activation image of m x K that does not fit in shared memory at once:
    # the decode kernel walks K in chunks (two images in turn); ragged N
    run(qtype, 200, 8192, m, seed=40 + m)


# q4_K from M = 4 splits K over a cluster of CTAs (4 CTAs when the slices
# keep >= 7 blocks, else 2) and reduces the slices through the CTAs' shared
# memory: clusters with fewer than 16 rows and a ragged row group (n = 37),
# several row groups per cluster so that the two partial-sum slots are reused
# (n = 2647), and the 2-CTA split (K = 3584: 14 blocks)
@pytest.mark.parametrize("n,k,m", [(37, 7168, 4), (37, 7168, 12), (2647, 7168, 5), (300, 3584, 8),
                                   (300, 3584, 16)])
@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q5_K])
def test_q4K_split_k(qtype, n, k, m):
    run(qtype, n, k, m, seed=n + m)


@pytest.mark.parametrize("qtype", CODECS)
def test_deterministic_and_row_independent(qtype):
    n, k = 200, 4096
    w = dev_u8(synth.weights(qtype, n, k, seed=3))
    x = synth.activations(6, k, seed=4)
    xd = dev_bf16(x)
    a = kq.qmv(xd, w, qtype)
    b = kq.qmv(xd, w, qtype)
    assert torch.equal(a, b)
    # row 2 alone vs in a batch of 6: identical bits are not promised across
    # different m (other kernels), but the same row in the same batch shape is
    x2 = x.copy()
    x2[[0, 1, 3, 4, 5]] = synth.activations(5, k, seed=9)
    c = kq.qmv(dev_bf16(x2), w, qtype)
    assert torch.equal(a[2], c[2])


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q5_K])
def test_one_row_long_k_falls_back(qtype):
    # K = 65536: the one-row column form's activation image and raw copy do
    # not fit in shared memory, so the call takes the scale-in-operand form
    # (split over a cluster or with the image built from x in place)
    run(qtype, 40, 65536, 1, seed=77)


@pytest.mark.parametrize("qtype", [kq.Q8_0, kq.Q6_K])
@pytest.mark.parametrize("n,k", [(2600, 4096), (2664, 14336), (150, 1024)])
def test_one_and_two_row_groups(qtype, n, k):
    # 17 or 18 rows per CTA (1 or 2 rows per CTA at N = 150) leave row groups
    # of one or two rows in the 16-row tensor-core items; K = 14336 splits
    # every row over several stages
    run(qtype, n, k, 1, seed=n + k)
    run(qtype, n, k, 2, seed=n + k + 1)
