"""The decode products over the whole activation range.

The pages fix no range for the activations (mlx-kquant bindings.cpp,
`quantized_matmul`: x is any float array), and the qmv bound is a relative
one ("within relative error 1e-3"), so it must hold whatever the magnitude of
x: tiny (N(0, sigma^2) down to sigma = 1e-5), large (beyond the binary16
range), rows of very different magnitude in one batch, and rows where a few
large entries sit among small ones.  Every call is checked against the fp64
oracle with the qmv bound (per element 1e-3 * sum |x w| and max-norm 1e-3).
Shapes reach the staged kernel (M <= 2; q4_K / q5_K up to M = 16), the
K-split q4_K / q5_K kernel (M >= 4), the general kernel (q8_0 / q6_K at
M >= 3; q6_K with 630-byte rows at K = 768), the exact fp32 kernel (q4_0 at
M >= 3) and the decode MoE kernels (gather_qmv,
moe_glu_gather)."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmv, dev_bf16, dev_u8, zero_weights_at

pytestmark = pytest.mark.gpu
CODECS = [kq.Q4_K, kq.Q6_K, kq.Q8_0, kq.Q5_K, kq.Q4_0]


def run(qtype, n, k, x, seed=0, w=None):
    w = synth.weights(qtype, n, k, seed=seed) if w is None else w
    y = kq.qmv(dev_bf16(x), dev_u8(w), qtype).cpu().numpy()
    ref, absdot = oracle.matmul(qtype, w, k, x, absdot=True)
    return check_qmv(y, ref, absdot)


def outliers_at(m, k, cols, small, big, seed):
    """N(0, small^2) rows with +-big at the given columns."""
    x = oracle.bf16_to_f32(synth.activations_scaled([small] * m, k, seed=seed)).copy()
    sign = np.where(np.random.default_rng(seed).random((m, len(cols))) < 0.5, -1.0, 1.0)
    x[:, cols] = (big * sign).astype(np.float32)
    return synth.f32_to_bf16_bits(x)


# Large activations where every weight row decodes to an exact zero (the
# format's code offset): sum |x w| then holds only the small terms, so the
# large products must cancel exactly.  The codes are centred on the offset
# in binary16 before the MMA, which makes each such product an exact zero.
ZERO_COLS = [3, 700, 1333, 2047]


@pytest.mark.parametrize("qtype", [kq.Q8_0, kq.Q6_K, kq.Q4_0])
@pytest.mark.parametrize("m", [1, 2, 3, 7, 16])
def test_outliers_on_zero_weights(qtype, m):
    k, n = 2048, 16 * 6 + 5
    w = zero_weights_at(qtype, synth.weights(qtype, n, k, seed=70), ZERO_COLS)
    run(qtype, n, k, outliers_at(m, k, ZERO_COLS, 1e-3, 1e4, seed=71 + m), w=w)


@pytest.mark.parametrize("qtype", [kq.Q8_0, kq.Q6_K, kq.Q4_0])
def test_decode_moe_outliers_on_zero_weights(qtype):
    tokens, top_k, experts, n, k = 3, 2, 4, 150, 2048
    wg = zero_weights_at(qtype, synth.weights(qtype, n, k, seed=72, experts=experts), ZERO_COLS)
    wu = zero_weights_at(qtype, synth.weights(qtype, n, k, seed=73, experts=experts), ZERO_COLS)
    ids = synth.routing(tokens, experts, top_k, seed=74)
    x = outliers_at(tokens * top_k, k, ZERO_COLS, 1e-3, 1e4, seed=75)
    y = torch.full((tokens * top_k, n), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.gather_qmv(dev_bf16(x), dev_u8(wg), qtype, torch.from_numpy(ids).cuda(), out=y, err=err)
    assert int(err.item()) == 0
    ref, a = oracle.gather_qmv(qtype, wg, k, x, ids, absdot=True)
    check_qmv(y.cpu().numpy(), ref, a)
    # the gate/up GLU with one activation row per token
    xt = outliers_at(tokens, k, ZERO_COLS, 1e-3, 1e4, seed=76)
    out = kq.moe_glu_gather(dev_bf16(xt), dev_u8(wg), dev_u8(wu), qtype, torch.from_numpy(ids).cuda())
    ref, g, u, ag, au = oracle.moe_glu_gather(qtype, wg, wu, k, xt, ids)
    dg, du = 1e-3 * ag, 1e-3 * au
    a = np.abs(oracle.glu(oracle.ACT_SILU, g, np.ones_like(g)))
    tol = 1.2 * dg * (np.abs(u) + du) + (a + 1.2 * dg) * du + 1e-5 * np.abs(ref) + 1e-300
    yv = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(yv))
    assert float(np.max(np.abs(yv - ref) / tol)) <= 1.0


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("sigma", [1e-2, 1e-3, 1e-5])
@pytest.mark.parametrize("m", [1, 2, 3, 9, 16])
def test_small_activations(qtype, sigma, m):
    x = synth.activations_scaled([sigma] * m, 4096, seed=m)
    run(qtype, 16 * 9 + 5, 4096, x, seed=int(-np.log10(sigma)))


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("sigma", [1e4, 1e8, 1e30])
def test_large_activations(qtype, sigma):
    # beyond binary16's 65504: the power-of-two scaling brings them in range
    x = synth.activations_scaled([sigma, sigma / 7], 2048, seed=3)
    run(qtype, 100, 2048, x, seed=4)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("scales", [[1e-4, 1e2], [1e-6, 1e-2, 1.0, 1e2, 1e5], [1e2] + [1e-4] * 8,
                                    [10.0 ** (e % 9 - 4) for e in range(16)]])
def test_rows_of_mixed_scale(qtype, scales):
    x = synth.activations_scaled(scales, 3072, seed=len(scales))
    run(qtype, 16 * 6 + 1, 3072, x, seed=5)


@pytest.mark.parametrize("qtype", CODECS)
@pytest.mark.parametrize("m", [1, 2, 5])
def test_outliers_among_small_values(qtype, m):
    x = synth.activations_outliers(m, 4096, small=1e-3, big=1e4, per_row=3, seed=10 + m)
    run(qtype, 16 * 7 + 9, 4096, x, seed=11)


@pytest.mark.parametrize("qtype", [kq.Q6_K, kq.Q4_K, kq.Q8_0])
@pytest.mark.parametrize("m", [1, 7])
def test_general_kernel_unaligned_rows(qtype, m):
    # K = 768: q6_K rows of 630 bytes (not a 16-byte multiple) take the
    # general kernel's staging path
    for x in (synth.activations_scaled([1e-5] * m, 768, seed=20 + m),
              synth.activations_outliers(m, 768, small=1e-3, big=3e4, per_row=2, seed=21 + m)):
        run(qtype, 50, 768, x, seed=22)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q5_K])
@pytest.mark.parametrize("m", [4, 8, 16])
def test_q4K_split_k_small_and_mixed(qtype, m):
    # K = 7168: the q4_K / q5_K kernel splits K over a cluster of CTAs, each
    # slice scaled on its own before the slices are summed
    x = synth.activations_scaled([10.0 ** (-5 + (i % 8)) for i in range(m)], 7168, seed=30 + m)
    run(qtype, 37, 7168, x, seed=31)


@pytest.mark.parametrize("m", [3, 16])
def test_exact_kernel_q4_0(m):
    # q4_0 from M = 3 takes the exact fp32 kernel
    x = synth.activations_scaled([1e-5, 1e5, 1.0] * (m // 3) + [1e-2] * (m % 3), 2048, seed=40)
    run(kq.Q4_0, 70, 2048, x, seed=41)


@pytest.mark.parametrize("qtype", CODECS)
def test_gather_qmv_small_and_outliers(qtype):
    tokens, top_k, experts, n, k = 3, 2, 4, 200, 2048
    w = synth.weights(qtype, n, k, seed=50, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=51)
    for x in (synth.activations_scaled([1e-5, 1e-3, 1e-2, 1e-5, 1e3, 1e-1], k, seed=52),
              synth.activations_outliers(tokens * top_k, k, small=1e-3, big=1e4, per_row=2, seed=53)):
        y = torch.full((tokens * top_k, n), float("nan"), device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        kq.gather_qmv(dev_bf16(x), dev_u8(w), qtype, torch.from_numpy(ids).cuda(), out=y, err=err)
        assert int(err.item()) == 0
        ref, a = oracle.gather_qmv(qtype, w, k, x, ids, absdot=True)
        check_qmv(y.cpu().numpy(), ref, a)


@pytest.mark.parametrize("qtype", CODECS)
def test_moe_glu_gather_small_activations(qtype):
    tokens, top_k, experts, n, k = 3, 2, 5, 150, 2048
    wg = synth.weights(qtype, n, k, seed=60, experts=experts)
    wu = synth.weights(qtype, n, k, seed=61, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=62)
    x = synth.activations_scaled([1e-5, 1e-3, 1e-2], k, seed=63)
    out = kq.moe_glu_gather(dev_bf16(x), dev_u8(wg), dev_u8(wu), qtype, torch.from_numpy(ids).cuda())
    ref, g, u, ag, au = oracle.moe_glu_gather(qtype, wg, wu, k, x, ids)
    # silu(g) ~ g/2 near 0: the product of two small sums; the propagated
    # bound of the gate and up sums (each within 1e-3 * sum |x w|)
    dg, du = 1e-3 * ag, 1e-3 * au
    a = np.abs(oracle.glu(oracle.ACT_SILU, g, np.ones_like(g)))
    tol = 1.2 * dg * (np.abs(u) + du) + (a + 1.2 * dg) * du + 1e-5 * np.abs(ref) + 1e-300
    y = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(y))
    assert float(np.max(np.abs(y - ref) / tol)) <= 1.0


@pytest.mark.parametrize("qtype", CODECS)
def test_non_finite_activation_flagged(qtype):
    k = 512
    w = dev_u8(synth.weights(qtype, 16, k, seed=5))
    for bad in (np.inf, np.nan):
        x = np.zeros((1, k), np.float32)
        x[0, 3] = bad
        kq.read_device_status(clear=True)
        kq.qmv(dev_bf16(synth.f32_to_bf16_bits(x)), w, qtype)
        torch.cuda.synchronize()
        assert kq.read_device_status(clear=True) & kq.DEV_X_RANGE
    # a finite row far beyond binary16 range is not flagged
    x = np.zeros((1, k), np.float32)
    x[0, 3] = 1e30
    kq.qmv(dev_bf16(synth.f32_to_bf16_bits(x)), w, qtype)
    torch.cuda.synchronize()
    assert kq.read_device_status(clear=True) == 0
