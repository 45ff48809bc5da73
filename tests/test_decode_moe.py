"""Decode MoE on the GPU vs the CPU oracle: gather_qmv (one output row per
(token, slot) pair; qmv tolerance), the inverse sort order (exact) and the
unsort + score mix gather_mix (bit-exact: both sides round each fp32 product
and sum in slot order)."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmv, dev_bf16, dev_u8

pytestmark = pytest.mark.gpu


def run_gather_qmv(qtype, w, k, x, ids, x_per_token=False):
    n = w.shape[1]
    out = torch.full((ids.size, n), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.gather_qmv(dev_bf16(x), dev_u8(w), qtype, torch.from_numpy(ids.astype(np.int32)).cuda(),
                  x_per_token=x_per_token, out=out, err=err)
    return out.cpu().numpy(), int(err.item())


def check_pairs(qtype, w, k, x, ids, y, x_per_token=False, rows=None):
    ref, a = oracle.gather_qmv(qtype, w, k, x, ids, x_per_token=x_per_token, absdot=True)
    rows = np.arange(ids.size) if rows is None else rows
    check_qmv(y[rows], ref[rows], a[rows])


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0, kq.Q5_K, kq.Q4_0])
@pytest.mark.parametrize("tokens,top_k,experts,n", [(1, 2, 8, 300), (3, 4, 5, 1000), (16, 2, 4, 520)])
def test_gather_qmv_vs_oracle(qtype, tokens, top_k, experts, n):
    k = 2048
    w = synth.weights(qtype, n, k, seed=tokens, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=tokens + 1)
    x = synth.activations(tokens * top_k, k, seed=tokens + 2)
    y, e = run_gather_qmv(qtype, w, k, x, ids)
    assert e == 0
    check_pairs(qtype, w, k, x, ids, y)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q8_0, kq.Q5_K, kq.Q4_0])
def test_gather_qmv_x_per_token(qtype):
    tokens, top_k, experts, n, k = 4, 2, 6, 257, 4096
    w = synth.weights(qtype, n, k, seed=61, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=62)
    x = synth.activations(tokens, k, seed=63)
    y, e = run_gather_qmv(qtype, w, k, x, ids, x_per_token=True)
    assert e == 0
    check_pairs(qtype, w, k, x, ids, y, x_per_token=True)


@pytest.mark.parametrize("qtype", [kq.Q6_K, kq.Q4_K, kq.Q4_0, kq.Q5_K])
def test_gather_qmv_crowded_expert_and_repeated_ids(qtype):
    # five tokens all route slot 0 to expert 1 (more pairs than one batch of
    # the q6_K kernel), token 2 names expert 3 twice
    tokens, top_k, experts, n, k = 5, 2, 4, 200, 2048
    ids = np.array([[1, 0], [1, 2], [1, 3], [1, 3], [1, 1]], np.int32)
    ids[2] = [3, 3]
    w = synth.weights(qtype, n, k, seed=71, experts=experts)
    x = synth.activations(tokens * top_k, k, seed=72)
    y, e = run_gather_qmv(qtype, w, k, x, ids)
    assert e == 0
    check_pairs(qtype, w, k, x, ids, y)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q8_0])
def test_gather_qmv_many_pairs(qtype):
    # 512 pairs over 64 experts: q4_K forms ~64 virtual experts of up to 16
    # pairs (2 CTAs and several row groups each), q8_0 ~256 of up to 2 pairs,
    # more than one launch of 148 CTAs holds
    tokens, top_k, experts, n, k = 64, 8, 64, 192, 2048
    w = synth.weights(qtype, n, k, seed=81, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=82)
    x = synth.activations(tokens * top_k, k, seed=83)
    y, e = run_gather_qmv(qtype, w, k, x, ids)
    assert e == 0
    check_pairs(qtype, w, k, x, ids, y)


def test_gather_qmv_bad_id_flagged_row_unwritten():
    tokens, top_k, experts, n, k = 2, 2, 3, 64, 2048
    ids = np.array([[0, 2], [5, 1]], np.int32)
    w = synth.weights(kq.Q8_0, n, k, seed=91, experts=experts)
    x = synth.activations(4, k, seed=92)
    y, e = run_gather_qmv(kq.Q8_0, w, k, x, ids)
    assert e & kq.DEV_BAD_EXPERT
    assert np.all(np.isnan(y[2]))
    check_pairs(kq.Q8_0, w, k, x, ids, y, rows=np.array([0, 1, 3]))


def test_gather_qmv_full_bank_sampled():
    # the prefill MoE bank (8 experts x 14336 x 4096 q4_K), 4 decode tokens
    # routed top-2 with one activation row per token; all rows of 8 sampled
    # columns and 2 full pairs
    experts, n, k, tokens, top_k = 8, 14336, 4096, 4, 2
    w = synth.weights(kq.Q4_K, n, k, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=5)
    x = synth.activations(tokens, k, seed=6)
    y, e = run_gather_qmv(kq.Q4_K, w, k, x, ids, x_per_token=True)
    assert e == 0
    g = np.random.default_rng(7)
    cols = np.sort(g.choice(n, 8, replace=False))
    ref, a = oracle.gather_qmv(kq.Q4_K, w[:, cols], k, x, ids, x_per_token=True, absdot=True)
    check_qmv(y[:, cols], ref, a)
    for p in (0, 7):
        e_p = int(ids.reshape(-1)[p])
        ref, a = oracle.matmul(kq.Q4_K, w[e_p], k, x[p // top_k:p // top_k + 1], absdot=True)
        check_qmv(y[p:p + 1], ref, a)


@pytest.mark.parametrize("tokens,experts,top_k", [(512, 8, 2), (37, 5, 3), (1, 4, 1)])
def test_inverse_order_exact(tokens, experts, top_k):
    ids = synth.routing(tokens, experts, top_k, seed=tokens)
    _, pair, _, inv = kq.moe_sort(torch.from_numpy(ids).cuda(), experts, with_inverse=True)
    _, ref_pair = oracle.moe_sort(ids, experts)
    assert np.array_equal(pair.cpu().numpy(), ref_pair)
    assert np.array_equal(inv.cpu().numpy(), oracle.inverse_order(ref_pair))


@pytest.mark.parametrize("tokens,top_k,n", [(512, 2, 14336), (37, 3, 260), (1, 8, 4)])
def test_gather_mix_bit_exact(tokens, top_k, n):
    experts = 8
    ids = synth.routing(tokens, experts, top_k, seed=3)
    g = np.random.default_rng(tokens)
    y = g.standard_normal((tokens * top_k, n)).astype(np.float32)
    sc = g.random((tokens, top_k)).astype(np.float32)
    _, pair, _, inv = kq.moe_sort(torch.from_numpy(ids).cuda(), experts, with_inverse=True)
    out = kq.gather_mix(torch.from_numpy(y).cuda(), inv, torch.from_numpy(sc).cuda()).cpu().numpy()
    ref = oracle.gather_mix(y, oracle.inverse_order(oracle.moe_sort(ids, experts)[1]), sc)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_gather_mix_bad_entry_flagged_and_skipped():
    y = np.arange(12, dtype=np.float32).reshape(3, 4)
    inv = np.array([0, 9, 2, 1], np.int32)                   # 9 is past the 3 rows of y
    sc = np.array([[1.0, 5.0], [0.5, 2.0]], np.float32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kq.gather_mix(torch.from_numpy(y).cuda(), torch.from_numpy(inv).cuda(), torch.from_numpy(sc).cuda(),
                        err=err).cpu().numpy()
    assert int(err.item()) & kq.DEV_BAD_RANGE
    assert np.array_equal(out[0], y[0])
    assert np.array_equal(out[1], oracle.gather_mix(y, inv[2:], sc[1:])[0])


def test_prefill_moe_end_to_end_mix():
    # sort -> tile map -> gather_qmm -> gather_mix: the mix of the GPU's expert
    # outputs equals the oracle's mix of the same outputs bit for bit
    experts, n, k, tokens, top_k = 4, 128, 1024, 40, 2
    w = synth.weights(kq.Q4_K, n, k, experts=experts, seed=13)
    x = synth.activations(tokens, k, seed=14)
    ids = synth.routing(tokens, experts, top_k, seed=15)
    sc = np.random.default_rng(16).random((tokens, top_k)).astype(np.float32)
    sids, pair, xs, inv = kq.moe_sort(torch.from_numpy(ids).cuda(), experts, dev_bf16(x), with_inverse=True)
    m, c = kq.expert_tile_map(sids, experts)
    y = kq.gather_qmm(xs, dev_u8(w), kq.Q4_K, m, c)
    out = kq.gather_mix(y, inv, torch.from_numpy(sc).cuda()).cpu().numpy()
    ref = oracle.gather_mix(y.cpu().numpy(), inv.cpu().numpy(), sc)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def check_glu(y, out, g, u, ag, au, act):
    """|y - out| within the propagated qmv bound: the gate and up sums each
    carry at most 1e-3 * sum|x w|, and act is 1.2-Lipschitz in g (silu, gelu
    and their limited forms) and linear in u; plus fp32 rounding of act."""
    dg, du = 1e-3 * ag, 1e-3 * au
    a = np.abs(oracle.glu(act, g, np.ones_like(g), limit=4.0))
    tol = 1.2 * dg * (np.abs(u) + du) + (a + 1.2 * dg) * du + 1e-5 * np.abs(out) + 1e-30
    err = np.abs(y.astype(np.float64) - out)
    assert np.all(np.isfinite(y))
    worst = float(np.max(err / tol))
    assert worst <= 1.0, f"error / bound = {worst:.3f}"


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0, kq.Q5_K, kq.Q4_0])
@pytest.mark.parametrize("act", [kq.ACT_SILU, kq.ACT_GELU_TANH, kq.ACT_SILU_LIMIT])
@pytest.mark.parametrize("tokens", [1, 3])
def test_moe_glu_gather_vs_oracle(qtype, act, tokens):
    # one token: every virtual expert has one activation row (the q4_K / q5_K
    # column form); three: batched rows
    top_k, experts, n, k = 2, 5, 333, 2048
    wg = synth.weights(qtype, n, k, seed=101, experts=experts)
    wu = synth.weights(qtype, n, k, seed=102, experts=experts)
    ids = synth.routing(tokens, experts, top_k, seed=103)
    x = synth.activations(tokens, k, seed=104)
    # scale x so that the products reach the region where the activations bend
    x = synth.f32_to_bf16_bits(oracle.bf16_to_f32(x) * 40.0)
    out = torch.full((tokens * top_k, n), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.moe_glu_gather(dev_bf16(x), dev_u8(wg), dev_u8(wu), qtype, torch.from_numpy(ids).cuda(), act=act, limit=4.0,
                      out=out, err=err)
    assert int(err.item()) == 0
    ref, g, u, ag, au = oracle.moe_glu_gather(qtype, wg, wu, k, x, ids, act=act, limit=4.0)
    assert np.mean(np.abs(g) > 1.0) > 0.2          # the activations are exercised off their linear part
    check_glu(out.cpu().numpy(), ref, g, u, ag, au, act)


def test_moe_glu_gather_full_bank_sampled():
    experts, n, k, tokens, top_k = 8, 14336, 4096, 4, 2
    wg = synth.weights(kq.Q4_K, n, k, experts=experts, seed=0)
    wu = synth.weights(kq.Q4_K, n, k, experts=experts, seed=1)
    ids = synth.routing(tokens, experts, top_k, seed=5)
    x = synth.activations(tokens, k, seed=6)
    y = kq.moe_glu_gather(dev_bf16(x), dev_u8(wg), dev_u8(wu), kq.Q4_K, torch.from_numpy(ids).cuda()).cpu().numpy()
    cols = np.sort(np.random.default_rng(8).choice(n, 16, replace=False))
    ref, g, u, ag, au = oracle.moe_glu_gather(kq.Q4_K, wg[:, cols], wu[:, cols], k, x, ids)
    check_glu(y[:, cols], ref, g, u, ag, au, kq.ACT_SILU)


def test_equal_length_banks_and_expert_slices():
    # q4_K and q4_0 rows of K values are equally long (K/32 * 18 bytes): one
    # buffer refilled with either codec's bytes is decoded as the codec the
    # call names (the library keeps no state per weight pointer), and a slice
    # of whole experts of a bank (an offset pointer) is the bank it views
    tokens, top_k, experts, n, k = 1, 2, 8, 300, 2048
    assert kq.row_bytes(kq.Q4_K, k) == kq.row_bytes(kq.Q4_0, k)
    ids = synth.routing(tokens, experts, top_k, seed=2)
    x = synth.activations(tokens * top_k, k, seed=3)
    buf = torch.empty(experts, n, kq.row_bytes(kq.Q4_K, k), dtype=torch.uint8, device="cuda")

    def run(qtype, bank, rid):
        out = torch.full((tokens * top_k, n), float("nan"), device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        kq.gather_qmv(dev_bf16(x), bank, qtype, torch.from_numpy(rid).cuda(), out=out, err=err)
        return out.cpu().numpy(), int(err.item())

    for qtype, seed in ((kq.Q4_K, 1), (kq.Q4_0, 1), (kq.Q4_K, 4)):
        w = synth.weights(qtype, n, k, seed=seed, experts=experts)
        buf.copy_(torch.from_numpy(w))
        y, e = run(qtype, buf, ids)
        assert e == 0
        check_pairs(qtype, w, k, x, ids, y)
    # experts 3..7 of the last bank's buffer
    sub = synth.routing(tokens, experts - 3, top_k, seed=5)
    y, e = run(kq.Q4_K, buf[3:], sub)
    assert e == 0
    check_pairs(kq.Q4_K, w[3:], k, x, sub, y)


def test_decode_moe_edge_cases():
    # one pair; zero tokens (nothing enqueued); top-8 mix over the smallest N
    w = synth.weights(kq.Q4_K, 64, 256, seed=1, experts=2)
    x = synth.activations(1, 256, seed=2)
    ids = np.array([[1]], np.int32)
    y, e = run_gather_qmv(kq.Q4_K, w, 256, x, ids)
    assert e == 0
    check_pairs(kq.Q4_K, w, 256, x, ids, y)
    empty = torch.empty(0, 2, dtype=torch.int32, device="cuda")
    out = kq.gather_qmv(dev_bf16(x), dev_u8(w), kq.Q4_K, empty)
    assert out.shape == (0, 64)
    g = np.random.default_rng(3)
    yv = g.standard_normal((24, 4)).astype(np.float32)
    inv = g.permutation(24).astype(np.int32)
    sc = g.random((3, 8)).astype(np.float32)
    o = kq.gather_mix(torch.from_numpy(yv).cuda(), torch.from_numpy(inv).cuda(), torch.from_numpy(sc).cuda())
    ref = oracle.gather_mix(yv, inv, sc)
    assert np.array_equal(o.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("k,n", [(768, 201), (11008, 257)])
def test_gather_qmv_q6K_rows_not_16_byte_multiple(k, n):
    # q6_K rows of 630 / 9030 bytes: staged from the 16-byte boundary below
    # each row and decoded at the row's own offset; the bank's size is not a
    # multiple of 16 either, so its last row ends past the last 16-byte
    # boundary (every expert is routed, the last one included)
    tokens, top_k, experts = 4, 2, 4
    assert synth.row_bytes(kq.Q6_K, k) % 16 != 0 and (experts * n * synth.row_bytes(kq.Q6_K, k)) % 16 != 0
    w = synth.weights(kq.Q6_K, n, k, seed=k, experts=experts)
    ids = np.array([[0, 3], [1, 2], [3, 1], [2, 0]], np.int32)
    x = synth.activations(tokens * top_k, k, seed=k + 1)
    y, e = run_gather_qmv(kq.Q6_K, w, k, x, ids)
    assert e == 0
    check_pairs(kq.Q6_K, w, k, x, ids, y)
    xt = synth.activations(tokens, k, seed=k + 2)
    y, e = run_gather_qmv(kq.Q6_K, w, k, xt, ids, x_per_token=True)
    assert e == 0
    check_pairs(kq.Q6_K, w, k, xt, ids, y, x_per_token=True)


def test_moe_glu_gather_q6K_k11008():
    tokens, top_k, experts, n, k = 3, 2, 4, 129, 11008
    wg = synth.weights(kq.Q6_K, n, k, seed=111, experts=experts)
    wu = synth.weights(kq.Q6_K, n, k, seed=112, experts=experts)
    ids = np.array([[3, 0], [1, 3], [2, 1]], np.int32)
    x = synth.activations(tokens, k, seed=113)
    out = kq.moe_glu_gather(dev_bf16(x), dev_u8(wg), dev_u8(wu), kq.Q6_K, torch.from_numpy(ids).cuda())
    ref, g, u, ag, au = oracle.moe_glu_gather(kq.Q6_K, wg, wu, k, x, ids)
    check_glu(out.cpu().numpy(), ref, g, u, ag, au, kq.ACT_SILU)
