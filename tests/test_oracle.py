"""Pins for the CPU oracle, independent of the oracle's own code.

Each test fixes a property the oracle must satisfy by a route other than the
oracle itself: hand-built blocks whose values follow from the closed form
d*sc*q - dmin*m, a full sweep of the fp16 scale field against numpy's binary16
conversion, the installed ``gguf.quants.dequantize`` library routine on random
blocks, exact rational brute force on tiny matmuls, and hand-worked tile maps
(tests/golden/).  No GPU is needed.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
Q8_0, Q4_K, Q6_K = oracle.Q8_0, oracle.Q4_K, oracle.Q6_K
Q5_K, Q4_0 = oracle.Q5_K, oracle.Q4_0


def bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


# ----------------------------------------------------------------------------
# block geometry (README "Codec reference" table)
# ----------------------------------------------------------------------------
def test_codec_table_matches_readme_and_gguf():
    import gguf
    rows = [l.split() for l in open(os.path.join(GOLDEN, "codec_table.txt")) if l[0] != "#"]
    assert len(rows) == 5
    for name, vpb, _bits, bpb, tid in rows:
        vpb, bpb, tid = int(vpb), int(bpb), int(tid)
        assert oracle.block_info(tid) == (vpb, bpb)
        assert synth.BLOCK_VALUES[tid] == vpb and synth.BLOCK_BYTES[tid] == bpb
        gt = gguf.GGMLQuantizationType(tid)
        assert gt.name.lower() == name
        assert tuple(gguf.GGML_QUANT_SIZES[gt]) == (vpb, bpb)


# ----------------------------------------------------------------------------
# fp16 scale field: every binary16 pattern, through the q8_0 decoder with q=1
# ----------------------------------------------------------------------------
def test_fp16_scale_all_patterns():
    pat = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blocks = np.zeros((65536, 34), dtype=np.uint8)
    blocks[:, 0:2] = pat.view(np.uint8).reshape(-1, 2)
    blocks[:, 2:] = 1  # every code = +1  ->  y = d * 1 = d
    y = oracle.dequantize(Q8_0, blocks.reshape(65536, 34), 32)[:, 0]
    ref = pat.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(y), nan)
    assert np.array_equal(bits(y)[~nan], bits(ref)[~nan])   # incl. subnormals and -0.0


# ----------------------------------------------------------------------------
# q4_K hand-built blocks
# ----------------------------------------------------------------------------
def q4k_block(d=1.0, dmin=0.0, scale_bytes=None, qs=None):
    b = np.zeros(144, dtype=np.uint8)
    b[0:2] = np.array([d], dtype=np.float16).view(np.uint8)
    b[2:4] = np.array([dmin], dtype=np.float16).view(np.uint8)
    if scale_bytes is not None:
        b[4:16] = scale_bytes
    if qs is not None:
        b[16:144] = qs
    return b


def test_q4k_codes_pass_through():
    # d=1, dmin=0, every 6-bit scale code 1, every min code 0: y equals the code.
    # Scale codes 0..3 are the low six bits of bytes 0..3; codes 4..7 take their
    # low four bits from the low nibbles of bytes 8..11; min codes 0..3 live in
    # bytes 4..7, min codes 4..7 in the high nibbles of bytes 8..11.
    s = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], dtype=np.uint8)
    # value 64c + l is the low nibble of qs[32c + l], 64c + 32 + l its high nibble;
    # choose both nibbles = l mod 16 so that value v carries code v mod 16.
    qs = np.array([(l % 16) | ((l % 16) << 4) for c in range(4) for l in range(32)], dtype=np.uint8)
    y = oracle.dequantize(Q4_K, q4k_block(1.0, 0.0, s, qs)[None], 256)[0]
    assert np.array_equal(y, (np.arange(256) % 16).astype(np.float32))


def _single_field(kind, j):
    """Scale bytes with exactly one 6-bit code (scale or min of sub-block j) = 63."""
    s = np.zeros(12, dtype=np.uint8)
    if kind == "sc":
        if j < 4:
            s[j] = 63
        else:
            s[j + 4] = 0x0F      # low four bits
            s[j - 4] = 0xC0      # bits 4..5 from the top two bits
    else:
        if j < 4:
            s[j + 4] = 63
        else:
            s[j + 4] = 0xF0      # low four bits from the high nibble
            s[j] = 0xC0          # bits 4..5
    return s


@pytest.mark.parametrize("kind", ["sc", "m"])
@pytest.mark.parametrize("j", range(8))
def test_q4k_single_field(kind, j):
    # d = dmin = 1, all codes q = 1: y = sc_j - m_j, so only sub-block j moves.
    blk = q4k_block(1.0, 1.0, _single_field(kind, j), np.full(128, 0x11, dtype=np.uint8))
    y = oracle.dequantize(Q4_K, blk[None], 256)[0]
    sub = np.zeros(256, dtype=np.int64)
    for v in range(256):
        sub[v] = 2 * (v // 64) + (v % 64) // 32
    expect = np.where(sub == j, 63.0 if kind == "sc" else -63.0, 0.0).astype(np.float32)
    assert np.array_equal(y, expect)


def test_q4k_min_only():
    # dmin = 1, every min code 63, every scale code 0, q = 0: y = -63 everywhere.
    s = np.zeros(12, dtype=np.uint8)
    for j in range(8):
        s = s | _single_field("m", j)
    y = oracle.dequantize(Q4_K, q4k_block(2.0, 1.0, s, np.zeros(128, np.uint8))[None], 256)[0]
    assert np.array_equal(y, np.full(256, -63.0, dtype=np.float32))


def test_q4k_scale_product_rounding():
    # y = fp32(fp32(d)*sc)*q - fp32(dmin*m): with d = 1/3 in fp16, sc = 63, q = 15
    # the two-rounding result is reproduced from numpy float32 scalars.
    s = _single_field("sc", 2) | _single_field("m", 2)
    d = np.float16(1.0 / 3.0)
    dmin = np.float16(0.1)
    blk = q4k_block(float(d), float(dmin), s, np.full(128, 0xFF, dtype=np.uint8))
    y = oracle.dequantize(Q4_K, blk[None], 256)[0]
    f = np.float32
    expect = f(f(f(d) * f(63)) * f(15)) - f(f(dmin) * f(63))
    assert bits(y[64 + 0]) == bits(expect)            # sub-block 2 = low nibbles of c = 1
    assert bits(y[0]) == bits(f(f(f(d) * f(0)) * f(15)) - f(f(dmin) * f(0)))


# ----------------------------------------------------------------------------
# q6_K hand-built blocks
# ----------------------------------------------------------------------------
def q6k_block(codes, scales, d=1.0):
    """codes: 256 ints in 0..63 placed by the q6_K layout; scales: 16 int8."""
    b = np.zeros(210, dtype=np.uint8)
    ql, qh = np.zeros(128, np.uint8), np.zeros(64, np.uint8)
    for v in range(256):
        h, t, l = v // 128, (v % 128) // 32, v % 32
        c = int(codes[v])
        ql[64 * h + 32 * (t & 1) + l] |= (c & 15) << (4 * (t >> 1))
        qh[32 * h + l] |= (c >> 4) << (2 * t)
    b[0:128], b[128:192] = ql, qh
    b[192:208] = np.asarray(scales, dtype=np.int8).view(np.uint8)
    b[208:210] = np.array([d], dtype=np.float16).view(np.uint8)
    return b


def test_q6k_all_codes():
    codes = np.arange(256) % 64
    y = oracle.dequantize(Q6_K, q6k_block(codes, np.ones(16))[None], 256)[0]
    assert np.array_equal(y, (codes - 32).astype(np.float32))     # q spans -32..31


def test_q6k_negative_scales():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 64, 256)
    scales = np.arange(16) - 8          # includes negative and zero scales
    y = oracle.dequantize(Q6_K, q6k_block(codes, scales, d=0.5)[None], 256)[0]
    expect = np.array([0.5 * scales[v // 16] * (codes[v] - 32) for v in range(256)], dtype=np.float32)
    assert np.array_equal(y, expect)


# ----------------------------------------------------------------------------
# q8_0 hand-built blocks and zero blocks
# ----------------------------------------------------------------------------
def test_q8_0_all_codes():
    b = np.zeros((8, 34), dtype=np.uint8)
    b[:, 0:2] = np.array([1.0], dtype=np.float16).view(np.uint8)
    b[:, 2:] = np.arange(256, dtype=np.uint32).astype(np.uint8).reshape(8, 32)
    y = oracle.dequantize(Q8_0, b.reshape(1, 8 * 34), 256)[0]
    assert np.array_equal(y, np.arange(256, dtype=np.uint32).astype(np.uint8).view(np.int8).astype(np.float32))


def test_zero_blocks_signed_zero():
    # q4_K and q8_0: 0*q - 0 = +0.0.  q6_K: code 0 means q = -32, (0*sc)*(-32) = -0.0.
    y4 = oracle.dequantize(Q4_K, np.zeros((1, 144), np.uint8), 256)
    y8 = oracle.dequantize(Q8_0, np.zeros((1, 34), np.uint8), 32)
    y6 = oracle.dequantize(Q6_K, np.zeros((1, 210), np.uint8), 256)
    assert np.all(bits(y4) == 0) and np.all(bits(y8) == 0)
    assert np.all(bits(y6) == 0x80000000)


# ----------------------------------------------------------------------------
# library cross-check: gguf.quants.dequantize on seeded random blocks
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("qtype", [Q4_K, Q6_K, Q8_0, Q5_K, Q4_0])
def test_matches_gguf_quants(qtype):
    import gguf
    k = 2048
    w = synth.weights(qtype, 24, k, seed=11)
    ref = gguf.quants.dequantize(w, gguf.GGMLQuantizationType(qtype)).astype(np.float32)
    y = oracle.dequantize(qtype, w, k)
    assert np.array_equal(bits(y), bits(ref))
    # fully random bytes too (any fp16 d, any int8 scale): where a scale is
    # NaN or infinite, only the position of the non-finite values is compared
    raw = np.random.default_rng(3).integers(0, 256, size=(64, synth.row_bytes(qtype, 256)), dtype=np.uint8)
    with np.errstate(invalid="ignore", over="ignore"):
        ref = gguf.quants.dequantize(raw, gguf.GGMLQuantizationType(qtype)).astype(np.float32)
    y = oracle.dequantize(qtype, raw, 256)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(y), fin)
    assert np.array_equal(bits(y)[fin], bits(ref)[fin])


# ----------------------------------------------------------------------------
# matmul: exact rational brute force and a library dot product
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("qtype,k", [(Q4_K, 256), (Q6_K, 512), (Q8_0, 256), (Q5_K, 256), (Q4_0, 256)])
def test_matmul_brute_force(qtype, k):
    import gguf
    n, m = 5, 3
    w = synth.weights(qtype, n, k, seed=21)
    x = synth.activations(m, k, seed=22)
    wd = gguf.quants.dequantize(w, gguf.GGMLQuantizationType(qtype)).astype(np.float32)
    xf = oracle.bf16_to_f32(x)
    y, a = oracle.matmul(qtype, w, k, x, absdot=True)
    for i in range(m):
        for j in range(n):
            exact = sum(Fraction(float(xf[i, t])) * Fraction(float(wd[j, t])) for t in range(k))
            aex = sum(abs(Fraction(float(xf[i, t])) * Fraction(float(wd[j, t]))) for t in range(k))
            # fp64 sequential summation error bound: k * eps * sum|terms|
            bound = k * 2.0 ** -53 * float(aex)
            assert abs(y[i, j] - float(exact)) <= bound
            assert abs(a[i, j] - float(aex)) <= bound


@pytest.mark.parametrize("qtype", [Q4_K, Q6_K, Q8_0])
def test_matmul_numpy_and_invariants(qtype):
    import gguf
    n, k, m = 37, 1024, 4
    w = synth.weights(qtype, n, k, seed=31)
    x = synth.activations(m, k, seed=32)
    wd = gguf.quants.dequantize(w, gguf.GGMLQuantizationType(qtype)).astype(np.float64)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    y = oracle.matmul(qtype, w, k, x)
    ref = xf @ wd.T
    assert np.all(np.abs(y - ref) <= 2 * k * 2.0 ** -53 * (np.abs(xf) @ np.abs(wd).T))
    # not transposed by mistake: a single nonzero activation picks one column of W
    e = np.zeros((1, k), np.float32)
    e[0, 7] = 1.0
    ye = oracle.matmul(qtype, w, k, synth.f32_to_bf16_bits(e))
    assert np.array_equal(ye[0], wd[:, 7])
    # scaling x by 2 (exact in bf16) scales y by exactly 2
    x2 = synth.f32_to_bf16_bits(2.0 * oracle.bf16_to_f32(x))
    assert np.array_equal(oracle.matmul(qtype, w, k, x2), 2.0 * y)
    # row independence: a row's result does not depend on the other rows
    y1 = oracle.matmul(qtype, w, k, x[2:3])
    assert np.array_equal(y1[0], y[2])
    # the fp32 baseline stays within fp32 summation error of the fp64 value
    y32 = oracle.matmul_f32(qtype, w, k, x)
    _, a = oracle.matmul(qtype, w, k, x, absdot=True)
    assert np.all(np.abs(y32 - y) <= (k + 1) * 2.0 ** -24 * a)


# ----------------------------------------------------------------------------
# MoE: sort, tile map (golden, hand-worked) and gather semantics
# ----------------------------------------------------------------------------
def _golden_tile_cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "tile_map_cases.txt")):
        p = line.split()
        if not p or p[0] == "#":
            continue
        if p[0] == "case":
            cur = (int(p[1]), [int(s) for s in p[2].split(",")], [])
            cases.append(cur)
        else:
            cur[2].append(tuple(int(v) for v in p[1:]))
    return cases


@pytest.mark.parametrize("case", _golden_tile_cases())
def test_tile_map_golden(case):
    n_experts, seg, expect = case
    ids = np.repeat(np.arange(n_experts), seg).astype(np.uint32)
    tiles = oracle.tile_map(ids, n_experts)
    assert sorted(tiles) == sorted(expect)
    assert len(tiles) <= oracle.map_capacity(len(ids), n_experts)


def test_moe_sort_is_stable():
    ids = np.array([[2, 0], [0, 1], [2, 1]], dtype=np.int32)   # 3 tokens, top-2
    sids, pair = oracle.moe_sort(ids, 3)
    assert sids.tolist() == [0, 0, 1, 1, 2, 2]
    assert pair.tolist() == [1, 2, 3, 5, 0, 4]                  # equal experts keep pair order
    x = np.arange(3 * 4, dtype=np.uint16).reshape(3, 4)
    xs = oracle.gather_rows(x, pair, 2)
    assert np.array_equal(xs, x[[0, 1, 1, 2, 0, 2]])


def test_routing_distinct_experts():
    r = synth.routing(512, 8, 2)
    assert r.shape == (512, 2) and np.all(r[:, 0] != r[:, 1])
    assert r.min() >= 0 and r.max() < 8


def test_gather_single_expert_equals_matmul():
    k, n, rows = 256, 16, 70
    w = synth.weights(Q4_K, n, k, seed=41, experts=1)
    x = synth.activations(rows, k, seed=42)
    ids = np.zeros(rows, np.uint32)
    tiles = oracle.tile_map(ids, 1)
    assert tiles == [(0, 0, 64), (0, 64, 6)]
    y = oracle.gather_qmm(Q4_K, w, k, x, tiles)
    assert np.array_equal(y, oracle.matmul(Q4_K, w[0], k, x))


def test_gather_uncovered_rows_unwritten():
    k, n = 256, 8
    w = synth.weights(Q8_0, n, k, seed=43, experts=2)
    x = synth.activations(10, k, seed=44)
    y = oracle.gather_qmm(Q8_0, w, k, x, [(1, 2, 3)])
    assert np.all(np.isnan(y[:2])) and np.all(np.isnan(y[5:]))
    assert np.array_equal(y[2:5], oracle.matmul(Q8_0, w[1], k, x[2:5]))


# ----------------------------------------------------------------------------
# decode MoE: gather_qmv (one output row per (token, slot) pair) and the
# unsort + score mix gather_mix
# ----------------------------------------------------------------------------
def test_gather_qmv_one_hot_picks_expert_columns():
    # Two q8_0 experts of hand-built blocks (d = 1, so W = the int8 codes) and a
    # third expert of q8_0 blocks with d = 0.5.  A one-hot activation row at
    # column c returns column c of the routed expert's matrix, so every output
    # follows from the closed form d * q without the oracle's decoder.
    n, k = 4, 64
    codes = np.arange(3 * n * k, dtype=np.int64).reshape(3, n, k) % 251 - 125
    d = [1.0, 1.0, 0.5]
    w = np.zeros((3, n, 2 * 34), dtype=np.uint8)
    for e in range(3):
        for b in range(2):
            w[e, :, 34 * b:34 * b + 2] = np.array([d[e]], dtype=np.float16).view(np.uint8)
            w[e, :, 34 * b + 2:34 * b + 34] = codes[e, :, 32 * b:32 * b + 32].astype(np.int8).view(np.uint8)
    ids = np.array([[2, 0], [1, 2], [0, 1]], dtype=np.int32)      # 3 tokens, top-2
    cols = [5, 40, 63, 0, 33, 17]                                 # one per pair
    x = np.zeros((6, k), np.float32)
    for p, c in enumerate(cols):
        x[p, c] = 1.0
    y = oracle.gather_qmv(Q8_0, w, k, synth.f32_to_bf16_bits(x), ids)
    for p, c in enumerate(cols):
        e = ids.reshape(-1)[p]
        assert np.array_equal(y[p], d[e] * codes[e, :, c].astype(np.float64))


def test_gather_qmv_reductions():
    # all pairs on one expert: the plain product; one activation row per token:
    # the per-pair product with that row repeated for every slot; a bad id
    # leaves its row unwritten
    n, k, t, top_k = 9, 512, 3, 2
    w = synth.weights(Q6_K, n, k, seed=51, experts=3)
    xp = synth.activations(t * top_k, k, seed=52)
    same = np.ones((t, top_k), np.int32)
    assert np.array_equal(oracle.gather_qmv(Q6_K, w, k, xp, same), oracle.matmul(Q6_K, w[1], k, xp))
    ids = np.array([[0, 2], [2, 1], [1, 0]], np.int32)
    xt = synth.activations(t, k, seed=53)
    a = oracle.gather_qmv(Q6_K, w, k, xt, ids, x_per_token=True)
    b = oracle.gather_qmv(Q6_K, w, k, np.repeat(xt, top_k, axis=0), ids)
    assert np.array_equal(a, b)
    bad = ids.copy()
    bad[1, 0] = 7
    yb = oracle.gather_qmv(Q6_K, w, k, xp, bad)
    assert np.all(np.isnan(yb[2])) and np.array_equal(np.delete(yb, 2, 0), np.delete(oracle.gather_qmv(Q6_K, w, k, xp, ids), 2, 0))


def test_inverse_order_and_gather_mix_unsort():
    ids = np.array([[2, 0], [0, 1], [2, 1]], dtype=np.int32)
    _, pair = oracle.moe_sort(ids, 3)
    inv = oracle.inverse_order(pair)
    assert inv.tolist() == [4, 0, 1, 2, 5, 3]                    # worked by hand from the sort above
    # top-1 with score 1: the mix is the unsort permutation, exactly
    y = np.random.default_rng(5).standard_normal((6, 8)).astype(np.float32)
    out = oracle.gather_mix(y, inv, np.ones((6, 1), np.float32))
    assert np.array_equal(out, y[inv])


def test_gather_mix_exact_values_and_order():
    # exactly representable products and sums: out[0] = 0.5*y[1] + 0.25*y[0]
    y = np.array([[4.0, -8.0], [2.0, 6.0], [1.0, 1.0]], np.float32)
    inv = np.array([1, 0, 2, 1], np.int32)                       # 2 tokens, top-2
    sc = np.array([[0.5, 0.25], [2.0, -1.0]], np.float32)
    out = oracle.gather_mix(y, inv, sc)
    assert out.tolist() == [[2.0, 1.0], [0.0, -4.0]]
    # fp32 rounding at every step, slots in ascending order: 1e8 + 1 rounds back
    # to 1e8 in fp32 (its spacing there is 8), so the result is 0, not the exact 1
    y = np.array([[1e8], [1.0], [-1e8]], np.float32)
    out = oracle.gather_mix(y, np.array([0, 1, 2], np.int32), np.ones((1, 3), np.float32))
    assert out[0, 0] == 0.0
    out = oracle.gather_mix(y, np.array([0, 2, 1], np.int32), np.ones((1, 3), np.float32))
    assert out[0, 0] == 1.0
    # a product is rounded to fp32 before it is added (no fused multiply-add):
    # (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24 rounds to 1 + 2^-11 in fp32, so adding
    # -(1 + 2^-11) gives 0 (a fused form would keep 2^-24)
    a = np.float32(1 + 2.0 ** -12)
    y = np.array([[a], [-(1 + 2.0 ** -11)]], np.float32)
    out = oracle.gather_mix(y, np.array([0, 1], np.int32), np.array([[a, 1.0]], np.float32))
    assert out[0, 0] == 0.0


def test_glu_activations():
    import math
    from scipy.special import expit
    g = np.linspace(-12, 12, 2401)
    u = np.random.default_rng(9).standard_normal(g.size)
    one = np.ones_like(g)
    # odd-part identities of both activations: a(g) - a(-g) = g
    for act in (oracle.ACT_SILU, oracle.ACT_GELU_TANH):
        assert np.allclose(oracle.glu(act, g, one) - oracle.glu(act, -g, one), g, rtol=0, atol=1e-12)
    # silu against the library logistic function
    assert np.allclose(oracle.glu(oracle.ACT_SILU, g, u), g * expit(g) * u, rtol=1e-14, atol=1e-300)
    # the tanh form stays within 1e-3 of the exact gelu g * Phi(g) (Phi from erf)
    exact = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in g])
    assert np.max(np.abs(oracle.glu(oracle.ACT_GELU_TANH, g, one) - exact)) < 1e-3
    # and it is exactly the tanh form: torch's own float64 implementation of
    # gelu(approximate="tanh") agrees to 1e-14 absolutely everywhere and to
    # 1e-12 relative where the value is not a cancellation residue of
    # 1 + tanh (|gelu| > 1e-2); a wrong constant such as 0.8 for sqrt(2/pi),
    # or 0.0447 for 0.044715, is off by more than 1e-5 absolute and 1e-3
    # relative
    import torch
    ref = torch.nn.functional.gelu(torch.from_numpy(g), approximate="tanh").numpy()
    got = oracle.glu(oracle.ACT_GELU_TANH, g, one)
    big = np.abs(ref) > 1e-2
    assert np.max(np.abs(got - ref)[big] / np.abs(ref[big])) < 1e-12
    assert np.max(np.abs(got - ref)) < 1e-14
    # two points worked by hand from the definition, to 1e-15
    for v, want in ((1.0, 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * 1.044715))),
                    (-2.0, -1.0 * (1 + math.tanh(math.sqrt(2 / math.pi) * (-2.0 - 0.35772))))):
        assert abs(float(oracle.glu(oracle.ACT_GELU_TANH, np.array([v]), np.ones(1))[0]) - want) <= 1e-15 * abs(want)
    # silu with a limit: the gate is capped from above, the up value clipped both ways
    lim = 3.0
    out = oracle.glu(oracle.ACT_SILU_LIMIT, g, 10 * u, limit=lim)
    assert np.allclose(out, oracle.glu(oracle.ACT_SILU, np.minimum(g, lim), np.clip(10 * u, -lim, lim)))
    assert np.all(np.abs(out) <= lim * lim * expit(lim) + 1e-12)


def test_moe_glu_gather_one_hot():
    # q8_0 hand blocks (d = 1): a one-hot token row returns one column of each
    # routed expert's gate and up matrix, so g and u are the int8 codes there
    n, k, e = 3, 32, 2
    gc = (np.arange(e * n * k).reshape(e, n, k) % 17 - 8).astype(np.int8)
    uc = (np.arange(e * n * k).reshape(e, n, k) % 13 - 6).astype(np.int8)
    def bank(c):
        w = np.zeros((e, n, 34), np.uint8)
        w[:, :, 0:2] = np.array([1.0], np.float16).view(np.uint8)
        w[:, :, 2:] = c.view(np.uint8)
        return w
    x = np.zeros((2, k), np.float32)
    x[0, 4] = 1.0
    x[1, 30] = 1.0
    ids = np.array([[1, 0], [0, 1]], np.int32)
    out, g, u, _, _ = oracle.moe_glu_gather(Q8_0, bank(gc), bank(uc), k, synth.f32_to_bf16_bits(x), ids)
    for p in range(4):
        t, ex, c = p // 2, ids.reshape(-1)[p], (4, 30)[p // 2]
        assert np.array_equal(g[p], gc[ex, :, c].astype(np.float64))
        assert np.array_equal(u[p], uc[ex, :, c].astype(np.float64))
        assert np.array_equal(out[p], oracle.glu(oracle.ACT_SILU, g[p], u[p]))


# ----------------------------------------------------------------------------
# encoder: float -> wire bytes
# ----------------------------------------------------------------------------
def test_float_to_half_matches_numpy():
    g = np.random.default_rng(21)
    bits32 = g.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32)
    x = bits32.view(np.float32)
    x = x[np.isfinite(x)]
    # ties: binary16 midpoints in every binade, subnormal range, overflow edge
    h = np.arange(0, 0x7c00, 7, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float32)
    hi = (h + 1).view(np.float16).astype(np.float32)
    ties = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    edge = np.array([65504, 65519.99, 65520, 65536, 1e-8, 2.0**-24, 2.0**-25, 3 * 2.0**-26, 0.0, -0.0],
                    np.float32)
    for v in (x, ties, -ties, edge, -edge):
        with np.errstate(over="ignore"):
            ref = v.astype(np.float16).view(np.uint16)
        assert np.array_equal(oracle.float_to_half_bits(v), ref)


def test_quantize_q8_0_matches_gguf():
    import gguf
    g = np.random.default_rng(22)
    w = (g.standard_normal((40, 512)) * g.uniform(1e-3, 10, (40, 1))).astype(np.float32)
    w[3, :32] = 0.0                                     # an all-zero block
    w[4, :32] = np.arange(32) - 15.5                    # x * (1/d) lands on halves
    w[5, 32:64] = 127.0 * np.sign(np.arange(32) - 16)   # codes at the extremes
    ref = gguf.quants.quantize(w, gguf.GGMLQuantizationType.Q8_0)
    assert np.array_equal(oracle.quantize(Q8_0, w), ref)


def _canonical_q4k(g, nblk):
    """q4_K blocks that the encoder must reproduce exactly: d = 2^-8,
    dmin = 2^-9, 6-bit codes with 63 present, every sub-block using codes 0
    and 15 (so its range is exactly 15 d sc_j and its min exactly -dmin m_j)."""
    blocks = np.zeros((nblk, 144), np.uint8)
    for b in range(nblk):
        sc = g.integers(1, 64, 8)
        m = g.integers(0, 64, 8)
        sc[g.integers(8)] = 63
        m[g.integers(8)] = 63
        q = g.integers(0, 16, 256)
        for j in range(8):
            pos = g.choice(32, 2, replace=False)
            q[32 * j + pos[0]], q[32 * j + pos[1]] = 0, 15
        blk = blocks[b]
        blk[0:2] = np.array([2.0 ** -8], np.float16).view(np.uint8)
        blk[2:4] = np.array([2.0 ** -9], np.float16).view(np.uint8)
        s = blk[4:16]
        for j in range(4):                              # the layout the decoder reads
            s[j] = sc[j] | ((sc[j + 4] >> 4) << 6)
            s[j + 4] = m[j] | ((m[j + 4] >> 4) << 6)
            s[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
        for c in range(4):
            for l in range(32):
                blk[16 + 32 * c + l] = q[64 * c + l] | (q[64 * c + 32 + l] << 4)
    return blocks


def _canonical_q6k(g, nblk):
    """q6_K blocks the encoder must reproduce exactly: d = 2^-10, int8 scales
    in 1..127 with 127 present, codes q in -31..31 with +-31 in every
    sub-block (so max|x| is exactly 31 d sc_j)."""
    blocks = np.zeros((nblk, 210), np.uint8)
    for b in range(nblk):
        sc = g.integers(1, 128, 16)
        sc[g.integers(16)] = 127
        q = g.integers(-31, 32, 256)
        for j in range(16):
            q[16 * j + g.integers(16)] = 31 if g.integers(2) else -31
        c = q + 32
        blk = blocks[b]
        for v in range(256):
            h, t, l = v // 128, (v % 128) // 32, v % 32
            blk[64 * h + l + 32 * (t & 1)] |= (c[v] & 15) << (4 * (t >> 1))
            blk[128 + 32 * h + l] |= (c[v] >> 4) << (2 * t)
        blk[192:208] = sc.astype(np.int8).view(np.uint8)
        blk[208:210] = np.array([2.0 ** -10], np.float16).view(np.uint8)
    return blocks


@pytest.mark.parametrize("qtype", [Q4_K, Q6_K])
def test_quantize_reproduces_canonical_blocks(qtype):
    g = np.random.default_rng(23)
    blocks = (_canonical_q4k if qtype == Q4_K else _canonical_q6k)(g, 24)
    x = oracle.dequantize(qtype, blocks.reshape(1, -1), 24 * 256)
    assert np.array_equal(oracle.quantize(qtype, x).reshape(24, -1), blocks)


def test_quantize_zero_blocks():
    z = np.zeros((1, 256), np.float32)
    assert np.all(oracle.quantize(Q4_K, z) == 0)
    assert np.all(oracle.quantize(Q8_0, z) == 0)
    # q6_K: d = 0 and scales 0, every code q = 0 stored as 32 = 0b10_0000: low
    # nibbles 0, each 2-bit high field 2, so every qh byte is 0b10101010
    b = oracle.quantize(Q6_K, z)[0]
    assert np.all(b[:128] == 0) and np.all(b[128:192] == 0xAA) and np.all(b[192:] == 0)


@pytest.mark.parametrize("qtype", [Q4_K, Q6_K, Q8_0])
def test_quantize_round_trip_bound(qtype):
    # per-value error of decode(encode(x)) within the bound that follows from
    # the sub-block range and the binary16 super-block scales, computed from x
    # alone; and at most a few per cent of values beyond half a quantization
    # step (only values clipped at the top of a sub-block's range)
    g = np.random.default_rng(24)
    x = (g.standard_normal((16, 1024)) * g.uniform(1e-2, 3, (16, 1))).astype(np.float32)
    y = oracle.dequantize(qtype, oracle.quantize(qtype, x), 1024).astype(np.float64)
    err = np.abs(y - x)
    xs = x.astype(np.float64)
    eps = 1e-6 * np.abs(xs).max()
    if qtype == Q8_0:
        a = np.abs(xs.reshape(-1, 32)).max(axis=1, keepdims=True)
        assert np.all(err.reshape(-1, 32) <= a / 254 * (1 + 2.0 ** -10) + a * 2.0 ** -11 + eps)
        return
    sb = xs.reshape(-1, 256)
    if qtype == Q4_K:
        sub = sb.reshape(-1, 8, 32)
        lo, hi = np.minimum(sub.min(axis=2), 0), sub.max(axis=2)
        s = (hi - lo) / 15
        df = s.max(axis=1, keepdims=True) / 63 * (1 + 2.0 ** -10)
        dmf = (-lo).max(axis=1, keepdims=True) / 63 * (1 + 2.0 ** -10)
        half = s / 2 + df / 4
        bound = half + 7.5 * df + dmf / 2
        e = err.reshape(-1, 8, 32)
    else:
        sub = sb.reshape(-1, 16, 16)
        s = np.abs(sub).max(axis=2) / 31
        df = s.max(axis=1, keepdims=True) / 127 * (1 + 2.0 ** -10)
        half = s / 2 + df / 4
        bound = half + 15.5 * df
        e = err.reshape(-1, 16, 16)
    assert np.all(e <= bound[..., None] + eps)
    assert np.mean(e > half[..., None] + eps) < 0.05



# ----------------------------------------------------------------------------
# q5_K and q4_0 hand-built blocks
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("bit", range(8))
def test_q5k_high_bit(bit):
    # d = 1, dmin = 0, every scale code 1, every nibble 0, qh bytes with only
    # bit `bit` set: sub-block `bit` reads 16 everywhere, every other value 0
    b = np.zeros(176, np.uint8)
    b[0:2] = np.array([1.0], np.float16).view(np.uint8)
    b[4:16] = [1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1]
    b[16:48] = 1 << bit
    y = oracle.dequantize(Q5_K, b[None], 256)[0]
    sub = np.array([2 * (v // 64) + (v % 64) // 32 for v in range(256)])
    assert np.array_equal(y, np.where(sub == bit, 16.0, 0.0).astype(np.float32))


def test_q5k_codes_and_min():
    # nibbles l mod 16 in both halves, high bits all set, d = 1, dmin = 1,
    # scale codes 1, min codes 3: y = (code + 16) - 3
    b = np.zeros(176, np.uint8)
    b[0:4] = np.array([1.0, 1.0], np.float16).view(np.uint8)
    b[4:16] = [1, 1, 1, 1, 3, 3, 3, 3, 0x31, 0x31, 0x31, 0x31]
    b[16:48] = 0xFF
    b[48:176] = [(l % 16) | ((l % 16) << 4) for c in range(4) for l in range(32)]
    y = oracle.dequantize(Q5_K, b[None], 256)[0]
    assert np.array_equal(y, (np.arange(256) % 16 + 16 - 3).astype(np.float32))


def test_q4_0_all_codes():
    b = np.zeros((1, 18), np.uint8)
    b[0, 0:2] = np.array([0.5], np.float16).view(np.uint8)
    b[0, 2:] = [l | ((15 - l) << 4) for l in range(16)]
    y = oracle.dequantize(Q4_0, b, 32)[0]
    expect = np.concatenate([np.arange(16) - 8, (15 - np.arange(16)) - 8]) * 0.5
    assert np.array_equal(y, expect.astype(np.float32))
