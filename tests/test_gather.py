"""MoE path on the GPU vs the CPU oracle: stable expert sort (exact), tile map
(exact, compared as a set), segment gather GEMM (qmm tolerance), data errors
flagged without faults, uncovered rows left unwritten."""
import numpy as np
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq
import oracle
import synth
from tests._util import check_qmm, dev_bf16, dev_u8, row_norms_w, row_norms_x

pytestmark = pytest.mark.gpu


def tiles_of(m, c):
    m = m.cpu().numpy().astype(np.int64)
    c = int(c.cpu().numpy()[0])
    return [tuple(int(v) for v in m[i]) for i in range(c)]


@pytest.mark.parametrize("tokens,experts,top_k", [(512, 8, 2), (37, 5, 3), (1, 4, 1), (3000, 64, 4)])
def test_sort_and_tile_map_exact(tokens, experts, top_k):
    ids = synth.routing(tokens, experts, top_k, seed=tokens)
    k = 64
    x = synth.activations(tokens, k, seed=1)
    sids, pair, xs = kq.moe_sort(torch.from_numpy(ids).cuda(), experts, dev_bf16(x))
    ref_ids, ref_pair = oracle.moe_sort(ids, experts)
    assert np.array_equal(sids.cpu().numpy().view(np.uint32), ref_ids)
    assert np.array_equal(pair.cpu().numpy(), ref_pair)
    assert np.array_equal(xs.view(torch.int16).cpu().numpy().view(np.uint16), oracle.gather_rows(x, ref_pair, top_k))
    m, c = kq.expert_tile_map(sids, experts)
    assert sorted(tiles_of(m, c)) == sorted(oracle.tile_map(ref_ids, experts))


def test_tile_map_golden_segments():
    seg = [0, 1, 64, 65, 0, 129, 63, 0]
    ids = np.repeat(np.arange(len(seg)), seg).astype(np.uint32)
    m, c = kq.expert_tile_map(torch.from_numpy(ids.view(np.int32)).cuda(), len(seg))
    assert sorted(tiles_of(m, c)) == sorted(oracle.tile_map(ids, len(seg)))


def test_tile_map_flags_bad_ids():
    ids = np.array([0, 2, 1, 9], dtype=np.int32)           # unsorted and out of range
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.expert_tile_map(torch.from_numpy(ids).cuda(), 4, err=err)
    e = int(err.item())
    assert e & kq.DEV_UNSORTED and e & kq.DEV_BAD_EXPERT


def run_gather(qtype, experts, n, k, tiles, rows, seed=0):
    w = synth.weights(qtype, n, k, seed=seed, experts=experts)
    x = synth.activations(rows, k, seed=seed + 1)
    tm = torch.tensor(np.array(tiles, dtype=np.int64).reshape(-1, 3), dtype=torch.int32).cuda()
    cnt = torch.tensor([len(tiles)], dtype=torch.int32).cuda()
    out = torch.full((rows, n), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kq.gather_qmm(dev_bf16(x), dev_u8(w), qtype, tm, cnt, out=out, err=err)
    y = out.cpu().numpy()
    return w, x, y, int(err.item())


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q6_K, kq.Q8_0])
def test_gather_vs_oracle(qtype):
    experts, n, k = 5, 200, 2048
    ids = np.sort(np.random.default_rng(3).integers(0, experts, 700)).astype(np.uint32)
    ids = ids[ids != 2]                                     # an expert with no rows
    tiles = oracle.tile_map(ids, experts)
    rng = np.random.default_rng(4)
    tiles = [tiles[i] for i in rng.permutation(len(tiles))]  # tile order is unspecified
    w, x, y, e = run_gather(qtype, experts, n, k, tiles, len(ids), seed=5)
    assert e == 0
    ref = oracle.gather_qmm(qtype, w, k, x, tiles)
    wn = np.stack([row_norms_w(qtype, w[i], k) for i in range(experts)])
    xn = row_norms_x(x)
    for ex in range(experts):
        r = np.nonzero(ids == ex)[0]
        if r.size:
            check_qmm(y[r], ref[r], xn[r], wn[ex], k)


def test_gather_many_tiles_per_expert_and_single_expert_equals_qmm():
    n, k, rows = 130, 2048, 700                               # 11 tiles for one expert
    ids = np.zeros(rows, np.uint32)
    tiles = oracle.tile_map(ids, 1)
    w, x, y, e = run_gather(kq.Q4_K, 1, n, k, tiles, rows, seed=7)
    assert e == 0
    yq = kq.qmm(dev_bf16(x), dev_u8(w[0]), kq.Q4_K).cpu().numpy()
    ref = oracle.matmul(kq.Q4_K, w[0], k, x)
    check_qmm(y, ref, row_norms_x(x), row_norms_w(kq.Q4_K, w[0], k), k)
    check_qmm(yq, ref, row_norms_x(x), row_norms_w(kq.Q4_K, w[0], k), k)


def test_gather_bad_tiles_skipped_and_uncovered_rows_unwritten():
    n, k, rows = 128, 256, 200
    tiles = [(0, 0, 64), (5, 64, 10), (1, 64, 0), (1, 70, 65), (1, 190, 20), (1, 100, 30)]
    w, x, y, e = run_gather(kq.Q4_K, 2, n, k, tiles, rows, seed=9)
    assert e & kq.DEV_BAD_EXPERT and e & kq.DEV_BAD_ROWS and e & kq.DEV_BAD_RANGE
    assert np.all(np.isnan(y[64:100])) and np.all(np.isnan(y[130:]))   # never written
    ref = oracle.gather_qmm(kq.Q4_K, w, k, x, [(0, 0, 64), (1, 100, 30)])
    check_qmm(y[:64], ref[:64], row_norms_x(x[:64]), row_norms_w(kq.Q4_K, w[0], k), k)
    check_qmm(y[100:130], ref[100:130], row_norms_x(x[100:130]), row_norms_w(kq.Q4_K, w[1], k), k)


def test_c4_full_size_sampled():
    experts, n, k, tokens, top_k = 8, 14336, 4096, 512, 2
    w = synth.weights(kq.Q4_K, n, k, experts=experts)
    x = synth.activations(tokens, k)
    ids = synth.routing(tokens, experts, top_k)
    sids, pair, xs = kq.moe_sort(torch.from_numpy(ids).cuda(), experts, dev_bf16(x))
    m, c = kq.expert_tile_map(sids, experts)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = kq.gather_qmm(xs, dev_u8(w), kq.Q4_K, m, c, err=err).cpu().numpy()
    assert int(err.item()) == 0
    ref_ids, ref_pair = oracle.moe_sort(ids, experts)
    xs_ref = oracle.gather_rows(x, ref_pair, top_k)
    g = np.random.default_rng(77)
    rows = np.sort(g.choice(tokens * top_k, 32, replace=False))
    cols = np.sort(g.choice(n, 32, replace=False))
    xn = row_norms_x(xs_ref)
    for r in rows:
        e = int(ref_ids[r])
        ref = oracle.matmul(kq.Q4_K, w[e], k, xs_ref[r:r + 1])
        check_qmm(y[r:r + 1], ref, xn[r:r + 1], row_norms_w(kq.Q4_K, w[e], k), k)
    for e in range(experts):
        rr = np.nonzero(ref_ids == e)[0]
        ref = oracle.matmul(kq.Q4_K, w[e][cols], k, xs_ref[rr])
        check_qmm(y[rr][:, cols], ref, xn[rr], row_norms_w(kq.Q4_K, w[e][cols], k), k)


@pytest.mark.parametrize("qtype", [kq.Q4_K, kq.Q8_0])
def test_gather_row_runs_and_split_tiles(qtype):
    # expert 0: one run of 202 rows over four tiles; expert 1: a 5-row run (the
    # second CTA of a pair then holds no row); expert 2: two tiles that are not
    # adjacent (rows 271..279 belong to no tile and stay unwritten)
    n, k, rows = 300, 1024, 300
    tiles = [(0, 0, 64), (0, 64, 64), (0, 128, 64), (0, 192, 10), (1, 202, 5), (2, 207, 64), (2, 280, 20)]
    w, x, y, e = run_gather(qtype, 3, n, k, tiles[::-1], rows, seed=11)
    assert e == 0
    assert np.all(np.isnan(y[271:280]))
    ref = oracle.gather_qmm(qtype, w, k, x, tiles)
    xn = row_norms_x(x)
    for ex, (lo, hi) in enumerate([(0, 202), (202, 207), (207, 300)]):
        r = np.array([i for i in range(lo, hi) if not 271 <= i < 280])
        check_qmm(y[r], ref[r], xn[r], row_norms_w(qtype, w[ex], k), k)


@pytest.mark.parametrize("shuffle", [False, True])
def test_gather_more_than_1024_tiles(shuffle):
    # 70 000 sorted rows over 3 experts: 1096 map tiles, more than one launch
    # window of 1024 map slots; the device-built map (grouped by expert, rows
    # in order) and the same tiles shuffled; every row against the oracle, no
    # flag raised
    experts, n, k, rows = 3, 64, 256, 70000
    ids = np.repeat(np.arange(experts), [30001, 25000, 14999]).astype(np.uint32)
    if shuffle:
        tiles = oracle.tile_map(ids, experts)
        assert len(tiles) > 1024
        tiles = [tiles[i] for i in np.random.default_rng(21).permutation(len(tiles))]
        w, x, y, e = run_gather(kq.Q4_K, experts, n, k, tiles, rows, seed=20)
    else:
        w = synth.weights(kq.Q4_K, n, k, seed=20, experts=experts)
        x = synth.activations(rows, k, seed=21)
        m, c = kq.expert_tile_map(torch.from_numpy(ids.view(np.int32)).cuda(), experts)
        tiles = tiles_of(m, c)
        assert len(tiles) > 1024
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full((rows, n), float("nan"), device="cuda")
        kq.gather_qmm(dev_bf16(x), dev_u8(w), kq.Q4_K, m, c, out=out, err=err)
        y, e = out.cpu().numpy(), int(err.item())
    assert e == 0
    assert np.all(np.isfinite(y))
    ref = oracle.gather_qmm(kq.Q4_K, w, k, x, tiles)
    xn = row_norms_x(x)
    for ex in range(experts):
        r = np.nonzero(ids == ex)[0]
        check_qmm(y[r], ref[r], xn[r], row_norms_w(kq.Q4_K, w[ex], k), k)


def test_gather_q6K_rows_not_16_byte_multiple():
    # K = 11008: 9030-byte rows; three experts' segments through the flat view
    experts, n, k = 3, 200, 11008
    ids = np.sort(np.random.default_rng(31).integers(0, experts, 300)).astype(np.uint32)
    tiles = oracle.tile_map(ids, experts)
    w, x, y, e = run_gather(kq.Q6_K, experts, n, k, tiles, len(ids), seed=32)
    assert e == 0
    ref = oracle.gather_qmm(kq.Q6_K, w, k, x, tiles)
    xn = row_norms_x(x)
    for ex in range(experts):
        r = np.nonzero(ids == ex)[0]
        check_qmm(y[r], ref[r], xn[r], row_norms_w(kq.Q6_K, w[ex], k), k)
