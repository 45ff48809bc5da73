"""CPU oracle for the GGUF block-quantized matmul path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, nothing
else.  It shares no code with the CUDA library (``gguf_quant_dequant_q4_b200``)
and never imports it.

The arithmetic lives in ``kq_oracle.c`` (plain C, gcc -O2 -ffp-contract=off,
OpenMP over output rows only).  This module compiles it, marshals numpy arrays,
and states the MoE semantics in plain numpy:

* ``dequantize``   exact fp32 decode (mlx-kquant bindings.cpp, ``dequantize``).
* ``matmul``       y = x @ dequant(w).T in fp64 (bindings.cpp,
                   ``quantized_matmul`` with transpose=True).
* ``moe_sort``     stable sort of (token, slot) pairs by expert id; x rows
                   gathered into expert-sorted order (mlx-kquant README,
                   "Performance": sorted MoE prefill batches; bindings.cpp
                   ``gather_qmm_seg``, whose rows come grouped by expert).
* ``tile_map``     (expert, row_start, num_rows) tiles of at most 64 rows,
                   only the last tile of a segment partial (bindings.cpp,
                   ``expert_tile_map``).
* ``gather_qmm``   y[r] = x_sorted[r] @ dequant(w[e(r)]).T for every row
                   covered by a tile (bindings.cpp, ``gather_qmm_seg``;
                   hanzo-ml quantized/mod.rs, ``indexed_moe_forward`` CPU
                   fallback that groups rows per expert and runs one
                   quantized matmul per expert).
* ``gather_qmv``   decode-shaped MoE product, one output row per (token,
                   slot) pair: y[p] = x[row(p)] @ dequant(w[ids[p]]).T
                   (bindings.cpp, ``gather_qmv_kq``: an activation row of
                   its own for each expert slot, x [T, R, K], indices [T, R], output
                   [T, R, N]; with one activation row per token the same
                   product feeds the gate/up projections of
                   ``moe_glu_gather_kq``).
* ``moe_glu_gather`` act(x W_g^T) * (x W_u^T) per pair from the fp64 gate
                   and up products, act silu, gelu (tanh form) or silu with
                   a limit (bindings.cpp, ``moe_glu_gather_kq``).
* ``quantize``     float -> wire bytes (bindings.cpp, ``quantize``: float
                   weights in, wire bytes out): q8_0 by
                   ggml's absmax rule, q4_K / q6_K by min/max and absmax
                   scales in fixed fp32 steps (see kq_oracle.c).
* ``inverse_order`` / ``gather_mix``  unsort and score mix of expert-sorted
                   rows: out[t] = sum_s scores[t, s] * y[inv_order[t k + s]]
                   (bindings.cpp, ``gather_mix``: f32 accumulation; hanzo-ml
                   quantized/mod.rs ``moe_combine``: the per-slot outputs
                   reduced by the router weights).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None

Q4_0, Q8_0, Q4_K, Q5_K, Q6_K = 2, 8, 12, 13, 14
TILE_ROWS = 64


def build(force: bool = False) -> str:
    """Compile kq_oracle.c into oracle/_build/liboracle.so (idempotent)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, ip = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_block_info.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        lib.oracle_dequantize.argtypes = [ctypes.c_int, ip, i64, i64, ip]
        lib.oracle_matmul_f64.argtypes = [ctypes.c_int, ip, i64, i64, ip, i64, ip, ip]
        lib.oracle_matmul_f32.argtypes = [ctypes.c_int, ip, i64, i64, ip, i64, ip]
        lib.oracle_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_quantize.argtypes = [ctypes.c_int, ip, i64, i64, ip]
        lib.oracle_float_to_half.argtypes = [ip, i64, ip]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def block_info(qtype: int) -> tuple[int, int]:
    v, b = ctypes.c_int(), ctypes.c_int()
    if _load().oracle_block_info(qtype, ctypes.byref(v), ctypes.byref(b)):
        raise ValueError(f"unknown codec {qtype}")
    return v.value, b.value


def threads() -> int:
    return _load().oracle_threads()


def set_threads(n: int) -> None:
    """Thread count of the parallel loops (0: all host cores)."""
    _load().oracle_set_threads(int(n))


def _check_w(qtype: int, w: np.ndarray, k: int) -> np.ndarray:
    vpb, bpb = block_info(qtype)
    if k % vpb:
        raise ValueError("K must be a multiple of the block size")
    w = np.ascontiguousarray(w, dtype=np.uint8)
    if w.shape[-1] != k // vpb * bpb:
        raise ValueError("row byte count does not match K")
    return w


def dequantize(qtype: int, w: np.ndarray, k: int) -> np.ndarray:
    """Wire bytes [..., N, row_bytes] -> fp32 [..., N, K] (exact)."""
    w = _check_w(qtype, w, k)
    rows = int(np.prod(w.shape[:-1]))
    out = np.empty(w.shape[:-1] + (k,), dtype=np.float32)
    if _load().oracle_dequantize(qtype, _ptr(w), rows, k, _ptr(out)):
        raise RuntimeError("oracle_dequantize failed")
    return out


def matmul(qtype: int, w: np.ndarray, k: int, x_bf16: np.ndarray, absdot: bool = False):
    """fp64 y[M, N] = x @ dequant(w).T; with absdot also sum_k |x*w|."""
    w = _check_w(qtype, w, k)
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    n, m = w.shape[0], x.shape[0]
    y = np.empty((m, n), dtype=np.float64)
    a = np.empty((m, n), dtype=np.float64) if absdot else None
    rc = _load().oracle_matmul_f64(qtype, _ptr(w), n, k, _ptr(x), m, _ptr(y),
                                   _ptr(a) if absdot else None)
    if rc:
        raise RuntimeError("oracle_matmul_f64 failed")
    return (y, a) if absdot else y


def matmul_f32(qtype: int, w: np.ndarray, k: int, x_bf16: np.ndarray) -> np.ndarray:
    """fp32 sequential-k y[M, N] (timed CPU baseline only)."""
    w = _check_w(qtype, w, k)
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    n, m = w.shape[0], x.shape[0]
    y = np.empty((m, n), dtype=np.float32)
    if _load().oracle_matmul_f32(qtype, _ptr(w), n, k, _ptr(x), m, _ptr(y)):
        raise RuntimeError("oracle_matmul_f32 failed")
    return y


def bf16_to_f32(x_bf16: np.ndarray) -> np.ndarray:
    return (np.asarray(x_bf16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def moe_sort(topk_ids: np.ndarray, n_experts: int):
    """Stable sort of the (token, slot) pairs by expert id.

    Returns (sorted_expert_ids uint32 [rows], sorted_pair int32 [rows]) with
    sorted_pair[r] = token * top_k + slot of the pair placed at sorted row r.
    Pairs with equal expert keep (token, slot) order."""
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    if ids.size and (ids.min() < 0 or ids.max() >= n_experts):
        raise ValueError("expert id out of range")
    order = np.argsort(ids, kind="stable")
    return ids[order].astype(np.uint32), order.astype(np.int32)


def gather_rows(x_bf16: np.ndarray, sorted_pair: np.ndarray, top_k: int) -> np.ndarray:
    """x_sorted[r] = x[sorted_pair[r] // top_k]."""
    return np.ascontiguousarray(np.asarray(x_bf16)[np.asarray(sorted_pair) // top_k])


def tile_map(sorted_ids: np.ndarray, n_experts: int, tile: int = TILE_ROWS):
    """Tiles (expert, row_start, num_rows) covering every expert segment of an
    ascending expert-id array, each at most `tile` rows, only the last tile of a
    segment partial; experts without rows get no tile."""
    ids = np.asarray(sorted_ids, dtype=np.int64)
    if ids.size and np.any(np.diff(ids) < 0):
        raise ValueError("ids must be sorted ascending")
    tiles = []
    for e in range(n_experts):
        idx = np.nonzero(ids == e)[0]
        if idx.size == 0:
            continue
        start, cnt = int(idx[0]), int(idx.size)
        for off in range(0, cnt, tile):
            tiles.append((e, start + off, min(tile, cnt - off)))
    return tiles


def map_capacity(rows: int, n_experts: int, tile: int = TILE_ROWS) -> int:
    """Upper bound on the number of tiles: ceil(rows / tile) + n_experts."""
    return -(-rows // tile) + n_experts


def gather_qmm(qtype: int, w_bank: np.ndarray, k: int, x_sorted: np.ndarray, tiles,
               absdot: bool = False):
    """fp64 y[rows, N]; rows covered by no tile are NaN (left unwritten)."""
    rows = x_sorted.shape[0]
    n = w_bank.shape[1]
    y = np.full((rows, n), np.nan)
    a = np.full((rows, n), np.nan) if absdot else None
    for e, s, c in tiles:
        r = matmul(qtype, w_bank[e], k, x_sorted[s:s + c], absdot=absdot)
        if absdot:
            y[s:s + c], a[s:s + c] = r
        else:
            y[s:s + c] = r
    return (y, a) if absdot else y


def gather_qmv(qtype: int, w_bank: np.ndarray, k: int, x_bf16: np.ndarray, ids: np.ndarray,
               x_per_token: bool = False, absdot: bool = False):
    """fp64 y[P, N] for the P = T * top_k (token, slot) pairs of ids [T, top_k]:
    y[p] = x[p] @ dequant(w_bank[ids.flat[p]]).T, or x[p // top_k] when x holds
    one row per token.  Rows of pairs whose id is out of range are NaN
    (left unwritten).  Each row is independent; rows of one expert are simply
    computed together."""
    ids = np.asarray(ids, dtype=np.int64)
    top_k = ids.shape[-1] if ids.ndim > 1 else 1
    flat = ids.reshape(-1)
    x = np.asarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    rows = np.arange(flat.size) // top_k if x_per_token else np.arange(flat.size)
    n = w_bank.shape[1]
    y = np.full((flat.size, n), np.nan)
    a = np.full((flat.size, n), np.nan) if absdot else None
    for e in range(w_bank.shape[0]):
        sel = np.nonzero(flat == e)[0]
        if sel.size == 0:
            continue
        r = matmul(qtype, w_bank[e], k, x[rows[sel]], absdot=absdot)
        if absdot:
            y[sel], a[sel] = r
        else:
            y[sel] = r
    return (y, a) if absdot else y


def inverse_order(sorted_pair: np.ndarray) -> np.ndarray:
    """inv[sorted_pair[r]] = r: the sorted row of every (token, slot) pair."""
    sp = np.asarray(sorted_pair, dtype=np.int64)
    inv = np.empty(sp.size, dtype=np.int32)
    inv[sp] = np.arange(sp.size, dtype=np.int32)
    return inv


def gather_mix(y: np.ndarray, inv_order: np.ndarray, scores: np.ndarray) -> np.ndarray:
    """out[t] = sum over s = 0, 1, .. of scores[t, s] * y[inv_order[t k + s]], in
    fp32: each product rounded to fp32, then added to the running fp32 sum
    (which starts at zero), slots in ascending order."""
    y = np.asarray(y, dtype=np.float32)
    sc = np.asarray(scores, dtype=np.float32)
    t, kk = sc.shape
    inv = np.asarray(inv_order, dtype=np.int64).reshape(t, kk)
    out = np.zeros((t, y.shape[1]), dtype=np.float32)
    for s in range(kk):
        prod = (sc[:, s:s + 1] * y[inv[:, s]]).astype(np.float32)
        out = (out + prod).astype(np.float32)
    return out


ACT_SILU, ACT_GELU_TANH, ACT_SILU_LIMIT = 0, 1, 2


def glu(act: int, g: np.ndarray, u: np.ndarray, limit: float = 0.0) -> np.ndarray:
    """act(g) * u in fp64: silu(g) = g / (1 + exp(-g)); gelu in the tanh form
    0.5 g (1 + tanh(sqrt(2 / pi) (g + 0.044715 g^3))); silu with limit L:
    silu(min(g, L)) * clip(u, -L, L)."""
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    if act == ACT_SILU_LIMIT:
        g = np.minimum(g, limit)
        u = np.clip(u, -limit, limit)
    if act == ACT_GELU_TANH:
        a = 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))
    else:
        with np.errstate(over="ignore"):   # exp(-g) = inf for g << 0 gives silu = -0
            a = g / (1.0 + np.exp(-g))
    return a * u


def moe_glu_gather(qtype: int, gate_bank: np.ndarray, up_bank: np.ndarray, k: int, x_bf16: np.ndarray,
                   ids: np.ndarray, act: int = ACT_SILU, limit: float = 0.0):
    """(out, g, u, ag, au): out[p] = act(g[p], u[p]) with the fp64 per-pair
    products g = x[t] @ dequant(gate[e]).T and u = x[t] @ dequant(up[e]).T
    (one activation row per token), and their sums of |x w| (ag, au)."""
    g, ag = gather_qmv(qtype, gate_bank, k, x_bf16, ids, x_per_token=True, absdot=True)
    u, au = gather_qmv(qtype, up_bank, k, x_bf16, ids, x_per_token=True, absdot=True)
    return glu(act, g, u, limit), g, u, ag, au


def float_to_half_bits(x: np.ndarray) -> np.ndarray:
    """binary32 -> binary16 bits, round to nearest even (the encoder's rounding)."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, dtype=np.uint16)
    _load().oracle_float_to_half(_ptr(x), x.size, _ptr(out))
    return out


def quantize(qtype: int, w: np.ndarray) -> np.ndarray:
    """fp32 [..., K] -> wire bytes [..., row_bytes] (fixed fp32 steps)."""
    vpb, bpb = block_info(qtype)
    w = np.ascontiguousarray(w, dtype=np.float32)
    k = w.shape[-1]
    if k % vpb:
        raise ValueError("K must be a multiple of the block size")
    rows = int(np.prod(w.shape[:-1]))
    out = np.empty(w.shape[:-1] + (k // vpb * bpb,), dtype=np.uint8)
    if _load().oracle_quantize(qtype, _ptr(w), rows, k, _ptr(out)):
        raise RuntimeError("oracle_quantize failed")
    return out
