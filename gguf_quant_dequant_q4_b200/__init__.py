"""B200 (sm_100a) matrix products with GGUF block-quantized weights.

A thin Python binding over the C ABI in ``include/kq.h`` (shared library
``_lib/libkq.so``, built by ``python -m gguf_quant_dequant_q4_b200.build``).
This module only marshals arguments: torch provides device memory and the
current CUDA stream, every step of the computation runs in the library's
kernels.  There is no CPU fallback; calling an op without the built library or
without a CUDA device raises.

Codecs (ggml type ids): ``Q4_0 = 2``, ``Q8_0 = 8``, ``Q4_K = 12``, ``Q5_K = 13``,
``Q6_K = 14`` (q5_K and q4_0: dequantize and the tensor-core products).  Weights are
wire bytes ``uint8 [N, row_bytes]`` ("transpose=True" layout: y = x @ W.T),
activations ``bfloat16 [M, K]``, outputs ``float32``.
"""
from __future__ import annotations

import ctypes
import os

import torch

Q4_0, Q8_0, Q4_K, Q5_K, Q6_K = 2, 8, 12, 13, 14
NAMES = {Q4_0: "q4_0", Q8_0: "q8_0", Q4_K: "q4_K", Q5_K: "q5_K", Q6_K: "q6_K"}
_BLOCK = {Q4_0: (32, 18), Q8_0: (32, 34), Q4_K: (256, 144), Q5_K: (256, 176), Q6_K: (256, 210)}
TILE_ROWS = 64

DEV_BAD_EXPERT, DEV_BAD_ROWS, DEV_BAD_RANGE, DEV_UNSORTED = 0x1, 0x2, 0x4, 0x8
DEV_TIMEOUT, DEV_TOO_MANY, DEV_X_RANGE = 0x10, 0x20, 0x40

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libkq.so")

# Every entry point declared in include/kq.h: name -> (restype, argtypes)
_vp, _i64, _i32, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
SIGNATURES = {
    "kq_block_info": (_int, [_int, ctypes.POINTER(_int), ctypes.POINTER(_int)]),
    "kq_status_string": (ctypes.c_char_p, [_int]),
    "kq_last_cuda_error": (_int, []),
    "kq_read_device_status": (_int, [ctypes.POINTER(_i32), _int]),
    "kq_set_wait_limit": (_int, [_i64]),
    "kq_dequantize": (_int, [_int, _vp, _i64, _i64, _vp, _vp]),
    "kq_quantize": (_int, [_int, _vp, _i64, _i64, _vp, _vp]),
    "kq_qmv": (_int, [_int, _vp, _i64, _i64, _vp, _i64, _vp, _vp]),
    "kq_qmm": (_int, [_int, _vp, _i64, _i64, _vp, _i64, _vp, _vp]),
    "kq_moe_sort": (_int, [_vp, _i64, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "kq_expert_tile_map": (_int, [_vp, _i64, _i32, _vp, _i64, _vp, _vp, _vp]),
    "kq_gather_qmm": (_int, [_int, _vp, _i32, _i64, _i64, _vp, _i64, _vp, _vp, _i64, _vp, _vp, _vp]),
    "kq_gather_qmv": (_int, [_int, _vp, _i32, _i64, _i64, _vp, _i32, _vp, _i64, _i32, _vp, _vp, _vp]),
    "kq_gather_mix": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp, _vp, _vp]),
    "kq_moe_glu_gather": (_int, [_int, _vp, _vp, _i32, _i64, _i64, _vp, _vp, _i64, _i32, _i32, ctypes.c_float,
                                 _vp, _vp, _vp]),
}
ACT_SILU, ACT_GELU_TANH, ACT_SILU_LIMIT = 0, 1, 2

_lib = None


class KQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().kq_status_string(status).decode()
        if status == 4:
            msg += f" (cudaError {lib().kq_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [status {status}]")


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m gguf_quant_dequant_q4_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype, f.argtypes = res, args
        _lib = l
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise KQError(rc, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _need_cuda(*ts):
    # contiguity first: a strided view (say, some rows of every expert of a
    # bank) would otherwise be walked with the packed stride
    if any(t is not None and not t.is_contiguous() for t in ts):
        raise ValueError("all tensors must be contiguous")
    if any(t is not None and not t.is_cuda for t in ts):
        raise ValueError("all tensors must be CUDA tensors")


def _need(t, what: str, size: int, count: int | None = None, exact: bool = False) -> None:
    """Tensor ``t`` (if given) holds elements of ``size`` bytes, and at least
    (or exactly) ``count`` of them: the C ABI takes bare pointers, so a buffer
    shorter than the call's sizes would be read or written past its end."""
    if t is None:
        return
    if t.element_size() != size:
        raise TypeError(f"{what}: {size}-byte elements expected, got {t.dtype}")
    if count is not None and (t.numel() != count if exact else t.numel() < count):
        raise ValueError(f"{what}: {'exactly' if exact else 'at least'} {count} elements expected, got {t.numel()}")


def _whole_blocks(qtype: int, k: int) -> bool:
    # sizes the library accepts; anything else it rejects with its own status
    return qtype in _BLOCK and k > 0 and k % _BLOCK[qtype][0] == 0


def _need_bank(w, what: str, qtype: int, k: int, dims: int) -> None:
    """Weight bytes with ``dims`` dimensions whose rows hold ``k`` values."""
    _need(w, what, 1)
    if w.dim() != dims:
        raise ValueError(f"{what}: {dims} dimensions expected, got {w.dim()}")
    if _whole_blocks(qtype, k) and w.shape[-1] != row_bytes(qtype, k):
        raise ValueError(f"{what}: rows of {row_bytes(qtype, k)} bytes expected for k = {k}, got {w.shape[-1]}")


def block_info(qtype: int) -> tuple[int, int]:
    v, b = _int(), _int()
    _check(lib().kq_block_info(qtype, ctypes.byref(v), ctypes.byref(b)), "kq_block_info")
    return v.value, b.value


def row_bytes(qtype: int, k: int) -> int:
    vpb, bpb = _BLOCK[qtype]
    return k // vpb * bpb


def read_device_status(clear: bool = False) -> int:
    v = _i32()
    _check(lib().kq_read_device_status(ctypes.byref(v), int(clear)), "kq_read_device_status")
    return v.value


def set_wait_limit(ns: int = 0) -> None:
    """Time limit (ns) of the staged decode kernel's pipeline waits; 0 restores
    the default (2 s).  For fault-handling tests."""
    _check(lib().kq_set_wait_limit(int(ns)), "kq_set_wait_limit")


def _bf16_bits(x: torch.Tensor) -> torch.Tensor:
    if x.dtype == torch.bfloat16:
        return x
    if x.dtype in (torch.uint16, torch.int16):
        return x
    raise TypeError("activations must be bfloat16")


def dequantize(w: torch.Tensor, qtype: int, k: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 [..., N, K] decode of wire bytes [..., N, row_bytes] (bit-exact)."""
    rows = w.numel() // max(1, w.shape[-1]) if w.dim() else 0
    _need(w, "w", 1)
    if w.dim() and _whole_blocks(qtype, k) and w.shape[-1] != row_bytes(qtype, k):
        raise ValueError(f"w: rows of {row_bytes(qtype, k)} bytes expected for k = {k}, got {w.shape[-1]}")
    if out is None:
        out = torch.empty(*w.shape[:-1], k, dtype=torch.float32, device=w.device)
    _need(out, "out", 4, rows * k)
    _need_cuda(w, out)
    _check(lib().kq_dequantize(qtype, _ptr(w), rows, k, _ptr(out), _stream(stream)), "kq_dequantize")
    return out


def quantize(w: torch.Tensor, qtype: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Wire bytes uint8 [..., row_bytes] of fp32 weights [..., K]."""
    if w.dtype != torch.float32:
        raise TypeError("weights must be float32")
    k = w.shape[-1]
    rows = w.numel() // max(1, k)
    if out is None:
        out = torch.empty(*w.shape[:-1], row_bytes(qtype, k), dtype=torch.uint8, device=w.device)
    if _whole_blocks(qtype, k):
        _need(out, "out", 1, rows * row_bytes(qtype, k))
    _need_cuda(w, out)
    _check(lib().kq_quantize(qtype, _ptr(w), rows, k, _ptr(out), _stream(stream)), "kq_quantize")
    return out


def qmv(x: torch.Tensor, w: torch.Tensor, qtype: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[M, N] = x[M, K] @ dequant(w[N, :]).T for 1 <= M <= 16."""
    x = _bf16_bits(x)
    m, k = x.shape
    n = w.shape[0]
    _need_bank(w, "w", qtype, k, 2)
    if out is None:
        out = torch.empty(m, n, dtype=torch.float32, device=x.device)
    _need(out, "out", 4, m * n)
    _need_cuda(x, w, out)
    _check(lib().kq_qmv(qtype, _ptr(w), n, k, _ptr(x), m, _ptr(out), _stream(stream)), "kq_qmv")
    return out


def qmm(x: torch.Tensor, w: torch.Tensor, qtype: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[M, N] = x[M, K] @ dequant(w[N, :]).T on the tcgen05 tensor cores."""
    x = _bf16_bits(x)
    m, k = x.shape
    n = w.shape[0]
    _need_bank(w, "w", qtype, k, 2)
    if out is None:
        out = torch.empty(m, n, dtype=torch.float32, device=x.device)
    _need(out, "out", 4, m * n)
    _need_cuda(x, w, out)
    _check(lib().kq_qmm(qtype, _ptr(w), n, k, _ptr(x), m, _ptr(out), _stream(stream)), "kq_qmm")
    return out


def map_capacity(rows: int, n_experts: int) -> int:
    return -(-rows // TILE_ROWS) + n_experts


def moe_sort(topk_ids: torch.Tensor, n_experts: int, x: torch.Tensor | None = None, err: torch.Tensor | None = None,
             stream=None, with_inverse: bool = False):
    """Stable sort of routed pairs by expert: (sorted_ids, sorted_pair, x_sorted),
    plus inv_order (the sorted row of every pair) when with_inverse is set."""
    t, top_k = topk_ids.shape
    rows = t * top_k
    _need(topk_ids, "topk_ids", 4)
    _need(err, "err", 4, 1)
    dev = topk_ids.device
    sids = torch.empty(rows, dtype=torch.int32, device=dev)
    pair = torch.empty(rows, dtype=torch.int32, device=dev)
    inv = torch.empty(rows, dtype=torch.int32, device=dev) if with_inverse else None
    xs = None
    k = 0
    if x is not None:
        x = _bf16_bits(x)
        k = x.shape[1]
        _need(x, "x", 2, t * k)
        xs = torch.empty(rows, k, dtype=x.dtype, device=dev)
    _need_cuda(topk_ids, x, xs, err)
    _check(lib().kq_moe_sort(_ptr(topk_ids), t, top_k, n_experts, _ptr(x), k, _ptr(sids), _ptr(pair), _ptr(inv),
                             _ptr(xs), _ptr(err), _stream(stream)), "kq_moe_sort")
    return (sids, pair, xs, inv) if with_inverse else (sids, pair, xs)


def expert_tile_map(sorted_ids: torch.Tensor, n_experts: int, cap: int | None = None,
                    err: torch.Tensor | None = None, stream=None):
    """(map int32 [cap, 3] of (expert, row_start, num_rows), count int32 [1])."""
    rows = sorted_ids.numel()
    cap = map_capacity(rows, n_experts) if cap is None else cap
    _need(sorted_ids, "sorted_ids", 4)
    _need(err, "err", 4, 1)
    m = torch.empty(cap, 3, dtype=torch.int32, device=sorted_ids.device)
    c = torch.empty(1, dtype=torch.int32, device=sorted_ids.device)
    _need_cuda(sorted_ids, err)
    _check(lib().kq_expert_tile_map(_ptr(sorted_ids), rows, n_experts, _ptr(m), cap, _ptr(c), _ptr(err),
                                    _stream(stream)), "kq_expert_tile_map")
    return m, c


def gather_qmm(x_sorted: torch.Tensor, w_bank: torch.Tensor, qtype: int, tile_map: torch.Tensor,
               count: torch.Tensor, out: torch.Tensor | None = None, err: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """y[r] = x_sorted[r] @ dequant(w_bank[e(r)]).T for every row covered by a tile."""
    x_sorted = _bf16_bits(x_sorted)
    rows, k = x_sorted.shape
    e, n = w_bank.shape[0], w_bank.shape[1]
    _need_bank(w_bank, "w_bank", qtype, k, 3)
    _need(tile_map, "tile_map", 4)
    if tile_map.dim() != 2 or tile_map.shape[1] != 3:
        raise ValueError(f"tile_map: [cap, 3] expected, got {tuple(tile_map.shape)}")
    _need(count, "count", 4, 1)
    _need(err, "err", 4, 1)
    if out is None:
        out = torch.empty(rows, n, dtype=torch.float32, device=x_sorted.device)
    _need(out, "out", 4, rows * n)
    _need_cuda(x_sorted, w_bank, tile_map, count, out, err)
    _check(lib().kq_gather_qmm(qtype, _ptr(w_bank), e, n, k, _ptr(x_sorted), rows, _ptr(tile_map), _ptr(count),
                               tile_map.shape[0], _ptr(out), _ptr(err), _stream(stream)), "kq_gather_qmm")
    return out


def gather_qmv(x: torch.Tensor, w_bank: torch.Tensor, qtype: int, ids: torch.Tensor, x_per_token: bool = False,
               out: torch.Tensor | None = None, err: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode MoE product, one row per (token, slot) pair p = t * top_k + s:
    y[p] = x[p] @ dequant(w_bank[ids[t, s]]).T (x [T*top_k, K]), or
    x[t] @ ... with x_per_token (x [T, K]).  ids int32 [T, top_k]."""
    x = _bf16_bits(x)
    t, top_k = ids.shape
    k = x.shape[-1]
    e, n = w_bank.shape[0], w_bank.shape[1]
    _need_bank(w_bank, "w_bank", qtype, k, 3)
    _need(ids, "ids", 4)
    _need(err, "err", 4, 1)
    _need(x, "x", 2, (t if x_per_token else t * top_k) * k)
    if out is None:
        out = torch.empty(t * top_k, n, dtype=torch.float32, device=x.device)
    _need(out, "out", 4, t * top_k * n)
    _need_cuda(x, w_bank, ids, out, err)
    _check(lib().kq_gather_qmv(qtype, _ptr(w_bank), e, n, k, _ptr(x), int(bool(x_per_token)), _ptr(ids), t, top_k,
                               _ptr(out), _ptr(err), _stream(stream)), "kq_gather_qmv")
    return out


def gather_mix(y: torch.Tensor, inv_order: torch.Tensor, scores: torch.Tensor, out: torch.Tensor | None = None,
               err: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t] = sum_s scores[t, s] * y[inv_order[t * top_k + s]] (fp32, slots in order)."""
    rows, n = y.shape
    t, top_k = scores.shape
    _need(y, "y", 4)
    _need(inv_order, "inv_order", 4, t * top_k)
    _need(scores, "scores", 4)
    _need(err, "err", 4, 1)
    if out is None:
        out = torch.empty(t, n, dtype=torch.float32, device=y.device)
    _need(out, "out", 4, t * n)
    _need_cuda(y, inv_order, scores, out, err)
    _check(lib().kq_gather_mix(_ptr(y), rows, n, _ptr(inv_order), _ptr(scores), t, top_k, _ptr(out), _ptr(err),
                               _stream(stream)), "kq_gather_mix")
    return out


def moe_glu_gather(x: torch.Tensor, gate_bank: torch.Tensor, up_bank: torch.Tensor, qtype: int, ids: torch.Tensor,
                   act: int = ACT_SILU, limit: float = 0.0, out: torch.Tensor | None = None,
                   err: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t * top_k + s] = act(x[t] @ dequant(gate[e]).T, x[t] @ dequant(up[e]).T), e = ids[t, s]."""
    x = _bf16_bits(x)
    t, top_k = ids.shape
    k = x.shape[-1]
    e, n = gate_bank.shape[0], gate_bank.shape[1]
    _need_bank(gate_bank, "gate_bank", qtype, k, 3)
    _need_bank(up_bank, "up_bank", qtype, k, 3)
    if up_bank.shape != gate_bank.shape:
        raise ValueError(f"up_bank: shape {tuple(gate_bank.shape)} expected, got {tuple(up_bank.shape)}")
    _need(ids, "ids", 4)
    _need(err, "err", 4, 1)
    _need(x, "x", 2, t * k)
    if out is None:
        out = torch.empty(t * top_k, n, dtype=torch.float32, device=x.device)
    _need(out, "out", 4, t * top_k * n)
    _need_cuda(x, gate_bank, up_bank, ids, out, err)
    _check(lib().kq_moe_glu_gather(qtype, _ptr(gate_bank), _ptr(up_bank), e, n, k, _ptr(x), _ptr(ids), t, top_k,
                                   act, limit, _ptr(out), _ptr(err), _stream(stream)), "kq_moe_glu_gather")
    return out
