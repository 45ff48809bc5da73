"""The Python binding's buffer checks, on the CPU: the C ABI takes bare
pointers, so the binding compares every tensor's element size and element
count with the sizes of the call before anything reaches the library.  CPU
tensors serve as stand-ins: a call whose buffers are right gets as far as the
CUDA-device check; a call whose buffers are wrong stops before it."""
import pytest
import torch

import gguf_quant_dequant_q4_b200 as kq

CUDA = "CUDA tensors"


def u8(*shape):
    return torch.zeros(*shape, dtype=torch.uint8)


def bf(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


@pytest.mark.parametrize("fn", [kq.qmv, kq.qmm])
def test_matmul_buffers(fn):
    n, k = 8, 512
    w = u8(n, kq.row_bytes(kq.Q4_K, k))
    with pytest.raises(ValueError, match=CUDA):
        fn(bf(2, k), w, kq.Q4_K)
    with pytest.raises(ValueError, match=CUDA):
        fn(bf(2, k), w, kq.Q4_K, out=f32(2, n))
    # rows of the wrong length for k (here: k = 256 worth of bytes)
    with pytest.raises(ValueError, match="rows of 288 bytes"):
        fn(bf(2, k), u8(n, 144), kq.Q4_K)
    with pytest.raises(TypeError, match="1-byte elements"):
        fn(bf(2, k), torch.zeros(n, 288, dtype=torch.int16), kq.Q4_K)
    with pytest.raises(ValueError, match="2 dimensions"):
        fn(bf(2, k), u8(2, n, 288), kq.Q4_K)
    # an output too small or of the wrong element type
    with pytest.raises(ValueError, match="at least 16 elements"):
        fn(bf(2, k), w, kq.Q4_K, out=f32(1, n))
    with pytest.raises(TypeError, match="4-byte elements"):
        fn(bf(2, k), w, kq.Q4_K, out=torch.zeros(2, n, dtype=torch.float16))
    with pytest.raises(TypeError, match="bfloat16"):
        fn(f32(2, k), w, kq.Q4_K)


def test_matmul_sizes_the_library_rejects_pass_through():
    # k not a block multiple, or an unknown codec: no row check in Python,
    # the library answers with its own status (here: stopped at the device check)
    with pytest.raises(ValueError, match=CUDA):
        kq.qmv(bf(1, 100), u8(4, 10), kq.Q4_K)
    with pytest.raises(ValueError, match=CUDA):
        kq.qmv(bf(1, 256), u8(4, 10), 3)


def test_dequantize_and_quantize_buffers():
    k = 64
    w = u8(3, 5, kq.row_bytes(kq.Q8_0, k))
    with pytest.raises(ValueError, match=CUDA):
        kq.dequantize(w, kq.Q8_0, k)
    with pytest.raises(ValueError, match="rows of 68 bytes"):
        kq.dequantize(u8(3, 5, 34), kq.Q8_0, k)
    with pytest.raises(ValueError, match="at least 960 elements"):
        kq.dequantize(w, kq.Q8_0, k, out=f32(15, 63))
    wf = f32(6, 256)
    with pytest.raises(ValueError, match=CUDA):
        kq.quantize(wf, kq.Q6_K)
    with pytest.raises(ValueError, match="at least 1260 elements"):
        kq.quantize(wf, kq.Q6_K, out=u8(5, 210))
    with pytest.raises(TypeError, match="1-byte elements"):
        kq.quantize(wf, kq.Q6_K, out=torch.zeros(6, 105, dtype=torch.int16))


def test_prefill_moe_buffers():
    t, top_k, e, n, k = 5, 2, 4, 16, 256
    ids = i32(t, top_k)
    with pytest.raises(ValueError, match=CUDA):
        kq.moe_sort(ids, e, bf(t, k))
    with pytest.raises(TypeError, match="4-byte elements"):
        kq.moe_sort(ids.long(), e)
    with pytest.raises(ValueError, match="at least 1280 elements"):
        kq.moe_sort(ids, e, bf(t - 1, k))
    with pytest.raises(ValueError, match="at least 1 elements"):
        kq.moe_sort(ids, e, err=i32(0))
    with pytest.raises(TypeError, match="4-byte elements"):
        kq.expert_tile_map(ids.flatten().long(), e)
    bank = u8(e, n, kq.row_bytes(kq.Q4_K, k))
    tm, cnt = i32(9, 3), i32(1)
    with pytest.raises(ValueError, match=CUDA):
        kq.gather_qmm(bf(t * top_k, k), bank, kq.Q4_K, tm, cnt)
    with pytest.raises(ValueError, match=r"\[cap, 3\]"):
        kq.gather_qmm(bf(t * top_k, k), bank, kq.Q4_K, i32(27), cnt)
    with pytest.raises(ValueError, match="at least 1 elements"):
        kq.gather_qmm(bf(t * top_k, k), bank, kq.Q4_K, tm, i32(0))
    with pytest.raises(ValueError, match="3 dimensions"):
        kq.gather_qmm(bf(t * top_k, k), u8(e * n, 144), kq.Q4_K, tm, cnt)
    with pytest.raises(ValueError, match="at least 160 elements"):
        kq.gather_qmm(bf(t * top_k, k), bank, kq.Q4_K, tm, cnt, out=f32(t * top_k - 1, n))


def test_decode_moe_buffers():
    t, top_k, e, n, k = 3, 2, 4, 16, 512
    bank = u8(e, n, kq.row_bytes(kq.Q6_K, k))
    ids = i32(t, top_k)
    with pytest.raises(ValueError, match=CUDA):
        kq.gather_qmv(bf(t * top_k, k), bank, kq.Q6_K, ids)
    with pytest.raises(ValueError, match=CUDA):
        kq.gather_qmv(bf(t, k), bank, kq.Q6_K, ids, x_per_token=True)
    # one activation row per pair unless x_per_token
    with pytest.raises(ValueError, match="at least 3072 elements"):
        kq.gather_qmv(bf(t, k), bank, kq.Q6_K, ids)
    with pytest.raises(ValueError, match="rows of 420 bytes"):
        kq.gather_qmv(bf(t * top_k, k), u8(e, n, 210), kq.Q6_K, ids)
    with pytest.raises(ValueError, match="at least 96 elements"):
        kq.gather_qmv(bf(t * top_k, k), bank, kq.Q6_K, ids, out=f32(t, n))
    with pytest.raises(ValueError, match=CUDA):
        kq.moe_glu_gather(bf(t, k), bank, bank.clone(), kq.Q6_K, ids)
    with pytest.raises(ValueError, match="up_bank: shape"):
        kq.moe_glu_gather(bf(t, k), bank, u8(e - 1, n, 420), kq.Q6_K, ids)
    with pytest.raises(ValueError, match="at least 1536 elements"):
        kq.moe_glu_gather(bf(t - 1, k), bank, bank, kq.Q6_K, ids)
    y = f32(t * top_k, n)
    with pytest.raises(ValueError, match=CUDA):
        kq.gather_mix(y, i32(t * top_k), f32(t, top_k))
    with pytest.raises(ValueError, match="at least 6 elements"):
        kq.gather_mix(y, i32(t * top_k - 1), f32(t, top_k))
    with pytest.raises(TypeError, match="4-byte elements"):
        kq.gather_mix(y, i32(t * top_k), torch.zeros(t, top_k, dtype=torch.float64))
    with pytest.raises(ValueError, match="at least 48 elements"):
        kq.gather_mix(y, i32(t * top_k), f32(t, top_k), out=f32(t - 1, n))


def test_strided_views_are_refused_and_leading_slices_pass():
    # a bank sliced along its rows is a strided view: refused, never walked
    # with the packed stride; a slice of whole experts is contiguous (an offset
    # pointer) and goes through
    t, top_k, e, n, k = 2, 2, 6, 16, 256
    bank = u8(e, n, kq.row_bytes(kq.Q4_K, k))
    ids = i32(t, top_k)
    with pytest.raises(ValueError, match="contiguous"):
        kq.gather_qmv(bf(t * top_k, k), bank[:, : n // 2], kq.Q4_K, ids)
    with pytest.raises(ValueError, match=CUDA):
        kq.gather_qmv(bf(t * top_k, k), bank[2:5], kq.Q4_K, ids)
    with pytest.raises(ValueError, match="contiguous"):
        kq.qmv(bf(k, 2).t(), bank[0], kq.Q4_K)
    with pytest.raises(ValueError, match=CUDA):
        kq.qmv(bf(2, k), bank[0, 4:], kq.Q4_K)
