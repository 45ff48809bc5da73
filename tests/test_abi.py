"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/kq.h, and rejects bad arguments on the host before any
CUDA call (pointer arguments here are fake addresses that are never touched).
"""
import ctypes
import os
import re

import pytest

import gguf_quant_dequant_q4_b200 as kq
from gguf_quant_dequant_q4_b200 import build as kqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, ALIGN = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    kqbuild.build()
    return kq.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "kq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path():
    syms = declared_symbols()
    for s in ("kq_dequantize", "kq_qmv", "kq_qmm", "kq_moe_sort", "kq_expert_tile_map", "kq_gather_qmm",
              "kq_gather_qmv", "kq_gather_mix", "kq_moe_glu_gather"):
        assert s in syms


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert syms
    for s in syms:
        assert hasattr(lib, s), s
    # the Python binding knows every declared entry point and nothing else
    assert sorted(kq.SIGNATURES) == syms


def test_block_info_and_status_strings(lib):
    assert kq.block_info(kq.Q4_K) == (256, 144)
    assert kq.block_info(kq.Q6_K) == (256, 210)
    assert kq.block_info(kq.Q8_0) == (32, 34)
    assert kq.block_info(kq.Q5_K) == (256, 176)
    assert kq.block_info(kq.Q4_0) == (32, 18)
    v = ctypes.c_int()
    assert lib.kq_block_info(3, ctypes.byref(v), None) == UNSUPPORTED
    for s in range(6):
        assert lib.kq_status_string(s)
    assert lib.kq_status_string(99) == b"unknown status"


A = 0x10000           # a fake, 16-byte aligned device address (never dereferenced)
MIS = 0x10008


@pytest.mark.parametrize("fn", ["kq_qmv", "kq_qmm"])
def test_matmul_argument_checks(lib, fn):
    f = getattr(lib, fn)
    assert f(3, A, 16, 256, A, 1, A, None) == UNSUPPORTED            # unknown codec
    assert f(kq.Q4_K, A, 16, 100, A, 1, A, None) == INVALID           # K not a block multiple
    assert f(kq.Q4_K, A, 16, 0, A, 1, A, None) == INVALID
    assert f(kq.Q4_K, A, 16, 2**31, A, 1, A, None) == INVALID        # K past 32-bit counts
    assert f(kq.Q4_K, A, -1, 256, A, 1, A, None) == INVALID
    assert f(kq.Q4_K, None, 16, 256, A, 1, A, None) == INVALID        # null weights
    assert f(kq.Q4_K, MIS, 16, 256, A, 1, A, None) == ALIGN           # misaligned weights
    assert f(kq.Q4_K, A, 16, 256, None, 1, A, None) == INVALID        # null x
    assert f(kq.Q4_K, A, 16, 256, MIS, 1, A, None) == ALIGN
    assert f(kq.Q4_K, A, 16, 256, A, 1, MIS, None) == ALIGN
    assert f(kq.Q8_0, A, 0, 32, A, 1, A, None) == OK                  # empty: nothing to do
    if fn == "kq_qmv":
        assert f(kq.Q4_K, A, 16, 256, A, 0, A, None) == INVALID       # m must be 1..16
        assert f(kq.Q4_K, A, 16, 256, A, 17, A, None) == INVALID


def test_quantize_argument_checks(lib):
    f = lib.kq_quantize
    assert f(5, A, 4, 256, A, None) == UNSUPPORTED
    assert f(kq.Q4_K, A, 4, 255, A, None) == INVALID
    assert f(kq.Q4_K, A, -1, 256, A, None) == INVALID
    assert f(kq.Q8_0, A, 4, 2**31, A, None) == INVALID
    assert f(kq.Q4_K, None, 4, 256, A, None) == INVALID
    assert f(kq.Q4_K, A, 4, 256, MIS, None) == ALIGN
    assert f(kq.Q8_0, MIS, 4, 32, A, None) == ALIGN
    assert f(kq.Q6_K, None, 0, 256, None, None) == OK
    assert f(kq.Q5_K, A, 4, 256, A, None) == UNSUPPORTED              # no encoder for q5_K / q4_0


def test_dequantize_argument_checks(lib):
    f = lib.kq_dequantize
    assert f(5, A, 4, 256, A, None) == UNSUPPORTED
    assert f(kq.Q6_K, A, 4, 255, A, None) == INVALID
    assert f(kq.Q6_K, A, 4, 256, None, None) == INVALID
    assert f(kq.Q8_0, A, 4, 2**36, A, None) == INVALID
    assert f(kq.Q6_K, A, 4, 256, MIS, None) == ALIGN
    assert f(kq.Q6_K, A, 0, 256, None, None) == OK


def test_moe_argument_checks(lib):
    s = lib.kq_moe_sort
    assert s(A, 4, 0, 8, None, 0, A, A, None, None, None, None) == INVALID      # top_k < 1
    assert s(A, 4, 2, 0, None, 0, A, A, None, None, None, None) == INVALID      # no experts
    assert s(A, 4, 2, 257, None, 0, A, A, None, None, None, None) == INVALID
    assert s(A, 4, 2, 8, None, 64, A, A, None, A, None, None) == INVALID        # x_sorted without x
    assert s(A, 4, 2, 8, A, 60, A, A, A, A, None, None) == INVALID              # k % 8
    assert s(A, 2**62, 4, 8, None, 0, A, A, None, None, None, None) == INVALID  # no overflow of the count
    assert s(A, 4, 2, 8, A, 2**32, A, A, A, A, None, None) == INVALID           # k past 32-bit counts
    assert s(A, 0, 2, 8, None, 0, A, A, A, None, None, None) == OK
    t = lib.kq_expert_tile_map
    assert t(A, 1024, 8, A, 23, A, None, None) == INVALID                 # cap < ceil(1024/64) + 8
    assert t(A, 1024, 8, None, 24, A, None, None) == INVALID
    g = lib.kq_gather_qmm
    assert g(kq.Q4_K, A, 0, 64, 256, A, 10, A, A, 8, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 250, A, 10, A, A, 8, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 256, None, 10, A, A, 8, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 256, MIS, 10, A, A, 8, A, None, None) == ALIGN
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, A, 8, A, None, None) == OK


def test_decode_moe_argument_checks(lib):
    g = lib.kq_gather_qmv
    assert g(3, A, 8, 64, 256, A, 0, A, 1, 2, A, None, None) == UNSUPPORTED      # unknown codec
    assert g(kq.Q4_K, A, 0, 64, 256, A, 0, A, 1, 2, A, None, None) == INVALID    # no experts
    assert g(kq.Q4_K, A, 257, 64, 256, A, 0, A, 1, 2, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 250, A, 0, A, 1, 2, A, None, None) == INVALID    # K not a block multiple
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, 1, 0, A, None, None) == INVALID    # top_k < 1
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, 4097, 2, A, None, None) == INVALID  # more than 8192 pairs
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, 2**62, 4, A, None, None) == INVALID  # no overflow of the count
    assert g(kq.Q4_K, A, 8, 64, 256, None, 0, A, 1, 2, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, None, 1, 2, A, None, None) == INVALID
    assert g(kq.Q4_K, A, 8, 64, 256, MIS, 0, A, 1, 2, A, None, None) == ALIGN
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, 1, 2, MIS, None, None) == ALIGN
    assert g(kq.Q4_K, A, 8, 64, 256, A, 0, A, 0, 2, A, None, None) == OK         # no tokens
    f = lib.kq_moe_glu_gather
    assert f(kq.Q4_K, A, A, 8, 64, 256, A, A, 1, 2, 3, 0.0, A, None, None) == INVALID    # unknown act
    assert f(kq.Q4_K, A, A, 8, 64, 256, A, A, 1, 2, 2, 0.0, A, None, None) == INVALID    # limit must be > 0
    assert f(kq.Q4_K, A, None, 8, 64, 256, A, A, 1, 2, 0, 0.0, A, None, None) == INVALID  # null up bank
    assert f(kq.Q4_K, A, MIS, 8, 64, 256, A, A, 1, 2, 0, 0.0, A, None, None) == ALIGN
    assert f(kq.Q4_K, A, A, 8, 64, 256, A, A, 0, 2, 2, 1.0, A, None, None) == OK
    m = lib.kq_gather_mix
    assert m(A, 8, 6, A, A, 4, 2, A, None, None) == INVALID                      # n % 4
    assert m(A, 8, 8, A, A, 4, 0, A, None, None) == INVALID                      # top_k < 1
    assert m(A, 8, 8, A, A, 4, 65, A, None, None) == INVALID                     # top_k > 64
    assert m(A, 8, 4 * 256 * 65536, A, A, 4, 2, A, None, None) == INVALID        # past the grid's x extent
    assert m(A, 8, 8, None, A, 4, 2, A, None, None) == INVALID
    assert m(A, 8, 8, A, A, 4, 2, MIS, None, None) == ALIGN
    assert m(MIS, 8, 8, A, A, 4, 2, A, None, None) == ALIGN
    assert m(A, 8, 8, A, A, 0, 2, A, None, None) == OK


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(kq, "_lib", None)
    monkeypatch.setattr(kq, "LIB_PATH", "/nonexistent/libkq.so")
    with pytest.raises(RuntimeError, match="missing"):
        kq.lib()
