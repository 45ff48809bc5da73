"""The C ABI as a C program sees it, on the CPU: include/kq.h compiles as
strict C99 and as C++, a C consumer (tests/c/abi_consumer.c) links
libkq.so, and the entry points that need no GPU answer as the header says."""
import os
import shutil
import subprocess

import pytest

import gguf_quant_dequant_q4_b200 as kq
from gguf_quant_dequant_q4_b200 import build as kqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
OK, INVALID, UNSUPPORTED, ALIGN = 0, 1, 2, 3

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None or shutil.which("g++") is None,
                                reason="no host C/C++ compiler")


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    lib = kqbuild.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path_factory.mktemp("c_abi") / "abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE,
                    os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", libdir, "-lkq",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return dict(line.split(" ", 1) for line in out.splitlines())


def test_header_compiles_as_cxx():
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                    "-I", INCLUDE, "-x", "c++", "-"], input='#include "kq.h"\nint main() { return KQ_OK; }\n',
                   text=True, check=True)


def test_block_geometry_and_status_strings(consumer):
    for qt in (kq.Q4_0, kq.Q8_0, kq.Q4_K, kq.Q5_K, kq.Q6_K):
        vpb, bpb = kq.block_info(qt)
        assert consumer[f"block_info_{qt}"] == f"{OK} {vpb} {bpb}"
    assert consumer["block_info_unknown"] == str(UNSUPPORTED)
    assert consumer["status_string_0"] == "ok"
    assert consumer["status_string_3"] == "pointer not 16-byte aligned"


def test_host_checks(consumer):
    expect = {"qmv_k_not_block_multiple": INVALID, "qmv_m_17": INVALID, "qmv_unknown_codec": UNSUPPORTED,
              "qmv_misaligned_w": ALIGN, "qmv_empty": OK, "qmm_null_x": INVALID, "dequantize_empty": OK,
              "gather_qmv_too_many_pairs": INVALID, "tile_map_small_cap": INVALID, "glu_bad_act": INVALID,
              "mix_n_not_multiple_of_4": INVALID}
    for name, rc in expect.items():
        assert consumer[name] == str(rc), name
