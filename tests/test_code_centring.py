"""The decode kernels centre each code on its format's offset in binary16
before the MMA: the code's bits as a subnormal (code 2^-24) minus the offset
as a subnormal, one IEEE binary16 subtraction.  These checks restate that
arithmetic with numpy's IEEE binary16 (subnormals kept) for every code of
every format: the difference is exactly (code - offset) 2^-24, so a code
equal to the offset gives an exact zero operand.  They pin the bit patterns
the kernels use (byte ^ 0x80 for q8_0, nibble in place for the high half)."""
import numpy as np

U = np.float16(2.0 ** -24)   # the smallest binary16 subnormal


def sub16(a_bits, b_bits):
    a = np.array(a_bits, np.uint16).view(np.float16)
    b = np.array(b_bits, np.uint16).view(np.float16)
    return (a - b).astype(np.float64)


def test_binary16_subnormal_unit():
    assert np.float16(1).view(np.uint16) == 0x3C00
    assert np.array(1, np.uint16).view(np.float16) == U
    assert float(U) == 2.0 ** -24


def test_q8_0_codes_centred_exactly():
    # int8 code c as its byte b; the kernel's operand (b ^ 0x80) is 128 + c
    codes = np.arange(-128, 128)
    b = codes.astype(np.int8).view(np.uint8).astype(np.uint16)
    got = sub16(b ^ 0x80, np.full_like(b, 0x80))
    assert np.array_equal(got, codes * 2.0 ** -24)
    assert got[codes == 0][0] == 0.0


def test_q4_0_codes_centred_exactly():
    q = np.arange(16, dtype=np.uint16)
    lo = sub16(q, np.full_like(q, 8))                  # low nibble: (q - 8) 2^-24
    hi = sub16(q << 4, np.full_like(q, 0x80))          # high nibble in place: 16 (q - 8) 2^-24
    assert np.array_equal(lo, (q.astype(np.int64) - 8) * 2.0 ** -24)
    assert np.array_equal(hi, 16 * (q.astype(np.int64) - 8) * 2.0 ** -24)
    assert lo[8] == 0.0 and hi[8] == 0.0


def test_q6_K_codes_centred_exactly():
    c6 = np.arange(64, dtype=np.uint16)
    lo = sub16(c6, np.full_like(c6, 0x20))             # c6 - 32
    hi = sub16(c6 << 4, np.full_like(c6, 0x200))       # 16 (c6 - 32), still subnormal (< 1024 2^-24)
    assert np.all((c6 << 4) < 0x400)
    assert np.array_equal(lo, (c6.astype(np.int64) - 32) * 2.0 ** -24)
    assert np.array_equal(hi, 16 * (c6.astype(np.int64) - 32) * 2.0 ** -24)
    # the general kernel centres only the high 2-bit field h (4^tq h - 2 4^tq)
    for tq in range(4):
        h = np.arange(4, dtype=np.uint16) << (2 * tq)
        got = sub16(h, np.full_like(h, 2 << (2 * tq)))
        assert np.array_equal(got, (np.arange(4) - 2) * 4.0 ** tq * 2.0 ** -24)


def test_centred_products_are_exact_in_fp32():
    # a centred code times a binary16 activation is exact in fp32 (at most
    # 11 + 9 significant bits), so one code equal to the offset contributes
    # exactly 0 next to any activation, however large
    rng = np.random.default_rng(0)
    a = rng.standard_normal(1000).astype(np.float16)
    for code in (-128, -1, 0, 1, 127, 496):
        prod32 = (np.float32(code * 2.0 ** -24) * a.astype(np.float32)).astype(np.float64)
        assert np.array_equal(prod32, code * 2.0 ** -24 * a.astype(np.float64))
