// Exact fp32 decode of 8 values of a q5_K or q4_0 block by one lane, shared by
// kq_dequantize and the decode-and-dot qmv of these codecs.  Layouts: ggml's
// block formats, sizes from the mlx-kquant README "Codec reference" table
// (q5_k 256 values / 176 B, q4_0 32 / 18 B).  Every operation is rounded as
// written: y = fp32(fp32(d) sc) q - fp32(fp32(dmin) m) (q5_K), fp32(d) (q - 8)
// (q4_0).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace kq {

__device__ __forceinline__ float dec_h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
// small non-negative integer -> float, exactly: its bits in the mantissa of
// 2^23, minus 2^23 (an FADD instead of an integer conversion); `bias` is
// subtracted in the same exact step (|result| < 2^23)
__device__ __forceinline__ float dec_i2f(uint32_t code, float bias) {
    return __fsub_rn(__uint_as_float(0x4B000000u | code), 8388608.0f + bias);
}
__device__ __forceinline__ uint32_t dec_ldg_u16(const uint8_t* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// q5_K superblock (16-byte aligned): values 8 lane .. +7, chunk c = lane/8,
// half (lane/4) % 2, l = 8 (lane % 4) .. +7: the nibble of qs[32c + l] (low for
// the first half) plus 16 times bit 2c + half of qh[l]; scale/min codes packed
// as in q4_K (j < 4: low six bits of s[j], s[j+4]; j >= 4: nibbles of s[j+4]
// with the top two bits of s[j-4], s[j]).  Loading and decoding are separate
// so that callers can have several blocks' loads in flight.
struct RawQ5K {
    uint2 q, hb;
    uint32_t dd;      // d | dmin << 16
    uint32_t sc_m;    // the lane's scale code | min code << 8
};
__device__ __forceinline__ RawQ5K load_q5k(const uint8_t* blk, int lane) {
    const int c = lane >> 3, li = lane & 7, j = 2 * c + (li >> 2);
    RawQ5K r;
    r.q = __ldg(reinterpret_cast<const uint2*>(blk + 48 + 32 * c + 8 * (li & 3)));
    r.hb = __ldg(reinterpret_cast<const uint2*>(blk + 16 + 8 * (li & 3)));
    r.dd = __ldg(reinterpret_cast<const unsigned int*>(blk));
    const uint8_t* s = blk + 4;
    int sc, m;
    if (j < 4) {
        sc = __ldg(s + j) & 63;
        m = __ldg(s + j + 4) & 63;
    } else {
        sc = (__ldg(s + j + 4) & 0x0f) | ((__ldg(s + j - 4) >> 6) << 4);
        m = (__ldg(s + j + 4) >> 4) | ((__ldg(s + j) >> 6) << 4);
    }
    r.sc_m = static_cast<uint32_t>(sc) | (static_cast<uint32_t>(m) << 8);
    return r;
}
__device__ __forceinline__ void decode_q5k(const RawQ5K& r, int lane, float (&v)[8]) {
    const int c = lane >> 3, half = (lane & 7) >> 2, j = 2 * c + half;
    const float d = dec_h2f(static_cast<uint16_t>(r.dd & 0xffff));
    const float dmin = dec_h2f(static_cast<uint16_t>(r.dd >> 16));
    const float dl = __fmul_rn(d, static_cast<float>(r.sc_m & 0xff));
    const float ml = __fmul_rn(dmin, static_cast<float>(r.sc_m >> 8));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t word = i < 4 ? r.q.x : r.q.y, hw = i < 4 ? r.hb.x : r.hb.y;
        const uint32_t code = ((word >> (8 * (i & 3) + 4 * half)) & 15) | (((hw >> (8 * (i & 3) + j)) & 1) << 4);
        v[i] = __fsub_rn(__fmul_rn(dl, dec_i2f(code, 0.0f)), ml);
    }
}
__device__ __forceinline__ void decode8_q5k(const uint8_t* blk, int lane, float (&v)[8]) {
    decode_q5k(load_q5k(blk, lane), lane, v);
}

// q4_0 block (2-byte aligned): values 8 part .. +7 (part 0..3); values 0..15
// are the low nibbles of qs[0..15], values 16..31 the high nibbles.
struct RawQ40 {
    uint32_t d;
    uint32_t two[4];
};
__device__ __forceinline__ RawQ40 load_q4_0(const uint8_t* blk, int part) {
    RawQ40 r;
    r.d = dec_ldg_u16(blk);
    const uint8_t* qs = blk + 2 + 8 * (part & 1);
#pragma unroll
    for (int p = 0; p < 4; ++p) r.two[p] = dec_ldg_u16(qs + 2 * p);
    return r;
}
__device__ __forceinline__ void decode_q4_0(const RawQ40& r, int part, float (&v)[8]) {
    const float d = dec_h2f(static_cast<uint16_t>(r.d));
    const int sh = 4 * (part >> 1);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        v[2 * p] = __fmul_rn(d, dec_i2f((r.two[p] >> sh) & 15, 8.0f));
        v[2 * p + 1] = __fmul_rn(d, dec_i2f((r.two[p] >> (8 + sh)) & 15, 8.0f));
    }
}
__device__ __forceinline__ void decode8_q4_0(const uint8_t* blk, int part, float (&v)[8]) {
    decode_q4_0(load_q4_0(blk, part), part, v);
}

}  // namespace kq
