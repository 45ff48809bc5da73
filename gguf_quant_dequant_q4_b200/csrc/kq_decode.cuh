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
__device__ __forceinline__ uint32_t dec_ldg_u16(const uint8_t* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// q5_K superblock (16-byte aligned): values 8 lane .. +7, chunk c = lane/8,
// half (lane/4) % 2, l = 8 (lane % 4) .. +7: the nibble of qs[32c + l] (low for
// the first half) plus 16 times bit 2c + half of qh[l]; scale/min codes packed
// as in q4_K (j < 4: low six bits of s[j], s[j+4]; j >= 4: nibbles of s[j+4]
// with the top two bits of s[j-4], s[j]).
__device__ __forceinline__ void decode8_q5k(const uint8_t* blk, int lane, float (&v)[8]) {
    const uint4 h = __ldg(reinterpret_cast<const uint4*>(blk));
    const float d = dec_h2f(static_cast<uint16_t>(h.x & 0xffff));
    const float dmin = dec_h2f(static_cast<uint16_t>(h.x >> 16));
    const int c = lane >> 3, li = lane & 7, half = li >> 2;
    const int j = 2 * c + half;
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(blk + 48 + 32 * c + 8 * (li & 3)));
    const uint2 hb = __ldg(reinterpret_cast<const uint2*>(blk + 16 + 8 * (li & 3)));
    const uint8_t* s = blk + 4;
    int sc, m;
    if (j < 4) {
        sc = __ldg(s + j) & 63;
        m = __ldg(s + j + 4) & 63;
    } else {
        sc = (__ldg(s + j + 4) & 0x0f) | ((__ldg(s + j - 4) >> 6) << 4);
        m = (__ldg(s + j + 4) >> 4) | ((__ldg(s + j) >> 6) << 4);
    }
    const float dl = __fmul_rn(d, static_cast<float>(sc));
    const float ml = __fmul_rn(dmin, static_cast<float>(m));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t word = i < 4 ? q.x : q.y, hw = i < 4 ? hb.x : hb.y;
        const int code = ((word >> (8 * (i & 3) + 4 * half)) & 15) | (((hw >> (8 * (i & 3) + j)) & 1) << 4);
        v[i] = __fsub_rn(__fmul_rn(dl, static_cast<float>(code)), ml);
    }
}

// q4_0 block (2-byte aligned): values 8 part .. +7 (part 0..3); values 0..15
// are the low nibbles of qs[0..15], values 16..31 the high nibbles.
__device__ __forceinline__ void decode8_q4_0(const uint8_t* blk, int part, float (&v)[8]) {
    const float d = dec_h2f(static_cast<uint16_t>(dec_ldg_u16(blk)));
    const uint8_t* qs = blk + 2 + 8 * (part & 1);
    const int sh = 4 * (part >> 1);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t two = dec_ldg_u16(qs + 2 * p);
        v[2 * p] = __fmul_rn(d, static_cast<float>(static_cast<int>((two >> sh) & 15) - 8));
        v[2 * p + 1] = __fmul_rn(d, static_cast<float>(static_cast<int>((two >> (8 + sh)) & 15) - 8));
    }
}

}  // namespace kq
