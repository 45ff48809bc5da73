// kq_dequantize: GGUF wire bytes -> fp32, bit-exact.
//
// mlx-kquant bindings.cpp, `dequantize`; hanzo-ml quantized/mod.rs,
// `QTensor::dequantize` (to_float into f32).  Block sizes: mlx-kquant README,
// "Codec reference".  The decode order is fixed and every operation is a
// separately rounded fp32 op (__fmul_rn / __fsub_rn, never an FMA):
//   q4_K  (d*sc)*q - (dmin*m)     q6_K  (d*sc)*q     q8_0  d*q
//
// The kernel is write-bound (4 bytes out per 0.56..1.06 bytes in): one warp
// decodes one 256-value superblock (q4_K, q6_K) or eight 32-value blocks
// (q8_0) per step, every lane producing 8 consecutive outputs stored as two
// 16-byte streaming stores, so a warp writes 1 KB contiguously.
#include "kq_decode.cuh"
#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

__device__ __forceinline__ void store8(float* out, const float (&v)[8]) {
    float4* o = reinterpret_cast<float4*>(out);
    __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
    __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint16_t ldg_u16(const uint8_t* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// q4_K superblock b: lane i writes values 8i..8i+7.  Values 64c..64c+31 are
// the low nibbles of qs[32c..32c+31] (sub-block 2c), 64c+32..64c+63 the high
// nibbles of the same bytes (sub-block 2c+1).
__device__ __forceinline__ void dq_q4k(const uint8_t* blk, float* out, int lane) {
    const uint4 h = __ldg(reinterpret_cast<const uint4*>(blk));
    const float d = h2f(static_cast<uint16_t>(h.x & 0xffff));
    const float dmin = h2f(static_cast<uint16_t>(h.x >> 16));
    const int c = lane >> 3, li = lane & 7;
    const int j = 2 * c + (li >> 2);                 // sub-block of the 8 values
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(blk + 16 + 32 * c + 8 * (li & 3)));
    const uint8_t* s = blk + 4;
    int sc, m;
    if (j < 4) {
        sc = s[j] & 63;
        m = s[j + 4] & 63;
    } else {
        sc = (s[j + 4] & 0x0f) | ((s[j - 4] >> 6) << 4);
        m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
    const float dl = __fmul_rn(d, static_cast<float>(sc));
    const float ml = __fmul_rn(dmin, static_cast<float>(m));
    const int shift = (li >> 2) * 4;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t word = i < 4 ? q.x : q.y;
        const int code = (word >> (8 * (i & 3) + shift)) & 15;
        v[i] = __fsub_rn(__fmul_rn(dl, static_cast<float>(code)), ml);
    }
    store8(out + 8 * lane, v);
}

// q6_K superblock (2-byte aligned in memory): lane i writes values
// v = 8i..8i+7, v = 128h + 32t + l.  Low 4 bits: nibble t>>1 of
// ql[64h + 32(t&1) + l]; high 2 bits: bits 2t of qh[32h + l]; q = code - 32;
// scale sc[v/16].
__device__ __forceinline__ void dq_q6k(const uint8_t* blk, float* out, int lane) {
    const int v0 = 8 * lane;
    const int h = v0 >> 7, t = (v0 & 127) >> 5, l0 = v0 & 31;
    const uint8_t* ql = blk + 64 * h + 32 * (t & 1) + l0;
    const uint8_t* qh = blk + 128 + 32 * h + l0;
    const float d = h2f(ldg_u16(blk + 208));
    const int sc = static_cast<int8_t>(__ldg(blk + 192 + (v0 >> 4)));
    const float dl = __fmul_rn(d, static_cast<float>(sc));
    uint32_t lo[2], hi[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        lo[p] = ldg_u16(ql + 4 * p) | (static_cast<uint32_t>(ldg_u16(ql + 4 * p + 2)) << 16);
        hi[p] = ldg_u16(qh + 4 * p) | (static_cast<uint32_t>(ldg_u16(qh + 4 * p + 2)) << 16);
    }
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int lo4 = (lo[i >> 2] >> (8 * (i & 3) + 4 * (t >> 1))) & 15;
        const int hi2 = (hi[i >> 2] >> (8 * (i & 3) + 2 * t)) & 3;
        const int q = (lo4 | (hi2 << 4)) - 32;
        v[i] = __fmul_rn(dl, static_cast<float>(q));
    }
    store8(out + v0, v);
}

// q8_0: lane i handles block (i >> 2) of the warp's eight, values 8(i&3)..+7.
__device__ __forceinline__ void dq_q8_0(const uint8_t* blk, float* out, int part) {
    const float d = h2f(ldg_u16(blk));
    const uint8_t* qs = blk + 2 + 8 * part;
    float v[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t two = ldg_u16(qs + 2 * p);
        v[2 * p] = __fmul_rn(d, static_cast<float>(static_cast<int8_t>(two & 0xff)));
        v[2 * p + 1] = __fmul_rn(d, static_cast<float>(static_cast<int8_t>(two >> 8)));
    }
    store8(out + 8 * part, v);
}

// q5_K superblock b: lane i writes values 8i..8i+7 (decode in kq_decode.cuh).
__device__ __forceinline__ void dq_q5k(const uint8_t* blk, float* out, int lane) {
    float v[8];
    decode8_q5k(blk, lane, v);
    store8(out + 8 * lane, v);
}

// q4_0: lane i handles block (i >> 2) of the warp's eight, values 8(i&3)..+7.
__device__ __forceinline__ void dq_q4_0(const uint8_t* blk, float* out, int part) {
    float v[8];
    decode8_q4_0(blk, part, v);
    store8(out + 8 * part, v);
}

template <int QT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ w, int64_t nblocks,
                                                      float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    if constexpr (QT == KQ_Q4_K) {
        for (int64_t b = warp; b < nblocks; b += nwarps) dq_q4k(w + b * 144, out + b * 256, lane);
    } else if constexpr (QT == KQ_Q6_K) {
        for (int64_t b = warp; b < nblocks; b += nwarps) dq_q6k(w + b * 210, out + b * 256, lane);
    } else if constexpr (QT == KQ_Q5_K) {
        for (int64_t b = warp; b < nblocks; b += nwarps) dq_q5k(w + b * 176, out + b * 256, lane);
    } else {
        const int64_t units = (nblocks + 7) / 8;
        for (int64_t u = warp; u < units; u += nwarps) {
            const int64_t b = u * 8 + (lane >> 2);
            if (b < nblocks) {
                if constexpr (QT == KQ_Q4_0) dq_q4_0(w + b * 18, out + b * 32, lane & 3);
                else dq_q8_0(w + b * 34, out + b * 32, lane & 3);
            }
        }
    }
}

}  // namespace

int launch_dequantize(int type, const void* w, int64_t n_rows, int64_t k, float* out, cudaStream_t s) {
    const bool small = type == KQ_Q8_0 || type == KQ_Q4_0;   // 32-value blocks, eight per warp
    const int vpb = small ? 32 : 256;
    const int64_t nblocks = n_rows * (k / vpb);
    if (nblocks == 0) return KQ_OK;
    const int64_t units = small ? (nblocks + 7) / 8 : nblocks;
    const int sms = device_sm_count();
    int64_t grid = (units + 7) / 8;
    if (grid > static_cast<int64_t>(sms) * 16) grid = static_cast<int64_t>(sms) * 16;
    const uint8_t* wb = static_cast<const uint8_t*>(w);
    switch (type) {
    case KQ_Q4_K: dequant_kernel<KQ_Q4_K><<<static_cast<int>(grid), 256, 0, s>>>(wb, nblocks, out); break;
    case KQ_Q6_K: dequant_kernel<KQ_Q6_K><<<static_cast<int>(grid), 256, 0, s>>>(wb, nblocks, out); break;
    case KQ_Q5_K: dequant_kernel<KQ_Q5_K><<<static_cast<int>(grid), 256, 0, s>>>(wb, nblocks, out); break;
    case KQ_Q4_0: dequant_kernel<KQ_Q4_0><<<static_cast<int>(grid), 256, 0, s>>>(wb, nblocks, out); break;
    case KQ_Q8_0: dequant_kernel<KQ_Q8_0><<<static_cast<int>(grid), 256, 0, s>>>(wb, nblocks, out); break;
    default: return KQ_ERR_UNSUPPORTED;
    }
    return check_launch();
}

}  // namespace kq
