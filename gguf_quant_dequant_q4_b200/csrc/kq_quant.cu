// kq_quantize: fp32 weights -> GGUF wire bytes (q8_0, q4_K, q6_K).
//
// mlx-kquant bindings.cpp `quantize` (encode a float weight tensor into GGUF
// K-quant wire bytes; last dim a multiple of the codec's block); hanzo-ml
// quantized/mod.rs `QTensor::quantize`.  The pages give no encoding search, so
// the encoder is the plainest one the block formats allow:
//   q8_0  ggml's absmax rule: d = max|x| / 127, codes round(x * (1/d)) with
//         ties away from zero, d stored as binary16;
//   q4_K  per 32-value sub-block the range [min(0, min x), max x]: scale
//         (max - min) / 15 and min -min(0, min x); super-block scales
//         d = max scale / 63 and dmin = max min / 63 as binary16; 6-bit codes
//         round(scale / d) and round(min / dmin); value codes
//         round((x + dmin m_j) / (d sc_j)) in 0..15;
//   q6_K  per 16-value sub-block scale max|x| / 31; d = max scale / 127 as
//         binary16; int8 scale codes round(scale / d); value codes
//         round(x / (d sc_j)) in -32..31, stored + 32.
// Every step is one explicitly rounded fp32 operation in that order (the
// products d sc_j and dmin m_j are the decoder's own), so the bytes are
// reproducible; ties of signed zeros resolve as a sequential scan with strict
// comparisons would.
//
// One warp per 256 values (one q4_K / q6_K super-block or eight q8_0 blocks):
// lane l holds values 8l..8l+7 from two 16-byte loads (the warp reads 1 KB
// contiguous), sub-block statistics are shuffle reductions over the lanes of
// the sub-block, nibbles and 2-bit fields are paired across lanes by shuffles,
// and the block is assembled in shared memory, then stored with 16-byte
// (q4_K: 144 = 9 x 16 B, q8_0: 272 = 17 x 16 B per 8 blocks) or 2-byte
// (q6_K: 210 B) coalesced stores.  Bound: HBM (4 bytes read per value).
#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kWarps = 8;
constexpr int kStage = 288;   // shared staging bytes per warp (>= 272)

__device__ __forceinline__ int clampi(float v, int lo, int hi) {
    const int q = static_cast<int>(v);
    return q < lo ? lo : (q > hi ? hi : q);
}
// strict comparisons: the kept value wins ties, as in a sequential scan
__device__ __forceinline__ float kmax(float a, float b) { return b > a ? b : a; }
__device__ __forceinline__ float kmin(float a, float b) { return b < a ? b : a; }
template <int W>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = 1; o < W; o <<= 1) v = kmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int W>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
    for (int o = 1; o < W; o <<= 1) v = kmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
// maximum over the warp of values clipped below at +0 (a scan from +0 with
// strict comparisons never keeps -0)
__device__ __forceinline__ float warp_max_pos(float v) { return group_max<32>(v > 0.0f ? v : 0.0f); }

__device__ __forceinline__ uint32_t pack4(const int (&b)[8], int i0) {
    return static_cast<uint32_t>(b[i0] & 0xff) | (static_cast<uint32_t>(b[i0 + 1] & 0xff) << 8) |
           (static_cast<uint32_t>(b[i0 + 2] & 0xff) << 16) | (static_cast<uint32_t>(b[i0 + 3] & 0xff) << 24);
}

template <int QT>
__global__ void __launch_bounds__(kWarps * 32) quantize_kernel(const float* __restrict__ x, int64_t groups,
                                                               int64_t nvals, uint8_t* __restrict__ out) {
    __shared__ __align__(16) uint8_t stage_all[kWarps * kStage];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* st = stage_all + warp * kStage;
    const int64_t nw = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * kWarps + warp; g < groups; g += nw) {
        const int64_t v0 = g * 256 + 8 * lane;
        float v[8];
        const bool in = v0 < nvals;   // q8_0: the last group may hold fewer than 8 blocks
        if (in) {
            const float4 a = __ldcs(reinterpret_cast<const float4*>(x + v0));
            const float4 b = __ldcs(reinterpret_cast<const float4*>(x + v0) + 1);
            v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
        if constexpr (QT == KQ_Q8_0) {
            // block l/4, 4 lanes per block
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) a = kmax(a, fabsf(v[i]));
            a = group_max<4>(a);
            const float d = __fdiv_rn(a, 127.0f);
            const float id = d == 0.0f ? 0.0f : __fdiv_rn(1.0f, d);
            int q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = clampi(roundf(__fmul_rn(v[i], id)), -128, 127);
            const int b = lane >> 2;
            uint8_t* bb = st + 34 * b;
            if ((lane & 3) == 0) *reinterpret_cast<uint16_t*>(bb) = __half_as_ushort(__float2half_rn(d));
#pragma unroll
            for (int i = 0; i < 8; i += 2)
                *reinterpret_cast<uint16_t*>(bb + 2 + 8 * (lane & 3) + i) =
                    static_cast<uint16_t>((q[i] & 0xff) | ((q[i + 1] & 0xff) << 8));
            __syncwarp();
            const int64_t nb_left = (nvals - g * 256) / 32;
            uint8_t* o = out + g * 272;
            if (nb_left >= 8) {
                if (lane < 17) reinterpret_cast<uint4*>(o)[lane] = reinterpret_cast<const uint4*>(st)[lane];
            } else {
                for (int h = lane; h < 17 * nb_left; h += 32)
                    reinterpret_cast<uint16_t*>(o)[h] = reinterpret_cast<const uint16_t*>(st)[h];
            }
        } else if constexpr (QT == KQ_Q4_K) {
            // sub-block l/4 (32 values on 4 lanes)
            float lo = 0.0f, hi = v[0];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                lo = kmin(lo, v[i]);
                hi = kmax(hi, v[i]);
            }
            lo = group_min<4>(lo);
            hi = group_max<4>(hi);
            const float s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
            const float mn = -lo;
            const float smax = warp_max_pos(s), mmax = warp_max_pos(mn);
            const __half hd = __float2half_rn(__fdiv_rn(smax, 63.0f));
            const __half hm = __float2half_rn(__fdiv_rn(mmax, 63.0f));
            const float df = __half2float(hd), dmf = __half2float(hm);
            const int sc = df > 0.0f ? clampi(roundf(__fdiv_rn(s, df)), 0, 63) : 0;
            const int m = dmf > 0.0f ? clampi(roundf(__fdiv_rn(mn, dmf)), 0, 63) : 0;
            const float ds = __fmul_rn(df, static_cast<float>(sc));
            const float dm = __fmul_rn(dmf, static_cast<float>(m));
            int q[8], hq[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                q[i] = ds > 0.0f ? clampi(roundf(__fdiv_rn(__fadd_rn(v[i], dm), ds)), 0, 15) : 0;
            // value 64c + w: low nibble of byte 32c + w (w < 32), else high nibble of 32c + w - 32;
            // lane l holds w = 8(l%8)..+7 of c = l/8, its high-nibble partner is lane l + 4
#pragma unroll
            for (int i = 0; i < 8; ++i) hq[i] = __shfl_down_sync(0xffffffffu, q[i], 4);
            int scj[8], mj[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                scj[j] = __shfl_sync(0xffffffffu, sc, 4 * j);
                mj[j] = __shfl_sync(0xffffffffu, m, 4 * j);
            }
            if ((lane & 7) < 4) {
                int byt[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) byt[i] = q[i] | (hq[i] << 4);
                *reinterpret_cast<uint2*>(st + 16 + 32 * (lane >> 3) + 8 * (lane & 7)) =
                    make_uint2(pack4(byt, 0), pack4(byt, 4));
            }
            if (lane == 0) {
                // 6-bit codes: j < 4 in the low six bits of s[j] (scale) and
                // s[j+4] (min); j >= 4 low nibbles in s[j+4], top two bits in
                // the top bits of s[j-4] (scale) and s[j] (min)
                int sb[8], hb[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sb[j] = scj[j] | ((scj[j + 4] >> 4) << 6);
                    sb[j + 4] = mj[j] | ((mj[j + 4] >> 4) << 6);
                    hb[j] = (scj[j + 4] & 15) | ((mj[j + 4] & 15) << 4);
                }
                uint4 hdr;
                hdr.x = static_cast<uint32_t>(__half_as_ushort(hd)) | (static_cast<uint32_t>(__half_as_ushort(hm)) << 16);
                hdr.y = pack4(sb, 0);
                hdr.z = pack4(sb, 4);
                hdr.w = static_cast<uint32_t>(hb[0]) | (static_cast<uint32_t>(hb[1]) << 8) |
                        (static_cast<uint32_t>(hb[2]) << 16) | (static_cast<uint32_t>(hb[3]) << 24);
                *reinterpret_cast<uint4*>(st) = hdr;
            }
            __syncwarp();
            if (lane < 9) reinterpret_cast<uint4*>(out + g * 144)[lane] = reinterpret_cast<const uint4*>(st)[lane];
        } else {
            // q6_K: sub-block l/2 (16 values on 2 lanes); value 128h + 32t + l'' with
            // h = l/16, t = (l/4)%4, l'' = 8(l%4) + i
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) a = kmax(a, fabsf(v[i]));
            a = group_max<2>(a);
            const float s = __fdiv_rn(a, 31.0f);
            const float smax = warp_max_pos(s);
            const __half hd = __float2half_rn(__fdiv_rn(smax, 127.0f));
            const float df = __half2float(hd);
            const int sc = df > 0.0f ? clampi(roundf(__fdiv_rn(s, df)), -128, 127) : 0;
            const float ds = __fmul_rn(df, static_cast<float>(sc));
            int c[8], c8[8], h4[8], h8[8], h12[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = (ds > 0.0f ? clampi(roundf(__fdiv_rn(v[i], ds)), -32, 31) : 0) + 32;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c8[i] = __shfl_down_sync(0xffffffffu, c[i], 8);
                h4[i] = __shfl_down_sync(0xffffffffu, c[i] >> 4, 4);
                h8[i] = __shfl_down_sync(0xffffffffu, c[i] >> 4, 8);
                h12[i] = __shfl_down_sync(0xffffffffu, c[i] >> 4, 12);
            }
            const int h = lane >> 4, t = (lane >> 2) & 3, lq = 8 * (lane & 3);
            if (t < 2) {
                // ql[64h + 32t + l'']: low nibble from quarter t, high nibble from t + 2
                int byt[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) byt[i] = (c[i] & 15) | ((c8[i] & 15) << 4);
                *reinterpret_cast<uint2*>(st + 64 * h + 32 * t + lq) = make_uint2(pack4(byt, 0), pack4(byt, 4));
            }
            if (t == 0) {
                // qh[32h + l'']: the 2-bit high fields of quarters 0..3
                int byt[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) byt[i] = (c[i] >> 4) | (h4[i] << 2) | (h8[i] << 4) | (h12[i] << 6);
                *reinterpret_cast<uint2*>(st + 128 + 32 * h + lq) = make_uint2(pack4(byt, 0), pack4(byt, 4));
            }
            if ((lane & 1) == 0) st[192 + (lane >> 1)] = static_cast<uint8_t>(static_cast<int8_t>(sc));
            if (lane == 0) *reinterpret_cast<uint16_t*>(st + 208) = __half_as_ushort(hd);
            __syncwarp();
            uint16_t* o = reinterpret_cast<uint16_t*>(out + g * 210);
            for (int k2 = lane; k2 < 105; k2 += 32) o[k2] = reinterpret_cast<const uint16_t*>(st)[k2];
        }
        __syncwarp();   // the staging buffer is reused by the next group
    }
}

}  // namespace

int launch_quantize(int type, const float* x, int64_t n_rows, int64_t k, void* out, cudaStream_t s) {
    const int64_t nvals = n_rows * k;
    const int64_t groups = (nvals + 255) / 256;
    int64_t grid = (groups + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
    if (grid > cap) grid = cap;
    uint8_t* o = static_cast<uint8_t*>(out);
    switch (type) {
    case KQ_Q8_0: quantize_kernel<KQ_Q8_0><<<static_cast<unsigned>(grid), kWarps * 32, 0, s>>>(x, groups, nvals, o); break;
    case KQ_Q4_K: quantize_kernel<KQ_Q4_K><<<static_cast<unsigned>(grid), kWarps * 32, 0, s>>>(x, groups, nvals, o); break;
    case KQ_Q6_K: quantize_kernel<KQ_Q6_K><<<static_cast<unsigned>(grid), kWarps * 32, 0, s>>>(x, groups, nvals, o); break;
    default: return KQ_ERR_UNSUPPORTED;
    }
    return check_launch();
}

}  // namespace kq
