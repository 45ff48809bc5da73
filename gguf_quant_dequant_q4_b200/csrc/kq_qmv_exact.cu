// kq_qmv for q5_K and q4_0: y = x . W^T for 1 <= m <= 16, decode and dot in
// fp32 (mlx-kquant README "How it works": the scalar decode-then-dot matmul;
// bindings.cpp `quantized_matmul`).  These codecs have no tensor-core decode
// path here, so every weight is decoded exactly to fp32 (kq_decode.cuh) and
// multiplied by the bf16 activations (exact in fp32) with fp32 FMAs.
//
// One warp per weight row: q5_K lanes take 8 values of each 256-value block
// (the warp covers one block per step), q4_0 lanes take 8 values of one of
// eight 32-value blocks (the warp covers 256 values per step).  The activations
// are read through the read-only cache (every row reuses them); partial sums
// are reduced over the warp with shuffles in a fixed order (deterministic).
#include "kq_decode.cuh"
#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kWarpsPerCta = 8;

template <int QT, int MT>
__global__ void __launch_bounds__(kWarpsPerCta * 32) qmv_exact_kernel(const uint8_t* __restrict__ w, int64_t n,
                                                                     int64_t k, const uint16_t* __restrict__ x,
                                                                     int m, float* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = static_cast<int64_t>(gridDim.x) * kWarpsPerCta;
    const int64_t row_bytes = QT == KQ_Q5_K ? k / 256 * 176 : k / 32 * 18;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5); r < n; r += nw) {
        const uint8_t* row = w + r * row_bytes;
        float acc[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = 0.f;
        for (int64_t v0 = 0; v0 < k; v0 += 256) {
            float wv[8];
            int64_t col;   // first of the lane's 8 values
            if constexpr (QT == KQ_Q5_K) {
                decode8_q5k(row + (v0 / 256) * 176, lane, wv);
                col = v0 + 8 * lane;
            } else {
                const int64_t b = v0 / 32 + (lane >> 2);
                decode8_q4_0(row + b * 18, lane & 3, wv);
                col = b * 32 + 8 * (lane & 3);
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t < m) {
                    const uint4 xr = __ldg(reinterpret_cast<const uint4*>(x + t * k + col));
                    const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[t] = fmaf(wv[2 * i], __uint_as_float(xw[i] << 16), acc[t]);
                        acc[t] = fmaf(wv[2 * i + 1], __uint_as_float(xw[i] & 0xffff0000u), acc[t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t < m) y[t * n + r] = v;
        }
    }
}

template <int QT, int MT>
int launch_mt(const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y, cudaStream_t s) {
    int64_t grid = (n + kWarpsPerCta - 1) / kWarpsPerCta;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (grid > cap) grid = cap;
    qmv_exact_kernel<QT, MT><<<static_cast<unsigned>(grid), kWarpsPerCta * 32, 0, s>>>(
        static_cast<const uint8_t*>(w), n, k, x, m, y);
    return check_launch();
}

template <int QT>
int launch_codec_exact(const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y, cudaStream_t s) {
    if (k % 256 != 0) return KQ_ERR_UNSUPPORTED;   // whole warp steps of 256 values
    if (m <= 1) return launch_mt<QT, 1>(w, n, k, x, m, y, s);
    if (m <= 4) return launch_mt<QT, 4>(w, n, k, x, m, y, s);
    return launch_mt<QT, 16>(w, n, k, x, m, y, s);
}

}  // namespace

int launch_qmv_exact(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
                     cudaStream_t s) {
    switch (type) {
    case KQ_Q5_K: return launch_codec_exact<KQ_Q5_K>(w, n, k, x, m, y, s);
    case KQ_Q4_0: return launch_codec_exact<KQ_Q4_0>(w, n, k, x, m, y, s);
    default: return KQ_ERR_UNSUPPORTED;
    }
}

}  // namespace kq
