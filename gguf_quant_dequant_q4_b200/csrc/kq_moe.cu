// Expert grouping for the sorted MoE prefill path, entirely on the device.
//
// kq_moe_sort: stable counting sort of the routed (token, slot) pairs by
//   expert id, plus the row gather x_sorted[r] = x[pair(r) / top_k]
//   (mlx-kquant README "Performance": sorted MoE prefill batches take a
//   per-expert-segment GEMM; bindings.cpp `gather_qmm_seg`: rows pre-sorted
//   by expert).
// kq_expert_tile_map: (expert, row_start, num_rows <= 64) tiles of every
//   expert segment, only the last tile of a segment partial, plus the tile
//   count (bindings.cpp `expert_tile_map`).  No host synchronization.
#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kSortThreads = 1024;
constexpr int kMaxExperts = 256;

// One CTA.  Pass 1 histograms the ids; pass 2 walks the pairs in chunks of
// 1024 in order, ranking equal ids within a warp with __match_any_sync and
// across the warps of the chunk with per-warp counts, so equal experts keep
// their (token, slot) order.
__global__ void __launch_bounds__(kSortThreads) moe_sort_kernel(const int32_t* __restrict__ ids, int rows, int n_experts,
                                                                 uint32_t* __restrict__ sorted_ids,
                                                                 int32_t* __restrict__ sorted_pair,
                                                                 int32_t* __restrict__ inv, int32_t* err) {
    __shared__ int base[kMaxExperts];
    __shared__ int wcount[kSortThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < kMaxExperts; e += kSortThreads) base[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int i = tid; i < rows; i += kSortThreads) {
        const int e = ids[i];
        if (e < 0 || e >= n_experts) bad = 1;
        else atomicAdd(&base[e], 1);
    }
    if (bad && err) atomicOr(err, KQ_DEV_BAD_EXPERT);
    __syncthreads();
    __shared__ int valid;
    if (tid == 0) {
        int acc = 0;
        for (int e = 0; e < n_experts; ++e) {
            const int c = base[e];
            base[e] = acc;
            acc += c;
        }
        valid = acc;
    }
    __syncthreads();
    // rows left over by invalid ids are marked (id 0xffffffff, pair -1)
    for (int i = valid + tid; i < rows; i += kSortThreads) {
        sorted_ids[i] = 0xffffffffu;
        sorted_pair[i] = -1;
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int c0 = 0; c0 < rows; c0 += kSortThreads) {
        for (int i = tid; i < (kSortThreads / 32) * kMaxExperts; i += kSortThreads) (&wcount[0][0])[i] = 0;
        __syncthreads();
        const int i = c0 + tid;
        int e = i < rows ? ids[i] : -1;
        if (e >= n_experts) e = -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & lt);
        if (e >= 0 && rank == 0) wcount[warp][e] = __popc(same);
        __syncthreads();
        if (e >= 0) {
            int pos = base[e] + rank;
            for (int w = 0; w < warp; ++w) pos += wcount[w][e];
            sorted_ids[pos] = static_cast<uint32_t>(e);
            sorted_pair[pos] = i;
            if (inv) inv[i] = pos;
        } else if (inv && i < rows) {
            inv[i] = -1;
        }
        __syncthreads();
        // advance the per-expert bases by this chunk's counts
        for (int ee = tid; ee < n_experts; ee += kSortThreads) {
            int s = 0;
            for (int w = 0; w < kSortThreads / 32; ++w) s += wcount[w][ee];
            base[ee] += s;
        }
        __syncthreads();
    }
}

// x_sorted[r] = x[sorted_pair[r] / top_k]: one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x, int64_t k,
                                                          const int32_t* __restrict__ pair, int rows, int top_k,
                                                          uint16_t* __restrict__ xs, const uint32_t* __restrict__ sids,
                                                          int n_experts) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    for (int r = warp; r < rows; r += nw) {
        if (sids[r] >= static_cast<uint32_t>(n_experts) || pair[r] < 0) continue;
        const int tok = pair[r] / top_k;
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(tok) * k);
        uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(r) * k);
        for (int64_t c = lane; c < k / 8; c += 32) dst[c] = __ldg(src + c);
    }
}

// One CTA: per-expert counts (and a sortedness check), prefix sums of rows
// and of tiles, then every expert writes its tiles in ascending row order.
__global__ void __launch_bounds__(1024) tile_map_kernel(const uint32_t* __restrict__ ids, int rows, int n_experts,
                                                         uint32_t* __restrict__ map, uint32_t* __restrict__ count,
                                                         int32_t* err) {
    __shared__ int cnt[kMaxExperts], rstart[kMaxExperts], tstart[kMaxExperts];
    const int tid = threadIdx.x;
    for (int e = tid; e < kMaxExperts; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int i = tid; i < rows; i += blockDim.x) {
        const uint32_t e = ids[i];
        if (i > 0 && ids[i - 1] > e) bad |= KQ_DEV_UNSORTED;
        if (e >= static_cast<uint32_t>(n_experts)) bad |= KQ_DEV_BAD_EXPERT;
        else atomicAdd(&cnt[e], 1);
    }
    if (bad && err) atomicOr(err, bad);
    __syncthreads();
    if (tid == 0) {
        int r = 0, t = 0;
        for (int e = 0; e < n_experts; ++e) {
            rstart[e] = r;
            tstart[e] = t;
            r += cnt[e];
            t += (cnt[e] + 63) / 64;
        }
        *count = static_cast<uint32_t>(t);
    }
    __syncthreads();
    for (int e = 0; e < n_experts; ++e) {
        const int nt = (cnt[e] + 63) / 64;
        for (int j = tid; j < nt; j += blockDim.x) {
            const int left = cnt[e] - 64 * j;
            uint32_t* m = map + 3 * static_cast<int64_t>(tstart[e] + j);
            m[0] = static_cast<uint32_t>(e);
            m[1] = static_cast<uint32_t>(rstart[e] + 64 * j);
            m[2] = static_cast<uint32_t>(left < 64 ? left : 64);
        }
    }
}

// out[t, c..c+3] = sum over s of scores[t, s] * y[inv[t k + s], c..c+3]:
// one thread per (token, 4 columns), 16-byte loads and stores, fp32 product
// then sum per slot in ascending order (explicitly rounded, never fused).
__global__ void __launch_bounds__(256) gather_mix_kernel(const float* __restrict__ y, int64_t rows, int64_t n4,
                                                          const int32_t* __restrict__ inv,
                                                          const float* __restrict__ scores, int64_t n_tokens,
                                                          int top_k, float* __restrict__ out, int32_t* err) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int64_t t = blockIdx.y; t < n_tokens; t += gridDim.y) {
        if (c >= n4) continue;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < top_k; ++s) {
            const int64_t r = __ldg(inv + t * top_k + s);
            if (r < 0 || r >= rows) {
                if (c == 0 && err) atomicOr(err, KQ_DEV_BAD_RANGE);
                continue;
            }
            const float sc = __ldg(scores + t * top_k + s);
            const float4 v = __ldcs(reinterpret_cast<const float4*>(y + r * n4 * 4) + c);
            acc.x = __fadd_rn(acc.x, __fmul_rn(sc, v.x));
            acc.y = __fadd_rn(acc.y, __fmul_rn(sc, v.y));
            acc.z = __fadd_rn(acc.z, __fmul_rn(sc, v.z));
            acc.w = __fadd_rn(acc.w, __fmul_rn(sc, v.w));
        }
        __stcs(reinterpret_cast<float4*>(out + t * n4 * 4) + c, acc);
    }
}

}  // namespace

int launch_moe_sort(const int32_t* topk_ids, int64_t n_tokens, int top_k, int n_experts, const uint16_t* x,
                    int64_t k, uint32_t* sorted_ids, int32_t* sorted_pair, int32_t* inv_order, uint16_t* x_sorted,
                    int32_t* err_flag, cudaStream_t s) {
    const int rows = static_cast<int>(n_tokens * top_k);
    if (rows == 0) return KQ_OK;
    moe_sort_kernel<<<1, kSortThreads, 0, s>>>(topk_ids, rows, n_experts, sorted_ids, sorted_pair, inv_order,
                                                err_flag);
    int rc = check_launch();
    if (rc || !x_sorted) return rc;
    int grid = (rows + 7) / 8;
    const int cap = device_sm_count() * 8;
    if (grid > cap) grid = cap;
    gather_rows_kernel<<<grid, 256, 0, s>>>(x, k, sorted_pair, rows, top_k, x_sorted, sorted_ids, n_experts);
    return check_launch();
}

int launch_tile_map(const uint32_t* sorted_ids, int64_t rows, int n_experts, uint32_t* map, int64_t cap,
                    uint32_t* count, int32_t* err_flag, cudaStream_t s) {
    (void)cap;
    tile_map_kernel<<<1, 1024, 0, s>>>(sorted_ids, static_cast<int>(rows), n_experts, map, count, err_flag);
    return check_launch();
}

int launch_gather_mix(const float* y, int64_t rows, int64_t n, const int32_t* inv_order, const float* scores,
                      int64_t n_tokens, int top_k, float* out, int32_t* err_flag, cudaStream_t s) {
    const int64_t n4 = n / 4;
    const int64_t bx = (n4 + 255) / 256;
    if (bx > 65535) return KQ_ERR_INVALID_ARG;
    const int64_t by = n_tokens < 65535 ? n_tokens : 65535;
    gather_mix_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(by)), 256, 0, s>>>(
        y, rows, n4, inv_order, scores, n_tokens, top_k, out, err_flag);
    return check_launch();
}

}  // namespace kq
