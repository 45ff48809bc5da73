// kq_qmv: y = x . W^T for 1 <= m <= 16 activation rows (decode shape).
//
// mlx-kquant bindings.cpp `quantized_matmul` (x @ dequant(w).T); README "How
// it works": small row counts take a kernel that amortizes each weight read
// over all rows (`verify_qmv`); hanzo-ml quantized/mod.rs: decode runs the
// quantized matvec directly on the packed blocks.
//
// The path is HBM-bound, so the design goal is to spend as few instructions
// per weight as possible while reading every weight byte exactly once:
//
//  * One CTA per SM (at most) owns a balanced contiguous range of weight rows,
//    walked in 16-row groups, and all of K.  Its row segments (several blocks
//    per row) are streamed into a ring of shared-memory stages by 1-D bulk
//    async copies (one per row, issued by a producer warp, completion counted
//    on an mbarrier; rows that are not a 16-byte multiple are staged with
//    2-byte loads instead), so many kilobytes per SM are in flight without
//    registers.
//  * 16 consumer warps split the blocks of a stage.  A warp decodes its 16 rows into
//    m16n8k16 tensor-core A fragments whose entries are EXACT integers in
//    binary16: the codes themselves (q6_K, q8_0) or code * 6-bit scale
//    (q4_K, at most 945).  The activations, rounded once to binary16, are the
//    B fragments (pre-permuted per CTA into a shared-memory "image" so each
//    fragment is one 8-byte load).  The tensor core forms exact products and
//    accumulates them in fp32, so the only rounding besides fp32 summation is
//    x -> binary16.
//  * Binary16 codes: q4_K ORs its 4-bit code into the mantissa of 1024.0
//    (1024 + code, exactly) and removes the 1024 with the HFMA2 that also
//    applies its scale; q6_K and q8_0 put the code's bits in the mantissa with
//    exponent field 0, a subnormal code x 2^-24 (exact; the tensor core keeps
//    subnormal operands exact), and subtract the codec's own offset from that
//    subnormal before the MMA (q8_0: 128, q6_K: 2 from its high 2-bit field),
//    exactly, so that a zero weight contributes exactly zero; the 2^24 goes
//    into the per-block scale.
//  * q4_K (per-block scales d, dmin): each lane owns one 64-value group of a
//    block, so it decodes only its own two 6-bit scale/min pairs; the MMA
//    chain runs over the whole block and the min term sum_j m_j * X_j is one
//    more MMA on (m_j) x (X_j split into two binary16 halves).
//  * q6_K / q8_0 (per-16- or per-32-value scales): the chain stops at every
//    sub-block.  For m <= 4 the 8 MMA columns are shared out as
//    (token, sub-block slot) pairs, so one epilogue covers up to 8 sub-blocks
//    instead of wasting 7 of 8 columns.
//  * Activation range: before the binary16 rounding each token's activations
//    (per super-chunk of K) are multiplied by a power of two that puts their
//    largest magnitude at 2^T; the warps multiply their partial sums by the
//    inverse, so the relative precision does not depend on the scale of x.
//  * Partial sums of the 16 consumer warps go to shared memory and a reducer
//    warp adds them in a fixed order and stores y: no atomics, bitwise
//    reproducible.
#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kCWarps = 16;                 // consumer warps
constexpr int kProducerWarp = kCWarps;      // bulk-copy producer
constexpr int kReducerWarp = kCWarps + 1;   // cross-warp reduction and stores
constexpr int kThreads = 32 * (kCWarps + 2);
constexpr int kRows = 16;
constexpr int kOffW = 512;   // barriers, flags, a zero word and the activation scales live below
constexpr int kXMax = 320;   // largest |x| per token, bf16 bits, two buffers of 16 words
constexpr int kXInv = 448;   // inverse activation scale per token (16 floats)
constexpr int kMaxStages = 8;

template <int QT> struct Codec;
// Stage geometry is chosen per call: a stage is 16 rows x g blocks, g a
// multiple of GA (so every per-row copy starts 16-byte aligned), as large as
// shared memory allows; rows are padded to a stride of 16 mod 128 bytes.
// XT: target exponent of the scaled activations (largest magnitude in
// [2^XT, 2^(XT+1))): q4_K keeps its 32-value sums inside binary16 range,
// q6_K and q8_0 keep their smallest operands (x/256, x/64) normal.
template <> struct Codec<KQ_Q4_K> {
    static constexpr int VPB = 256, BPB = 144, GA = 8, XT = 9;
    static constexpr int IMG = 544;   // B image bytes per (token, block)
};
template <> struct Codec<KQ_Q6_K> {
    static constexpr int VPB = 256, BPB = 210, GA = 8, XT = 14;
    static constexpr int IMG = 1024;
};
template <> struct Codec<KQ_Q8_0> {
    static constexpr int VPB = 32, BPB = 34, GA = 8, XT = 14;
    static constexpr int IMG = 64;
};

struct QmvParams {
    const uint8_t* w;
    const uint16_t* x;
    float* y;
    int* status;
    int64_t n, k, row_bytes;
    int m, nblk, scb, ns, bulk, g, rs;
    uint32_t tokstride, off_img, off_pbuf, off_racc;
};

// binary16 constants
constexpr uint32_t kH1024 = 0x64006400u;    // (1024, 1024)
constexpr uint32_t kHm1024 = 0xE400E400u;   // (-1024, -1024)
constexpr uint32_t kH1_16 = 0x2C002C00u;    // (1/16, 1/16)
constexpr float kTwo24 = 16777216.0f;        // 2^24: a subnormal code's unit is 2^-24

// Shared-memory loads are volatile so that they are never moved across the
// mbarrier waits and __syncthreads that order them with the bulk copies.
__device__ __forceinline__ uint32_t lds32c(uint32_t a) { return lds32(a); }
__device__ __forceinline__ uint2 lds64c(uint32_t a) { return lds64(a); }
__device__ __forceinline__ uint4 lds128c(uint32_t a) { return lds128(a); }
__device__ __forceinline__ uint32_t ldsu16c(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ int ldss8c(uint32_t a) {
    int16_t v;
    asm volatile("ld.shared.s8 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
// 4 bytes at a 2-byte aligned address; `odd` = (a & 2) is warp-uniform.
__device__ __forceinline__ uint32_t lds32c_a2(uint32_t a, bool odd) {
    if (!odd) return lds32c(a);
    return __byte_perm(lds32c(a - 2), lds32c(a + 2), 0x5432);
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y));
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t x) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(x));
}
__device__ __forceinline__ float h16(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// Scaled bf16 pair -> binary16 pair, and the two binary16 values back as floats.
__device__ __forceinline__ uint32_t f16pair(float a, float b, float S) { return pack_f16x2(a * S, b * S); }
__device__ __forceinline__ float f16sum(uint32_t h) { return h16(h & 0xffff) + h16(h >> 16); }
// Scale 2^s of token m for the codec's target exponent (see xscale_exp).
template <int QT>
__device__ __forceinline__ float tok_scale(const uint32_t* xm, int m) {
    return exp2_int(xscale_exp(xm[m], Codec<QT>::XT));
}

// Largest |x| of every token over values [v0, v0 + nv) of K, as bf16 bit
// patterns, by atomic max into xm[token] (zeroed beforehand).  All consumer
// warps take part: 16 / m warps per token, each lane loading up to eight
// 16-byte chunks before it reduces, so the loads overlap.
__device__ void x_range(const QmvParams& p, int64_t v0, int nv, uint32_t* xm) {
    constexpr int U = 8;
    const int chunks = nv / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpt = p.m < kCWarps ? kCWarps / p.m : 1;
    const int m = warp / wpt, slot = warp % wpt;
    if (m >= p.m) return;   // warp-uniform
    uint32_t mx = 0;
    for (int c0 = slot * 32 * U; c0 < chunks; c0 += wpt * 32 * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + 32 * u + lane;
            v[u] = c < chunks ? ldg_nc_v4(p.x + static_cast<int64_t>(m) * p.k + v0 + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) mx = absmax8_bf16(mx, v[u]);
    }
    mx = __reduce_max_sync(0xffffffffu, max(mx & 0xFFFFu, mx >> 16));
    if (lane == 0 && mx) atomicMax(&xm[m], mx);
}

// ---------------------------------------------------------------------------
// Activation images.  For block bl of the current super-chunk and token m the
// image holds, for every MMA of that block and every lane column t, the two
// B registers of lane (g = token, t) in binary16 (of the scaled activations).
// ---------------------------------------------------------------------------
template <int QT>
__device__ void build_image(const QmvParams& p, int blk0, int nb, uint32_t img, const uint32_t* xm);

// q4_K: MMA (nib, u) of lane t uses values v = 64t + 32nib + 4u + {0,2 | 1,3};
// the extra 32 bytes per block hold (Xhi, Xlo) of sub-blocks 2t and 2t+1, the
// sums of their binary16 operands split into two binary16 parts.
template <>
__device__ void build_image<KQ_Q4_K>(const QmvParams& p, int blk0, int nb, uint32_t img, const uint32_t* xm) {
    const int items = p.m * nb * 4;
    for (int it = threadIdx.x; it < items; it += kCWarps * 32) {
        const int m = it / (nb * 4), rem = it % (nb * 4), bl = rem >> 2, t = rem & 3;
        const uint16_t* xs = p.x + static_cast<int64_t>(m) * p.k + static_cast<int64_t>(blk0 + bl) * 256 + 64 * t;
        const uint32_t base = img + m * p.tokstride + bl * 544;
        const float S = tok_scale<KQ_Q4_K>(xm, m);
        float X[2] = {0.f, 0.f};
#pragma unroll
        for (int nib = 0; nib < 2; ++nib) {
#pragma unroll
            for (int uu = 0; uu < 2; ++uu) {
                const uint4 r0 = ldg_nc_v4(xs + 32 * nib + 16 * uu);
                const uint4 r1 = ldg_nc_v4(xs + 32 * nib + 16 * uu + 8);
                const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int u = 4 * uu + q;
                    const float f0 = bf16lo_to_f32(wv[2 * q]), f1 = bf16hi_to_f32(wv[2 * q]);
                    const float f2 = bf16lo_to_f32(wv[2 * q + 1]), f3 = bf16hi_to_f32(wv[2 * q + 1]);
                    const uint32_t h02 = f16pair(f0, f2, S), h13 = f16pair(f1, f3, S);
                    X[nib] += f16sum(h02) + f16sum(h13);
                    sts64(base + (nib * 8 + u) * 32 + t * 8, h02, h13);
                }
            }
        }
        uint32_t e[2];
#pragma unroll
        for (int nib = 0; nib < 2; ++nib) {
            const __half hi = __float2half_rn(X[nib]);
            const __half lo = __float2half_rn(X[nib] - __half2float(hi));
            e[nib] = static_cast<uint32_t>(__half_as_ushort(hi)) | (static_cast<uint32_t>(__half_as_ushort(lo)) << 16);
        }
        sts64(base + 512 + t * 8, e[0], e[1]);
    }
}

// q8_0: MMA h (0, 1) of lane t uses values v = 8t + 4h + {0,2 | 1,3}.
template <>
__device__ void build_image<KQ_Q8_0>(const QmvParams& p, int blk0, int nb, uint32_t img, const uint32_t* xm) {
    const int items = p.m * nb;
    for (int it = threadIdx.x; it < items; it += kCWarps * 32) {
        const int m = it / nb, bl = it % nb;
        const uint16_t* xs = p.x + static_cast<int64_t>(m) * p.k + static_cast<int64_t>(blk0 + bl) * 32;
        const uint32_t base = img + m * p.tokstride + bl * 64;
        const float S = tok_scale<KQ_Q8_0>(xm, m);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint4 r = ldg_nc_v4(xs + 8 * t);
            const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float f0 = bf16lo_to_f32(wv[2 * h]), f1 = bf16hi_to_f32(wv[2 * h]);
                const float f2 = bf16lo_to_f32(wv[2 * h + 1]), f3 = bf16hi_to_f32(wv[2 * h + 1]);
                sts64(base + h * 32 + t * 8, f16pair(f0, f2, S), f16pair(f1, f3, S));
            }
        }
    }
}

// q6_K: sub-block j (16 values, j = 8h + 2tq + u) has a low-code MMA and a
// high-code MMA; lane t uses values 16j + 4t + {0,2 | 1,3}.  The low-code B
// is a = x/16 (tq < 2) or x/256 (tq >= 2, where the code sits in the high
// nibble); the high-code B is x / 4^tq (x scaled, then rounded to binary16).
// With the high 2 bits centred (h - 2) the MMAs give D = 2^-24 sum (c - 32)
// x / 16, c the 6-bit code.
template <>
__device__ void build_image<KQ_Q6_K>(const QmvParams& p, int blk0, int nb, uint32_t img, const uint32_t* xm) {
    const int items = p.m * nb * 16;
    for (int it = threadIdx.x; it < items; it += kCWarps * 32) {
        const int m = it / (nb * 16), rem = it % (nb * 16), bl = rem >> 4, j = rem & 15;
        const int tq = (j & 7) >> 1;
        const float S = tok_scale<KQ_Q6_K>(xm, m);
        const float slo = S * (tq < 2 ? 0.0625f : 0.00390625f), shi = S * exp2_int(-2 * tq);
        const uint16_t* xs = p.x + static_cast<int64_t>(m) * p.k + static_cast<int64_t>(blk0 + bl) * 256 + 16 * j;
        const uint32_t base = img + m * p.tokstride + bl * 1024 + j * 64;
        const uint4 r0 = ldg_nc_v4(xs), r1 = ldg_nc_v4(xs + 8);
        const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float f0 = bf16lo_to_f32(wv[2 * t]), f1 = bf16hi_to_f32(wv[2 * t]);
            const float f2 = bf16lo_to_f32(wv[2 * t + 1]), f3 = bf16hi_to_f32(wv[2 * t + 1]);
            sts64(base + t * 8, f16pair(f0, f2, slo), f16pair(f1, f3, slo));
            sts64(base + 32 + t * 8, f16pair(f0, f2, shi), f16pair(f1, f3, shi));
        }
    }
}

// ---------------------------------------------------------------------------
// Per-warp block processing
// ---------------------------------------------------------------------------
template <int NT>
struct Lane {
    int g, t;
    uint32_t tokb[NT];   // image base of the lane's B column (token) per n-tile
    int tok[NT];         // token index (clamped) of that column
    uint32_t bmask[8];   // slot variants: (1, 1) in binary16 if the lane's column has slot s, else 0
};

// q4_K, one superblock of 16 rows.  rowA/rowB: shared address of the block in
// rows g and g+8.  imgb: offset of the block inside a token image.
template <int NT>
__device__ __forceinline__ void q4k_block(const Lane<NT>& L, uint32_t rowA, uint32_t rowB, uint32_t imgb,
                                          float (&acc)[NT][4]) {
    const int t = L.t;
    const uint4 hA = lds128c(rowA), hB = lds128c(rowB);
    const uint4 qA0 = lds128c(rowA + 16 + 32 * t), qA1 = lds128c(rowA + 32 + 32 * t);
    const uint4 qB0 = lds128c(rowB + 16 + 32 * t), qB1 = lds128c(rowB + 32 + 32 * t);
    // 6-bit scale/min codes of sub-blocks 2t, 2t+1 as (code_2t, code_2t+1) in
    // bits 0..5 / 16..21.  For t < 2: sc = s[j] & 63, m = s[j+4] & 63.  For
    // t >= 2 (j >= 4, jj = j-4): sc = (s[j+4] & 15) | (s[jj] >> 6) << 4 and
    // m = (s[j+4] >> 4) | (s[j] >> 6) << 4.
    const bool lo = t < 2;
    const uint32_t jj0 = (2 * t) & 3;
    const uint32_t sel = 0x4040u | jj0 | ((jj0 + 1) << 8);
    const uint32_t mka = lo ? 0x003F003Fu : 0x000F000Fu, mkb = lo ? 0u : 0x00300030u;
    uint32_t S_lo[2], B_lo[2], S_hi[2], B_hi[2], M_lo[2], M_hi[2];
    float dd[2], dm[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const uint4 h = r ? hB : hA;
        const uint32_t asc = lo ? h.y : h.w;
        const uint32_t am = lo ? h.z : (h.w >> 4);
        const uint32_t scp = (__byte_perm(asc, 0, sel) & mka) | ((__byte_perm(h.y, 0, sel) >> 2) & mkb);
        const uint32_t mp = (__byte_perm(am, 0, sel) & mka) | ((__byte_perm(h.z, 0, sel) >> 2) & mkb);
        const uint32_t scf = hsub2_u32(scp | kH1024, kH1024);   // (sc_2t, sc_2t+1) exact
        const uint32_t mf = hsub2_u32(mp | kH1024, kH1024);
        S_lo[r] = __byte_perm(scf, 0, 0x1010);
        S_hi[r] = hmul2_u32(__byte_perm(scf, 0, 0x3232), kH1_16);
        B_lo[r] = hmul2_u32(S_lo[r], kHm1024);   // -1024 sc
        B_hi[r] = hmul2_u32(S_hi[r], kHm1024);   // -64 sc
        M_lo[r] = __byte_perm(mf, 0, 0x1010);
        M_hi[r] = __byte_perm(mf, 0, 0x3232);
        dd[r] = h16(h.x & 0xffff);
        dm[r] = h16(h.x >> 16);
    }
    const uint32_t wA[8] = {qA0.x, qA0.y, qA0.z, qA0.w, qA1.x, qA1.y, qA1.z, qA1.w};
    const uint32_t wB[8] = {qB0.x, qB0.y, qB0.z, qB0.w, qB1.x, qB1.y, qB1.z, qB1.w};
    float D[2][NT][4], Dm[NT][4];   // two independent MMA chains (word parity)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) D[0][nt][e] = D[1][nt][e] = Dm[nt][e] = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint32_t a = wA[u], b = wB[u], a8 = a >> 8, b8 = b >> 8;
        // low nibbles: 1024 + q, times sc, minus 1024 sc -> q*sc exactly
        {
            const uint32_t a0 = hfma2_u32(and_or(a, 0x000F000Fu, kH1024), S_lo[0], B_lo[0]);
            const uint32_t a1 = hfma2_u32(and_or(b, 0x000F000Fu, kH1024), S_lo[1], B_lo[1]);
            const uint32_t a2 = hfma2_u32(and_or(a8, 0x000F000Fu, kH1024), S_lo[0], B_lo[0]);
            const uint32_t a3 = hfma2_u32(and_or(b8, 0x000F000Fu, kH1024), S_lo[1], B_lo[1]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 bv = lds64c(L.tokb[nt] + imgb + u * 32 + t * 8);
                mma_f16(D[u & 1][nt], a0, a1, a2, a3, bv.x, bv.y);
            }
        }
        // high nibbles: 1024 + 16q, times sc/16, minus 64 sc -> q*sc exactly
        {
            const uint32_t a0 = hfma2_u32(and_or(a, 0x00F000F0u, kH1024), S_hi[0], B_hi[0]);
            const uint32_t a1 = hfma2_u32(and_or(b, 0x00F000F0u, kH1024), S_hi[1], B_hi[1]);
            const uint32_t a2 = hfma2_u32(and_or(a8, 0x00F000F0u, kH1024), S_hi[0], B_hi[0]);
            const uint32_t a3 = hfma2_u32(and_or(b8, 0x00F000F0u, kH1024), S_hi[1], B_hi[1]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 bv = lds64c(L.tokb[nt] + imgb + (8 + u) * 32 + t * 8);
                mma_f16(D[u & 1][nt], a0, a1, a2, a3, bv.x, bv.y);
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint2 bv = lds64c(L.tokb[nt] + imgb + 512 + t * 8);
        mma_f16(Dm[nt], M_lo[0], M_lo[1], M_hi[0], M_hi[1], bv.x, bv.y);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = e >> 1;
            acc[nt][e] = fmaf(dd[r], D[0][nt][e] + D[1][nt][e], fmaf(-dm[r], Dm[nt][e], acc[nt][e]));
        }
    }
}

// Column bookkeeping for the slot variants (q6_K, q8_0): column c of n-tile nt
// holds token c / S and sub-block slot c % S (S > 1), or token 8 nt + c.
template <int S, int NT>
__device__ __forceinline__ void col_info(int nt, int col, int m, int& tok, int& slot) {
    if (S > 1) {
        tok = col / S;
        slot = col % S;
    } else {
        tok = 8 * nt + col;
        slot = 0;
    }
    tok = tok < m ? tok : m - 1;
}

// q8_0: the warp's run of up to RUN consecutive 32-value blocks of one stage.
// rowA/rowB: shared address of row g / g+8 of the stage; lb0: first local
// block; nvalid: blocks present; imgb0: image offset of lb0.
template <int S, int NT, int RUN>
__device__ __forceinline__ void q8_run(const Lane<NT>& L, const QmvParams& p, uint32_t rowA, uint32_t rowB, int lb0,
                                       int nvalid, uint32_t imgb0, uint32_t zero_addr,
                                       float (&acc)[NT][4]) {
    const int t = L.t;
    float D[NT][4];
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        if (i % S == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) D[nt][e] = 0.f;
        }
        if (i < nvalid) {
            const int lb = lb0 + i;
            const uint32_t off = lb * 34 + 2 + 8 * t;
            const bool odd = (off & 2) != 0;
            const uint32_t a0w = lds32c_a2(rowA + off, odd), a1w = lds32c_a2(rowA + off + 4, odd);
            const uint32_t b0w = lds32c_a2(rowB + off, odd), b1w = lds32c_a2(rowB + off + 4, odd);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t wa = h ? a1w : a0w, wb = h ? b1w : b0w;
                // byte ^ 0x80 = q + 128 as a binary16 subnormal, less 128 2^-24:
                // the signed code as the subnormal q 2^-24 (exact)
                const uint32_t A0 = hsub2_u32(and_xor(wa, 0x00FF00FFu, 0x00800080u), 0x00800080u);
                const uint32_t A1 = hsub2_u32(and_xor(wb, 0x00FF00FFu, 0x00800080u), 0x00800080u);
                const uint32_t A2 = hsub2_u32(and_xor(wa >> 8, 0x00FF00FFu, 0x00800080u), 0x00800080u);
                const uint32_t A3 = hsub2_u32(and_xor(wb >> 8, 0x00FF00FFu, 0x00800080u), 0x00800080u);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint2 bv = lds64c(L.tokb[nt] + imgb0 + i * 64 + h * 32 + t * 8);
                    if (S > 1) {   // only the columns of this block's slot see its activations
                        bv.x = hmul2_u32(bv.x, L.bmask[i % S]);
                        bv.y = hmul2_u32(bv.y, L.bmask[i % S]);
                    }
                    mma_f16(D[nt], A0, A1, A2, A3, bv.x, bv.y);
                }
            }
        }
        if (i % S == S - 1 || i == RUN - 1) {
            // epilogue: y += 2^24 d D per column's block (D = 2^-24 sum q x)
            const int i0 = i - (i % S);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int tok, slot;
                    col_info<S, NT>(nt, 2 * t + (e & 1), p.m, tok, slot);
                    const int ib = i0 + slot;
                    if (ib < nvalid && ib <= i) {
                        const uint32_t row = (e >> 1) ? rowB : rowA;
                        const float d = h16(ldsu16c(row + (lb0 + ib) * 34)) * kTwo24;
                        acc[nt][e] = fmaf(d, D[nt][e], acc[nt][e]);
                    }
                }
            }
        }
    }
}

// q6_K: half h (sub-blocks j = 8h + 2tq + u, 128 values) of one 256-value
// block of 16 rows.  Two warps share a block, one half each.
template <int S, int NT>
__device__ __forceinline__ void q6k_half(const Lane<NT>& L, const QmvParams& p, uint32_t rowA, uint32_t rowB,
                                         bool odd, int h, uint32_t imgb, uint32_t zero_addr,
                                         float (&acc)[NT][4]) {
    const int t = L.t;
    const float dA = h16(ldsu16c(rowA + 208));
    const float dB = h16(ldsu16c(rowB + 208));
    // the lane's 4-byte pieces: ql[h][pp][u] and qh[h][u] for rows g and g+8
    uint32_t QLA[4], QLB[4], QHA[2], QHB[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t o = 64 * h + 32 * (i >> 1) + 16 * (i & 1) + 4 * t;
        QLA[i] = lds32c_a2(rowA + o, odd);
        QLB[i] = lds32c_a2(rowB + o, odd);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t o = 128 + 32 * h + 16 * i + 4 * t;
        QHA[i] = lds32c_a2(rowA + o, odd);
        QHB[i] = lds32c_a2(rowB + o, odd);
    }
    float D[NT][4];
#pragma unroll
    for (int jl = 0; jl < 8; ++jl) {
        const int tq = jl >> 1, u = jl & 1, pp = tq & 1;
        const int j = 8 * h + jl;
        if (jl % S == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) D[nt][e] = 0.f;
        }
        const uint32_t la = QLA[2 * pp + u], lb = QLB[2 * pp + u];
        const uint32_t ha = QHA[u], hb = QHB[u];
        // low 4 bits as binary16 subnormals: low nibble c (tq < 2) -> c 2^-24
        // with B = x/16, high nibble (tq >= 2) -> 16 c 2^-24 with B = x/256
        const uint32_t mlo = tq < 2 ? 0x000F000Fu : 0x00F000F0u;
        const uint32_t L0 = la & mlo, L1 = lb & mlo, L2 = (la >> 8) & mlo, L3 = (lb >> 8) & mlo;
        // high 2 bits h, left at bits 2tq..2tq+1 of each byte, less 2 (the
        // code offset 32 = 16 2): 4^tq (h - 2) 2^-24 (exact), with B =
        // x / 4^tq (all B scalings are exact powers of two, none above 1).
        // The two MMAs sum 2^-24 (c6 - 32) x / 16.
        const uint32_t mhi = 0x00030003u << (2 * tq), off = 0x00020002u << (2 * tq);
        const uint32_t H0 = hsub2_u32(ha & mhi, off), H1 = hsub2_u32(hb & mhi, off);
        const uint32_t H2 = hsub2_u32((ha >> 8) & mhi, off), H3 = hsub2_u32((hb >> 8) & mhi, off);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t a = L.tokb[nt] + imgb + j * 64 + t * 8;
            uint2 bl = lds64c(a), bh = lds64c(a + 32);
            if (S > 1) {   // only the columns of this sub-block's slot see its activations
                const uint32_t mk = L.bmask[jl % S];
                bl.x = hmul2_u32(bl.x, mk);
                bl.y = hmul2_u32(bl.y, mk);
                bh.x = hmul2_u32(bh.x, mk);
                bh.y = hmul2_u32(bh.y, mk);
            }
            mma_f16(D[nt], L0, L1, L2, L3, bl.x, bl.y);
            mma_f16(D[nt], H0, H1, H2, H3, bh.x, bh.y);
        }
        if (jl % S == S - 1) {
            const int j0 = j - (S - 1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int tok, slot;
                    col_info<S, NT>(nt, 2 * t + (e & 1), p.m, tok, slot);
                    const int jj = j0 + slot;
                    // sum (c - 32) x = 16 2^24 D
                    const uint32_t row = (e >> 1) ? rowB : rowA;
                    const float dr = (e >> 1) ? dB : dA;
                    const int sc = ldss8c(row + 192 + jj);
                    const float s = 268435456.0f * __fmul_rn(dr, static_cast<float>(sc));   // 16 2^24 d sc
                    acc[nt][e] = fmaf(s, D[nt][e], acc[nt][e]);
                }
            }
        }
    }
}

template <int QT, int S, int NT>
__global__ void __launch_bounds__(kThreads, 1) qmv_kernel(const QmvParams p) {
    using C = Codec<QT>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);           // [kMaxStages]
    uint64_t* empty = full + kMaxStages;                           // [kMaxStages]
    uint64_t* red_full = full + 2 * kMaxStages;                    // [2]
    uint64_t* red_empty = full + 2 * kMaxStages + 2;               // [2]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 256);
    volatile int* consumed = reinterpret_cast<volatile int*>(smem + 260);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t zero_addr = sbase + 272;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // balanced contiguous row range of this CTA
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * p.n / gridDim.x;
    const int64_t r1 = static_cast<int64_t>(blockIdx.x + 1) * p.n / gridDim.x;
    const int nrg = static_cast<int>((r1 - r0 + kRows - 1) / kRows);
    const int nsc = cdiv(p.nblk, p.scb);

    if (tid == 0) {
        for (int i = 0; i < p.ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], QT == KQ_Q4_K ? kCWarps / 2 : kCWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&red_full[i], kCWarps);
            mbar_init(&red_empty[i], 1);
        }
        *abort_flag = 0;
        *consumed = 0;
        fence_barrier_init();
    }
    if (tid < 4) sts32(zero_addr + 4 * tid, 0u);
    if (tid < 32) reinterpret_cast<uint32_t*>(smem + kXMax)[tid] = 0u;
    // Programmatic dependent launch: the next kernel in the stream may start
    // its prologue now.  This CTA's weight bytes are prefetched into L2 (a
    // hint; L2 is coherent, so it is safe even if an earlier kernel is still
    // writing them), then every thread waits for the earlier grids to finish
    // before touching memory they might produce.  Without the launch
    // attribute both instructions are no-ops.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kProducerWarp && p.bulk) {
        const uint8_t* base = p.w + r0 * p.row_bytes;
        const int64_t bytes = (r1 - r0) * p.row_bytes;
        for (int64_t o = static_cast<int64_t>(lane) * 65536; o < bytes; o += 32 * 65536) {
            const uint32_t sz = static_cast<uint32_t>(bytes - o < 65536 ? bytes - o : 65536);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + o), "r"(sz) : "memory");
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();

    auto stages_in = [&](int sc) { return cdiv(min(p.scb, p.nblk - sc * p.scb), p.g); };
    auto stage_addr = [&](int slot) { return sbase + kOffW + slot * (kRows * p.rs); };
    auto bwait = [&](uint64_t* bar, uint32_t parity) {
        if (*abort_flag) return false;
        if (!mbar_wait(bar, parity, p.status)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };

    if (warp == kProducerWarp) {
        // ------------------------------------------------ W stage producer
        int q = 0;   // global stage counter
        bool ok = true;
        for (int sc = 0; sc < nsc && ok; ++sc) {
            const int nst = stages_in(sc);
            for (int g = 0; g < nrg && ok; ++g) {
                const int64_t row0 = r0 + static_cast<int64_t>(g) * kRows;
                const int rv = static_cast<int>(r1 - row0 < kRows ? r1 - row0 : kRows);
                for (int si = 0; si < nst; ++si, ++q) {
                    const int slot = q % p.ns;
                    const int b0 = sc * p.scb + si * p.g;
                    const int nb = p.nblk - b0 < p.g ? p.nblk - b0 : p.g;
                    const uint32_t bytes = nb * C::BPB;
                    if (lane == 0) ok = bwait(&empty[slot], ((q / p.ns) & 1) ^ 1);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const uint8_t* src = p.w + row0 * p.row_bytes + static_cast<int64_t>(b0) * C::BPB;
                    if (p.bulk) {
                        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes * rv);
                        __syncwarp();
                        if (lane < rv)
                            bulk_g2s(smem + kOffW + slot * (kRows * p.rs) + lane * p.rs, src + lane * p.row_bytes,
                                     bytes, &full[slot]);
                    } else {
                        const int half = bytes / 2;
                        const uint32_t dst = stage_addr(slot);
                        for (int i = lane; i < rv * half; i += 32) {
                            const int r = i / half, c = i % half;
                            const unsigned short v =
                                __ldg(reinterpret_cast<const unsigned short*>(src + r * p.row_bytes) + c);
                            asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst + r * p.rs + 2 * c), "h"(v));
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&full[slot]);
                    }
                }
            }
        }
        // wind down after an abort: let copies in flight land
        if (*abort_flag && lane == 0)
            for (int qq = *consumed; qq < q; ++qq) mbar_wait(&full[qq % p.ns], (qq / p.ns) & 1, nullptr);
    } else if (warp == kReducerWarp) {
        // ------------------------------------------------ cross-warp reducer
        float* pbuf = reinterpret_cast<float*>(smem + p.off_pbuf);
        float* racc = reinterpret_cast<float*>(smem + p.off_racc);
        constexpr int PW = 32 * 4 * NT;   // floats per warp partial
        int it = 0;
        for (int sc = 0; sc < nsc; ++sc) {
            for (int g = 0; g < nrg; ++g, ++it) {
                const int b = it & 1;
                if (!bwait(&red_full[b], (it >> 1) & 1)) break;
                const int64_t row0 = r0 + static_cast<int64_t>(g) * kRows;
                const int rv = static_cast<int>(r1 - row0 < kRows ? r1 - row0 : kRows);
                const float* pb = pbuf + b * kCWarps * PW;
                // outputs (token, row): 16 rows x m tokens
                for (int o = lane; o < p.m * kRows; o += 32) {
                    const int tok = o / kRows, r = o % kRows;
                    float sum = 0.f;
                    const int slots = S > 1 ? S : 1;
                    for (int sl = 0; sl < slots; ++sl) {
                        const int c = S > 1 ? tok * S + sl : tok;   // column within the 8 (or 16) of the tiles
                        const int nt = c >> 3, cc = c & 7;
                        const int ln = 4 * (r & 7) + (cc >> 1);
                        const int e = 2 * (r >> 3) + (cc & 1);
                        const int idx = ln * 4 * NT + nt * 4 + e;
                        for (int w = 0; w < kCWarps; ++w) sum += pb[w * PW + idx];
                    }
                    float* ra = racc + (g * kRows + r) * 16 + tok;
                    if (nsc > 1) {
                        if (sc > 0) sum += *ra;
                        *ra = sum;
                    }
                    if (sc == nsc - 1 && r < rv) p.y[static_cast<int64_t>(tok) * p.n + row0 + r] = sum;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_empty[b]);
            }
            if (*abort_flag) break;
        }
    } else {
        // ------------------------------------------------ consumers (16 warps)
        Lane<NT> L;
        L.g = lane >> 2;
        L.t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            int tok, slot;
            col_info<S, NT>(nt, L.g, p.m, tok, slot);
            L.tok[nt] = tok;
            L.tokb[nt] = sbase + p.off_img + tok * p.tokstride;
        }
#pragma unroll
        for (int sl = 0; sl < 8; ++sl) L.bmask[sl] = (S > 1 && (L.g % S) == sl) ? 0x3C003C00u : 0u;
        // q4_K: two groups of 8 warps take alternate stages (a warp decodes a
        // whole block); the other codecs share every stage among all 16 warps
        const int grp = warp >> 3, wig = warp & 7;
        float* pbuf = reinterpret_cast<float*>(smem + p.off_pbuf);
        float* xinv = reinterpret_cast<float*>(smem + kXInv);
        constexpr int PW = 32 * 4 * NT;
        int q = 0, it = 0;
        // every consumer thread passes the same barriers, aborted or not
        for (int sc = 0; sc < nsc; ++sc) {
            const int blk0 = sc * p.scb;
            const int nbsc = p.nblk - blk0 < p.scb ? p.nblk - blk0 : p.scb;
            const int nst = stages_in(sc);
            // the super-chunk's activation scales (two buffers of maxima: the
            // other one is cleared for the next super-chunk), then its image
            uint32_t* xm = reinterpret_cast<uint32_t*>(smem + kXMax) + 16 * (sc & 1);
            asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32));
            if (!*abort_flag) x_range(p, static_cast<int64_t>(blk0) * C::VPB, nbsc * C::VPB, xm);
            if (tid < 16) xm[16 * (1 - 2 * (sc & 1)) + tid] = 0u;
            asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32));
            if (tid < p.m) {
                if (xm[tid] >= 0x7F80u) atomicOr(p.status, KQ_DEV_X_RANGE);   // Inf or NaN
                xinv[tid] = exp2_int(-xscale_exp(xm[tid], C::XT));
            }
            if (!*abort_flag) build_image<QT>(p, blk0, nbsc, sbase + p.off_img, xm);
            asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32));
            if (*abort_flag) continue;
            for (int g = 0; g < nrg; ++g, ++it) {
                float acc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
                bool ok = true;
                for (int si = 0; si < nst; ++si, ++q) {
                    const int slot = q % p.ns;
                    if (QT == KQ_Q4_K && (q & 1) != grp) continue;
                    if (!bwait(&full[slot], (q / p.ns) & 1)) {
                        ok = false;
                        break;
                    }
                    const int b0 = blk0 + si * p.g;
                    const int nb = p.nblk - b0 < p.g ? p.nblk - b0 : p.g;
                    const uint32_t st = stage_addr(slot);
                    const uint32_t rowA = st + L.g * p.rs, rowB = rowA + 8 * p.rs;
                    const int bl = si * p.g;   // first block of the stage within the super-chunk
                    if constexpr (QT == KQ_Q4_K) {
                        // group of 8 warps, a warp decodes whole blocks wig, wig + 8, ...
                        for (int lb = wig; lb < nb; lb += 8)
                            q4k_block<NT>(L, rowA + lb * 144, rowB + lb * 144, (bl + lb) * 544, acc);
                    } else if constexpr (QT == KQ_Q6_K) {
                        // half blocks: item i = (block i/2, half i%2)
                        for (int it2 = warp; it2 < 2 * nb; it2 += kCWarps) {
                            const int lb = it2 >> 1, lbi = bl + lb;
                            q6k_half<S, NT>(L, p, rowA + lb * 210, rowB + lb * 210, (lb & 1) != 0, it2 & 1,
                                            lbi * 1024, zero_addr, acc);
                        }
                    } else {
                        // runs of 4 consecutive blocks
                        for (int lb0 = 4 * warp; lb0 < nb; lb0 += 4 * kCWarps) {
                            const int nv = nb - lb0 < 4 ? nb - lb0 : 4;
                            const int lbi = bl + lb0;
                            q8_run<S, NT, 4>(L, p, rowA, rowB, lb0, nv, lbi * 64, zero_addr, acc);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&empty[slot]);
                        if (warp == 0) *consumed = q + 1;
                    }
                }
                if (!ok) break;
                // hand the warp's partial sums of this row group, unscaled, to
                // the reducer
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        int tok, slot;
                        col_info<S, NT>(nt, 2 * L.t + (e & 1), p.m, tok, slot);
                        acc[nt][e] *= xinv[tok];
                    }
                const int b = it & 1;
                if (!bwait(&red_empty[b], ((it >> 1) & 1) ^ 1)) break;
                float* dst = pbuf + (b * kCWarps + warp) * PW + lane * 4 * NT;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<float4*>(dst + 4 * nt) = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_full[b]);
            }
        }
    }
    __syncthreads();
}

template <int QT>
int launch_codec(const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y, cudaStream_t st) {
    using C = Codec<QT>;
    QmvParams p{};
    p.w = static_cast<const uint8_t*>(w);
    p.x = x;
    p.y = y;
    p.status = device_status_ptr();
    p.n = n;
    p.k = k;
    p.m = m;
    p.nblk = static_cast<int>(k / C::VPB);
    p.row_bytes = static_cast<int64_t>(p.nblk) * C::BPB;
    p.bulk = (p.row_bytes % 16 == 0) && (reinterpret_cast<uintptr_t>(w) % 16 == 0);
    const int optin = device_smem_optin();
    const int sms = device_sm_count();
    // One persistent CTA per SM, each owning a contiguous range of rows.
    const int64_t groups = (n + kRows - 1) / kRows;
    const int grid = static_cast<int>(groups < sms ? groups : sms);
    const int nt = (QT != KQ_Q4_K && m <= 4) ? 1 : (m > 8 ? 2 : 1);
    const int64_t rpc = (n + grid - 1) / grid;
    const int nrg = static_cast<int>((rpc + kRows - 1) / kRows);
    const uint32_t pbuf_bytes = 2u * kCWarps * 32 * 4 * nt * 4;
    // Pick the stage geometry: most bytes in flight (ns stages x 16 rows x g
    // blocks), then more stages, subject to the shared-memory budget that the
    // activation image, the partial-sum buffers and the barriers leave.
    int ns = 0, g = 0, scb = 0, rs = 0;
    uint32_t tokstride = 0, off_img = 0, off_pbuf = 0, off_racc = 0, total = 0;
    int64_t best = -1;
    const int gmax = cdiv(p.nblk, C::GA) * C::GA;
    for (int ns_try = 4; ns_try >= 2; --ns_try) {
        for (int g_try = gmax; g_try >= C::GA; g_try -= C::GA) {
            const int rs_try = ((g_try * C::BPB + 127) / 128) * 128 + 16;
            const uint32_t wbytes = kOffW + ns_try * kRows * rs_try;
            const uint32_t oi = (wbytes + 127) & ~127u;
            const int scb_full = cdiv(p.nblk, g_try) * g_try;
            // super-chunk: as many whole stages of blocks as the image allows
            for (int scb_try = scb_full; scb_try >= g_try; scb_try -= g_try) {
                const uint32_t base = scb_try * C::IMG;
                const uint32_t ts = base + ((32u - (base & 127u)) & 127u);
                const uint32_t op = (oi + m * ts + 15) & ~15u;
                const uint32_t orc = op + pbuf_bytes;
                const uint32_t tot = orc + (scb_try < scb_full ? nrg * kRows * 16 * 4 : 0);
                if (tot > static_cast<uint32_t>(optin)) continue;
                const int64_t inflight = static_cast<int64_t>(ns_try) * kRows * g_try * C::BPB;
                if (inflight > best) {
                    best = inflight;
                    ns = ns_try; g = g_try; scb = scb_try; rs = rs_try;
                    tokstride = ts; off_img = oi; off_pbuf = op; off_racc = orc; total = tot;
                }
                break;
            }
        }
    }
    if (best < 0) {
        // the activation image of all m rows does not fit: split the rows
        if (m == 1) return KQ_ERR_UNSUPPORTED;
        const int m1 = m / 2;
        const int rc = launch_codec<QT>(w, n, k, x, m1, y, st);
        if (rc) return rc;
        return launch_codec<QT>(w, n, k, x + static_cast<int64_t>(m1) * k, m - m1, y + static_cast<int64_t>(m1) * n, st);
    }
    p.ns = ns;
    p.g = g;
    p.rs = rs;
    p.scb = scb;
    p.tokstride = tokstride;
    p.off_img = off_img;
    p.off_pbuf = off_pbuf;
    p.off_racc = off_racc;
    auto launch = [&](auto kernel) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
        if (e != cudaSuccess) return record_cuda(e);
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = total;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = use_pdl() ? 1 : 0;
        return record_cuda(cudaLaunchKernelEx(&cfg, kernel, p));
    };
    if constexpr (QT == KQ_Q4_K) {
        return m > 8 ? launch(qmv_kernel<QT, 1, 2>) : launch(qmv_kernel<QT, 1, 1>);
    } else if constexpr (QT == KQ_Q8_0) {
        // runs of 4 blocks per warp: at most 4 sub-block slots per token
        if (m == 1) return launch(qmv_kernel<QT, 4, 1>);
        if (m == 2) return launch(qmv_kernel<QT, 4, 1>);
        if (m <= 4) return launch(qmv_kernel<QT, 2, 1>);
        if (m <= 8) return launch(qmv_kernel<QT, 1, 1>);
        return launch(qmv_kernel<QT, 1, 2>);
    } else {
        if (m == 1) return launch(qmv_kernel<QT, 8, 1>);
        if (m == 2) return launch(qmv_kernel<QT, 4, 1>);
        if (m <= 4) return launch(qmv_kernel<QT, 2, 1>);
        if (m <= 8) return launch(qmv_kernel<QT, 1, 1>);
        return launch(qmv_kernel<QT, 1, 2>);
    }
}

}  // namespace

int launch_qmv(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
               cudaStream_t s) {
    if (n == 0) return KQ_OK;
    const int rc = launch_qmv_stream(type, w, n, k, x, m, y, s);
    if (rc != KQ_ERR_UNSUPPORTED) return rc;
    switch (type) {
    case KQ_Q4_K: return launch_codec<KQ_Q4_K>(w, n, k, x, m, y, s);
    case KQ_Q6_K: return launch_codec<KQ_Q6_K>(w, n, k, x, m, y, s);
    case KQ_Q8_0: return launch_codec<KQ_Q8_0>(w, n, k, x, m, y, s);
    // exact fp32 decode-and-dot kernel
    case KQ_Q5_K:
    case KQ_Q4_0: return launch_qmv_exact(type, w, n, k, x, m, y, s);
    default: return KQ_ERR_UNSUPPORTED;
    }
}

}  // namespace kq
