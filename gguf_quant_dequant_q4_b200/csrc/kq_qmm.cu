// kq_qmm / kq_gather_qmm: prefill-shaped y = x . W^T on the tcgen05 tensor
// cores, with W decoded from its GGUF wire blocks inside the kernel.
//
// mlx-kquant bindings.cpp `quantized_matmul` and `gather_qmm_seg` (segment-
// walking gather GEMM over expert-sorted rows, map of (expert, row_start,
// num_rows <= 64) tiles, uncovered rows left unwritten); README
// "Performance": a single-pass matmul on the tensor units, per-expert-segment
// GEMM for sorted MoE prefill.  hanzo-ml quantized/mod.rs notes that a GEMM
// that re-reads the weight once per small row group wastes bandwidth; here
// every weight tile is read and decoded once per 256 output rows.
//
// Tile: 256 weight rows x up to 256 activation rows, K in steps of 64, on a
// CTA pair (a cluster of two CTAs on neighbouring SMs, tcgen05 cta_group::2,
// MMA M = 256): each CTA decodes its own 128 weight rows and loads half of
// the activation rows, so a pair reads each activation tile once for 256
// weight rows.  (With KQ_QMM_1SM=1 a single CTA takes 128 weight rows and all
// 256 activation rows, MMA M = 128.)  Persistent, one CTA per SM,
// warp-specialized:
//   warp 0      activation producer: TMA of bf16 activation tiles
//               (128B-swizzled 64-row boxes: over the CTA's half of a unit's
//               run of rows, or one per map tile when the tiles are not one run)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer (in the
//               first CTA of a pair; the full barriers it waits on live
//               there, and its commits arrive on both CTAs' empty barriers)
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, masked stores
//   warps 6..21 decoders: wire bytes -> bf16 A tile in the 128B-swizzled
//               K-major layout the tensor core reads (thread = one row and
//               one 16-value quarter of the 64-value step)
//   warp 22     raw weight producer: TMA of wire-byte tiles (2-D box, 128
//               rows x one 256-value block), with L2 prefetch ahead
// Accumulators are double-buffered in TMEM (2 x 256 columns) so the epilogue
// of one tile overlaps the main loop of the next.  All waits are bounded; a
// wait that runs out sets KQ_DEV_TIMEOUT and the CTA winds down, freeing its
// TMEM.  No TMA multicast is used anywhere.
#include <cuda.h>

#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kDecWarps = 16;    // decoder warps (thread = row x 16-value part)
constexpr int kThreads = (7 + kDecWarps) * 32;
constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBN = 256;          // activation rows per tile (MMA N max)
constexpr int kBK = 64;           // K per pipeline step (one 128-byte swizzle row)
constexpr int kMaxTiles = 1024;   // map tiles one gather launch takes (a window of the map)
constexpr uint32_t kHeader = 5120; // barriers, misc words, tile tables
constexpr int kDeqWarp0 = 6;   // warps 0..5: producer, MMA, 4 epilogue
constexpr int kRawWarp = kDeqWarp0 + kDecWarps;   // the raw weight producer
constexpr int kRawAhead = 2;   // raw stages prefetched into L2 ahead of their load (measured: 1-2 best)

template <int QT> struct QmmCodec;
// raw row bytes per stage (one 256-value block column of 128 weight rows)
template <> struct QmmCodec<KQ_Q4_K> {
    static constexpr int RAWB = 144;
};
template <> struct QmmCodec<KQ_Q6_K> {
    static constexpr int RAWB = 240;   // 210-byte block at offset 210b mod 16
};
template <> struct QmmCodec<KQ_Q8_0> {
    static constexpr int RAWB = 272;   // eight 34-byte blocks
};
template <> struct QmmCodec<KQ_Q5_K> {
    static constexpr int RAWB = 176;
};
template <> struct QmmCodec<KQ_Q4_0> {
    static constexpr int RAWB = 144;   // eight 18-byte blocks
};

struct Smem {
    static constexpr uint32_t kBars = 0;      // mbarriers (36)
    static constexpr uint32_t kMisc = 384;    // tmem base, abort flag, counts
    static constexpr uint32_t kTiles = 512;   // sorted tile ids (u16) + per-expert tables
};

struct QmmParams {
    int64_t n;            // weight rows per expert
    int64_t m;            // activation rows (dense) / rows of x_sorted (gather)
    int k;
    int n_experts;        // 0 = dense qmm
    int ntn;              // weight tiles per expert = ceil(n / 128)
    int units;            // dense: full units, then the tail's 64-row sub-units
    int units_main;       // dense: units covered by whole rounds of the grid
    int split;            // dense: sub-units per unit of the last round (1, 2 or 4)
    const uint32_t* map;
    const uint32_t* count;
    int64_t cap;
    int64_t win0;         // gather: first map tile of this launch's window of kMaxTiles
    int64_t row_bytes;    // flat raw view (rows not a 16-byte multiple): bytes per weight row
    float* y;
    int32_t* err;         // caller's flag (gather) or library status
    int* status;
};

// ---------------------------------------------------------------- PTX glue
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Rank-1 tiled load (the flat byte view of the weights); x a multiple of 16.
__device__ __forceinline__ void tma_load_1d(uint32_t dst, const CUtensorMap* map, int x, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrive on `bar` once the MMAs issued so far complete; for a CTA pair the
// arrival goes to the barrier at the same offset in both CTAs.
template <int CG>
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    if constexpr (CG == 2) {
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                smem_u32(bar)),
            "h"(static_cast<uint16_t>(3))
            : "memory");
    } else {
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(bar))
                     : "memory");
    }
}
template <int CG>
__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    if constexpr (CG == 2) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
            : "memory");
    }
}
// All 512 TMEM columns (two 256-column accumulators), address written to
// shared memory at `dst`; one whole warp, the same warp in both CTAs of a pair.
template <int CG>
__device__ __forceinline__ void tmem_alloc512(uint32_t dst) {
    if constexpr (CG == 2) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
}
template <int CG>
__device__ __forceinline__ void tmem_dealloc512(uint32_t tmem) {
    if constexpr (CG == 2) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}
// ---- CTA pairs (clusters of two): cluster helpers are in kq_device.cuh
// Arrive on an mbarrier given by its cluster shared-memory address (default
// .release.cta semantics: the data it publishes is this CTA's shared memory,
// read by the pair's tensor cores after the async-proxy fence, so no
// cluster-scope fence is needed).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
// Prefetch of a tile into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}
// Tiled load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (cluster address), no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t ldsu16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

// K-major operand in the 128-byte swizzle layout: rows of 128 bytes, groups of
// 8 rows 1024 bytes apart (stride byte offset), start advanced by 32 bytes per
// 16-element K slice.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}
// kind::f16 instruction descriptor: D f32, A and B bf16, both K-major, M =
// 128 (one CTA) or 256 (a CTA pair).
__device__ __forceinline__ uint32_t make_idesc(int n, int m) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// ------------------------------------------------------- bf16x2 arithmetic
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf16_bits(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
__device__ __forceinline__ float bf16_val(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ uint32_t dup(uint32_t b) { return b | (b << 16); }
// A scale s split into two bf16 parts, s ~= hi + lo to 16 significant bits.
__device__ __forceinline__ void split_scale(float s, uint32_t& hi2, uint32_t& lo2) {
    const uint32_t h = bf16_bits(s);
    hi2 = dup(h);
    lo2 = dup(bf16_bits(s - bf16_val(h)));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ float h16v(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// 32 bytes starting O bytes into the 16-byte aligned shared address `a`,
// as 8 little-endian words (O even, compile time).
template <int O>
__device__ __forceinline__ void lds32B(uint32_t a, uint32_t (&w)[8]) {
    uint32_t r[12];
    const uint4 c0 = lds128(a), c1 = lds128(a + 16);
    r[0] = c0.x; r[1] = c0.y; r[2] = c0.z; r[3] = c0.w;
    r[4] = c1.x; r[5] = c1.y; r[6] = c1.z; r[7] = c1.w;
    if constexpr (O != 0) {
        const uint4 c2 = lds128(a + 32);
        r[8] = c2.x; r[9] = c2.y; r[10] = c2.z; r[11] = c2.w;
    } else {
        r[8] = r[9] = r[10] = r[11] = 0;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if constexpr ((O & 3) == 0) w[i] = r[(O >> 2) + i];
        else w[i] = __byte_perm(r[(O >> 2) + i], r[(O >> 2) + i + 1], 0x5432);
    }
}

// 16 bytes starting O bytes after the 16-byte aligned shared address `a`, as 4
// little-endian words (O even, compile time).
template <int O>
__device__ __forceinline__ void lds16B(uint32_t a, uint32_t (&w)[4]) {
    if constexpr (O == 0) {
        const uint4 c = lds128(a);
        w[0] = c.x; w[1] = c.y; w[2] = c.z; w[3] = c.w;
    } else {
        const uint4 c0 = lds128(a), c1 = lds128(a + 16);
        const uint32_t r[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr ((O & 3) == 0) w[i] = r[(O >> 2) + i];
            else w[i] = __byte_perm(r[(O >> 2) + i], r[(O >> 2) + i + 1], 0x5432);
        }
    }
}

// ---------------------------------------------------------------- decoders
// A decoder thread owns one weight row r and one 16-value part p (0..3) of
// every 64-value K step.  At the start of each raw stage (one 256-value block
// row, four K steps q = 0..3) it decodes the scale terms of its four steps
// once; each step then turns 16 wire values into 8 bf16x2 words:
//   w = bf16( fp32(d*sc)*q - fp32(dmin*m) )  evaluated as
//   t = q*s_lo - mm ; w = q*s_hi + t   in bf16x2 FMA (s = s_hi + s_lo exact to
//   16 bits), so the result carries essentially one bf16 rounding.
constexpr uint32_t kB128 = 0x43004300u;   // bf16 (128, 128)
constexpr uint32_t kB160 = 0x43204320u;   // bf16 (160, 160)
constexpr uint32_t kB136 = 0x43084308u;   // bf16 (136, 136)
constexpr uint32_t kMagic = 0x43434343u;

struct StageScales {
    uint32_t hi[4], lo[4], nmm[4];
    float d[4];
};

// q4_K: step q, part p covers values 64q + 16p .. +15: nibble p>>1 of
// qs[32q + 16(p&1) ..], scale/min code j = 2q + (p>>1).
__device__ __forceinline__ void q4k_scales(uint32_t row, int p, StageScales& S) {
    const uint4 h = lds128(row);
    const float d = h16v(h.x & 0xffff), dmin = h16v(h.x >> 16);
    const int ph = p >> 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = 2 * q + ph;
        int sc, m;
        if (q < 2) {   // j < 4
            sc = (h.y >> (8 * j)) & 63;
            m = (h.z >> (8 * j)) & 63;
        } else {
            const int jj = j - 4;
            const uint32_t b8 = (h.w >> (8 * jj)) & 0xff;
            sc = (b8 & 15) | (((h.y >> (8 * jj + 6)) & 3) << 4);
            m = (b8 >> 4) | (((h.z >> (8 * jj + 6)) & 3) << 4);
        }
        split_scale(__fmul_rn(d, static_cast<float>(sc)), S.hi[q], S.lo[q]);
        S.nmm[q] = dup(bf16_bits(-__fmul_rn(dmin, static_cast<float>(m))));
    }
}

__device__ __forceinline__ void q4k_step(uint32_t row, int q, int p, const StageScales& S, uint32_t (&o)[8]) {
    const uint4 c = lds128(row + 16 + 32 * q + 16 * (p & 1));
    const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
    const uint32_t hi = S.hi[q], lo = S.lo[q], nmm = S.nmm[q];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t nib = (p >> 1) ? ((wv[i] >> 4) & 0x0F0F0F0Fu) : (wv[i] & 0x0F0F0F0Fu);
        const uint32_t v01 = bsub2(__byte_perm(nib, kMagic, 0x5140), kB128);   // (q0, q1) exact
        const uint32_t v23 = bsub2(__byte_perm(nib, kMagic, 0x7362), kB128);
        o[2 * i] = bfma2(v01, hi, bfma2(v01, lo, nmm));
        o[2 * i + 1] = bfma2(v23, hi, bfma2(v23, lo, nmm));
    }
}

// q6_K (block at byte O of the staged row): step q, part p covers
// h = q/2, quarter tq = 2(q&1) + (p>>1), l = 16(p&1) .. +15; low 4 bits nibble
// tq>>1 of ql[64h + 32(tq&1) + l], high 2 bits bits 2tq of qh[32h + l],
// scale sc[8h + 2tq + (p&1)].  y = fp32(d*sc) * (code - 32).
template <int O>
__device__ __forceinline__ void q6k_scales(uint32_t row, int p, StageScales& S) {
    const float d = h16v(ldsu16(row + O + 208));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int h = q >> 1, tq = 2 * (q & 1) + (p >> 1);
        int16_t scv;
        asm volatile("ld.shared.s8 %0, [%1];" : "=h"(scv) : "r"(row + O + 192 + 8 * h + 2 * tq + (p & 1)));
        split_scale(__fmul_rn(d, static_cast<float>(scv)), S.hi[q], S.lo[q]);
    }
}

template <int O>
__device__ __forceinline__ void q6k_step(uint32_t row, int q, int p, const StageScales& S, uint32_t (&o)[8]) {
    const int h = q >> 1, tq = 2 * (q & 1) + (p >> 1), sb = p & 1;
    uint32_t QL[4], QH[4];
    lds16B<O>(row + 64 * h + 32 * (tq & 1) + 16 * sb, QL);
    lds16B<O>(row + 128 + 32 * h + 16 * sb, QH);
    const int lsh = 4 * (tq >> 1), hsh = 2 * tq;
    const uint32_t hi = S.hi[q], lo = S.lo[q];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t c4 = ((QL[i] >> lsh) & 0x0F0F0F0Fu) | (((QH[i] >> hsh) & 0x03030303u) << 4);
        const uint32_t v01 = bsub2(__byte_perm(c4, kMagic, 0x5140), kB160);   // code - 32, exact
        const uint32_t v23 = bsub2(__byte_perm(c4, kMagic, 0x7362), kB160);
        o[2 * i] = bfma2(v01, hi, bmul2(v01, lo));
        o[2 * i + 1] = bfma2(v23, hi, bmul2(v23, lo));
    }
}

// The same q6_K step for a block at a run-time offset O (even, 0..14) of its
// 16-byte aligned window, as in the flat raw view where every weight row has
// its own offset: 16 bytes from five 4-byte loads joined by byte permutes
// with a per-thread selector (no divergence between threads of one warp).
__device__ __forceinline__ void lds16B_rt(uint32_t a, int O, uint32_t (&w)[4]) {
    const uint32_t base = a + static_cast<uint32_t>(O & ~3);
    const uint32_t sel = (O & 2) ? 0x5432u : 0x3210u;
    uint32_t r[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) r[i] = lds32(base + 4 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __byte_perm(r[i], r[i + 1], sel);
}
__device__ __forceinline__ void q6k_scales_rt(uint32_t row, int O, int p, StageScales& S) {
    const float d = h16v(ldsu16(row + O + 208));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int h = q >> 1, tq = 2 * (q & 1) + (p >> 1);
        int16_t scv;
        asm volatile("ld.shared.s8 %0, [%1];" : "=h"(scv) : "r"(row + O + 192 + 8 * h + 2 * tq + (p & 1)));
        split_scale(__fmul_rn(d, static_cast<float>(scv)), S.hi[q], S.lo[q]);
    }
}
__device__ __forceinline__ void q6k_step_rt(uint32_t row, int O, int q, int p, const StageScales& S,
                                            uint32_t (&o)[8]) {
    const int h = q >> 1, tq = 2 * (q & 1) + (p >> 1), sb = p & 1;
    uint32_t QL[4], QH[4];
    lds16B_rt(row + 64 * h + 32 * (tq & 1) + 16 * sb, O, QL);
    lds16B_rt(row + 128 + 32 * h + 16 * sb, O, QH);
    const int lsh = 4 * (tq >> 1), hsh = 2 * tq;
    const uint32_t hi = S.hi[q], lo = S.lo[q];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t c4 = ((QL[i] >> lsh) & 0x0F0F0F0Fu) | (((QH[i] >> hsh) & 0x03030303u) << 4);
        const uint32_t v01 = bsub2(__byte_perm(c4, kMagic, 0x5140), kB160);   // code - 32, exact
        const uint32_t v23 = bsub2(__byte_perm(c4, kMagic, 0x7362), kB160);
        o[2 * i] = bfma2(v01, hi, bmul2(v01, lo));
        o[2 * i + 1] = bfma2(v23, hi, bmul2(v23, lo));
    }
}

// q5_K: as q4_K with the codes at 48 and the fifth bit of value 64q + 16p + i
// in bit 2q + (p>>1) of qh[16(p&1) + i] (codes 0..31, exact in the same
// bf16 trick).
__device__ __forceinline__ void q5k_step(uint32_t row, int q, int p, const StageScales& S, uint32_t (&o)[8]) {
    const uint4 c = lds128(row + 48 + 32 * q + 16 * (p & 1));
    const uint4 hbits = lds128(row + 16 + 16 * (p & 1));
    const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
    const uint32_t hv[4] = {hbits.x, hbits.y, hbits.z, hbits.w};
    const int j = 2 * q + (p >> 1);
    const uint32_t hi = S.hi[q], lo = S.lo[q], nmm = S.nmm[q];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t nib = (p >> 1) ? ((wv[i] >> 4) & 0x0F0F0F0Fu) : (wv[i] & 0x0F0F0F0Fu);
        const uint32_t code = nib | (((hv[i] >> j) & 0x01010101u) << 4);
        const uint32_t v01 = bsub2(__byte_perm(code, kMagic, 0x5140), kB128);   // (q0, q1) exact
        const uint32_t v23 = bsub2(__byte_perm(code, kMagic, 0x7362), kB128);
        o[2 * i] = bfma2(v01, hi, bfma2(v01, lo, nmm));
        o[2 * i + 1] = bfma2(v23, hi, bfma2(v23, lo, nmm));
    }
}

// q4_0 (eight 18-byte blocks per staged row): step q, part p covers block
// bi = 2q + (p>>1), values 16(p&1) .. +15: the low (p&1 = 0) or high nibbles
// of its 16 code bytes.  code - 8 is exact in bf16 (the 128 + code trick,
// minus 136), multiplied by d split into two bf16 parts as in q6_K.
__device__ __forceinline__ void q40_scales(uint32_t row, int p, StageScales& S) {
#pragma unroll
    for (int q = 0; q < 4; ++q) split_scale(h16v(ldsu16(row + 18 * (2 * q + (p >> 1)))), S.hi[q], S.lo[q]);
}

template <int BI, int SB>
__device__ __forceinline__ void q40_step(uint32_t row, uint32_t hi, uint32_t lo, uint32_t (&o)[8]) {
    constexpr int L = 18 * BI + 2;
    uint32_t QW[4];
    lds16B<(L & 15)>(row + (L & ~15), QW);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = (QW[i] >> (4 * SB)) & 0x0F0F0F0Fu;
        const uint32_t v01 = bsub2(__byte_perm(u, kMagic, 0x5140), kB136);   // code - 8, exact
        const uint32_t v23 = bsub2(__byte_perm(u, kMagic, 0x7362), kB136);
        o[2 * i] = bfma2(v01, hi, bmul2(v01, lo));
        o[2 * i + 1] = bfma2(v23, hi, bmul2(v23, lo));
    }
}

// q8_0 (eight 34-byte blocks per staged row): step q, part p covers block
// bi = 2q + (p>>1), codes 16(p&1) .. +15.  y = fp32(d*q) rounded to bf16.
__device__ __forceinline__ void q8_scales(uint32_t row, int p, StageScales& S) {
#pragma unroll
    for (int q = 0; q < 4; ++q) S.d[q] = h16v(ldsu16(row + 34 * (2 * q + (p >> 1))));
}

template <int BI, int SB>
__device__ __forceinline__ void q8_step(uint32_t row, float d, uint32_t (&o)[8]) {
    constexpr int L = 34 * BI + 2 + 16 * SB;
    uint32_t QW[4];
    lds16B<(L & 15)>(row + (L & ~15), QW);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t u = QW[i] ^ 0x80808080u;   // q + 128
        float f[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t bits = __byte_perm(u, 0x4B000000u, 0x7650 + b);   // 2^23 + q + 128
            f[b] = __fmul_rn(d, __uint_as_float(bits) - 8388736.0f);
        }
        o[2 * i] = pack_bf16x2(f[0], f[1]);
        o[2 * i + 1] = pack_bf16x2(f[2], f[3]);
    }
}

template <int QT>
__device__ __forceinline__ void prep_scales(uint32_t row, int p, int o6, StageScales& S) {
    if constexpr (QT == KQ_Q4_K || QT == KQ_Q5_K) {
        q4k_scales(row, p, S);   // the same header
    } else if constexpr (QT == KQ_Q4_0) {
        q40_scales(row, p, S);
    } else if constexpr (QT == KQ_Q6_K) {
        switch (o6) {
        case 0: q6k_scales<0>(row, p, S); break;
        case 2: q6k_scales<2>(row, p, S); break;
        case 4: q6k_scales<4>(row, p, S); break;
        case 6: q6k_scales<6>(row, p, S); break;
        case 8: q6k_scales<8>(row, p, S); break;
        case 10: q6k_scales<10>(row, p, S); break;
        case 12: q6k_scales<12>(row, p, S); break;
        default: q6k_scales<14>(row, p, S); break;
        }
    } else {
        q8_scales(row, p, S);
    }
}

template <int QT>
__device__ __forceinline__ void decode_step(uint32_t row, int q, int p, int o6, const StageScales& S,
                                            uint32_t (&o)[8]) {
    if constexpr (QT == KQ_Q4_K) {
        q4k_step(row, q, p, S, o);
    } else if constexpr (QT == KQ_Q5_K) {
        q5k_step(row, q, p, S, o);
    } else if constexpr (QT == KQ_Q4_0) {
        const uint32_t hi = S.hi[q], lo = S.lo[q];
        switch (4 * q + p) {
        case 0: q40_step<0, 0>(row, hi, lo, o); break;
        case 1: q40_step<0, 1>(row, hi, lo, o); break;
        case 2: q40_step<1, 0>(row, hi, lo, o); break;
        case 3: q40_step<1, 1>(row, hi, lo, o); break;
        case 4: q40_step<2, 0>(row, hi, lo, o); break;
        case 5: q40_step<2, 1>(row, hi, lo, o); break;
        case 6: q40_step<3, 0>(row, hi, lo, o); break;
        case 7: q40_step<3, 1>(row, hi, lo, o); break;
        case 8: q40_step<4, 0>(row, hi, lo, o); break;
        case 9: q40_step<4, 1>(row, hi, lo, o); break;
        case 10: q40_step<5, 0>(row, hi, lo, o); break;
        case 11: q40_step<5, 1>(row, hi, lo, o); break;
        case 12: q40_step<6, 0>(row, hi, lo, o); break;
        case 13: q40_step<6, 1>(row, hi, lo, o); break;
        case 14: q40_step<7, 0>(row, hi, lo, o); break;
        default: q40_step<7, 1>(row, hi, lo, o); break;
        }
    } else if constexpr (QT == KQ_Q6_K) {
        switch (o6) {
        case 0: q6k_step<0>(row, q, p, S, o); break;
        case 2: q6k_step<2>(row, q, p, S, o); break;
        case 4: q6k_step<4>(row, q, p, S, o); break;
        case 6: q6k_step<6>(row, q, p, S, o); break;
        case 8: q6k_step<8>(row, q, p, S, o); break;
        case 10: q6k_step<10>(row, q, p, S, o); break;
        case 12: q6k_step<12>(row, q, p, S, o); break;
        default: q6k_step<14>(row, q, p, S, o); break;
        }
    } else {
        const float d = S.d[q];
        switch (4 * q + p) {
        case 0: q8_step<0, 0>(row, d, o); break;
        case 1: q8_step<0, 1>(row, d, o); break;
        case 2: q8_step<1, 0>(row, d, o); break;
        case 3: q8_step<1, 1>(row, d, o); break;
        case 4: q8_step<2, 0>(row, d, o); break;
        case 5: q8_step<2, 1>(row, d, o); break;
        case 6: q8_step<3, 0>(row, d, o); break;
        case 7: q8_step<3, 1>(row, d, o); break;
        case 8: q8_step<4, 0>(row, d, o); break;
        case 9: q8_step<4, 1>(row, d, o); break;
        case 10: q8_step<5, 0>(row, d, o); break;
        case 11: q8_step<5, 1>(row, d, o); break;
        case 12: q8_step<6, 0>(row, d, o); break;
        case 13: q8_step<6, 1>(row, d, o); break;
        case 14: q8_step<7, 0>(row, d, o); break;
        default: q8_step<7, 1>(row, d, o); break;
        }
    }
}

// ------------------------------------------------------------- work units
// A unit is (expert, up to 4 map tiles of that expert, one 128-row weight
// tile).  Dense qmm: one pseudo-expert whose tiles are rows 64i..64i+63.
struct Unit {
    int e, ntile, nt;         // expert, weight tile, number of 64-row tiles
    int rs[4], nr[4];         // row_start / num_rows of each tile
    // cont: the tiles are one run of rows [rs0, rs0 + rows) (full tiles back
    // to back, only the last one partial), as in every dense unit and in the
    // units of a map that tiles each expert segment in order
    int cont, rs0, rows;
};

struct Pipe {
    int idx = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1;
        }
    }
};

// Shared-memory stages per CTA: raw weight blocks (RST, 256 values each), A
// (decoded weights, AST) and B (activations, BST), KPS steps of 64 values of K
// each.  A CTA pair halves the activation stage.  Raw stages come from DRAM
// and have the longest latency to cover.  Every stage boundary costs the MMA
// issuing thread a wait and a release, which the shallow MMA queue does not
// hide, so where shared memory allows a stage holds two K steps.  The split
// between A and B stages is measured per codec: q4_K pairs are faster with
// three B stages, q6_K pairs (the heavier decoder) with three A stages.
template <int QT, int CG> struct Stages;
template <> struct Stages<KQ_Q4_K, 1> { static constexpr int RST = 3, AST = 3, BST = 3, KPS = 1; };
template <> struct Stages<KQ_Q6_K, 1> { static constexpr int RST = 3, AST = 2, BST = 3, KPS = 1; };
template <> struct Stages<KQ_Q8_0, 1> { static constexpr int RST = 3, AST = 2, BST = 2, KPS = 1; };
template <> struct Stages<KQ_Q4_K, 2> { static constexpr int RST = 3, AST = 2, BST = 3, KPS = 2; };
template <> struct Stages<KQ_Q6_K, 2> { static constexpr int RST = 2, AST = 3, BST = 2, KPS = 2; };
template <> struct Stages<KQ_Q8_0, 2> { static constexpr int RST = 3, AST = 3, BST = 4, KPS = 1; };
template <> struct Stages<KQ_Q5_K, 1> { static constexpr int RST = 3, AST = 2, BST = 3, KPS = 1; };
template <> struct Stages<KQ_Q5_K, 2> { static constexpr int RST = 2, AST = 2, BST = 3, KPS = 2; };
template <> struct Stages<KQ_Q4_0, 1> { static constexpr int RST = 3, AST = 3, BST = 3, KPS = 1; };
template <> struct Stages<KQ_Q4_0, 2> { static constexpr int RST = 3, AST = 2, BST = 3, KPS = 2; };

// The flat raw view (q6_K rows that are not a 16-byte multiple) loads each
// row's 240-byte window with its own tensor copy, whose shared-memory
// destination must be 128-byte aligned: rows of raw stages are then 256
// bytes apart, and fewer stages fit (two of each).
template <int QT, int CG, bool FLAT> struct StagesOf : Stages<QT, CG> {
    static constexpr int RAWB = QmmCodec<QT>::RAWB;
};
template <int CG> struct StagesOf<KQ_Q6_K, CG, true> {
    static constexpr int RST = 2, AST = 2, BST = CG == 2 ? 2 : 3, KPS = Stages<KQ_Q6_K, CG>::KPS;
    static constexpr int RAWB = 256;
};

template <int QT, int CG, bool FLAT = false>
constexpr uint32_t smem_bytes() {
    using S = StagesOf<QT, CG, FLAT>;
    return kHeader + 1024 + S::BST * S::KPS * (kBN / CG) * kBK * 2 + S::AST * S::KPS * kBM * kBK * 2 +
           S::RST * kBM * S::RAWB;
}

// FLAT (q6_K only): the weight rows are not a 16-byte multiple, so the raw
// tensor map is a rank-1 view of all the weight bytes; the raw producer loads
// each row's 16-byte aligned window of a block separately, and each decoder
// thread takes its row's offset in the window at run time.
template <int QT, int CG, bool FLAT = false>
__global__ void __launch_bounds__(kThreads, 1)
    qmm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
               const QmmParams p) {
    static_assert(!FLAT || QT == KQ_Q6_K, "the flat raw view serves q6_K");
    using C = QmmCodec<QT>;
    using SO = StagesOf<QT, CG, FLAT>;
    constexpr int RST = SO::RST;
    constexpr int AST = SO::AST;
    constexpr int BST = SO::BST;
    constexpr int KPS = SO::KPS;     // 64-value K steps per A/B stage
    constexpr int RAWB = SO::RAWB;   // shared-memory bytes of a raw stage row
    static_assert(RST <= 4 && AST <= 4 && BST <= 8, "barrier table holds 4 raw, 4 A and 8 B stages");
    static_assert(KPS == 1 || KPS == 2, "a raw stage (4 K steps) holds whole A/B stages");
    static_assert(smem_bytes<QT, CG, FLAT>() <= 232448, "shared memory per CTA");
    constexpr int kBNc = kBN / CG;                    // activation rows of a B stage in this CTA
    constexpr uint32_t kRawBytes = kBM * RAWB;
    constexpr uint32_t kAAtom = kBM * kBK * 2;       // 16 KB: one K step of A
    constexpr uint32_t kBAtom = kBNc * kBK * 2;      // 32 KB (one CTA) or 16 KB (pair): one K step of B
    constexpr uint32_t kABytes = KPS * kAAtom;
    constexpr uint32_t kBBytes = KPS * kBAtom;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sb = smem_u32(smem);
    // stage regions (1024-aligned): B stages, A stages, raw stages; the same
    // offsets in both CTAs of a pair, as the pair's MMA descriptors require
    const uint32_t base = (sb + kHeader + 1023) & ~1023u;
    const uint32_t bst = base, ast = bst + BST * kBBytes, rst = ast + AST * kABytes;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
    uint64_t* raw_full = bars;
    uint64_t* raw_empty = bars + 4;
    uint64_t* a_full = bars + 8;
    uint64_t* a_empty = bars + 12;
    uint64_t* b_full = bars + 16;
    uint64_t* b_empty = bars + 24;
    uint64_t* acc_full = bars + 32;
    uint64_t* acc_empty = bars + 34;
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + Smem::kMisc);
    // misc[0] tmem base, misc[1] abort, misc[2] number of chunks, misc[3] tiles
    uint16_t* tiles = reinterpret_cast<uint16_t*>(smem + Smem::kTiles);          // sorted valid tile ids
    int* cstart = reinterpret_cast<int*>(smem + Smem::kTiles + 2 * kMaxTiles);    // per expert chunk prefix [257]
    int* tstart = cstart + 257;                                                  // per expert tile prefix [257]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0;   // 0 = the pair's MMA-issuing CTA
    // full barriers the pair's MMA waits on live in CTA 0 of the pair
    auto lead = [&](uint64_t* bar) { return CG == 2 ? mapa_u32(smem_u32(bar), 0) : smem_u32(bar); };

    // ---- set-up: barriers, TMEM, work list
    if (tid == 0) {
        for (int i = 0; i < RST; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], kDecWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4 * CG);
        }
        for (int i = 0; i < AST; ++i) {
            mbar_init(&a_full[i], kDecWarps * CG);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < BST; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        misc[1] = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc512<CG>(sb + Smem::kMisc);
    int total_units;
    if (p.n_experts == 0) {
        total_units = p.units;
    } else {
        // Gather: this launch takes the window [win0, win0 + kMaxTiles) of
        // the map's first `count` tiles (a larger map is served by further
        // launches).  Validate the window, keep its valid tiles, group them by
        // expert in map order and cut each expert's list into chunks of 4.
        // Both CTAs of a pair build the same tables.
        int64_t cnt = static_cast<int64_t>(*p.count);
        if (cnt > p.cap) {
            if (tid == 0 && p.win0 == 0 && p.err) atomicOr(p.err, KQ_DEV_BAD_RANGE);
            cnt = p.cap;
        }
        const int wn = static_cast<int>(cnt - p.win0 < 0 ? 0 : (cnt - p.win0 < kMaxTiles ? cnt - p.win0 : kMaxTiles));
        const uint32_t* wmap_t = p.map + 3 * p.win0;   // the window's tiles
        for (int e = tid; e < 257; e += kThreads) cstart[e] = tstart[e] = 0;
        __syncthreads();
        // validity and per-expert counts
        auto tile_ok = [&](int i, uint32_t& e) {
            e = wmap_t[3 * i];
            const uint32_t rs = wmap_t[3 * i + 1], nr = wmap_t[3 * i + 2];
            int bad = 0;
            if (e >= static_cast<uint32_t>(p.n_experts)) bad |= KQ_DEV_BAD_EXPERT;
            if (nr == 0 || nr > 64) bad |= KQ_DEV_BAD_ROWS;
            if (static_cast<int64_t>(rs) + nr > p.m) bad |= KQ_DEV_BAD_RANGE;
            return bad;
        };
        for (int i = tid; i < wn; i += kThreads) {
            uint32_t e;
            const int bad = tile_ok(i, e);
            if (bad) {
                if (p.err) atomicOr(p.err, bad);
            } else {
                atomicAdd(&tstart[e + 1], 1);
            }
        }
        __syncthreads();
        // first slot of every expert's list (tstart), and a running fill
        // pointer per expert (cstart, turned into the chunk prefix below)
        if (tid == 0) {
            int tacc = 0;
            for (int e = 0; e < p.n_experts; ++e) {
                const int te = tstart[e + 1];
                tstart[e] = tacc;
                cstart[e] = tacc;
                tacc += te;
            }
            tstart[p.n_experts] = tacc;
        }
        __syncthreads();
        // place: one warp walks the window in map order, 32 tiles at a time;
        // a valid tile goes to its expert's next free slot (lanes of one
        // expert in a step ranked among themselves), so each expert's list
        // keeps map order, which is row order for kq_expert_tile_map's maps
        if (warp == 0) {
            for (int i0 = 0; i0 < wn; i0 += 32) {
                const int i = i0 + lane;
                uint32_t e = 0xFFFFFFFFu;
                if (i < wn && tile_ok(i, e) != 0) e = 0xFFFFFFFFu;
                const unsigned same = __match_any_sync(0xffffffffu, e);
                const unsigned below = same & ((1u << lane) - 1u);
                int pos = 0;
                if (e != 0xFFFFFFFFu) pos = cstart[e] + __popc(below);
                __syncwarp();
                if (e != 0xFFFFFFFFu) {
                    tiles[pos] = static_cast<uint16_t>(i);
                    if (below == 0) cstart[e] += __popc(same);
                }
                __syncwarp();
            }
        }
        __syncthreads();
        if (tid == 0) {
            int cacc = 0;
            for (int e = 0; e < p.n_experts; ++e) {
                cstart[e] = cacc;
                cacc += (tstart[e + 1] - tstart[e] + 3) / 4;
            }
            cstart[p.n_experts] = cacc;
            misc[2] = cacc;
        }
        total_units = 0;   // read after the barrier below
    }
    tc_fence_before();
    // the pair's barriers and TMEM are set up before any CTA of it goes on
    if constexpr (CG == 2) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    // gather: units are (chunk of <= 4 map tiles, weight tile); as for dense
    // qmm, the units of the last, partial round of the grid are split, here
    // into sub-units of one or two map tiles, so that they spread over more
    // CTAs (every thread derives the same split from the chunk count)
    int g_main = 0, g_split = 1;
    if (p.n_experts != 0) {
        total_units = static_cast<int>(misc[2]) * p.ntn;
        const int ng = static_cast<int>(gridDim.x) / CG;
        g_main = total_units;
        const int tail = total_units % ng;
        if (total_units > ng && tail != 0) {
            g_split = 4 * tail <= ng ? 4 : (2 * tail <= ng ? 2 : 1);
            g_main = total_units - tail;
            total_units = g_main + g_split * tail;
        }
    }
    // a unit is processed by one CTA (CG = 1) or one CTA pair (CG = 2)
    const int u0 = static_cast<int>(blockIdx.x) / CG, ustep = static_cast<int>(gridDim.x) / CG;

    auto get_unit = [&](int u, Unit& U) {
        if (p.n_experts == 0) {
            // units below units_main: (256 activation rows, weight tile); the
            // units of the last, partial round of the grid are split into
            // `split` sub-units of 256/split rows so that they spread over
            // more SMs (a sub-unit past the end of m has nt = 0: skipped)
            const int mtiles = static_cast<int>((p.m + kBN - 1) / kBN);
            int fu = u, sub = -1;
            if (u >= p.units_main) {
                fu = p.units_main + (u - p.units_main) / p.split;
                sub = (u - p.units_main) % p.split;
            }
            const int mt = fu % mtiles;
            U.e = 0;
            U.ntile = fu / mtiles;
            int64_t r0 = static_cast<int64_t>(mt) * kBN;
            int64_t left = p.m - r0;
            if (sub >= 0) {
                const int rows = kBN / p.split;
                r0 += static_cast<int64_t>(rows) * sub;
                left = left - static_cast<int64_t>(rows) * sub;
                left = left < 0 ? 0 : (left > rows ? rows : left);
            }
            U.nt = static_cast<int>(left >= kBN ? 4 : (left + 63) / 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                U.rs[i] = static_cast<int>(r0 + 64 * i);
                const int64_t ri = left - 64 * i;
                U.nr[i] = ri <= 0 ? 0 : (ri >= 64 ? 64 : static_cast<int>(ri));
            }
        } else {
            const int nch = static_cast<int>(misc[2]);
            int fu = u, sub = -1;
            if (u >= g_main) {
                fu = g_main + (u - g_main) / g_split;
                sub = (u - g_main) % g_split;
            }
            const int c = fu % nch;
            U.ntile = fu / nch;
            int lo = 0, hi = p.n_experts - 1;   // expert with cstart[e] <= c < cstart[e+1]
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (cstart[mid] <= c) lo = mid;
                else hi = mid - 1;
            }
            U.e = lo;
            int first = tstart[lo] + 4 * (c - cstart[lo]);
            int left = tstart[lo + 1] - first;
            if (sub >= 0) {   // sub-unit: tiles [sub * per, sub * per + per) of the chunk
                const int per = 4 / g_split;
                first += sub * per;
                left -= sub * per;
                left = left < 0 ? 0 : (left > per ? per : left);
            }
            U.nt = left >= 4 ? 4 : left;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i < U.nt) {
                    const int ti = tiles[first + i];
                    U.rs[i] = static_cast<int>(p.map[3 * (p.win0 + ti) + 1]);
                    U.nr[i] = static_cast<int>(p.map[3 * (p.win0 + ti) + 2]);
                } else {
                    U.rs[i] = 0;
                    U.nr[i] = 0;
                }
            }
        }
        U.cont = 1;
#pragma unroll
        for (int i = 1; i < 4; ++i)
            if (i < U.nt && (U.nr[i - 1] != 64 || U.rs[i] != U.rs[i - 1] + 64)) U.cont = 0;
        U.rs0 = U.rs[0];
        U.rows = U.nt > 0 ? 64 * (U.nt - 1) + U.nr[U.nt - 1] : 0;
    };
    // MMA N: one CTA trims it to the rows present.  A pair splits N evenly
    // between its CTAs (CTA r holds B rows [rN/2, (r+1)N/2)): a run of rows
    // takes N = rows rounded up to 32 (each CTA then holds a multiple of 16
    // rows, loaded as 64-row boxes from the run's start), tiles that are not
    // one run keep whole tiles per CTA, N = 128 (one each) or 256 (two each).
    auto mma_n = [&](const Unit& U) {
        if constexpr (CG == 2) return U.cont ? (U.rows + 31) & ~31 : (U.nt <= 2 ? 128 : 256);
        else return 64 * (U.nt - 1) + ((U.nr[U.nt - 1] + 15) & ~15);
    };
    auto aborted = [&]() { return misc[1] != 0; };
    auto bwait = [&](uint64_t* bar, uint32_t parity) {
        if (misc[1]) return false;
        if (!mbar_wait(bar, parity, p.status)) {
            misc[1] = 1;
            return false;
        }
        return true;
    };

    const int ksteps = p.k / kBK;
    const int nstages = ksteps / KPS;   // A/B stages per unit (ksteps is a multiple of 4)
    const int wtile_rows = kBM * CG;   // weight rows of a unit
    if (warp == 0) {
        // ------------------------------------------------ activation producer
        if (lane == 0) {
            Pipe bp;
            for (int u = u0; u < total_units && !aborted(); u += ustep) {
                Unit U;
                get_unit(u, U);
                if (U.nt == 0) continue;
                // this CTA's activation tiles of the unit: [t0, t1), at 64-row slots from 0
                int t0 = 0, t1 = U.nt;
                // a run of rows (pair): this CTA's rows start at `cr`; boxes
                // (64 rows each, slots from 0) are loaded while they start
                // inside the run, rows past it are never stored
                int cr = 0, cb = 0, boxes = U.nt;
                if constexpr (CG == 2) {
                    if (U.cont) {
                        const int half = mma_n(U) / 2;
                        cr = static_cast<int>(rank) * half;
                        boxes = 0;
                        for (int r = 0; r < 2; ++r)
                            for (int b = 0; 64 * b < half; ++b) {
                                const bool in = r * half + 64 * b < U.rows;
                                boxes += in;
                                if (r == static_cast<int>(rank)) cb += in;
                            }
                    } else {
                        const int tpc = mma_n(U) / 128;
                        t0 = static_cast<int>(rank) * tpc;
                        t1 = t0 + tpc < U.nt ? t0 + tpc : U.nt;
                    }
                }
                for (int st = 0; st < nstages; ++st) {
                    if (!bwait(&b_empty[bp.idx], bp.phase ^ 1)) break;
                    const uint32_t dst = bst + bp.idx * kBBytes;
                    if constexpr (CG == 2) {
                        // both CTAs' bytes land on CTA 0's full barrier; CTA 0
                        // expects the unit's total
                        if (rank == 0) mbar_arrive_expect_tx(&b_full[bp.idx], KPS * boxes * 8192);
                        const uint32_t fb = lead(&b_full[bp.idx]);
                        if (U.cont) {
#pragma unroll
                            for (int a = 0; a < KPS; ++a)
                                for (int b = 0; b < cb; ++b)
                                    tma_load_2d_pair(dst + a * kBAtom + b * 8192, &xmap, (st * KPS + a) * kBK,
                                                     U.rs0 + cr + 64 * b, fb);
                        } else {
#pragma unroll
                            for (int a = 0; a < KPS; ++a)
                                for (int i = t0; i < t1; ++i)
                                    tma_load_2d_pair(dst + a * kBAtom + (i - t0) * 8192, &xmap, (st * KPS + a) * kBK,
                                                     U.rs[i], fb);
                        }
                    } else {
                        mbar_arrive_expect_tx(&b_full[bp.idx], KPS * U.nt * 8192);
#pragma unroll
                        for (int a = 0; a < KPS; ++a)
                            for (int i = t0; i < t1; ++i)
                                tma_load_2d(dst + a * kBAtom + i * 8192, &xmap, (st * KPS + a) * kBK, U.rs[i], &b_full[bp.idx]);
                    }
                    bp.next(BST);
                }
            }
        }
    } else if (warp == kRawWarp) {
        // ------------------------------------------------ raw weight producer
        // One 256-value block column of this CTA's 128 weight rows per stage,
        // straight from the wire bytes; the block kRawAhead stages ahead is
        // prefetched into L2 so that the load it later issues finds it there.
        if constexpr (FLAT) {
            // flat view: lane l loads the windows of rows l, l + 32, l + 64,
            // l + 96 (240 bytes each, from the 16-byte boundary at or below
            // the block's first byte, into a 256-byte slot: a tensor copy's
            // shared-memory destination is 128-byte aligned; past the end of
            // the weights the tensor map fills zeros); lane 0 waits and sets
            // the byte count
            Pipe rp;
            const int nblk = ksteps / 4;
            for (int u = u0; u < total_units && !aborted(); u += ustep) {
                Unit U;
                get_unit(u, U);
                if (U.nt == 0) continue;
                const int64_t wrow = static_cast<int64_t>(U.e) * p.n + U.ntile * wtile_rows + kBM * static_cast<int>(rank);
                bool ok = true;
                for (int blk = 0; blk < nblk; ++blk) {
                    if (lane == 0) {
                        ok = bwait(&raw_empty[rp.idx], rp.phase ^ 1);
                        // 128 windows of C::RAWB (240) bytes land in 256-byte slots
                        if (ok) mbar_arrive_expect_tx(&raw_full[rp.idx], kBM * C::RAWB);
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
#pragma unroll
                    for (int j = 0; j < kBM / 32; ++j) {
                        const int r = lane + 32 * j;
                        const int64_t b0 = (wrow + r) * p.row_bytes + 210 * blk;
                        tma_load_1d(rst + rp.idx * kRawBytes + r * RAWB, &wmap, static_cast<int>(b0 & ~int64_t(15)),
                                    &raw_full[rp.idx]);
                    }
                    rp.next(RST);
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
        } else if (lane == 0) {
            Pipe rp;
            const int nblk = ksteps / 4;
            auto xcol = [&](int blk) {
                if constexpr (QT == KQ_Q4_K || QT == KQ_Q4_0) return 144 * blk;
                else if constexpr (QT == KQ_Q5_K) return 176 * blk;
                else if constexpr (QT == KQ_Q6_K) return (210 * blk) & ~15;
                else return 136 * blk;   // 2-byte elements
            };
            for (int u = u0; u < total_units && !aborted(); u += ustep) {
                Unit U;
                get_unit(u, U);
                if (U.nt == 0) continue;
                const int wrow = U.e * static_cast<int>(p.n) + U.ntile * wtile_rows + kBM * static_cast<int>(rank);
                for (int b = 0; b < kRawAhead && b < nblk; ++b) tma_prefetch_2d(&wmap, xcol(b), wrow);
                for (int blk = 0; blk < nblk; ++blk) {
                    if (blk + kRawAhead < nblk) tma_prefetch_2d(&wmap, xcol(blk + kRawAhead), wrow);
                    if (!bwait(&raw_empty[rp.idx], rp.phase ^ 1)) break;
                    mbar_arrive_expect_tx(&raw_full[rp.idx], kRawBytes);
                    tma_load_2d(rst + rp.idx * kRawBytes, &wmap, xcol(blk), wrow, &raw_full[rp.idx]);
                    rp.next(RST);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (CTA 0 of a pair)
        if (lane == 0 && rank == 0) {
            Pipe ap, bp, cp;
            for (int u = u0; u < total_units && !aborted(); u += ustep) {
                Unit U;
                get_unit(u, U);
                if (U.nt == 0) continue;
                const uint32_t idesc = make_idesc(mma_n(U), kBM * CG);
                if (!bwait(&acc_empty[cp.idx], cp.phase ^ 1)) break;
                tc_fence_after();
                const uint32_t dt = tmem + cp.idx * 256;
                bool ok = true;
                // The issue loop is on the critical path of the tensor pipe
                // (the MMA queue is shallow: whatever this thread does between
                // two MMAs can leave the pipe idle), so the bookkeeping of a
                // stage sits between the MMAs of the next one: the previous
                // stage's release (commit) after the first MMA, the poll of
                // the next stage after the second.  The bounded wait runs
                // only when a stage is not complete yet.
                bool ra = false, rb = false;   // stage seen complete by the poll
                int pa = -1, pb = -1;          // stages whose release is pending
                for (int st = 0; st < nstages; ++st) {
                    if (!ra && !mbar_try_wait(&a_full[ap.idx], ap.phase) && !bwait(&a_full[ap.idx], ap.phase)) {
                        ok = false;
                        break;
                    }
                    if (!rb && !mbar_try_wait(&b_full[bp.idx], bp.phase) && !bwait(&b_full[bp.idx], bp.phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(ast + ap.idx * kABytes);
                    const uint64_t bd = sw128_desc(bst + bp.idx * kBBytes);
                    tc_mma<CG>(dt, ad, bd, idesc, st != 0);
                    if (pa >= 0) {
                        tc_commit<CG>(&a_empty[pa]);
                        tc_commit<CG>(&b_empty[pb]);
                    }
                    tc_mma<CG>(dt, ad + 2, bd + 2, idesc, 1);
                    Pipe an = ap, bn = bp;
                    an.next(AST);
                    bn.next(BST);
                    ra = st + 1 < nstages && mbar_try_wait(&a_full[an.idx], an.phase);
                    rb = st + 1 < nstages && mbar_try_wait(&b_full[bn.idx], bn.phase);
                    // descriptor start addresses advance 32 bytes (2 units) per
                    // 16-value K slice inside an atom, one atom per K step
#pragma unroll
                    for (int kk = 2; kk < KPS * (kBK / 16); ++kk) {
                        const int a = kk / (kBK / 16), sl = kk % (kBK / 16);
                        tc_mma<CG>(dt, ad + (a * kAAtom >> 4) + 2 * sl, bd + (a * kBAtom >> 4) + 2 * sl, idesc, 1);
                    }
                    pa = ap.idx;
                    pb = bp.idx;
                    ap = an;
                    bp = bn;
                }
                if (pa >= 0) {
                    tc_commit<CG>(&a_empty[pa]);
                    tc_commit<CG>(&b_empty[pb]);
                }
                if (!ok) break;
                tc_commit<CG>(&acc_full[cp.idx]);
                cp.next(2);
            }
        }
    } else if (warp < kDeqWarp0) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        Pipe cp;
        for (int u = u0; u < total_units && !aborted(); u += ustep) {
            Unit U;
            get_unit(u, U);
            if (U.nt == 0) continue;
            const int nmma = mma_n(U);
            if (!bwait(&acc_full[cp.idx], cp.phase)) break;
            tc_fence_after();
            const int64_t nrow = static_cast<int64_t>(U.ntile) * wtile_rows + kBM * static_cast<int>(rank) + 32 * q + lane;
            const bool row_ok = nrow < p.n;
            const uint32_t tbase = tmem + cp.idx * 256 + (static_cast<uint32_t>(32 * q) << 16);
            for (int c0 = 0; c0 < nmma; c0 += 16) {
                // activation row of column c0 and the valid rows of this
                // 16-column chunk (column j is B row j: a run's row rs0 + j,
                // else row j % 64 of tile j / 64)
                int nv;
                int64_t ar;
                if (CG == 2 && U.cont) {
                    nv = U.rows - c0;
                    ar = static_cast<int64_t>(U.rs0) + c0;
                } else {
                    const int ti = c0 >> 6, r0 = c0 & 63;
                    nv = U.nr[ti] - r0;
                    ar = static_cast<int64_t>(U.rs[ti]) + r0;
                }
                if (nv <= 0) continue;          // warp-uniform
                uint32_t v[16];
                tmem_ld16(tbase + c0, v);
                if (row_ok) {
                    // y is written once and never read here: streaming stores
                    float* yp = p.y + ar * p.n + nrow;
                    if (nv >= 16) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) __stcs(yp + i * p.n, __uint_as_float(v[i]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (i < nv) __stcs(yp + i * p.n, __uint_as_float(v[i]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2) mbar_arrive_remote(lead(&acc_empty[cp.idx]));
                else mbar_arrive(&acc_empty[cp.idx]);
            }
            cp.next(2);
        }
    } else {
        // ------------------------------------------------ decoders
        const int dt = tid - kDeqWarp0 * 32;   // 0..511
        const int r = dt & 127, part = dt >> 7;
        // swizzled offsets of the thread's two 16-byte chunks (2p, 2p+1) in an A stage
        const uint32_t rowb = (r >> 3) * 1024 + (r & 7) * 128;
        const uint32_t so0 = rowb + (((2 * part) ^ (r & 7)) << 4), so1 = rowb + (((2 * part + 1) ^ (r & 7)) << 4);
        Pipe rp, ap;
        StageScales S;
        for (int u = u0; u < total_units && !aborted(); u += ustep) {
            Unit U;
            get_unit(u, U);
            if (U.nt == 0) continue;
            bool ok = true;
            // flat view: this thread's row starts at rbyte (its window offset
            // moves with every block)
            int64_t rbyte = 0;
            if constexpr (FLAT)
                rbyte = (static_cast<int64_t>(U.e) * p.n + U.ntile * wtile_rows + kBM * static_cast<int>(rank) + r) *
                        p.row_bytes;
            for (int ks0 = 0; ks0 < ksteps && ok; ks0 += 4) {
                const uint32_t row = rst + rp.idx * kRawBytes + r * RAWB;
                const int o6 = QT != KQ_Q6_K ? 0
                               : FLAT        ? static_cast<int>((rbyte + 210 * (ks0 >> 2)) & 15)
                                             : (210 * (ks0 >> 2)) & 15;
                if (!bwait(&raw_full[rp.idx], rp.phase)) {
                    ok = false;
                    break;
                }
                if constexpr (FLAT) q6k_scales_rt(row, o6, part, S);
                else prep_scales<QT>(row, part, o6, S);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int a = q % KPS;   // K step within the A stage
                    if (a == 0 && !bwait(&a_empty[ap.idx], ap.phase ^ 1)) {
                        ok = false;
                        break;
                    }
                    uint32_t o[8];
                    if constexpr (FLAT) q6k_step_rt(row, o6, q, part, S, o);
                    else decode_step<QT>(row, q, part, o6, S, o);
                    const uint32_t ab = ast + ap.idx * kABytes + a * kAAtom;
                    sts128(ab + so0, o[0], o[1], o[2], o[3]);
                    sts128(ab + so1, o[4], o[5], o[6], o[7]);
                    if (a == KPS - 1) {
                        fence_proxy_async();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (CG == 2) mbar_arrive_remote(lead(&a_full[ap.idx]));
                            else mbar_arrive(&a_full[ap.idx]);
                        }
                        ap.next(AST);
                    }
                }
                if (!ok) break;
                if (lane == 0) mbar_arrive(&raw_empty[rp.idx]);
                rp.next(RST);
            }
            if (!ok) break;
        }
    }

    // ---- tear-down: neither CTA of a pair leaves while the other may still
    // read its shared memory or signal its barriers
    __syncwarp();
    tc_fence_before();
    if constexpr (CG == 2) cluster_sync();
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc512<CG>(tmem);
    }
}

// ------------------------------------------------------------------ host
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encoder() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    }
    return fn;
}

int make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* ptr, uint64_t inner, uint64_t outer,
             uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
    EncodeTiled enc = get_encoder();
    if (!enc) return KQ_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * esize};
    const cuuint32_t box[2] = {box_in, box_out};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KQ_OK : KQ_ERR_INVALID_ARG;
}

// Rank-1 byte map over `bytes` bytes at w (16-byte aligned), boxes of `box`
// bytes (a multiple of 16); reads past the end are zero-filled.
int make_map_1d(CUtensorMap* m, const void* w, uint64_t bytes, uint32_t box) {
    EncodeTiled enc = get_encoder();
    if (!enc) return KQ_ERR_CUDA;
    const cuuint64_t dims[1] = {bytes};
    const cuuint64_t strides[1] = {bytes};   // unused at rank 1
    const cuuint32_t boxd[1] = {box};
    const cuuint32_t estr[1] = {1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, const_cast<void*>(w), dims, strides, boxd, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KQ_OK : KQ_ERR_INVALID_ARG;
}

// Launch with units of 128 (one CTA) or 256 (a CTA pair) weight rows; a pair
// is a cluster of two CTAs on neighbouring SMs.
template <int QT, int CG, bool FLAT = false>
int launch_cg(const CUtensorMap& wmap, const CUtensorMap& xmap, QmmParams p, cudaStream_t s) {
    constexpr uint32_t smem = smem_bytes<QT, CG, FLAT>();
    auto kern = qmm_kernel<QT, CG, FLAT>;
    static bool attr_set[64] = {false};
    static int slots[64] = {0};   // CTAs of this kernel resident at once, per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return record_cuda(e);
        int n = device_sm_count();
        if (CG == 2) {
            cudaLaunchConfig_t q = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = 2;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            q.gridDim = dim3(2 * (n / 2), 1, 1);
            q.blockDim = dim3(kThreads, 1, 1);
            q.dynamicSmemBytes = smem;
            q.attrs = at;
            q.numAttrs = 1;
            int clusters = 0;
            e = cudaOccupancyMaxActiveClusters(&clusters, kern, &q);
            if (e != cudaSuccess) return record_cuda(e);
            n = 2 * clusters;
        }
        if (n < CG) return KQ_ERR_UNSUPPORTED;
        slots[dev] = n;
        attr_set[dev] = true;
    }
    const int groups = slots[dev] / CG;   // CTAs or CTA pairs resident at once
    p.ntn = static_cast<int>((p.n + kBM * CG - 1) / (kBM * CG));
    p.units = p.n_experts == 0 ? static_cast<int>((p.m + kBN - 1) / kBN) * p.ntn : 0;
    p.units_main = p.units;
    p.split = 1;
    int ng = groups;
    if (p.n_experts == 0 && p.units < ng) ng = p.units;
    if (ng < 1) return KQ_OK;
    if (p.n_experts == 0 && p.units > ng && p.units % ng != 0 && p.m > 64) {
        // the last, partial round: its units become sub-units, as many per
        // unit as still fit in one round of the grid
        const int tail = p.units % ng;
        p.split = 4 * tail <= ng ? 4 : (2 * tail <= ng ? 2 : 1);
        p.units_main = p.units - tail;
        p.units = p.units_main + p.split * tail;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CG;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(ng * CG), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = at;
    cfg.numAttrs = CG == 2 ? 1 : 0;
    // gather: one launch per window of kMaxTiles map slots (the valid-tile
    // count is on the device; a window past it has no units)
    const int64_t windows = p.n_experts == 0 ? 1 : (p.cap + kMaxTiles - 1) / kMaxTiles;
    for (int64_t w = 0; w < (windows > 0 ? windows : 1); ++w) {
        p.win0 = w * kMaxTiles;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, wmap, xmap, p);
        if (e != cudaSuccess) return record_cuda(e);
    }
    return check_launch();
}

template <int QT>
int launch_impl(const void* w, int64_t w_rows, int64_t n, int64_t k, const uint16_t* x, int64_t x_rows, int n_experts,
                const uint32_t* map, const uint32_t* count, int64_t cap, float* y, int32_t* err, cudaStream_t s) {
    using C = QmmCodec<QT>;
    const int vpb = (QT == KQ_Q8_0 || QT == KQ_Q4_0) ? 32 : 256;
    const int bpb = QT == KQ_Q4_K ? 144 : QT == KQ_Q5_K ? 176 : QT == KQ_Q6_K ? 210 : QT == KQ_Q4_0 ? 18 : 34;
    const int64_t row_bytes = k / vpb * bpb;
    if (k % 256 != 0) return KQ_ERR_UNSUPPORTED;        // 256-value raw stages
    // rows that are not a 16-byte multiple (q6_K with K / 256 not a multiple
    // of 8) take the flat raw view: a rank-1 map over all the weight bytes,
    // whose coordinates (bytes, 32-bit) must cover the last tile's rows
    const bool flat = row_bytes % 16 != 0;
    if (flat && (QT != KQ_Q6_K || (w_rows + 2 * kBM) * row_bytes >= (int64_t(1) << 31))) return KQ_ERR_UNSUPPORTED;
    CUtensorMap wmap, xmap;
    int rc;
    if (flat)
        rc = make_map_1d(&wmap, w, static_cast<uint64_t>(w_rows * row_bytes), C::RAWB);
    else if constexpr (QT == KQ_Q8_0)
        rc = make_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w, row_bytes / 2, w_rows, C::RAWB / 2, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        rc = make_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w, row_bytes, w_rows, C::RAWB, kBM,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    rc = make_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, k, x_rows, kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;

    QmmParams p{};
    p.n = n;
    p.m = x_rows;
    p.k = static_cast<int>(k);
    p.n_experts = n_experts;
    p.map = map;
    p.count = count;
    p.cap = cap;
    p.y = y;
    p.err = err;
    p.status = device_status_ptr();
    p.row_bytes = row_bytes;
    if constexpr (QT == KQ_Q6_K) {
        if (flat) return use_pair_mma() ? launch_cg<QT, 2, true>(wmap, xmap, p, s) : launch_cg<QT, 1, true>(wmap, xmap, p, s);
    }
    return use_pair_mma() ? launch_cg<QT, 2>(wmap, xmap, p, s) : launch_cg<QT, 1>(wmap, xmap, p, s);
}

}  // namespace

int launch_qmm(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m, float* y,
               cudaStream_t s) {
    if (n == 0 || m == 0) return KQ_OK;
    switch (type) {
    case KQ_Q4_K: return launch_impl<KQ_Q4_K>(w, n, n, k, x, m, 0, nullptr, nullptr, 0, y, nullptr, s);
    case KQ_Q6_K: return launch_impl<KQ_Q6_K>(w, n, n, k, x, m, 0, nullptr, nullptr, 0, y, nullptr, s);
    case KQ_Q8_0: return launch_impl<KQ_Q8_0>(w, n, n, k, x, m, 0, nullptr, nullptr, 0, y, nullptr, s);
    case KQ_Q5_K: return launch_impl<KQ_Q5_K>(w, n, n, k, x, m, 0, nullptr, nullptr, 0, y, nullptr, s);
    case KQ_Q4_0: return launch_impl<KQ_Q4_0>(w, n, n, k, x, m, 0, nullptr, nullptr, 0, y, nullptr, s);
    default: return KQ_ERR_UNSUPPORTED;
    }
}

int launch_gather_qmm(int type, const void* w_bank, int n_experts, int64_t n, int64_t k, const uint16_t* x_sorted,
                      int64_t rows, const uint32_t* map, const uint32_t* count, int64_t cap, float* y,
                      int32_t* err_flag, cudaStream_t s) {
    if (n == 0 || rows == 0) return KQ_OK;
    const int64_t wr = static_cast<int64_t>(n_experts) * n;
    switch (type) {
    case KQ_Q4_K:
        return launch_impl<KQ_Q4_K>(w_bank, wr, n, k, x_sorted, rows, n_experts, map, count, cap, y, err_flag, s);
    case KQ_Q6_K:
        return launch_impl<KQ_Q6_K>(w_bank, wr, n, k, x_sorted, rows, n_experts, map, count, cap, y, err_flag, s);
    case KQ_Q8_0:
        return launch_impl<KQ_Q8_0>(w_bank, wr, n, k, x_sorted, rows, n_experts, map, count, cap, y, err_flag, s);
    case KQ_Q5_K:
        return launch_impl<KQ_Q5_K>(w_bank, wr, n, k, x_sorted, rows, n_experts, map, count, cap, y, err_flag, s);
    case KQ_Q4_0:
        return launch_impl<KQ_Q4_0>(w_bank, wr, n, k, x_sorted, rows, n_experts, map, count, cap, y, err_flag, s);
    default: return KQ_ERR_UNSUPPORTED;
    }
}

}  // namespace kq
