// kq_qmv for 1 <= m <= 2 (q8_0, q6_K, q4_0) or m <= 16 (q4_K, q5_K):
// y = x . W^T; also the decode MoE products (gather and GLU modes).
//
// mlx-kquant bindings.cpp `quantized_matmul` (x @ dequant(w).T) and README
// "How it works" (small row counts take a kernel that amortizes each weight
// read over all rows); hanzo-ml quantized/mod.rs (decode multiplies directly
// on the packed blocks).  Block layouts: mlx-kquant README, "Codec
// reference"; gguf-py constants (q4_K 144 B, q5_K 176 B, q6_K 210 B, q8_0
// 34 B, q4_0 18 B).
//
// Streaming.  One CTA per SM owns a balanced contiguous range of rows.  A
// producer warp streams 16-row stages (whole rows when they fit, else equal
// row slices) into a ring of shared-memory slots with one 1-D bulk copy per
// row; big contiguous copies are what keeps HBM busy.  Before the first
// stage it copies the activation rows, so they land first.  16 consumer
// warps build the activation image, then split every stage into work items
// and release the slot through an mbarrier; the producer never waits for
// anything else.
//
// Arithmetic is the exact-integer tensor-core scheme: a lane turns its codes
// into binary16 integers, the activations rounded once to binary16 are the B
// operand of m16n8k16 MMAs, and the tensor core accumulates exact products in
// fp32; per-block scales are applied in fp32 once a block is complete.
// Before that rounding each run of activations (a block, or a 16-value run of
// q6_K) is scaled by a power of two that puts its largest magnitude at 2^T
// (T per codec), and the inverse scale is applied to its fp32 sums, so the
// relative precision does not depend on the activations' magnitude.  Codes
// enter the MMA as binary16 subnormals (the code's bits in the mantissa,
// exponent field 0: code x 2^-24, exact; the tensor core keeps subnormal
// operands exact), centred on the codec's offset before the MMA (q8_0: 128
// of the unsigned view of the int8 code, q4_0: 8, q6_K: 32) by one exact
// sub.f16x2, so a zero weight contributes exactly zero however large its
// activation; the 2^24 goes into the per-block scale.  q4_K / q5_K at m >= 2
// multiply their codes by the 6-bit scale exactly in binary16 instead (1024 +
// code, scaled and the 1024 removed by one HFMA2).  The activation operand of
// every MMA is precomputed per CTA into a shared-memory image in fragment
// order (one 8-byte load per MMA); B lanes whose column does not receive a
// given word read a zero block instead of being masked.  The lane-to-byte
// mappings:
//
//  * q8_0, item = 16 rows x 8 blocks: lane t owns blocks 2t and 2t+1 (68
//    bytes, word aligned) and feeds one 32-bit word per MMA.  Words 0..8 hold
//    codes of the even block only (its fp16 scale bytes and the odd block's
//    get a zero activation), words 9..16 those of the odd block, so MMA
//    column 2t + parity collects exactly lane t's block of that parity.
//  * q4_0, item = 16 rows x 8 blocks: as q8_0 with 36-byte spans and two MMAs
//    per word (low nibbles against x, high nibbles in place against x/16).
//  * q6_K, item = 16 rows x 1 block: lane t owns a quarter (half h, 16-value
//    run lh) of the block for all four q; nibble and 2-bit field are merged
//    into the 6-bit code with two LOP3s; columns 2t, 2t+1 hold its low- and
//    high-nibble sub-blocks of the current pass.  The four lanes of a row read
//    their words in a rotated order, which keeps the loads free of bank
//    conflicts.
//  * q4_K / q5_K, item = 16 rows x 1 block: lane t owns values 64t..64t+63.
//    At m >= 2 one column per token, the scale in the operand (q sc <= 945,
//    <= 1953 with q5_K's fifth bit) and the min term as one more MMA on
//    (m_j) x (X_j split into two binary16 halves).  At m = 1 (Q4C) the
//    columns separate lane t's two sub-blocks instead, and scale and min are
//    applied in the fp32 epilogue.
//
// Partial sums of the 16 warps are combined in a fixed order by the last
// warp to finish a row group: results are bitwise reproducible.
#include <algorithm>
#include <type_traits>

#include "kq_device.cuh"
#include "kq_launch.h"

namespace kq {
namespace {

constexpr int kCW = 16;                  // consumer warps
static_assert((kCW & (kCW - 1)) == 0, "warp round robin uses a power-of-two mask");
constexpr int kProd = kCW;               // producer warp
constexpr int kThreads = 32 * (kCW + 1);
constexpr int kRows = 16;
constexpr int kMaxStages = 6;
constexpr int kMaxGroups = 64;           // row groups per CTA (counters)
constexpr uint32_t kHdr = 1024;          // barriers and counters

struct SP {
    const uint8_t* w;
    const uint16_t* x;
    float* y;
    int* status;
    int64_t n, k, row_bytes;   // k: values of K this CTA covers (its slice)
    int m, nblk, g, spr, ns;   // nblk: blocks of the slice
    // x_global 1: build the image from x in global memory (no room for a raw
    // copy); ks: CTAs of a cluster splitting K (q4_K; 1: no split; the token
    // stride of x is then ks k); strict 1: the wait limit is shorter than the
    // default, the activation wait tests its phase (see spin_wait).  Packed:
    // a larger parameter block was measured to slow the kernel down.
    uint32_t x_global : 8, ks : 8, strict : 1;
    uint32_t rs;   // shared-memory stride of a stage row
    uint32_t off_stage, off_img, img_tok, off_xs, xs_tok, off_zero, off_part, off_xraw;
    uint32_t off_red;   // split: receive slots of the cluster reduction
};
static_assert(sizeof(SP) == 120, "kernel parameter block size");

// Gather mode (decode MoE, one output row per (token, slot) pair): the pairs
// of an expert-id list are grouped by expert into "virtual experts" of at most
// m pairs (ascending expert id, pairs in (token, slot) order, an expert with
// more than m pairs takes several); the CTAs of a launch are spread evenly
// over virtual experts [vbase, vbase + vcount), each CTA covering a
// contiguous range of its expert's rows.  x row of pair q: q / xdiv; y row:
// q.  A separate parameter type, so that the dense kernels keep their block.
struct SPG : SP {
    const int32_t* ids;   // [pairs] expert id of every (token, slot) pair
    int32_t* err;         // caller's device flag word (nullable)
    int pairs, xdiv, n_experts, vbase, vcount;
};
// GLU mode (decode MoE gate/up pair, one activation row per token): the
// gate bank is w, the up bank w2; logical row group 2g + h of a CTA is its
// row group g of the gate (h = 0) or up (h = 1) matrix.  The gate sums wait
// in a small buffer for the up sums of the same rows, and act(gate) * up is
// stored.
struct SPGLU : SPG {
    const uint8_t* w2;
    int act;       // 0: silu, 1: gelu (tanh form), 2: silu with limit
    float limit;
};
constexpr uint32_t kGList = 512;     // gather: pair list of the CTA (16 ints)
constexpr uint32_t kGMisc = 576;     // gather: expert, pairs present, row range
constexpr uint32_t kGCount = 1024;   // gather: pairs per expert (256 ints)
constexpr uint32_t kGHdr = 2048;     // gather header size

// Row groups are walked with a partial last group (fewer than 16 rows) moved
// to the front: its small stage lands first and its decode overlaps the full
// stages still in flight instead of trailing the kernel.
__device__ __forceinline__ int group_order(int rg, int nrg, int64_t rows) {
    if (nrg < 2 || rows % kRows == 0) return rg;
    return rg == 0 ? nrg - 1 : rg - 1;
}

constexpr uint32_t kH1024 = 0x64006400u;    // binary16 (1024, 1024)
constexpr uint32_t kHm1024 = 0xE400E400u;   // (-1024, -1024)
constexpr uint32_t kH1_16 = 0x2C002C00u;    // (1/16, 1/16)
constexpr float kTwo24 = 16777216.0f;        // 2^24: a subnormal code's unit is 2^-24

// Volatile so that the conversions stay next to the MMA that consumes them.
__device__ __forceinline__ uint32_t vand_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm volatile("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t vand_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm volatile("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// a - b per binary16 half.  On codes held as subnormals (integer multiples
// of 2^-24 below 2^-14 in magnitude) the difference is exact: it centres a
// code on the format's offset before the MMA, so that a large activation
// meets a zero weight as an exact zero.
__device__ __forceinline__ uint32_t vhsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm volatile("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vhfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm volatile("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y));
}
__device__ __forceinline__ void sts16(uint32_t a, __half x) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(__half_as_ushort(x)));
}
__device__ __forceinline__ void sts8(uint32_t a, uint32_t x) {
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(a), "r"(x));
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t x) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(x));
}
__device__ __forceinline__ int lds_s8(uint32_t a) {
    int16_t v;
    asm volatile("ld.shared.s8 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float h2f(uint32_t h) { return __half2float(__ushort_as_half(static_cast<unsigned short>(h))); }

// Time limit of the pipeline waits of this kernel, per device (default
// kWaitLimitNs; kq_set_wait_limit shortens it for fault-handling tests).  Read
// only once a wait has not completed at its first poll.
__device__ uint64_t g_wait_ns = kWaitLimitNs;
// Host copy, per device, of whether g_wait_ns is shorter than the default.
bool g_strict_wait[64];
__device__ __forceinline__ uint64_t wait_limit() { return *static_cast<volatile uint64_t*>(&g_wait_ns); }

// Bounded spin on an mbarrier phase (no suspend hint: these waits are short
// and a sleeping warp can wake up late).  False after the time limit, with
// KQ_DEV_TIMEOUT recorded.  Under a limit shorter than the default (a
// test's) the time is taken at every poll and a completion seen after the
// limit counts as run out.  `test_first` (the activation wait, once per CTA,
// with a short limit): the phase is only tested, never waited on, so that
// wait runs out unless the copy has already landed.  The per-stage waits
// keep the plain form: a blocking first poll and no extra work.
__device__ __forceinline__ bool spin_wait(uint64_t* bar, uint32_t parity, int* status, bool test_first = false) {
    if (test_first ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns(), limit = wait_limit();
    const bool strict = limit < kWaitLimitNs;
    for (int i = 0;; ++i) {
        const bool done = test_first ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity);
        if (done && !strict) return true;
        if (strict || (i & 255) == 255) {
            if (global_ns() - t0 > limit) {
                if (status) atomicOr(status, KQ_DEV_TIMEOUT);
                return false;
            }
            if (done) return true;
        }
    }
}

// Bounded wait that lets the warp sleep until the phase completes (the
// producer: it must not take issue slots from the decoding warps).  `limit`
// is the time limit (the pipeline's, or kWaitLimitNs for the wind-down); a
// shorter limit than the default makes the wait strict, as in spin_wait.
__device__ __forceinline__ bool sleep_wait(uint64_t* bar, uint32_t parity, int* status, uint64_t limit) {
    const bool strict = limit < kWaitLimitNs;
    if (strict ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        const bool done = strict ? mbar_test_wait(bar, parity) : mbar_try_wait_sleep(bar, parity);
        if (done && !strict) return true;
        if (global_ns() - t0 > limit) {
            if (status) atomicOr(status, KQ_DEV_TIMEOUT);
            return false;
        }
        if (done) return true;
    }
}

// Raw bf16 activations, copied into shared memory before the image is built.
__device__ __forceinline__ uint32_t xaddr(const SP& p, uint32_t sb, int tok, int64_t i) {
    return sb + p.off_xraw + 2u * static_cast<uint32_t>(tok * p.k + i);
}
__device__ __forceinline__ float xval(const SP& p, uint32_t sb, int tok, int64_t i) {
    return __uint_as_float(lds_u16(xaddr(p, sb, tok, i)) << 16);
}
// Binary16 of an activation times its power-of-two scale.
__device__ __forceinline__ __half hx(float v, float scale) { return __float2half_rn(v * scale); }
__device__ __forceinline__ uint32_t hpair(__half lo, __half hi) {
    return static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}


// Lane roles in the m16n8k16 fragments (lane = 4 g + t): A rows g and g+8,
// k-slots 2t, 2t+1, 2t+8, 2t+9; B column g; D columns 2t, 2t+1.
struct Lane {
    int g, t;
};

// ===========================================================================
// q8_0
// ===========================================================================
template <int NT>
struct Q8 {
    static constexpr int kVPB = 32, kBPB = 34;
    static constexpr int kItemBlocks = 8;
    static constexpr uint32_t kItemImg = 17 * 32;   // image bytes per item (8 blocks) and token
    static constexpr uint32_t kZero = kItemImg;
    static constexpr int kAccPerLane = 2 * NT;
    // a block's scaled activations stay below 2^15: far inside binary16
    static constexpr int kXT = 14;
    static constexpr bool kSplit = false;

    // rowA/rowB: shared address of the item (8 blocks) in rows g / g+8;
    // gi: global item index (block 8 gi).
    static __device__ __forceinline__ void item(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                uint32_t rowB, int gi, float (&acc)[2 * NT]) {
        const int t = L.t;
        const bool act = (L.g >> 1) == t;   // B lanes whose column holds lane t's blocks
        uint32_t bb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t img = sb + p.off_img + nt * p.img_tok + gi * kItemImg + 8 * t;
            const uint32_t zero = sb + p.off_zero + 8 * t;
            bb[nt][0] = (act && (L.g & 1) == 0) ? img : zero;
            bb[nt][1] = (act && (L.g & 1) == 1) ? img : zero;
        }
        float D[NT][2][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) D[nt][c][e] = 0.f;
        const uint32_t a0 = rowA + 68 * t, b0 = rowB + 68 * t;
        float dE[2], dO[2];
#pragma unroll
        for (int mu = 0; mu < 17; ++mu) {
            const uint32_t wa = lds32(a0 + 4 * mu), wb = lds32(b0 + 4 * mu);
            if (mu == 0) {   // fp16 d of the even block: bytes 0..1 of the span
                dE[0] = h2f(wa & 0xffff) * kTwo24;
                dE[1] = h2f(wb & 0xffff) * kTwo24;
            }
            if (mu == 8) {   // the odd block's d: bytes 34..35
                dO[0] = h2f(wa >> 16) * kTwo24;
                dO[1] = h2f(wb >> 16) * kTwo24;
            }
            const int par = mu >= 9 ? 1 : 0;
            // byte ^ 0x80 = 128 + code as a binary16 subnormal, less 128 2^-24:
            // the signed code as the subnormal code 2^-24
            const uint32_t A0 = vhsub2(vand_xor(wa, 0x00FF00FFu, 0x00800080u), 0x00800080u);
            const uint32_t A1 = vhsub2(vand_xor(wb, 0x00FF00FFu, 0x00800080u), 0x00800080u);
            const uint32_t A2 = vhsub2(vand_xor(wa >> 8, 0x00FF00FFu, 0x00800080u), 0x00800080u);
            const uint32_t A3 = vhsub2(vand_xor(wb >> 8, 0x00FF00FFu, 0x00800080u), 0x00800080u);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 bv = lds64(bb[nt][par] + 32 * mu);
                mma_f16(D[nt][mu & 1], A0, A1, A2, A3, bv.x, bv.y);
            }
        }
        // D = 2^-24 sum code a with a = x 2^s (s per token and block):
        // y += 2^(24-s) d D for columns 2t (even block) and 2t+1 (odd block)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 xv = lds64(sb + p.off_xs + nt * p.xs_tok + 8 * (4 * gi + t));
            const float iv[2] = {__uint_as_float(xv.x), __uint_as_float(xv.y)};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e >> 1, odd = e & 1;
                const float Ds = D[nt][0][e] + D[nt][1][e];
                acc[2 * nt + r] = fmaf((odd ? dO[r] : dE[r]) * iv[odd], Ds, acc[2 * nt + r]);
            }
        }
    }

    // Partial sums of this warp for a row group -> part[row][tok].
    static __device__ __forceinline__ void store_part(const SP& p, const Lane& L, float (&acc)[2 * NT], float* part) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float v = acc[2 * nt + r];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                if (L.t == 0) part[(L.g + 8 * r) * p.m + nt] = v;
            }
    }

    // Image entry (item, mu, t') = binary16 of the scaled activations of the
    // 4 raw bytes at offset 272 item + 68 t' + 4 mu of a row, as (byte0,
    // byte2 | byte1, byte3); scale bytes get 0.  Eight neighbouring lanes
    // share the span of lane t' (blocks b0 = 8 item + 2 t' and b0 + 1), each
    // with 8 values of one block: they agree on the block's scale 2^s (its
    // largest |x| at 2^14) by two shuffles, and lane 0 of the block stores
    // 2^-s (4 bytes per block, in block order).  Every warp runs the same
    // number of rounds, so the shuffles always see the whole warp.  Returns
    // whether this thread met a non-finite activation.
    static __device__ bool build(const SP& p, uint32_t sb, int64_t xoff) {
        bool bad = false;
        const int spans = p.nblk / 2, total = p.m * spans * 8;
        for (int w0 = threadIdx.x & ~31; w0 < total; w0 += kCW * 32) {
            const int e = w0 + (threadIdx.x & 31);
            const bool in = e < total;
            const int sp = e >> 3, tok = sp / spans, s2 = sp - tok * spans;   // s2 = 4 item + t'
            const int it = s2 >> 2, tt = s2 & 3, odd = (e >> 2) & 1, qq = e & 3;
            const int blk = 2 * s2 + odd;
            const uint4 v = in ? lds128(xaddr(p, sb, tok, 32 * blk + 8 * qq)) : make_uint4(0u, 0u, 0u, 0u);
            uint32_t mx = absmax8_bf16(0u, v);
            mx = max(mx & 0xFFFFu, mx >> 16);
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            bad |= in && mx >= 0x7F80u;
            const int se = xscale_exp(mx, kXT);
            const float S = exp2_int(se);
            if (!in) continue;   // lanes out of range occur in the last round only
            if (qq == 0) sts32(sb + p.off_xs + tok * p.xs_tok + 4 * blk, __float_as_uint(exp2_int(-se)));
            // value 8 qq + i of the block is byte j = 8 qq + i + 2 (+ 34) of the span
            const uint32_t ent = sb + p.off_img + tok * p.img_tok + it * kItemImg + tt * 8;
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float f = (i & 1) ? bf16hi_to_f32(wv[i >> 1]) : bf16lo_to_f32(wv[i >> 1]);
                const int j = 8 * qq + i + 2 + 34 * odd, b = j & 3;
                sts16(ent + (j >> 2) * 32 + 4 * (b & 1) + 2 * (b >> 1), hx(f, S));
            }
            if (qq == 0) {   // the block's scale bytes: span bytes 0, 1 (even) or 34, 35 (odd)
                const int j0 = 34 * odd, b = j0 & 3;
                sts16(ent + (j0 >> 2) * 32 + 4 * (b & 1) + 2 * (b >> 1), __float2half_rn(0.f));
                sts16(ent + ((j0 + 1) >> 2) * 32 + 4 * ((b + 1) & 1) + 2 * ((b + 1) >> 1), __float2half_rn(0.f));
            }
        }
        return bad;
    }
};

// ===========================================================================
// q4_0
// ===========================================================================
// q4_0 (18 bytes per 32 values): fp16 d, then 16 bytes whose low nibbles are
// values 0..15 and high nibbles values 16..31; y = d (code - 8).  Item = 16
// rows x 8 blocks (144 bytes of a row).  Lane t owns blocks 2t and 2t+1 (36
// bytes, word aligned) and feeds two MMAs per word: the low nibbles as
// binary16 subnormals less 8 2^-24 ((code - 8) 2^-24, exact) against x, the
// high nibbles in place less 128 2^-24 (16 (code - 8) 2^-24) against x/16.
// Words 0..4 hold the even block (its d in bytes 0..1, the odd block's d in
// bytes 18..19: zero activations), words 5..8 the odd block, so MMA column
// 2t + parity collects exactly lane t's block of that parity.
template <int NT>
struct Q40 {
    static constexpr int kVPB = 32, kBPB = 18;
    static constexpr int kItemBlocks = 8;
    static constexpr uint32_t kItemImg = 18 * 32;   // 9 words x (low, high) per item and token
    static constexpr uint32_t kZero = kItemImg;
    static constexpr int kAccPerLane = 2 * NT;
    static constexpr int kXT = 14;
    static constexpr bool kSplit = false;

    static __device__ __forceinline__ void item(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                uint32_t rowB, int gi, float (&acc)[2 * NT]) {
        const int t = L.t;
        const bool act = (L.g >> 1) == t;
        uint32_t bb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t img = sb + p.off_img + nt * p.img_tok + gi * kItemImg + 8 * t;
            const uint32_t zero = sb + p.off_zero + 8 * t;
            bb[nt][0] = (act && (L.g & 1) == 0) ? img : zero;
            bb[nt][1] = (act && (L.g & 1) == 1) ? img : zero;
        }
        float D[NT][2][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) D[nt][c][e] = 0.f;
        const uint32_t a0 = rowA + 36 * t, b0 = rowB + 36 * t;
        float dE[2], dO[2];
#pragma unroll
        for (int mu = 0; mu < 9; ++mu) {
            const uint32_t wa = lds32(a0 + 4 * mu), wb = lds32(b0 + 4 * mu);
            if (mu == 0) {   // the even block's d: bytes 0..1 of the span
                dE[0] = h2f(wa & 0xffff) * kTwo24;
                dE[1] = h2f(wb & 0xffff) * kTwo24;
            }
            if (mu == 4) {   // the odd block's d: bytes 18..19
                dO[0] = h2f(wa >> 16) * kTwo24;
                dO[1] = h2f(wb >> 16) * kTwo24;
            }
            const int par = mu >= 5 ? 1 : 0;
            const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
            // low nibbles as subnormals (c - 8) 2^-24, high nibbles in place:
            // 16 (c - 8) 2^-24
            const uint32_t L0 = vhsub2(vand_or(wa, 0x000F000Fu, 0u), 0x00080008u);
            const uint32_t L1 = vhsub2(vand_or(wb, 0x000F000Fu, 0u), 0x00080008u);
            const uint32_t L2 = vhsub2(vand_or(wa8, 0x000F000Fu, 0u), 0x00080008u);
            const uint32_t L3 = vhsub2(vand_or(wb8, 0x000F000Fu, 0u), 0x00080008u);
            const uint32_t H0 = vhsub2(vand_or(wa, 0x00F000F0u, 0u), 0x00800080u);
            const uint32_t H1 = vhsub2(vand_or(wb, 0x00F000F0u, 0u), 0x00800080u);
            const uint32_t H2 = vhsub2(vand_or(wa8, 0x00F000F0u, 0u), 0x00800080u);
            const uint32_t H3 = vhsub2(vand_or(wb8, 0x00F000F0u, 0u), 0x00800080u);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 bl = lds64(bb[nt][par] + 64 * mu), bh = lds64(bb[nt][par] + 64 * mu + 32);
                mma_f16(D[nt][mu & 1], L0, L1, L2, L3, bl.x, bl.y);
                mma_f16(D[nt][mu & 1], H0, H1, H2, H3, bh.x, bh.y);
            }
        }
        // D = 2^-24 sum (c - 8) a (a = x 2^s, the high half against
        // x 2^s / 16): y += 2^(24-s) d D
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 xv = lds64(sb + p.off_xs + nt * p.xs_tok + 8 * (4 * gi + t));
            const float iv[2] = {__uint_as_float(xv.x), __uint_as_float(xv.y)};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e >> 1, odd = e & 1;
                const float Ds = D[nt][0][e] + D[nt][1][e];
                acc[2 * nt + r] = fmaf((odd ? dO[r] : dE[r]) * iv[odd], Ds, acc[2 * nt + r]);
            }
        }
    }

    static __device__ __forceinline__ void store_part(const SP& p, const Lane& L, float (&acc)[2 * NT], float* part) {
        Q8<NT>::store_part(p, L, acc, part);
    }

    // Image entries (item, mu, low / high, t') = binary16 of the scaled
    // activations of the 4 raw bytes at offset 144 item + 36 t' + 4 mu of a
    // row, as (byte0, byte2 | byte1, byte3): the low nibble's value (x 2^s)
    // or the high nibble's (x 2^s / 16); d bytes get 0.  Eight neighbouring
    // lanes share the span of lane t' (blocks b0 = 8 item + 2 t' and
    // b0 + 1), each with 4 code bytes of one block (low values 4 qq + c, high
    // values 16 + 4 qq + c): they agree on the block's scale 2^s by two
    // shuffles, and lane 0 of the block stores 2^-s (4 bytes per block, in
    // block order).  Returns whether this thread met a non-finite activation.
    static __device__ bool build(const SP& p, uint32_t sb, int64_t xoff) {
        bool bad = false;
        const int spans = p.nblk / 2, total = p.m * spans * 8;
        for (int w0 = threadIdx.x & ~31; w0 < total; w0 += kCW * 32) {
            const int e = w0 + (threadIdx.x & 31);
            const bool in = e < total;
            const int sp = e >> 3, tok = sp / spans, s2 = sp - tok * spans;   // s2 = 4 item + t'
            const int it = s2 >> 2, tt = s2 & 3, odd = (e >> 2) & 1, qq = e & 3;
            const int blk = 2 * s2 + odd;
            uint2 lo = make_uint2(0u, 0u), hi = make_uint2(0u, 0u);
            if (in) {
                lo = lds64(xaddr(p, sb, tok, 32 * blk + 4 * qq));
                hi = lds64(xaddr(p, sb, tok, 32 * blk + 16 + 4 * qq));
            }
            uint32_t mx = absmax8_bf16(0u, make_uint4(lo.x, lo.y, hi.x, hi.y));
            mx = max(mx & 0xFFFFu, mx >> 16);
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            bad |= in && mx >= 0x7F80u;
            const int se = xscale_exp(mx, kXT);
            const float S = exp2_int(se), S16 = S * 0.0625f;
            if (!in) continue;   // lanes out of range occur in the last round only
            if (qq == 0) sts32(sb + p.off_xs + tok * p.xs_tok + 4 * blk, __float_as_uint(exp2_int(-se)));
            // code byte 4 qq + c of the block is byte j = 4 qq + c + 2 (+ 18) of the span
            const uint32_t ent = sb + p.off_img + tok * p.img_tok + it * kItemImg + tt * 8;
            const uint32_t lw[2] = {lo.x, lo.y}, hw[2] = {hi.x, hi.y};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int j = 4 * qq + c + 2 + 18 * odd, b = j & 3;
                const uint32_t a = ent + (j >> 2) * 64 + 4 * (b & 1) + 2 * (b >> 1);
                const float fl = (c & 1) ? bf16hi_to_f32(lw[c >> 1]) : bf16lo_to_f32(lw[c >> 1]);
                const float fh = (c & 1) ? bf16hi_to_f32(hw[c >> 1]) : bf16lo_to_f32(hw[c >> 1]);
                sts16(a, hx(fl, S));
                sts16(a + 32, hx(fh, S16));
            }
            if (qq == 0) {   // the block's d bytes: span bytes 0, 1 (even) or 18, 19 (odd)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int j = 18 * odd + c, b = j & 3;
                    const uint32_t a = ent + (j >> 2) * 64 + 4 * (b & 1) + 2 * (b >> 1);
                    sts16(a, __float2half_rn(0.f));
                    sts16(a + 32, __float2half_rn(0.f));
                }
            }
        }
        return bad;
    }
};

// ===========================================================================
// q6_K
// ===========================================================================
// (a & m) | (b & ~m) in one LOP3.
__device__ __forceinline__ uint32_t vbitsel(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm volatile("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

template <int NT>
struct Q6 {
    static constexpr int kVPB = 256, kBPB = 210;
    static constexpr int kItemBlocks = 1;
    static constexpr uint32_t kBlkImg = 512;   // image bytes per block and token
    static constexpr uint32_t kZero = 512;
    static constexpr int kAccPerLane = 2 * NT;
    // a run's scaled activations below 2^15: its x/16 and x/256 operands stay
    // normal binary16 numbers down to 2^-22 of the run's largest magnitude
    static constexpr int kXT = 14;
    static constexpr bool kSplit = false;

    // Word at shared address a: 4-byte aligned (MODE 0), 2 bytes past a
    // 4-byte boundary (MODE 1), or either, per thread (MODE 2: rows at their
    // own offsets, when a row is not a 16-byte multiple).
    template <int MODE>
    static __device__ __forceinline__ uint32_t word(uint32_t a) {
        if constexpr (MODE == 1) return __byte_perm(lds32(a - 2), lds32(a + 2), 0x5432);
        else if constexpr (MODE == 2) {
            const uint32_t al = a & ~3u;
            return __byte_perm(lds32(al), lds32(al + 4), (a & 2u) ? 0x5432u : 0x3210u);
        } else return lds32(a);
    }

    // One block of 16 rows.  Lane t owns quarter (h = t >> 1, lh = t & 1):
    // values v = 128h + 32q + l, l in [16 lh, 16 lh + 16), all four q, i.e.
    // sub-blocks j = 8h + 2q + lh.  Its 6-bit codes come from nibble q >> 1 of
    // ql[64h + 32 (q & 1) + l] and bits 2q of qh[32h + l].  For each pass
    // qp = q & 1 and word k the lane feeds two MMAs: the low nibbles (q = qp,
    // c6 - 32 as a subnormal, activations x/16) into column 2t and the high
    // nibbles (q = qp + 2, 16 (c6 - 32), x/256) into column 2t + 1.  The four lanes of
    // a row read their words in the order (k + t) mod 4, which spreads them over
    // all 32 banks; the activation image follows the same order.
    template <int ODD>
    static __device__ __forceinline__ void block(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                 uint32_t rowB, int gb, float (&acc)[2 * NT]) {
        const int t = L.t, h = t >> 1, lh = t & 1;
        const bool act = (L.g >> 1) == t;   // B lanes whose columns hold lane t's sub-blocks
        uint32_t bb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t img = sb + p.off_img + nt * p.img_tok + gb * kBlkImg + 8 * t;
            const uint32_t zero = sb + p.off_zero + 8 * t;
            bb[nt][0] = (act && (L.g & 1) == 0) ? img : zero;
            bb[nt][1] = (act && (L.g & 1) == 1) ? img : zero;
        }
        // scales of the lane's sub-blocks: sc[8h + 2q + lh], and 16 d
        float sc[2][4], d16[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t row = r ? rowB : rowA;
#pragma unroll
            for (int q = 0; q < 4; ++q) sc[r][q] = static_cast<float>(lds_s8(row + 192 + 8 * h + lh + 2 * q));
            d16[r] = 268435456.0f * h2f(lds_u16(row + 208));   // 2^28 d = 16 d 2^24
        }
        // the lane's 4 qh words (rows g, g+8), in its rotated order
        const uint32_t rot[4] = {4u * ((0 + t) & 3), 4u * ((1 + t) & 3), 4u * ((2 + t) & 3), 4u * ((3 + t) & 3)};
        uint32_t ha[4], hb[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            ha[k] = word<ODD>(rowA + 128 + 32 * h + 16 * lh + rot[k]);
            hb[k] = word<ODD>(rowB + 128 + 32 * h + 16 * lh + rot[k]);
        }
#pragma unroll
        for (int qp = 0; qp < 2; ++qp) {
            float D[2][NT][4];   // two chains (k parity)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) D[c][nt][e] = 0.f;
            // field qp (and qp + 2) of each qh byte moved next to its nibble:
            // bits 4-5 (low nibble) / 8-9 (high nibble); bytes 1 and 3 also >> 8
            constexpr int kSh[2] = {4, 2};
            const int sh = kSh[qp];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t wa = word<ODD>(rowA + 64 * h + 32 * qp + 16 * lh + rot[k]);
                const uint32_t wb = word<ODD>(rowB + 64 * h + 32 * qp + 16 * lh + rot[k]);
                const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
                const uint32_t sa02 = ha[k] << sh, sa13 = ha[k] >> (8 - sh);
                const uint32_t sb02 = hb[k] << sh, sb13 = hb[k] >> (8 - sh);
                // low nibble + field qp -> c6 as a subnormal (c6 2^-24), less
                // 32 2^-24: the centred code, exact
                const uint32_t L0 = vhsub2(vbitsel(wa, vand_or(sa02, 0x00300030u, 0u), 0x000F000Fu), 0x00200020u);
                const uint32_t L1 = vhsub2(vbitsel(wb, vand_or(sb02, 0x00300030u, 0u), 0x000F000Fu), 0x00200020u);
                const uint32_t L2 = vhsub2(vbitsel(wa8, vand_or(sa13, 0x00300030u, 0u), 0x000F000Fu), 0x00200020u);
                const uint32_t L3 = vhsub2(vbitsel(wb8, vand_or(sb13, 0x00300030u, 0u), 0x000F000Fu), 0x00200020u);
                // high nibble + field qp + 2 -> 16 c6 as a subnormal, less 512 2^-24
                const uint32_t H0 = vhsub2(vbitsel(wa, vand_or(sa02, 0x03000300u, 0u), 0x00F000F0u), 0x02000200u);
                const uint32_t H1 = vhsub2(vbitsel(wb, vand_or(sb02, 0x03000300u, 0u), 0x00F000F0u), 0x02000200u);
                const uint32_t H2 = vhsub2(vbitsel(wa8, vand_or(sa13, 0x03000300u, 0u), 0x00F000F0u), 0x02000200u);
                const uint32_t H3 = vhsub2(vbitsel(wb8, vand_or(sb13, 0x03000300u, 0u), 0x00F000F0u), 0x02000200u);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint2 bl = lds64(bb[nt][0] + 32 * (8 * qp + k));
                    const uint2 bh = lds64(bb[nt][1] + 32 * (8 * qp + 4 + k));
                    mma_f16(D[k & 1][nt], L0, L1, L2, L3, bl.x, bl.y);
                    mma_f16(D[k & 1][nt], H0, H1, H2, H3, bh.x, bh.y);
                }
            }
            // column 2t: D = 2^-24 sum (c - 32) a with a = x 2^s/16, column
            // 2t + 1: D = 2^-24 sum 16 (c - 32) a with a = x 2^s/256 (s per
            // 16-value run); both are 2^-24 2^s sum (c - 32) x / 16:
            // y += 2^28 d sc_j 2^-s D
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 xv = lds64(sb + p.off_xs + nt * p.xs_tok + ((gb * 4 + t) * 2 + qp) * 8);
                const float iv[2] = {__uint_as_float(xv.x), __uint_as_float(xv.y)};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = e >> 1, c = e & 1;
                    const float Ds = D[0][nt][e] + D[1][nt][e];
                    acc[2 * nt + r] = fmaf(__fmul_rn(d16[r], sc[r][qp + 2 * c]) * iv[c], Ds, acc[2 * nt + r]);
                }
            }
        }
    }

    static __device__ __forceinline__ void item(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                uint32_t rowB, int gb, float (&acc)[2 * NT]) {
        if (gb & 1) block<1>(p, sb, L, rowA, rowB, gb, acc);
        else block<0>(p, sb, L, rowA, rowB, gb, acc);
    }
    // rows A and B at their own byte offsets (rows not a 16-byte multiple)
    static __device__ __forceinline__ void item_rt(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                   uint32_t rowB, int gb, float (&acc)[2 * NT]) {
        block<2>(p, sb, L, rowA, rowB, gb, acc);
    }

    static __device__ __forceinline__ void store_part(const SP& p, const Lane& L, float (&acc)[2 * NT], float* part) {
        Q8<NT>::store_part(p, L, acc, part);
    }

    // One thread per 16-value run (token, block, quarter t' = (h, lh), qp,
    // s): q = qp + 2s, values v = 128h + 32q + 16 lh + l, l = 0..15.  Its
    // scale 2^e puts the run's largest |x| at 2^14; image entry (block,
    // E = 8 qp + 4 s + k, t') = binary16 of x[v] 2^e / 16 (s = 0) or / 256
    // (s = 1) for l = 4 ((k + t') mod 4) + {0, 2 | 1, 3}; the runs'
    // {2^-e_s=0, 2^-e_s=1} per (block, t', qp).  Returns whether this thread
    // met a non-finite activation.
    static __device__ bool build(const SP& p, uint32_t sb, int64_t xoff) {
        bool bad = false;
        const int per_tok = p.nblk * 16;
        for (int e = threadIdx.x; e < p.m * per_tok; e += kCW * 32) {
            const int tok = e / per_tok, rem = e % per_tok;
            const int blk = rem >> 4, tt = (rem >> 2) & 3, qp = (rem >> 1) & 1, sl = rem & 1;
            const int h = tt >> 1, lh = tt & 1, q = qp + 2 * sl;
            const uint32_t xs = xaddr(p, sb, tok, blk * 256 + 128 * h + 32 * q + 16 * lh);
            const uint4 v0 = lds128(xs), v1 = lds128(xs + 16);
            uint32_t mx = absmax8_bf16(0u, v0);
            mx = absmax8_bf16(mx, v1);
            mx = max(mx & 0xFFFFu, mx >> 16);
            bad |= mx >= 0x7F80u;
            const int se = xscale_exp(mx, kXT);
            const float sc = exp2_int(se) * (sl ? 0.00390625f : 0.0625f);
            const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const uint32_t img = sb + p.off_img + tok * p.img_tok + blk * kBlkImg + (8 * qp + 4 * sl) * 32 + tt * 8;
            // values 4g .. 4g+3 (words 2g, 2g+1) go to entry k = (g - t') mod 4
            // as binary16 pairs (4g, 4g+2 | 4g+1, 4g+3)
#pragma unroll
            for (int g = 0; g < 4; ++g)
                sts64(img + ((g - tt) & 3) * 32,
                      pack_f16x2(bf16lo_to_f32(wv[2 * g]) * sc, bf16lo_to_f32(wv[2 * g + 1]) * sc),
                      pack_f16x2(bf16hi_to_f32(wv[2 * g]) * sc, bf16hi_to_f32(wv[2 * g + 1]) * sc));
            sts32(sb + p.off_xs + tok * p.xs_tok + ((blk * 4 + tt) * 2 + qp) * 8 + 4 * sl,
                  __float_as_uint(exp2_int(-se)));
        }
        return bad;
    }
};

// ===========================================================================
// q4_K (and q5_K: FIVE)
// ===========================================================================
// q5_K (176 B) has q4_K's header (d, dmin, packed 6-bit scales and mins), then
// qh[32], then the 4-bit codes at byte 48: value 64c + l takes bit 2c of
// qh[l] as its fifth bit, value 64c + 32 + l bit 2c + 1; q = 0..31.  The
// image, the scales and the min term are q4_K's; only the code assembly
// differs: 1024 + q (low) and 1024 + 16 q (high) still hold q sc exactly
// after the scale FMA (q sc <= 1953 < 2048).
template <int NT, bool FIVE = false>
struct Q4 {
    static constexpr int kVPB = 256, kBPB = FIVE ? 176 : 144;
    static constexpr bool kSplit = true;   // the K-split (cluster) kernel serves it
    static constexpr int kItemBlocks = 1;
    static constexpr uint32_t kBlkImg = 544;
    static constexpr uint32_t kZero = kBlkImg;
    static constexpr int kAccPerLane = 4 * NT;
    // a block's scaled activations below 2^10: a sub-block sum X_j (32
    // values) stays below 2^15, inside the binary16 range of its two-part split
    static constexpr int kXT = 9;

    static __device__ __forceinline__ void item(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                uint32_t rowB, int gb, float (&acc)[4 * NT]) {
        const int t = L.t;
        uint32_t bb[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tok = 8 * nt + L.g;
            bb[nt] = tok < p.m ? sb + p.off_img + tok * p.img_tok + gb * kBlkImg + 8 * t : sb + p.off_zero + 8 * t;
        }
        const uint4 hA = lds128(rowA), hB = lds128(rowB);
        constexpr uint32_t kQs = FIVE ? 48 : 16;   // first code byte
        const uint4 qA0 = lds128(rowA + kQs + 32 * t), qA1 = lds128(rowA + kQs + 16 + 32 * t);
        const uint4 qB0 = lds128(rowB + kQs + 32 * t), qB1 = lds128(rowB + kQs + 16 + 32 * t);
        uint32_t fA[8], fB[8];   // q5_K: qh[4u .. 4u+3] >> 2t (the lane's two bits at bits 0, 1 of each byte)
        if constexpr (FIVE) {
            const uint4 hA0 = lds128(rowA + 16), hA1 = lds128(rowA + 32);
            const uint4 hB0 = lds128(rowB + 16), hB1 = lds128(rowB + 32);
            const uint32_t ha[8] = {hA0.x, hA0.y, hA0.z, hA0.w, hA1.x, hA1.y, hA1.z, hA1.w};
            const uint32_t hb[8] = {hB0.x, hB0.y, hB0.z, hB0.w, hB1.x, hB1.y, hB1.z, hB1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                fA[u] = ha[u] >> (2 * t);
                fB[u] = hb[u] >> (2 * t);
            }
        }
        // 6-bit scale/min codes of sub-blocks 2t, 2t+1 as (code_2t, code_2t+1)
        // in bits 0..5 / 16..21.  t < 2: sc = s[j] & 63, m = s[j+4] & 63;
        // t >= 2 (j >= 4): sc = (s[j+4] & 15) | (s[j-4] >> 6) << 4,
        // m = (s[j+4] >> 4) | (s[j] >> 6) << 4.
        const bool lo = t < 2;
        const uint32_t jj0 = (2 * t) & 3;
        const uint32_t sel = 0x4040u | jj0 | ((jj0 + 1) << 8);
        const uint32_t mka = lo ? 0x003F003Fu : 0x000F000Fu, mkb = lo ? 0u : 0x00300030u;
        uint32_t S_lo[2], B_lo[2], S_hi[2], B_hi[2], M_lo[2], M_hi[2];
        float dd[2], dm[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint4 hh = r ? hB : hA;
            const uint32_t asc = lo ? hh.y : hh.w;
            const uint32_t am = lo ? hh.z : (hh.w >> 4);
            const uint32_t scp = (__byte_perm(asc, 0, sel) & mka) | ((__byte_perm(hh.y, 0, sel) >> 2) & mkb);
            const uint32_t mp = (__byte_perm(am, 0, sel) & mka) | ((__byte_perm(hh.z, 0, sel) >> 2) & mkb);
            const uint32_t scf = hsub2_u32(scp | kH1024, kH1024);   // (sc_2t, sc_2t+1) exactly
            const uint32_t mf = hsub2_u32(mp | kH1024, kH1024);
            S_lo[r] = __byte_perm(scf, 0, 0x1010);
            S_hi[r] = hmul2_u32(__byte_perm(scf, 0, 0x3232), kH1_16);
            B_lo[r] = hmul2_u32(S_lo[r], kHm1024);   // -1024 sc
            B_hi[r] = hmul2_u32(S_hi[r], kHm1024);   // -64 sc
            M_lo[r] = __byte_perm(mf, 0, 0x1010);
            M_hi[r] = __byte_perm(mf, 0, 0x3232);
            dd[r] = h2f(hh.x & 0xffff);
            dm[r] = h2f(hh.x >> 16);
        }
        const uint32_t wA[8] = {qA0.x, qA0.y, qA0.z, qA0.w, qA1.x, qA1.y, qA1.z, qA1.w};
        const uint32_t wB[8] = {qB0.x, qB0.y, qB0.z, qB0.w, qB1.x, qB1.y, qB1.z, qB1.w};
        // independent MMA chains: four for one n-tile, two per n-tile for two
        // (the same MMAs in flight, fewer accumulator registers)
        constexpr int CH = NT == 1 ? 4 : 2;
        float D[CH][NT][4], Dm[NT][4];
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) D[c][nt][e] = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t a = wA[u], b = wB[u], a8 = a >> 8, b8 = b >> 8;
            uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
            if constexpr (FIVE) {
                // fifth bit: bit 0 (low codes) / bit 1 (high codes) of each
                // byte of f moved to bit 4 / bit 8 of its 16-bit lane
                const uint32_t fa = fA[u], fb = fB[u];
                // low nibbles: 1024 + nib + 16 h, times sc, minus 1024 sc -> q sc exactly
                a0 = vhfma2(vbitsel(a, vand_or(fa << 4, 0x00100010u, kH1024), 0x000F000Fu), S_lo[0], B_lo[0]);
                a1 = vhfma2(vbitsel(b, vand_or(fb << 4, 0x00100010u, kH1024), 0x000F000Fu), S_lo[1], B_lo[1]);
                a2 = vhfma2(vbitsel(a8, vand_or(fa >> 4, 0x00100010u, kH1024), 0x000F000Fu), S_lo[0], B_lo[0]);
                a3 = vhfma2(vbitsel(b8, vand_or(fb >> 4, 0x00100010u, kH1024), 0x000F000Fu), S_lo[1], B_lo[1]);
                // high nibbles: 1024 + 16 nib + 256 h = 1024 + 16 q, times sc / 16, minus 64 sc
                c0 = vhfma2(vbitsel(a, vand_or(fa << 7, 0x01000100u, kH1024), 0x00F000F0u), S_hi[0], B_hi[0]);
                c1 = vhfma2(vbitsel(b, vand_or(fb << 7, 0x01000100u, kH1024), 0x00F000F0u), S_hi[1], B_hi[1]);
                c2 = vhfma2(vbitsel(a8, vand_or(fa >> 1, 0x01000100u, kH1024), 0x00F000F0u), S_hi[0], B_hi[0]);
                c3 = vhfma2(vbitsel(b8, vand_or(fb >> 1, 0x01000100u, kH1024), 0x00F000F0u), S_hi[1], B_hi[1]);
            } else {
                // low nibbles: (1024 + q) sc - 1024 sc = q sc exactly
                a0 = vhfma2(vand_or(a, 0x000F000Fu, kH1024), S_lo[0], B_lo[0]);
                a1 = vhfma2(vand_or(b, 0x000F000Fu, kH1024), S_lo[1], B_lo[1]);
                a2 = vhfma2(vand_or(a8, 0x000F000Fu, kH1024), S_lo[0], B_lo[0]);
                a3 = vhfma2(vand_or(b8, 0x000F000Fu, kH1024), S_lo[1], B_lo[1]);
                // high nibbles: (1024 + 16 q) sc / 16 - 64 sc = q sc exactly
                c0 = vhfma2(vand_or(a, 0x00F000F0u, kH1024), S_hi[0], B_hi[0]);
                c1 = vhfma2(vand_or(b, 0x00F000F0u, kH1024), S_hi[1], B_hi[1]);
                c2 = vhfma2(vand_or(a8, 0x00F000F0u, kH1024), S_hi[0], B_hi[0]);
                c3 = vhfma2(vand_or(b8, 0x00F000F0u, kH1024), S_hi[1], B_hi[1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 bl = lds64(bb[nt] + u * 32);
                const uint2 bh = lds64(bb[nt] + (8 + u) * 32);
                mma_f16(D[u % CH][nt], a0, a1, a2, a3, bl.x, bl.y);
                mma_f16(D[u % CH][nt], c0, c1, c2, c3, bh.x, bh.y);
            }
        }
        // y += 2^-s (d D - dmin sum_j m_j X_j), 2^-s of this block for the
        // column's token: tokens 2t, 2t + 1 of the n-tile, one 2-byte load
        // from the [block][16 tokens] table of biased exponents 127 - s
        // (entries past m are never stored)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 bv = lds64(bb[nt] + 512);
            const uint32_t eb = lds_u16(sb + p.off_xs + 16 * gb + 8 * nt + 2 * t);
            const float iv[2] = {__uint_as_float((eb & 0xFFu) << 23), __uint_as_float((eb >> 8) << 23)};
#pragma unroll
            for (int e = 0; e < 4; ++e) Dm[nt][e] = 0.f;
            mma_f16(Dm[nt], M_lo[0], M_lo[1], M_hi[0], M_hi[1], bv.x, bv.y);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e >> 1;
                float Ds = D[0][nt][e] + D[1][nt][e];
                if constexpr (CH == 4) Ds = (D[0][nt][e] + D[1][nt][e]) + (D[2][nt][e] + D[3][nt][e]);
                acc[4 * nt + e] = fmaf(iv[e & 1], fmaf(dd[r], Ds, -dm[r] * Dm[nt][e]), acc[4 * nt + e]);
            }
        }
    }

    static __device__ __forceinline__ void store_part(const SP& p, const Lane& L, float (&acc)[4 * NT], float* part) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * nt + 2 * L.t + (e & 1);
                if (tok < p.m) part[(L.g + 8 * (e >> 1)) * p.m + tok] = acc[4 * nt + e];
            }
    }

    // Image per block and token: MMA (nib, u) of lane t uses the scaled
    // values v = 64t + 32nib + 4u + {0,2 | 1,3}; the last 32 bytes hold (Xhi,
    // Xlo) of sub-blocks 2t and 2t+1, the sums of their binary16 operands.
    // Sixteen neighbouring lanes share a (token, block), one per (t, nib,
    // half uu of u): 16 values each.  They agree on the block's scale 2^s
    // (largest |x| at 2^9) by four shuffles and add the two halves of a
    // sub-block sum by one; 127 - s (the biased exponent of 2^-s) goes to the
    // [block][16 tokens] byte table.  Every warp runs the same number of
    // rounds, so the shuffles always see the whole warp.
    // Returns whether this thread met a non-finite activation.
    static __device__ bool build(const SP& p, uint32_t sb, int64_t xoff) {
        bool bad = false;
        const int total = p.m * p.nblk * 16;
        // the 16 values of lane e: (token, block) e / 16, t, nib, uu from e
        // mod 16; read a round ahead, so that a round's loads (from global
        // memory when the image is built from x in place) are in flight while
        // the previous round converts
        auto load = [&](int e, uint4 (&r)[2]) {
            r[0] = r[1] = make_uint4(0u, 0u, 0u, 0u);
            if (e >= total) return;
            const int q = e >> 4, tok = q / p.nblk, bl = q - tok * p.nblk;
            const int64_t xi = static_cast<int64_t>(bl) * 256 + 64 * ((e >> 2) & 3) + 32 * ((e >> 1) & 1) + 16 * (e & 1);
            if (p.x_global) {
                const uint16_t* xg = p.x + static_cast<int64_t>(tok) * p.k * p.ks + xoff + xi;
                r[0] = ldg_nc_v4(xg);
                r[1] = ldg_nc_v4(xg + 8);
            } else {
                const uint32_t xs = xaddr(p, sb, tok, xi);
                r[0] = lds128(xs);
                r[1] = lds128(xs + 16);
            }
        };
        uint4 nx[2];
        load((threadIdx.x & ~31) + (threadIdx.x & 31), nx);
        for (int w0 = threadIdx.x & ~31; w0 < total; w0 += kCW * 32) {
            const int e = w0 + (threadIdx.x & 31);
            const bool in = e < total;
            const int q = e >> 4, tok = q / p.nblk, bl = q - tok * p.nblk;
            const int uu = e & 1, nib = (e >> 1) & 1, t = (e >> 2) & 3;
            const uint32_t base = sb + p.off_img + tok * p.img_tok + bl * kBlkImg;
            const uint4 r[2] = {nx[0], nx[1]};
            load(e + kCW * 32, nx);
            uint32_t mx = absmax8_bf16(absmax8_bf16(0u, r[0]), r[1]);
            mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            bad |= in && mx >= 0x7F80u;
            const int se = xscale_exp(mx, kXT);
            const float S = exp2_int(se);
            if (in && (e & 15) == 0) sts8(sb + p.off_xs + 16 * bl + tok, static_cast<uint32_t>(127 - se));
            float X = 0.f;
            const uint32_t wv[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int u = 4 * uu + qq;
                // binary16 pairs (v0, v2) and (v1, v3) of the scaled values
                const uint32_t h02 = pack_f16x2(bf16lo_to_f32(wv[2 * qq]) * S, bf16lo_to_f32(wv[2 * qq + 1]) * S);
                const uint32_t h13 = pack_f16x2(bf16hi_to_f32(wv[2 * qq]) * S, bf16hi_to_f32(wv[2 * qq + 1]) * S);
                X = add_f16hi(h13, add_f16hi(h02, add_f16lo(h13, add_f16lo(h02, X))));
                if (in) sts64(base + (nib * 8 + u) * 32 + t * 8, h02, h13);
            }
            // the sub-block sum: this half plus the other (lane e ^ 1), in uu order
            const float Xo = __shfl_xor_sync(0xffffffffu, X, 1);
            if (in && uu == 0) {
                const float Xs = X + Xo;
                const __half hi = __float2half_rn(Xs);
                const __half lo = __float2half_rn(Xs - __half2float(hi));
                sts32(base + 512 + t * 8 + 4 * nib, hpair(hi, lo));
            }
        }
        return bad;
    }
};

// ===========================================================================
// q4_K and q5_K at one activation row (column form)
// ===========================================================================
// With a single token the 8 MMA columns are free to separate sub-blocks, as in
// q6_K: lane t's low nibbles (sub-block 2t) go to column 2t, its high nibbles
// (sub-block 2t+1) to column 2t+1, each B lane of another column reading a
// zero block.  The codes then enter the MMA as plain binary16 subnormals (q
// 2^-24; the high nibble in place, 16 q 2^-24, against x/16) and the 6-bit
// scales and mins are applied once per block in the fp32 epilogue:
//   y += 2^-s (d sc_2t 2^24 D_2t + d sc_2t+1 2^24 D_2t+1 - dmin (m_2t X_2t + m_2t+1 X_2t+1)),
// X_j the fp32 sum of sub-block j's binary16 operands as the MMA consumed
// them (x 2^s, resp. 16 binary16(x 2^s / 16)).  No per-code scale product,
// no min-term MMA.  q5_K: the fifth bit merged into the code (q <= 31).
template <bool FIVE = false>
struct Q4C {
    static constexpr int kVPB = 256, kBPB = FIVE ? 176 : 144;
    static constexpr bool kSplit = false;
    static constexpr int kItemBlocks = 1;
    // image per block: 16 MMAs x 4 lanes x 8 bytes, then X_2t, X_2t+1 (fp32) per lane
    static constexpr uint32_t kBlkImg = 544;
    static constexpr uint32_t kZero = 512;
    static constexpr int kAccPerLane = 2;
    // a block's scaled activations below 2^15: far inside binary16
    static constexpr int kXT = 14;

    static __device__ __forceinline__ void item(const SP& p, uint32_t sb, const Lane& L, uint32_t rowA,
                                                uint32_t rowB, int gb, float (&acc)[2]) {
        const int t = L.t;
        const uint32_t img = sb + p.off_img + gb * kBlkImg;
        const uint32_t zero = sb + p.off_zero + 8 * t;
        // B lanes whose column holds lane t's low (2t) or high (2t+1) sub-block
        const uint32_t blo = L.g == 2 * t ? img + 8 * t : zero;
        const uint32_t bhi = L.g == 2 * t + 1 ? img + 256 + 8 * t : zero;
        const uint4 hA = lds128(rowA), hB = lds128(rowB);
        constexpr uint32_t kQs = FIVE ? 48 : 16;   // first code byte
        const uint4 qA0 = lds128(rowA + kQs + 32 * t), qA1 = lds128(rowA + kQs + 16 + 32 * t);
        const uint4 qB0 = lds128(rowB + kQs + 32 * t), qB1 = lds128(rowB + kQs + 16 + 32 * t);
        uint32_t fA[8], fB[8];   // q5_K: qh[4u .. 4u+3] >> 2t (the lane's two bits at bits 0, 1 of each byte)
        if constexpr (FIVE) {
            const uint4 hA0 = lds128(rowA + 16), hA1 = lds128(rowA + 32);
            const uint4 hB0 = lds128(rowB + 16), hB1 = lds128(rowB + 32);
            const uint32_t ha[8] = {hA0.x, hA0.y, hA0.z, hA0.w, hA1.x, hA1.y, hA1.z, hA1.w};
            const uint32_t hb[8] = {hB0.x, hB0.y, hB0.z, hB0.w, hB1.x, hB1.y, hB1.z, hB1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                fA[u] = ha[u] >> (2 * t);
                fB[u] = hb[u] >> (2 * t);
            }
        }
        const uint32_t wA[8] = {qA0.x, qA0.y, qA0.z, qA0.w, qA1.x, qA1.y, qA1.z, qA1.w};
        const uint32_t wB[8] = {qB0.x, qB0.y, qB0.z, qB0.w, qB1.x, qB1.y, qB1.z, qB1.w};
        float D[4][4];   // four independent MMA chains
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) D[c][e] = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t a = wA[u], b = wB[u], a8 = a >> 8, b8 = b >> 8;
            uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
            if constexpr (FIVE) {
                const uint32_t fa = fA[u], fb = fB[u];
                a0 = vbitsel(a, vand_or(fa << 4, 0x00100010u, 0u), 0x000F000Fu);
                a1 = vbitsel(b, vand_or(fb << 4, 0x00100010u, 0u), 0x000F000Fu);
                a2 = vbitsel(a8, vand_or(fa >> 4, 0x00100010u, 0u), 0x000F000Fu);
                a3 = vbitsel(b8, vand_or(fb >> 4, 0x00100010u, 0u), 0x000F000Fu);
                c0 = vbitsel(a, vand_or(fa << 7, 0x01000100u, 0u), 0x00F000F0u);
                c1 = vbitsel(b, vand_or(fb << 7, 0x01000100u, 0u), 0x00F000F0u);
                c2 = vbitsel(a8, vand_or(fa >> 1, 0x01000100u, 0u), 0x00F000F0u);
                c3 = vbitsel(b8, vand_or(fb >> 1, 0x01000100u, 0u), 0x00F000F0u);
            } else {
                a0 = vand_or(a, 0x000F000Fu, 0u);
                a1 = vand_or(b, 0x000F000Fu, 0u);
                a2 = vand_or(a8, 0x000F000Fu, 0u);
                a3 = vand_or(b8, 0x000F000Fu, 0u);
                c0 = vand_or(a, 0x00F000F0u, 0u);
                c1 = vand_or(b, 0x00F000F0u, 0u);
                c2 = vand_or(a8, 0x00F000F0u, 0u);
                c3 = vand_or(b8, 0x00F000F0u, 0u);
            }
            const uint2 bl = lds64(blo + u * 32);
            const uint2 bh = lds64(bhi + u * 32);
            mma_f16(D[u & 3], a0, a1, a2, a3, bl.x, bl.y);
            mma_f16(D[u & 3], c0, c1, c2, c3, bh.x, bh.y);
        }
        // 6-bit scale/min codes of sub-blocks 2t, 2t+1 as (code_2t, code_2t+1)
        // in bits 0..5 / 16..21.  t < 2: sc = s[j] & 63, m = s[j+4] & 63;
        // t >= 2 (j >= 4): sc = (s[j+4] & 15) | (s[j-4] >> 6) << 4,
        // m = (s[j+4] >> 4) | (s[j] >> 6) << 4.
        const bool lo = t < 2;
        const uint32_t jj0 = (2 * t) & 3;
        const uint32_t sel = 0x4040u | jj0 | ((jj0 + 1) << 8);
        const uint32_t mka = lo ? 0x003F003Fu : 0x000F000Fu, mkb = lo ? 0u : 0x00300030u;
        const uint2 xv = lds64(img + 512 + 8 * t);   // X_2t, X_2t+1
        const float X0 = __uint_as_float(xv.x), X1 = __uint_as_float(xv.y);
        const float iv = __uint_as_float(static_cast<uint32_t>(lds_u16(sb + p.off_xs + 16 * gb) & 0xFFu) << 23);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint4 hh = r ? hB : hA;
            const uint32_t asc = lo ? hh.y : hh.w;
            const uint32_t am = lo ? hh.z : (hh.w >> 4);
            const uint32_t scp = (__byte_perm(asc, 0, sel) & mka) | ((__byte_perm(hh.y, 0, sel) >> 2) & mkb);
            const uint32_t mp = (__byte_perm(am, 0, sel) & mka) | ((__byte_perm(hh.z, 0, sel) >> 2) & mkb);
            const float d24 = h2f(hh.x & 0xffff) * kTwo24, dm = h2f(hh.x >> 16);
            const float D0 = (D[0][2 * r] + D[1][2 * r]) + (D[2][2 * r] + D[3][2 * r]);
            const float D1 = (D[0][2 * r + 1] + D[1][2 * r + 1]) + (D[2][2 * r + 1] + D[3][2 * r + 1]);
            const float sc0 = static_cast<float>(scp & 0xFFFFu), sc1 = static_cast<float>(scp >> 16);
            const float m0 = static_cast<float>(mp & 0xFFFFu), m1 = static_cast<float>(mp >> 16);
            const float v = fmaf(__fmul_rn(d24, sc0), D0, fmaf(__fmul_rn(d24, sc1), D1, -dm * fmaf(m0, X0, m1 * X1)));
            acc[r] = fmaf(iv, v, acc[r]);
        }
    }

    static __device__ __forceinline__ void store_part(const SP& p, const Lane& L, float (&acc)[2], float* part) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            float v = acc[r];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            if (L.t == 0) part[(L.g + 8 * r) * p.m] = v;
        }
    }

    // Image per (token, block): entry (nib, u, t) = binary16 of lane t's values
    // 64t + 32nib + 4u + {0,2 | 1,3}, scaled by 2^s (nib 0) or 2^s / 16 (nib
    // 1, against the high nibble in place), at 256 nib + 32 u + 8 t; then the
    // fp32 sums X_2t, X_2t+1 at 512 + 8t.  Sixteen neighbouring lanes share a
    // block, one per (t, nib, half uu of u): they agree on the block's scale
    // 2^s (largest |x| at 2^14) by four shuffles and add the two halves of a
    // sub-block sum by one; 127 - s goes to the [block][16 tokens] byte table.
    // Every warp runs the same number of rounds, so the shuffles always see
    // the whole warp.  Returns whether this thread met a non-finite activation.
    static __device__ bool build(const SP& p, uint32_t sb, int64_t xoff) {
        bool bad = false;
        const int total = p.m * p.nblk * 16;
        for (int w0 = threadIdx.x & ~31; w0 < total; w0 += kCW * 32) {
            const int e = w0 + (threadIdx.x & 31);
            const bool in = e < total;
            const int q = e >> 4, tok = q / p.nblk, bl = q - tok * p.nblk;
            const int uu = e & 1, nib = (e >> 1) & 1, t = (e >> 2) & 3;
            uint4 r[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if (in) {
                const uint32_t xs = xaddr(p, sb, tok, static_cast<int64_t>(bl) * 256 + 64 * t + 32 * nib + 16 * uu);
                r[0] = lds128(xs);
                r[1] = lds128(xs + 16);
            }
            uint32_t mx = absmax8_bf16(absmax8_bf16(0u, r[0]), r[1]);
            mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            bad |= in && mx >= 0x7F80u;
            const int se = xscale_exp(mx, kXT);
            const float S = exp2_int(se) * (nib ? 0.0625f : 1.0f);
            const uint32_t base = sb + p.off_img + tok * p.img_tok + bl * kBlkImg;
            if (in && (e & 15) == 0) sts8(sb + p.off_xs + 16 * bl + tok, static_cast<uint32_t>(127 - se));
            float X = 0.f;
            const uint32_t wv[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int u = 4 * uu + qq;
                const uint32_t h02 = pack_f16x2(bf16lo_to_f32(wv[2 * qq]) * S, bf16lo_to_f32(wv[2 * qq + 1]) * S);
                const uint32_t h13 = pack_f16x2(bf16hi_to_f32(wv[2 * qq]) * S, bf16hi_to_f32(wv[2 * qq + 1]) * S);
                X = add_f16hi(h13, add_f16hi(h02, add_f16lo(h13, add_f16lo(h02, X))));
                if (in) sts64(base + nib * 256 + u * 32 + t * 8, h02, h13);
            }
            // the sub-block sum: this half plus the other (lane e ^ 1); the
            // high sub-block's operands stand for 16 times their value
            const float Xs = (X + __shfl_xor_sync(0xffffffffu, X, 1)) * (nib ? 16.0f : 1.0f);
            if (in && uu == 0) sts32(base + 512 + t * 8 + 4 * nib, __float_as_uint(Xs));
        }
        return bad;
    }
};

// ===========================================================================
// Kernel
// ===========================================================================
// SPLIT: the launch is in clusters of p.ks CTAs that split K (compiled out
// otherwise, so the unsplit kernel carries none of it).
// Gather mode, all threads: this CTA's virtual expert (its expert, pairs and
// row range) from the id list.  False when the launch has no virtual expert
// for this CTA.
__device__ bool gather_setup(const SPG& p, uint8_t* smem, int64_t& r0, int64_t& r1, int& ge, int& gm) {
    int* cnt = reinterpret_cast<int*>(smem + kGCount);
    int* glist = reinterpret_cast<int*>(smem + kGList);
    volatile int* gmisc = reinterpret_cast<volatile int*>(smem + kGMisc);
    volatile long long* grange = reinterpret_cast<volatile long long*>(smem + kGMisc + 16);
    const int tid = threadIdx.x;
    for (int e = tid; e < p.n_experts; e += kThreads) cnt[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int q = tid; q < p.pairs; q += kThreads) {
        const int e = p.ids[q];
        if (e < 0 || e >= p.n_experts) bad = 1;
        else atomicAdd(&cnt[e], 1);
    }
    if (bad && p.err) atomicOr(p.err, KQ_DEV_BAD_EXPERT);
    __syncthreads();
    if (tid < 32) {
        const int lane = tid;
        // virtual experts per expert, lane l holding experts 8l .. 8l + 7
        int loc[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * lane + i;
            loc[i] = e < p.n_experts ? (cnt[e] + p.m - 1) / p.m : 0;
            sum += loc[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int vj = min(p.vcount, total - p.vbase);
        if (lane == 0) gmisc[0] = -1;
        __syncwarp();
        if (vj > 0) {
            // CTA c serves virtual expert floor(c vj / G); the CTAs of one
            // virtual expert split its rows evenly
            const int64_t G = gridDim.x, c = blockIdx.x;
            const int vl = static_cast<int>(c * vj / G);
            const int64_t cf = (static_cast<int64_t>(vl) * G + vj - 1) / vj;
            const int64_t cn = (static_cast<int64_t>(vl + 1) * G + vj - 1) / vj - cf;
            const int v = p.vbase + vl;
            const int excl = incl - sum;
            if (v >= excl && v < incl) {
                int acc = excl, e = -1, b = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (e < 0 && v < acc + loc[i]) {
                        e = 8 * lane + i;
                        b = v - acc;
                    }
                    acc += loc[i];
                }
                gmisc[0] = e;
                gmisc[1] = b;
                gmisc[2] = min(p.m, cnt[e] - b * p.m);
                grange[0] = (c - cf) * p.n / cn;
                grange[1] = (c - cf + 1) * p.n / cn;
            }
        }
        __syncwarp();
        // the pairs of the virtual expert: ranks [b m, b m + present) among
        // the pairs of expert e, in (token, slot) order
        const int e = gmisc[0];
        if (e >= 0) {
            const int lo = gmisc[1] * p.m, hi = lo + gmisc[2];
            int seen = 0;
            for (int q0 = 0; q0 < p.pairs && seen < hi; q0 += 32) {
                const int q = q0 + lane;
                const bool hit = q < p.pairs && p.ids[q] == e;
                const unsigned bal = __ballot_sync(0xffffffffu, hit);
                const int rk = seen + __popc(bal & ((1u << lane) - 1u));
                if (hit && rk >= lo && rk < hi) glist[rk - lo] = q;
                seen += __popc(bal);
            }
        }
    }
    __syncthreads();
    ge = gmisc[0];
    if (ge < 0) return false;
    gm = gmisc[2];
    r0 = grange[0];
    r1 = grange[1];
    return true;
}

// The weight bank a stage is read from (GLU: gate or up) and its size.
template <class P>
__device__ __forceinline__ const uint8_t* bank_of(const P& p, bool up) {
    if constexpr (std::is_same<P, SPGLU>::value) return up ? p.w2 : p.w;
    else return p.w;
}
template <class P>
__device__ __forceinline__ int64_t bank_bytes(const P& p) {
    if constexpr (std::is_same<P, SP>::value) return p.n * p.row_bytes;
    else return static_cast<int64_t>(p.n_experts) * p.n * p.row_bytes;
}

// act(g) * u of the GLU epilogue, in fp32: silu(g) = g / (1 + e^-g); gelu in
// its tanh form 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))); silu with
// limit: silu(min(g, L)) * clamp(u, -L, L).
__device__ __forceinline__ float glu_act(int act, float limit, float g, float u) {
    if (act == 2) {
        g = fminf(g, limit);
        u = fminf(fmaxf(u, -limit), limit);
    }
    float a;
    if (act == 1) a = 0.5f * g * (1.0f + tanhf(0.7978845608028654f * (g + 0.044715f * g * g * g)));
    else a = g / (1.0f + expf(-g));
    return a * u;
}

template <class C, bool SPLIT, class P = SP>
__global__ void __launch_bounds__(kThreads, 1) qmv_stream_kernel(const P p) {
    constexpr bool GATHER = !std::is_same<P, SP>::value;
    constexpr bool GLU = std::is_same<P, SPGLU>::value;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // [kMaxStages]
    uint64_t* empty = full + kMaxStages;                   // [kMaxStages]
    uint64_t* xbar = full + 2 * kMaxStages;
    uint64_t* pfree = xbar + 1;                            // [2] partial-sum slots released
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 128);
    int* grp_done = reinterpret_cast<int*>(smem + 256);   // [kMaxGroups]
    const uint32_t sb = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // A cluster of p.ks CTAs owns a balanced contiguous range of rows; CTA
    // `rank` of it covers blocks [rank nblk, (rank + 1) nblk) of every row.
    const int ks = SPLIT ? p.ks : 1;
    const int rank = SPLIT ? static_cast<int>(cluster_ctarank()) : 0;
    const int ncl = static_cast<int>(gridDim.x) / ks, cl = static_cast<int>(blockIdx.x) / ks;
    int64_t r0 = static_cast<int64_t>(cl) * p.n / ncl;
    int64_t r1 = static_cast<int64_t>(cl + 1) * p.n / ncl;
    const uint32_t stage_bytes = kRows * p.rs;
    const int64_t kb0 = static_cast<int64_t>(rank) * p.nblk;   // first block of the slice

    if (tid == 0) {
        for (int i = 0; i < p.ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kCW);
        }
        mbar_init(xbar, 1);
        if (SPLIT || GATHER) {
            mbar_init(&pfree[0], 1);
            mbar_init(&pfree[1], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid < kMaxGroups) grp_done[tid] = 0;
    __syncthreads();
    // Programmatic dependent launch: the next kernel may start its prologue;
    // this one waits for the earlier grids before it reads x or W.  (Asking L2
    // for the first weight stages before the wait was measured to slow down
    // the tail of the earlier grid more than it gained.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // gather: the expert's weights, the pairs present (x rows gathered and y
    // rows scattered through the pair list) and the row range
    const uint8_t* wbase = p.w;
    const uint8_t* wbase2 = nullptr;
    int gm = p.m;
    const int* glist = reinterpret_cast<const int*>(smem + kGList);
    if constexpr (GATHER) {
        int ge = 0;
        if (!gather_setup(p, smem, r0, r1, ge, gm)) return;
        wbase = p.w + static_cast<int64_t>(ge) * p.n * p.row_bytes;
        if constexpr (GLU) wbase2 = p.w2 + static_cast<int64_t>(ge) * p.n * p.row_bytes;
    }
    const int nrg = cdiv(r1 - r0, kRows);
    const int nlg = GLU ? 2 * nrg : nrg;   // logical row groups (GLU: gate and up)

    if (warp == kProd) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            if (p.x_global) {
                mbar_arrive(xbar);
            } else {
                const uint32_t row = 2u * static_cast<uint32_t>(p.k);
                mbar_arrive_expect_tx(xbar, row * p.m);
                for (int tok = 0; tok < p.m; ++tok) {
                    // gather: token slots past the pairs present repeat the last pair's row
                    int64_t xr = tok;
                    if constexpr (GATHER) xr = glist[tok < gm ? tok : gm - 1] / p.xdiv;
                    bulk_g2s(smem + p.off_xraw + tok * row, p.x + xr * p.k * ks + kb0 * C::kVPB, row, xbar);
                }
            }
        }
        // ring position: stage q goes to slot q mod ns, whose previous fill
        // (phase parity ^ 1) must have been released first
        int q = 0, slot = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int rg = 0; rg < nlg && ok; ++rg) {
            const int gi = GLU ? rg >> 1 : rg;
            const int64_t row0 = r0 + static_cast<int64_t>(group_order(gi, nrg, r1 - r0)) * kRows;
            const int rv = static_cast<int>(r1 - row0 < kRows ? r1 - row0 : kRows);
            const uint8_t* wsrc = (GLU && (rg & 1)) ? wbase2 : wbase;
            for (int st = 0; st < p.spr; ++st, ++q) {
                if (lane == 0 && q >= p.ns) ok = sleep_wait(&empty[slot], phase ^ 1, p.status, wait_limit());
                ok = __shfl_sync(0xffffffffu, ok, 0) && !*abort_flag;
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                const int b0 = st * p.g;
                const int nb = p.nblk - b0 < p.g ? p.nblk - b0 : p.g;
                const uint32_t bytes = static_cast<uint32_t>(nb) * C::kBPB;
                bool rt = false;
                if constexpr (C::kBPB == 210 && GATHER) rt = (p.row_bytes & 15) != 0;
                if (rt) {
                    // rows that are not a 16-byte multiple (decode MoE q6_K):
                    // each row's span is copied from the 16-byte boundary at or
                    // below its first byte, so it lands at its own offset in
                    // the slot; the copy stops at the last 16-byte boundary of
                    // the bank and the bytes after it (the bank's last row only)
                    // are stored one by one before the stage is announced
                    const uint8_t* bank = bank_of(p, GLU && (rg & 1));
                    const int64_t lim = bank_bytes(p) & ~int64_t(15);
                    uint32_t nb16 = 0;
                    if (lane < rv) {
                        const int64_t a0 = (wsrc - bank) + (row0 + lane) * p.row_bytes + (kb0 + b0) * C::kBPB;
                        const int64_t s0 = a0 & ~int64_t(15), end = a0 + bytes;
                        const int64_t ce = ((end + 15) & ~int64_t(15)) < lim ? ((end + 15) & ~int64_t(15)) : lim;
                        nb16 = ce > s0 ? static_cast<uint32_t>(ce - s0) : 0u;
                        uint8_t* dst = smem + p.off_stage + slot * stage_bytes + lane * p.rs;
                        for (int64_t b = ce > a0 ? ce : a0; b < end; ++b)
                            asm volatile("st.shared.u8 [%0], %1;" ::"r"(smem_u32(dst + (b - s0))),
                                         "r"(static_cast<uint32_t>(__ldg(bank + b))));
                    }
                    const uint32_t tx = __reduce_add_sync(0xffffffffu, nb16);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_expect_tx(&full[slot], tx);
                    __syncwarp();
                    if (nb16) {
                        const int64_t a0 = (wsrc - bank) + (row0 + lane) * p.row_bytes + (kb0 + b0) * C::kBPB;
                        bulk_g2s(smem + p.off_stage + slot * stage_bytes + lane * p.rs, bank + (a0 & ~int64_t(15)),
                                 nb16, &full[slot]);
                    }
                } else {
                    if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes * rv);
                    __syncwarp();
                    if (lane < rv)
                        bulk_g2s(smem + p.off_stage + slot * stage_bytes + lane * p.rs,
                                 wsrc + (row0 + lane) * p.row_bytes + (kb0 + b0) * C::kBPB, bytes, &full[slot]);
                }
                if (++slot == p.ns) {
                    slot = 0;
                    phase ^= 1;
                }
            }
        }
        // The copies this warp issued land before the CTA exits, also when a
        // consumer gave up on a wait after the last stage was issued: the x
        // copy and the latest fill of every slot (each slot's last phase, so
        // a completed wait returns at once), with the full time limit.
        if (lane == 0) {
            sleep_wait(xbar, 0, nullptr, kWaitLimitNs);
            for (int qq = q - p.ns > 0 ? q - p.ns : 0; qq < q; ++qq)
                sleep_wait(&full[qq % p.ns], (qq / p.ns) & 1, nullptr, kWaitLimitNs);
        }
    } else {
        // --------------------------------------------------------- consumers
        Lane L;
        L.g = lane >> 2;
        L.t = lane & 3;
        if (!spin_wait(xbar, 0, p.status, p.strict)) *abort_flag = 1;
        // the activation image with its per-block (or per-run) scales
        bool bad = false;
        if (!*abort_flag) {
            bad |= C::build(p, sb, kb0 * C::kVPB);
            for (uint32_t o = 4 * tid; o < C::kZero; o += 4 * kCW * 32) sts32(sb + p.off_zero + o, 0u);
        }
        if (bad) atomicOr(p.status, KQ_DEV_X_RANGE);   // an activation is Inf or NaN
        asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");   // image ready (x copy now dead)
        float* part = reinterpret_cast<float*>(smem + p.off_part);
        const int items_per_row = p.nblk / C::kItemBlocks;
        int slot = 0;   // ring slot and fill parity of the next stage
        uint32_t phase = 0;
        for (int rg = 0; rg < nlg && !*abort_flag; ++rg) {
            const int gi = GLU ? rg >> 1 : rg;
            const int64_t row0 = r0 + static_cast<int64_t>(group_order(gi, nrg, r1 - r0)) * kRows;
            const int rv = static_cast<int>(r1 - row0 < kRows ? r1 - row0 : kRows);
            float acc[C::kAccPerLane];
#pragma unroll
            for (int i = 0; i < C::kAccPerLane; ++i) acc[i] = 0.f;
            // items of the row group, round robin over warps across stages
            bool ok = true;
            for (int st = 0; st < p.spr; ++st) {
                const int i0 = st * p.g / C::kItemBlocks;
                const int i1 = min(items_per_row, (st + 1) * p.g / C::kItemBlocks);
                // items continue the round robin of the previous row groups, so
                // that rows with fewer items than warps still spread over all
                const int rot = SPLIT ? rg * items_per_row : 0;
                const int first = i0 + ((warp - i0 - rot) & (kCW - 1));
                // every warp waits for the stage, items or not, so that its
                // release below always belongs to this fill of the slot
                if (!spin_wait(&full[slot], phase, p.status)) {
                    *abort_flag = 1;
                    ok = false;
                } else {
                    const uint32_t stg = sb + p.off_stage + slot * stage_bytes;
                    uint32_t rowA = stg + L.g * p.rs, rowB = rowA + 8 * p.rs;
                    bool rt = false;
                    if constexpr (C::kBPB == 210 && GATHER) {
                        // rows that are not a 16-byte multiple sit at their own
                        // offsets in the slot (see the producer)
                        if (p.row_bytes & 15) {
                            rt = true;
                            const int64_t ab = (wbase - p.w) + static_cast<int64_t>(st * p.g) * C::kBPB;
                            rowA += static_cast<uint32_t>((ab + (row0 + L.g) * p.row_bytes) & 15);
                            rowB += static_cast<uint32_t>((ab + (row0 + L.g + 8) * p.row_bytes) & 15);
                        }
                    }
                    for (int it = first; it < i1; it += kCW) {
                        const uint32_t off = static_cast<uint32_t>(it * C::kItemBlocks - st * p.g) * C::kBPB;
                        if constexpr (C::kBPB == 210 && GATHER) {
                            if (rt) C::item_rt(p, sb, L, rowA + off, rowB + off, it, acc);
                            else C::item(p, sb, L, rowA + off, rowB + off, it, acc);
                        } else {
                            C::item(p, sb, L, rowA + off, rowB + off, it, acc);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                if (++slot == p.ns) {
                    slot = 0;
                    phase ^= 1;
                }
                if (!ok) break;
            }
            if (!ok) break;
            // partial sums -> shared memory; the last warp of the row group sums
            // the 16 partials in warp order and stores y (or, when the cluster
            // splits K, this CTA's share of y for the cluster reduction).  With
            // two slots (K split, gather), row group rg reuses the slot of rg - 2
            // once its sum is done; gather also reuses the two arrival counters,
            // so a CTA may own any number of rows.
            constexpr bool kReuse = SPLIT || GATHER;
            const int pslot = kReuse ? (rg & 1) : rg;
            if (kReuse && rg >= 2) {
                if (!spin_wait(&pfree[rg & 1], ((rg >> 1) - 1) & 1, p.status)) {
                    *abort_flag = 1;
                    break;
                }
            }
            float* pw = part + (pslot * kCW + warp) * kRows * p.m;
            C::store_part(p, L, acc, pw);
            __threadfence_block();
            __syncwarp();
            int last = 0;
            int* gdone = &grp_done[GATHER ? (rg & 1) : rg];
            if (lane == 0) last = atomicAdd(gdone, 1) == kCW - 1;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                __threadfence_block();
                // split: the sum of this slice goes to the CTA that owns the
                // row group (rg mod ks), into its receive slot for this rank
                const uint32_t recv = sb + p.off_red +
                                      4u * static_cast<uint32_t>(((rg / ks) * ks + rank) * kRows * p.m);
                const uint32_t dst = SPLIT ? mapa_u32(recv, static_cast<uint32_t>(rg % ks)) : 0u;
                if constexpr (SPLIT) {
                    // element f = r m + tok of the row group, four per 16-byte
                    // load, the 16 partials added in warp order
                    const int nv4 = kRows * p.m / 4;
                    const uint32_t pbase = sb + p.off_part + 16u * static_cast<uint32_t>(pslot * kCW * nv4);
                    for (int f4 = lane; f4 < nv4; f4 += 32) {
                        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int w = 0; w < kCW; ++w) {
                            const uint4 v = lds128(pbase + 16u * static_cast<uint32_t>(w * nv4 + f4));
                            sum[0] += __uint_as_float(v.x);
                            sum[1] += __uint_as_float(v.y);
                            sum[2] += __uint_as_float(v.z);
                            sum[3] += __uint_as_float(v.w);
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) st_cluster_f32(dst + 16u * f4 + 4u * c, sum[c]);
                    }
                } else {
                    for (int o = lane; o < kRows * p.m; o += 32) {
                        const int tok = o / kRows, r = o % kRows;
                        float sum = 0.f;
                        for (int w = 0; w < kCW; ++w) sum += part[((pslot * kCW + w) * kRows + r) * p.m + tok];
                        if constexpr (GLU) {
                            // gate sums wait behind the two partial slots for the up sums
                            float* gbuf = part + 2 * kCW * kRows * p.m;
                            if ((rg & 1) == 0) gbuf[o] = sum;
                            else if (r < rv && tok < gm)
                                p.y[static_cast<int64_t>(glist[tok]) * p.n + row0 + r] = glu_act(p.act, p.limit, gbuf[o], sum);
                        } else if constexpr (GATHER) {
                            if (r < rv && tok < gm) p.y[static_cast<int64_t>(glist[tok]) * p.n + row0 + r] = sum;
                        } else {
                            if (r < rv) p.y[static_cast<int64_t>(tok) * p.n + row0 + r] = sum;
                        }
                    }
                }
                __syncwarp();
                // the slot's next row group counts from zero; it starts only
                // after the release below
                if (GATHER && lane == 0) *gdone = 0;
                if (kReuse && lane == 0) mbar_arrive(&pfree[rg & 1]);
            }
        }
    }
    if constexpr (SPLIT) {
        // Every CTA of the cluster has pushed its slice sums of every row
        // group to the row group's owner; the owner adds them in slice order.
        // Nothing touches another CTA's shared memory after this barrier.
        __syncwarp();
        cluster_sync();
        if (!*abort_flag) {
            for (int rg = rank; rg < nrg; rg += ks) {
                const int64_t row0 = r0 + static_cast<int64_t>(group_order(rg, nrg, r1 - r0)) * kRows;
                const int rv = static_cast<int>(r1 - row0 < kRows ? r1 - row0 : kRows);
                const float* recv = reinterpret_cast<const float*>(smem + p.off_red) + (rg / ks) * ks * kRows * p.m;
                for (int f = tid; f < kRows * p.m; f += kThreads) {
                    const int r = f / p.m, tok = f - r * p.m;
                    if (r >= rv) continue;
                    float sum = 0.f;
                    for (int j = 0; j < ks; ++j) sum += recv[j * kRows * p.m + f];
                    p.y[static_cast<int64_t>(tok) * p.n + row0 + r] = sum;
                }
            }
        }
    } else {
        __syncthreads();
    }
}

constexpr uint32_t align16(uint32_t v) { return (v + 15u) & ~15u; }

// CTAs of this kernel resident at once when launched in clusters of ks
// (one CTA per SM; clusters are placed within a GPC, so for ks > 2 fewer
// than all SMs can be used), cached per device.
template <class C>
int resident_ctas(int ks, uint32_t smem) {
    static int cache[64][4] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    const int slot = ks == 1 ? 0 : (ks == 2 ? 1 : (ks == 4 ? 2 : 3));
    if (cache[dev][slot]) return cache[dev][slot];
    const int sms = device_sm_count();
    int n = sms;
    if constexpr (!C::kSplit) {
        if (ks > 1) return 0;
    } else if (ks > 1) {
        // the query needs the launch's shared-memory size to be allowed
        if (cudaFuncSetAttribute(qmv_stream_kernel<C, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cudaLaunchConfig_t q{};
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = ks;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        q.gridDim = dim3(sms / ks * ks);
        q.blockDim = dim3(kThreads);
        q.dynamicSmemBytes = smem;
        q.attrs = at;
        q.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, qmv_stream_kernel<C, true>, &q) != cudaSuccess) {
            cudaGetLastError();
            clusters = 0;
        }
        n = clusters * ks;
    }
    cache[dev][slot] = n;
    return n;
}

// Gather-mode arguments (decode MoE); see SPG.
struct GatherArgs {
    const int32_t* ids;
    int32_t* err;
    int pairs, xdiv, n_experts;
    const void* w2;   // GLU mode: the up bank (w is the gate bank)
    int act;
    float limit;
};

// ks: CTAs of a cluster that split K (1, 2, 4, 8; a divisor of the block
// count), each covering nblk / ks blocks of every row of the cluster's rows.
// ga: gather mode (ks = 1), n the rows of one expert.
template <class C>
int launch_stream(const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y, cudaStream_t st,
                  uint32_t img_tok, uint32_t xs_tok, int ks = 1, const GatherArgs* ga = nullptr) {
    SP p{};
    p.w = static_cast<const uint8_t*>(w);
    p.x = x;
    p.y = y;
    p.status = device_status_ptr();
    {
        int dev = 0;
        cudaGetDevice(&dev);
        p.strict = dev >= 0 && dev < 64 && g_strict_wait[dev] ? 1 : 0;
    }
    p.n = n;
    p.m = m;
    const int nblk_all = static_cast<int>(k / C::kVPB);
    if (ks < 1 || nblk_all % ks != 0 || (ga && ks != 1)) return KQ_ERR_UNSUPPORTED;
    p.ks = ks;
    p.nblk = nblk_all / ks;
    p.k = static_cast<int64_t>(p.nblk) * C::kVPB;
    p.row_bytes = static_cast<int64_t>(nblk_all) * C::kBPB;
    // rows that are not a 16-byte multiple: q6_K decode MoE only (each row's
    // copy starts at a 16-byte boundary, the row at its offset past it)
    const bool unaligned = p.row_bytes % 16 != 0;
    if (unaligned && !(ga && C::kBPB == 210)) return KQ_ERR_UNSUPPORTED;
    if (!unaligned && (static_cast<int64_t>(p.nblk) * C::kBPB) % 16 != 0) return KQ_ERR_UNSUPPORTED;   // slice copies
    p.img_tok = img_tok;
    p.xs_tok = xs_tok;
    const uint32_t optin = static_cast<uint32_t>(device_smem_optin());
    const int slots = resident_ctas<C>(ks, optin);
    // Shared-memory layout for at most nrg_max row groups per CTA (gather
    // mode: any number, in two reused slots); the total size, or 0 when it
    // does not fit.
    auto layout = [&](int nrg_max) -> uint32_t {
        if (!ga && nrg_max > kMaxGroups) return 0;
        // fixed part of the layout
        p.off_img = ga ? kGHdr : kHdr;
        p.off_xs = align16(p.off_img + m * img_tok);
        p.off_zero = align16(p.off_xs + m * xs_tok);
        p.off_part = align16(p.off_zero + C::kZero);
        p.off_xraw = p.off_part;   // the raw x copy is dead before any partial sum is written
        // split: two row-group slots of partial sums, reused in turn
        uint32_t part = static_cast<uint32_t>(ks > 1 || ga ? 2 : nrg_max) * kCW * kRows * m * 4;
        if (ga && ga->w2) part += kRows * m * 4;   // GLU: the gate sums of a row group
        // receive slots of the row groups this CTA owns: ceil(nrg / ks) x ks slices
        const uint32_t red = ks > 1 ? static_cast<uint32_t>(cdiv(nrg_max, ks) * ks) * kRows * m * 4 : 0;
        uint32_t xraw = static_cast<uint32_t>(m) * static_cast<uint32_t>(p.k) * 2;
        // q4_K can build its image from global memory when the raw copy would
        // crowd out the weight stages (not in gather mode, whose x rows are
        // gathered by the copy)
        p.x_global = (C::kSplit && p.off_part + xraw + red + 2u * kRows * 2048u > optin) ? 1 : 0;
        if (p.x_global && ga) return 0;
        if (p.x_global) xraw = 0;
        p.off_red = align16(p.off_part + (part > xraw ? part : xraw));
        p.off_stage = (p.off_red + red + 127u) & ~127u;
        // stage geometry: whole rows if two or more stages fit, else the fewest
        // equal row slices (a multiple of the item size, copies 16-byte sized)
        // that do; the deepest ring that fits
        const int ga_blk = C::kItemBlocks * (C::kBPB % 16 == 0 ? 1 : 8 / C::kItemBlocks);
        p.ns = 0;
        for (int s = 1; s <= 16 && p.ns == 0; ++s) {
            const int g = cdiv(cdiv(p.nblk, s), ga_blk) * ga_blk;
            if (s > 1 && g >= p.nblk) continue;
            const uint32_t rs = ((static_cast<uint32_t>(g) * C::kBPB + (unaligned ? 32u : 0u) + 127u) & ~127u) + 16;
            for (int ns = kMaxStages; ns >= 2; --ns) {
                if (p.off_stage + static_cast<uint32_t>(ns) * kRows * rs <= optin) {
                    p.ns = ns;
                    p.g = g;
                    p.rs = rs;
                    p.spr = cdiv(p.nblk, g);
                    break;
                }
            }
        }
        if (p.ns == 0) return 0;
        return p.off_stage + static_cast<uint32_t>(p.ns) * kRows * p.rs;
    };
    int grid = 0, launches = 1, vcount = 0;
    uint32_t total = 0;
    if (!ga) {
        const int64_t gmax = (n + 7) / 8;   // at least 8 rows per cluster
        int64_t ncl = slots / ks;
        if (ncl > gmax) ncl = gmax;
        if (ncl < 1) return KQ_ERR_UNSUPPORTED;
        grid = static_cast<int>(ncl) * ks;
        total = layout(cdiv(cdiv(n, ncl), kRows));
    } else {
        // Every CTA takes one virtual expert, any number of its rows; a
        // launch serves up to one virtual expert per CTA, and there are
        // enough launches for the most virtual experts the pairs can form.
        grid = slots;
        total = layout(2);
        vcount = grid;
        if (total == 0) return KQ_ERR_UNSUPPORTED;
        const int64_t vmax = std::min<int64_t>(ga->pairs, cdiv(ga->pairs, m) + std::min(ga->n_experts, ga->pairs));
        launches = static_cast<int>(cdiv(vmax, vcount));
    }
    if (total == 0) return KQ_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = total;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (use_pdl()) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (ks > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = ks;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (ga) {
        SPGLU g{};
        static_cast<SP&>(g) = p;
        g.ids = ga->ids;
        g.err = ga->err;
        g.pairs = ga->pairs;
        g.xdiv = ga->xdiv;
        g.n_experts = ga->n_experts;
        g.vcount = vcount;
        g.w2 = static_cast<const uint8_t*>(ga->w2);
        g.act = ga->act;
        g.limit = ga->limit;
        auto kg = qmv_stream_kernel<C, false, SPG>;
        auto kglu = qmv_stream_kernel<C, false, SPGLU>;
        cudaError_t e = ga->w2 ? cudaFuncSetAttribute(kglu, cudaFuncAttributeMaxDynamicSharedMemorySize, total)
                               : cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
        if (e != cudaSuccess) return record_cuda(e);
        for (int j = 0; j < launches; ++j) {
            g.vbase = j * vcount;
            const int rc = ga->w2 ? record_cuda(cudaLaunchKernelEx(&cfg, kglu, g))
                                  : record_cuda(cudaLaunchKernelEx(&cfg, kg, static_cast<const SPG&>(g)));
            if (rc) return rc;
        }
        return KQ_OK;
    }
    auto kernel = qmv_stream_kernel<C, false>;
    if constexpr (C::kSplit) {   // the K split is built for q4_K and q5_K
        if (ks > 1) kernel = qmv_stream_kernel<C, true>;
    } else if (ks > 1) {
        return KQ_ERR_UNSUPPORTED;
    }
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, total);
    if (e != cudaSuccess) return record_cuda(e);
    return record_cuda(cudaLaunchKernelEx(&cfg, kernel, p));
}

// q4_K keeps its inverse scales in one [block][16 tokens] byte table in the
// per-token X region: the per-token stride that makes m of them hold it.
uint32_t q4_inv_tok(int nblk, int m) { return align16(static_cast<uint32_t>(cdiv(nblk * 16, m))); }

}  // namespace

// Pipeline wait limit of the staged decode kernel on the current device
// (ns == 0: the default).
int set_stream_wait_limit(uint64_t ns) {
    const uint64_t v = ns ? ns : kWaitLimitNs;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64) g_strict_wait[dev] = v < kWaitLimitNs;
    return record_cuda(cudaMemcpyToSymbol(g_wait_ns, &v, sizeof(v)));
}

namespace {
// q4_K and q5_K (FIVE) on the staged kernel.  From M = 4 the activation
// image of a whole row crowds out the weight stages (and from M = 8 it no
// longer fits): K is then split over a cluster of 4 (else 2) CTAs, each
// covering a slice of at least 7 blocks.  Below M = 4 the split's cluster
// reduction costs more than it saves (measured).
template <bool FIVE>
int launch_q4family(const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y, cudaStream_t s) {
    const int nblk = static_cast<int>(k / 256);
    int ks = 1;
    if (m >= 4) {
        if (nblk % 4 == 0 && nblk / 4 >= 7) ks = 4;
        else if (nblk % 2 == 0 && nblk / 2 >= 7) ks = 2;
    }
    if (m == 1) {   // one row: the column form (scales in the epilogue)
        const int rc = launch_stream<Q4C<FIVE>>(w, n, k, x, 1, y, s, nblk * Q4C<FIVE>::kBlkImg, q4_inv_tok(nblk, 1));
        if (rc != KQ_ERR_UNSUPPORTED) return rc;
    }
    for (;;) {
        // per-token image stride 32 bytes past a multiple of 128: the 8
        // tokens of an MMA's B fragment then read disjoint banks
        uint32_t it = (nblk / ks) * Q4<1, FIVE>::kBlkImg;
        it += (32u - it % 128u + 128u) % 128u;
        const int rc = m <= 8 ? launch_stream<Q4<1, FIVE>>(w, n, k, x, m, y, s, it, q4_inv_tok(nblk / ks, m), ks)
                              : launch_stream<Q4<2, FIVE>>(w, n, k, x, m, y, s, it, q4_inv_tok(nblk / ks, m), ks);
        if (rc != KQ_ERR_UNSUPPORTED || ks == 1) return rc;
        ks = 1;
    }
}
}  // namespace

// Staged qmv for the shapes it covers; KQ_ERR_UNSUPPORTED otherwise (the
// caller then takes the general kernel).
int launch_qmv_stream(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int m, float* y,
                      cudaStream_t s) {
    switch (type) {
    case KQ_Q8_0: {
        const int nblk = static_cast<int>(k / 32);
        if (m > 2 || nblk % 8 != 0) return KQ_ERR_UNSUPPORTED;
        const uint32_t it = (nblk / 8) * Q8<1>::kItemImg, xt = nblk * 4;
        return m == 1 ? launch_stream<Q8<1>>(w, n, k, x, m, y, s, it, xt) : launch_stream<Q8<2>>(w, n, k, x, m, y, s, it, xt);
    }
    case KQ_Q6_K: {
        const int nblk = static_cast<int>(k / 256);
        if (m > 2 || nblk % 8 != 0) return KQ_ERR_UNSUPPORTED;
        const uint32_t it = nblk * Q6<1>::kBlkImg, xt = nblk * 16 * 4;
        return m == 1 ? launch_stream<Q6<1>>(w, n, k, x, m, y, s, it, xt) : launch_stream<Q6<2>>(w, n, k, x, m, y, s, it, xt);
    }
    case KQ_Q4_K: return launch_q4family<false>(w, n, k, x, m, y, s);
    case KQ_Q5_K: return launch_q4family<true>(w, n, k, x, m, y, s);
    case KQ_Q4_0: {
        const int nblk = static_cast<int>(k / 32);
        if (m > 2 || nblk % 8 != 0) return KQ_ERR_UNSUPPORTED;
        const uint32_t it = (nblk / 8) * Q40<1>::kItemImg, xt = nblk * 4;
        return m == 1 ? launch_stream<Q40<1>>(w, n, k, x, m, y, s, it, xt) : launch_stream<Q40<2>>(w, n, k, x, m, y, s, it, xt);
    }
    default: return KQ_ERR_UNSUPPORTED;
    }
}

// Decode MoE product on the staged kernel: at most m_cap pairs of one expert
// per virtual expert (q8_0 and q6_K take up to 2 activation rows, q4_K up to
// 16 while the activation image fits; fewer when shared memory requires).
int launch_gather_qmv(int type, const void* w_bank, const void* w_bank2, int act, float limit, int n_experts,
                      int64_t n, int64_t k, const uint16_t* x, int xdiv, const int32_t* ids, int pairs, int m_cap,
                      float* y, int32_t* err_flag, cudaStream_t s) {
    GatherArgs ga{ids, err_flag, pairs, xdiv, n_experts, w_bank2, act, limit};
    const int nblk = static_cast<int>(k / (type == KQ_Q8_0 || type == KQ_Q4_0 ? 32 : 256));
    int rc = KQ_ERR_UNSUPPORTED;
    switch (type) {
    case KQ_Q8_0: {
        if (nblk % 8 != 0) return KQ_ERR_UNSUPPORTED;
        const uint32_t it = (nblk / 8) * Q8<1>::kItemImg, xt = nblk * 4;
        rc = m_cap >= 2 ? launch_stream<Q8<2>>(w_bank, n, k, x, 2, y, s, it, xt, 1, &ga) : KQ_ERR_UNSUPPORTED;
        if (rc == KQ_ERR_UNSUPPORTED) rc = launch_stream<Q8<1>>(w_bank, n, k, x, 1, y, s, it, xt, 1, &ga);
        return rc;
    }
    case KQ_Q6_K: {   // any k % 256 == 0 (rows that are not a 16-byte multiple included)
        const uint32_t it = nblk * Q6<1>::kBlkImg, xt = nblk * 16 * 4;
        rc = m_cap >= 2 ? launch_stream<Q6<2>>(w_bank, n, k, x, 2, y, s, it, xt, 1, &ga) : KQ_ERR_UNSUPPORTED;
        if (rc == KQ_ERR_UNSUPPORTED) rc = launch_stream<Q6<1>>(w_bank, n, k, x, 1, y, s, it, xt, 1, &ga);
        return rc;
    }
    case KQ_Q4_K:
    case KQ_Q5_K: {
        uint32_t it = nblk * Q4<1>::kBlkImg;
        it += (32u - it % 128u + 128u) % 128u;
        for (int m = m_cap < 16 ? m_cap : 16; m >= 1; --m) {
            if (m == 1) {   // one row per virtual expert: the column form
                const uint32_t it1 = nblk * Q4C<>::kBlkImg;
                rc = type == KQ_Q4_K ? launch_stream<Q4C<false>>(w_bank, n, k, x, 1, y, s, it1, q4_inv_tok(nblk, 1), 1, &ga)
                                     : launch_stream<Q4C<true>>(w_bank, n, k, x, 1, y, s, it1, q4_inv_tok(nblk, 1), 1, &ga);
                if (rc != KQ_ERR_UNSUPPORTED) return rc;
            }
            if (type == KQ_Q4_K)
                rc = m <= 8 ? launch_stream<Q4<1>>(w_bank, n, k, x, m, y, s, it, q4_inv_tok(nblk, m), 1, &ga)
                            : launch_stream<Q4<2>>(w_bank, n, k, x, m, y, s, it, q4_inv_tok(nblk, m), 1, &ga);
            else
                rc = m <= 8 ? launch_stream<Q4<1, true>>(w_bank, n, k, x, m, y, s, it, q4_inv_tok(nblk, m), 1, &ga)
                            : launch_stream<Q4<2, true>>(w_bank, n, k, x, m, y, s, it, q4_inv_tok(nblk, m), 1, &ga);
            if (rc != KQ_ERR_UNSUPPORTED) return rc;
        }
        return rc;
    }
    case KQ_Q4_0: {
        if (nblk % 8 != 0) return KQ_ERR_UNSUPPORTED;
        const uint32_t it = (nblk / 8) * Q40<1>::kItemImg, xt = nblk * 4;
        rc = m_cap >= 2 ? launch_stream<Q40<2>>(w_bank, n, k, x, 2, y, s, it, xt, 1, &ga) : KQ_ERR_UNSUPPORTED;
        if (rc == KQ_ERR_UNSUPPORTED) rc = launch_stream<Q40<1>>(w_bank, n, k, x, 1, y, s, it, xt, 1, &ga);
        return rc;
    }
    default: return KQ_ERR_UNSUPPORTED;
    }
}

}  // namespace kq
