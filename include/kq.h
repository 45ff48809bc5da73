/*
 * kq.h - C ABI of the B200 (sm_100a) library for matrix products with GGUF
 * block-quantized weights: y = x . W^T where W is stored as q4_K, q6_K,
 * q8_0, q5_K or q4_0 wire blocks, plus the encoder that writes such blocks,
 * the MoE routing helpers and the MoE epilogues.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument is a DEVICE pointer (memory the caller allocated on
 *    the current CUDA device, e.g. through torch), unless a comment says
 *    "host".  The library allocates no device memory on any call below and
 *    keeps no state other than the lazily created per-device kernel attribute
 *    settings.  The caller owns every buffer.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every compute call is asynchronous on that stream: it only
 *    validates its arguments on the host and enqueues kernels.  No call
 *    synchronizes with the device.
 *  - W is the codec's wire bytes for an [n, k] matrix, row-major, rows
 *    contiguous: row r starts at byte r * row_bytes with
 *    row_bytes = (k / values_per_block) * bytes_per_block.  This is the
 *    layout the mlx-kquant `quantized_matmul` op takes with transpose=True
 *    (bindings.cpp docstring: the weight operand is uint8 wire bytes, N rows
 *    of K values in that mode), the README's product x @ dequant(w).T.
 *  - Activations x are bfloat16 [m, k] row-major (passed as uint16_t bit
 *    patterns), any finite value.  The tensor-core decode kernels
 *    (kq_qmv, kq_gather_qmv, kq_moe_glu_gather) scale each run of
 *    activations (a block, a 16-value run of q6_K, or a row slice) by a
 *    power of two taken from its largest magnitude, round it to binary16
 *    and apply the inverse scale to the fp32 sums, so their relative error
 *    does not depend on the magnitude of x.  Codes enter the MMA centred on
 *    their format's offset (q8_0 code, q4_0 code - 8, q6_K code - 32,
 *    exactly), so a weight that decodes to 0 contributes exactly 0 however
 *    large its activation.  Within one run, values below about 2^-29 of the
 *    run's largest magnitude fall into binary16's subnormal range and lose
 *    relative precision.  A non-finite activation sets KQ_DEV_X_RANGE (its
 *    outputs are then NaN or infinite).  qmm/gather use bf16 as is, and the
 *    exact fp32 kernel (q4_0 at m >= 3) widens it to fp32 exactly.
 *  - Outputs y are fp32 [m, n] row-major.
 *  - Return value: a kq_status.  A non-zero status means nothing was enqueued
 *    (argument errors) or that the CUDA launch failed (KQ_ERR_CUDA; the
 *    cudaError_t is available from kq_last_cuda_error()).  Nothing throws.
 *  - Alignment: W, x, y and out must be 16-byte aligned, else
 *    KQ_ERR_ALIGNMENT.  Weight rows whose byte length is not a multiple of 16
 *    (q6_K with k / 256 not a multiple of 8) are accepted everywhere, on
 *    slower copy paths; kq_qmm / kq_gather_qmm need k % 256 == 0
 *    (KQ_ERR_UNSUPPORTED otherwise).
 *  - `k` must be a multiple of the codec's values_per_block, as the reference
 *    requires (bindings.cpp `dequantize`: the last dimension holds whole
 *    blocks), and at most 2^31 - 1; otherwise KQ_ERR_INVALID_ARG.
 *  - Environment (read once per process; A/B levers, not needed in use):
 *    KQ_NO_PDL=1 launches the decode kernels (kq_qmv, kq_gather_qmv,
 *    kq_moe_glu_gather) without programmatic dependent launch, so a launch
 *    no longer overlaps its start-up with the end of the previous kernel on
 *    the stream (the kernels and their results are unchanged);
 *    KQ_QMM_1SM=1 runs kq_qmm / kq_gather_qmm on single CTAs (128 weight
 *    rows per unit, MMA M = 128) instead of CTA pairs, a performance lever
 *    that the test suite does not cover.
 */
#ifndef KQ_H
#define KQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ggml / GGUF type ids of the supported codecs. */
typedef enum {
    KQ_Q4_0 = 2,   /* 32 values, 18 bytes: fp16 d, 16 B of 4-bit codes (q-8) */
    KQ_Q8_0 = 8,   /* 32 values, 34 bytes: fp16 d, 32 x int8               */
    KQ_Q4_K = 12,  /* 256 values, 144 bytes: fp16 d, fp16 dmin, 12 B packed
                      6-bit scale/min codes, 128 B of 4-bit codes             */
    KQ_Q5_K = 13,  /* 256 values, 176 bytes: as q4_K plus 32 B of fifth bits
                      (qh) before the 128 B of 4-bit codes                    */
    KQ_Q6_K = 14   /* 256 values, 210 bytes: 128 B low nibbles, 64 B high
                      2-bit pairs, 16 x int8 scales, fp16 d                   */
} kq_type;

typedef enum {
    KQ_OK = 0,
    KQ_ERR_INVALID_ARG = 1,   /* bad size, null pointer, bad capacity       */
    KQ_ERR_UNSUPPORTED = 2,   /* unknown codec id                           */
    KQ_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned           */
    KQ_ERR_CUDA = 4,          /* a CUDA runtime call failed                 */
    KQ_ERR_DEVICE_DATA = 5    /* reserved for device-side data errors       */
} kq_status;

/* Bits the kernels OR into a caller's int32 device error word (err_flag).
 * The caller zeroes the word before the call and reads it afterwards. */
#define KQ_DEV_BAD_EXPERT   0x1   /* tile or routing id >= n_experts           */
#define KQ_DEV_BAD_ROWS     0x2   /* tile num_rows == 0 or > 64                */
#define KQ_DEV_BAD_RANGE    0x4   /* tile rows past `rows`, count > cap        */
#define KQ_DEV_UNSORTED     0x8   /* expert ids not ascending                  */
#define KQ_DEV_TIMEOUT      0x10  /* a bounded pipeline wait ran out            */
#define KQ_DEV_TOO_MANY     0x20  /* reserved: not set by this version         */
#define KQ_DEV_X_RANGE      0x40  /* an activation is infinite or NaN         */

/* Block geometry of a codec (host only).  Returns KQ_OK or
 * KQ_ERR_UNSUPPORTED.  Source: mlx-kquant README, "Codec reference" table. */
int kq_block_info(int type, int* values_per_block, int* bytes_per_block);

/* Static, thread-safe description of a kq_status value. */
const char* kq_status_string(int status);

/* cudaError_t of the most recent KQ_ERR_CUDA on the calling host thread. */
int kq_last_cuda_error(void);

/* Library-wide device status word: bits KQ_DEV_* set by kernels that have no
 * err_flag argument (kq_qmv, kq_qmm).  Host call, synchronous: it first waits
 * for all work on the current device (every stream, cudaDeviceSynchronize),
 * then reads the word.  `clear` != 0 resets the word after reading.  The word
 * is shared by every call and stream of the device: a bit cannot be traced to
 * the call that set it. */
int kq_read_device_status(int32_t* host_status, int clear);

/*
 * kq_set_wait_limit - time limit, in ns, of every pipeline wait of the staged
 * decode kernel (kq_qmv on the shapes it covers: m <= 2 for q8_0 / q6_K /
 * q4_0, q4_K / q5_K while their activation image fits; kq_gather_qmv,
 * kq_moe_glu_gather) on the current device, for launches made after the
 * call; ns <= 0 restores the default of 2 s.  Host call, synchronous.  A wait
 * that runs out sets KQ_DEV_TIMEOUT in the library status word and the kernel
 * winds down (letting its own copies land) without finishing: its outputs
 * are then incomplete.  Under a limit shorter than the default the first
 * wait for the activation copy only tests it, so that wait runs out unless
 * the copy has landed.  A short limit exists so that fault-handling tests
 * can make a wait run out on purpose; production code has no reason to call
 * it.  No counterpart on the pages (the failure handling of this library).
 */
int kq_set_wait_limit(int64_t ns);

/*
 * kq_dequantize - decode wire bytes to fp32, bit-exactly (all five codecs).
 * mlx-kquant bindings.cpp, `dequantize` (wire bytes in, a float array out);
 * hanzo-ml quantized/mod.rs, `QTensor::dequantize` (decodes to f32 through
 * its to_float routine).
 *   w    [n_rows, row_bytes] wire bytes
 *   out  [n_rows, k] fp32; element (r, c) = decode of value c of row r,
 *        computed in fp32 as (d*sc)*q - (dmin*m) (q4_K, q5_K), (d*sc)*q
 *        (q6_K), d*q (q8_0, q4_0), each operation rounded separately (no FMA).
 * n_rows >= 0; n_rows == 0 enqueues nothing.
 */
int kq_dequantize(int type, const void* w, int64_t n_rows, int64_t k, float* out, void* stream);

/*
 * kq_quantize - encode fp32 weights into wire bytes (the step before the
 * products).  mlx-kquant bindings.cpp, `quantize` (float weights in, wire
 * bytes out; the last dimension holds whole blocks); hanzo-ml
 * quantized/mod.rs `QTensor::quantize`.
 *   w    [n_rows, k] fp32, finite (scales must stay in binary16 range)
 *   out  [n_rows, row_bytes] wire bytes
 * The pages give no encoding search; this one is fixed step by step in fp32:
 * q8_0 d = max|x|/127, codes round(x * (1/d)) (ggml's rule, identical bytes);
 * q4_K per 32 values scale (max - min(0, min))/15 and min -min(0, min x),
 * 6-bit codes against binary16 d = max scale/63 and dmin = max min/63,
 * codes round((x + dmin*m)/(d*sc)); q6_K per 16 values scale max|x|/31, int8
 * codes against binary16 d = max scale/127, codes round(x/(d*sc)) + 32.
 * Rounding is to nearest with ties away from zero.  The importance matrix
 * of the pages' op is not supported.  n_rows == 0 enqueues nothing.
 */
int kq_quantize(int type, const float* w, int64_t n_rows, int64_t k, void* out, void* stream);

/*
 * kq_qmv - decode-shaped product y = x . W^T for 1 <= m <= 16 rows of x.
 * All five codecs take the staged tensor-core kernel (q8_0, q6_K, q4_0 for
 * m <= 2; q4_K, q5_K for every m).  q8_0 and q6_K at m >= 3 take the
 * general tensor-core kernel; q4_0 at m >= 3 takes a plainer one (every
 * weight decoded exactly to fp32 and multiplied by the activations with
 * fp32 FMAs).  q4_0 needs k % 256 == 0.
 * mlx-kquant bindings.cpp, `quantized_matmul` (x @ dequant(w), transpose=True);
 * README "How it works": small row counts take a weight-read-amortizing
 * kernel (`verify_qmv`).  Every weight byte is read once for all m rows.
 *   w [n, row_bytes], x [m, k] bf16, y [m, n] fp32.
 * Arithmetic: quantization codes and integer scale products are exact in the
 * tensor-core operands, activations (scaled by a power of two per row) are
 * rounded to binary16, accumulation is fp32.  Results are deterministic (no
 * atomics).
 * m outside 1..16 -> KQ_ERR_INVALID_ARG.
 */
int kq_qmv(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m,
           float* y, void* stream);

/*
 * kq_qmm - prefill-shaped product y = x . W^T for any m >= 1 on the
 * tcgen05 tensor cores: W tiles are dequantized to bf16 in shared memory,
 * x is read as bf16, products accumulate in fp32 in tensor memory.
 * mlx-kquant bindings.cpp `quantized_matmul`; README "Performance"
 * (single-pass matmul on the tensor units).
 *   w [n, row_bytes], x [m, k] bf16, y [m, n] fp32.
 * k % 256 == 0 (else KQ_ERR_UNSUPPORTED); m, n <= 2^31 - 1 (else
 * KQ_ERR_INVALID_ARG).  q6_K rows that are not a 16-byte multiple are read
 * through a flat byte view whose coordinates are 32-bit: the weight bytes
 * plus two tiles of rows must stay below 2^31 bytes (else
 * KQ_ERR_UNSUPPORTED; kq_gather_qmm likewise for the whole bank).
 */
int kq_qmm(int type, const void* w, int64_t n, int64_t k, const uint16_t* x, int64_t m,
           float* y, void* stream);

/*
 * kq_moe_sort - group routed (token, slot) pairs by expert for a sorted MoE
 * prefill: a stable counting sort by expert id, plus the row gather of x.
 * mlx-kquant README "Performance" (sorted MoE prefill batches route to a
 * per-expert-segment GEMM) and bindings.cpp `gather_qmm_seg` (its rows come
 * in already grouped by expert).
 *   topk_ids    [n_tokens, top_k] int32 expert ids, each in [0, n_experts)
 *   x           [n_tokens, k] bf16 (may be NULL when x_sorted is NULL)
 *   sorted_ids  [n_tokens*top_k] uint32 out: expert id of sorted row r
 *   sorted_pair [n_tokens*top_k] int32 out: token*top_k + slot of sorted row r
 *   inv_order   [n_tokens*top_k] int32 out (nullable): the sorted row of pair
 *               token*top_k + slot (the inverse permutation, as
 *               kq_gather_mix takes it); -1 for a pair with a bad id
 *   x_sorted    [n_tokens*top_k, k] bf16 out (nullable): x[sorted_pair/top_k]
 *   err_flag    int32 device word (nullable): KQ_DEV_BAD_EXPERT on bad ids
 * Pairs with equal expert id keep (token, slot) order.  1 <= n_experts <= 256,
 * n_tokens*top_k <= 2^30, and with x_sorted: x non-NULL, k a positive
 * multiple of 8 (16-byte rows) of at most 2^31 - 1; else KQ_ERR_INVALID_ARG.
 */
int kq_moe_sort(const int32_t* topk_ids, int64_t n_tokens, int32_t top_k, int32_t n_experts,
                const uint16_t* x, int64_t k, uint32_t* sorted_ids, int32_t* sorted_pair,
                int32_t* inv_order, uint16_t* x_sorted, int32_t* err_flag, void* stream);

/*
 * kq_expert_tile_map - build the tile map of a segment-walking gather GEMM on
 * the device, without a host round trip.
 * mlx-kquant bindings.cpp, `expert_tile_map`: tile each expert segment of
 * the ascending id array into 64-row tiles (expert, row_start, num_rows)
 * where only the last tile of a segment can be partial, plus the valid-tile
 * count.  Tile order is unspecified (here: grouped by expert, ascending).
 * Slots past the count are left untouched.
 *   sorted_ids [rows] uint32 ascending expert ids
 *   map        [cap, 3] uint32 out,  count [1] uint32 out
 *   cap must be >= ceil(rows / 64) + n_experts, else KQ_ERR_INVALID_ARG.
 *   err_flag (nullable): KQ_DEV_BAD_EXPERT (id >= n_experts),
 *   KQ_DEV_UNSORTED (ids not ascending; the map is then unspecified).
 */
int kq_expert_tile_map(const uint32_t* sorted_ids, int64_t rows, int32_t n_experts,
                       uint32_t* map, int64_t cap, uint32_t* count, int32_t* err_flag,
                       void* stream);

/*
 * kq_gather_qmm - MoE segment GEMM: for every valid tile (e, start, n) of the
 * map, y[r, :] = x_sorted[r, :] . dequant(W[e])^T for start <= r < start + n.
 * mlx-kquant bindings.cpp, `gather_qmm_seg`: "valid tiles never span experts
 * and must cover every x row exactly once (uncovered output rows are left
 * unwritten)"; num_rows <= 64.  Each CTA pair owns one (expert, 256 weight
 * rows) unit at a time and streams up to four of that expert's tiles through
 * the tensor cores, so each expert weight tile is decoded once per four map
 * tiles.  Any number of tiles:
 * the map is taken in windows of 1024 slots, one kernel launch per window
 * (ceil(cap / 1024) launches; a window past the device-side count has no
 * work), and an expert's tiles are grouped in map order within a window.
 *   w_bank [n_experts, n, row_bytes], x_sorted [rows, k] bf16,
 *   map [cap, 3], count [1] (device), y [rows, n] fp32.
 *   err_flag (nullable): tiles with e >= n_experts (KQ_DEV_BAD_EXPERT),
 *   num_rows 0 or > 64 (KQ_DEV_BAD_ROWS), rows past `rows` or count > cap
 *   (KQ_DEV_BAD_RANGE) are skipped and flagged; they never fault.
 */
int kq_gather_qmm(int type, const void* w_bank, int32_t n_experts, int64_t n, int64_t k,
                  const uint16_t* x_sorted, int64_t rows, const uint32_t* map,
                  const uint32_t* count, int64_t cap, float* y, int32_t* err_flag,
                  void* stream);

/*
 * kq_gather_qmv - decode-shaped MoE product with one output row per
 * (token, slot) pair: y[p, :] = x[row(p), :] . dequant(W[ids[p]])^T for the
 * p = token*top_k + slot pairs of ids [n_tokens, top_k].
 * mlx-kquant bindings.cpp, `gather_qmv_kq` (a matvec over a stack of
 * expert weight matrices, as in the MoE down projection, with its own
 * activation row for every expert slot: x [T, R, K], w (n_experts, N,
 * bytes_per_row), indices [T, R], output [T, R, N]).  With x_per_token != 0 x holds one row per token,
 * row(p) = p / top_k, which is the gate/up product of `moe_glu_gather_kq`
 * before its GLU; else row(p) = p.
 *   w_bank [n_experts, n, row_bytes], x [n_tokens*top_k or n_tokens, k] bf16,
 *   ids [n_tokens*top_k] int32, y [n_tokens*top_k, n] fp32.
 * No host round trip: the pairs are grouped by expert on the device and each
 * routed expert's weights are read once for all of its pairs (in batches of
 * up to 2 (q8_0, q6_K, q4_0) or 16 (q4_K, q5_K) activation rows; an expert
 * with more pairs than a batch is streamed once per batch).  Arithmetic as
 * kq_qmv.  All five codecs.
 * Limits: 1 <= n_experts <= 256, 1 <= n_tokens*top_k <= 8192; k % 256 == 0,
 * else KQ_ERR_UNSUPPORTED (q6_K rows that are not a 16-byte multiple, k / 256
 * not a multiple of 8, take a slower copy path: each row is staged from the
 * 16-byte boundary below it and decoded at its own byte offset).
 *   err_flag (nullable): KQ_DEV_BAD_EXPERT for ids outside [0, n_experts);
 *   the rows of those pairs are left unwritten.
 */
int kq_gather_qmv(int type, const void* w_bank, int32_t n_experts, int64_t n, int64_t k,
                  const uint16_t* x, int32_t x_per_token, const int32_t* ids, int64_t n_tokens,
                  int32_t top_k, float* y, int32_t* err_flag, void* stream);

/* GLU activations of kq_moe_glu_gather. */
#define KQ_ACT_SILU        0   /* silu(g) * u, silu(g) = g / (1 + exp(-g))          */
#define KQ_ACT_GELU_TANH   1   /* gelu(g) * u, gelu in its tanh approximation:
                                  0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))   */
#define KQ_ACT_SILU_LIMIT  2   /* silu(min(g, limit)) * clamp(u, -limit, limit)     */

/*
 * kq_moe_glu_gather - decode MoE gate/up products and their GLU in one
 * dispatch: out[p, :] = act(x[t, :] . dequant(Wg[e])^T, x[t, :] . dequant(Wu[e])^T)
 * for the pairs p = t*top_k + s of ids [n_tokens, top_k], e = ids[p].
 * mlx-kquant bindings.cpp, `moe_glu_gather_kq` (the gate and up matvecs of
 * an expert load each activation once, and act(g) * u is applied before the
 * dispatch ends; act 'silu' (default), 'gelu' (tanh approx),
 * 'silu_limit' (requires limit > 0); x [T, K], gate_w and up_w
 * (n_experts, N, bytes_per_row), indices [T, R], output [T, R, N]).
 * Each routed expert's gate and up rows are streamed once; every CTA takes
 * 16 gate rows, then the same 16 up rows, and applies act in fp32 to the
 * two fp32 sums (arithmetic of the sums as kq_qmv).
 *   gate_bank, up_bank [n_experts, n, row_bytes], x [n_tokens, k] bf16,
 *   ids [n_tokens*top_k] int32, out [n_tokens*top_k, n] fp32.
 *   act one of KQ_ACT_*; KQ_ACT_SILU_LIMIT needs limit > 0.
 * Limits and errors as kq_gather_qmv.
 */
int kq_moe_glu_gather(int type, const void* gate_bank, const void* up_bank, int32_t n_experts,
                      int64_t n, int64_t k, const uint16_t* x, const int32_t* ids, int64_t n_tokens,
                      int32_t top_k, int32_t act, float limit, float* out, int32_t* err_flag,
                      void* stream);

/*
 * kq_gather_mix - unsort and score mix of expert-sorted MoE outputs:
 * out[t, :] = sum over s = 0 .. top_k-1 of scores[t, s] * y[inv_order[t*top_k + s], :].
 * mlx-kquant bindings.cpp, `gather_mix` (fused unsort and score mix for
 * sorted-prefill MoE, f32 accumulation, N a multiple of 4); hanzo-ml
 * quantized/mod.rs `moe_combine` (the per-slot outputs reduced by the router
 * weights).  fp32 throughout, in a fixed order: each product rounded to
 * fp32, then added to the running sum (which starts at 0), slots ascending;
 * no fused multiply-add, so results are bit-reproducible.
 *   y [rows, n] fp32 (e.g. kq_gather_qmm's output), inv_order
 *   [n_tokens*top_k] int32 (kq_moe_sort's), scores [n_tokens, top_k] fp32,
 *   out [n_tokens, n] fp32.  n % 4 == 0, n <= 67107840 (4 x 256 x 65535)
 *   and 1 <= top_k <= 64, else KQ_ERR_INVALID_ARG.
 *   err_flag (nullable): KQ_DEV_BAD_RANGE for an inv_order entry outside
 *   [0, rows); that term is left out of the sum.
 */
int kq_gather_mix(const float* y, int64_t rows, int64_t n, const int32_t* inv_order,
                  const float* scores, int64_t n_tokens, int32_t top_k, float* out,
                  int32_t* err_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KQ_H */
