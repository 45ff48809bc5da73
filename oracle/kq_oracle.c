/*
 * CPU oracle for GGUF block-quantized weights (q4_K, q6_K, q8_0).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; it is compiled with
 * gcc -O2 -ffp-contract=off (no fused multiply-add, no fast-math) so every
 * floating-point operation below is rounded exactly where it is written.
 *
 * What it computes, and where that is stated:
 *  - dequantize: wire bytes -> float ("dequantize" op docstring, mlx-kquant
 *    bindings.cpp; "QTensor::dequantize -> to_float into f32", hanzo-ml
 *    quantized/mod.rs).  Block sizes: mlx-kquant README, "Codec reference"
 *    table (q4_k 256 values / 144 B, q6_k 256 / 210 B, q8_0 32 / 34 B).  The
 *    field layout inside a block is not printed on the pages; the pages say
 *    the codecs are ggml's (README, "Acknowledgements") and that the scalar
 *    decoder is bit-exact against the gguf.quants reference (README, "How it
 *    works").  The layout decoded here is ggml's public block format; the
 *    test suite pins it against the installed gguf.quants.dequantize and
 *    against hand-built blocks with closed-form values.
 *  - matmul: y = x @ dequant(w).T with w laid out [N, K] ("quantized_matmul"
 *    docstring, transpose=True, mlx-kquant bindings.cpp; README "Using
 *    K-quant ops directly").  The reference value accumulates in fp64; an
 *    fp32 sequential-k variant is provided for timing only.
 *
 * Parity pins for every function live in tests/test_oracle.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define T_Q8_0 8
#define T_Q4_K 12
#define T_Q6_K 14

/* IEEE-754 binary16 -> binary32, exact for every input (subnormals, +-0,
 * inf; NaN stays NaN).  Written from the binary16 definition: value =
 * (-1)^s * 2^(e-15) * (1 + f/1024) for 1 <= e <= 30, and
 * (-1)^s * 2^-14 * (f/1024) for e = 0. */
static float half_to_float(uint16_t h) {
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    float v;
    if (e == 0)
        v = ldexpf((float)f, -24);               /* f * 2^-24, exact */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexpf((float)(f + 1024), e - 25);   /* (1024 + f) * 2^(e-25) */
    return s ? -v : v;
}

static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* bfloat16 bits -> float: the upper half of a binary32. */
static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* q4_K: the 12 bytes s[0..11] hold eight 6-bit scale codes sc[j] and eight
 * 6-bit min codes m[j].  For j < 4 the low six bits of s[j] and s[j+4] are
 * sc[j] and m[j].  For j >= 4 the low nibble of s[j+4] gives the low four
 * bits of sc[j] and its high nibble the low four bits of m[j]; the two top
 * bits of s[j-4] and of s[j] supply bits 4..5 of sc[j] and m[j]. */
static void q4k_scale_min(const uint8_t* s, int j, int* sc, int* m) {
    if (j < 4) {
        *sc = s[j] & 63;
        *m = s[j + 4] & 63;
    } else {
        *sc = (s[j + 4] & 0x0f) | ((s[j - 4] >> 6) << 4);
        *m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

/* q4_K block (144 B): d (fp16) at 0, dmin (fp16) at 2, packed scales at 4,
 * 128 bytes of nibbles at 16.  Value 64c + l (c = 0..3, l = 0..31) is the low
 * nibble of qs[32c + l] (sub-block 2c); value 64c + 32 + l is its high
 * nibble (sub-block 2c + 1).  y = (d*sc)*q - (dmin*m), each product and the
 * difference rounded to fp32. */
static void dq_q4k(const uint8_t* b, float* out) {
    float d = half_to_float(rd16(b));
    float dmin = half_to_float(rd16(b + 2));
    const uint8_t* s = b + 4;
    const uint8_t* qs = b + 16;
    for (int j = 0; j < 8; ++j) {
        int sc, m;
        q4k_scale_min(s, j, &sc, &m);
        float dl = d * (float)sc;
        float ml = dmin * (float)m;
        int c = j / 2, hi = j % 2;
        for (int l = 0; l < 32; ++l) {
            int byte = qs[32 * c + l];
            int q = hi ? (byte >> 4) : (byte & 15);
            float t = dl * (float)q;
            out[64 * c + 32 * hi + l] = t - ml;
        }
    }
}

/* q6_K block (210 B): ql[128] at 0, qh[64] at 128, int8 scales[16] at 192,
 * d (fp16) at 208.  Value v = 128h + 32t + l (h = 0..1, t = 0..3,
 * l = 0..31): low four bits = nibble (t >> 1) of ql[64h + 32(t & 1) + l],
 * high two bits = bits 2t..2t+1 of qh[32h + l]; q = code - 32; the scale is
 * scales[v / 16].  y = (d*sc)*q, each product rounded to fp32. */
static void dq_q6k(const uint8_t* b, float* out) {
    const uint8_t* ql = b;
    const uint8_t* qh = b + 128;
    const int8_t* sc = (const int8_t*)(b + 192);
    float d = half_to_float(rd16(b + 208));
    for (int v = 0; v < 256; ++v) {
        int h = v / 128, t = (v % 128) / 32, l = v % 32;
        int lo = (ql[64 * h + 32 * (t & 1) + l] >> (4 * (t >> 1))) & 15;
        int hi = (qh[32 * h + l] >> (2 * t)) & 3;
        int q = (lo | (hi << 4)) - 32;
        float dl = d * (float)sc[v / 16];
        out[v] = dl * (float)q;
    }
}

/* q8_0 block (34 B): d (fp16) at 0, 32 int8 codes at 2.  y = d*q. */
static void dq_q8_0(const uint8_t* b, float* out) {
    float d = half_to_float(rd16(b));
    const int8_t* qs = (const int8_t*)(b + 2);
    for (int i = 0; i < 32; ++i) out[i] = d * (float)qs[i];
}

int oracle_block_info(int type, int* values, int* bytes) {
    switch (type) {
    case T_Q4_K: *values = 256; *bytes = 144; return 0;
    case T_Q6_K: *values = 256; *bytes = 210; return 0;
    case T_Q8_0: *values = 32; *bytes = 34; return 0;
    default: return -1;
    }
}

static void dq_row(int type, const uint8_t* row, int64_t k, float* out) {
    int vpb, bpb;
    oracle_block_info(type, &vpb, &bpb);
    for (int64_t b = 0; b < k / vpb; ++b) {
        const uint8_t* blk = row + b * bpb;
        float* o = out + b * vpb;
        if (type == T_Q4_K) dq_q4k(blk, o);
        else if (type == T_Q6_K) dq_q6k(blk, o);
        else dq_q8_0(blk, o);
    }
}

/* W [n_rows, k/vpb*bpb] wire bytes -> out [n_rows, k] fp32. */
int oracle_dequantize(int type, const uint8_t* w, int64_t n_rows, int64_t k, float* out) {
    int vpb, bpb;
    if (oracle_block_info(type, &vpb, &bpb) || k % vpb) return -1;
    int64_t rb = k / vpb * bpb;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) dq_row(type, w + r * rb, k, out + r * k);
    return 0;
}

/* y[m, n] = sum_k x[m, k] * W[n, k], x given as bf16 bits [m, k], W decoded
 * exactly to fp32 and both promoted to fp64; fp64 accumulation in k order.
 * absdot[m, n] = sum_k |x[m, k] * W[n, k]| (the scale the tolerance uses).
 * absdot may be NULL. */
int oracle_matmul_f64(int type, const uint8_t* w, int64_t n, int64_t k, const uint16_t* x,
                      int64_t m, double* y, double* absdot) {
    int vpb, bpb;
    if (oracle_block_info(type, &vpb, &bpb) || k % vpb) return -1;
    int64_t rb = k / vpb * bpb;
    double* xd = (double*)malloc(sizeof(double) * (size_t)(m * k));
    if (!xd) return -2;
    for (int64_t i = 0; i < m * k; ++i) xd[i] = (double)bf16_to_float(x[i]);
    int fail = 0;
#pragma omp parallel
    {
        float* wr = (float*)malloc(sizeof(float) * (size_t)k);
        if (!wr) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t j = 0; j < n; ++j) {
                dq_row(type, w + j * rb, k, wr);
                for (int64_t i = 0; i < m; ++i) {
                    const double* xr = xd + i * k;
                    double acc = 0.0, aacc = 0.0;
                    for (int64_t t = 0; t < k; ++t) {
                        double p = xr[t] * (double)wr[t];
                        acc += p;
                        aacc += fabs(p);
                    }
                    y[i * n + j] = acc;
                    if (absdot) absdot[i * n + j] = aacc;
                }
            }
            free(wr);
        }
    }
    free(xd);
    return fail ? -2 : 0;
}

/* fp32 variant used only as the timed CPU baseline: each product and each
 * partial sum rounded to fp32, k in order. */
int oracle_matmul_f32(int type, const uint8_t* w, int64_t n, int64_t k, const uint16_t* x,
                      int64_t m, float* y) {
    int vpb, bpb;
    if (oracle_block_info(type, &vpb, &bpb) || k % vpb) return -1;
    int64_t rb = k / vpb * bpb;
    float* xf = (float*)malloc(sizeof(float) * (size_t)(m * k));
    if (!xf) return -2;
    for (int64_t i = 0; i < m * k; ++i) xf[i] = bf16_to_float(x[i]);
    int fail = 0;
#pragma omp parallel
    {
        float* wr = (float*)malloc(sizeof(float) * (size_t)k);
        if (!wr) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t j = 0; j < n; ++j) {
                dq_row(type, w + j * rb, k, wr);
                for (int64_t i = 0; i < m; ++i) {
                    const float* xr = xf + i * k;
                    float acc = 0.0f;
                    for (int64_t t = 0; t < k; ++t) {
                        float p = xr[t] * wr[t];
                        acc = acc + p;
                    }
                    y[i * n + j] = acc;
                }
            }
            free(wr);
        }
    }
    free(xf);
    return fail ? -2 : 0;
}

/* Number of OpenMP threads the parallel loops above use. */
int oracle_threads(void) {
    int t = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            t = omp_get_num_threads();
#endif
        }
    }
    return t;
}
