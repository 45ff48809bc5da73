/*
 * CPU oracle for GGUF block-quantized weights (q4_K, q6_K, q8_0; decoders also
 * for q5_K and q4_0).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; it is compiled with
 * gcc -O2 -ffp-contract=off (no fused multiply-add, no fast-math) so every
 * floating-point operation below is rounded exactly where it is written.
 *
 * What it computes, and where that is stated:
 *  - dequantize: wire bytes -> float (the `dequantize` op docstring,
 *    mlx-kquant bindings.cpp; QTensor::dequantize, which decodes to f32
 *    through to_float, hanzo-ml quantized/mod.rs).  Block sizes: mlx-kquant README, "Codec reference"
 *    table (q4_k 256 values / 144 B, q5_k 256 / 176 B, q6_k 256 / 210 B, q8_0
 *    32 / 34 B, q4_0 32 / 18 B).  The
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
 *  - quantize: float -> wire bytes (the `quantize` op docstring, mlx-kquant
 *    bindings.cpp: float weights in, wire bytes out; hanzo-ml
 *    quantized/mod.rs QTensor::quantize).  The pages give no
 *    encoding search.  q8_0 follows ggml's published rule (absmax / 127,
 *    round half away from zero), pinned against gguf.quants.quantize.  q4_K
 *    and q6_K take the plainest reading: per sub-block min/max (q4_K) or
 *    absmax (q6_K) scales, 6-bit / int8 scale codes against an fp16 super-
 *    block scale, then the codes; every step below is one fp32 operation
 *    in a fixed order.  Those two are pinned by round-trip error bounds, not
 *    against ggml's own (search-based) encoder.
 *
 * Parity pins for every function live in tests/test_oracle.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define T_Q4_0 2
#define T_Q8_0 8
#define T_Q4_K 12
#define T_Q5_K 13
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

/* q5_K block (176 B): d and dmin (fp16) at 0 and 2, the 12 packed 6-bit
 * scale/min bytes at 4 (packed as in q4_K), qh[32] at 16, qs[128] at 48.
 * Value 64c + l (c = 0..3, l = 0..31) is the low nibble of qs[32c + l] plus 16
 * times bit 2c of qh[l], in sub-block 2c; value 64c + 32 + l is the high nibble
 * of the same byte plus 16 times bit 2c + 1 of qh[l], in sub-block 2c + 1.
 * y = fp32(fp32(d) * sc) * q - fp32(fp32(dmin) * m), q in 0..31. */
static void dq_q5k(const uint8_t* b, float* out) {
    float d = half_to_float(rd16(b)), dmin = half_to_float(rd16(b + 2));
    const uint8_t* s = b + 4;
    const uint8_t* qh = b + 16;
    const uint8_t* qs = b + 48;
    for (int c = 0; c < 4; ++c) {
        for (int half = 0; half < 2; ++half) {
            int j = 2 * c + half, sc, m;
            q4k_scale_min(s, j, &sc, &m);
            float dl = d * (float)sc, ml = dmin * (float)m;
            for (int l = 0; l < 32; ++l) {
                int nib = half ? (qs[32 * c + l] >> 4) : (qs[32 * c + l] & 15);
                int q = nib + 16 * ((qh[l] >> j) & 1);
                out[64 * c + 32 * half + l] = dl * (float)q - ml;
            }
        }
    }
}

/* q4_0 block (18 B): d (fp16) at 0, qs[16] at 2.  Value l (l = 0..15) is the
 * low nibble of qs[l] minus 8, value 16 + l the high nibble minus 8;
 * y = fp32(d) * q. */
static void dq_q4_0(const uint8_t* b, float* out) {
    float d = half_to_float(rd16(b));
    for (int l = 0; l < 16; ++l) {
        out[l] = d * (float)((b[2 + l] & 15) - 8);
        out[16 + l] = d * (float)((b[2 + l] >> 4) - 8);
    }
}

int oracle_block_info(int type, int* values, int* bytes) {
    switch (type) {
    case T_Q4_K: *values = 256; *bytes = 144; return 0;
    case T_Q6_K: *values = 256; *bytes = 210; return 0;
    case T_Q8_0: *values = 32; *bytes = 34; return 0;
    case T_Q5_K: *values = 256; *bytes = 176; return 0;
    case T_Q4_0: *values = 32; *bytes = 18; return 0;
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
        else if (type == T_Q5_K) dq_q5k(blk, o);
        else if (type == T_Q4_0) dq_q4_0(blk, o);
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

/* Thread count of the parallel loops (the timed baseline runs once on one
 * thread and once on all host cores); n <= 0 restores the default. */
void oracle_set_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    extern int omp_get_num_procs(void);
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
#else
    (void)n;
#endif
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


/* ------------------------------------------------------------------ encoder */

/* binary32 -> binary16, round to nearest, ties to even (IEEE-754 default).
 * Written from the binary16 definition: normal numbers 2^(e-15) (1 + f/1024)
 * for 1 <= e <= 30, subnormals 2^-14 (f / 1024); the 11-bit significand of
 * |v| is rounded with rintf (default rounding mode: nearest, ties to even);
 * a carry into bit 11 moves to the next binade; from 65520 on (the midpoint
 * between 65504 and 2^16) the result is infinity. */
static uint16_t float_to_half(float v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    float a = fabsf(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00u);
    if (a >= 65520.0f) return (uint16_t)(sign | 0x7c00u);
    if (a < ldexpf(1.0f, -14)) {                       /* subnormal range (and zero) */
        float m = rintf(ldexpf(a, 24));                /* units of 2^-24, exact scaling */
        return (uint16_t)(sign | (uint16_t)m);         /* m == 1024 is the smallest normal */
    }
    int e;
    frexpf(a, &e);                                     /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                            /* a in [2^e, 2^(e+1)) */
    float m = rintf(ldexpf(a, 10 - e));                /* significand in [1024, 2048] */
    if (m >= 2048.0f) {
        m = 1024.0f;
        e += 1;
    }
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0f));
}

int oracle_float_to_half(const float* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_half(in[i]);
    return 0;
}

static int clampi(float v, int lo, int hi) {
    int q = (int)v;
    return q < lo ? lo : (q > hi ? hi : q);
}

static void wr16(uint8_t* p, uint16_t h) {
    p[0] = (uint8_t)(h & 0xff);
    p[1] = (uint8_t)(h >> 8);
}

/* q8_0: d = max|x| / 127, codes round(x * (1/d)) (half away from zero),
 * d stored as binary16. */
static void qz_q8_0(const float* x, uint8_t* b) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float d = amax / 127.0f;
    float id = d == 0.0f ? 0.0f : 1.0f / d;
    wr16(b, float_to_half(d));
    for (int i = 0; i < 32; ++i) {
        float p = x[i] * id;
        b[2 + i] = (uint8_t)(int8_t)clampi(roundf(p), -128, 127);
    }
}

/* q4_K: sub-block j (values 32j..32j+31) spans [lo_j, hi_j] with
 * lo_j = min(0, min x) and hi_j = max x; its scale is (hi_j - lo_j) / 15 and
 * its min -lo_j.  The super-block scales d = max scale / 63 and
 * dmin = max min / 63 are stored as binary16; the 6-bit codes are the
 * rounded ratios to the stored values; each value's 4-bit code is
 * round((x + dmin*m_j) / (d*sc_j)), using the decoder's own products. */
static void qz_q4k(const float* x, uint8_t* b) {
    float sc_f[8], mn_f[8], smax = 0.0f, mmax = 0.0f;
    for (int j = 0; j < 8; ++j) {
        float lo = 0.0f, hi = x[32 * j];
        for (int i = 0; i < 32; ++i) {
            float v = x[32 * j + i];
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        sc_f[j] = (hi - lo) / 15.0f;
        mn_f[j] = -lo;
        if (sc_f[j] > smax) smax = sc_f[j];
        if (mn_f[j] > mmax) mmax = mn_f[j];
    }
    uint16_t hd = float_to_half(smax / 63.0f), hm = float_to_half(mmax / 63.0f);
    float df = half_to_float(hd), dmf = half_to_float(hm);
    int sc[8], m[8];
    for (int j = 0; j < 8; ++j) {
        sc[j] = df > 0.0f ? clampi(roundf(sc_f[j] / df), 0, 63) : 0;
        m[j] = dmf > 0.0f ? clampi(roundf(mn_f[j] / dmf), 0, 63) : 0;
    }
    memset(b, 0, 144);
    wr16(b, hd);
    wr16(b + 2, hm);
    uint8_t* s = b + 4;
    for (int j = 0; j < 4; ++j) {
        s[j] = (uint8_t)(sc[j] | ((sc[j + 4] >> 4) << 6));
        s[j + 4] = (uint8_t)(m[j] | ((m[j + 4] >> 4) << 6));
        s[j + 8] = (uint8_t)((sc[j + 4] & 0x0f) | ((m[j + 4] & 0x0f) << 4));
    }
    uint8_t* qs = b + 16;
    for (int v = 0; v < 256; ++v) {
        int j = v / 32;
        float ds = df * (float)sc[j];
        float dm = dmf * (float)m[j];
        int q = ds > 0.0f ? clampi(roundf((x[v] + dm) / ds), 0, 15) : 0;
        int c = v / 64, w = v % 64;
        if (w < 32) qs[32 * c + w] |= (uint8_t)q;
        else qs[32 * c + w - 32] |= (uint8_t)(q << 4);
    }
}

/* q6_K: sub-block j (values 16j..16j+15) has scale max|x| / 31; the
 * super-block scale d = max scale / 127 is stored as binary16, the int8
 * scale codes are the rounded ratios to it, and each value's 6-bit code is
 * round(x / (d*sc_j)) + 32, clamped to 0..63. */
static void qz_q6k(const float* x, uint8_t* b) {
    float s_f[16], smax = 0.0f;
    for (int j = 0; j < 16; ++j) {
        float a = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float v = fabsf(x[16 * j + i]);
            if (v > a) a = v;
        }
        s_f[j] = a / 31.0f;
        if (s_f[j] > smax) smax = s_f[j];
    }
    uint16_t hd = float_to_half(smax / 127.0f);
    float df = half_to_float(hd);
    int sc[16];
    for (int j = 0; j < 16; ++j) sc[j] = df > 0.0f ? clampi(roundf(s_f[j] / df), -128, 127) : 0;
    memset(b, 0, 210);
    uint8_t *ql = b, *qh = b + 128;
    for (int v = 0; v < 256; ++v) {
        int j = v / 16;
        float ds = df * (float)sc[j];
        int q = ds > 0.0f ? clampi(roundf(x[v] / ds), -32, 31) : 0;
        int c = q + 32;
        int h = v / 128, t = (v % 128) / 32, l = v % 32;
        ql[64 * h + l + 32 * (t & 1)] |= (uint8_t)((c & 0x0f) << (4 * (t >> 1)));
        qh[32 * h + l] |= (uint8_t)((c >> 4) << (2 * t));
    }
    for (int j = 0; j < 16; ++j) b[192 + j] = (uint8_t)(int8_t)sc[j];
    wr16(b + 208, hd);
}

int oracle_quantize(int type, const float* x, int64_t n_rows, int64_t k, uint8_t* out) {
    int vpb, bpb;
    if (oracle_block_info(type, &vpb, &bpb) || k % vpb) return 1;
    if (type != T_Q8_0 && type != T_Q4_K && type != T_Q6_K) return 1;   /* encoders of the three codecs */
    int64_t nb = n_rows * (k / vpb);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i) {
        const float* xb = x + i * vpb;
        uint8_t* ob = out + i * bpb;
        if (type == T_Q8_0) qz_q8_0(xb, ob);
        else if (type == T_Q4_K) qz_q4k(xb, ob);
        else qz_q6k(xb, ob);
    }
    return 0;
}
