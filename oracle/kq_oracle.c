/*
 * kq_oracle.c -- CPU oracle for block-quantized (GGUF-style) matrix products.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or constant with the CUDA library; the two meet only through the
 * seeded byte generator in synth/.
 *
 * What it computes, written out plainly (no tiling, no fusion, no reordering):
 *
 *   decode:    every block is turned into its weights by the codec's own
 *              definition (below), once as the IEEE fp32 operation sequence
 *              the definition names (the bit-exact reference for dequantize)
 *              and once as the exact real value held in fp64;
 *   matmul:    Y[m][n] = sum_k W[n][k] * X[m][k], in fp64
 *              (mlx-kquant bindings.cpp, `quantized_matmul`: x @ dequant(w)
 *              with w laid out [N, K]);
 *   matmul_id: Y[t][s][n] = sum_k W[ids[t][s]][n][k] * X[t][k], in fp64
 *              (mlx-native 0.21.0 quantized_matmul_id_ggml.rs, module doc:
 *              output[token*top_k+slot][col] = sum_k dequant(weight[expert]
 *              [col][k]) * input[token][k]); an id outside [0, E) gives a NaN
 *              row (same file, `quantized_matmul_id_ggml` doc: invalid routing
 *              metadata writes a non-finite poison sentinel).
 *
 * Codec definitions followed:
 *
 *   Q8_0  (ds4_metal.m, MSL preamble `struct block_q8_0 { half d;
 *          int8_t qs[QK8_0]; }`, QK8_0 = 32; row bytes (K/32)*34 in
 *          `ds4_gpu_make_q8_0_mv_args`):  w_i = float(d) * float(q_i).
 *
 *   TQ1_G128 (ternel_packed_model.py, format constants BLOCK_BYTES = 28,
 *          BLOCK_SIZE = 128, MAX_FULL_CODE_BYTE = 242, MAX_TAIL_CODE_BYTE = 26;
 *          `_trit_table_source` / `_direct_trit_table_source`: digit i of a
 *          code byte p is (p / 3^i) % 3 and the weight is (digit - 1) * scale;
 *          illegal bytes decode to zero; `_GET_ROWS_SOURCE`: slot = j / 5 and
 *          digit = j % 5 for j < 125, the tail slot 25 holds weights
 *          125..127 as digits 0..2; layout docstring: 26 code bytes plus a raw
 *          little-endian fp16 scale).  Reading (byte order inside the
 *          canonical block is not printed): bytes 0..24 full codes, byte 25
 *          tail, bytes 26..27 scale.
 *
 *   Q4_K and Q2_K are named on the pages (mlx-native GgmlType, kernel names
 *          `kernel_mul_mv_id_q4_K_f32`, `kernel_mul_mv_id_q2_K_f32`) but their
 *          bit layouts are not printed there.  Reading: the public GGUF block
 *          layouts, which the pages require byte-for-byte ("native U8 GGUF
 *          blocks" fed straight to the kernels):
 *            Q4_K, 144 B / 256 w: fp16 d @0, fp16 dmin @2, 12 packed 6-bit
 *              scale/min bytes @4, 128 nibble bytes @16;
 *              w = float(d)*sc*q - float(dmin)*m.
 *            Q2_K, 84 B / 256 w: 16 scale/min bytes @0 (low nibble scale,
 *              high nibble min), 64 quant bytes @16 (four 2-bit quants each),
 *              fp16 d @80, fp16 dmin @82;  w = float(d)*sc*q - float(dmin)*m.
 *          Q5_K and Q6_K (named in the same GgmlType table) follow their
 *          GGUF layouts the same way (see q5_k_block, q6_k_block).
 *          Parity unpinned against an external GGUF file (none is at hand):
 *          the tests pin these two decoders to blocks built by packers written
 *          separately from this file, field by field.
 *
 * Products in the fp32 decode are exact (at most 21 significant bits), so the
 * one rounding is the final subtraction; the decode result is unique.
 * Compile with -ffp-contract=off so each C operator is one IEEE operation.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { KQO_Q8_0 = 8, KQO_Q2_K = 10, KQO_Q4_K = 12, KQO_Q5_K = 13, KQO_Q6_K = 14, KQO_TQ1_G128 = 1001 };

int kqo_block_weights(int type) {
    switch (type) {
    case KQO_Q8_0: return 32;
    case KQO_Q2_K: return 256;
    case KQO_Q4_K: return 256;
    case KQO_Q5_K: return 256;
    case KQO_Q6_K: return 256;
    case KQO_TQ1_G128: return 128;
    default: return 0;
    }
}

int kqo_block_bytes(int type) {
    switch (type) {
    case KQO_Q8_0: return 34;  /* 2-byte half + 32 int8 */
    case KQO_Q2_K: return 84;  /* 16 + 64 + 2 + 2 */
    case KQO_Q4_K: return 144; /* 2 + 2 + 12 + 128 */
    case KQO_Q5_K: return 176; /* 2 + 2 + 12 + 32 + 128 */
    case KQO_Q6_K: return 210; /* 128 + 64 + 16 + 2 */
    case KQO_TQ1_G128: return 28;
    default: return 0;
    }
}

/* IEEE 754 binary16 -> real value, from the format's definition
 * (sign, 5-bit biased exponent, 10-bit fraction).  Exact in double. */
static double half_value(const uint8_t *p) {
    unsigned h = (unsigned)p[0] | ((unsigned)p[1] << 8);
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* ---- per-codec decode of one block into fp32 (IEEE op sequence) and fp64 ---- */

static void q8_0_block(const uint8_t *b, float *w32, double *w64) {
    double d = half_value(b);
    float df = (float)d;
    for (int i = 0; i < 32; ++i) {
        int q = (int)(int8_t)b[2 + i];
        if (w32) w32[i] = df * (float)q;
        if (w64) w64[i] = d * (double)q;
    }
}

/* 6-bit scale and min of sub-block j from the 12 packed bytes s[0..11]
 * (GGUF Q4_K packing: sub-blocks 0..3 keep their scale and min in the low six
 * bits of s[j] and s[j+4]; sub-blocks 4..7 take their low four bits from the
 * nibbles of s[j+4] and their top two bits from the spare high bits of s[j-4]
 * (scale) and s[j] (min)). */
static void q4_k_scale_min(const uint8_t *s, int j, int *sc, int *m) {
    if (j < 4) {
        *sc = s[j] & 63;
        *m = s[j + 4] & 63;
    } else {
        *sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        *m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

static void q4_k_block(const uint8_t *b, float *w32, double *w64) {
    double d = half_value(b), dmin = half_value(b + 2);
    float df = (float)d, dminf = (float)dmin;
    const uint8_t *s = b + 4, *qs = b + 16;
    /* Four chunks of 64 weights; chunk c uses quant bytes qs[32c .. 32c+31]:
     * the low nibbles are weights 64c+0..31 (sub-block 2c), the high nibbles
     * weights 64c+32..63 (sub-block 2c+1). */
    for (int c = 0; c < 4; ++c) {
        for (int half = 0; half < 2; ++half) {
            int j = 2 * c + half, sc, m;
            q4_k_scale_min(s, j, &sc, &m);
            for (int l = 0; l < 32; ++l) {
                int byte = qs[32 * c + l];
                int q = half ? (byte >> 4) : (byte & 15);
                int idx = 64 * c + 32 * half + l;
                if (w32) w32[idx] = df * (float)sc * (float)q - dminf * (float)m;
                if (w64) w64[idx] = d * sc * q - dmin * m;
            }
        }
    }
}

static void q2_k_block(const uint8_t *b, float *w32, double *w64) {
    const uint8_t *s = b, *qs = b + 16;
    double d = half_value(b + 80), dmin = half_value(b + 82);
    float df = (float)d, dminf = (float)dmin;
    /* Two halves of 128 weights; half h uses qs[32h .. 32h+31].  Within a half,
     * bit pair j (bits 2j..2j+1) of byte 32h+l is weight 128h + 32j + l, and
     * weights come in sub-blocks of 16: sub-block 8h + 2j + l/16. */
    for (int h = 0; h < 2; ++h) {
        for (int j = 0; j < 4; ++j) {
            for (int l = 0; l < 32; ++l) {
                int q = (qs[32 * h + l] >> (2 * j)) & 3;
                int sb = s[8 * h + 2 * j + l / 16];
                int sc = sb & 15, m = sb >> 4;
                int idx = 128 * h + 32 * j + l;
                if (w32) w32[idx] = df * (float)sc * (float)q - dminf * (float)m;
                if (w64) w64[idx] = d * sc * q - dmin * m;
            }
        }
    }
}

/* Q5_K, 176 B / 256 w (GGUF reading): fp16 d @0, fp16 dmin @2, the 12
 * packed 6-bit scale/min bytes @4 (Q4_K's packing), qh[32] @16, qs[128] @48.
 * Chunk c (64 weights) takes qs[32c .. 32c+31]: weight 64c+l is the low
 * nibble of qs[32c+l] plus 16 times bit 2c of qh[l], in sub-block 2c;
 * weight 64c+32+l the high nibble plus 16 times bit 2c+1 of qh[l], in
 * sub-block 2c+1.  w = float(d)*sc*q - float(dmin)*m (products exact). */
static void q5_k_block(const uint8_t *b, float *w32, double *w64) {
    double d = half_value(b), dmin = half_value(b + 2);
    float df = (float)d, dminf = (float)dmin;
    const uint8_t *s = b + 4, *qh = b + 16, *qs = b + 48;
    for (int c = 0; c < 4; ++c) {
        for (int half = 0; half < 2; ++half) {
            int j = 2 * c + half, sc, m;
            q4_k_scale_min(s, j, &sc, &m);
            for (int l = 0; l < 32; ++l) {
                int byte = qs[32 * c + l];
                int q = (half ? (byte >> 4) : (byte & 15)) + 16 * ((qh[l] >> j) & 1);
                int idx = 64 * c + 32 * half + l;
                if (w32) w32[idx] = df * (float)sc * (float)q - dminf * (float)m;
                if (w64) w64[idx] = d * sc * q - dmin * m;
            }
        }
    }
}

/* Q6_K, 210 B / 256 w (GGUF reading): ql[128] @0 (low four bits), qh[64]
 * @128 (high two bits), int8 scales[16] @192, fp16 d @208.  Half h (128
 * weights) takes ql[64h ..], qh[32h ..], scales[8h ..]; for l in 0..31:
 *   weight 128h+l    : low nibble of ql[64h+l]    | bits 0-1 of qh[32h+l] << 4
 *   weight 128h+32+l : low nibble of ql[64h+32+l] | bits 2-3 << 4
 *   weight 128h+64+l : high nibble of ql[64h+l]   | bits 4-5 << 4
 *   weight 128h+96+l : high nibble of ql[64h+32+l]| bits 6-7 << 4
 * each minus 32, in sub-blocks of 16 (scale index 8h + position / 16).
 * w = (float(d) * sc) * q: d*sc is exact, the product with q rounds once. */
static void q6_k_block(const uint8_t *b, float *w32, double *w64) {
    const uint8_t *ql = b, *qh = b + 128;
    const int8_t *sc = (const int8_t *)(b + 192);
    double d = half_value(b + 208);
    float df = (float)d;
    for (int h = 0; h < 2; ++h) {
        for (int l = 0; l < 32; ++l) {
            int hb = qh[32 * h + l];
            int q[4];
            q[0] = ((ql[64 * h + l] & 15) | (((hb >> 0) & 3) << 4)) - 32;
            q[1] = ((ql[64 * h + 32 + l] & 15) | (((hb >> 2) & 3) << 4)) - 32;
            q[2] = ((ql[64 * h + l] >> 4) | (((hb >> 4) & 3) << 4)) - 32;
            q[3] = ((ql[64 * h + 32 + l] >> 4) | (((hb >> 6) & 3) << 4)) - 32;
            for (int r = 0; r < 4; ++r) {
                int idx = 128 * h + 32 * r + l;
                int s = sc[8 * h + idx % 128 / 16];
                if (w32) {
                    float ds = df * (float)s;
                    w32[idx] = ds * (float)q[r];
                }
                if (w64) w64[idx] = d * s * q[r];
            }
        }
    }
}

/* Base-3 digit i of a code byte; bytes above the largest legal value decode
 * to the "zero weight" digit 1 for every position. */
static int tq1_digit(int code, int i, int max_legal) {
    if (code > max_legal) return 1;
    int p = 1;
    for (int r = 0; r < i; ++r) p *= 3;
    return (code / p) % 3;
}

static void tq1_block(const uint8_t *b, float *w32, double *w64) {
    double scale = half_value(b + 26);
    float sf = (float)scale;
    for (int j = 0; j < 128; ++j) {
        int t;
        if (j < 125) t = tq1_digit(b[j / 5], j % 5, 242);
        else t = tq1_digit(b[25], j - 125, 26);
        if (w32) w32[j] = (float)(t - 1) * sf;
        if (w64) w64[j] = (double)(t - 1) * scale;
    }
}

/* Decode `rows` rows of K weights each; row r starts at w + r*row_stride.
 * Either output may be NULL.  Returns 0, or -1 on a bad type / shape. */
int kqo_decode(int type, const uint8_t *w, int64_t rows, int64_t k, int64_t row_stride,
               float *out32, double *out64) {
    int qk = kqo_block_weights(type), bb = kqo_block_bytes(type);
    if (qk == 0 || k % qk) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t blk = 0; blk < k / qk; ++blk) {
            const uint8_t *b = w + r * row_stride + blk * bb;
            float *o32 = out32 ? out32 + r * k + blk * qk : NULL;
            double *o64 = out64 ? out64 + r * k + blk * qk : NULL;
            switch (type) {
            case KQO_Q8_0: q8_0_block(b, o32, o64); break;
            case KQO_Q4_K: q4_k_block(b, o32, o64); break;
            case KQO_Q2_K: q2_k_block(b, o32, o64); break;
            case KQO_Q5_K: q5_k_block(b, o32, o64); break;
            case KQO_Q6_K: q6_k_block(b, o32, o64); break;
            case KQO_TQ1_G128: tq1_block(b, o32, o64); break;
            }
        }
    }
    return 0;
}

/* Row gather (Ternary Bonsai ternel_packed_model.py, `_GET_ROWS_SOURCE`:
 * decode exactly the requested rows; an id outside the table reads as an
 * all-zero row): out[t][:] = fp32 decode of row ids[t] of w. */
int kqo_get_rows(int type, const uint8_t *w, int64_t rows, int64_t k, int64_t row_stride,
                 const int32_t *ids, int64_t n_ids, float *out) {
    int qk = kqo_block_weights(type);
    if (qk == 0 || k % qk) return -1;
    for (int64_t t = 0; t < n_ids; ++t) {
        float *o = out + t * k;
        if (ids[t] < 0 || ids[t] >= rows) {
            for (int64_t c = 0; c < k; ++c) o[c] = 0.0f;
            continue;
        }
        kqo_decode(type, w + (int64_t)ids[t] * row_stride, 1, k, row_stride, o, NULL);
    }
    return 0;
}

/* Count the TQ1_G128 blocks holding a byte above the legal maximum and report
 * the first (row-major block index), or -1 if none. */
int64_t kqo_tq1_first_illegal(const uint8_t *w, int64_t rows, int64_t k, int64_t row_stride) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t blk = 0; blk < k / 128; ++blk) {
            const uint8_t *b = w + r * row_stride + blk * 28;
            int bad = b[25] > 26;
            for (int i = 0; i < 25; ++i) bad |= b[i] > 242;
            if (bad) return r * (k / 128) + blk;
        }
    return -1;
}

/* ---- products ---- */

typedef struct {
    int type;
    const uint8_t *w;
    int64_t n, k, row_stride;
    const double *x;    /* [m][k] */
    int64_t m;
    double *y;          /* [m][n] */
    int64_t n0, n1;     /* weight rows this worker owns */
    int status;
} matmul_job;

static void *matmul_worker(void *arg) {
    matmul_job *j = (matmul_job *)arg;
    double *row = (double *)malloc(sizeof(double) * (size_t)j->k);
    if (!row) { j->status = -2; return NULL; }
    for (int64_t n = j->n0; n < j->n1; ++n) {
        kqo_decode(j->type, j->w + n * j->row_stride, 1, j->k, j->row_stride, NULL, row);
        for (int64_t mm = 0; mm < j->m; ++mm) {
            const double *xr = j->x + mm * j->k;
            double acc = 0.0;
            for (int64_t kk = 0; kk < j->k; ++kk) acc += row[kk] * xr[kk];
            j->y[mm * j->n + n] = acc;
        }
    }
    free(row);
    return NULL;
}

/* Y[m][n] = sum_k W[n][k] X[m][k] in fp64.  Weight rows are split statically
 * over `threads` POSIX threads (1 = run on the caller's thread). */
int kqo_matmul(int type, const uint8_t *w, int64_t n, int64_t k, int64_t row_stride,
               const double *x, int64_t m, double *y, int threads) {
    int qk = kqo_block_weights(type);
    if (qk == 0 || k % qk || n < 0 || m < 0) return -1;
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (threads > n && n > 0) threads = (int)n;
    matmul_job jobs[256];
    pthread_t tids[256];
    for (int t = 0; t < threads; ++t) {
        jobs[t] = (matmul_job){type, w, n, k, row_stride, x, m, y,
                               n * t / threads, n * (t + 1) / threads, 0};
    }
    if (threads == 1) {
        matmul_worker(&jobs[0]);
        return jobs[0].status;
    }
    for (int t = 0; t < threads; ++t) pthread_create(&tids[t], NULL, matmul_worker, &jobs[t]);
    int st = 0;
    for (int t = 0; t < threads; ++t) {
        pthread_join(tids[t], NULL);
        if (jobs[t].status) st = jobs[t].status;
    }
    return st;
}

/* Y[t][s][n] = sum_k W[ids[t][s]][n][k] X[t][k]; W_e starts at w + e*expert_stride.
 * Invalid ids give a NaN row.  Single-threaded. */
int kqo_matmul_id(int type, const uint8_t *w, int64_t n_experts, int64_t n, int64_t k,
                  int64_t row_stride, int64_t expert_stride, const double *x, int64_t n_tokens,
                  const int32_t *ids, int64_t top_k, double *y) {
    int qk = kqo_block_weights(type);
    if (qk == 0 || k % qk) return -1;
    double *row = (double *)malloc(sizeof(double) * (size_t)k);
    if (!row) return -2;
    for (int64_t t = 0; t < n_tokens; ++t) {
        for (int64_t s = 0; s < top_k; ++s) {
            int32_t e = ids[t * top_k + s];
            double *yr = y + (t * top_k + s) * n;
            if (e < 0 || e >= n_experts) {
                for (int64_t c = 0; c < n; ++c) yr[c] = NAN;
                continue;
            }
            for (int64_t c = 0; c < n; ++c) {
                kqo_decode(type, w + e * expert_stride + c * row_stride, 1, k, row_stride, NULL, row);
                double acc = 0.0;
                for (int64_t kk = 0; kk < k; ++kk) acc += row[kk] * x[t * k + kk];
                yr[c] = acc;
            }
        }
    }
    free(row);
    return 0;
}
