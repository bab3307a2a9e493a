/*
 * qattn_oracle.c -- plain, slow, obviously-correct CPU oracle for the smoothed-K INT8 attention
 * forward (prefill) described on the SageAttention summary page
 * ("SAGEATTENTION: accurate 8-bit attention for plug-and-play inference acceleration",
 * aibr.jp/archives/102657).
 *
 * The file also holds, each in its own section further down, the oracle's parts for the
 * ThriftAttention page ("ThriftAttention: Selective Mixed Precision for Long-Context FP4
 * Attention", gist.science/ja/paper/2605.23081, method section): the block-mean key-tile
 * selection, NVFP4 quantization, and the FP4-path attention with FP16 promotion.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and the CPU-baseline leg
 * of the benchmark may load this library.  The product path (the CUDA library) never calls it and
 * shares no code, header, table or helper with it.
 *
 * What the page fixes, and where (section names of that page):
 *   - K is smoothed before quantization so that extreme values do not inflate the INT8 scale
 *     (dialogue answer on accuracy; sec. 2 "differences from prior work"; sec. 3 "core technical
 *     elements").
 *   - Q and K are quantized to INT8 and Q K^T runs as an integer product with 32-bit accumulation
 *     (sec. 3: the Tensor Core instruction mma(u8.u8.s32)).
 *   - P V runs in FP16 (sec. 2 and 3: FP16 accumulation, mma(f16.f16.f16)).
 *   - The kernel follows FlashAttention's blockwise softmax (sec. 4); blockwise evaluation is exact
 *     up to rounding, so the oracle evaluates the plain row softmax.
 * The page gives no formula, block size, scale rule or rounding mode.  The readings used here:
 *   - smoothing: K'[n,c] = K[n,c] - mean_n K[n,c], the mean over all N tokens of the sequence, per
 *     (batch, kv head, channel); the sum is exact in int64 fixed point (every fp16 value is an
 *     integer multiple of 2^-24), mean = (float)((double)sum / (N * 2^24)), K' = (float)K - mean
 *     in binary32;
 *   - quantization: blocks of 128 consecutive Q rows and 64 consecutive K rows (all d channels)
 *     per (batch, head); scale = amax / 127 (binary32 division), code = clamp(rint(x / scale),
 *     -127, 127) with binary32 division and round-half-even; amax == 0 gives scale 0, codes 0;
 *   - dequantization: S = S_int * sQ * sK / sqrt(d) in binary64;
 *   - causal: key j is visible to query i iff j <= i (square prefill);
 *   - GQA: query head h reads kv head h / (H / Hkv).
 * Everything after the int32 product is binary64.  Compile with -O2 -ffp-contract=off and without
 * -ffast-math, so that every binary32 operation above rounds exactly once to nearest-even.
 *
 * Layouts (all row-major, contiguous):
 *   q, out: [B, H, N, d]; k, v: [B, Hkv, N, d]; fp16 arrays are passed as raw uint16 bit patterns.
 *   q_scale: [B, H, ceil(N/128)]; k_scale: [B, Hkv, ceil(N/64)]; k_mean: [B, Hkv, d].
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_QBLOCK 128
#define ORACLE_KBLOCK 64
#define ORACLE_SBLOCK 256  /* block-sparse selection: query rows per selection block */
#define ORACLE_KTILE 128   /* block-sparse selection: keys per key tile */

/* ------------------------------------------------------------------------------------------------
 * IEEE 754 binary16, written from the format's definition: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; exponent 0 encodes subnormals m * 2^-24, exponent 31 encodes inf/NaN.
 * ---------------------------------------------------------------------------------------------- */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + m), e - 25);
    }
    return sign ? -v : v;
}

/* Round a binary64 value to the nearest binary16 (ties to even); overflow gives +-inf. */
uint16_t oracle_f64_to_f16(double x) {
    uint16_t sign = 0;
    if (isnan(x)) return 0x7E00;
    if (signbit(x)) { sign = 0x8000; x = -x; }
    if (x == 0.0) return sign;
    if (x < ldexp(1.0, -14)) {                  /* subnormal range: units of 2^-24 */
        double q = rint(ldexp(x, 24));          /* exact scaling, then round-half-even */
        return (uint16_t)(sign | (uint16_t)q);  /* q == 1024 is the smallest normal, still right */
    }
    int e;
    (void)frexp(x, &e);                         /* x = f * 2^e, f in [0.5, 1) */
    e -= 1;                                     /* x in [2^e, 2^(e+1)) */
    double q = rint(ldexp(x, 10 - e));          /* 11-bit significand in [1024, 2048] */
    if (q == 2048.0) { q = 1024.0; e += 1; }
    if (e + 15 >= 31) return (uint16_t)(sign | 0x7C00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)q - 1024));
}

/* ------------------------------------------------------------------------------------------------
 * Smoothing of K (page sec. 3, first technical element).
 * ---------------------------------------------------------------------------------------------- */

/* K * 2^24 as an exact integer: every binary16 value is an integer multiple of 2^-24 and
 * |K| <= 65504 < 2^16, so |K * 2^24| < 2^40. */
static int64_t k_fixed(uint16_t h) {
    return (int64_t)(oracle_f16_to_f64(h) * 16777216.0);
}

/* sums[(b*Hkv+g)*d + c] = sum over n of K[b,g,n,c] * 2^24, exact (|sum| < 2^57 for N <= 2^17). */
void oracle_k_channel_sums(const uint16_t* k, int B, int Hkv, int N, int d, int64_t* sums) {
    for (long bg = 0; bg < (long)B * Hkv; ++bg) {
        for (int c = 0; c < d; ++c) sums[bg * d + c] = 0;
        for (int n = 0; n < N; ++n) {
            const uint16_t* row = k + (bg * N + n) * (long)d;
            for (int c = 0; c < d; ++c) sums[bg * d + c] += k_fixed(row[c]);
        }
    }
}

/* mean = (float)((double)sum / (N * 2^24)): one rounding to binary64, one division, one
 * rounding to binary32. */
float oracle_mean_from_sum(int64_t sum, int N) {
    double den = (double)N * 16777216.0;
    return (float)((double)sum / den);
}

/* ------------------------------------------------------------------------------------------------
 * Per-block symmetric INT8 quantization (page sec. 3: INT8 operands; block sizes, scale rule and
 * rounding per the reading in the file header).
 * x holds `rows` rows of `d` binary32 values; writes codes and returns the block scale.
 * ---------------------------------------------------------------------------------------------- */
float oracle_quantize_block(const float* x, int rows, int d, int8_t* codes) {
    float amax = 0.0f;
    for (long i = 0; i < (long)rows * d; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        memset(codes, 0, (size_t)rows * d);
        return 0.0f;
    }
    float s = amax / 127.0f;
    for (long i = 0; i < (long)rows * d; ++i) {
        float t = x[i] / s;
        float r = rintf(t);          /* default rounding mode: nearest, ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        codes[i] = (int8_t)r;
    }
    return s;
}

/* The whole pre-processing: smoothing of K, then per-block quantization of Q and K'.
 * smooth = 0 skips the smoothing (mean taken as 0); used only for the negative control.
 * k_mean may be NULL. */
void oracle_smooth_quant(const uint16_t* q, const uint16_t* k, int B, int H, int Hkv, int N, int d,
                         int smooth, int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                         float* k_mean) {
    int nqb = (N + ORACLE_QBLOCK - 1) / ORACLE_QBLOCK;
    int nkb = (N + ORACLE_KBLOCK - 1) / ORACLE_KBLOCK;
    int64_t* sums = (int64_t*)calloc((size_t)B * Hkv * d, sizeof(int64_t));
    float* mean = (float*)calloc((size_t)B * Hkv * d, sizeof(float));
    float* buf = (float*)malloc(sizeof(float) * (size_t)ORACLE_QBLOCK * d);
    if (smooth) {
        oracle_k_channel_sums(k, B, Hkv, N, d, sums);
        for (long i = 0; i < (long)B * Hkv * d; ++i) mean[i] = oracle_mean_from_sum(sums[i], N);
    }
    if (k_mean) memcpy(k_mean, mean, sizeof(float) * (size_t)B * Hkv * d);
    for (long bg = 0; bg < (long)B * Hkv; ++bg) {
        for (int blk = 0; blk < nkb; ++blk) {
            int r0 = blk * ORACLE_KBLOCK;
            int rows = N - r0 < ORACLE_KBLOCK ? N - r0 : ORACLE_KBLOCK;
            for (int r = 0; r < rows; ++r)
                for (int c = 0; c < d; ++c) {
                    float kv = (float)oracle_f16_to_f64(k[(bg * N + r0 + r) * (long)d + c]);
                    buf[(long)r * d + c] = kv - mean[bg * d + c];
                }
            k_scale[bg * nkb + blk] =
                oracle_quantize_block(buf, rows, d, k_i8 + (bg * N + r0) * (long)d);
        }
    }
    for (long bh = 0; bh < (long)B * H; ++bh) {
        for (int blk = 0; blk < nqb; ++blk) {
            int r0 = blk * ORACLE_QBLOCK;
            int rows = N - r0 < ORACLE_QBLOCK ? N - r0 : ORACLE_QBLOCK;
            for (int r = 0; r < rows; ++r)
                for (int c = 0; c < d; ++c)
                    buf[(long)r * d + c] = (float)oracle_f16_to_f64(q[(bh * N + r0 + r) * (long)d + c]);
            q_scale[bh * nqb + blk] =
                oracle_quantize_block(buf, rows, d, q_i8 + (bh * N + r0) * (long)d);
        }
    }
    free(buf);
    free(mean);
    free(sums);
}

/* ------------------------------------------------------------------------------------------------
 * INT8 Q K^T with exact 32-bit accumulation (page sec. 3, mma(u8.u8.s32); signed codes per the
 * symmetric quantization).  out[i][j] = sum_c q[b,h,i0+i,c] * k[b,g(h),j0+j,c], no masking.
 * ---------------------------------------------------------------------------------------------- */
void oracle_qk_int32(const int8_t* q_i8, const int8_t* k_i8, int B, int H, int Hkv, int N, int d,
                     int b, int h, int i0, int ni, int j0, int nj, int32_t* out) {
    (void)B;
    int g = h / (H / Hkv);
    const int8_t* qb = q_i8 + ((long)b * H + h) * (long)N * d;
    const int8_t* kb = k_i8 + ((long)b * Hkv + g) * (long)N * d;
    for (int i = 0; i < ni; ++i)
        for (int j = 0; j < nj; ++j) {
            int32_t acc = 0;
            for (int c = 0; c < d; ++c)
                acc += (int32_t)qb[(long)(i0 + i) * d + c] * (int32_t)kb[(long)(j0 + j) * d + c];
            out[(long)i * nj + j] = acc;
        }
}

/* ------------------------------------------------------------------------------------------------
 * Attention rows, binary64 (page sec. 4: FlashAttention-style blockwise softmax, evaluated here
 * as the plain two-pass row softmax it is exactly equal to).
 * ---------------------------------------------------------------------------------------------- */

typedef struct {
    /* quantized mode */
    const int8_t* q_i8; const float* q_scale; const int8_t* k_i8; const float* k_scale;
    /* full-precision mode */
    const uint16_t* q16; const uint16_t* k16; int smooth;
    const uint16_t* v16;
    int B, H, Hkv, N, d, causal, quantized;
    const int64_t* row_bh; const int64_t* row_i; long nrows;
    const uint8_t* tile_mask;  /* block-sparse mode: [B*H][ceil(N/256)][ceil(N/128)], or NULL */
    double* out;
    double* kmean64;   /* full-precision mode: exact per-channel means, [B*Hkv, d] */
    long next;         /* work counter */
    pthread_mutex_t lock;
} attn_job;

static void attn_one_row(attn_job* J, long r, double* s, double* acc) {
    int H = J->H, Hkv = J->Hkv, N = J->N, d = J->d;
    long bh = J->row_bh[r];
    int i = (int)J->row_i[r];
    int b = (int)(bh / H), h = (int)(bh % H);
    int g = h / (H / Hkv);
    long bg = (long)b * Hkv + g;
    int nvis = J->causal ? i + 1 : N;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
    double m = -INFINITY;
    /* block-sparse mode: keys of unselected 128-key tiles are left out (weight 0) */
    const uint8_t* sel = NULL;
    if (J->tile_mask) {
        int nsb = (N + ORACLE_SBLOCK - 1) / ORACLE_SBLOCK, nkt = (N + ORACLE_KTILE - 1) / ORACLE_KTILE;
        sel = J->tile_mask + (bh * nsb + i / ORACLE_SBLOCK) * (long)nkt;
    }
    if (J->quantized) {
        int nkb = (N + ORACLE_KBLOCK - 1) / ORACLE_KBLOCK;
        int nqb = (N + ORACLE_QBLOCK - 1) / ORACLE_QBLOCK;
        const int8_t* qrow = J->q_i8 + (bh * N + i) * (long)d;
        double sq = (double)J->q_scale[bh * nqb + i / ORACLE_QBLOCK];
        for (int j = 0; j < nvis; ++j) {
            const int8_t* krow = J->k_i8 + (bg * N + j) * (long)d;
            int32_t acc32 = 0;
            for (int c = 0; c < d; ++c) acc32 += (int32_t)qrow[c] * (int32_t)krow[c];
            double sk = (double)J->k_scale[bg * nkb + j / ORACLE_KBLOCK];
            s[j] = (double)acc32 * sq * sk * inv_sqrt_d;
            if (sel && !sel[j / ORACLE_KTILE]) s[j] = -INFINITY;
            if (s[j] > m) m = s[j];
        }
    } else {
        const uint16_t* qrow = J->q16 + (bh * N + i) * (long)d;
        for (int j = 0; j < nvis; ++j) {
            const uint16_t* krow = J->k16 + (bg * N + j) * (long)d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) {
                double kc = oracle_f16_to_f64(krow[c]);
                if (J->smooth) kc -= J->kmean64[bg * d + c];
                dot += oracle_f16_to_f64(qrow[c]) * kc;
            }
            s[j] = dot * inv_sqrt_d;
            if (s[j] > m) m = s[j];
        }
    }
    double l = 0.0;
    for (int j = 0; j < nvis; ++j) { s[j] = s[j] == -INFINITY ? 0.0 : exp(s[j] - m); l += s[j]; }
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    for (int j = 0; j < nvis; ++j) {
        const uint16_t* vrow = J->v16 + (bg * N + j) * (long)d;
        for (int c = 0; c < d; ++c) acc[c] += s[j] * oracle_f16_to_f64(vrow[c]);
    }
    for (int c = 0; c < d; ++c) J->out[r * d + c] = acc[c] / l;
}

static void* attn_worker(void* arg) {
    attn_job* J = (attn_job*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)J->N);
    double* acc = (double*)malloc(sizeof(double) * (size_t)J->d);
    for (;;) {
        long r0;
        pthread_mutex_lock(&J->lock);
        r0 = J->next;
        J->next += 16;
        pthread_mutex_unlock(&J->lock);
        if (r0 >= J->nrows) break;
        long r1 = r0 + 16 < J->nrows ? r0 + 16 : J->nrows;
        for (long r = r0; r < r1; ++r) attn_one_row(J, r, s, acc);
    }
    free(acc);
    free(s);
    return NULL;
}

static void run_rows(attn_job* J, int nthreads) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    J->next = 0;
    pthread_mutex_init(&J->lock, NULL);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, attn_worker, J);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J->lock);
}

/* Output rows of the quantized attention: out[r, :] for the query row (bh = row_bh[r],
 * i = row_i[r]), computed from the INT8 codes and block scales, binary64 after the int32 product.
 * Returns the number of threads used. */
int oracle_attention_quantized(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                               const float* k_scale, const uint16_t* v, int B, int H, int Hkv,
                               int N, int d, int causal, const int64_t* row_bh,
                               const int64_t* row_i, long nrows, double* out, int nthreads) {
    attn_job J;
    memset(&J, 0, sizeof(J));
    J.q_i8 = q_i8; J.q_scale = q_scale; J.k_i8 = k_i8; J.k_scale = k_scale; J.v16 = v;
    J.B = B; J.H = H; J.Hkv = Hkv; J.N = N; J.d = d; J.causal = causal; J.quantized = 1;
    J.row_bh = row_bh; J.row_i = row_i; J.nrows = nrows; J.out = out;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    run_rows(&J, nthreads);
    return nthreads;
}

/* oracle_attention_quantized restricted to selected key tiles: query row i of head bh sees key
 * j only if tile_mask[bh][i / 256][j / 128] != 0 (and j <= i when causal). */
int oracle_attention_quantized_sparse(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                      const float* k_scale, const uint16_t* v, int B, int H,
                                      int Hkv, int N, int d, int causal, const uint8_t* tile_mask,
                                      const int64_t* row_bh, const int64_t* row_i, long nrows,
                                      double* out, int nthreads) {
    attn_job J;
    memset(&J, 0, sizeof(J));
    J.q_i8 = q_i8; J.q_scale = q_scale; J.k_i8 = k_i8; J.k_scale = k_scale; J.v16 = v;
    J.B = B; J.H = H; J.Hkv = Hkv; J.N = N; J.d = d; J.causal = causal; J.quantized = 1;
    J.row_bh = row_bh; J.row_i = row_i; J.nrows = nrows; J.out = out; J.tile_mask = tile_mask;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    run_rows(&J, nthreads);
    return nthreads;
}

/* Full-precision attention rows, softmax(Q K'^T / sqrt(d)) V in binary64 from the fp16 inputs,
 * with K' = K - (exact binary64 per-channel mean) when smooth != 0, else K' = K.  This is the
 * unquantized reference the quantized result is measured against. */
int oracle_attention_fp64(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H,
                          int Hkv, int N, int d, int causal, int smooth, const int64_t* row_bh,
                          const int64_t* row_i, long nrows, double* out, int nthreads) {
    attn_job J;
    memset(&J, 0, sizeof(J));
    J.q16 = q; J.k16 = k; J.v16 = v; J.smooth = smooth;
    J.B = B; J.H = H; J.Hkv = Hkv; J.N = N; J.d = d; J.causal = causal; J.quantized = 0;
    J.row_bh = row_bh; J.row_i = row_i; J.nrows = nrows; J.out = out;
    J.kmean64 = (double*)calloc((size_t)B * Hkv * d, sizeof(double));
    if (smooth) {
        for (long bg = 0; bg < (long)B * Hkv; ++bg)
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) acc += oracle_f16_to_f64(k[(bg * N + n) * (long)d + c]);
                J.kmean64[bg * d + c] = acc / (double)N;
            }
    }
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    run_rows(&J, nthreads);
    free(J.kmean64);
    return nthreads;
}

/* ------------------------------------------------------------------------------------------------
 * Block importance and selection for block-sparse attention.  The page "ThriftAttention:
 * Selective Mixed Precision for Long-Context FP4 Attention" (gist.science, technical summary,
 * method, heuristic block selection) scores each (query block, key block) pair by the dot
 * product of the two blocks' mean vectors and singles out the top-k pairs; its results section
 * compares against sparse top-k attention, which computes those pairs and drops the rest.  That
 * dropping variant is what is built here.  Readings: query blocks of 256 rows (a pair of
 * 128-row attention tiles), key blocks of 128 keys (one key tile); means taken over the block's
 * rows that exist (< N) of the fp16 inputs, exactly (int64 fixed point, one binary64 rounding);
 * score = sum over channels c = 0..d-1, in that order, of fma(qmean[c], kmean[c], acc) in
 * binary64; per query block the candidates are the key blocks it may see (all, or those at or
 * below its last row when causal), the diagonal key blocks (its own rows' tiles) are always
 * kept when causal, and the topk highest-scoring other candidates (ties to the lower index)
 * are added; the list is in ascending order.  The means of K are taken on K itself: subtracting
 * the channel mean would shift every score of a query block by the same amount.
 * ---------------------------------------------------------------------------------------------- */

/* means[o][blk][c] of x[o][n][c] over rows n of block blk (rows_per_block rows, the last one
 * shorter when N is not a multiple). */
void oracle_block_means(const uint16_t* x, long outer, int N, int d, int rows_per_block,
                        double* means) {
    int nb = (N + rows_per_block - 1) / rows_per_block;
    for (long o = 0; o < outer; ++o)
        for (int blk = 0; blk < nb; ++blk) {
            int n0 = blk * rows_per_block;
            int n1 = n0 + rows_per_block < N ? n0 + rows_per_block : N;
            for (int c = 0; c < d; ++c) {
                int64_t sum = 0;
                for (int n = n0; n < n1; ++n) sum += k_fixed(x[(o * N + n) * (long)d + c]);
                means[(o * nb + blk) * (long)d + c] = (double)sum / ((double)(n1 - n0) * 16777216.0);
            }
        }
}

/* scores[bh][i][j] = qmeans[bh][i] . kmeans[bh's kv head][j], fma chain over c in order. */
void oracle_block_scores(const double* qmeans, const double* kmeans, int B, int H, int Hkv, int nsb,
                         int nkt, int d, double* scores) {
    for (long bh = 0; bh < (long)B * H; ++bh) {
        long bg = (bh / H) * Hkv + (bh % H) / (H / Hkv);
        for (int i = 0; i < nsb; ++i)
            for (int j = 0; j < nkt; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc = fma(qmeans[(bh * nsb + i) * (long)d + c], kmeans[(bg * nkt + j) * (long)d + c], acc);
                scores[(bh * nsb + i) * (long)nkt + j] = acc;
            }
    }
}

/* list[bh][i][0 .. count[bh][i]) = the selected key tiles of query block i, ascending. */
void oracle_select_blocks(const double* scores, int B, int H, int N, int causal, int topk,
                          int32_t* list, int32_t* count) {
    int nsb = (N + ORACLE_SBLOCK - 1) / ORACLE_SBLOCK, nkt = (N + ORACLE_KTILE - 1) / ORACLE_KTILE;
    uint8_t* pick = (uint8_t*)malloc((size_t)nkt);
    for (long bh = 0; bh < (long)B * H; ++bh)
        for (int i = 0; i < nsb; ++i) {
            const double* sc = scores + (bh * nsb + i) * (long)nkt;
            int last = causal ? 2 * i + 1 : nkt - 1;       /* highest key tile the block may see */
            if (last > nkt - 1) last = nkt - 1;
            memset(pick, 0, (size_t)nkt);
            if (causal)
                for (int j = 2 * i; j <= last; ++j) pick[j] = 1;
            for (int r = 0; r < topk; ++r) {
                int best = -1;
                for (int j = 0; j <= last; ++j)
                    if (!pick[j] && (best < 0 || sc[j] > sc[best])) best = j;
                if (best < 0) break;
                pick[best] = 1;
            }
            int n = 0;
            int32_t* out = list + (bh * nsb + i) * (long)nkt;
            for (int j = 0; j < nkt; ++j)
                if (pick[j]) out[n++] = j;
            count[bh * nsb + i] = n;
        }
    free(pick);
}

/* ------------------------------------------------------------------------------------------------
 * NVFP4 quantization: the operand format of the FP4 path of the ThriftAttention page
 * ("ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention",
 * gist.science/ja/paper/2605.23081, method section, "FP4 path": the blocks that are not promoted
 * to FP16 are computed in FP4 using the NVFP4 micro-scaling format of Blackwell GPUs).
 * The page names the format but does not define it.  The reading used here is the format as NVIDIA
 * publishes it: FP4 E2M1 elements in blocks of 16, one unsigned FP8 E4M3 scale per block and one
 * binary32 scale per tensor; the tensor is one (batch, head) slice.  Steps, every binary32
 * operation rounded once to nearest-even:
 *   x'    = (float)x - mean[c]          (mean optional: the smoothing of K, subtracted per channel)
 *   amax  = max |x'| over the slice;    g = amax / 2688  (2688 = 448 * 6: largest scale * largest
 *                                                         element)
 *   per block of 16:  bmax = max |x'|;  s = E4M3(bmax / (6 * g))   (6 * g rounded first)
 *                     sc = s * g;       code_i = E2M1(x'_i / sc)
 *   decoded value x^ = E2M1value(code) * E4M3value(s) * g.
 * Both conversions round to nearest, ties to even, and saturate to the largest finite value
 * (448, 6).  A block whose scale rounds to 0, and every block of a slice with amax == 0, gets
 * scale byte 0 and codes 0.  A code whose value is zero is written as +0 (code 0).
 * Packing: two codes per byte, the element with the lower index in bits 0-3.
 * ---------------------------------------------------------------------------------------------- */

/* E2M1 value of a 4-bit code: 1 sign bit, 2 exponent bits (bias 1), 1 fraction bit; exponent 0
 * encodes 0 and 0.5 (subnormal), no infinities or NaN.  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_decode(uint8_t code) {
    int e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (code & 8) ? -v : v;
}

/* Nearest E2M1 code to x, ties to the even fraction bit, |x| >= 6 saturating to 6.  Inside each
 * binade of the format the representable magnitudes are the integer multiples of one spacing
 * (0.5 below 2, 1 in [2, 4), 2 in [4, 8)), so rounding is rint(|x| / spacing) with ties to even,
 * and an even multiple is exactly an even fraction bit. */
uint8_t oracle_e2m1_encode(float x) {
    double m = fabs((double)x);
    double spacing = (m < 2.0) ? 0.5 : (m < 4.0) ? 1.0 : 2.0;
    double v = rint(m / spacing) * spacing;    /* exact: spacing is a power of two */
    if (v > 6.0) v = 6.0;
    uint8_t mag;
    if (v < 2.0) mag = (uint8_t)(v * 2.0);                      /* 0, 0.5, 1, 1.5 -> 0..3 */
    else if (v < 4.0) mag = (uint8_t)(4 + (int)(v - 2.0));      /* 2, 3 -> 4, 5 */
    else mag = (uint8_t)(v == 4.0 ? 6 : 7);                     /* 4, 6 -> 6, 7 */
    if (mag == 0) return 0;
    return (x < 0.0f) ? (uint8_t)(mag | 8) : mag;
}

/* Value of an unsigned E4M3 byte (the FP8 E4M3 format with the sign bit 0): 4 exponent bits
 * (bias 7), 3 fraction bits; exponent 0 encodes subnormals m * 2^-9; 0x7F is NaN, 448 the
 * largest finite value. */
double oracle_ue4m3_decode(uint8_t code) {
    int e = (code >> 3) & 15, m = code & 7;
    if (code == 0x7F) return NAN;
    return (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
}

/* Nearest E4M3 byte to x >= 0, ties to the even fraction bit, values above 448 saturating to 448. */
uint8_t oracle_ue4m3_encode(float x) {
    double v = (double)x;
    if (!(v > 0.0)) return 0;
    if (v >= 448.0) return 0x7E;
    if (v < ldexp(1.0, -6)) {                  /* subnormal range: units of 2^-9 */
        return (uint8_t)rint(ldexp(v, 9));     /* 8 is the smallest normal, code 0x08: still right */
    }
    int e;
    (void)frexp(v, &e);
    e -= 1;                                    /* v in [2^e, 2^(e+1)), e in [-6, 8] */
    double q = rint(ldexp(v, 3 - e));          /* 4-bit significand in [8, 16] */
    if (q == 16.0) { q = 8.0; e += 1; }
    int code = ((e + 7) << 3) | ((int)q - 8);
    return (uint8_t)(code > 0x7E ? 0x7E : code);
}

/* One block of 16 values (binary32, already smoothed) with the slice's global scale g. */
static void nvfp4_block(const float* x, float g, uint8_t* codes16, uint8_t* scale) {
    float bmax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > bmax) bmax = a;
    }
    uint8_t s = 0;
    if (g > 0.0f) {
        float sixg = 6.0f * g;
        float t = bmax / sixg;
        s = oracle_ue4m3_encode(t);
    }
    *scale = s;
    if (s == 0) {
        for (int i = 0; i < 16; ++i) codes16[i] = 0;
        return;
    }
    float sc = (float)oracle_ue4m3_decode(s) * g;   /* the E4M3 value is exact in binary32 */
    for (int i = 0; i < 16; ++i) {
        float q = x[i] / sc;
        codes16[i] = oracle_e2m1_encode(q);
    }
}

/* x: fp16 [S][R][C]; mean: binary32 [S][C] or NULL.
 * along_rows == 0: blocks of 16 consecutive channels of one row (C % 16 == 0);
 *   codes [S][R][C/2] bytes, scales [S][R][C/16].
 * along_rows == 1: blocks of 16 consecutive rows of one channel, written transposed; rows
 *   R .. Rp-1 (Rp = R rounded up to 128, one key tile) are zero padding;
 *   codes [S][C][Rp/2] bytes, scales [S][C][Rp/16].
 * gscale [S]: g of each slice.  Returns 0, or -1 on a bad argument. */
int oracle_quant_nvfp4(const uint16_t* x, const float* mean, int S, int R, int C, int along_rows,
                       uint8_t* codes, uint8_t* scales, float* gscale) {
    if (S < 1 || R < 1 || C < 1) return -1;
    if (!along_rows && C % 16 != 0) return -1;
    int Rp = (R + 127) / 128 * 128;
    float* xs = (float*)malloc(sizeof(float) * (size_t)R * C);
    float blk[16];
    uint8_t c16[16];
    for (long s = 0; s < S; ++s) {
        float amax = 0.0f;
        for (long r = 0; r < R; ++r)
            for (int c = 0; c < C; ++c) {
                float v = (float)oracle_f16_to_f64(x[(s * R + r) * C + c]);
                if (mean) v = v - mean[s * C + c];
                xs[r * C + c] = v;
                if (fabsf(v) > amax) amax = fabsf(v);
            }
        float g = amax / 2688.0f;
        gscale[s] = g;
        if (!along_rows) {
            for (long r = 0; r < R; ++r)
                for (int b = 0; b < C / 16; ++b) {
                    nvfp4_block(xs + r * C + b * 16, g, c16, scales + (s * R + r) * (C / 16) + b);
                    uint8_t* out = codes + (s * R + r) * (C / 2) + b * 8;
                    for (int i = 0; i < 8; ++i) out[i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
                }
        } else {
            for (int c = 0; c < C; ++c)
                for (int b = 0; b < Rp / 16; ++b) {
                    for (int i = 0; i < 16; ++i) {
                        long r = (long)b * 16 + i;
                        blk[i] = (r < R) ? xs[r * C + c] : 0.0f;
                    }
                    nvfp4_block(blk, g, c16, scales + (s * C + c) * (Rp / 16) + b);
                    uint8_t* out = codes + (s * C + c) * (Rp / 2) + b * 8;
                    for (int i = 0; i < 8; ++i) out[i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
                }
        }
    }
    free(xs);
    return 0;
}

/* ------------------------------------------------------------------------------------------------
 * Attention on the FP4 path (ThriftAttention page, method section: "FP4 path" computes the blocks
 * in NVFP4; "online merge" combines blocks with FlashAttention-2's online softmax; the FP4 path's
 * probability blocks use a two-level quantization adapted from SageAttention3, whose details the
 * page does not give).  Every key tile here is on the FP4 path (no promotion).  Readings:
 *   - Q (per query head) and smoothed K (per kv head) are NVFP4 along the channels, V NVFP4 along
 *     the tokens (transposed, Np tokens per channel row); decoded values as oracle_quant_nvfp4;
 *   - scores x_j = S_ij * log2(e) / sqrt(d) in binary64 from the decoded Q and K;
 *   - key tiles of 128 in order; per tile m' = max(m, max_j x_j), corr = 2^(m - m'),
 *     p_j = 2^(x_j - m') rounded to binary32;
 *   - two-level quantization of the tile's P row: level 1, a per-row binary32 scale
 *     gP = max_j p_j / 2688 that maps the row into the E2M1 x E4M3 range; level 2, NVFP4 blocks of
 *     16 keys with gP as the global scale (the same binary32 steps as oracle_quant_nvfp4);
 *   - l = l * corr + sum_j p^_j over the dequantized p^ (the values the P V product uses);
 *     acc = acc * corr + sum_j p^_j v^_j;  out = acc / l.
 * The GPU's scores carry f32 accumulation and its exponentials binary32 rounding, so an FP4
 * decision taken within a relative 2^-16 of a tie may go the other way there.  For each output
 * row the oracle also returns a slack: the sum, over such decisions, of the largest change that
 * decision can make to the row's output (code: one E2M1 step times its scale; block scale: the
 * whole block's p plus two steps per element), times (max |v^| + max |out|) / l.
 * ---------------------------------------------------------------------------------------------- */

static double nvfp4_value(const uint8_t* codes, const uint8_t* scales, long row, int rowlen, int j,
                          double g) {
    uint8_t byte = codes[row * (rowlen / 2) + j / 2];
    uint8_t nib = (j & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_decode(nib) * oracle_ue4m3_decode(scales[row * (rowlen / 16) + j / 16]) * g;
}

/* E2M1 code of q, and whether a relative perturbation of 2^-16 could change it. */
static int e2m1_near_tie(float q) {
    const double d = ldexp(1.0, -16);
    return oracle_e2m1_encode((float)(q * (1.0 - d))) != oracle_e2m1_encode((float)(q * (1.0 + d)));
}

static int ue4m3_near_tie(float t) {
    const double d = ldexp(1.0, -16);
    return oracle_ue4m3_encode((float)(t * (1.0 - d))) != oracle_ue4m3_encode((float)(t * (1.0 + d)));
}

/* q_codes [B*H][N][d/2], q_scales [B*H][N][d/16], q_g [B*H]; k_* likewise over B*Hkv;
 * vt_codes [B*Hkv][d][Np/2], vt_scales [B*Hkv][d][Np/16], v_g [B*Hkv].
 * Promotion (the FP16 path of the same page's method section: the top-k query-key block pairs are
 * computed in FP16; NULL promote = none): promote [B*H][ceil(N/256)][ceil(N/128)] marks the key
 * tiles of each 256-row query block that run in FP16, from fp16 q [B*H][N][d], k and v
 * [B*Hkv][N][d]; their scores use the smoothed keys, x_j = sum_c q_c (k_jc - k_mean_c) log2(e) /
 * sqrt(d) (k_mean [B*Hkv][d], the mean the FP4 K was smoothed with), p_j is rounded to binary32
 * and then to fp16, and l and P V take those fp16 values and fp16 V.
 * Rows (row_bh[r], row_i[r]) for r < nrows; out [nrows][d], slack [nrows].  Returns 0, or -1 on a
 * bad argument. */
int oracle_attention_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* q_g,
                           const uint8_t* k_codes, const uint8_t* k_scales, const float* k_g,
                           const uint8_t* vt_codes, const uint8_t* vt_scales, const float* v_g,
                           const uint16_t* q16, const uint16_t* k16, const uint16_t* v16,
                           const float* k_mean, const uint8_t* promote,
                           int B, int H, int Hkv, int N, int Np, int d, int causal,
                           const long* row_bh, const long* row_i, long nrows, double* out,
                           double* slack) {
    if (B < 1 || H < 1 || Hkv < 1 || N < 1 || H % Hkv || d % 16 || Np < N || Np % 16) return -1;
    if (promote && (!q16 || !k16 || !v16 || !k_mean)) return -1;
    const double sl2 = 1.4426950408889634 / sqrt((double)d);
    const double rel = ldexp(1.0, -16);
    const long nsb = (N + 255) / 256, nkt = (N + 127) / 128;
    double* q = (double*)malloc(sizeof(double) * d);
    double* acc = (double*)malloc(sizeof(double) * d);
    double x[128], ph[128], risk[128];
    float p[128];
    for (long r = 0; r < nrows; ++r) {
        const long bh = row_bh[r], i = row_i[r];
        const long b = bh / H, h = bh % H, bg = b * Hkv + h / (H / Hkv);
        for (int c = 0; c < d; ++c) q[c] = nvfp4_value(q_codes, q_scales, bh * N + i, d, c, q_g[bh]);
        const long last = causal ? i : N - 1;
        /* l, acc: the online softmax; rv, rp: the risk sums against |v| and against |out|,
         * rescaled with l */
        double m = -INFINITY, l = 0.0, rv = 0.0, rp = 0.0;
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (long t0 = 0; t0 <= last; t0 += 128) {
            const int n = (int)((last - t0 + 1) < 128 ? (last - t0 + 1) : 128);   /* visible keys */
            if (promote && promote[(bh * nsb + i / 256) * nkt + t0 / 128]) {
                /* FP16 path: smoothed scores from the fp16 operands, fp16 P, fp16 V */
                double tmx = -INFINITY;
                for (int j = 0; j < n; ++j) {
                    double sdot = 0.0;
                    for (int c = 0; c < d; ++c)
                        sdot += oracle_f16_to_f64(q16[(bh * N + i) * (long)d + c]) *
                                (oracle_f16_to_f64(k16[(bg * N + t0 + j) * (long)d + c]) -
                                 (double)k_mean[bg * d + c]);
                    x[j] = sdot * sl2;
                    if (x[j] > tmx) tmx = x[j];
                }
                const double mn = m > tmx ? m : tmx;
                const double corr = exp2(m - mn);
                l *= corr;
                rv *= corr;
                rp *= corr;
                for (int c = 0; c < d; ++c) acc[c] *= corr;
                for (int j = 0; j < n; ++j) {
                    const float pf = (float)exp2(x[j] - mn);
                    const double p16 = oracle_f16_to_f64(oracle_f64_to_f16((double)pf));
                    l += p16;
                    for (int c = 0; c < d; ++c)
                        acc[c] += p16 * oracle_f16_to_f64(v16[(bg * N + t0 + j) * (long)d + c]);
                }
                m = mn;
                continue;
            }
            double tmax = -INFINITY;
            for (int j = 0; j < n; ++j) {
                double sdot = 0.0;
                for (int c = 0; c < d; ++c)
                    sdot += q[c] * nvfp4_value(k_codes, k_scales, bg * N + t0 + j, d, c, k_g[bg]);
                x[j] = sdot * sl2;
                if (x[j] > tmax) tmax = x[j];
            }
            const double mn = m > tmax ? m : tmax;
            const double corr = exp2(m - mn);
            float pmax = 0.0f;
            for (int j = 0; j < 128; ++j) {
                p[j] = j < n ? (float)exp2(x[j] - mn) : 0.0f;
                if (p[j] > pmax) pmax = p[j];
                risk[j] = 0.0;
                ph[j] = 0.0;
            }
            /* level 1: the row's binary32 scale; level 2: NVFP4 blocks of 16 keys */
            const float gp = pmax / 2688.0f;
            for (int blk = 0; blk < 8; ++blk) {
                float bmax = 0.0f;
                for (int e = 0; e < 16; ++e)
                    if (p[blk * 16 + e] > bmax) bmax = p[blk * 16 + e];
                if (!(gp > 0.0f)) continue;
                const float sixg = 6.0f * gp;
                const float t = bmax / sixg;
                const uint8_t sb = oracle_ue4m3_encode(t);
                const float sc = sb ? (float)oracle_ue4m3_decode(sb) * gp : 0.0f;
                for (int e = 0; e < 16 && sb; ++e) {
                    const int j = blk * 16 + e;
                    const float qq = p[j] / sc;
                    ph[j] = oracle_e2m1_decode(oracle_e2m1_encode(qq)) * (double)sc;
                    if (e2m1_near_tie(qq)) {
                        double lo = oracle_e2m1_decode(oracle_e2m1_encode((float)(qq * (1.0 - rel))));
                        double hi = oracle_e2m1_decode(oracle_e2m1_encode((float)(qq * (1.0 + rel))));
                        risk[j] += fabs(hi - lo) * (double)sc;
                    }
                }
                if (ue4m3_near_tie(t)) {
                    /* the scale may round to a neighbour (one E4M3 step, or 0): every p^ of the
                     * block may move by up to its own size plus two code steps */
                    const double big = 2.0 * 2.0 * (double)bmax / 6.0 + 1e-300;
                    for (int e = 0; e < 16; ++e) risk[blk * 16 + e] += p[blk * 16 + e] + big;
                }
            }
            l *= corr;
            rv *= corr;
            rp *= corr;
            for (int c = 0; c < d; ++c) acc[c] *= corr;
            for (int j = 0; j < n; ++j) {
                l += ph[j];
                double vm = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double v = nvfp4_value(vt_codes, vt_scales, bg * d + c, Np, (int)(t0 + j),
                                                 v_g[bg]);
                    acc[c] += ph[j] * v;
                    if (fabs(v) > vm) vm = fabs(v);
                }
                rv += risk[j] * vm;
                rp += risk[j];
            }
            m = mn;
        }
        double omax = 0.0;
        for (int c = 0; c < d; ++c) {
            out[r * d + c] = acc[c] / l;
            if (fabs(out[r * d + c]) > omax) omax = fabs(out[r * d + c]);
        }
        slack[r] = (rv + rp * omax) / l;
    }
    free(q);
    free(acc);
    return 0;
}

/* ------------------------------------------------------------------------------------------------
 * Adaptive quantization (SageAttention summary page, aibr.jp/archives/102657: the dialogue and
 * sec. 2-4 -- the quantization strength is chosen per layer or head, so that the important parts
 * keep more precision while the others run faster; +11.7 % speed without metric loss).  The page
 * names no variants.  The coarser variant here keeps the INT8 Q K^T and runs P V in FP8 E4M3
 * (twice the FP16 tensor rate on Blackwell) instead of FP16; the choice between the two is made
 * per (batch, kv head) by calibration.  Readings:
 *   - V in E4M3 per (batch, kv head) slice: amax = max |v|, sV = amax / 448 (binary32 division;
 *     448 is the largest E4M3 value), code = E4M3(v / sV) with binary32 division, nearest-even,
 *     saturating at 448; amax == 0 gives sV = 0 and codes 0; a zero code is +0 (0x00) whatever
 *     the sign of the input.  Stored transposed ([slice][channel][Np] bytes, Np = N rounded up to
 *     128, zero padding), the K-major operand of the P V product.
 *   - P in E4M3 follows FlashAttention's online softmax over key tiles of 128 (page sec. 4),
 *     with the running maximum moved only when it grows by more than 4 (log2 units): per tile
 *     the maximum t of the scaled scores of the tile's visible keys; if t > m + 4 (or on the first
 *     tile) the accumulated O and l are scaled by 2^(m - t) and m = t; then per key p = 2^(y),
 *     y = S_int * c + (4 - m) (one binary32 fused multiply-add; c = (sQ * sK) * sl2 in binary32,
 *     sl2 = binary32(log2(e) / sqrt(d))), so that p <= 2^(4 + 4) = 256 < 448; p^ = E4M3(p);
 *     l += p^; O += p^ v^ with v^ the E4M3 code values; out = O * sV / l.  The scaled maximum of
 *     a 64-key scale block is (max S_int over its visible keys) * c, one binary32 product.
 *   - The GPU computes 2^(y) with MUFU ex2 (binary32, a few ulp), so an E4M3 decision taken
 *     within a relative 2^-16 of a rounding tie may go the other way there: for each output row
 *     the oracle returns a slack, the sum over such decisions of one E4M3 step times
 *     (max |v^| sV + max |out|) / l.
 * ---------------------------------------------------------------------------------------------- */

/* E4M3 byte of x (sign bit 7, then the unsigned byte of |x|), nearest-even, saturating at 448;
 * a zero magnitude is +0. */
uint8_t oracle_e4m3_encode(float x) {
    uint8_t mag = oracle_ue4m3_encode(fabsf(x));
    if (mag == 0) return 0;
    return (x < 0.0f) ? (uint8_t)(mag | 0x80) : mag;
}

double oracle_e4m3_decode(uint8_t code) {
    double v = oracle_ue4m3_decode((uint8_t)(code & 0x7F));
    return (code & 0x80) ? -v : v;
}

/* v: fp16 [S][R][C]; codes [S][C][Rp] (Rp = R rounded up to 128, rows R .. Rp-1 zero);
 * scale [S].  Returns 0, or -1 on a bad argument. */
int oracle_quant_v_fp8(const uint16_t* v, int S, int R, int C, uint8_t* codes, float* scale) {
    if (S < 1 || R < 1 || C < 1) return -1;
    const long Rp = (R + 127) / 128 * 128;
    for (long s = 0; s < S; ++s) {
        float amax = 0.0f;
        for (long r = 0; r < R; ++r)
            for (int c = 0; c < C; ++c) {
                float a = fabsf((float)oracle_f16_to_f64(v[(s * R + r) * C + c]));
                if (a > amax) amax = a;
            }
        const float sv = amax / 448.0f;
        scale[s] = sv;
        for (int c = 0; c < C; ++c)
            for (long r = 0; r < Rp; ++r) {
                uint8_t code = 0;
                if (r < R && amax > 0.0f)
                    code = oracle_e4m3_encode((float)oracle_f16_to_f64(v[(s * R + r) * C + c]) / sv);
                codes[(s * C + c) * Rp + r] = code;
            }
    }
    return 0;
}

/* E4M3 code of p >= 0 and whether a relative perturbation of 2^-16 could change it; *step is
 * the distance between the two codes that perturbation can give. */
static uint8_t e4m3_with_risk(float p, double* step) {
    const double d = ldexp(1.0, -16);
    const uint8_t lo = oracle_ue4m3_encode((float)(p * (1.0 - d)));
    const uint8_t hi = oracle_ue4m3_encode((float)(p * (1.0 + d)));
    *step = (lo != hi) ? oracle_ue4m3_decode(hi) - oracle_ue4m3_decode(lo) : 0.0;
    return oracle_ue4m3_encode(p);
}

/* Attention with INT8 Q K^T (as oracle_attention_quantized) and FP8 P V, row by row in the online
 * order above.  q_i8 [B*H][N][d], q_scale [B*H][ceil(N/128)], k_i8 [B*Hkv][N][d],
 * k_scale [B*Hkv][ceil(N/64)], vt8 [B*Hkv][d][Np], v_scale [B*Hkv].  Rows (row_bh[r], row_i[r]);
 * out [nrows][d], slack [nrows].  Returns 0, or -1 on a bad argument. */
int oracle_attention_pv8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                         const float* k_scale, const uint8_t* vt8, const float* v_scale, int B,
                         int H, int Hkv, int N, int Np, int d, int causal, const long* row_bh,
                         const long* row_i, long nrows, double* out, double* slack) {
    if (B < 1 || H < 1 || Hkv < 1 || N < 1 || H % Hkv || Np < N || Np % 128) return -1;
    const float sl2 = (float)(1.4426950408889634 / sqrt((double)d));
    const int nqb = (N + ORACLE_QBLOCK - 1) / ORACLE_QBLOCK, nkb = (N + ORACLE_KBLOCK - 1) / ORACLE_KBLOCK;
    double* acc = (double*)malloc(sizeof(double) * d);
    int32_t s[128];
    double ph[128], step[128];
    for (long r = 0; r < nrows; ++r) {
        const long bh = row_bh[r], i = row_i[r];
        const long b = bh / H, h = bh % H, bg = b * Hkv + h / (H / Hkv);
        const int8_t* qrow = q_i8 + (bh * N + i) * (long)d;
        const float sq = q_scale[bh * nqb + i / ORACLE_QBLOCK];
        const long last = causal ? i : N - 1;
        float m = -INFINITY;
        double l = 0.0, rv = 0.0, rp = 0.0, vmax = 0.0;
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (int c = 0; c < d; ++c)
            for (long j = 0; j <= last; ++j) {
                double a = fabs(oracle_e4m3_decode(vt8[(bg * d + c) * (long)Np + j]));
                if (a > vmax) vmax = a;
            }
        for (long t0 = 0; t0 <= last; t0 += 128) {
            const int n = (int)((last - t0 + 1) < 128 ? (last - t0 + 1) : 128);   /* visible keys */
            float cb[2], t = -INFINITY;
            for (int blk = 0; blk < 2; ++blk) {
                const long kb = (t0 + 64 * blk) / ORACLE_KBLOCK;
                cb[blk] = kb < nkb ? (sq * k_scale[bg * nkb + kb]) * sl2 : 0.0f;
                int32_t mx = 0;
                int any = 0;
                for (int j = 64 * blk; j < 64 * blk + 64 && j < n; ++j) {
                    int32_t a = 0;
                    const int8_t* krow = k_i8 + (bg * N + t0 + j) * (long)d;
                    for (int c = 0; c < d; ++c) a += (int32_t)qrow[c] * (int32_t)krow[c];
                    s[j] = a;
                    if (!any || a > mx) mx = a;
                    any = 1;
                }
                if (any) {
                    const float tb = (float)mx * cb[blk];
                    if (tb > t) t = tb;
                }
            }
            if (t > m + 4.0f) {
                const double alpha = (m == -INFINITY) ? 0.0 : exp2((double)m - (double)t);
                l *= alpha;
                rv *= alpha;
                rp *= alpha;
                for (int c = 0; c < d; ++c) acc[c] *= alpha;
                m = t;
            }
            const float g = 4.0f - m;
            for (int j = 0; j < n; ++j) {
                const float y = fmaf((float)s[j], cb[j / 64], g);
                const float p = (float)exp2((double)y);
                ph[j] = oracle_ue4m3_decode(e4m3_with_risk(p, &step[j]));
            }
            for (int j = 0; j < n; ++j) {
                l += ph[j];
                for (int c = 0; c < d; ++c)
                    acc[c] += ph[j] * oracle_e4m3_decode(vt8[(bg * d + c) * (long)Np + t0 + j]);
                rv += step[j] * vmax;
                rp += step[j];
            }
        }
        double omax = 0.0;
        for (int c = 0; c < d; ++c) {
            out[r * d + c] = acc[c] * (double)v_scale[bg] / l;
            if (fabs(out[r * d + c]) > omax) omax = fabs(out[r * d + c]);
        }
        slack[r] = (rv * (double)v_scale[bg] + rp * omax) / l;
    }
    free(acc);
    return 0;
}
