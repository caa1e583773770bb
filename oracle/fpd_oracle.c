/*
 * fpd_oracle.c -- the CPU oracle for paged FP8 (E4M3) decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this library; the product path never calls it.
 * It shares no code with the CUDA kernels.
 *
 * What it computes, in fp64, for every sequence b and query head h.  The
 * operation is the one the grouped-nf4-gemm solutions page
 * "fp8-paged-attention-for-moe-serving" names (its title and summary): one
 * decode query per sequence attending, through a block table, to a paged
 * E4M3 K/V cache, with an optional sliding window, optional attention sinks
 * and a caller-chosen softmax scale.
 *
 *   g     = Hq / Hkv, kvh = h / g            (consecutive query heads share a
 *                                           KV head: GQA)
 *   L     = seq_lens[b]
 *   start = window_left >= 0 ? max(0, L - 1 - window_left) : 0
 *           (FlashInfer's window_left, passed through by the vLLM FlashInfer
 *            backend in the NVFP4 KV-cache gist: the query sees itself and the
 *            window_left keys before it)
 *   for j in [start, L):   page = block_table[b][j / bt], slot = j % bt
 *       k_j = k_scale * e4m3(k_cache[page][slot][kvh][:])
 *       v_j = v_scale * e4m3(v_cache[page][slot][kvh][:])
 *       s_j = sm_scale * sum_d q[b][h][d] * k_j[d]
 *   sigma = sinks ? sinks[h] : -inf         (a sink is a logit with no value:
 *                                           it only enters the denominator)
 *   m   = max(max_j s_j, sigma)
 *   Z   = sum_j exp(s_j - m) + exp(sigma - m)
 *   out = sum_j exp(s_j - m) / Z * v_j
 *   lse = m + ln Z                          (natural log, sink included)
 *
 * Per-tensor scales: the cache writer of the gist stores x / scale, so a stored
 * code decodes to e4m3(code) * scale.
 *
 * E4M3 is the OCP "e4m3fn" format (the CUDA type __nv_fp8_e4m3 named in the
 * gist's quantisation helpers): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent 0 is subnormal; S.1111.111 is NaN; there are no infinities.
 *
 * The file also holds the oracle of the FP8 cache write that fills such a
 * cache (fpd_oracle_cache_write, below the E4M3 codec), and the merge of
 * partial results over disjoint key sets that context-parallel decode needs
 * (fpd_oracle_merge, at the end).
 *
 * Several query tokens per sequence (speculative / multi-token decode): the
 * sequence's q_len newest tokens are queries.  Query i (0 <= i < q_len) sits at
 * position p = L - q_len + i and sees the keys j in [start_i, p] (causal), with
 * start_i = max(0, p - window_left) under a window; q, out and lse gain a
 * q_len axis after B.  q_len = 1 is the formula above.
 *
 * Interface variants (the layouts and forms the gist's FlashInfer backend and
 * cache writer use): the query may be IEEE fp16 instead of bf16, and the
 * pages may be head-major, [num_blocks, Hkv, bt, D] ("HND"), instead of
 * token-major [num_blocks, bt, Hkv, D] ("NHD"); only the addressing of
 * element [page][slot][kvh][d] changes.
 *
 * NVFP4 pages (the format of the NVFP4 KV-cache serving gist, its cache writer
 * and the FlashInfer paged reader it routes to): each K or V element is an
 * E2M1 code (4 bits; element 2i of a row in the low nibble of byte i) times
 * the E4M3 scale of its block of 16 elements, times the per-tensor scale:
 *   k_j[d] = k_scale * e2m1(code) * e4m3(sf[d / 16])
 * Pages are head-major; a page holds a data region [Hkv][bt][D/2] and a
 * scale region [Hkv][bt][D/16] per side, at caller-given page strides.
 *
 * Degenerate cases: L == 0 gives out = 0 and lse = sigma (-inf without sinks).
 * A stored NaN code inside the attended range propagates NaN (plain
 * arithmetic); codes outside the attended range are never read.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E4M3 (e4m3fn) code -> exact real value. */
double fpd_oracle_e4m3_to_f64(uint8_t code)
{
    const int sign = code >> 7;
    const int expo = (code >> 3) & 0xF;
    const int mant = code & 0x7;
    double mag;
    if (expo == 0xF && mant == 0x7)
        return NAN;
    if (expo == 0)
        mag = ldexp((double)mant / 8.0, -6);          /* subnormal: 2^-6 * m/8 */
    else
        mag = ldexp(1.0 + (double)mant / 8.0, expo - 7); /* normal: 2^(e-7) * (1+m/8) */
    return sign ? -mag : mag;
}

/* bf16 bit pattern -> real value (bf16 is the top half of an IEEE binary32). */
double fpd_oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 bit pattern -> real value: 1 sign, 5 exponent (bias 15), 10
 * mantissa bits; exponent 0 is subnormal (2^-14 * m / 1024); exponent 31 is
 * inf (m = 0) or NaN. */
double fpd_oracle_f16_to_f64(uint16_t bits)
{
    const int s = bits >> 15, e = (bits >> 10) & 0x1F, m = bits & 0x3FF;
    const double sign = s ? -1.0 : 1.0;
    if (e == 0x1F)
        return m ? NAN : sign * INFINITY;
    if (e == 0)
        return sign * ldexp((double)m / 1024.0, -14);
    return sign * ldexp(1.0 + (double)m / 1024.0, e - 15);
}

/* E2M1 code (low 4 bits) -> real value: 1 sign, 2 exponent (bias 1), 1
 * mantissa bit; exponent 0 is subnormal (0 or 0.5).  Values 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6 and their negatives; no inf or NaN. */
double fpd_oracle_e2m1_to_f64(uint8_t code)
{
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Real value -> E2M1 code: nearest value, ties to the even code, saturating
 * at +-6; the sign of zero is kept.  A search over the 8 codes, which are
 * increasing in value.  (NaN has no E2M1 code; it gives +0 here.) */
uint8_t fpd_oracle_f64_to_e2m1(double x)
{
    const uint8_t sign = signbit(x) ? 0x8 : 0x0;
    const double a = fabs(x);
    int best = 0, c;
    double best_d;
    if (isnan(x))
        return 0;
    if (a >= 6.0)
        return (uint8_t)(sign | 0x7);
    best_d = a;
    for (c = 1; c <= 7; ++c) {
        const double d = fabs(a - fpd_oracle_e2m1_to_f64((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* Byte offset of element [page][slot][kvh][0]: token-major pages
 * [num_blocks, bt, Hkv, D], or head-major [num_blocks, Hkv, bt, D] (hnd). */
static size_t page_row(int hnd, int page, int slot, int kvh, int bt, int Hkv, int D)
{
    if (hnd)
        return (((size_t)page * Hkv + kvh) * bt + slot) * (size_t)D;
    return (((size_t)page * bt + slot) * Hkv + kvh) * (size_t)D;
}

/*
 * Real value -> E4M3 code: the nearest representable value, ties to the even
 * code (mantissa LSB 0), saturating to +-448 (S.1111.110) beyond the largest
 * finite value, so +-inf saturate too; NaN gives the NaN code S.1111.111.
 * The sign of zero is kept.  Written as the definition: a search over the
 * 127 non-negative finite codes, which are increasing in value.
 */
uint8_t fpd_oracle_f64_to_e4m3(double x)
{
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    int best = 0, c;
    double best_d;
    if (isnan(x))
        return (uint8_t)(sign | 0x7F);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    best_d = a; /* distance to code 0 (+0) */
    for (c = 1; c <= 0x7E; ++c) {
        const double d = fabs(a - fpd_oracle_e4m3_to_f64((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(sign | best);
}

/*
 * FP8 KV-cache write (test infrastructure, like everything in this file).
 * The per-tensor quantisation of the cache writer in the NVFP4 KV-cache gist
 * (its standalone writer kernel and host wrapper): the scale's reciprocal is
 * taken in fp32 and every element is multiplied by it in fp32 before
 * rounding, i.e. stored = e4m3_rne_sat(float(x) * (1.0f / scale)).  Token t
 * goes to slot s = slot_mapping[t] = page * bt + offset of the
 * [num_blocks, bt, Hkv, D] caches; a negative slot is a padded token and is
 * skipped.  key and value are bf16 bit patterns [num_tokens, Hkv, D] with a
 * token stride of key_stride / value_stride elements.  hnd selects head-major
 * pages [num_blocks, Hkv, bt, D].  Returns the number of slots past the end of
 * the cache (skipped), or -1 for a bad argument.
 */
int fpd_oracle_cache_write_x(const uint16_t *key, const uint16_t *value,
                             const int64_t *slot_mapping, int num_tokens, int Hkv, int D,
                             long key_stride, long value_stride, float k_scale, float v_scale,
                             uint8_t *k_cache, uint8_t *v_cache, int num_blocks, int bt, int hnd)
{
    const float kr = 1.0f / k_scale, vr = 1.0f / v_scale;
    const int64_t n_slots = (int64_t)num_blocks * bt;
    int bad = 0, t, h, d;
    if (num_tokens < 0 || Hkv <= 0 || D <= 0 || num_blocks <= 0 || bt <= 0)
        return -1;
    for (t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= n_slots) {
            ++bad;
            continue;
        }
        for (h = 0; h < Hkv; ++h) {
            for (d = 0; d < D; ++d) {
                const size_t dst =
                    page_row(hnd, (int)(slot / bt), (int)(slot % bt), h, bt, Hkv, D) + d;
                const float xk = (float)fpd_oracle_bf16_to_f64(key[t * key_stride + (long)h * D + d]);
                const float xv = (float)fpd_oracle_bf16_to_f64(value[t * value_stride + (long)h * D + d]);
                const float yk = xk * kr, yv = xv * vr; /* fp32 products, round to nearest */
                k_cache[dst] = fpd_oracle_f64_to_e4m3((double)yk);
                v_cache[dst] = fpd_oracle_f64_to_e4m3((double)yv);
            }
        }
    }
    return bad;
}

/* Token-major pages (the default layout). */
int fpd_oracle_cache_write(const uint16_t *key, const uint16_t *value, const int64_t *slot_mapping,
                           int num_tokens, int Hkv, int D, long key_stride, long value_stride,
                           float k_scale, float v_scale, uint8_t *k_cache, uint8_t *v_cache,
                           int num_blocks, int bt)
{
    return fpd_oracle_cache_write_x(key, value, slot_mapping, num_tokens, Hkv, D, key_stride,
                                    value_stride, k_scale, v_scale, k_cache, v_cache,
                                    num_blocks, bt, 0);
}

typedef struct {
    const uint16_t *q;
    const uint8_t *k_cache, *v_cache;
    const int32_t *block_table, *seq_lens;
    int B, Hq, Hkv, D, num_blocks, bt, max_blocks, q_len;
    double k_scale, v_scale, sm_scale;
    int window_left;
    int q_f16;           /* q holds IEEE fp16 bit patterns instead of bf16 */
    int kv_hnd;          /* head-major pages [num_blocks, Hkv, bt, D] */
    int nvfp4;           /* NVFP4 pages: k_cache/v_cache hold the E2M1 data */
    const uint8_t *k_sf, *v_sf;           /* NVFP4 block scales (E4M3) */
    long data_page_stride, sf_page_stride; /* NVFP4 bytes between pages */
    const float *sinks;
    double *out, *lse;
    const int32_t *rows; /* list of (b * q_len + i) * Hq + h to compute, or NULL for all */
    int n_rows;
    int next;            /* work counter */
    int status;
    pthread_mutex_t mu;
} job_t;

/* Byte offset of element [page][slot][kvh][0] in the job's cache layout. */
static size_t cache_row(const job_t *J, int page, int slot, int kvh)
{
    return page_row(J->kv_hnd, page, slot, kvh, J->bt, J->Hkv, J->D);
}

/* NVFP4 element [page][slot][kvh][d] of one side without the per-tensor scale:
 * data [page][kvh][slot][D/2] (two codes per byte, even d low), block scales
 * [page][kvh][slot][D/16]. */
static double nvfp4_elem(const job_t *J, const uint8_t *data, const uint8_t *sf, int page,
                         int slot, int kvh, int d)
{
    const size_t row = (size_t)kvh * J->bt + slot;
    const uint8_t byte = data[(size_t)page * J->data_page_stride + row * (J->D / 2) + d / 2];
    const uint8_t code = (d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
    const uint8_t sfc = sf[(size_t)page * J->sf_page_stride + row * (J->D / 16) + d / 16];
    return fpd_oracle_e2m1_to_f64(code) * fpd_oracle_e4m3_to_f64(sfc);
}

static double q_value(const job_t *J, uint16_t bits)
{
    return J->q_f16 ? fpd_oracle_f16_to_f64(bits) : fpd_oracle_bf16_to_f64(bits);
}

static int one_row(const job_t *J, int row, double *s, double *acc)
{
    const int Q = J->q_len;
    const int b = row / (Q * J->Hq), i = (row / J->Hq) % Q, h = row % J->Hq;
    const int g = J->Hq / J->Hkv;
    const int kvh = h / g;
    const int D = J->D;
    const int L = J->seq_lens[b];
    double *o = J->out + (size_t)row * D;
    const uint16_t *qr = J->q + (size_t)row * D;
    const double sigma = J->sinks ? (double)J->sinks[h] : -INFINITY;
    int p, start, end, j, d;
    double m, Z;

    if (L < 0 || L > J->max_blocks * J->bt)
        return -2;
    p = L - Q + i;              /* the query's own position; it sees keys up to p */
    end = p + 1 > 0 ? p + 1 : 0;
    start = (J->window_left >= 0) ? p - J->window_left : 0;
    if (start < 0)
        start = 0;

    /* logits */
    m = sigma;
    for (j = start; j < end; ++j) {
        const int page = J->block_table[(size_t)b * J->max_blocks + j / J->bt];
        const uint8_t *kr;
        double dot = 0.0;
        if (page < 0 || page >= J->num_blocks)
            return -3;
        if (J->nvfp4) {
            for (d = 0; d < D; ++d)
                dot += q_value(J, qr[d]) *
                       (J->k_scale * nvfp4_elem(J, J->k_cache, J->k_sf, page, j % J->bt, kvh, d));
        } else {
        kr = J->k_cache + cache_row(J, page, j % J->bt, kvh);
        for (d = 0; d < D; ++d)
            dot += q_value(J, qr[d]) * (J->k_scale * fpd_oracle_e4m3_to_f64(kr[d]));
        }
        s[j - start] = J->sm_scale * dot;
        if (s[j - start] > m || isnan(s[j - start]))
            m = s[j - start];
    }

    /* softmax weights, denominator and weighted sum of values */
    for (d = 0; d < D; ++d)
        acc[d] = 0.0;
    Z = 0.0;
    if (m == -INFINITY) { /* no keys and no sink */
        for (d = 0; d < D; ++d)
            o[d] = 0.0;
        J->lse[row] = -INFINITY;
        return 0;
    }
    for (j = start; j < end; ++j) {
        const int page = J->block_table[(size_t)b * J->max_blocks + j / J->bt];
        const uint8_t *vr = J->v_cache + cache_row(J, page, j % J->bt, kvh);
        const double p = exp(s[j - start] - m);
        Z += p;
        if (J->nvfp4) {
            for (d = 0; d < D; ++d)
                acc[d] += p * (J->v_scale *
                               nvfp4_elem(J, J->v_cache, J->v_sf, page, j % J->bt, kvh, d));
        } else {
        for (d = 0; d < D; ++d)
            acc[d] += p * (J->v_scale * fpd_oracle_e4m3_to_f64(vr[d]));
        }
    }
    Z += exp(sigma - m);
    for (d = 0; d < D; ++d)
        o[d] = acc[d] / Z;
    J->lse[row] = m + log(Z);
    return 0;
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int total = J->rows ? J->n_rows : J->B * J->q_len * J->Hq;
    int maxL = J->max_blocks * J->bt;
    double *s = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)J->D);
    for (;;) {
        int i, row, st;
        pthread_mutex_lock(&J->mu);
        i = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (i >= total)
            break;
        row = J->rows ? J->rows[i] : i;
        st = one_row(J, row, s, acc);
        if (st != 0) {
            pthread_mutex_lock(&J->mu);
            if (J->status == 0)
                J->status = st;
            pthread_mutex_unlock(&J->mu);
        }
    }
    free(s);
    free(acc);
    return NULL;
}

/*
 * Decode attention over the paged cache, q_len query tokens per sequence.
 *   q            bf16 bits [B, q_len, Hq, D]
 *   k/v_cache    E4M3 codes [num_blocks, bt, Hkv, D]
 *   block_table  [B, max_blocks], seq_lens [B] (including the q_len new tokens)
 *   sinks        float [Hq] or NULL
 *   out          double [B * q_len * Hq, D]  (only the listed rows are written)
 *   lse          double [B * q_len * Hq]
 *   rows/n_rows  rows ((b * q_len + i) * Hq + h) to compute; NULL computes all.
 *   n_threads    worker threads (<= 0: 1)
 *   q_f16        q holds IEEE fp16 bit patterns instead of bf16
 *   kv_hnd       the caches are head-major [num_blocks, Hkv, bt, D]
 * Returns 0, -1 for bad shapes, -2 for a sequence length outside
 * [0, max_blocks * bt], -3 for a block-table entry outside [0, num_blocks).
 */
int fpd_oracle_decode_x(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        int B, int q_len, int Hq, int Hkv, int D, int num_blocks, int bt,
                        int max_blocks, double k_scale, double v_scale, double sm_scale,
                        int window_left, const float *sinks, double *out, double *lse,
                        const int32_t *rows, int n_rows, int n_threads, int q_f16, int kv_hnd)
{
    job_t J;
    pthread_t *th;
    int t, i;
    if (B < 0 || q_len < 1 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || bt <= 0 ||
        max_blocks < 0 || num_blocks < 0)
        return -1;
    if (rows) {
        for (i = 0; i < n_rows; ++i)
            if (rows[i] < 0 || rows[i] >= B * q_len * Hq)
                return -1;
    }
    memset(&J, 0, sizeof J);
    J.q = q; J.k_cache = k_cache; J.v_cache = v_cache;
    J.block_table = block_table; J.seq_lens = seq_lens;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.num_blocks = num_blocks; J.bt = bt;
    J.max_blocks = max_blocks; J.q_len = q_len;
    J.k_scale = k_scale; J.v_scale = v_scale; J.sm_scale = sm_scale;
    J.window_left = window_left; J.sinks = sinks; J.out = out; J.lse = lse;
    J.q_f16 = q_f16; J.kv_hnd = kv_hnd;
    J.rows = rows; J.n_rows = n_rows;
    pthread_mutex_init(&J.mu, NULL);
    if (n_threads < 1)
        n_threads = 1;
    th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (t = 0; t < n_threads; ++t)
        pthread_create(&th[t], NULL, worker, &J);
    for (t = 0; t < n_threads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return J.status;
}

/*
 * Decode over NVFP4 pages (head-major).  k_data / v_data: E2M1 codes,
 * [page][kvh][slot][D/2] bytes at data_page_stride bytes per page; k_sf / v_sf:
 * E4M3 block scales [page][kvh][slot][D/16] at sf_page_stride bytes per page
 * (the writer's page [K data | K scales | V data | V scales] is four such
 * pointers with one stride).  Everything else as fpd_oracle_decode_x.
 */
int fpd_oracle_decode_nvfp4(const uint16_t *q, const uint8_t *k_data, const uint8_t *k_sf,
                            const uint8_t *v_data, const uint8_t *v_sf, long data_page_stride,
                            long sf_page_stride, const int32_t *block_table,
                            const int32_t *seq_lens, int B, int q_len, int Hq, int Hkv, int D,
                            int num_blocks, int bt, int max_blocks, double k_scale,
                            double v_scale, double sm_scale, int window_left,
                            const float *sinks, double *out, double *lse, const int32_t *rows,
                            int n_rows, int n_threads, int q_f16)
{
    job_t J;
    pthread_t *th;
    int t, i;
    if (B < 0 || q_len < 1 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || D % 16 != 0 ||
        bt <= 0 || max_blocks < 0 || num_blocks < 0 || data_page_stride <= 0 ||
        sf_page_stride <= 0)
        return -1;
    if (rows) {
        for (i = 0; i < n_rows; ++i)
            if (rows[i] < 0 || rows[i] >= B * q_len * Hq)
                return -1;
    }
    memset(&J, 0, sizeof J);
    J.q = q; J.k_cache = k_data; J.v_cache = v_data; J.k_sf = k_sf; J.v_sf = v_sf;
    J.nvfp4 = 1; J.kv_hnd = 1;
    J.data_page_stride = data_page_stride; J.sf_page_stride = sf_page_stride;
    J.block_table = block_table; J.seq_lens = seq_lens;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.num_blocks = num_blocks; J.bt = bt;
    J.max_blocks = max_blocks; J.q_len = q_len;
    J.k_scale = k_scale; J.v_scale = v_scale; J.sm_scale = sm_scale;
    J.window_left = window_left; J.sinks = sinks; J.out = out; J.lse = lse;
    J.q_f16 = q_f16;
    J.rows = rows; J.n_rows = n_rows;
    pthread_mutex_init(&J.mu, NULL);
    if (n_threads < 1)
        n_threads = 1;
    th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (t = 0; t < n_threads; ++t)
        pthread_create(&th[t], NULL, worker, &J);
    for (t = 0; t < n_threads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return J.status;
}

/*
 * NVFP4 KV-cache write: the per-block quantisation of the gist's NVFP4 cache
 * writer (its writer kernel and quantisation helper), with the reciprocals
 * taken exactly in fp32 where the gist uses approximate ones:
 *   gs    = 1 / scale                         (the per-tensor "global" scale)
 *   sf    = e4m3_rne_sat((amax16 * (1/6)) * gs)   amax16 = max |x| of 16 elements
 *   osc   = sf == 0 ? 0 : 1 / (e4m3(sf) * (1 / gs))
 *   code  = e2m1_rne_sat(x * osc)
 * every product and reciprocal rounded to fp32.  Token t goes to slot
 * s = slot_mapping[t] (page s / bt, in-page slot s % bt); negative slots are
 * skipped, slots past the end counted and skipped.  Layout as in
 * fpd_oracle_decode_nvfp4.  Returns the count of out-of-range slots, or -1.
 */
int fpd_oracle_cache_write_nvfp4(const uint16_t *key, const uint16_t *value,
                                 const int64_t *slot_mapping, int num_tokens, int Hkv, int D,
                                 long key_stride, long value_stride, float k_scale,
                                 float v_scale, uint8_t *k_data, uint8_t *k_sf, uint8_t *v_data,
                                 uint8_t *v_sf, long data_page_stride, long sf_page_stride,
                                 int num_blocks, int bt)
{
    const int64_t n_slots = (int64_t)num_blocks * bt;
    int bad = 0, t, side, h, blk, i;
    if (num_tokens < 0 || Hkv <= 0 || D <= 0 || D % 16 != 0 || num_blocks <= 0 || bt <= 0)
        return -1;
    for (t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        int page, off;
        if (slot < 0)
            continue;
        if (slot >= n_slots) {
            ++bad;
            continue;
        }
        page = (int)(slot / bt);
        off = (int)(slot % bt);
        for (side = 0; side < 2; ++side) {
            const uint16_t *src = side ? value + t * value_stride : key + t * key_stride;
            const float gs = 1.0f / (side ? v_scale : k_scale);
            uint8_t *data = side ? v_data : k_data;
            uint8_t *sf = side ? v_sf : k_sf;
            for (h = 0; h < Hkv; ++h) {
                const size_t row = (size_t)h * bt + off;
                for (blk = 0; blk < D / 16; ++blk) {
                    float x[16], amax = 0.0f, sf_f, sf_v, osc;
                    uint8_t sfc, codes[16];
                    for (i = 0; i < 16; ++i) {
                        x[i] = (float)fpd_oracle_bf16_to_f64(src[(long)h * D + blk * 16 + i]);
                        if (fabsf(x[i]) > amax)
                            amax = fabsf(x[i]);
                    }
                    sf_f = (amax * (1.0f / 6.0f)) * gs;
                    sfc = fpd_oracle_f64_to_e4m3((double)sf_f);
                    sf_v = (float)fpd_oracle_e4m3_to_f64(sfc);
                    osc = sf_v == 0.0f ? 0.0f : 1.0f / (sf_v * (1.0f / gs));
                    for (i = 0; i < 16; ++i) {
                        const float y = x[i] * osc;
                        codes[i] = fpd_oracle_f64_to_e2m1((double)y);
                    }
                    for (i = 0; i < 8; ++i)
                        data[(size_t)page * data_page_stride + row * (D / 2) + blk * 8 + i] =
                            (uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4));
                    sf[(size_t)page * sf_page_stride + row * (D / 16) + blk] = sfc;
                }
            }
        }
    }
    return bad;
}

/* bf16 q, token-major pages. */
int fpd_oracle_decode_q(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        int B, int q_len, int Hq, int Hkv, int D, int num_blocks, int bt,
                        int max_blocks, double k_scale, double v_scale, double sm_scale,
                        int window_left, const float *sinks, double *out, double *lse,
                        const int32_t *rows, int n_rows, int n_threads)
{
    return fpd_oracle_decode_x(q, k_cache, v_cache, block_table, seq_lens, B, q_len, Hq, Hkv,
                               D, num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                               window_left, sinks, out, lse, rows, n_rows, n_threads, 0, 0);
}

/* One query token per sequence: q bf16 bits [B, Hq, D]. */
int fpd_oracle_decode(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                      const int32_t *block_table, const int32_t *seq_lens,
                      int B, int Hq, int Hkv, int D, int num_blocks, int bt, int max_blocks,
                      double k_scale, double v_scale, double sm_scale, int window_left,
                      const float *sinks, double *out, double *lse,
                      const int32_t *rows, int n_rows, int n_threads)
{
    return fpd_oracle_decode_q(q, k_cache, v_cache, block_table, seq_lens, B, 1, Hq, Hkv, D,
                               num_blocks, bt, max_blocks, k_scale, v_scale, sm_scale,
                               window_left, sinks, out, lse, rows, n_rows, n_threads);
}

/*
 * The merge of partial results (context-parallel decode).  When the keys of a
 * row are split into R disjoint parts, part r giving the attention over its
 * own keys without a sink, O_r = sum_{j in r} e^(s_j - m_r) v_j / Z_r and
 * lse_r = m_r + ln Z_r, the attention over all keys follows from the split-KV
 * merge of partial O and LSE (FlashInfer PR #5591, Summary), since
 * e^(lse_r) = sum_{j in r} e^(s_j):
 *   M   = max(max_r lse_r, sigma)
 *   Z   = sum_r e^(lse_r - M) + e^(sigma - M)
 *   out = sum_r e^(lse_r - M) O_r / Z,   lse = M + ln Z
 * A part with no key (lse_r = -inf) weighs nothing; with no part and no sink
 * out = 0 and lse = -inf, as in the decode.
 *   o_parts [R][rows][D], lse_parts [R][rows]; row = (token, head), head
 *   innermost, so its sink is sinks[row % Hq].
 */
void fpd_oracle_merge(const double *o_parts, const double *lse_parts, int R, long rows, int D,
                      int Hq, const float *sinks, double *out, double *lse)
{
    long row;
    int r, d;
    for (row = 0; row < rows; ++row) {
        const double sigma = sinks ? (double)sinks[row % Hq] : -INFINITY;
        double M = sigma, Z = 0.0;
        double *o = out + (size_t)row * D;
        for (r = 0; r < R; ++r)
            if (lse_parts[(size_t)r * rows + row] > M)
                M = lse_parts[(size_t)r * rows + row];
        for (d = 0; d < D; ++d)
            o[d] = 0.0;
        if (M == -INFINITY) {
            lse[row] = -INFINITY;
            continue;
        }
        for (r = 0; r < R; ++r) {
            const double l = lse_parts[(size_t)r * rows + row];
            const double w = l == -INFINITY ? 0.0 : exp(l - M);
            Z += w;
            for (d = 0; d < D; ++d)
                o[d] += w * o_parts[((size_t)r * rows + row) * D + d];
        }
        Z += exp(sigma - M);
        for (d = 0; d < D; ++d)
            o[d] /= Z;
        lse[row] = M + log(Z);
    }
}
