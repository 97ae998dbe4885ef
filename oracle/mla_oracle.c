/*
 * Plain fp64 CPU oracle for paged MLA latent-attention decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this file.  It shares no code,
 * header, table or helper with the CUDA library, and the library never calls
 * it.
 *
 * What it computes (one query row = one (sequence b, query token t, head h)):
 *
 *   n      = number of cached positions the row may see
 *   kv_j   = dequantised 576-value row of position j, looked up through the
 *            page table: page = page_table[b][j / 16], slot = j % 16
 *   s_j    = sm_scale * ( q_lat . kv_j[0:512] + q_pe . kv_j[512:576] )
 *   M      = max_j s_j,   Z = sum_j exp(s_j - M),   lse = M + ln Z
 *   out[d] = sum_j exp(s_j - M) / Z * kv_j[d]          for d < 512
 *
 * Sources: the compressed KV history of 576 values per position and its
 * per-position byte count ("Inside Kimi K3 optimisation work", section 1,
 * DCP paragraph); 16-token pages ("Kimi K2.6 DFlash on 8x MI300X", hardware
 * stack, BLOCK_SIZE=16); every query head attends to the cached positions on
 * its own ("Inside Kimi K3 optimisation work", section 4, head padding);
 * partial answers carry normalisation information and merge exactly
 * (section 1, DCP; section 4, history split).  The 512 + 64 split of the 576
 * values, the value = latent reading and the per-token FP8 scale are the
 * plainest reading of the problem statement: the pages give only the
 * 576-value total and a dynamically computed FP8 scale.
 *
 * Visibility: without an explicit per-token count, query token t of a
 * sequence with ctx cached positions sits at position ctx - T + t (the last T
 * cached positions are the query tokens themselves) and sees every position
 * up to and including itself: n = ctx - T + t + 1.
 *
 * An empty visible set gives out = 0 and lse = -inf.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_PAGE 16
#define ORACLE_DL 512
#define ORACLE_DR 64
#define ORACLE_D (ORACLE_DL + ORACLE_DR)

enum { ORACLE_KV_BF16 = 0, ORACLE_KV_FP8 = 1 };

/* bfloat16 is the upper half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_f64(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* FP8 e4m3fn from its format definition: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); the single
 * pattern S.1111.111 is NaN; there is no infinity; largest finite is 448. */
double oracle_e4m3_to_f64(uint8_t byte) {
    int sign = byte >> 7;
    int e = (byte >> 3) & 0xF;
    int m = byte & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* FP8 e4m3fn encoding of a binary32 value, written from the same format
 * definition: round to nearest, ties to even, magnitudes above 448 clamped to
 * 448 (the cache writer clamps before it rounds), the sign kept (-0 -> 0x80).
 * Subnormal codes m = 0..7 step 2^-9; a subnormal that rounds up to 8 steps
 * is the smallest normal, whose code is also 8. */
uint8_t oracle_e4m3_encode(float q) {
    uint8_t sign = signbit(q) ? 0x80 : 0x00;
    double a = fabs((double)q);
    if (a > 448.0) a = 448.0;
    if (a < ldexp(1.0, -6)) {                   /* subnormal range, quantum 2^-9 */
        double n = a / ldexp(1.0, -9);          /* exact: a power-of-two scaling */
        double r = nearbyint(n);                /* default rounding: ties to even */
        return (uint8_t)(sign | (uint8_t)r);
    }
    int k;
    frexp(a, &k);                               /* a = f 2^k, f in [0.5, 1) */
    int e = k - 1;                              /* a in [2^e, 2^(e+1)) */
    double n = a / ldexp(1.0, e - 3);           /* in [8, 16), exact */
    double r = nearbyint(n);
    if (r == 16.0) {
        e += 1;
        r = 8.0;
    }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)r - 8)));
}

/* The cache writer for one token of an FP8 cache ("Kimi K2.6 DFlash on 8x
 * MI300X", comparison of FP8 and BF16 KV: the FP8 cache computes a dynamic
 * scale as it is written; here one fp32 scale per token):
 *   x_d = widen(bf16 value d), d < 576       (c_kv 0..511 then k_pe)
 *   scale = max_d |x_d| / 448 in binary32, or 1 when that is 0
 *   code_d = e4m3(clamp(x_d / scale, -448, 448)), the division in binary32. */
/* static_scale > 0: a per-tensor scale given by the caller replaces the
 * row's own (a static, calibrated scale). */
void oracle_quantize_row_e4m3(const uint16_t *row, uint8_t *codes, float *scale_out, float static_scale) {
    float x[ORACLE_D];
    float amax = 0.0f;
    for (int d = 0; d < ORACLE_D; ++d) {
        x[d] = (float)oracle_bf16_to_f64(row[d]);
        float ax = fabsf(x[d]);
        if (ax > amax) amax = ax;
    }
    float scale = amax / 448.0f;
    if (!(scale > 0.0f)) scale = 1.0f;
    if (static_scale > 0.0f) scale = static_scale;
    for (int d = 0; d < ORACLE_D; ++d) {
        float q = x[d] / scale;
        if (q > 448.0f) q = 448.0f;
        if (q < -448.0f) q = -448.0f;
        codes[d] = oracle_e4m3_encode(q);
    }
    *scale_out = scale;
}

/* Append: token t of sequence b (its c_kv and k_pe, bf16) is cached position
 * ctx_lens[b] - T + t, i.e. the context already counts the new tokens, as in
 * the decode.  Returns 0, or -1 if a context or page index is out of range
 * (nothing is written for such a token). */
int oracle_append_kv(int B, int T, const uint16_t *c_kv_new, const uint16_t *k_pe_new, void *kv_pages, int kv_dtype,
                     float *kv_scale, int kv_scale_per_tensor, int num_pages, const int32_t *page_table,
                     int page_table_stride, int max_pages, const int32_t *ctx_lens) {
    int rc = 0;
    for (int b = 0; b < B; ++b) {
        int ctx = ctx_lens[b];
        if (ctx < T || ctx > max_pages * ORACLE_PAGE) {
            rc = -1;
            continue;
        }
        for (int t = 0; t < T; ++t) {
            int pos = ctx - T + t;
            int page = page_table[(int64_t)b * page_table_stride + pos / ORACLE_PAGE];
            if (page < 0 || page >= num_pages) {
                rc = -1;
                continue;
            }
            int64_t slot = (int64_t)page * ORACLE_PAGE + pos % ORACLE_PAGE;
            uint16_t row[ORACLE_D];
            memcpy(row, c_kv_new + ((int64_t)b * T + t) * ORACLE_DL, ORACLE_DL * sizeof(uint16_t));
            memcpy(row + ORACLE_DL, k_pe_new + ((int64_t)b * T + t) * ORACLE_DR, ORACLE_DR * sizeof(uint16_t));
            if (kv_dtype == ORACLE_KV_BF16) {
                memcpy((uint16_t *)kv_pages + slot * ORACLE_D, row, sizeof row);
            } else {
                float s;
                oracle_quantize_row_e4m3(row, (uint8_t *)kv_pages + slot * ORACLE_D, &s,
                                         kv_scale_per_tensor ? kv_scale[0] : 0.0f);
                if (!kv_scale_per_tensor) kv_scale[slot] = s;
            }
        }
    }
    return rc;
}

typedef struct {
    int B, T, H;
    const uint16_t *q_lat;   /* [B,T,H,512] bf16 bits */
    const uint16_t *q_pe;    /* [B,T,H,64]  bf16 bits */
    const void *kv_pages;    /* [P,16,576] bf16 bits or e4m3fn bytes */
    int kv_dtype;
    const float *kv_scale;   /* [P,16] for FP8, or [1] with kv_scale_per_tensor; else NULL */
    int kv_scale_per_tensor;
    int num_pages;
    const int32_t *page_table;
    int page_table_stride;
    const int32_t *ctx_lens; /* [B] */
    const int32_t *vis_lens; /* [B,T] or NULL */
    double sm_scale;
} oracle_problem;

/* One dequantised KV value: element d of the row stored at (page, slot). */
static double kv_value(const oracle_problem *p, int64_t page, int slot, int d) {
    int64_t row = page * ORACLE_PAGE + slot;
    if (p->kv_dtype == ORACLE_KV_BF16) {
        const uint16_t *kv = (const uint16_t *)p->kv_pages;
        return oracle_bf16_to_f64(kv[row * ORACLE_D + d]);
    } else {
        const uint8_t *kv = (const uint8_t *)p->kv_pages;
        return oracle_e4m3_to_f64(kv[row * ORACLE_D + d]) * (double)p->kv_scale[p->kv_scale_per_tensor ? 0 : row];
    }
}

static int visible_count(const oracle_problem *p, int b, int t) {
    if (p->vis_lens) return p->vis_lens[(int64_t)b * p->T + t];
    return p->ctx_lens[b] - p->T + t + 1;
}

/* Returns 0, or a negative code when the row's inputs are inconsistent. */
static int decode_row(const oracle_problem *p, int64_t row, double *out, double *lse,
                      double *scores) {
    int h = (int)(row % p->H);
    int t = (int)((row / p->H) % p->T);
    int b = (int)(row / ((int64_t)p->H * p->T));
    int ctx = p->ctx_lens[b];
    int n = visible_count(p, b, t);
    const uint16_t *ql = p->q_lat + row * ORACLE_DL;
    const uint16_t *qp = p->q_pe + row * ORACLE_DR;

    if (ctx < 0 || n < 0 || n > ctx) return -2;
    for (int d = 0; d < ORACLE_DL; ++d) out[d] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return 0;
    }
    /* scores s_j over the visible positions, through the page table */
    for (int j = 0; j < n; ++j) {
        int32_t page = p->page_table[(int64_t)b * p->page_table_stride + j / ORACLE_PAGE];
        int slot = j % ORACLE_PAGE;
        double dot = 0.0;
        if (page < 0 || page >= p->num_pages) return -3;
        for (int d = 0; d < ORACLE_DL; ++d)
            dot += oracle_bf16_to_f64(ql[d]) * kv_value(p, page, slot, d);
        for (int d = 0; d < ORACLE_DR; ++d)
            dot += oracle_bf16_to_f64(qp[d]) * kv_value(p, page, slot, ORACLE_DL + d);
        scores[j] = p->sm_scale * dot;
    }
    double M = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (scores[j] > M) M = scores[j];
    double Z = 0.0;
    for (int j = 0; j < n; ++j) Z += exp(scores[j] - M);
    *lse = M + log(Z);
    /* out = softmax-weighted sum of the latent part of the visible rows */
    for (int j = 0; j < n; ++j) {
        int32_t page = p->page_table[(int64_t)b * p->page_table_stride + j / ORACLE_PAGE];
        int slot = j % ORACLE_PAGE;
        double w = exp(scores[j] - M) / Z;
        for (int d = 0; d < ORACLE_DL; ++d) out[d] += w * kv_value(p, page, slot, d);
    }
    return 0;
}

typedef struct {
    const oracle_problem *p;
    const int64_t *rows;     /* NULL: all rows */
    int64_t n_rows;
    double *out;
    double *lse;
    int64_t next;            /* shared work cursor */
    pthread_mutex_t lock;
    int status;
    int max_ctx;
} oracle_job;

static void *worker(void *arg) {
    oracle_job *job = (oracle_job *)arg;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(job->max_ctx > 0 ? job->max_ctx : 1));
    for (;;) {
        int64_t i;
        pthread_mutex_lock(&job->lock);
        i = job->next++;
        pthread_mutex_unlock(&job->lock);
        if (i >= job->n_rows) break;
        int64_t row = job->rows ? job->rows[i] : i;
        int rc = decode_row(job->p, row, job->out + i * ORACLE_DL, job->lse + i, scores);
        if (rc) {
            pthread_mutex_lock(&job->lock);
            if (!job->status) job->status = rc;
            pthread_mutex_unlock(&job->lock);
        }
    }
    free(scores);
    return NULL;
}

static int run_rows(const oracle_problem *p, const int64_t *rows, int64_t n_rows,
                    double *out, double *lse, int n_threads) {
    oracle_job job;
    int max_ctx = 0;
    int64_t total_rows = (int64_t)p->B * p->T * p->H;
    if (p->B <= 0 || p->T <= 0 || p->H <= 0) return -1;
    for (int b = 0; b < p->B; ++b)
        if (p->ctx_lens[b] > max_ctx) max_ctx = p->ctx_lens[b];
    for (int64_t i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= total_rows) return -1;
    memset(&job, 0, sizeof job);
    job.p = p;
    job.rows = rows;
    job.n_rows = n_rows;
    job.out = out;
    job.lse = lse;
    job.max_ctx = max_ctx;
    pthread_mutex_init(&job.lock, NULL);
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    for (int k = 0; k < n_threads; ++k) pthread_create(&th[k], NULL, worker, &job);
    for (int k = 0; k < n_threads; ++k) pthread_join(th[k], NULL);
    pthread_mutex_destroy(&job.lock);
    return job.status;
}

/* Decode every row (rows == NULL) or the listed flat rows b*T*H + t*H + h.
 * out: [n_rows, 512] fp64, lse: [n_rows] fp64.  Returns 0 on success. */
int oracle_mla_decode(int B, int T, int H, const uint16_t *q_lat, const uint16_t *q_pe,
                      const void *kv_pages, int kv_dtype, const float *kv_scale, int kv_scale_per_tensor,
                      int num_pages,
                      const int32_t *page_table, int page_table_stride, const int32_t *ctx_lens,
                      const int32_t *vis_lens, double sm_scale, const int64_t *rows,
                      int64_t n_rows, double *out, double *lse, int n_threads) {
    oracle_problem p;
    p.B = B;
    p.T = T;
    p.H = H;
    p.q_lat = q_lat;
    p.q_pe = q_pe;
    p.kv_pages = kv_pages;
    p.kv_dtype = kv_dtype;
    p.kv_scale = kv_scale;
    p.kv_scale_per_tensor = kv_scale_per_tensor;
    p.num_pages = num_pages;
    p.page_table = page_table;
    p.page_table_stride = page_table_stride;
    p.ctx_lens = ctx_lens;
    p.vis_lens = vis_lens;
    p.sm_scale = sm_scale;
    if (kv_dtype != ORACLE_KV_BF16 && kv_dtype != ORACLE_KV_FP8) return -1;
    if (kv_dtype == ORACLE_KV_FP8 && !kv_scale) return -1;
    if (!rows) n_rows = (int64_t)B * T * H;
    return run_rows(&p, rows, n_rows, out, lse, n_threads);
}

/* Merge n_parts partial results of the same rows, each normalised within its
 * own part and carrying that part's log-sum-exp:
 *   L = max_i lse_i,  w_i = exp(lse_i - L),  out = sum_i w_i out_i / sum_i w_i,
 *   lse = L + ln sum_i w_i.
 * Parts with lse = -inf weigh nothing; if every part is -inf the row is empty:
 * out = 0, lse = -inf.  A NaN lse in any part makes the row NaN (out and lse).
 * out_parts: [n_parts, rows, dv]; lse_parts: [n_parts, rows]. */
int oracle_mla_merge(int n_parts, int64_t rows, int dv, const double *out_parts,
                     const double *lse_parts, double *out, double *lse) {
    if (n_parts <= 0 || rows < 0 || dv <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        double L = -INFINITY;
        int poisoned = 0;
        for (int i = 0; i < n_parts; ++i) {
            double l = lse_parts[(int64_t)i * rows + r];
            if (isnan(l)) poisoned = 1;
            else if (l > L) L = l;
        }
        double *o = out + r * dv;
        /* a NaN normaliser (a part computed from invalid input) poisons the row,
           also when every part is NaN and no maximum exists */
        if (poisoned) {
            for (int d = 0; d < dv; ++d) o[d] = NAN;
            lse[r] = NAN;
            continue;
        }
        for (int d = 0; d < dv; ++d) o[d] = 0.0;
        if (L == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double W = 0.0;
        for (int i = 0; i < n_parts; ++i) {
            double l = lse_parts[(int64_t)i * rows + r];
            if (l == -INFINITY) continue;
            double w = exp(l - L);
            const double *oi = out_parts + ((int64_t)i * rows + r) * dv;
            W += w;
            for (int d = 0; d < dv; ++d) o[d] += w * oi[d];
        }
        for (int d = 0; d < dv; ++d) o[d] /= W;
        lse[r] = L + log(W);
    }
    return 0;
}
