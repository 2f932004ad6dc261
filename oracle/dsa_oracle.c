/*
 * dsa_oracle.c -- float64 CPU oracle for the DSA sparse-attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; the two only read the same
 * seeded input bytes.
 *
 * What it computes, step by step, in the order the pages give them:
 *
 *  1. Lightning Indexer relevance scoring with head-weight weighting.
 *     "Day0 Adaptation and Performance Optimization for Novel Long-Sequence
 *     Reasoning Models", section 1 (Sparse Index Branch) and section 3 (the
 *     index stage fuses relevance scoring, head-weight weighting and Top-K);
 *     "Day0 Adaptation and Sparse Attention Optimization for Long-Sequence LLM
 *     Inference", section 4 (index generation = scoring, multi-head weight
 *     aggregation, Top-K).  The pages give no formula; the gate used here is
 *     the ReLU form of the Lightning Indexer:
 *         score(t, s) = sum_h w[t,h] * max(0, sum_d q[t,h,d] * k[s,d])
 *     for every position s the query token t can see (0..pos(t), causal).
 *     fp8 keys: k[s,d] = e4m3(code[s,d]) * scale[s, d/64] (one fp32 scale per
 *     64 contiguous elements of a key; "Day0 Adaptation and Performance
 *     Optimization ...", section 4, every N elements share a scaling factor).
 *     MXFP8 index queries and keys (same page, section 4: full quantization of
 *     index Q/K in the MXFP8 format, every 32 elements share a scaling factor;
 *     "Optimizing and Deploying Ultra-Long Sequence Inference Architectures",
 *     section II item 1): x[d] = e4m3(code[d]) * 2^(e[d/32] - 127), e an
 *     8-bit power-of-two scale shared by 32 contiguous elements of one vector.
 *
 *  2. Top-K selection.  "Large Model Inference Acceleration: Day-0
 *     Adaptation ...", section 1.1 (a Top-K pass picks the most important
 *     positions).  Done here as a FULL SORT of the visible positions by
 *     (score descending, position ascending) -- the lower position wins a
 *     tie -- keeping the first min(K, visible).  The kept set is written in
 *     ascending position order and padded with -1.
 *
 *  3. Sparse Flash Attention over the selected rows of the MLA latent cache.
 *     "Day0 Adaptation and Sparse Attention Optimization ...", section 4
 *     (the sparse read stage gathers the selected KV entries and computes
 *     attention); "Optimizing and Deploying Ultra-Long Sequence Inference
 *     Architectures", section I.  Each cache row is [512 latent | 64 RoPE];
 *     the key is the whole 576-wide row, the value is the 512-wide latent:
 *         l_j  = sm_scale * sum_{d<576} q[t,g,d] * kv[s_j,d]
 *         p_j  = exp(l_j - max l) / sum_i exp(l_i - max l)
 *         o    = sum_j p_j * kv[s_j, 0:512],   lse = max l + ln sum_i exp(l_i - max l)
 *     Rows with index -1 are skipped.
 *
 *  4. Indexer prolog (input preparation of the index stage).  "Day0
 *     Adaptation and Performance Optimization ...", section 3 (query
 *     projection, key RMS normalization, query quantization, head-weight
 *     projection) and section 4 (projections kept in bf16, index Q/K in
 *     MXFP8); "Large Model Inference Acceleration ...", section 1.2.  The
 *     projections and the normalized key are returned in float64; the
 *     encoders (e4m3fn, MXFP8 groups of 32, e4m3fn with one fp32 scale per
 *     64) turn them into the stored formats.
 *
 * All arithmetic is IEEE float64, no fused multiply-add contraction
 * (built with -ffp-contract=off), summation in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK 64
#define ORACLE_DQK 576
#define ORACLE_DV 512

/* bf16 bits -> double: the bf16 value is the top half of a float32. */
static double bf16_to_f64(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* MX shared scale (8 exponent bits, no mantissa) -> double: 2^(e - 127);
 * 0xFF is NaN (the generator never produces it). */
double oracle_e8m0_to_f64(uint8_t e) {
    if (e == 0xFF) return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* OCP e4m3fn code -> double.  Sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN (returned as
 * NaN; the generator never produces it). */
double oracle_e4m3_to_f64(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

typedef struct {
    int32_t B, T, H_I, D_I, K;
    int32_t key_fp8;                 /* 0: bf16 keys, 1: e4m3 codes + fp32 scales, 2: MXFP8 */
    const int32_t* seq_lens;         /* [B] */
    const int32_t* cu_q;             /* [B+1] */
    const int32_t* block_table;      /* [B, max_blocks] */
    int32_t max_blocks;
    const uint16_t* q_idx;           /* [T, H_I, D_I] bf16 bits */
    const float* w;                  /* [T, H_I] */
    const void* k_idx;               /* [nblk, 64, D_I] bf16 bits or u8 codes */
    const float* k_scale;            /* [nblk, 64, D_I/64] fp32, [nblk, 64, D_I/32] u8 (MXFP8) or NULL */
    int32_t q_mx;                    /* 1: q_idx holds e4m3 codes [T, H_I, D_I] (MXFP8 queries) */
    const uint8_t* q_scale;          /* [T, H_I, D_I/32] shared scales of MXFP8 queries, or NULL */
} oracle_indexer_args;

/* Sequence and absolute position of query token t. */
static void token_place(const int32_t* cu_q, const int32_t* seq_lens, int B, int t,
                        int* b_out, int64_t* pos_out) {
    int b = 0;
    while (b + 1 < B + 1 && cu_q[b + 1] <= t) b++;
    int nq = cu_q[b + 1] - cu_q[b];
    *b_out = b;
    *pos_out = (int64_t)seq_lens[b] - nq + (t - cu_q[b]);
}

static int64_t phys_row(const oracle_indexer_args* a, int b, int64_t pos) {
    int64_t blk = a->block_table[(int64_t)b * a->max_blocks + pos / ORACLE_BLOCK];
    return blk * ORACLE_BLOCK + pos % ORACLE_BLOCK;
}

/* Key element d of logical position pos of sequence b, as a double. */
static double key_elem(const oracle_indexer_args* a, int64_t row, int d) {
    if (!a->key_fp8) {
        const uint16_t* k = (const uint16_t*)a->k_idx;
        return bf16_to_f64(k[row * a->D_I + d]);
    } else if (a->key_fp8 == 2) {
        /* MXFP8: the code times the shared scale of its 32-element group */
        const uint8_t* k = (const uint8_t*)a->k_idx;
        const uint8_t* e = (const uint8_t*)a->k_scale;
        return oracle_e4m3_to_f64(k[row * a->D_I + d]) * oracle_e8m0_to_f64(e[row * (a->D_I / 32) + d / 32]);
    } else {
        const uint8_t* k = (const uint8_t*)a->k_idx;
        double sc = (double)a->k_scale[row * (a->D_I / 64) + d / 64];
        return oracle_e4m3_to_f64(k[row * a->D_I + d]) * sc;
    }
}

/* Query element d of head h of token t, as a double: bf16 bits, or (MXFP8
 * queries) the code times the shared scale of its 32-element group. */
static double query_elem(const oracle_indexer_args* a, int t, int h, int d) {
    int64_t i = ((int64_t)t * a->H_I + h) * a->D_I + d;
    if (!a->q_mx) return bf16_to_f64(a->q_idx[i]);
    const uint8_t* qc = (const uint8_t*)a->q_idx;
    return oracle_e4m3_to_f64(qc[i]) *
           oracle_e8m0_to_f64(a->q_scale[((int64_t)t * a->H_I + h) * (a->D_I / 32) + d / 32]);
}

/* Step 1 for one token: scores of positions 0..pos into out[0..pos]. */
static void score_token(const oracle_indexer_args* a, int t, double* out, int64_t* npos_out) {
    int b;
    int64_t pos;
    token_place(a->cu_q, a->seq_lens, a->B, t, &b, &pos);
    int H = a->H_I, D = a->D_I;
    double* q = (double*)malloc(sizeof(double) * (size_t)H * D);
    double* k = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < H; h++)
        for (int d = 0; d < D; d++) q[h * D + d] = query_elem(a, t, h, d);
    for (int64_t s = 0; s <= pos; s++) {
        int64_t row = phys_row(a, b, s);
        for (int d = 0; d < D; d++) k[d] = key_elem(a, row, d);
        double acc = 0.0;
        for (int h = 0; h < H; h++) {
            double dot = 0.0;
            for (int d = 0; d < D; d++) dot += q[h * D + d] * k[d];
            double relu = dot > 0.0 ? dot : 0.0;
            acc += (double)a->w[(int64_t)t * H + h] * relu;
        }
        out[s] = acc;
    }
    *npos_out = pos + 1;
    free(q);
    free(k);
}

typedef struct { double score; int64_t pos; } scored_pos;

/* Order: score descending, then position ascending (lower position wins). */
static int cmp_rank(const void* x, const void* y) {
    const scored_pos* a = (const scored_pos*)x;
    const scored_pos* b = (const scored_pos*)y;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->pos > b->pos) - (a->pos < b->pos);
}

static int cmp_i64(const void* x, const void* y) {
    int64_t a = *(const int64_t*)x, b = *(const int64_t*)y;
    return (a > b) - (a < b);
}

/*
 * Steps 1+2 for the tokens listed in `tokens` (n_tokens entries).
 * out_idx   [n_tokens, K] int32: selected positions ascending, -1 padded.
 * out_score [n_tokens, K] double: score of each selected position (NaN pad).
 * out_kth   [n_tokens] double: the K-th largest visible score (smallest kept
 *           score), or -inf when fewer than K positions are visible.
 * out_all   optional [n_tokens, all_stride] double: every visible score.
 */
int oracle_indexer_topk(const oracle_indexer_args* a, const int32_t* tokens, int n_tokens,
                        int32_t* out_idx, double* out_score, double* out_kth,
                        double* out_all, int64_t all_stride) {
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; i++) {
        int t = tokens[i];
        int b;
        int64_t pos;
        token_place(a->cu_q, a->seq_lens, a->B, t, &b, &pos);
        int64_t nvis = pos + 1;
        double* sc = (double*)malloc(sizeof(double) * (size_t)nvis);
        scored_pos* sp = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)nvis);
        int64_t* keep = (int64_t*)malloc(sizeof(int64_t) * (size_t)(a->K > 0 ? a->K : 1));
        if (!sc || !sp || !keep) { rc = -1; free(sc); free(sp); free(keep); continue; }
        score_token(a, t, sc, &nvis);
        if (out_all) memcpy(out_all + (int64_t)i * all_stride, sc, sizeof(double) * (size_t)nvis);
        for (int64_t s = 0; s < nvis; s++) { sp[s].score = sc[s]; sp[s].pos = s; }
        qsort(sp, (size_t)nvis, sizeof(scored_pos), cmp_rank);
        int64_t nk = nvis < a->K ? nvis : a->K;
        for (int64_t j = 0; j < nk; j++) keep[j] = sp[j].pos;
        out_kth[i] = (nvis >= a->K && a->K > 0) ? sp[a->K - 1].score : -INFINITY;
        qsort(keep, (size_t)nk, sizeof(int64_t), cmp_i64);
        for (int64_t j = 0; j < a->K; j++) {
            int64_t o = (int64_t)i * a->K + j;
            out_idx[o] = j < nk ? (int32_t)keep[j] : -1;
            out_score[o] = j < nk ? sc[keep[j]] : NAN;
        }
        free(sc);
        free(sp);
        free(keep);
    }
    return rc;
}

/* Step 1 alone: the score of each (token, position) pair listed. */
int oracle_indexer_score_pairs(const oracle_indexer_args* a, const int32_t* tokens,
                               const int64_t* positions, int64_t n_pairs, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_pairs; i++) {
        int b;
        int64_t pos;
        int t = tokens[i];
        token_place(a->cu_q, a->seq_lens, a->B, t, &b, &pos);
        int64_t s = positions[i];
        if (s < 0 || s > pos) { out[i] = NAN; continue; }
        int64_t row = phys_row(a, b, s);
        double acc = 0.0;
        for (int h = 0; h < a->H_I; h++) {
            double dot = 0.0;
            for (int d = 0; d < a->D_I; d++)
                dot += query_elem(a, t, h, d) * key_elem(a, row, d);
            acc += (double)a->w[(int64_t)t * a->H_I + h] * (dot > 0.0 ? dot : 0.0);
        }
        out[i] = acc;
    }
    return 0;
}

typedef struct {
    int32_t B, T, H, K;
    double sm_scale;
    const int32_t* seq_lens;
    const int32_t* cu_q;
    const int32_t* block_table;
    int32_t max_blocks;
    const uint16_t* q;               /* [T, H, 576] bf16 bits */
    const void* kv;                  /* [nblk, 64, 576] bf16 bits, or e4m3 codes (kv_fp8) */
    const int32_t* idx;              /* [T, K] logical positions, -1 = skip */
    int32_t kv_fp8;                  /* 1: kv holds e4m3 codes with per-row tile scales */
    const float* kv_scale;           /* [nblk, 64, 5] fp32: one scale per 128 elements of a row */
} oracle_attn_args;

/*
 * Element d of latent cache row `row`.  FP8 latent cache ("Day0 Adaptation and
 * Performance Optimization ...", section 4: FP8 KV cache quantized per token and
 * per head in tiles of 128 elements; "Large Model Inference Acceleration ...",
 * section 2.2): the 576-element row is cut into tiles of 128 (the last one, the
 * RoPE part, has 64) and each tile has its own fp32 scale:
 *     kv[row, d] = e4m3(code[row, d]) * scale[row, d / 128].
 */
static double kv_elem(const oracle_attn_args* a, int64_t row, int d) {
    if (!a->kv_fp8) return bf16_to_f64(((const uint16_t*)a->kv)[row * ORACLE_DQK + d]);
    return oracle_e4m3_to_f64(((const uint8_t*)a->kv)[row * ORACLE_DQK + d]) * (double)a->kv_scale[row * 5 + d / 128];
}

/*
 * Step 3 for the tokens listed: out_o [n_tokens, H, 512] double,
 * out_lse [n_tokens, H] double (-inf when no row is selected; o is then 0).
 */
int oracle_sparse_attn(const oracle_attn_args* a, const int32_t* tokens, int n_tokens,
                       double* out_o, double* out_lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; i++) {
        int t = tokens[i];
        int b = 0;
        while (b + 1 < a->B + 1 && a->cu_q[b + 1] <= t) b++;
        const int32_t* sel = a->idx + (int64_t)t * a->K;
        double* logit = (double*)malloc(sizeof(double) * (size_t)a->K);
        int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)a->K);
        int n = 0;
        for (int j = 0; j < a->K; j++) {
            if (sel[j] < 0) continue;
            int64_t p = sel[j];
            rows[n++] = (int64_t)a->block_table[(int64_t)b * a->max_blocks + p / ORACLE_BLOCK] * ORACLE_BLOCK
                        + p % ORACLE_BLOCK;
        }
        for (int g = 0; g < a->H; g++) {
            const uint16_t* qg = a->q + ((int64_t)t * a->H + g) * ORACLE_DQK;
            double* o = out_o + ((int64_t)i * a->H + g) * ORACLE_DV;
            for (int d = 0; d < ORACLE_DV; d++) o[d] = 0.0;
            if (n == 0) { out_lse[(int64_t)i * a->H + g] = -INFINITY; continue; }
            double m = -INFINITY;
            for (int j = 0; j < n; j++) {
                double dot = 0.0;
                for (int d = 0; d < ORACLE_DQK; d++) dot += bf16_to_f64(qg[d]) * kv_elem(a, rows[j], d);
                logit[j] = a->sm_scale * dot;
                if (logit[j] > m) m = logit[j];
            }
            double den = 0.0;
            for (int j = 0; j < n; j++) den += exp(logit[j] - m);
            for (int j = 0; j < n; j++) {
                double p = exp(logit[j] - m) / den;
                for (int d = 0; d < ORACLE_DV; d++) o[d] += p * kv_elem(a, rows[j], d);
            }
            out_lse[(int64_t)i * a->H + g] = m + log(den);
        }
        free(logit);
        free(rows);
    }
    return 0;
}

/*
 * Indexer prolog: the input preparation of the index stage ("Day0 Adaptation
 * and Performance Optimization for Novel Long-Sequence Reasoning Models",
 * section 3: query projection, key normalization, query quantization and
 * head-weight projection; "Large Model Inference Acceleration ...", section
 * 1.2).  For each new token t with hidden state x[t, 0:d] and the weight rows
 * wt = [W_q (H_I*D_I rows) ; W_k (D_I rows) ; W_w (H_I rows)], each [d]:
 *     p[n]      = sum_c x[t,c] * wt[n,c]
 *     q[t,h,i]  = p[h*D_I + i]
 *     k[t,i]    = p[HD + i] / sqrt(mean_j p[HD + j]^2 + eps) * gamma[i]   (RMS normalization)
 *     w[t,h]    = p[HD + D_I + h]
 * with HD = H_I*D_I.  Returned in float64, before any rounding or encoding.
 */
typedef struct {
    int32_t T, d, H_I, D_I;
    const uint16_t* x;               /* [T, d] bf16 bits */
    const uint16_t* wt;              /* [H_I*D_I + D_I + H_I, d] bf16 bits */
    const float* gamma;              /* [D_I] */
    double eps;
} oracle_prolog_args;

int oracle_indexer_prolog(const oracle_prolog_args* a, double* q_out, double* k_out, double* w_out) {
    const int HD = a->H_I * a->D_I, n_out = HD + a->D_I + a->H_I;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < a->T; t++) {
        double* p = (double*)malloc(sizeof(double) * (size_t)n_out);
        for (int n = 0; n < n_out; n++) {
            double acc = 0.0;
            for (int c = 0; c < a->d; c++)
                acc += bf16_to_f64(a->x[(int64_t)t * a->d + c]) * bf16_to_f64(a->wt[(int64_t)n * a->d + c]);
            p[n] = acc;
        }
        for (int i = 0; i < HD; i++) q_out[(int64_t)t * HD + i] = p[i];
        double ms = 0.0;
        for (int i = 0; i < a->D_I; i++) ms += p[HD + i] * p[HD + i];
        ms /= (double)a->D_I;
        double r = 1.0 / sqrt(ms + a->eps);
        for (int i = 0; i < a->D_I; i++) k_out[(int64_t)t * a->D_I + i] = p[HD + i] * r * (double)a->gamma[i];
        for (int h = 0; h < a->H_I; h++) w_out[(int64_t)t * a->H_I + h] = p[HD + a->D_I + h];
        free(p);
    }
    return 0;
}

/*
 * e4m3fn encoding of a real value: the nearest finite e4m3fn value, an exact tie
 * going to the code with an even mantissa, magnitudes beyond the largest finite
 * value (448) saturated to +-448.  Written as a search over the 127 non-negative
 * finite codes, each decoded by oracle_e4m3_to_f64.
 */
uint8_t oracle_e4m3_encode(double v) {
    double a = fabs(v);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 126; c++) {
        double d = fabs(oracle_e4m3_to_f64((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) { bd = d; best = c; }
    }
    if (best == 0) return 0;                          /* +0 for both signs of a zero result */
    return (uint8_t)(best | (v < 0.0 ? 0x80 : 0));
}

/*
 * MXFP8 encoding of n values (n a multiple of 32), 32 consecutive values per
 * group ("Day0 Adaptation ...", section 4: every 32 elements share one scale;
 * the OCP MX rule for the shared scale): X = 2^(floor(log2 amax) - 8), 8 being
 * the exponent of the largest e4m3fn power of two, clamped to 2^-127..2^127;
 * stored as the byte log2(X) + 127.  An all-zero group takes X = 1.  Each value
 * is stored as oracle_e4m3_encode(v / X).
 */
void oracle_mx_encode(const double* v, int64_t n, uint8_t* codes, uint8_t* scales) {
    for (int64_t g = 0; g < n / 32; g++) {
        double amax = 0.0;
        for (int i = 0; i < 32; i++) amax = fmax(amax, fabs(v[g * 32 + i]));
        int e = 0;
        if (amax > 0.0) {
            int ex;
            frexp(amax, &ex);                         /* amax = m * 2^ex, m in [0.5, 1) */
            e = ex - 1 - 8;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
        }
        scales[g] = (uint8_t)(e + 127);
        for (int i = 0; i < 32; i++) codes[g * 32 + i] = oracle_e4m3_encode(ldexp(v[g * 32 + i], -e));
    }
}

/*
 * e4m3fn encoding with one fp32 scale per `group` consecutive values: s is
 * amax / 448 rounded to fp32 (1 for an all-zero group) and each value is stored
 * as oracle_e4m3_encode(v / s).
 */
void oracle_fp8_group_encode(const double* v, int64_t n, int group, uint8_t* codes, float* scales) {
    for (int64_t g = 0; g < n / group; g++) {
        double amax = 0.0;
        for (int i = 0; i < group; i++) amax = fmax(amax, fabs(v[g * group + i]));
        float sc = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
        scales[g] = sc;
        for (int i = 0; i < group; i++) codes[g * group + i] = oracle_e4m3_encode(v[g * group + i] / (double)sc);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
