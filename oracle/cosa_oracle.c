/*
 * CoSA oracle: a plain, slow, single-source CPU restatement of what the
 * two CoSA stages compute.  TEST INFRASTRUCTURE ONLY: only tests/, the smoke
 * check and the benchmark's CPU-baseline leg load this library; the product
 * path never does.  It shares no code, header or constant with the CUDA path.
 *
 * Source: "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
 * Co-Designed Sparse Attention" (gist.science/paper/2607.25291), technical
 * summary:
 *   Sec. 2.1  online-softmax accumulation is independent of the order of the
 *             KV blocks; the proxy emits a computation-order mask.
 *   Sec. 2.2  KAP: downsample Q and K, approximate scores, MaxPool over keys,
 *             MaxNorm, HRM ("have rowmax") flags, flag-grouped sorting under
 *             a moderate budget.
 *   Sec. 2.3  OSK: mask-skipped blocks are never visited; retained blocks are
 *             skipped in-kernel when the local-vs-running max difference says
 *             they are negligible; the rest are computed.
 *   Sec. 1    the "bucket effect": one row vetoes a block skip.
 * The pages give no formulas; each open point is fixed as follows (and the
 * CUDA path implements the same readings independently):
 *   pooling     mean of s consecutive tokens, summed in fp32 in token order,
 *               times 1/s, rounded to bf16 (round-to-nearest-even): the
 *               pooled vectors are a quantised code that decides the
 *               selection, so they are formed in the kernel's precision.
 *   scores      raw dot products of pooled rows (no 1/sqrt(d)), computed in
 *               fp64 and rounded to fp32; every selection decision after that
 *               (max, subtract, compare) is taken in fp32.
 *   causality   pooled key c is visible to pooled row r iff some token pair
 *               is causal: s*c <= off + s*r + s-1.
 *   MaxPool     max over the visible pooled keys of each KV block.
 *   MaxNorm     z = Bs - rowmax (log-domain normalisation, z <= 0).
 *   HRM         block j is flagged for Q-block I iff j is the smallest block
 *               index attaining rowmax for some pooled row r of I.
 *   aggregate   score[I,j] = max over the pooled rows r of I of z[r,j].
 *   budget      n_I causally visible blocks, bp = round(beta*1e4),
 *               k_I = max(1, ceil(n_I*bp/1e4)) in integer arithmetic.
 *   sort        (HRM desc, score desc, block index asc); keep k_I.
 *   skip test   row vote: m_loc = -inf, or (m_run finite and
 *               fp32(m_loc - m_run) < T) with T = fp32(ln(eps)*sqrt(d)) in
 *               raw-logit units; a block is skipped iff every row of the
 *               Q-block votes skip; eps = 0 never skips.
 *   softmax     fp64, scale 1/sqrt(d), in visit order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, Nq, Nkv, d;
    int bq, bk, s;
    int paged;      /* 0: K,V [B,Hkv,Nkv,d]; 1: K,V [num_pages,Hkv,bk,d] + page_table [B][nKB] */
    int num_pages;
} or_shape;

/* ---------------------------------------------------------------- scalars */

static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* float -> bf16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static int cdiv(int a, int b) { return (a + b - 1) / b; }

static int n_qblocks(const or_shape* sh) { return cdiv(sh->Nq, sh->bq); }
static int n_kblocks(const or_shape* sh) { return cdiv(sh->Nkv, sh->bk); }

/* ------------------------------------------------------------- addressing */

static const uint16_t* q_row(const or_shape* sh, const uint16_t* q, int b, int h, int i) {
    return q + (((size_t)b * sh->Hq + h) * sh->Nq + i) * sh->d;
}

/* Token c of kv-head g in batch b, through the page table when paged. */
static const uint16_t* kv_row(const or_shape* sh, const uint16_t* x, const int32_t* pt, int b, int g, int c) {
    if (!sh->paged) return x + (((size_t)b * sh->Hkv + g) * sh->Nkv + c) * sh->d;
    int page = pt[(size_t)b * n_kblocks(sh) + c / sh->bk];
    return x + (((size_t)page * sh->Hkv + g) * sh->bk + (c % sh->bk)) * sh->d;
}

/* ------------------------------------------------------------- stage 1: KAP */

/* Downsampling (Sec. 2.2 "downsamples queries and keys"): pooled row r is
 * the mean of tokens s*r .. s*r+s-1. */
static void pool_row(const or_shape* sh, const uint16_t* const* rows, float* out) {
    for (int e = 0; e < sh->d; ++e) {
        float acc = 0.0f;
        for (int t = 0; t < sh->s; ++t) acc = acc + bf16_to_f32(rows[t][e]);
        out[e] = bf16_to_f32(f32_to_bf16_rne(acc * (1.0f / (float)sh->s)));
    }
}

/* Pooled Q rows of one head: [Nq/s][d]. */
static void pool_q_head(const or_shape* sh, const uint16_t* q, int b, int h, float* qp) {
    const uint16_t* rows[64];
    for (int r = 0; r < sh->Nq / sh->s; ++r) {
        for (int t = 0; t < sh->s; ++t) rows[t] = q_row(sh, q, b, h, r * sh->s + t);
        pool_row(sh, rows, qp + (size_t)r * sh->d);
    }
}

/* Pooled K rows of one kv-head: [Nkv/s][d]. */
static void pool_k_head(const or_shape* sh, const uint16_t* k, const int32_t* pt, int b, int g, float* kp) {
    const uint16_t* rows[64];
    for (int c = 0; c < sh->Nkv / sh->s; ++c) {
        for (int t = 0; t < sh->s; ++t) rows[t] = kv_row(sh, k, pt, b, g, c * sh->s + t);
        pool_row(sh, rows, kp + (size_t)c * sh->d);
    }
}

/* Number of KV blocks with at least one key visible to some query of
 * Q-block I (the blocks a causal dense kernel would visit). */
static int causal_blocks(const or_shape* sh, int I) {
    int off = sh->Nkv - sh->Nq;
    int last_q = (I + 1) * sh->bq < sh->Nq ? (I + 1) * sh->bq - 1 : sh->Nq - 1;
    int n = (off + last_q) / sh->bk + 1;
    int nkb = n_kblocks(sh);
    return n < nkb ? n : nkb;
}

/* Budget (Sec. 2.2 "moderate budget"): k = max(1, ceil(n * bp / 10000)). */
static int budget_blocks(int n, int bp) {
    long long k = ((long long)n * bp + 9999) / 10000;
    if (k < 1) k = 1;
    if (k > n) k = n;
    return (int)k;
}

typedef struct { int j; int hrm; float score; } rank_entry;

/* Flag-grouped sorting (Sec. 2.2): HRM blocks first, then by estimated score,
 * block index ascending among equals. */
static int rank_cmp(const void* pa, const void* pb) {
    const rank_entry* a = (const rank_entry*)pa;
    const rank_entry* b = (const rank_entry*)pb;
    if (a->hrm != b->hrm) return a->hrm ? -1 : 1;
    if (a->score != b->score) return a->score > b->score ? -1 : 1;
    return a->j < b->j ? -1 : (a->j > b->j);
}

/* KAP for one (b, h, Q-block I), with the pooled Q of head h and pooled K of
 * its kv-head already formed.  Writes order[0..k_I-1]; returns k_I. */
static int kap_one(const or_shape* sh, const float* qp, const float* kp, int I, int bp,
                   int32_t* order, int32_t* hrm_count, float* score_out, uint8_t* hrm_out,
                   float* bs /* [rows][nKB] scratch */, rank_entry* ent) {
    const int s = sh->s, d = sh->d, nkb = n_kblocks(sh);
    const int off = sh->Nkv - sh->Nq;
    const int r0 = I * sh->bq / s;
    const int r1 = ((I + 1) * sh->bq < sh->Nq ? (I + 1) * sh->bq : sh->Nq) / s;
    const int nrows = r1 - r0;
    const int n_valid = causal_blocks(sh, I);
    const int kpb = sh->bk / s;            /* pooled keys per KV block */
    const int nkp = sh->Nkv / s;

    /* approximate scores + MaxPool over the keys of each block */
    for (int rr = 0; rr < nrows; ++rr) {
        const int r = r0 + rr;
        const float* qv = qp + (size_t)r * d;
        for (int j = 0; j < nkb; ++j) {
            float m = -INFINITY;
            for (int c = j * kpb; c < (j + 1) * kpb && c < nkp; ++c) {
                if ((long long)s * c > (long long)off + (long long)s * r + (s - 1)) continue;
                const float* kv = kp + (size_t)c * d;
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += (double)qv[e] * (double)kv[e];
                float sc = (float)acc;
                if (sc > m) m = sc;
            }
            bs[(size_t)rr * nkb + j] = m;
        }
    }
    /* MaxNorm, HRM flags, aggregation over the rows of the Q-block */
    for (int j = 0; j < n_valid; ++j) { ent[j].j = j; ent[j].hrm = 0; ent[j].score = -INFINITY; }
    for (int rr = 0; rr < nrows; ++rr) {
        const float* row = bs + (size_t)rr * nkb;
        float rowmax = -INFINITY;
        int jstar = -1;
        for (int j = 0; j < nkb; ++j)
            if (row[j] > rowmax) { rowmax = row[j]; jstar = j; }
        if (jstar < 0) continue;           /* a row with no visible key (cannot happen for off >= 0) */
        if (jstar < n_valid) ent[jstar].hrm = 1;
        for (int j = 0; j < n_valid; ++j) {
            float z = row[j] - rowmax;
            if (z > ent[j].score) ent[j].score = z;
        }
    }
    int nh = 0;
    for (int j = 0; j < n_valid; ++j) {
        nh += ent[j].hrm;
        if (score_out) score_out[j] = ent[j].score;
        if (hrm_out) hrm_out[j] = (uint8_t)ent[j].hrm;
    }
    if (score_out) for (int j = n_valid; j < nkb; ++j) score_out[j] = -INFINITY;
    if (hrm_out) for (int j = n_valid; j < nkb; ++j) hrm_out[j] = 0;
    qsort(ent, (size_t)n_valid, sizeof(rank_entry), rank_cmp);
    const int k = budget_blocks(n_valid, bp);
    for (int t = 0; t < k; ++t) order[t] = ent[t].j;
    *hrm_count = nh;
    return k;
}

static int resolve_sel(const or_shape* sh, const int32_t* sel, int nsel, int idx, int* b, int* h, int* I) {
    if (sel) { *b = sel[3 * idx]; *h = sel[3 * idx + 1]; *I = sel[3 * idx + 2]; }
    else {
        int nqb = n_qblocks(sh);
        *I = idx % nqb; *h = (idx / nqb) % sh->Hq; *b = idx / (nqb * sh->Hq);
    }
    (void)nsel;
    return (*b >= 0 && *b < sh->B && *h >= 0 && *h < sh->Hq && *I >= 0 && *I < n_qblocks(sh)) ? 0 : -1;
}

static int check_shape(const or_shape* sh) {
    if (sh->B < 0 || sh->Hq <= 0 || sh->Hkv <= 0 || sh->Hq % sh->Hkv) return -1;
    if (sh->Nq < 0 || sh->Nkv < sh->Nq || sh->d <= 0) return -1;
    if (sh->s <= 0 || sh->s > 64 || sh->bq % sh->s || sh->bk % sh->s) return -1;
    if (sh->Nq % sh->s || sh->Nkv % sh->s) return -1;
    return 0;
}

int oracle_kmax(const or_shape* sh, double budget) {
    if (check_shape(sh) || sh->Nq == 0) return 0;
    int bp = (int)lround(budget * 10000.0);
    return budget_blocks(causal_blocks(sh, n_qblocks(sh) - 1), bp);
}

int oracle_causal_blocks(const or_shape* sh, int I) { return causal_blocks(sh, I); }
int oracle_budget_blocks(int n, double budget) { return budget_blocks(n, (int)lround(budget * 10000.0)); }

/* Pool a [rows][d] bf16 matrix with stride s into [rows/s][d] bf16. */
void oracle_pool(const uint16_t* x, int rows, int d, int s, uint16_t* out) {
    or_shape sh = {0};
    sh.d = d; sh.s = s;
    const uint16_t* r[64];
    float* tmp = (float*)malloc(sizeof(float) * (size_t)d);
    for (int p = 0; p < rows / s; ++p) {
        for (int t = 0; t < s; ++t) r[t] = x + ((size_t)p * s + t) * d;
        pool_row(&sh, r, tmp);
        for (int e = 0; e < d; ++e) out[(size_t)p * d + e] = f32_to_bf16_rne(tmp[e]);
    }
    free(tmp);
}

/* Stage 1 over a list of (b, h, I) triples (sel, nsel) or over every
 * (b, h, I) in row-major order (sel == NULL).  order is [n][kmax], padded
 * with -1; block_score / hrm (optional) are [n][nKB]. */
int oracle_kap(const or_shape* sh, const uint16_t* q, const uint16_t* k, const int32_t* page_table,
               double budget, const int32_t* sel, int nsel, int kmax,
               int32_t* order, int32_t* count, int32_t* hrm_count,
               float* block_score, uint8_t* hrm, int nthreads) {
    if (check_shape(sh)) return -1;
    const int nqb = n_qblocks(sh), nkb = n_kblocks(sh), G = sh->Hq / sh->Hkv, d = sh->d;
    const int n = sel ? nsel : sh->B * sh->Hq * nqb;
    const int bp = (int)lround(budget * 10000.0);
    if (bp < 0 || bp > 10000) return -1;
    if (n == 0) return 0;
    if (kmax < oracle_kmax(sh, budget)) return -2;
    const size_t kp_sz = (size_t)(sh->Nkv / sh->s) * d;
    const size_t qp_sz = (size_t)(sh->Nq / sh->s) * d;
    /* pooled K of every (b, kv-head) and pooled Q of every (b, head) used */
    float* kp = (float*)malloc(sizeof(float) * kp_sz * (size_t)sh->B * sh->Hkv + 1);
    float* qp = (float*)malloc(sizeof(float) * qp_sz * (size_t)sh->B * sh->Hq + 1);
    char* qdone = (char*)calloc((size_t)sh->B * sh->Hq, 1);
    for (int i = 0; i < n; ++i) {
        int b, h, I;
        if (resolve_sel(sh, sel, nsel, i, &b, &h, &I)) { free(kp); free(qp); free(qdone); return -3; }
        qdone[(size_t)b * sh->Hq + h] = 1;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bg = 0; bg < sh->B * sh->Hkv; ++bg)
        pool_k_head(sh, k, page_table, bg / sh->Hkv, bg % sh->Hkv, kp + kp_sz * bg);
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bh = 0; bh < sh->B * sh->Hq; ++bh)
        if (qdone[bh]) pool_q_head(sh, q, bh / sh->Hq, bh % sh->Hq, qp + qp_sz * bh);
    int err = 0;
#ifdef _OPENMP
#pragma omp parallel
#endif
    {
        float* bs = (float*)malloc(sizeof(float) * (size_t)(sh->bq / sh->s) * nkb + 1);
        rank_entry* ent = (rank_entry*)malloc(sizeof(rank_entry) * (size_t)nkb + 1);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int i = 0; i < n; ++i) {
            int b, h, I;
            resolve_sel(sh, sel, nsel, i, &b, &h, &I);
            int32_t* ord = order + (size_t)i * kmax;
            for (int t = 0; t < kmax; ++t) ord[t] = -1;
            int c = kap_one(sh, qp + qp_sz * ((size_t)b * sh->Hq + h),
                            kp + kp_sz * ((size_t)b * sh->Hkv + h / G), I, bp, ord, hrm_count + i,
                            block_score ? block_score + (size_t)i * nkb : NULL,
                            hrm ? hrm + (size_t)i * nkb : NULL, bs, ent);
            count[i] = c;
            if (c > kmax) err = -2;
        }
        free(bs);
        free(ent);
    }
    free(kp); free(qp); free(qdone);
    return err;
}

/* ------------------------------------------------------------- stage 2: OSK */

/* T = fp32(ln(eps) * sqrt(d)); eps = 0 gives -inf (never skip). */
float oracle_skip_threshold(double eps, int d) {
    if (eps <= 0.0) return -INFINITY;
    return (float)(log(eps) * sqrt((double)d));
}

/* OSK for one (b, h, I) (Sec. 2.3): visit order[0..count-1]; per block, the
 * in-kernel skip test on exact logits, else the online-softmax update. */
static void osk_one(const or_shape* sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const int32_t* pt, int b, int h, int I, const int32_t* order, int count,
                    float T, int apply_skip, double* out, double* lse, uint8_t* skipped,
                    double* margin, double* qf, double* srow) {
    const int d = sh->d, bq = sh->bq, bk = sh->bk, g = h / (sh->Hq / sh->Hkv);
    const int off = sh->Nkv - sh->Nq;
    const int i0 = I * bq;
    const int nrows = (i0 + bq < sh->Nq ? bq : sh->Nq - i0);
    const double scale = 1.0 / sqrt((double)d);
    float m_run[256];
    double m_acc[256], l[256];
    for (int r = 0; r < nrows; ++r) {
        const uint16_t* qr = q_row(sh, q, b, h, i0 + r);
        for (int e = 0; e < d; ++e) qf[(size_t)r * d + e] = (double)bf16_to_f32(qr[e]);
        m_run[r] = -INFINITY; m_acc[r] = -INFINITY; l[r] = 0.0;
        for (int e = 0; e < d; ++e) out[(size_t)r * d + e] = 0.0;
    }
    for (int t = 0; t < count; ++t) {
        const int j = order[t];
        const int c0 = j * bk, c1 = (c0 + bk < sh->Nkv ? c0 + bk : sh->Nkv);
        /* exact logits of the block and the tile-wide skip vote; the block's
         * margin is the largest row distance above the threshold (< 0 iff
         * every row votes skip), reported so callers can tell fragile
         * decisions from robust ones */
        int all_skip = 1;
        double mg = -INFINITY;
        for (int r = 0; r < nrows; ++r) {
            float m_loc = -INFINITY;
            for (int c = c0; c < c1; ++c) {
                double* sv = srow + (size_t)r * bk + (c - c0);
                if (c > off + i0 + r) { *sv = -INFINITY; continue; }
                const uint16_t* kr = kv_row(sh, k, pt, b, g, c);
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += qf[(size_t)r * d + e] * (double)bf16_to_f32(kr[e]);
                *sv = acc;
                if ((float)acc > m_loc) m_loc = (float)acc;
            }
            int vote = (m_loc == -INFINITY) ||
                       (m_run[r] != -INFINITY && (float)(m_loc - m_run[r]) < T);
            if (!vote) all_skip = 0;
            if (m_loc != -INFINITY) {
                double dr = (m_run[r] == -INFINITY || T == -INFINITY)
                                ? INFINITY : (double)(float)(m_loc - m_run[r]) - (double)T;
                if (dr > mg) mg = dr;
            }
            srow[(size_t)bk * 256 + r] = m_loc;          /* keep m_loc for the update below */
        }
        if (skipped) skipped[t] = (uint8_t)(apply_skip && all_skip);
        if (margin) margin[t] = mg;
        if (apply_skip && all_skip) continue;
        for (int r = 0; r < nrows; ++r) {
            float m_loc = (float)srow[(size_t)bk * 256 + r];
            if (m_loc > m_run[r]) m_run[r] = m_loc;
            double mb = -INFINITY;
            for (int c = c0; c < c1; ++c) if (srow[(size_t)r * bk + (c - c0)] > mb) mb = srow[(size_t)r * bk + (c - c0)];
            if (mb == -INFINITY) continue;
            double m_new = mb > m_acc[r] ? mb : m_acc[r];
            double alpha = (m_acc[r] == -INFINITY) ? 0.0 : exp((m_acc[r] - m_new) * scale);
            l[r] *= alpha;
            double* o = out + (size_t)r * d;
            for (int e = 0; e < d; ++e) o[e] *= alpha;
            for (int c = c0; c < c1; ++c) {
                double sv = srow[(size_t)r * bk + (c - c0)];
                if (sv == -INFINITY) continue;
                double p = exp((sv - m_new) * scale);
                l[r] += p;
                const uint16_t* vr = kv_row(sh, v, pt, b, g, c);
                for (int e = 0; e < d; ++e) o[e] += p * (double)bf16_to_f32(vr[e]);
            }
            m_acc[r] = m_new;
        }
    }
    for (int r = 0; r < nrows; ++r) {
        double* o = out + (size_t)r * d;
        if (l[r] > 0.0) {
            for (int e = 0; e < d; ++e) o[e] /= l[r];
            if (lse) lse[r] = m_acc[r] * scale + log(l[r]);
        } else {
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            if (lse) lse[r] = -INFINITY;
        }
    }
    for (int r = nrows; r < bq; ++r) {
        for (int e = 0; e < d; ++e) out[(size_t)r * d + e] = 0.0;
        if (lse) lse[r] = -INFINITY;
    }
}

/* Stage 2 over a selection (or everything).  order/count as produced by
 * oracle_kap (or any caller-chosen visit order).  out [n][bq][d], lse
 * [n][bq] (optional), skipped [n][kmax] (optional, 1 = skipped in-kernel),
 * margin [n][kmax] (optional: per visit, the largest row value of
 * fp32(m_loc - m_run) - T; negative iff the block is skipped, +inf where a
 * row had no running max yet or eps = 0, -inf where no row saw a key).
 * eps = 0 disables the in-kernel skip. */
int oracle_osk(const or_shape* sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
               const int32_t* page_table, const int32_t* sel, int nsel,
               const int32_t* order, const int32_t* count, int kmax, double eps,
               double* out, double* lse, uint8_t* skipped, double* margin, int nthreads) {
    if (check_shape(sh) || sh->bq > 256 || eps < 0.0 || eps >= 1.0) return -1;
    const int n = sel ? nsel : sh->B * sh->Hq * n_qblocks(sh);
    const float T = oracle_skip_threshold(eps, sh->d);
    for (int i = 0; i < n; ++i) {
        int b, h, I;
        if (resolve_sel(sh, sel, nsel, i, &b, &h, &I)) return -3;
        if (count[i] < 0 || count[i] > kmax) return -2;
        for (int t = 0; t < count[i]; ++t)
            if (order[(size_t)i * kmax + t] < 0 || order[(size_t)i * kmax + t] >= n_kblocks(sh)) return -2;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* qf = (double*)malloc(sizeof(double) * (size_t)sh->bq * sh->d);
        double* srow = (double*)malloc(sizeof(double) * ((size_t)sh->bk * 256 + 256));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int i = 0; i < n; ++i) {
            int b, h, I;
            resolve_sel(sh, sel, nsel, i, &b, &h, &I);
            if (skipped) memset(skipped + (size_t)i * kmax, 0, (size_t)kmax);
            if (margin) for (int t = 0; t < kmax; ++t) margin[(size_t)i * kmax + t] = NAN;
            osk_one(sh, q, k, v, page_table, b, h, I, order + (size_t)i * kmax, count[i], T, eps > 0.0,
                    out + (size_t)i * sh->bq * sh->d, lse ? lse + (size_t)i * sh->bq : NULL,
                    skipped ? skipped + (size_t)i * kmax : NULL, margin ? margin + (size_t)i * kmax : NULL,
                    qf, srow);
        }
        free(qf);
        free(srow);
    }
    return 0;
}

/* ---------------------------------------------------------- dense reference */

/* Textbook two-pass causal softmax attention in fp64 for the rows of one
 * Q-block, over the keys of the listed blocks (or of every block when
 * blocks == NULL).  This is the "dense attention" the speedup is quoted
 * against, and, restricted to a block list, the closed form that OSK with
 * eps = 0 must reproduce. */
static void dense_one(const or_shape* sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const int32_t* pt, int b, int h, int I, const int32_t* blocks, int nblocks,
                      double* out, double* lse, double* sbuf, char* use) {
    const int d = sh->d, bq = sh->bq, bk = sh->bk, g = h / (sh->Hq / sh->Hkv);
    const int off = sh->Nkv - sh->Nq, nkb = n_kblocks(sh);
    const int i0 = I * bq, nrows = (i0 + bq < sh->Nq ? bq : sh->Nq - i0);
    const double scale = 1.0 / sqrt((double)d);
    memset(use, blocks ? 0 : 1, (size_t)nkb);
    if (blocks) for (int t = 0; t < nblocks; ++t) use[blocks[t]] = 1;
    for (int r = 0; r < nrows; ++r) {
        const uint16_t* qr = q_row(sh, q, b, h, i0 + r);
        const int last = off + i0 + r;
        double m = -INFINITY;
        for (int c = 0; c <= last && c < sh->Nkv; ++c) {
            sbuf[c] = -INFINITY;
            if (!use[c / bk]) continue;
            const uint16_t* kr = kv_row(sh, k, pt, b, g, c);
            double acc = 0.0;
            for (int e = 0; e < d; ++e) acc += (double)bf16_to_f32(qr[e]) * (double)bf16_to_f32(kr[e]);
            sbuf[c] = acc * scale;
            if (sbuf[c] > m) m = sbuf[c];
        }
        double* o = out + (size_t)r * d;
        for (int e = 0; e < d; ++e) o[e] = 0.0;
        if (m == -INFINITY) { if (lse) lse[r] = -INFINITY; continue; }
        double l = 0.0;
        for (int c = 0; c <= last && c < sh->Nkv; ++c) {
            if (sbuf[c] == -INFINITY) continue;
            double p = exp(sbuf[c] - m);
            l += p;
            const uint16_t* vr = kv_row(sh, v, pt, b, g, c);
            for (int e = 0; e < d; ++e) o[e] += p * (double)bf16_to_f32(vr[e]);
        }
        for (int e = 0; e < d; ++e) o[e] /= l;
        if (lse) lse[r] = m + log(l);
    }
    for (int r = nrows; r < bq; ++r) {
        for (int e = 0; e < d; ++e) out[(size_t)r * d + e] = 0.0;
        if (lse) lse[r] = -INFINITY;
    }
}

/* Dense over a selection.  order == NULL: full causal attention; else the
 * keys of blocks order[i][0..count[i]-1] only. */
int oracle_dense(const or_shape* sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const int32_t* page_table, const int32_t* sel, int nsel,
                 const int32_t* order, const int32_t* count, int kmax,
                 double* out, double* lse, int nthreads) {
    if (check_shape(sh)) return -1;
    const int n = sel ? nsel : sh->B * sh->Hq * n_qblocks(sh);
    for (int i = 0; i < n; ++i) {
        int b, h, I;
        if (resolve_sel(sh, sel, nsel, i, &b, &h, &I)) return -3;
        if (order) {
            if (count[i] < 0 || count[i] > kmax) return -2;
            for (int t = 0; t < count[i]; ++t)
                if (order[(size_t)i * kmax + t] < 0 || order[(size_t)i * kmax + t] >= n_kblocks(sh)) return -2;
        }
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double* sbuf = (double*)malloc(sizeof(double) * (size_t)sh->Nkv + 8);
        char* use = (char*)malloc((size_t)n_kblocks(sh) + 1);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int i = 0; i < n; ++i) {
            int b, h, I;
            resolve_sel(sh, sel, nsel, i, &b, &h, &I);
            dense_one(sh, q, k, v, page_table, b, h, I, order ? order + (size_t)i * kmax : NULL,
                      order ? count[i] : 0, out + (size_t)i * sh->bq * sh->d,
                      lse ? lse + (size_t)i * sh->bq : NULL, sbuf, use);
        }
        free(sbuf);
        free(use);
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
