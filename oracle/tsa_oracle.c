/*
 * Token Sparse Attention layer: CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * restatement that the CUDA library is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg load it.  It shares no
 * code, header, table or constant with the CUDA library, and the library never
 * calls it.
 *
 * All arithmetic is IEEE double on the exact values of the inputs (fp32, or
 * bf16 given as its raw 16 bits).  Parallelism is a plain split of independent
 * (batch, head) problems over pthreads; within one problem every sum runs in
 * index order.
 *
 * Sources (cited by page and section):
 *   [notes]  papernotes.org notes, "Token Sparse Attention: Efficient
 *            Long-Context Inference with Interleaved Token Selection":
 *            方法详解 › 整体框架 (overall framework), 关键设计 1
 *            (Compress-then-Decompress), 关键设计 2 (Dynamic Token Coverage).
 *   [blog]   bxzpzcl.cn post on the same paper: §1.1 核心算法实现细节
 *            (compress / attend / decompress, with a code sketch) and
 *            §2.1 重要性评估机制 (recent-query scoring, head and layer score,
 *            coverage budget).
 *   [gist]   gist.science summary: §2 Methodology, "Core Architecture" and
 *            "Dynamic Token Coverage".
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   scoring is causal (recent query p sees keys t <= p) and uses the same
 *   1/sqrt(d) scale as attention; "pool" after the column sum adds nothing in
 *   the method as benchmarked (orc_pool gives the max / mean variants);
 *   "normalize" is division by the total; the coverage cumulative sum is taken
 *   in 2^-62 fixed point; top-k ties go to the lower token index; S_h is listed
 *   in ascending token order; GQA query head h reads KV head h / (H / Hkv).
 *
 * Pins: every function below is checked by tests/test_oracle.py against
 * closed forms, library routines (torch float64 SDPA / softmax) or brute force
 * on tiny inputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Element decoding.  dtype 0 = IEEE fp32, dtype 1 = bfloat16 (the upper 16  */
/* bits of an fp32 word, stored as uint16).                                  */
/* ------------------------------------------------------------------------ */
static double elem(const void *base, int dtype, size_t i) {
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t w = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* A tiny work splitter: run fn(arg, item) for item in [0, n) on nthreads.   */
/* ------------------------------------------------------------------------ */
typedef void (*item_fn)(void *arg, long item);
typedef struct {
    item_fn fn;
    void *arg;
    long n, next;
    pthread_mutex_t mu;
} pool_t;

static void *pool_worker(void *p_) {
    pool_t *p = (pool_t *)p_;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        long it = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (it >= p->n) return NULL;
        p->fn(p->arg, it);
    }
}

static void run_items(item_fn fn, void *arg, long n, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads == 1 || n <= 1) {
        for (long i = 0; i < n; ++i) fn(arg, i);
        return;
    }
    pool_t p;
    p.fn = fn; p.arg = arg; p.n = n; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    pthread_t th[256];
    int started = 0;
    for (int t = 0; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, pool_worker, &p) == 0) ++started;
    if (started == 0) pool_worker(&p);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------------ */
/* Step 1: Dynamic Token Coverage scoring.                                   */
/*   [notes] 关键设计 2; [blog] §2.1 "轻量级注意力评分" and "头级重要性计算";  */
/*   [gist] §2 "Scoring".                                                    */
/* The last q_eff = min(q, L) queries (positions p = L - q_eff + i) attend    */
/* to the keys t <= p of their head's KV group with a softmax; the weights   */
/* are summed over the queries: s_h[t] = sum_i A[i, t].                      */
/* Then u[t] = sum_h s_h[t] and s_l = u / sum_t u ([blog] §2.1 "层级预算分配"). */
/* ------------------------------------------------------------------------ */
typedef struct {
    int B, L, H, Hkv, d, dtype, qe;
    const void *Qr;   /* [B, qe, H, d]: the last qe query rows */
    const void *K;    /* [B, L, Hkv, d] */
    double scale;
    double *s_h;      /* [B, H, L] */
} score_job;

static void score_item(void *arg, long item) {
    score_job *j = (score_job *)arg;
    const int b = (int)(item / j->H), h = (int)(item % j->H);
    const int G = j->H / j->Hkv, kv = h / G, L = j->L, d = j->d;
    double *z = (double *)malloc(sizeof(double) * (size_t)L);
    double *sh = j->s_h + ((size_t)b * j->H + h) * L;
    for (int t = 0; t < L; ++t) sh[t] = 0.0;
    for (int i = 0; i < j->qe; ++i) {
        const int p = L - j->qe + i;
        const size_t qoff = (((size_t)b * j->qe + i) * j->H + h) * d;
        double zmax = -INFINITY;
        for (int t = 0; t <= p; ++t) {
            const size_t koff = (((size_t)b * L + t) * j->Hkv + kv) * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += elem(j->Qr, j->dtype, qoff + c) * elem(j->K, j->dtype, koff + c);
            z[t] = j->scale * acc;
            if (z[t] > zmax) zmax = z[t];
        }
        double den = 0.0;
        for (int t = 0; t <= p; ++t) den += exp(z[t] - zmax);
        for (int t = 0; t <= p; ++t) sh[t] += exp(z[t] - zmax) / den;
    }
    free(z);
}

int orc_score(int B, int L, int H, int Hkv, int d, int dtype, int q,
              const void *Qrecent, const void *K, double scale,
              double *s_h, double *s_l, int nthreads) {
    if (B < 1 || L < 1 || H < 1 || Hkv < 1 || H % Hkv || d < 1 || q < 1) return 1;
    score_job j = {B, L, H, Hkv, d, dtype, q < L ? q : L, Qrecent, K, scale, s_h};
    run_items(score_item, &j, (long)B * H, nthreads);
    for (int b = 0; b < B; ++b) {
        double *sl = s_l + (size_t)b * L, tot = 0.0;
        for (int t = 0; t < L; ++t) {
            double u = 0.0;
            for (int h = 0; h < H; ++h) u += s_h[((size_t)b * H + h) * L + t];
            sl[t] = u;
            tot += u;
        }
        for (int t = 0; t < L; ++t) sl[t] /= tot;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 2: layer budget.  [notes] 关键设计 2; [blog] §2.1 "层级预算分配";     */
/* [gist] §2 "Budget Allocation".  Sort s_l ascending, take the smallest k   */
/* whose cumulative mass reaches tau, keep L' = L - k.                       */
/* The mass is summed in unsigned 2^-62 fixed point: m[t] = floor(s_l*2^62), */
/* T = ceil(tau*2^62).  Both products are exact in double.  If the mass      */
/* never reaches T, k = L and L' = 0.                                        */
/* ------------------------------------------------------------------------ */
typedef struct { float v; int t; } vt_pair;

static int cmp_asc(const void *a_, const void *b_) {
    const vt_pair *a = (const vt_pair *)a_, *b = (const vt_pair *)b_;
    if (a->v < b->v) return -1;
    if (a->v > b->v) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

static int cmp_desc(const void *a_, const void *b_) {
    const vt_pair *a = (const vt_pair *)a_, *b = (const vt_pair *)b_;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

/* real_disagree (optional) counts batch elements where a long-double        */
/* cumulative sum of the same sorted values would pick a different k.        */
int orc_budget(int B, int L, const float *s_l, double tau, int32_t *Lkeep,
               int32_t *real_disagree) {
    if (B < 1 || L < 1 || !(tau >= 0.0 && tau < 1.0)) return 1;
    const double two62 = 4611686018427387904.0; /* 2^62 */
    const uint64_t T = (uint64_t)ceil(tau * two62);
    vt_pair *v = (vt_pair *)malloc(sizeof(vt_pair) * (size_t)L);
    int32_t dis = 0;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < L; ++t) {
            v[t].v = s_l[(size_t)b * L + t];
            v[t].t = t;
            if (!(v[t].v >= 0.0f && v[t].v <= 1.0f)) { free(v); return 2; }
        }
        qsort(v, (size_t)L, sizeof(vt_pair), cmp_asc);
        int k = L;
        uint64_t cum = 0;
        if (T == 0) k = 0;
        for (int kk = 1; k != 0 && kk <= L; ++kk) {
            cum += (uint64_t)floor((double)v[kk - 1].v * two62);
            if (cum >= T) { k = kk; break; }
        }
        int kr = L;
        long double cr = 0.0L;
        if (tau == 0.0) kr = 0;
        for (int kk = 1; kr != 0 && kk <= L; ++kk) {
            cr += (long double)v[kk - 1].v;
            if (cr >= (long double)tau) { kr = kk; break; }
        }
        if (kr != k) ++dis;
        Lkeep[b] = L - k;
    }
    free(v);
    if (real_disagree) *real_disagree = dis;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Budget variant for the ablation: a fixed sparsity ratio s instead of the  */
/* coverage threshold.  [notes] 消融实验 (Fixed s = 0.3 / s = 0.5 against the  */
/* dynamic budget) and 关键设计 2 (a one-size "cut 30%" is what the coverage  */
/* budget replaces).  Reading: s is the fraction of tokens pruned, so        */
/* k = floor(s * L) (in double) and L' = L - k, the same for every batch     */
/* element.                                                                  */
/* ------------------------------------------------------------------------ */
int orc_budget_fixed(int B, int L, double s, int32_t *Lkeep) {
    if (B < 1 || L < 1 || !(s >= 0.0 && s <= 1.0)) return 1;
    const int k = (int)floor(s * (double)L);
    for (int b = 0; b < B; ++b) Lkeep[b] = L - k;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Score variant: pooling of the head scores along the token axis.          */
/* [notes] 关键设计 2: the column sums are pooled to give s_h before the     */
/* layer score.  The pages name no pooling kind or window; the two plain     */
/* readings are built: kind 1 = max, kind 2 = mean, over the window          */
/* [t - r, t + r] (width = 2r + 1, odd) clipped to [0, L): the mean divides  */
/* by the number of in-range tokens.  Then u[t] = sum_h pooled[t] and        */
/* s_l = u / sum_t u, as in step 1.                                          */
/* ------------------------------------------------------------------------ */
int orc_pool(int B, int H, int L, const double *s_h, int kind, int width,
             double *out, double *s_l) {
    if (B < 1 || H < 1 || L < 1 || width < 1 || (width & 1) == 0 || (kind != 1 && kind != 2))
        return 1;
    const int rad = width / 2;
    for (long row = 0; row < (long)B * H; ++row) {
        const double *in = s_h + (size_t)row * L;
        double *o = out + (size_t)row * L;
        for (int t = 0; t < L; ++t) {
            const int lo = t - rad < 0 ? 0 : t - rad, hi = t + rad > L - 1 ? L - 1 : t + rad;
            double acc = kind == 1 ? -INFINITY : 0.0;
            for (int u = lo; u <= hi; ++u) {
                if (kind == 1) { if (in[u] > acc) acc = in[u]; }
                else acc += in[u];
            }
            o[t] = kind == 1 ? acc : acc / (double)(hi - lo + 1);
        }
    }
    for (int b = 0; b < B; ++b) {
        double *sl = s_l + (size_t)b * L, tot = 0.0;
        for (int t = 0; t < L; ++t) {
            double u = 0.0;
            for (int h = 0; h < H; ++h) u += out[((size_t)b * H + h) * L + t];
            sl[t] = u;
            tot += u;
        }
        for (int t = 0; t < L; ++t) sl[t] /= tot;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 3: per-head top-L' selection.  [notes] 关键设计 2 (each head takes    */
/* its own top-k_keep); [gist] §2 "Head-Wise Selection".  Order tokens by    */
/* (s_h descending, t ascending), keep the first L'.  idx[b,h,:] receives    */
/* the kept tokens in ascending order, then the remaining L - L' tokens in   */
/* ascending order (so every row of idx is a permutation of 0..L-1).         */
/* ------------------------------------------------------------------------ */
int orc_select(int B, int H, int L, const float *s_h, const int32_t *Lkeep,
               int32_t *idx) {
    if (B < 1 || H < 1 || L < 1) return 1;
    vt_pair *v = (vt_pair *)malloc(sizeof(vt_pair) * (size_t)L);
    unsigned char *keep = (unsigned char *)malloc((size_t)L);
    for (int b = 0; b < B; ++b) {
        const int Lk = Lkeep[b];
        if (Lk < 0 || Lk > L) { free(v); free(keep); return 2; }
        for (int h = 0; h < H; ++h) {
            const float *s = s_h + ((size_t)b * H + h) * L;
            int32_t *out = idx + ((size_t)b * H + h) * L;
            for (int t = 0; t < L; ++t) { v[t].v = s[t]; v[t].t = t; keep[t] = 0; }
            qsort(v, (size_t)L, sizeof(vt_pair), cmp_desc);
            for (int i = 0; i < Lk; ++i) keep[v[i].t] = 1;
            int a = 0, r = Lk;
            for (int t = 0; t < L; ++t) {
                if (keep[t]) out[a++] = t;
                else out[r++] = t;
            }
        }
    }
    free(v);
    free(keep);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Steps 4-5: compress and attend.  [notes] 整体框架 and 关键设计 1; [blog]    */
/* §1.1 (gather, softmax(Q̂K̂ᵀ/√d)V̂); [gist] §2 "Compression".                */
/* Row i of head h: query token t_i = idx[b,h,i] (identity when idx is NULL) */
/* attends to the kept keys t_j (j < L') whose ORIGINAL position satisfies   */
/* t_j <= t_i (causal on original positions).  Q from head h, K and V from   */
/* KV head h / (H / Hkv).  Output rows are requested as (b, h, i) triples.   */
/* ------------------------------------------------------------------------ */
typedef struct {
    int B, L, H, Hkv, d, dtype;
    const void *Q, *K, *V;
    const int32_t *idx, *Lkeep;
    double scale;
    const int32_t *rows;
    double *out;
} attend_job;

static void attend_item(void *arg, long item) {
    attend_job *j = (attend_job *)arg;
    const int b = j->rows[3 * item], h = j->rows[3 * item + 1], i = j->rows[3 * item + 2];
    const int L = j->L, d = j->d, G = j->H / j->Hkv, kv = h / G;
    const int Lk = j->Lkeep ? j->Lkeep[b] : L;
    double *o = j->out + (size_t)item * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (i < 0 || i >= Lk) return;
    const int32_t *S = j->idx ? j->idx + ((size_t)b * j->H + h) * L : NULL;
    const int ti = S ? S[i] : i;
    const size_t qoff = (((size_t)b * L + ti) * j->H + h) * d;
    double *z = (double *)malloc(sizeof(double) * (size_t)Lk);
    double zmax = -INFINITY;
    for (int jj = 0; jj < Lk; ++jj) {
        const int tj = S ? S[jj] : jj;
        if (tj > ti) { z[jj] = -INFINITY; continue; }
        const size_t koff = (((size_t)b * L + tj) * j->Hkv + kv) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += elem(j->Q, j->dtype, qoff + c) * elem(j->K, j->dtype, koff + c);
        z[jj] = j->scale * acc;
        if (z[jj] > zmax) zmax = z[jj];
    }
    double den = 0.0;
    for (int jj = 0; jj < Lk; ++jj)
        if (z[jj] != -INFINITY) den += exp(z[jj] - zmax);
    for (int jj = 0; jj < Lk; ++jj) {
        if (z[jj] == -INFINITY) continue;
        const int tj = S ? S[jj] : jj;
        const double w = exp(z[jj] - zmax) / den;
        const size_t voff = (((size_t)b * L + tj) * j->Hkv + kv) * d;
        for (int c = 0; c < d; ++c) o[c] += w * elem(j->V, j->dtype, voff + c);
    }
    free(z);
}

int orc_attend_rows(int B, int L, int H, int Hkv, int d, int dtype,
                    const void *Q, const void *K, const void *V,
                    const int32_t *idx, const int32_t *Lkeep, double scale,
                    long n_rows, const int32_t *rows, double *out, int nthreads) {
    if (B < 1 || L < 1 || H < 1 || Hkv < 1 || H % Hkv || d < 1) return 1;
    for (long r = 0; r < n_rows; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= H)
            return 2;
    attend_job j = {B, L, H, Hkv, d, dtype, Q, K, V, idx, Lkeep, scale, rows, out};
    run_items(attend_item, &j, n_rows, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Step 6: decompress and residual.  [notes] 关键设计 1 (scatter Ô back into  */
/* a zero L×d tensor, unselected rows stay 0, then X_{l+1} = X_l +           */
/* Decompress(Ô)); [blog] §1.1 解压缩阶段; [gist] §2 "Decompression".         */
/* Oh holds [B, H, L, d] rows of which the first Lkeep[b] are meaningful.    */
/* O_dec (optional) receives the decompressed tensor before the residual.    */
/* ------------------------------------------------------------------------ */
int orc_decompress_residual(int B, int L, int H, int d, int dtype,
                            const double *Oh, const int32_t *idx,
                            const int32_t *Lkeep, const void *X,
                            double *O_dec, double *Y) {
    if (B < 1 || L < 1 || H < 1 || d < 1) return 1;
    const size_t row = (size_t)H * d;
    double *O = O_dec ? O_dec : (double *)malloc(sizeof(double) * (size_t)B * L * row);
    memset(O, 0, sizeof(double) * (size_t)B * L * row);
    for (int b = 0; b < B; ++b) {
        const int Lk = Lkeep ? Lkeep[b] : L;
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < Lk; ++i) {
                const int t = idx ? idx[((size_t)b * H + h) * L + i] : i;
                const double *src = Oh + (((size_t)b * H + h) * L + i) * d;
                double *dst = O + ((size_t)b * L + t) * row + (size_t)h * d;
                for (int c = 0; c < d; ++c) dst[c] = src[c];
            }
    }
    for (size_t e = 0; e < (size_t)B * L * row; ++e) Y[e] = elem(X, dtype, e) + O[e];
    if (!O_dec) free(O);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Sparse-layer choice by inter-layer representation drift.  [notes] 关键设计 */
/* 3 (R_l = E_t[ ||h_{l+1,t} - h_{l,t}||_2 / (||h_{l,t}||_2 + eps) ], rank,  */
/* sparse layers = { l : R^_l <= delta }, delta = 0.5 by default); [blog] §2 */
/* (only the layers in the lower 50% of the drift ranking, i.e. below the    */
/* median, are made sparse).  Readings: R^_l = rank_l / N with rank_l the     */
/* 1-based position in ascending R (ties: lower layer first); the mean runs  */
/* over all T calibration tokens; eps is the caller's (the pages give none).  */
/* h holds N + 1 states [N + 1, T, D]: h_0 the input of layer 0, h_{l+1} the  */
/* output of layer l.                                                        */
/* ------------------------------------------------------------------------ */
int orc_drift(int N, long T, int D, int dtype, const void *h, double eps, double *R) {
    if (N < 1 || T < 1 || D < 1 || !(eps >= 0.0)) return 1;
    for (int l = 0; l < N; ++l) {
        double acc = 0.0;
        for (long t = 0; t < T; ++t) {
            const size_t a = ((size_t)l * T + t) * D, b = ((size_t)(l + 1) * T + t) * D;
            double dd = 0.0, hh = 0.0;
            for (int c = 0; c < D; ++c) {
                const double x = elem(h, dtype, a + c), y = elem(h, dtype, b + c);
                dd += (y - x) * (y - x);
                hh += x * x;
            }
            acc += sqrt(dd) / (sqrt(hh) + eps);
        }
        R[l] = acc / (double)T;
    }
    return 0;
}

int orc_drift_mask(int N, const double *R, double delta, int32_t *mask) {
    if (N < 1 || !(delta >= 0.0 && delta <= 1.0)) return 1;
    for (int l = 0; l < N; ++l) {
        int rank = 1;
        for (int m = 0; m < N; ++m)
            if (R[m] < R[l] || (R[m] == R[l] && m < l)) ++rank;
        mask[l] = ((double)rank / (double)N <= delta) ? 1 : 0;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block-sparse pattern inside the compressed space: [notes] 关键发现 (token  */
/* sparsity stacked on block-level sparsity is the most valuable pairing)    */
/* and [blog] §3.2 与现有方案的兼容性 ("token selection first, then block-    */
/* sparse computation").  The block choice is this project's own definition: */
/* the pages give none.  In head h's compressed                              */
/* order (position i is token S_h[i]):                                       */
/*   query pair p = positions [256p, 256p + 256), key block j = positions    */
/*   [128j, 128j + 128);                                                     */
/*   z[p][j] = scale * < mean of the pair's Q rows, mean of block j's K rows > */
/*   for the blocks j < 2p before the pair's own (diagonal) blocks;         */
/*   kept: j = 0, the diagonal blocks 2p and 2p + 1, and every j < 2p with   */
/*   z[p][j] >= max_j z[p][j] - theta, the threshold taken in fp32 on fp32   */
/*   logits (the precision the GPU decides in);                              */
/*   attention: row i attends to the keys i' <= i whose block is kept for    */
/*   the pair of i.                                                          */
/* z has shape [B, H, NP, NB] with NP = ceil(L / 256), NB = ceil(L / 128);   */
/* entries that do not exist are NaN.                                        */
/* ------------------------------------------------------------------------ */
int orc_block_logits(int B, int L, int H, int Hkv, int d, int dtype, const void *Q,
                     const void *K, const int32_t *idx, const int32_t *Lkeep, double scale,
                     double *z) {
    if (B < 1 || L < 1 || H < 1 || Hkv < 1 || H % Hkv || d < 1) return 1;
    const int NP = (L + 255) / 256, NB = (L + 127) / 128, G = H / Hkv;
    double *qb = (double *)malloc(sizeof(double) * (size_t)d);
    double *kb = (double *)malloc(sizeof(double) * (size_t)d);
    for (size_t e = 0; e < (size_t)B * H * NP * NB; ++e) z[e] = NAN;
    for (int b = 0; b < B; ++b) {
        const int Lk = Lkeep[b];
        for (int h = 0; h < H; ++h) {
            const int32_t *S = idx + ((size_t)b * H + h) * L;
            for (int p = 0; 256 * p < Lk; ++p) {
                const int i1 = 256 * p + 256 < Lk ? 256 * p + 256 : Lk;
                for (int c = 0; c < d; ++c) qb[c] = 0.0;
                for (int i = 256 * p; i < i1; ++i)
                    for (int c = 0; c < d; ++c)
                        qb[c] += elem(Q, dtype, (((size_t)b * L + S[i]) * H + h) * d + c);
                for (int c = 0; c < d; ++c) qb[c] /= (double)(i1 - 256 * p);
                for (int j = 0; j < 2 * p; ++j) {
                    for (int c = 0; c < d; ++c) kb[c] = 0.0;
                    for (int i = 128 * j; i < 128 * j + 128; ++i)
                        for (int c = 0; c < d; ++c)
                            kb[c] += elem(K, dtype, (((size_t)b * L + S[i]) * Hkv + h / G) * d + c);
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += qb[c] * (kb[c] / 128.0);
                    z[(((size_t)b * H + h) * NP + p) * NB + j] = scale * acc;
                }
            }
        }
    }
    free(qb);
    free(kb);
    return 0;
}

int orc_block_select(int B, int H, int L, const int32_t *Lkeep, const float *z, float theta,
                     uint8_t *keep) {
    if (B < 1 || H < 1 || L < 1 || !(theta >= 0.0f)) return 1;
    const int NP = (L + 255) / 256, NB = (L + 127) / 128;
    memset(keep, 0, (size_t)B * H * NP * NB);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int p = 0; 256 * p < Lkeep[b]; ++p) {
                const float *zr = z + (((size_t)b * H + h) * NP + p) * NB;
                uint8_t *kr = keep + (((size_t)b * H + h) * NP + p) * NB;
                kr[0] = 1;
                kr[2 * p] = 1;
                if (256 * p + 128 < Lkeep[b]) kr[2 * p + 1] = 1;
                if (p == 0) continue;
                float m = zr[0];
                for (int j = 1; j < 2 * p; ++j) if (zr[j] > m) m = zr[j];
                const float thr = m - theta; /* one fp32 subtraction */
                for (int j = 1; j < 2 * p; ++j) if (zr[j] >= thr) kr[j] = 1;
            }
    return 0;
}

int orc_attend_block_rows(int B, int L, int H, int Hkv, int d, int dtype, const void *Q,
                          const void *K, const void *V, const int32_t *idx,
                          const int32_t *Lkeep, const uint8_t *keep, double scale,
                          const int32_t *rows, long nrows, double *out) {
    if (B < 1 || L < 1 || H < 1 || Hkv < 1 || H % Hkv || d < 1) return 1;
    const int NP = (L + 255) / 256, NB = (L + 127) / 128, G = H / Hkv;
    double *z = (double *)malloc(sizeof(double) * (size_t)L);
    for (long r = 0; r < nrows; ++r) {
        const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        double *o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (i < 0 || i >= Lkeep[b]) continue;
        const int32_t *S = idx + ((size_t)b * H + h) * L;
        const uint8_t *kr = keep + (((size_t)b * H + h) * NP + i / 256) * NB;
        const size_t qoff = (((size_t)b * L + S[i]) * H + h) * d;
        double zmax = -INFINITY;
        for (int jj = 0; jj <= i; ++jj) {
            z[jj] = -INFINITY;
            if (!kr[jj / 128]) continue;
            const size_t koff = (((size_t)b * L + S[jj]) * Hkv + h / G) * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += elem(Q, dtype, qoff + c) * elem(K, dtype, koff + c);
            z[jj] = scale * acc;
            if (z[jj] > zmax) zmax = z[jj];
        }
        double den = 0.0;
        for (int jj = 0; jj <= i; ++jj) if (z[jj] != -INFINITY) den += exp(z[jj] - zmax);
        for (int jj = 0; jj <= i; ++jj) {
            if (z[jj] == -INFINITY) continue;
            const double w = exp(z[jj] - zmax) / den;
            const size_t voff = (((size_t)b * L + S[jj]) * Hkv + h / G) * d;
            for (int c = 0; c < d; ++c) o[c] += w * elem(V, dtype, voff + c);
        }
    }
    free(z);
    return 0;
}
