/*
 * vggt_oracle.c -- plain fp64 CPU oracle for the VGGT alternating-attention
 * hot path: frame attention, global attention, and AVGGT's training-free
 * Subsampled Global Attention (SGA).
 *
 * TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg are the only callers.  The CUDA
 * library never links, loads or calls this file, and the two share no code,
 * headers, tables or helpers.
 *
 * What it follows:
 *  - "VGGT CVPR25 Best Paper" notes, section "Alternating-Attention":
 *    frame-wise self-attention attends within one view, global
 *    self-attention treats all views' tokens as one sequence, no
 *    cross-attention.
 *  - VGGT-Omega notes, improvement one "Register Attention": in some global
 *    layers cross-frame attention is restricted to the register tokens (16
 *    per frame plus one camera token); image tokens take no part in it.
 *    Read here as global attention whose queries and keys are the special
 *    tokens of all frames (mode ORACLE_REGISTER; patch rows are not outputs).
 *  - "AVGGT: Rethinking Global Attention for Accelerating VGGT", technical
 *    summary section 3 (Methodology), step two "Subsampling Global
 *    Attention": every query kept; K/V kept on a uniform s_h x s_w grid of
 *    the patch tokens (one token per window, the middle one; all special
 *    tokens kept); each token's own (diagonal) term preserved; all dropped
 *    K/V columns replaced by one mean key / mean value; the kept part, the
 *    diagonal and the mean term share one softmax normalisation.
 *    The exact form used (multiplicity M_i = |D| - [i in D] on the mean
 *    column, logit q.kbar*scale + ln M_i) is the plainest reading that makes
 *    "the dropped columns are approximated by their mean" an equation: each
 *    dropped column other than the query's own is replaced by (kbar, vbar).
 *
 * Readings where the pages are silent:
 *  - token order inside a frame: the n_special special tokens first, then
 *    the h x w patch grid row-major;
 *  - window rule on one axis of length n with stride s: windows
 *    [a*s, min((a+1)*s, n)) for a = 0 .. ceil(n/s)-1 (a shorter last window
 *    included); the kept coordinate is a*s + (len-1)/2 (integer division);
 *  - the diagonal term is added only for a query whose own key was dropped;
 *  - the mean is over all of D (the query's own dropped key included);
 *  - M_i = 0 means no mean column at all (no ln 0); |D| = 0 means no mean.
 *
 * Layout: Q, K, V hold bf16 bit patterns, row-major [S][H][d], S = N*L,
 * L = n_special + h*w; token t = n*L + p.  Every bf16 is widened exactly to
 * double; every sum is in double; softmax is two-pass (max, then sum of
 * exp(x - max)) with libm exp().
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORACLE_FRAME = 0, ORACLE_GLOBAL = 1, ORACLE_SGA = 2, ORACLE_REGISTER = 3 };

static double widen(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_hardware_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Kept coordinates on one axis, by walking the windows one by one.
 * ("AVGGT" summary, section 3 step two: one representative per window,
 * the middle one -- "the middle one in each 3x3" in its analogy.) */
int oracle_axis_kept(int n, int s, int32_t *out)
{
    int cnt = 0;
    if (n <= 0 || s <= 0)
        return 0;
    for (int start = 0; start < n; start += s) {
        int len = (start + s <= n) ? s : (n - start);
        if (out)
            out[cnt] = start + (len - 1) / 2;
        cnt++;
    }
    return cnt;
}

/* Per-position keep mask for one frame: specials always kept, patches kept
 * iff both their row and column are window centres. Returns kept count. */
static int frame_keep_mask(int n_special, int h, int w, int s_h, int s_w,
                           unsigned char *keep /* [n_special + h*w] */)
{
    int L = n_special + h * w;
    memset(keep, 0, (size_t)L);
    for (int p = 0; p < n_special; p++)
        keep[p] = 1;
    int32_t *rk = (int32_t *)malloc(sizeof(int32_t) * (size_t)(h > 0 ? h : 1));
    int32_t *ck = (int32_t *)malloc(sizeof(int32_t) * (size_t)(w > 0 ? w : 1));
    int nr = oracle_axis_kept(h, s_h, rk);
    int nc = oracle_axis_kept(w, s_w, ck);
    for (int a = 0; a < nr; a++)
        for (int b = 0; b < nc; b++)
            keep[n_special + rk[a] * w + ck[b]] = 1;
    free(rk);
    free(ck);
    int kept = 0;
    for (int p = 0; p < L; p++)
        kept += keep[p];
    return kept;
}

/* SGA index: kept token list (ascending) and per-token multiplicity
 * M_t = |D| - [t in D].  Either output pointer may be NULL; the counts are
 * always returned.  Built by scanning every token against the window mask. */
int oracle_sga_build_index(int N, int n_special, int h, int w, int s_h, int s_w,
                           int32_t *kept_idx, int32_t *mult,
                           int64_t *n_kept_out, int64_t *n_dropped_out)
{
    if (N < 0 || n_special < 0 || h < 0 || w < 0 || s_h < 1 || s_w < 1)
        return -1;
    int L = n_special + h * w;
    unsigned char *keep = (unsigned char *)malloc((size_t)(L > 0 ? L : 1));
    frame_keep_mask(n_special, h, w, s_h, s_w, keep);
    int64_t S = (int64_t)N * L;
    int64_t nk = 0, nd = 0;
    for (int64_t t = 0; t < S; t++) {
        int p = (int)(t % L);
        if (keep[p])
            nk++;
        else
            nd++;
    }
    int64_t pos = 0;
    for (int64_t t = 0; t < S; t++) {
        int p = (int)(t % L);
        if (keep[p]) {
            if (kept_idx)
                kept_idx[pos] = (int32_t)t;
            pos++;
        }
        if (mult)
            mult[t] = (int32_t)(nd - (keep[p] ? 0 : 1));
    }
    free(keep);
    if (n_kept_out)
        *n_kept_out = nk;
    if (n_dropped_out)
        *n_dropped_out = nd;
    return 0;
}

/* Mean key and mean value per head over the dropped set D, summed directly
 * over D in double (not "total minus kept").  kbar, vbar: [H][d].
 * Returns -1 if |D| = 0 (the means are then undefined and not written). */
int oracle_sga_means(const uint16_t *k, const uint16_t *v, int N, int n_special,
                     int h, int w, int H, int d, int s_h, int s_w,
                     double *kbar, double *vbar)
{
    int L = n_special + h * w;
    unsigned char *keep = (unsigned char *)malloc((size_t)(L > 0 ? L : 1));
    frame_keep_mask(n_special, h, w, s_h, s_w, keep);
    int64_t S = (int64_t)N * L;
    size_t HD = (size_t)H * (size_t)d;
    memset(kbar, 0, sizeof(double) * HD);
    memset(vbar, 0, sizeof(double) * HD);
    int64_t nd = 0;
    for (int64_t t = 0; t < S; t++) {
        if (keep[t % L])
            continue;
        nd++;
        const uint16_t *kr = k + (size_t)t * HD;
        const uint16_t *vr = v + (size_t)t * HD;
        for (size_t e = 0; e < HD; e++) {
            kbar[e] += widen(kr[e]);
            vbar[e] += widen(vr[e]);
        }
    }
    free(keep);
    if (nd == 0)
        return -1;
    for (size_t e = 0; e < HD; e++) {
        kbar[e] /= (double)nd;
        vbar[e] /= (double)nd;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention for sampled query rows.                                         */

typedef struct {
    int mode;
    const uint16_t *q, *k, *v;
    int N, n_special, h, w, H, d;
    double scale;
    /* SGA state (mode == ORACLE_SGA) */
    const int32_t *kept;   /* ascending kept token list */
    int64_t n_kept, n_dropped;
    const unsigned char *keep; /* per-position keep mask, [L] */
    const double *kbar, *vbar; /* [H][d], valid iff n_dropped > 0 */
    /* work */
    const int64_t *rows;
    int64_t row_begin, row_end;
    double *out; /* [nrows][H][d] */
    double *lse; /* [nrows][H] or NULL */
    int status;
} job_t;

static double dot_q_bf16(const double *qd, const uint16_t *kr, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; c++)
        acc += qd[c] * widen(kr[c]);
    return acc;
}

static void *attn_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int H = J->H, d = J->d;
    const int L = J->n_special + J->h * J->w;
    const int64_t S = (int64_t)J->N * L;
    const size_t HD = (size_t)H * (size_t)d;

    int64_t max_keys;
    if (J->mode == ORACLE_FRAME)
        max_keys = L;
    else if (J->mode == ORACLE_GLOBAL)
        max_keys = S;
    else if (J->mode == ORACLE_REGISTER)
        max_keys = (int64_t)J->N * J->n_special;
    else
        max_keys = J->n_kept + 2;

    double *logit = (double *)malloc(sizeof(double) * (size_t)(max_keys > 0 ? max_keys : 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
    if (!logit || !qd || !acc) {
        J->status = -2;
        free(logit); free(qd); free(acc);
        return NULL;
    }

    for (int64_t r = J->row_begin; r < J->row_end; r++) {
        const int64_t i = J->rows[r];
        const int64_t frame = i / L;
        for (int hh = 0; hh < H; hh++) {
            const uint16_t *qr = J->q + (size_t)i * HD + (size_t)hh * d;
            for (int c = 0; c < d; c++)
                qd[c] = widen(qr[c]);

            /* Pass 1: every logit of this query's key list. */
            int64_t nl = 0;
            int has_diag = 0, has_mean = 0;
            int64_t M_i = 0;
            if (J->mode == ORACLE_FRAME || J->mode == ORACLE_GLOBAL) {
                int64_t j0 = (J->mode == ORACLE_FRAME) ? frame * L : 0;
                int64_t j1 = (J->mode == ORACLE_FRAME) ? (frame + 1) * L : S;
                for (int64_t j = j0; j < j1; j++)
                    logit[nl++] = J->scale *
                        dot_q_bf16(qd, J->k + (size_t)j * HD + (size_t)hh * d, d);
            } else if (J->mode == ORACLE_REGISTER) {
                for (int64_t n = 0; n < J->N; n++)
                    for (int sp = 0; sp < J->n_special; sp++) {
                        int64_t j = n * L + sp;
                        logit[nl++] = J->scale *
                            dot_q_bf16(qd, J->k + (size_t)j * HD + (size_t)hh * d, d);
                    }
            } else {
                for (int64_t a = 0; a < J->n_kept; a++) {
                    int64_t j = J->kept[a];
                    logit[nl++] = J->scale *
                        dot_q_bf16(qd, J->k + (size_t)j * HD + (size_t)hh * d, d);
                }
                int i_dropped = !J->keep[i % L];
                M_i = J->n_dropped - (i_dropped ? 1 : 0);
                if (i_dropped) {
                    has_diag = 1;
                    logit[nl++] = J->scale *
                        dot_q_bf16(qd, J->k + (size_t)i * HD + (size_t)hh * d, d);
                }
                if (M_i > 0) {
                    has_mean = 1;
                    const double *kb = J->kbar + (size_t)hh * d;
                    double s = 0.0;
                    for (int c = 0; c < d; c++)
                        s += qd[c] * kb[c];
                    logit[nl++] = J->scale * s + log((double)M_i);
                }
            }

            double m = -INFINITY;
            for (int64_t a = 0; a < nl; a++)
                if (logit[a] > m)
                    m = logit[a];

            /* Pass 2: normaliser and weighted values, in the same order. */
            double denom = 0.0;
            for (int c = 0; c < d; c++)
                acc[c] = 0.0;
            int64_t a = 0;
            if (J->mode == ORACLE_FRAME || J->mode == ORACLE_GLOBAL) {
                int64_t j0 = (J->mode == ORACLE_FRAME) ? frame * L : 0;
                for (; a < nl; a++) {
                    double e = exp(logit[a] - m);
                    denom += e;
                    const uint16_t *vr = J->v + (size_t)(j0 + a) * HD + (size_t)hh * d;
                    for (int c = 0; c < d; c++)
                        acc[c] += e * widen(vr[c]);
                }
            } else if (J->mode == ORACLE_REGISTER) {
                for (; a < nl; a++) {
                    double e = exp(logit[a] - m);
                    denom += e;
                    const int64_t j = (a / J->n_special) * L + (a % J->n_special);
                    const uint16_t *vr = J->v + (size_t)j * HD + (size_t)hh * d;
                    for (int c = 0; c < d; c++)
                        acc[c] += e * widen(vr[c]);
                }
            } else {
                for (; a < J->n_kept; a++) {
                    double e = exp(logit[a] - m);
                    denom += e;
                    const uint16_t *vr = J->v + (size_t)J->kept[a] * HD + (size_t)hh * d;
                    for (int c = 0; c < d; c++)
                        acc[c] += e * widen(vr[c]);
                }
                if (has_diag) {
                    double e = exp(logit[a++] - m);
                    denom += e;
                    const uint16_t *vr = J->v + (size_t)i * HD + (size_t)hh * d;
                    for (int c = 0; c < d; c++)
                        acc[c] += e * widen(vr[c]);
                }
                if (has_mean) {
                    double e = exp(logit[a++] - m);
                    denom += e;
                    const double *vb = J->vbar + (size_t)hh * d;
                    for (int c = 0; c < d; c++)
                        acc[c] += e * vb[c];
                }
            }
            double *o = J->out + ((size_t)r * H + hh) * d;
            for (int c = 0; c < d; c++)
                o[c] = acc[c] / denom;
            if (J->lse)
                J->lse[(size_t)r * H + hh] = m + log(denom);
        }
    }
    free(logit);
    free(qd);
    free(acc);
    return NULL;
}

/* Attention outputs for the query tokens rows[0..nrows), all heads.
 * mode 0: frame attention (keys = the query's own frame);
 * mode 1: global attention (keys = all S tokens);
 * mode 2: SGA with stride (s_h, s_w) (ignored for the other modes);
 * mode 3: register attention (queries and keys: the special tokens of all
 *         frames; every row must be a special token).
 * out: [nrows][H][d] double; lse: [nrows][H] double (natural log of the
 * softmax normaliser including the max), may be NULL.
 * nthreads <= 0 uses every online core.  Returns 0 on success. */
int oracle_attn(int mode, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                int N, int n_special, int h, int w, int H, int d, double scale,
                int s_h, int s_w, const int64_t *rows, int64_t nrows,
                double *out, double *lse, int nthreads)
{
    if (mode < 0 || mode > 3 || N < 1 || n_special < 0 || h < 0 || w < 0 ||
        H < 1 || d < 1 || nrows < 0)
        return -1;
    const int L = n_special + h * w;
    if (L < 1)
        return -1;
    const int64_t S = (int64_t)N * L;
    for (int64_t r = 0; r < nrows; r++) {
        if (rows[r] < 0 || rows[r] >= S)
            return -1;
        /* register attention is defined for the special-token rows only */
        if (mode == ORACLE_REGISTER && rows[r] % L >= n_special)
            return -1;
    }

    int32_t *kept = NULL;
    unsigned char *keep = NULL;
    double *kbar = NULL, *vbar = NULL;
    int64_t n_kept = 0, n_dropped = 0;
    if (mode == ORACLE_SGA) {
        if (s_h < 1 || s_w < 1)
            return -1;
        oracle_sga_build_index(N, n_special, h, w, s_h, s_w, NULL, NULL, &n_kept, &n_dropped);
        kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_kept > 0 ? n_kept : 1));
        oracle_sga_build_index(N, n_special, h, w, s_h, s_w, kept, NULL, NULL, NULL);
        keep = (unsigned char *)malloc((size_t)L);
        frame_keep_mask(n_special, h, w, s_h, s_w, keep);
        size_t HD = (size_t)H * (size_t)d;
        kbar = (double *)calloc(HD, sizeof(double));
        vbar = (double *)calloc(HD, sizeof(double));
        if (n_dropped > 0)
            oracle_sga_means(k, v, N, n_special, h, w, H, d, s_h, s_w, kbar, vbar);
    }

    if (nthreads <= 0)
        nthreads = oracle_hardware_threads();
    if (nthreads > nrows)
        nthreads = nrows > 0 ? (int)nrows : 1;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * (size_t)nthreads);
    int64_t per = nrows / nthreads, extra = nrows % nthreads, begin = 0;
    for (int t = 0; t < nthreads; t++) {
        job_t *J = &jobs[t];
        J->mode = mode; J->q = q; J->k = k; J->v = v;
        J->N = N; J->n_special = n_special; J->h = h; J->w = w; J->H = H; J->d = d;
        J->scale = scale;
        J->kept = kept; J->n_kept = n_kept; J->n_dropped = n_dropped; J->keep = keep;
        J->kbar = kbar; J->vbar = vbar;
        J->rows = rows; J->out = out; J->lse = lse; J->status = 0;
        int64_t cnt = per + (t < extra ? 1 : 0);
        J->row_begin = begin; J->row_end = begin + cnt;
        begin += cnt;
    }
    int status = 0;
    if (nthreads == 1) {
        attn_worker(&jobs[0]);
        status = jobs[0].status;
    } else {
        for (int t = 0; t < nthreads; t++)
            pthread_create(&tid[t], NULL, attn_worker, &jobs[t]);
        for (int t = 0; t < nthreads; t++) {
            pthread_join(tid[t], NULL);
            if (jobs[t].status)
                status = jobs[t].status;
        }
    }
    free(tid); free(jobs); free(kept); free(keep); free(kbar); free(vbar);
    return status;
}

/* ---------------------------------------------------------------------
 * Fused QKV projection with 2D rotary position embedding.
 *
 * What it follows: the trunk's attention layers take Q, K and V from a
 * linear projection of the tokens, and a rotary position embedding (RoPE)
 * is applied to Q and K before each attention ("Feed-forward optimization
 * in Visual Geometry Grounded and 3DGS", Cut3R part, section 3.5
 * architecture details, position encoding).  The pages give no formula,
 * so the plainest 2D form is taken:
 *  - y[t][n] = sum_c x[t][c] * W[n][c] + b[n], n in [0, 3C), C = H*d
 *    (W in the out x in layout of a linear layer);
 *    Q = y[:, 0:C], K = y[:, C:2C], V = y[:, 2C:3C], each [S][H][d];
 *  - a patch token at grid (r, c) has position r for the first half of
 *    each head's d dimensions and c for the second half; special tokens are
 *    not rotated;
 *  - within a half of width e = d/2, dimensions i and i + e/2 form a pair
 *    (i < e/2) rotated by the angle pos * base^(-2i/e):
 *      a' = a cos - b sin,   b' = b cos + a sin.
 * Everything in double; bias is fp32, x and W bf16.
 * --------------------------------------------------------------------- */
typedef struct {
    const uint16_t *x, *w;
    const float *bias;
    int C, d, L, n_special, pw;
    double base;
    const int64_t *rows;
    int64_t r0, r1;
    double *q, *k, *v;
} QkvJob;

static void rope_half(double *x, int e, double pos, double base)
{
    for (int i = 0; i < e / 2; ++i) {
        const double ang = pos * pow(base, -2.0 * i / e);
        const double a = x[i], b = x[i + e / 2];
        x[i] = a * cos(ang) - b * sin(ang);
        x[i + e / 2] = b * cos(ang) + a * sin(ang);
    }
}

static void *qkv_worker(void *arg)
{
    QkvJob *J = (QkvJob *)arg;
    const int C = J->C;
    double *xr = (double *)malloc(sizeof(double) * (size_t)C);
    double *y = (double *)malloc(sizeof(double) * 3 * (size_t)C);
    for (int64_t r = J->r0; r < J->r1; ++r) {
        const int64_t t = J->rows[r];
        for (int c = 0; c < C; ++c)
            xr[c] = widen(J->x[t * C + c]);
        for (int n = 0; n < 3 * C; ++n) {
            double acc = 0.0;
            const uint16_t *wn = J->w + (size_t)n * C;
            for (int c = 0; c < C; ++c)
                acc += xr[c] * widen(wn[c]);
            y[n] = acc + (J->bias ? (double)J->bias[n] : 0.0);
        }
        const int p = (int)(t % J->L);
        if (p >= J->n_special) {
            const int g = p - J->n_special;
            const double pr = g / J->pw, pc = g % J->pw;
            for (int part = 0; part < 2; ++part)  /* Q, then K */
                for (int h = 0; h < C / J->d; ++h) {
                    double *head = y + part * C + h * J->d;
                    rope_half(head, J->d / 2, pr, J->base);
                    rope_half(head + J->d / 2, J->d / 2, pc, J->base);
                }
        }
        memcpy(J->q + r * C, y, sizeof(double) * C);
        memcpy(J->k + r * C, y + C, sizeof(double) * C);
        memcpy(J->v + r * C, y + 2 * C, sizeof(double) * C);
    }
    free(xr);
    free(y);
    return NULL;
}

/* q, k, v: double [nrows][C] for the token indices in rows.  d must be
 * divisible by 4 (two halves of even width).  Returns 0, or -1 on bad
 * arguments. */
int oracle_qkv_rope(const uint16_t *x, const uint16_t *w, const float *bias, int N, int n_special, int ph,
                    int pw, int H, int d, double base, const int64_t *rows, int64_t nrows, double *q,
                    double *k, double *v, int nthreads)
{
    if (N < 1 || n_special < 0 || ph < 0 || pw < 0 || H < 1 || d < 4 || d % 4 || !(base > 0.0) || nrows < 0)
        return -1;
    if (ph * pw > 0 && pw == 0)
        return -1;
    const int L = n_special + ph * pw;
    const int64_t S = (int64_t)N * L;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= S)
            return -1;
    if (nthreads <= 0)
        nthreads = oracle_hardware_threads();
    if (nthreads > 256)
        nthreads = 256;
    if (nthreads > nrows)
        nthreads = nrows > 0 ? (int)nrows : 1;
    pthread_t tid[256];
    QkvJob jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (QkvJob){x, w, bias, H * d, d, L, n_special, pw > 0 ? pw : 1, base, rows,
                           nrows * t / nthreads, nrows * (t + 1) / nthreads, q, k, v};
        pthread_create(&tid[t], NULL, qkv_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(tid[t], NULL);
    return 0;
}

/* Output projection of an attention layer, fp64: y[r][n] = sum_c
 * x[rows[r]][c] * W[n][c] + b[n] (x bf16 [*, n_in], W bf16 [n_out, n_in],
 * b fp32 or NULL), y double [nrows][n_out].  Returns 0, or -1 on bad
 * arguments. */
int oracle_linear(const uint16_t *x, const uint16_t *w, const float *bias, int64_t n_rows_x, int n_in, int n_out,
                  const int64_t *rows, int64_t nrows, double *y)
{
    if (n_in < 1 || n_out < 1 || nrows < 0)
        return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[r] < 0 || rows[r] >= n_rows_x)
            return -1;
        const uint16_t *xr = x + rows[r] * n_in;
        for (int n = 0; n < n_out; ++n) {
            double acc = 0.0;
            for (int c = 0; c < n_in; ++c)
                acc += widen(xr[c]) * widen(w[(size_t)n * n_in + c]);
            y[r * n_out + n] = acc + (bias ? (double)bias[n] : 0.0);
        }
    }
    return 0;
}
