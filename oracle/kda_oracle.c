/*
 * kda_oracle.c -- plain, slow fp64 CPU oracle for the KDA forward scan and the
 * modality-aware short convolution (mShortConv).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the definition the CUDA path is checked
 * against.  Only the test-suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it; the product path never does.  It shares no code, header, table
 * or helper with the CUDA library.
 *
 * Sources (page title, section / equation):
 *  - "Chimera: hybrid attention + Chinchilla scaling" (pchao.org translation of the
 *    Chimera paper), section 3.3, Eq. 14: the per-head state update
 *        S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *    with S_t in R^{dk x dv} the state AFTER token t, alpha_t in (0,1)^{dk} a
 *    per-key-channel forget gate and beta_t in (0,1) one scalar per head and token.
 *    The same section says the state is reset to S_0 = 0 at every packed-sample
 *    boundary.  Eq. 15 reads the state out as S_t^T q_t.
 *  - agifrontier.github.io summary of the same paper, section on the single-stream
 *    hybrid design: the clean LaTeX form of Eq. 14, which fixes the parenthesisation
 *    (decay first, then the rank-one erase, then the write).
 *  - pchao.org translation, section 3.4 (modality-aware short convolution): text
 *    tokens get a causal 1-D depthwise conv, visual tokens a depthwise 3-D conv over
 *    (time, height, width) that is causal in time; an image is the one-frame case;
 *    no kernel crosses a segment boundary; outputs return to their packed positions.
 *    The agifrontier summary adds that the 3-D conv is symmetric in space and that an
 *    image is convolved as a 2-D plane.
 *  - pchao.org translation, section 3.3 Eq. 12: time-first raster order
 *    m = i*H*W + j*W + k inside a visual segment.
 *
 * Readings taken where the paper is silent (each is listed in the design notes):
 *  - alpha is passed as g = ln(alpha) (g <= 0); the oracle forms alpha = exp(g).
 *  - no 1/sqrt(dk) scaling and no normalisation inside the scan.
 *  - text conv: y[t] = sum_{j<Kt} w[c,j] * x[t-(Kt-1)+j], zero before the segment.
 *  - image conv: 3x3, y[r,s] = sum_{a,e} w[c,a,e] x[r-1+a, s-1+e], zero outside.
 *  - video conv: 3x3x3, y[f,r,s] = sum_{tau,a,e} w[c,tau,a,e] x[f-2+tau, r-1+a, s-1+e],
 *    frames before the segment's first frame and out-of-grid positions are zero.
 *  - no bias, no activation after the conv.
 *  - L2 normalisation of conv outputs (fused path) uses no epsilon; a zero vector
 *    stays zero.
 *
 * All arithmetic is in double.  Inputs are read at their stored precision
 * (fp32, bf16 bit patterns or fp64) and promoted exactly.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

static double rd(const void* p, int dtype, int64_t i)
{
    if (dtype == OR_F32) return (double)((const float*)p)[i];
    if (dtype == OR_BF16) {
        uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return ((const double*)p)[i];
}

/* ------------------------------------------------------------------------- */
/* KDA token-by-token scan                                                    */
/* ------------------------------------------------------------------------- */

typedef struct {
    const void *q, *k, *v, *g, *beta;
    int dtype;
    const double* S0;         /* [B,H,Dk,Dv] or NULL (zeros) */
    double* o;                /* element strides below; NULL: not written */
    int64_t o_sb, o_st, o_sh; /* o[b*o_sb + t*o_st + h*o_sh + j] */
    double* ST;               /* [B,H,Dk,Dv] or NULL */
    int B, T, H, Dk, Dv;
    const int* pairs;         /* n_pairs (b,h) pairs, flattened; NULL: all */
    int n_pairs;
    int next;                 /* work counter */
    pthread_mutex_t mu;
} kda_job;

static void kda_one_head(kda_job* J, int b, int h)
{
    const int T = J->T, H = J->H, Dk = J->Dk, Dv = J->Dv;
    double* S = (double*)calloc((size_t)Dk * Dv, sizeof(double));
    double* kS = (double*)calloc((size_t)Dv, sizeof(double));
    if (!S || !kS) { free(S); free(kS); return; }
    const int64_t sbase = ((int64_t)b * H + h) * Dk * Dv;
    if (J->S0) memcpy(S, J->S0 + sbase, sizeof(double) * Dk * Dv);

    for (int t = 0; t < T; ++t) {
        const int64_t tok = (int64_t)b * T + t;
        const int64_t ik = (tok * H + h) * Dk;  /* q, k, g row */
        const int64_t iv = (tok * H + h) * Dv;  /* v row */
        const double beta = rd(J->beta, J->dtype, tok * H + h);

        /* Diag(alpha_t) S_{t-1}: row i of the state decays by alpha_t[i] = exp(g_t[i]). */
        for (int i = 0; i < Dk; ++i) {
            const double a = exp(rd(J->g, J->dtype, ik + i));
            for (int j = 0; j < Dv; ++j) S[(int64_t)i * Dv + j] *= a;
        }
        /* (I - beta k k^T) applied to the decayed state: subtract beta k (k^T S). */
        for (int j = 0; j < Dv; ++j) kS[j] = 0.0;
        for (int i = 0; i < Dk; ++i) {
            const double ki = rd(J->k, J->dtype, ik + i);
            for (int j = 0; j < Dv; ++j) kS[j] += ki * S[(int64_t)i * Dv + j];
        }
        for (int i = 0; i < Dk; ++i) {
            const double ki = rd(J->k, J->dtype, ik + i);
            for (int j = 0; j < Dv; ++j) S[(int64_t)i * Dv + j] -= beta * ki * kS[j];
        }
        /* + beta k v^T */
        for (int i = 0; i < Dk; ++i) {
            const double bk = beta * rd(J->k, J->dtype, ik + i);
            for (int j = 0; j < Dv; ++j) S[(int64_t)i * Dv + j] += bk * rd(J->v, J->dtype, iv + j);
        }
        /* readout with the state after token t: o_t = S_t^T q_t */
        if (J->o) {
            double* orow = J->o + (int64_t)b * J->o_sb + (int64_t)t * J->o_st + (int64_t)h * J->o_sh;
            for (int j = 0; j < Dv; ++j) orow[j] = 0.0;
            for (int i = 0; i < Dk; ++i) {
                const double qi = rd(J->q, J->dtype, ik + i);
                for (int j = 0; j < Dv; ++j) orow[j] += S[(int64_t)i * Dv + j] * qi;
            }
        }
    }
    if (J->ST) memcpy(J->ST + sbase, S, sizeof(double) * Dk * Dv);
    free(S);
    free(kS);
}

static void* kda_worker(void* arg)
{
    kda_job* J = (kda_job*)arg;
    const int total = J->pairs ? J->n_pairs : J->B * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int w = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (w >= total) break;
        int b, h;
        if (J->pairs) { b = J->pairs[2 * w]; h = J->pairs[2 * w + 1]; }
        else { b = w / J->H; h = w % J->H; }
        kda_one_head(J, b, h);
    }
    return NULL;
}

/* Runs the scan for every listed (b,h) pair (all pairs when `pairs` is NULL).
 * Returns 0 on success, -1 on bad arguments. */
int oracle_kda_forward(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, int dtype, const double* S0,
                       double* o, int64_t o_sb, int64_t o_st, int64_t o_sh,
                       double* ST, int B, int T, int H, int Dk, int Dv,
                       const int* pairs, int n_pairs, int nthreads)
{
    if (!q || !k || !v || !g || !beta) return -1;
    if (B < 0 || T < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (dtype != OR_F32 && dtype != OR_BF16 && dtype != OR_F64) return -1;
    if (pairs) {
        for (int i = 0; i < n_pairs; ++i)
            if (pairs[2 * i] < 0 || pairs[2 * i] >= B || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= H)
                return -1;
    }
    kda_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.dtype = dtype;
    J.S0 = S0; J.o = o; J.o_sb = o_sb; J.o_st = o_st; J.o_sh = o_sh; J.ST = ST;
    J.B = B; J.T = T; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.pairs = pairs; J.n_pairs = n_pairs; J.next = 0;
    pthread_mutex_init(&J.mu, NULL);
    const int total = pairs ? n_pairs : B * H;
    int nt = nthreads < 1 ? 1 : nthreads;
    if (nt > total) nt = total > 0 ? total : 1;
    pthread_t* th = (pthread_t*)calloc((size_t)nt, sizeof(pthread_t));
    for (int i = 1; i < nt; ++i) pthread_create(&th[i], NULL, kda_worker, &J);
    kda_worker(&J);
    for (int i = 1; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* mShortConv: direct loops per segment                                       */
/* ------------------------------------------------------------------------- */

/* Field order mirrors the library's segment record so that one packed Python
 * structure can describe both; the definition here is the oracle's own. */
typedef struct {
    int32_t modality;   /* 0 text, 1 image, 2 video */
    int32_t pad0;
    int64_t start;      /* first token of the segment in the packed row */
    int32_t F, Hgt, Wid;
    int32_t weight_set;
} oracle_segment;

typedef struct {
    const void* x;
    int dtype;
    double* y;
    int B, T, C, c_lo, c_hi;
    const oracle_segment* segs;
    int n_segs, Kt;
    const float *w_text, *w_image, *w_video;
    int next;
    pthread_mutex_t mu;
} conv_job;

static double xat(const conv_job* J, int b, int64_t pos, int c)
{
    return rd(J->x, J->dtype, ((int64_t)b * J->T + pos) * J->C + c);
}

static void conv_channel(conv_job* J, int b, int c)
{
    for (int s = 0; s < J->n_segs; ++s) {
        const oracle_segment* sg = &J->segs[s];
        const int64_t st = sg->start;
        if (sg->modality == 0) {
            const int64_t len = sg->Wid;
            const float* w = J->w_text + ((int64_t)sg->weight_set * J->C + c) * J->Kt;
            for (int64_t t = 0; t < len; ++t) {
                double acc = 0.0;
                for (int j = 0; j < J->Kt; ++j) {
                    const int64_t src = t - (J->Kt - 1) + j;   /* causal: the last tap is t */
                    if (src < 0) continue;                      /* zero before the segment */
                    acc += (double)w[j] * xat(J, b, st + src, c);
                }
                J->y[((int64_t)b * J->T + st + t) * J->C + c] = acc;
            }
        } else if (sg->modality == 1) {
            const int Hh = sg->Hgt, Ww = sg->Wid;
            const float* w = J->w_image + ((int64_t)sg->weight_set * J->C + c) * 9;
            for (int r = 0; r < Hh; ++r)
                for (int q = 0; q < Ww; ++q) {
                    double acc = 0.0;
                    for (int a = 0; a < 3; ++a)
                        for (int e = 0; e < 3; ++e) {
                            const int rr = r - 1 + a, qq = q - 1 + e;
                            if (rr < 0 || rr >= Hh || qq < 0 || qq >= Ww) continue;
                            acc += (double)w[a * 3 + e] * xat(J, b, st + (int64_t)rr * Ww + qq, c);
                        }
                    J->y[((int64_t)b * J->T + st + (int64_t)r * Ww + q) * J->C + c] = acc;
                }
        } else {
            const int Ff = sg->F, Hh = sg->Hgt, Ww = sg->Wid;
            const float* w = J->w_video + ((int64_t)sg->weight_set * J->C + c) * 27;
            for (int f = 0; f < Ff; ++f)
                for (int r = 0; r < Hh; ++r)
                    for (int q = 0; q < Ww; ++q) {
                        double acc = 0.0;
                        for (int tau = 0; tau < 3; ++tau)
                            for (int a = 0; a < 3; ++a)
                                for (int e = 0; e < 3; ++e) {
                                    const int ff = f - 2 + tau, rr = r - 1 + a, qq = q - 1 + e;
                                    if (ff < 0 || rr < 0 || rr >= Hh || qq < 0 || qq >= Ww) continue;
                                    const int64_t m = ((int64_t)ff * Hh + rr) * Ww + qq; /* Eq. 12 order */
                                    acc += (double)w[(tau * 3 + a) * 3 + e] * xat(J, b, st + m, c);
                                }
                        const int64_t m = ((int64_t)f * Hh + r) * Ww + q;
                        J->y[((int64_t)b * J->T + st + m) * J->C + c] = acc;
                    }
        }
    }
}

static void* conv_worker(void* arg)
{
    conv_job* J = (conv_job*)arg;
    const int nc = J->c_hi - J->c_lo;
    const int total = J->B * nc;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int w = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (w >= total) break;
        conv_channel(J, w / nc, J->c_lo + w % nc);
    }
    return NULL;
}

static int64_t seg_len(const oracle_segment* s)
{
    if (s->modality == 0) return s->Wid;
    if (s->modality == 1) return (int64_t)s->Hgt * s->Wid;
    return (int64_t)s->F * s->Hgt * s->Wid;
}

/* y[b,t,c] (fp64, [B,T,C]) for channels c_lo..c_hi-1; positions not covered by a
 * segment are left untouched.  Returns 0, or -1 on a bad segment table. */
int oracle_mshortconv(const void* x, int dtype, double* y, int B, int T, int C,
                      int c_lo, int c_hi, const oracle_segment* segs, int n_segs, int Kt,
                      const float* w_text, const float* w_image, const float* w_video,
                      int nthreads)
{
    if (!x || !y || !segs || B < 0 || T < 0 || C <= 0 || Kt <= 0) return -1;
    if (c_lo < 0 || c_hi > C || c_lo >= c_hi) return -1;
    for (int s = 0; s < n_segs; ++s) {
        const oracle_segment* sg = &segs[s];
        if (sg->modality < 0 || sg->modality > 2) return -1;
        if (sg->start < 0 || sg->start + seg_len(&segs[s]) > T) return -1;
        if (sg->modality == 0 && !w_text) return -1;
        if (sg->modality == 1 && !w_image) return -1;
        if (sg->modality == 2 && !w_video) return -1;
    }
    conv_job J;
    memset(&J, 0, sizeof J);
    J.x = x; J.dtype = dtype; J.y = y; J.B = B; J.T = T; J.C = C; J.c_lo = c_lo; J.c_hi = c_hi;
    J.segs = segs; J.n_segs = n_segs; J.Kt = Kt;
    J.w_text = w_text; J.w_image = w_image; J.w_video = w_video;
    pthread_mutex_init(&J.mu, NULL);
    const int total = B * (c_hi - c_lo);
    int nt = nthreads < 1 ? 1 : nthreads;
    if (nt > total) nt = total > 0 ? total : 1;
    pthread_t* th = (pthread_t*)calloc((size_t)nt, sizeof(pthread_t));
    for (int i = 1; i < nt; ++i) pthread_create(&th[i], NULL, conv_worker, &J);
    conv_worker(&J);
    for (int i = 1; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

/* In-place L2 normalisation of every (row, head) vector of length D in an fp64
 * array of n_rows * H * D values; a zero vector stays zero. */
void oracle_l2norm_heads(double* x, int64_t n_rows, int H, int D)
{
    for (int64_t r = 0; r < n_rows * H; ++r) {
        double* p = x + r * D;
        double ss = 0.0;
        for (int i = 0; i < D; ++i) ss += p[i] * p[i];
        if (ss == 0.0) continue;
        const double inv = 1.0 / sqrt(ss);
        for (int i = 0; i < D; ++i) p[i] *= inv;
    }
}
