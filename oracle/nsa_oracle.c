/*
 * nsa_oracle.c -- plain, slow, fp64 CPU oracle for the Native Sparse Attention
 * (NSA) per-layer operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * Sources (the pages, cited by page title and section):
 *  - "硬件对齐+原生训练！DeepSeek NSA打造高效稀疏Attention" (m.youleyou.com),
 *    section 二 "NSA核心工作": overall framework (remapped K/V, three mapping
 *    strategies, sigmoid gates), 令牌压缩 (token compression with block length l,
 *    stride d, learnable map with intra-block position encoding), 令牌选择
 *    (importance scores from the compressed branch's attention, mapping to
 *    selection blocks when the blockings differ, sum over the heads of a GQA
 *    group, top-n with 1 initial + 2 local blocks always kept), 滑动窗口 (window
 *    branch), 最终输出计算 (gated sum), 效率分析 (decode reads).
 *  - "DeepseekNativelySparseAttention" (xookee.cn), sections
 *    "压缩注意力机制解析 2.2-2.4" (mean-pool / MLP compression, softmax(QK^T/sqrt(d_k))V)
 *    and "滑动窗口注意力 2.4" / "加权融合不同注意力结果" (O = g_cmp O_cmp +
 *    g_sel O_sel + g_win O_win, g = sigmoid(MLP(x))).
 * Every formula on the first page was lost in extraction; the readings adopted
 * where the pages are silent are stated next to the code that applies them.
 *
 * Conventions: 0-based token index t; bf16 tensors are passed as uint16 bit
 * patterns; all arithmetic is fp64.  Layouts (row-major, contiguous):
 *   q [B,T,H,dk]  k [B,T,G,dk]  v [B,T,G,dv]  gates [B,T,H,3] (cmp, slc, win)
 *   kc [B,C,G,dk] vc [B,C,G,dv]  with C = floor((T-l)/d)+1 compressed blocks
 *   W_K [dk, l*dk], E_K [l, dk], W_V [dv, l*dv], E_V [l, dv]
 *   idx [B,T,G,n] int32 ascending, padded with -1
 * Rows are addressed by r = b*T + t.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t B, T, H, G, dk, dv;
    int64_t l, d, lp, n, fi, fl, w;
    int64_t phi;       /* 0 = mean-pool, 1 = linear map + position embedding */
    int64_t score_map; /* 0 = overlap-weighted, 1 = unweighted overlap sum */
    int64_t cmp_exact; /* 0 = K~/V~ rounded to bf16 (the operator); 1 = kept in fp64
                          (only for finite-difference gradient checks) */
    double scale;      /* softmax scale; <= 0 selects 1/sqrt(dk) */
} ocfg_t;

/* ------------------------------------------------------------------ bf16 */

double oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round an fp64 value to the nearest bf16, ties to even, in one step (no
 * intermediate rounding to fp32). */
uint16_t oracle_double_to_bf16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a) || isnan(a)) return (uint16_t)(sign | 0x7F80u | (isnan(a) ? 0x40u : 0u));
    int e;
    (void)frexp(a, &e);                /* a = m * 2^e with 0.5 <= m < 1 */
    int q = e - 8;                      /* bf16 keeps 8 significant bits */
    if (q < -133) q = -133;             /* subnormal quantum 2^-133 */
    double r = nearbyint(ldexp(a, -q)); /* default rounding mode: ties to even */
    double y = ldexp(r, q);
    if (y >= 3.3961775292304e38) return (uint16_t)(sign | 0x7F80u); /* overflow to inf */
    float f = (float)y; /* exact: y has at most 9 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

static inline double bf(uint16_t h) { return oracle_bf16_to_double(h); }

/* --------------------------------------------------------- config helpers */

static double cfg_scale(const ocfg_t* c)
{
    return c->scale > 0.0 ? c->scale : 1.0 / sqrt((double)c->dk);
}

/* number of compressed blocks over a sequence of length T */
int64_t oracle_num_cmp_blocks(const ocfg_t* c, int64_t T)
{
    return T >= c->l ? (T - c->l) / c->d + 1 : 0;
}

/* number of selection blocks over a sequence of length T */
int64_t oracle_num_sel_blocks(const ocfg_t* c, int64_t T)
{
    return (T + c->lp - 1) / c->lp;
}

/* Compressed block i covers tokens [i*d, i*d + l).  Reading: a block is
 * visible to query t once it is complete, i*d + l - 1 <= t (causality of the
 * compressed keys; token compression section). */
int64_t oracle_ncmp_visible(const ocfg_t* c, int64_t t)
{
    if (t + 1 < c->l) return 0;
    return (t + 1 - c->l) / c->d + 1;
}

/* Weight with which compressed block i feeds selection block j.  Block i is
 * made of the l/d stride-d segments i, i+1, ..., i+l/d-1; segment s lies in
 * selection block floor(s*d / l').  Reading of the "blockings differ" case of
 * the importance-score paragraph: the selection score sums the compressed
 * probabilities of the blocks that overlap j, each counted once per shared
 * segment (score_map 0), or once (score_map 1).  With l = l' = d this is the
 * identity, as the page states for equal blockings. */
static int64_t map_weight(const ocfg_t* c, int64_t i, int64_t j)
{
    int64_t cps = c->l / c->d, cnt = 0;
    for (int64_t u = 0; u < cps; ++u)
        if (((i + u) * c->d) / c->lp == j) cnt++;
    if (c->score_map == 1) return cnt > 0 ? 1 : 0;
    return cnt;
}

/* ------------------------------------------------------------ key lists */

/* compressed keys visible to t: 0 .. N_cmp(t)-1 */
static int64_t cmp_keys(const ocfg_t* c, int64_t t, int64_t* keys)
{
    int64_t nv = oracle_ncmp_visible(c, t);
    for (int64_t i = 0; i < nv; ++i) keys[i] = i;
    return nv;
}

/* tokens of the selected blocks, u <= t, ascending */
static int64_t sel_keys(const ocfg_t* c, int64_t t, const int32_t* idx_row, int64_t* keys)
{
    int64_t nk = 0;
    for (int64_t a = 0; a < c->n; ++a) {
        int32_t j = idx_row[a];
        if (j < 0) continue;
        for (int64_t u = (int64_t)j * c->lp; u < ((int64_t)j + 1) * c->lp; ++u)
            if (u <= t) keys[nk++] = u;
    }
    return nk;
}

/* window: the last w tokens up to and including t */
static int64_t win_keys(const ocfg_t* c, int64_t t, int64_t* keys)
{
    int64_t lo = t - c->w + 1;
    if (lo < 0) lo = 0;
    int64_t nk = 0;
    for (int64_t u = lo; u <= t; ++u) keys[nk++] = u;
    return nk;
}

/* --------------------------------------------------------------- phi */

/* Token compression (token compression section; mean-pool / MLP options of
 * the compressed-attention explainer).  Mean: average of the block's l rows.
 * Linear (reading of "learnable MLP with intra-block position encoding"): one
 * linear layer without bias or non-linearity applied to the position-major
 * flattening of (block rows + position embedding).  The result is rounded to
 * bf16 (the storage type of the compressed keys/values).  exact outputs are
 * optional (NULL to skip). */
void oracle_phi(const ocfg_t* c, const uint16_t* k, const uint16_t* v, const uint16_t* wk,
                const uint16_t* ek, const uint16_t* wv, const uint16_t* ev, uint16_t* kc,
                uint16_t* vc, double* kc_exact, double* vc_exact)
{
    const int64_t C = oracle_num_cmp_blocks(c, c->T);
    for (int pass = 0; pass < 2; ++pass) {
        const int64_t D = pass == 0 ? c->dk : c->dv;
        const uint16_t* X = pass == 0 ? k : v;
        const uint16_t* W = pass == 0 ? wk : wv;
        const uint16_t* E = pass == 0 ? ek : ev;
        uint16_t* Y = pass == 0 ? kc : vc;
        double* Yx = pass == 0 ? kc_exact : vc_exact;
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int64_t b = 0; b < c->B; ++b)
            for (int64_t i = 0; i < C; ++i) {
                double* x = (double*)malloc(sizeof(double) * (size_t)(c->l * D));
                for (int64_t g = 0; g < c->G; ++g) {
                    for (int64_t j = 0; j < c->l; ++j)
                        for (int64_t ch = 0; ch < D; ++ch) {
                            int64_t tok = i * c->d + j;
                            double val = bf(X[((b * c->T + tok) * c->G + g) * D + ch]);
                            if (c->phi == 1) val += bf(E[j * D + ch]);
                            x[j * D + ch] = val;
                        }
                    for (int64_t o = 0; o < D; ++o) {
                        double acc = 0.0;
                        if (c->phi == 0) {
                            for (int64_t j = 0; j < c->l; ++j) acc += x[j * D + o];
                            acc /= (double)c->l;
                        } else {
                            const uint16_t* wr = W + o * (c->l * D);
                            for (int64_t e = 0; e < c->l * D; ++e) acc += bf(wr[e]) * x[e];
                        }
                        int64_t off = ((b * C + i) * c->G + g) * D + o;
                        Y[off] = oracle_double_to_bf16(acc);
                        if (Yx) Yx[off] = acc;
                    }
                }
                free(x);
            }
    }
}

/* ------------------------------------------------------------- attention */

/* softmax(scale * q.K_u) over the key list, output sum_u p_u V_u.
 * Returns the natural-log LSE of the scaled logits (-inf when empty, with o = 0
 * and no probabilities). */
static double attend(int64_t dk, int64_t dv, double scale, const double* qv, const uint16_t* K,
                     const uint16_t* V, int64_t kstride, int64_t vstride, const int64_t* keys,
                     int64_t nk, double* p, double* o)
{
    for (int64_t ch = 0; ch < dv; ++ch) o[ch] = 0.0;
    if (nk == 0) return -INFINITY;
    double mx = -INFINITY;
    for (int64_t a = 0; a < nk; ++a) {
        const uint16_t* kr = K + keys[a] * kstride;
        double s = 0.0;
        for (int64_t ch = 0; ch < dk; ++ch) s += qv[ch] * bf(kr[ch]);
        p[a] = scale * s;
        if (p[a] > mx) mx = p[a];
    }
    double sum = 0.0;
    for (int64_t a = 0; a < nk; ++a) {
        p[a] = exp(p[a] - mx);
        sum += p[a];
    }
    for (int64_t a = 0; a < nk; ++a) {
        p[a] /= sum;
        const uint16_t* vr = V + keys[a] * vstride;
        for (int64_t ch = 0; ch < dv; ++ch) o[ch] += p[a] * bf(vr[ch]);
    }
    return mx + log(sum);
}

/* the same, over fp64 keys/values (the compressed branch) */
static double attend_d(int64_t dk, int64_t dv, double scale, const double* qv, const double* K,
                       const double* V, int64_t kstride, int64_t vstride, const int64_t* keys,
                       int64_t nk, double* p, double* o)
{
    for (int64_t ch = 0; ch < dv; ++ch) o[ch] = 0.0;
    if (nk == 0) return -INFINITY;
    double mx = -INFINITY;
    for (int64_t a = 0; a < nk; ++a) {
        const double* kr = K + keys[a] * kstride;
        double s = 0.0;
        for (int64_t ch = 0; ch < dk; ++ch) s += qv[ch] * kr[ch];
        p[a] = scale * s;
        if (p[a] > mx) mx = p[a];
    }
    double sum = 0.0;
    for (int64_t a = 0; a < nk; ++a) {
        p[a] = exp(p[a] - mx);
        sum += p[a];
    }
    for (int64_t a = 0; a < nk; ++a) {
        p[a] /= sum;
        const double* vr = V + keys[a] * vstride;
        for (int64_t ch = 0; ch < dv; ++ch) o[ch] += p[a] * vr[ch];
    }
    return mx + log(sum);
}

static void load_q(const ocfg_t* c, const uint16_t* q, int64_t r, int64_t h, double* qv)
{
    const uint16_t* qr = q + (r * c->H + h) * c->dk;
    for (int64_t ch = 0; ch < c->dk; ++ch) qv[ch] = bf(qr[ch]);
}

/* Top-n block selection (top-n paragraph; hyperparameter paragraph: 1 initial
 * and 2 local blocks always active).  Candidates are the blocks 0..b_t with
 * b_t = floor(t/l'); the local blocks are b_t and the ones before it.  When
 * there are at most n candidates all are taken.  Otherwise the forced blocks
 * are kept and the remaining n - fi - fl are the highest scores among the
 * other candidates, ties going to the lower block index.  Output ascending,
 * padded with -1. */
static void topn_row(const ocfg_t* c, int64_t t, const double* score, int32_t* out)
{
    int64_t bt = t / c->lp, ncand = bt + 1, m = 0;
    if (ncand <= c->n) {
        for (int64_t j = 0; j < ncand; ++j) out[m++] = (int32_t)j;
    } else {
        char* chosen = (char*)calloc((size_t)ncand, 1);
        for (int64_t j = 0; j < c->fi; ++j) chosen[j] = 1;
        for (int64_t j = bt - c->fl + 1; j <= bt; ++j) chosen[j] = 1;
        int64_t rest = c->n - c->fi - c->fl;
        for (int64_t it = 0; it < rest; ++it) {
            int64_t best = -1;
            for (int64_t j = 0; j < ncand; ++j) {
                if (chosen[j]) continue;
                if (best < 0 || score[j] > score[best]) best = j;
            }
            if (best < 0) break;
            chosen[best] = 1;
        }
        for (int64_t j = 0; j < ncand; ++j)
            if (chosen[j]) out[m++] = (int32_t)j;
        free(chosen);
    }
    for (; m < c->n; ++m) out[m] = -1;
}

void oracle_topn(const ocfg_t* c, int64_t nrows, const int64_t* rows, const double* pgrp,
                 int32_t* idx)
{
    const int64_t NS = oracle_num_sel_blocks(c, c->T);
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < nrows; ++a) {
        int64_t t = rows[a] % c->T;
        for (int64_t g = 0; g < c->G; ++g)
            topn_row(c, t, pgrp + (a * c->G + g) * NS, idx + (a * c->G + g) * c->n);
    }
}

/* Per-row forward.  kc/vc are the compressed keys/values [B,C,G,*] the caller
 * provides (normally from oracle_phi).  idx_in, when non-NULL, replaces the
 * oracle's own selection for these rows ([nrows,G,n]); idx_out receives the
 * selection used.  Optional outputs may be NULL:
 *   lse [nrows,H,3], pgrp [nrows,G,Nsel], pcmp [nrows,H,C], obr [nrows,H,3,dv].
 * out [nrows,H,dv] = g_cmp o_cmp + g_slc o_slc + g_win o_win (final output
 * computation paragraph; gated-fusion section of the explainer). */
static void forward_rows_impl(const ocfg_t* c, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const uint16_t* kw, const uint16_t* vw,
                              const float* gates, int64_t qrow0,
                              const double* kc, const double* vc, int64_t nrows,
                              const int64_t* rows, const int32_t* idx_in, double* out,
                              int32_t* idx_out, double* lse, double* pgrp, double* pcmp,
                              double* obr)
{
    const int64_t C = oracle_num_cmp_blocks(c, c->T);
    const int64_t NS = oracle_num_sel_blocks(c, c->T);
    const int64_t Hg = c->H / c->G;
    const double sc = cfg_scale(c);
#pragma omp parallel for schedule(dynamic)
    for (int64_t a = 0; a < nrows; ++a) {
        const int64_t r = rows[a], b = r / c->T, t = r % c->T;
        int64_t maxk = C + c->T + 1;
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)maxk);
        double* p = (double*)malloc(sizeof(double) * (size_t)maxk);
        double* qv = (double*)malloc(sizeof(double) * (size_t)c->dk);
        double* ob = (double*)malloc(sizeof(double) * (size_t)(3 * c->dv));
        double* ps = (double*)malloc(sizeof(double) * (size_t)NS);
        int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)c->n);
        for (int64_t g = 0; g < c->G; ++g) {
            /* 1. compressed attention for every head of the group, and the
             * group's selection-block importance scores */
            for (int64_t j = 0; j < NS; ++j) ps[j] = 0.0;
            double* ocmp = (double*)malloc(sizeof(double) * (size_t)(Hg * c->dv));
            for (int64_t hh = 0; hh < Hg; ++hh) {
                int64_t h = g * Hg + hh;
                load_q(c, q, r - qrow0, h, qv);
                int64_t nk = cmp_keys(c, t, keys);
                const double* K = kc + (b * C * c->G + g) * c->dk;
                const double* V = vc + (b * C * c->G + g) * c->dv;
                double l0 = attend_d(c->dk, c->dv, sc, qv, K, V, c->G * c->dk, c->G * c->dv, keys,
                                   nk, p, ocmp + hh * c->dv);
                if (lse) lse[(a * c->H + h) * 3 + 0] = l0;
                if (pcmp) {
                    for (int64_t i = 0; i < C; ++i) pcmp[(a * c->H + h) * C + i] = 0.0;
                    for (int64_t i = 0; i < nk; ++i) pcmp[(a * c->H + h) * C + i] = p[i];
                }
                /* importance scores: map compressed probabilities to selection
                 * blocks, then sum over the heads of the group (shared-score
                 * paragraph for GQA/MQA) */
                for (int64_t i = 0; i < nk; ++i) {
                    int64_t jlo = (i * c->d) / c->lp;
                    int64_t jhi = ((i + c->l / c->d - 1) * c->d) / c->lp;
                    for (int64_t j = jlo; j <= jhi && j < NS; ++j)
                        ps[j] += (double)map_weight(c, i, j) * p[i];
                }
            }
            if (pgrp)
                for (int64_t j = 0; j < NS; ++j) pgrp[(a * c->G + g) * NS + j] = ps[j];
            /* 2. selection */
            if (idx_in)
                memcpy(sel, idx_in + (a * c->G + g) * c->n, sizeof(int32_t) * (size_t)c->n);
            else
                topn_row(c, t, ps, sel);
            if (idx_out) memcpy(idx_out + (a * c->G + g) * c->n, sel, sizeof(int32_t) * (size_t)c->n);
            /* 3. selected and window branches, 4. gated merge */
            for (int64_t hh = 0; hh < Hg; ++hh) {
                int64_t h = g * Hg + hh;
                load_q(c, q, r - qrow0, h, qv);
                const uint16_t* K = k + (b * c->T * c->G + g) * c->dk;
                const uint16_t* V = v + (b * c->T * c->G + g) * c->dv;
                for (int64_t ch = 0; ch < c->dv; ++ch) ob[ch] = ocmp[hh * c->dv + ch];
                int64_t nk = sel_keys(c, t, sel, keys);
                double l1 = attend(c->dk, c->dv, sc, qv, K, V, c->G * c->dk, c->G * c->dv, keys, nk,
                                   p, ob + c->dv);
                nk = win_keys(c, t, keys);
                const uint16_t* KW = kw + (b * c->T * c->G + g) * c->dk;
                const uint16_t* VW = vw + (b * c->T * c->G + g) * c->dv;
                double l2 = attend(c->dk, c->dv, sc, qv, KW, VW, c->G * c->dk, c->G * c->dv, keys, nk,
                                   p, ob + 2 * c->dv);
                if (lse) {
                    lse[(a * c->H + h) * 3 + 1] = l1;
                    lse[(a * c->H + h) * 3 + 2] = l2;
                }
                const float* gr = gates + ((r - qrow0) * c->H + h) * 3;
                for (int64_t ch = 0; ch < c->dv; ++ch)
                    out[(a * c->H + h) * c->dv + ch] = (double)gr[0] * ob[ch] +
                                                       (double)gr[1] * ob[c->dv + ch] +
                                                       (double)gr[2] * ob[2 * c->dv + ch];
                if (obr)
                    for (int64_t br = 0; br < 3; ++br)
                        for (int64_t ch = 0; ch < c->dv; ++ch)
                            obr[((a * c->H + h) * 3 + br) * c->dv + ch] = ob[br * c->dv + ch];
            }
            free(ocmp);
        }
        free(keys);
        free(p);
        free(qv);
        free(ob);
        free(ps);
        free(sel);
    }
}

void oracle_forward_rows(const ocfg_t* c, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const float* gates, const double* kc, const double* vc,
                         int64_t nrows, const int64_t* rows, const int32_t* idx_in, double* out,
                         int32_t* idx_out, double* lse, double* pgrp, double* pcmp, double* obr)
{
    forward_rows_impl(c, q, k, v, k, v, gates, 0, kc, vc, nrows, rows, idx_in, out, idx_out, lse, pgrp,
                      pcmp, obr);
}

/* The same rows with independent keys/values per branch (page 2, sliding-window
 * paragraph: the branches keep separate keys and values so that the window
 * branch's local patterns do not shortcut the other two): the compressed
 * branch reads kc/vc (phi of its own k/v, computed by the caller), the
 * selected branch k/v, the window branch kw/vw ([B,T,G,*] bf16 each).  The
 * selection still comes from the compressed branch's probabilities. */
void oracle_forward_rows_branches(const ocfg_t* c, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const uint16_t* kw, const uint16_t* vw,
                                  const float* gates, const double* kc, const double* vc, int64_t nrows,
                                  const int64_t* rows, const int32_t* idx_in, double* out,
                                  int32_t* idx_out, double* lse, double* pgrp, double* pcmp, double* obr)
{
    forward_rows_impl(c, q, k, v, kw, vw, gates, 0, kc, vc, nrows, rows, idx_in, out, idx_out, lse, pgrp,
                      pcmp, obr);
}

/* Number of keys each branch reads for query t (compressed, selected,
 * window), built by the same key-list code the attention uses.  The selected
 * count does not depend on which blocks win, so any scores do. */
void oracle_key_counts(const ocfg_t* c, int64_t t, int64_t* out3)
{
    const int64_t NS = oracle_num_sel_blocks(c, t + 1);
    double* sc = (double*)calloc((size_t)(NS + 1), sizeof(double));
    for (int64_t j = 0; j < NS; ++j) sc[j] = (double)((j * 7919) % 1000); /* arbitrary */
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)c->n);
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(t + 2 + oracle_num_cmp_blocks(c, t + 1)));
    topn_row(c, t, sc, sel);
    out3[0] = cmp_keys(c, t, keys);
    out3[1] = sel_keys(c, t, sel, keys);
    out3[2] = win_keys(c, t, keys);
    free(sc);
    free(sel);
    free(keys);
}

/* ---------------------------------------------------------------- decode */

/* Decode (efficiency-analysis paragraph on decoding): one query per sequence
 * at position t = L-1 over caches that already hold the current token.
 * Sequence s owns k/v cache rows [kv_off[s], kv_off[s+1]) ([*,G,dk]/[*,G,dv])
 * and compressed rows [cmp_off[s], cmp_off[s+1]) which must number
 * N_cmp(L-1).  Returns 0, or -1 when a compressed-cache length is wrong. */
int oracle_decode(const ocfg_t* c0, int64_t S, const uint16_t* q, const uint16_t* kcache,
                  const uint16_t* vcache, const int64_t* kv_off, const uint16_t* kccache,
                  const uint16_t* vccache, const int64_t* cmp_off, const float* gates,
                  double* out, int32_t* idx, double* lse, double* pgrp_out, int64_t ns_stride)
{
    int bad = 0;
    for (int64_t s = 0; s < S; ++s) {
        ocfg_t c = *c0;
        c.B = 1;
        c.T = kv_off[s + 1] - kv_off[s];
        int64_t t = c.T - 1;
        if (cmp_off[s + 1] - cmp_off[s] != oracle_ncmp_visible(&c, t)) {
            bad = 1;
            continue;
        }
        /* the rows function sizes compressed arrays by C(T); at t = T-1 this
         * equals N_cmp(T-1), the cache length */
        int64_t row = t;
        double* pg = NULL;
        const int64_t NS = oracle_num_sel_blocks(&c, c.T);
        if (pgrp_out) pg = (double*)malloc(sizeof(double) * (size_t)(c.G * NS));
        /* q and gates hold one row per sequence: row t of this call is
         * sequence s's row */
        int64_t nc = cmp_off[s + 1] - cmp_off[s];
        double* kcd = (double*)malloc(sizeof(double) * (size_t)((nc > 0 ? nc : 1) * c.G * c.dk));
        double* vcd = (double*)malloc(sizeof(double) * (size_t)((nc > 0 ? nc : 1) * c.G * c.dv));
        for (int64_t e = 0; e < nc * c.G * c.dk; ++e) kcd[e] = bf(kccache[cmp_off[s] * c.G * c.dk + e]);
        for (int64_t e = 0; e < nc * c.G * c.dv; ++e) vcd[e] = bf(vccache[cmp_off[s] * c.G * c.dv + e]);
        forward_rows_impl(&c, q + s * c.H * c.dk, kcache + kv_off[s] * c.G * c.dk,
                          vcache + kv_off[s] * c.G * c.dv, kcache + kv_off[s] * c.G * c.dk,
                          vcache + kv_off[s] * c.G * c.dv, gates + s * c.H * 3, t, kcd, vcd, 1,
                          &row, NULL, out + s * c.H * c.dv, idx + s * c.G * c.n,
                          lse ? lse + s * c.H * 3 : NULL, pg, NULL, NULL);
        free(kcd);
        free(vcd);
        if (pgrp_out) {
            /* pgrp_out is [S,G,ns_stride]; this sequence's Nsel blocks go at the
             * front of each group's slot, the rest is zero */
            for (int64_t g = 0; g < c.G; ++g) {
                double* dst = pgrp_out + (s * c.G + g) * ns_stride;
                for (int64_t j = 0; j < ns_stride; ++j) dst[j] = j < NS ? pg[g * NS + j] : 0.0;
            }
            free(pg);
        }
    }
    return bad ? -1 : 0;
}

/* -------------------------------------------------------------- backward */

/* Backward of the operator with the selection held fixed (the selection is a
 * discrete choice; no gradient flows through the importance scores).  Per
 * branch c with dO_c = g_c dO: softmax backward
 *   dP_u = <dO_c, V_u>, D = <dO_c, o_c>, dS_u = P_u (dP_u - D),
 *   dq += scale sum_u dS_u K_u, dK_u += scale dS_u q, dV_u += P_u dO_c,
 * d(gate_c) = <dO, o_c> (the gate values as passed, i.e. after the sigmoid).
 * The compressed branch's dK~/dV~ go back through phi: mean spreads dK~/l to
 * every member token; linear gives d x = W^T dK~ for the flattened block,
 * scattered onto the overlapping blocks' tokens.  The bf16 rounding of K~/V~
 * is treated as the identity in the backward (it is a storage format).
 * With cfg->cmp_exact the forward statistics use the unrounded K~/V~ too.
 *
 * Rows t >= t_lo only.  Every contribution to the key/value gradient of a
 * token u comes from rows t >= u (a compressed block becomes visible only once
 * complete), so dk/dv are exact for tokens u >= t_lo and dq/dgates for rows
 * t >= t_lo; entries below t_lo hold partial sums.  t_lo = 0 is the full
 * backward.  Outputs (fp64, zeroed here): dq [B,T,H,dk], dk [B,T,G,dk],
 * dv [B,T,G,dv], dgates [B,T,H,3].  idx [B,T,G,n]. */
static void backward_core(const ocfg_t* c, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const float* gates, const uint16_t* wk,
                          const uint16_t* ek, const uint16_t* wv, const uint16_t* ev,
                          const uint16_t* dout, const int32_t* idx, int64_t t_lo,
                          const uint8_t* row_on, double* dq, double* dk, double* dv,
                          double* dgates, double* dkc_out, double* dvc_out)
{
    const int64_t B = c->B, T = c->T, H = c->H, G = c->G, dK = c->dk, dV = c->dv;
    const int64_t C = oracle_num_cmp_blocks(c, T);
    const int64_t Hg = H / G;
    const double sc = cfg_scale(c);
    memset(dq, 0, sizeof(double) * (size_t)(B * T * H * dK));
    memset(dk, 0, sizeof(double) * (size_t)(B * T * G * dK));
    memset(dv, 0, sizeof(double) * (size_t)(B * T * G * dV));
    memset(dgates, 0, sizeof(double) * (size_t)(B * T * H * 3));
    const size_t nkc = (size_t)(B * (C > 0 ? C : 1) * G * dK), nvc = (size_t)(B * (C > 0 ? C : 1) * G * dV);
    uint16_t* kcb = (uint16_t*)malloc(sizeof(uint16_t) * nkc);
    uint16_t* vcb = (uint16_t*)malloc(sizeof(uint16_t) * nvc);
    double* kc = (double*)calloc(nkc, sizeof(double));
    double* vc = (double*)calloc(nvc, sizeof(double));
    if (C > 0) oracle_phi(c, k, v, wk, ek, wv, ev, kcb, vcb, kc, vc);
    if (!c->cmp_exact) {
        for (size_t e = 0; e < nkc; ++e) kc[e] = C > 0 ? bf(kcb[e]) : 0.0;
        for (size_t e = 0; e < nvc; ++e) vc[e] = C > 0 ? bf(vcb[e]) : 0.0;
    }
    free(kcb);
    free(vcb);
    double* dkc = (double*)calloc((size_t)(B * (C > 0 ? C : 1) * G * dK), sizeof(double));
    double* dvc = (double*)calloc((size_t)(B * (C > 0 ? C : 1) * G * dV), sizeof(double));

#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t g = 0; g < G; ++g) {
            int64_t maxk = C + T + 1;
            int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)maxk);
            double* p = (double*)malloc(sizeof(double) * (size_t)maxk);
            double* qv = (double*)malloc(sizeof(double) * (size_t)dK);
            double* o = (double*)malloc(sizeof(double) * (size_t)dV);
            double* dO = (double*)malloc(sizeof(double) * (size_t)dV);
            for (int64_t t = (t_lo > 0 ? t_lo : 0); t < T; ++t) {
                const int64_t r = b * T + t;
                if (row_on && !row_on[r]) continue;
                for (int64_t hh = 0; hh < Hg; ++hh) {
                    const int64_t h = g * Hg + hh;
                    load_q(c, q, r, h, qv);
                    for (int64_t ch = 0; ch < dV; ++ch) dO[ch] = bf(dout[(r * H + h) * dV + ch]);
                    const float* gr = gates + (r * H + h) * 3;
                    for (int br = 0; br < 3; ++br) {
                        const uint16_t *Kb = NULL, *Vb = NULL;
                        const double *Kd = NULL, *Vd = NULL;
                        double *dKb, *dVb;
                        int64_t nk;
                        if (br == 0) {
                            nk = cmp_keys(c, t, keys);
                            Kd = kc + (b * C * G + g) * dK;
                            Vd = vc + (b * C * G + g) * dV;
                            dKb = dkc + (b * C * G + g) * dK;
                            dVb = dvc + (b * C * G + g) * dV;
                            attend_d(dK, dV, sc, qv, Kd, Vd, G * dK, G * dV, keys, nk, p, o);
                        } else {
                            nk = br == 1 ? sel_keys(c, t, idx + (r * G + g) * c->n, keys)
                                         : win_keys(c, t, keys);
                            Kb = k + (b * T * G + g) * dK;
                            Vb = v + (b * T * G + g) * dV;
                            dKb = dk + (b * T * G + g) * dK;
                            dVb = dv + (b * T * G + g) * dV;
                            attend(dK, dV, sc, qv, Kb, Vb, G * dK, G * dV, keys, nk, p, o);
                        }
                        double dgate = 0.0;
                        for (int64_t ch = 0; ch < dV; ++ch) dgate += dO[ch] * o[ch];
                        dgates[(r * H + h) * 3 + br] = dgate;
                        const double gc = (double)gr[br];
                        const double Dc = gc * dgate;
                        for (int64_t a = 0; a < nk; ++a) {
                            double dP = 0.0;
                            for (int64_t ch = 0; ch < dV; ++ch)
                                dP += gc * dO[ch] * (Vd ? Vd[keys[a] * G * dV + ch]
                                                        : bf(Vb[keys[a] * G * dV + ch]));
                            double dS = p[a] * (dP - Dc);
                            double* dqr = dq + (r * H + h) * dK;
                            for (int64_t ch = 0; ch < dK; ++ch)
                                dqr[ch] += sc * dS * (Kd ? Kd[keys[a] * G * dK + ch]
                                                         : bf(Kb[keys[a] * G * dK + ch]));
                            double* dkr = dKb + keys[a] * G * dK;
                            for (int64_t ch = 0; ch < dK; ++ch) dkr[ch] += sc * dS * qv[ch];
                            double* dvr = dVb + keys[a] * G * dV;
                            for (int64_t ch = 0; ch < dV; ++ch) dvr[ch] += p[a] * gc * dO[ch];
                        }
                    }
                }
            }
            free(keys);
            free(p);
            free(qv);
            free(o);
            free(dO);
        }

    /* phi transposed: compressed-key gradients back onto the tokens */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t g = 0; g < G; ++g)
            for (int pass = 0; pass < 2; ++pass) {
                const int64_t D = pass == 0 ? dK : dV;
                const double* dY = pass == 0 ? dkc : dvc;
                const uint16_t* W = pass == 0 ? wk : wv;
                double* dX = pass == 0 ? dk : dv;
                for (int64_t i = 0; i < C; ++i) {
                    const double* dy = dY + ((b * C + i) * G + g) * D;
                    for (int64_t j = 0; j < c->l; ++j) {
                        double* dx = dX + ((b * T + i * c->d + j) * G + g) * D;
                        for (int64_t ch = 0; ch < D; ++ch) {
                            double acc = 0.0;
                            if (c->phi == 0) {
                                acc = dy[ch] / (double)c->l;
                            } else {
                                for (int64_t o2 = 0; o2 < D; ++o2)
                                    acc += bf(W[o2 * (c->l * D) + j * D + ch]) * dy[o2];
                            }
                            dx[ch] += acc;
                        }
                    }
                }
            }
    if (dkc_out && C > 0) memcpy(dkc_out, dkc, sizeof(double) * (size_t)(B * C * G * dK));
    if (dvc_out && C > 0) memcpy(dvc_out, dvc, sizeof(double) * (size_t)(B * C * G * dV));
    free(kc);
    free(vc);
    free(dkc);
    free(dvc);
}

void oracle_backward_tail(const ocfg_t* c, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const float* gates, const uint16_t* wk,
                          const uint16_t* ek, const uint16_t* wv, const uint16_t* ev,
                          const uint16_t* dout, const int32_t* idx, int64_t t_lo, double* dq,
                          double* dk, double* dv, double* dgates, double* dkc_out, double* dvc_out)
{
    backward_core(c, q, k, v, gates, wk, ek, wv, ev, dout, idx, t_lo, NULL, dq, dk, dv, dgates,
                  dkc_out, dvc_out);
}

/* The same backward restricted to the query rows r = b*T + t listed in
 * rows[0 .. nrows): the gradient of sum over the listed rows of <dout, out>,
 * i.e. every row outside the list contributes nothing (as if its dout were
 * zero).  dq/dgates are those of the listed rows (zero elsewhere); dk, dv and
 * the compressed-key gradients sum the listed rows' contributions over every
 * key they read, at any position.  Outputs as oracle_backward_tail. */
void oracle_backward_rows(const ocfg_t* c, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const float* gates, const uint16_t* wk,
                          const uint16_t* ek, const uint16_t* wv, const uint16_t* ev,
                          const uint16_t* dout, const int32_t* idx, int64_t nrows,
                          const int64_t* rows, double* dq, double* dk, double* dv,
                          double* dgates, double* dkc_out, double* dvc_out)
{
    uint8_t* on = (uint8_t*)calloc((size_t)(c->B * c->T), 1);
    for (int64_t a = 0; a < nrows; ++a)
        if (rows[a] >= 0 && rows[a] < c->B * c->T) on[rows[a]] = 1;
    backward_core(c, q, k, v, gates, wk, ek, wv, ev, dout, idx, 0, on, dq, dk, dv, dgates,
                  dkc_out, dvc_out);
    free(on);
}

/* Gradients of the linear phi's parameters (token compression: K~[i] =
 * W vec(k_blk + E), vec position-major) from the compressed-key gradients
 * dY = dK~ [B,C,G,D] of the backward above:
 *   dW[o, x]  = sum over (b, i, g) of dY[b,i,g,o] * X[b,i,g,x],  X = vec(k_blk + E)
 *   dE[j, ch] = sum over (b, i, g) and o of W[o, j*D + ch] * dY[b,i,g,o]
 * (the bf16 rounding of K~ treated as the identity, as above).  One call per
 * tensor: x = k with W_K, E_K (D = d_k) or v with W_V, E_V (D = d_v).
 * Outputs fp64, zeroed here: dW [D, l*D], dE [l, D]. */
void oracle_phi_param_grads(const ocfg_t* c, int64_t D, const uint16_t* x, const uint16_t* W,
                            const uint16_t* E, const double* dY, double* dW, double* dE)
{
    const int64_t B = c->B, T = c->T, G = c->G, l = c->l, K = c->l * D;
    const int64_t C = oracle_num_cmp_blocks(c, T);
    memset(dW, 0, sizeof(double) * (size_t)(D * K));
    memset(dE, 0, sizeof(double) * (size_t)K);
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < D; ++o)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t i = 0; i < C; ++i)
                for (int64_t g = 0; g < G; ++g) {
                    const double dy = dY[((b * C + i) * G + g) * D + o];
                    for (int64_t j = 0; j < l; ++j)
                        for (int64_t ch = 0; ch < D; ++ch)
                            dW[o * K + j * D + ch] +=
                                dy * (bf(x[((b * T + i * c->d + j) * G + g) * D + ch]) + bf(E[j * D + ch]));
                }
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < K; ++e) {
        double acc = 0.0;
        for (int64_t b = 0; b < B; ++b)
            for (int64_t i = 0; i < C; ++i)
                for (int64_t g = 0; g < G; ++g)
                    for (int64_t o = 0; o < D; ++o)
                        acc += bf(W[o * K + e]) * dY[((b * C + i) * G + g) * D + o];
        dE[e] = acc;
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
