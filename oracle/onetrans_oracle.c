/*
 * OneTrans block-stack forward: plain CPU fp64 ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path never calls it and shares no code with it.
 *
 * What it computes (OneTrans, "OneTrans: Unified Feature Interaction and
 * Sequence Modeling with One Transformer in Industrial Recommender", summary
 * page, block / pyramid / KV-cache paragraphs; blog page, "Mixed
 * Parameterization" and "Cross-Request KV Caching" designs):
 *
 *   tokens   : S-tokens (behaviour rows) first, then N NS-tokens per candidate.
 *   block    : pre-norm RMSNorm -> attention -> residual -> RMSNorm -> FFN
 *              (GELU) -> residual.  All S-tokens share one QKV/O/FFN set and
 *              one gain vector; NS position n has its own private set.
 *   mask     : S-token t sees S-tokens 0..t; NS-token n sees every S-token of
 *              the layer and NS-tokens 0..n of its own candidate.
 *   pyramid  : layer l takes L_l S rows, computes K/V for all of them and
 *              queries only for the tail q_l rows; the next layer's S input is
 *              that tail (L_{l+1} = q_l), in order.
 *   KV cache : S never attends to NS, so the S-side K/V of every layer are a
 *              per-user quantity; candidates are scored against them.
 *   sparse MoE (cfg->moe_experts = E > 0; the OneTrans-V2 summary page names
 *              a sparse mixture of experts for capacity, without a recipe):
 *              the shared S-side FFN of every block becomes E expert FFNs of
 *              the same shape.  With z = n(h; g2) the FFN's normalised input,
 *              a linear router gives logits W_r z; the top-k logits (ties to
 *              the lower expert index) are softmax-ed into gates g_j, and
 *              y = h + sum_j g_j W2_e(j) GELU(W1_e(j) z).  NS tokens keep
 *              their private dense FFNs.
 *   full attention (cfg->full_attn = 1; summary page, limitations paragraph:
 *              full attention matches causal attention offline, causal wins
 *              only through the KV cache): every token sees every token of
 *              its own candidate's sequence, S and NS alike.  S then depends
 *              on the candidate, so only the joint formulation runs it.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   RMSNorm n(x; g) = x * (mean(x^2) + eps)^(-1/2) * g, eps from the config;
 *   no biases; attention scale 1/sqrt(head_dim); exact-erf GELU; no
 *   positional encoding; no final norm; heads concatenated along d.
 *
 * Storage: every input is passed as float32, which holds the bf16 / fp32
 * values of the runs exactly; all arithmetic is fp64 (double).
 *
 * FP8 modes (the V2 podcast page credits kernel fusion and FP8 and says no
 * more; the workload fixes e4m3 with per-tensor fp32 scales):
 *   fp8 = 2 (per-tensor): every projection input tensor -- the input of the
 *     QKV, O, W1 or W2 projection of one layer and one parameter set (S, or
 *     NS position n) -- has one fixed fp32 scale s from cfg->act_scale; each
 *     value is quantised as e4m3(x / s), round to nearest even, saturating
 *     at +-448.  A calibrated scale does not depend on the batch, so a
 *     candidate's result stays independent of the other candidates.
 *   fp8 = 1 (per-row, the calibration pass): every input row gets its own
 *     scale s = amax(row)/448 (s = 1 for an all-zero row).
 *   In both modes every weight matrix is quantised with one scale
 *   amax(W)/448, the product is computed in fp64 on the quantised values and
 *   multiplied by both scales, and attention stays unquantised.
 *   cfg->act_amax, if not NULL, receives max |x| over every row that entered
 *   each projection input tensor (max-accumulated): the per-tensor amax a
 *   calibration turns into scales amax/448.
 *   Layout of act_scale / act_amax: [layer][set][4], set 0 = S, 1 + n = NS
 *   position n; the 4 inputs in the order QKV, O, W1, W2.
 *
 * Layouts (row-major):
 *   Wqkv [3d][d] (rows Q | K | V), Wo [d][d], W1 [ffn][d], W2 [d][ffn],
 *   S-side weights indexed [layer], NS-side [layer][n].
 *   KV cache per user: for layer l, K [L_l][d] then V [L_l][d]; layers packed
 *   in order, so layer l starts at 2*d*sum_{j<l} L_j.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_MAX_LAYERS 64

typedef struct {
    int layers, d, heads, ffn, n_ns, L0;
    int q[ORC_MAX_LAYERS]; /* query tail per layer; L_{l+1} = q[l] */
    double eps;
    int fp8;                  /* 0 off, 1 per-row scales, 2 per-tensor scales */
    const double *act_scale;  /* fp8 == 2: [layers][1 + n_ns][4] */
    double *act_amax;         /* optional, same layout: max |input| seen */
    int full_attn;            /* 1: full (non-causal) attention, joint form only */
    int moe_experts;          /* E > 0: the S-side FFN is a sparse mixture of E experts */
    int moe_topk;             /* experts per S row (1 or 2) */
} orc_cfg;

enum { ORC_IN_QKV = 0, ORC_IN_O = 1, ORC_IN_W1 = 2, ORC_IN_W2 = 3 };

typedef struct {
    const float *Wqkv_s, *Wo_s, *W1_s, *W2_s, *g1_s, *g2_s;
    const float *Wqkv_ns, *Wo_ns, *W1_ns, *W2_ns, *g1_ns, *g2_ns;
    const float *W_router; /* [layers][E][d] (moe_experts > 0) */
    const float *W1_moe;   /* [layers][E][ffn][d] */
    const float *W2_moe;   /* [layers][E][d][ffn] */
} orc_weights;

/* ------------------------------------------------------------------------- */
/* e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinity,  */
/* largest finite 448, subnormal quantum 2^-9): round to nearest, ties to     */
/* even, saturating.  Written from the format's definition.                   */
static double e4m3_round(double v)
{
    double a = fabs(v);
    if (a >= 448.0) return copysign(448.0, v);
    if (a == 0.0) return v;
    int e;
    frexp(a, &e);           /* a = m * 2^e, m in [0.5, 1) */
    int E = e - 1;          /* a in [2^E, 2^(E+1)) */
    if (E < -6) E = -6;     /* below the normal range the quantum stays 2^-9 */
    double quantum = ldexp(1.0, E - 3);
    double r = nearbyint(a / quantum) * quantum; /* ties to even */
    return copysign(r, v);
}

double orc_e4m3_round(double v) { return e4m3_round(v); }

/* Quantise n values with one per-block scale; returns the scale. */
static double quantise_block(const double *x, long n, double *xq)
{
    double amax = 0.0;
    for (long i = 0; i < n; ++i) if (fabs(x[i]) > amax) amax = fabs(x[i]);
    double s = amax > 0.0 ? amax / 448.0 : 1.0;
    for (long i = 0; i < n; ++i) xq[i] = e4m3_round(x[i] / s);
    return s;
}

/* A weight matrix as the projections read it: plain, or quantised + scale,
 * with the quantisation rule of its input tensor. */
typedef struct {
    const float *w; /* [out][in] */
    double *wq;     /* quantised copy (fp8 mode) */
    double s;
    int out, in;
    int fp8;        /* input rule: 0 none, 1 per-row scale, 2 per-tensor scale xs */
    double xs;      /* per-tensor input scale (fp8 == 2) */
    double *amax;   /* if not NULL: max |input| of this tensor, accumulated */
} mat_t;

static mat_t mat_plain(const float *w, int out, int in)
{
    mat_t m = {w, NULL, 1.0, out, in, 0, 1.0, NULL};
    return m;
}

static mat_t mat_make(const float *w, int out, int in, int fp8)
{
    mat_t m = mat_plain(w, out, in);
    m.fp8 = fp8;
    if (fp8) {
        long n = (long)out * in;
        double *tmp = (double *)malloc(sizeof(double) * n);
        m.wq = (double *)malloc(sizeof(double) * n);
        for (long i = 0; i < n; ++i) tmp[i] = w[i];
        m.s = quantise_block(tmp, n, m.wq);
        free(tmp);
    }
    return m;
}

static void mat_free(mat_t *m) { free(m->wq); m->wq = NULL; }

/* Record max |x| of one input row into the tensor's amax slot. */
static void record_amax(const mat_t *m, const double *x)
{
    if (!m->amax) return;
    double a = 0.0;
    for (int k = 0; k < m->in; ++k) if (fabs(x[k]) > a) a = fabs(x[k]);
#pragma omp critical(orc_amax)
    {
        if (a > *m->amax) *m->amax = a;
    }
}

/* Quantise one input row by the matrix's input rule; returns its scale. */
static double quantise_input(const mat_t *m, const double *x, double *xq)
{
    if (m->fp8 == 1) return quantise_block(x, m->in, xq);
    for (int k = 0; k < m->in; ++k) xq[k] = e4m3_round(x[k] / m->xs);
    return m->xs;
}

/* y[o] = sum_k W[o][k] x[k] for o in [o0, o0+nout).  In fp8 mode the input
 * row x (the whole projection input, all `in` values) is quantised first,
 * with its own scale (per-row) or the tensor's (per-tensor).  xq is scratch
 * of `in` doubles. */
static void project(const mat_t *m, const double *x, int o0, int nout, double *y, double *xq)
{
    int in = m->in;
    record_amax(m, x);
    if (!m->wq) {
        for (int o = 0; o < nout; ++o) {
            const float *row = m->w + (long)(o0 + o) * in;
            double acc = 0.0;
            for (int k = 0; k < in; ++k) acc += (double)row[k] * x[k];
            y[o] = acc;
        }
        return;
    }
    double sx = quantise_input(m, x, xq);
    for (int o = 0; o < nout; ++o) {
        const double *row = m->wq + (long)(o0 + o) * in;
        double acc = 0.0;
        for (int k = 0; k < in; ++k) acc += row[k] * xq[k];
        y[o] = acc * sx * m->s;
    }
}

/* RMSNorm: y = x * (mean(x^2) + eps)^(-1/2) * g */
static void rmsnorm(const double *x, const float *g, int d, double eps, double *y)
{
    double ss = 0.0;
    for (int k = 0; k < d; ++k) ss += x[k] * x[k];
    double r = 1.0 / sqrt(ss / d + eps);
    for (int k = 0; k < d; ++k) y[k] = x[k] * r * (double)g[k];
}

static double gelu(double z) { return 0.5 * z * (1.0 + erf(z / sqrt(2.0))); }

/* softmax(q.k_j / sqrt(hd)) over the given key rows, then sum p_j v_j.
 * Keys come from up to two row sets (S rows then NS rows), each [rows][d],
 * read at column offset h*hd. */
static void attend(const double *q, int hd, int coff, int d,
                   const double *K1, const double *V1, int n1,
                   const double *K2, const double *V2, int n2,
                   double *out, double *sc)
{
    double scale = 1.0 / sqrt((double)hd);
    double mx = -INFINITY;
    for (int j = 0; j < n1 + n2; ++j) {
        const double *k = j < n1 ? K1 + (long)j * d : K2 + (long)(j - n1) * d;
        double s = 0.0;
        for (int e = 0; e < hd; ++e) s += q[e] * k[coff + e];
        s *= scale;
        sc[j] = s;
        if (s > mx) mx = s;
    }
    double sum = 0.0;
    for (int j = 0; j < n1 + n2; ++j) { sc[j] = exp(sc[j] - mx); sum += sc[j]; }
    for (int e = 0; e < hd; ++e) out[e] = 0.0;
    for (int j = 0; j < n1 + n2; ++j) {
        const double *v = j < n1 ? V1 + (long)j * d : V2 + (long)(j - n1) * d;
        double p = sc[j] / sum;
        for (int e = 0; e < hd; ++e) out[e] += p * v[coff + e];
    }
}

/* Everything one block needs for one parameter set (S shared or NS position n). */
typedef struct {
    mat_t qkv, o, w1, w2;
    const float *g1, *g2;
    int moe_E, moe_k;        /* S set with a mixture of experts: E, top-k */
    const float *router;     /* [E][d] */
    mat_t *ew1, *ew2;        /* [E] expert W1 [ffn][d], W2 [d][ffn] */
} pset_t;

/* Attach the input rule of tensor (layer l, set, input t) to a matrix. */
static void mat_input(const orc_cfg *c, mat_t *m, int l, int set, int t)
{
    long slot = ((long)l * (1 + c->n_ns) + set) * 4 + t;
    if (c->fp8 == 2) m->xs = c->act_scale[slot];
    if (c->act_amax) m->amax = c->act_amax + slot;
}

/* Parameter set `set` (0 = S, 1 + n = NS position n) of layer l. */
static pset_t pset_make(const orc_cfg *c, int l, int set, const float *Wqkv, const float *Wo,
                        const float *W1, const float *W2, const float *g1, const float *g2)
{
    int d = c->d, f = c->ffn;
    pset_t p;
    p.qkv = mat_make(Wqkv, 3 * d, d, c->fp8);
    p.o = mat_make(Wo, d, d, c->fp8);
    p.w1 = mat_make(W1, f, d, c->fp8);
    p.w2 = mat_make(W2, d, f, c->fp8);
    mat_input(c, &p.qkv, l, set, ORC_IN_QKV);
    mat_input(c, &p.o, l, set, ORC_IN_O);
    mat_input(c, &p.w1, l, set, ORC_IN_W1);
    mat_input(c, &p.w2, l, set, ORC_IN_W2);
    p.g1 = g1;
    p.g2 = g2;
    p.moe_E = 0;
    p.moe_k = 0;
    p.router = NULL;
    p.ew1 = p.ew2 = NULL;
    return p;
}

static void pset_free(pset_t *p)
{
    mat_free(&p->qkv); mat_free(&p->o); mat_free(&p->w1); mat_free(&p->w2);
    free(p->ew1);
    free(p->ew2);
}

static pset_t s_params(const orc_cfg *c, const orc_weights *w, int l)
{
    long d = c->d, f = c->ffn;
    if (c->moe_experts > 0) {
        /* the dense S FFN weights are not used: point them at expert 0 */
        long E = c->moe_experts;
        pset_t p = pset_make(c, l, 0, w->Wqkv_s + l * 3 * d * d, w->Wo_s + l * d * d,
                             w->W1_moe + l * E * f * d, w->W2_moe + l * E * d * f, w->g1_s + l * d,
                             w->g2_s + l * d);
        p.moe_E = (int)E;
        p.moe_k = c->moe_topk;
        p.router = w->W_router + l * E * d;
        p.ew1 = (mat_t *)malloc(sizeof(mat_t) * E);
        p.ew2 = (mat_t *)malloc(sizeof(mat_t) * E);
        for (long e = 0; e < E; ++e) {
            p.ew1[e] = mat_plain(w->W1_moe + (l * E + e) * f * d, (int)f, (int)d);
            p.ew2[e] = mat_plain(w->W2_moe + (l * E + e) * d * f, (int)d, (int)f);
        }
        return p;
    }
    return pset_make(c, l, 0, w->Wqkv_s + l * 3 * d * d, w->Wo_s + l * d * d, w->W1_s + l * f * d,
                     w->W2_s + l * d * f, w->g1_s + l * d, w->g2_s + l * d);
}

/* Router of a mixture of experts: the top-k of the logits W_r z (ties to
 * the lower expert index) and their softmax gates. */
static void moe_route(const pset_t *p, const double *z, int d, int *sel, double *gate)
{
    double logit[64];
    for (int e = 0; e < p->moe_E; ++e) {
        const float *r = p->router + (long)e * d;
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += (double)r[k] * z[k];
        logit[e] = acc;
    }
    for (int j = 0; j < p->moe_k; ++j) {
        int best = -1;
        for (int e = 0; e < p->moe_E; ++e) {
            int taken = 0;
            for (int i = 0; i < j; ++i) taken |= sel[i] == e;
            if (!taken && (best < 0 || logit[e] > logit[best])) best = e;
        }
        sel[j] = best;
    }
    double mx = logit[sel[0]], sum = 0.0;
    for (int j = 0; j < p->moe_k; ++j) { gate[j] = exp(logit[sel[j]] - mx); sum += gate[j]; }
    for (int j = 0; j < p->moe_k; ++j) gate[j] /= sum;
}

static pset_t ns_params(const orc_cfg *c, const orc_weights *w, int l, int n)
{
    long d = c->d, f = c->ffn, ln = (long)l * c->n_ns + n;
    return pset_make(c, l, 1 + n, w->Wqkv_ns + ln * 3 * d * d, w->Wo_ns + ln * d * d, w->W1_ns + ln * f * d,
                     w->W2_ns + ln * d * f, w->g1_ns + ln * d, w->g2_ns + ln * d);
}

/* Second half of the block for one row: h = x + a.Wo^T; y = h + W2 GELU(W1 n(h)),
 * or with a mixture of experts y = h + sum_j g_j W2_e(j) GELU(W1_e(j) n(h)). */
static void block_tail(const orc_cfg *c, const pset_t *p, const double *x, const double *a, double *y,
                       double *scr /* >= 3d + 2 ffn */)
{
    int d = c->d, f = c->ffn;
    double *h = scr, *z = scr + d, *t = scr + 2 * d, *hid = scr + 3 * d, *xq = hid + f;
    project(&p->o, a, 0, d, t, xq);
    for (int k = 0; k < d; ++k) h[k] = x[k] + t[k];
    rmsnorm(h, p->g2, d, c->eps, z);
    if (p->moe_E > 0) {
        int sel[2];
        double gate[2];
        moe_route(p, z, d, sel, gate);
        for (int k = 0; k < d; ++k) y[k] = h[k];
        for (int j = 0; j < p->moe_k; ++j) {
            project(&p->ew1[sel[j]], z, 0, f, hid, xq);
            for (int k = 0; k < f; ++k) hid[k] = gelu(hid[k]);
            project(&p->ew2[sel[j]], hid, 0, d, t, xq);
            for (int k = 0; k < d; ++k) y[k] += gate[j] * t[k];
        }
        return;
    }
    project(&p->w1, z, 0, f, hid, xq);
    for (int k = 0; k < f; ++k) hid[k] = gelu(hid[k]);
    project(&p->w2, hid, 0, d, t, xq);
    for (int k = 0; k < d; ++k) y[k] = h[k] + t[k];
}

static int rows_at(const orc_cfg *c, int l) { return l == 0 ? c->L0 : c->q[l - 1]; }

long orc_kv_layer_offset(const orc_cfg *c, int l)
{
    long off = 0;
    for (int j = 0; j < l; ++j) off += 2L * c->d * rows_at(c, j);
    return off;
}

long orc_kv_user_elems(const orc_cfg *c) { return orc_kv_layer_offset(c, c->layers); }

static int check_cfg(const orc_cfg *c)
{
    if (c->layers < 1 || c->layers > ORC_MAX_LAYERS || c->d < 1 || c->heads < 1 ||
        c->d % c->heads || c->ffn < 1 || c->n_ns < 0 || c->L0 < 1 || c->fp8 < 0 || c->fp8 > 2)
        return 1;
    if (c->moe_experts < 0 || c->moe_experts > 64 ||
        (c->moe_experts > 0 && (c->moe_topk < 1 || c->moe_topk > 2 || c->moe_topk > c->moe_experts ||
                                c->fp8)))
        return 1;
    if (c->fp8 == 2) {
        if (!c->act_scale) return 1;
        for (long i = 0; i < (long)c->layers * (1 + c->n_ns) * 4; ++i)
            if (!(c->act_scale[i] > 0.0)) return 1;
    }
    int L = c->L0;
    for (int l = 0; l < c->layers; ++l) {
        if (c->q[l] < 1 || c->q[l] > L) return 1;
        L = c->q[l];
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* S-side for U users ("encode once per user"): per-layer K/V into the cache  */
/* and the final S tail rows.  S is [U][L0][d]; s_out is [U][q_last][d].      */
int orc_encode_user(const orc_cfg *c, const orc_weights *w, const float *S, int U,
                    double *kv, double *s_out)
{
    if (check_cfg(c) || c->full_attn) return 1; /* S would depend on the candidate */
    int d = c->d, H = c->heads, hd = d / H, f = c->ffn;
    long kv_user = orc_kv_user_elems(c);
    for (int u = 0; u < U; ++u) {
        int L = c->L0;
        double *X = (double *)malloc(sizeof(double) * (long)L * d);
        for (long i = 0; i < (long)L * d; ++i) X[i] = S[(long)u * c->L0 * d + i];
        for (int l = 0; l < c->layers; ++l) {
            int q = c->q[l];
            pset_t p = s_params(c, w, l);
            double *K = kv + (long)u * kv_user + orc_kv_layer_offset(c, l);
            double *V = K + (long)L * d;
            double *Q = (double *)malloc(sizeof(double) * (long)q * d);
            double *Y = (double *)malloc(sizeof(double) * (long)q * d);
#pragma omp parallel
            {
                double *xn = (double *)malloc(sizeof(double) * d);
                double *qkv = (double *)malloc(sizeof(double) * 3 * d);
                double *xq = (double *)malloc(sizeof(double) * (d > f ? d : f));
#pragma omp for schedule(static)
                for (int t = 0; t < L; ++t) {
                    rmsnorm(X + (long)t * d, p.g1, d, c->eps, xn);
                    project(&p.qkv, xn, 0, 3 * d, qkv, xq);
                    memcpy(K + (long)t * d, qkv + d, sizeof(double) * d);
                    memcpy(V + (long)t * d, qkv + 2 * d, sizeof(double) * d);
                    if (t >= L - q) memcpy(Q + (long)(t - (L - q)) * d, qkv, sizeof(double) * d);
                }
                free(xn); free(qkv); free(xq);
            }
#pragma omp parallel
            {
                double *a = (double *)malloc(sizeof(double) * d);
                double *sc = (double *)malloc(sizeof(double) * L);
                double *scr = (double *)malloc(sizeof(double) * (3 * d + 2 * f + d));
#pragma omp for schedule(dynamic, 4)
                for (int i = 0; i < q; ++i) {
                    int t = L - q + i; /* S query t sees S keys 0..t */
                    for (int h = 0; h < H; ++h)
                        attend(Q + (long)i * d + h * hd, hd, h * hd, d, K, V, t + 1, NULL, NULL, 0,
                               a + h * hd, sc);
                    block_tail(c, &p, X + (long)t * d, a, Y + (long)i * d, scr);
                }
                free(a); free(sc); free(scr);
            }
            pset_free(&p);
            free(Q);
            free(X);
            X = Y;
            L = q;
        }
        memcpy(s_out + (long)u * L * d, X, sizeof(double) * (long)L * d);
        free(X);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Appending S rows to encoded users (sequence KV caching across requests,     */
/* summary page, KV-cache paragraph; the pages give no schedule for it).      */
/* Reading: the pyramid windows stay anchored at their first row, so every    */
/* layer's row set and query tail grow by the `delta` new rows: c is the grown */
/* configuration (L0 and each q[l] include the new rows) and the previous      */
/* encode used L0 - delta and q[l] - delta.  An old row then sees exactly the */
/* keys it saw before at every layer (the mask is causal and no window loses  */
/* a row), so its K/V and outputs are unchanged; only the new rows are run:   */
/* per layer their K/V join the old ones, and new row t attends to keys 0..t. */
/* kv_old is the previous cache, S_new [U][delta][d]; kv_new receives the      */
/* cache in the grown layout, out_new [U][delta][d] the new rows' outputs of  */
/* the last layer (the last delta rows of the grown S output).               */
int orc_encode_append(const orc_cfg *c, const orc_weights *w, const double *kv_old,
                      const float *S_new, int U, int delta, double *kv_new, double *out_new)
{
    if (check_cfg(c) || c->full_attn || delta < 1) return 1;
    orc_cfg old = *c;
    old.L0 -= delta;
    for (int l = 0; l < c->layers; ++l) old.q[l] -= delta;
    if (check_cfg(&old)) return 1;
    int d = c->d, H = c->heads, hd = d / H, f = c->ffn;
    long kv_user = orc_kv_user_elems(c), kv_user_old = orc_kv_user_elems(&old);
    for (int u = 0; u < U; ++u) {
        double *X = (double *)malloc(sizeof(double) * (long)delta * d);
        for (long i = 0; i < (long)delta * d; ++i) X[i] = S_new[(long)u * delta * d + i];
        for (int l = 0; l < c->layers; ++l) {
            int L = rows_at(c, l), Lo = L - delta;
            pset_t p = s_params(c, w, l);
            double *K = kv_new + (long)u * kv_user + orc_kv_layer_offset(c, l);
            double *V = K + (long)L * d;
            const double *Ko = kv_old + (long)u * kv_user_old + orc_kv_layer_offset(&old, l);
            const double *Vo = Ko + (long)Lo * d;
            memcpy(K, Ko, sizeof(double) * (long)Lo * d);
            memcpy(V, Vo, sizeof(double) * (long)Lo * d);
            double *Q = (double *)malloc(sizeof(double) * (long)delta * d);
            double *Y = (double *)malloc(sizeof(double) * (long)delta * d);
            double *xn = (double *)malloc(sizeof(double) * d);
            double *qkv = (double *)malloc(sizeof(double) * 3 * d);
            double *xq = (double *)malloc(sizeof(double) * (d > f ? d : f));
            for (int i = 0; i < delta; ++i) {
                int t = Lo + i;
                rmsnorm(X + (long)i * d, p.g1, d, c->eps, xn);
                project(&p.qkv, xn, 0, 3 * d, qkv, xq);
                memcpy(Q + (long)i * d, qkv, sizeof(double) * d);
                memcpy(K + (long)t * d, qkv + d, sizeof(double) * d);
                memcpy(V + (long)t * d, qkv + 2 * d, sizeof(double) * d);
            }
            free(xn); free(qkv); free(xq);
#pragma omp parallel
            {
                double *a = (double *)malloc(sizeof(double) * d);
                double *sc = (double *)malloc(sizeof(double) * L);
                double *scr = (double *)malloc(sizeof(double) * (3 * d + 2 * f + d));
#pragma omp for schedule(dynamic, 4)
                for (int i = 0; i < delta; ++i) {
                    int t = Lo + i; /* the new row t sees keys 0..t: the old rows and new rows up to itself */
                    for (int h = 0; h < H; ++h)
                        attend(Q + (long)i * d + h * hd, hd, h * hd, d, K, V, t + 1, NULL, NULL, 0,
                               a + h * hd, sc);
                    block_tail(c, &p, X + (long)i * d, a, Y + (long)i * d, scr);
                }
                free(a); free(sc); free(scr);
            }
            pset_free(&p);
            free(Q);
            free(X);
            X = Y;
        }
        memcpy(out_new + (long)u * delta * d, X, sizeof(double) * (long)delta * d);
        free(X);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* NS-side per candidate against the cached S K/V ("NS-side runs per          */
/* candidate").  ns_in / ns_out are [U][C][N][d].                             */
int orc_score_candidates(const orc_cfg *c, const orc_weights *w, const double *kv, int U,
                         const double *ns_in, int C, double *ns_out)
{
    if (check_cfg(c) || c->full_attn) return 1;
    int d = c->d, H = c->heads, hd = d / H, f = c->ffn, N = c->n_ns;
    long kv_user = orc_kv_user_elems(c);
    pset_t *P = (pset_t *)malloc(sizeof(pset_t) * (long)c->layers * (N > 0 ? N : 1));
    for (int l = 0; l < c->layers; ++l)
        for (int n = 0; n < N; ++n) P[(long)l * N + n] = ns_params(c, w, l, n);
#pragma omp parallel
    {
        double *X = (double *)malloc(sizeof(double) * (long)N * d + 1);
        double *Y = (double *)malloc(sizeof(double) * (long)N * d + 1);
        double *Q = (double *)malloc(sizeof(double) * (long)N * d + 1);
        double *K = (double *)malloc(sizeof(double) * (long)N * d + 1);
        double *V = (double *)malloc(sizeof(double) * (long)N * d + 1);
        double *xn = (double *)malloc(sizeof(double) * d);
        double *qkv = (double *)malloc(sizeof(double) * 3 * d);
        double *xq = (double *)malloc(sizeof(double) * (d > f ? d : f));
        double *a = (double *)malloc(sizeof(double) * d);
        double *sc = (double *)malloc(sizeof(double) * ((long)c->L0 + N));
        double *scr = (double *)malloc(sizeof(double) * (3 * d + 2 * f + d));
#pragma omp for schedule(dynamic, 1)
        for (long uc = 0; uc < (long)U * C; ++uc) {
            int u = (int)(uc / C);
            memcpy(X, ns_in + uc * N * d, sizeof(double) * (long)N * d);
            for (int l = 0; l < c->layers; ++l) {
                int L = rows_at(c, l);
                const double *KS = kv + (long)u * kv_user + orc_kv_layer_offset(c, l);
                const double *VS = KS + (long)L * d;
                for (int n = 0; n < N; ++n) {
                    const pset_t *p = &P[(long)l * N + n];
                    rmsnorm(X + (long)n * d, p->g1, d, c->eps, xn);
                    project(&p->qkv, xn, 0, 3 * d, qkv, xq);
                    memcpy(Q + (long)n * d, qkv, sizeof(double) * d);
                    memcpy(K + (long)n * d, qkv + d, sizeof(double) * d);
                    memcpy(V + (long)n * d, qkv + 2 * d, sizeof(double) * d);
                }
                for (int n = 0; n < N; ++n) {
                    /* NS token n sees all L S keys and NS keys 0..n of this candidate */
                    for (int h = 0; h < H; ++h)
                        attend(Q + (long)n * d + h * hd, hd, h * hd, d, KS, VS, L, K, V, n + 1,
                               a + h * hd, sc);
                    block_tail(c, &P[(long)l * N + n], X + (long)n * d, a, Y + (long)n * d, scr);
                }
                double *tmp = X; X = Y; Y = tmp;
            }
            memcpy(ns_out + uc * N * d, X, sizeof(double) * (long)N * d);
        }
        free(X); free(Y); free(Q); free(K); free(V); free(xn); free(qkv); free(xq); free(a);
        free(sc); free(scr);
    }
    for (long i = 0; i < (long)c->layers * N; ++i) pset_free(&P[i]);
    free(P);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Joint formulation: every candidate's own token sequence [S rows; NS rows]  */
/* run through the stack with no cache, each token picking its parameter set  */
/* by type and position and its visible keys by the S/NS mask rule (or, with  */
/* full attention, every key of the sequence).                                */
/* s_out [U][C][q_last][d]; kv [U][C][cache]; ns_out [U][C][N][d].            */
int orc_full_forward_joint(const orc_cfg *c, const orc_weights *w, const float *S, int U,
                           const double *ns_in, int C, double *s_out, double *kv, double *ns_out)
{
    if (check_cfg(c)) return 1;
    int d = c->d, H = c->heads, hd = d / H, f = c->ffn, N = c->n_ns;
    long kv_user = orc_kv_user_elems(c);
    int qlast = c->q[c->layers - 1];
    for (long uc = 0; uc < (long)U * C; ++uc) {
        int u = (int)(uc / C);
        int L = c->L0;
        long T = L + N;
        double *X = (double *)malloc(sizeof(double) * T * d);
        for (long i = 0; i < (long)L * d; ++i) X[i] = S[(long)u * c->L0 * d + i];
        memcpy(X + (long)L * d, ns_in + uc * N * d, sizeof(double) * (long)N * d);
        for (int l = 0; l < c->layers; ++l) {
            int q = c->q[l];
            T = L + N;
            pset_t *P = (pset_t *)malloc(sizeof(pset_t) * (N + 1));
            P[0] = s_params(c, w, l);
            for (int n = 0; n < N; ++n) P[1 + n] = ns_params(c, w, l, n);
            double *Qa = (double *)malloc(sizeof(double) * T * d);
            double *Ka = (double *)malloc(sizeof(double) * T * d);
            double *Va = (double *)malloc(sizeof(double) * T * d);
            long nq = q + N; /* query rows: S tail rows L-q..L-1, then all NS rows */
            double *Y = (double *)malloc(sizeof(double) * nq * d);
#pragma omp parallel
            {
                double *xn = (double *)malloc(sizeof(double) * d);
                double *qkv = (double *)malloc(sizeof(double) * 3 * d);
                double *xq = (double *)malloc(sizeof(double) * (d > f ? d : f));
#pragma omp for schedule(static)
                for (long i = 0; i < T; ++i) {
                    const pset_t *p = i < L ? &P[0] : &P[1 + (i - L)];
                    rmsnorm(X + i * d, p->g1, d, c->eps, xn);
                    project(&p->qkv, xn, 0, 3 * d, qkv, xq);
                    memcpy(Qa + i * d, qkv, sizeof(double) * d);
                    memcpy(Ka + i * d, qkv + d, sizeof(double) * d);
                    memcpy(Va + i * d, qkv + 2 * d, sizeof(double) * d);
                }
                free(xn); free(qkv); free(xq);
            }
            double *kvl = kv + uc * kv_user + orc_kv_layer_offset(c, l);
            memcpy(kvl, Ka, sizeof(double) * (long)L * d);
            memcpy(kvl + (long)L * d, Va, sizeof(double) * (long)L * d);
#pragma omp parallel
            {
                double *a = (double *)malloc(sizeof(double) * d);
                double *sc = (double *)malloc(sizeof(double) * T);
                double *Kv = (double *)malloc(sizeof(double) * T * d);
                double *Vv = (double *)malloc(sizeof(double) * T * d);
                double *scr = (double *)malloc(sizeof(double) * (3 * d + 2 * f + d));
#pragma omp for schedule(dynamic, 4)
                for (long r = 0; r < nq; ++r) {
                    long i = r < q ? (L - q + r) : (L + (r - q)); /* sequence position */
                    int is_ns = i >= L;
                    /* gather the keys token i may see, by the S/NS mask rule */
                    int nv = 0;
                    for (long j = 0; j < T; ++j) {
                        int j_ns = j >= L;
                        int ok = c->full_attn ? 1 : is_ns ? (!j_ns || j <= i) : (!j_ns && j <= i);
                        if (ok) {
                            memcpy(Kv + (long)nv * d, Ka + j * d, sizeof(double) * d);
                            memcpy(Vv + (long)nv * d, Va + j * d, sizeof(double) * d);
                            ++nv;
                        }
                    }
                    for (int h = 0; h < H; ++h)
                        attend(Qa + i * d + h * hd, hd, h * hd, d, Kv, Vv, nv, NULL, NULL, 0,
                               a + h * hd, sc);
                    const pset_t *p = is_ns ? &P[1 + (i - L)] : &P[0];
                    block_tail(c, p, X + i * d, a, Y + r * d, scr);
                }
                free(a); free(sc); free(Kv); free(Vv); free(scr);
            }
            for (int n = 0; n <= N; ++n) pset_free(&P[n]);
            free(P); free(Qa); free(Ka); free(Va); free(X);
            X = Y; /* [q S tail rows; N NS rows] is the next layer's sequence */
            L = q;
        }
        memcpy(s_out + uc * (long)qlast * d, X, sizeof(double) * (long)qlast * d);
        memcpy(ns_out + uc * (long)N * d, X + (long)qlast * d, sizeof(double) * (long)N * d);
        free(X);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* One projection of `rows` input rows under an FP8 rule, exactly as the      */
/* block's projections run it (fp8 0 / 1 / 2 as in the config; xs is the     */
/* per-tensor scale of rule 2; amax, if not NULL, accumulates max |x|).      */
/* x [rows][in], W [out][in] -> y [rows][out].                                */
int orc_project_rows(const double *x, long rows, int in, const float *W, int out, int fp8,
                     double xs, double *amax, double *y)
{
    if (rows < 0 || in < 1 || out < 1 || fp8 < 0 || fp8 > 2 || (fp8 == 2 && !(xs > 0.0)))
        return 1;
    mat_t m = mat_make(W, out, in, fp8);
    m.xs = xs;
    m.amax = amax;
    double *xq = (double *)malloc(sizeof(double) * in);
    for (long r = 0; r < rows; ++r) project(&m, x + r * in, 0, out, y + r * out, xq);
    free(xq);
    mat_free(&m);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Auto-Split: one projection of the concatenated static features, sliced     */
/* into N tokens of width d (token n = output columns n*d .. n*d+d-1).         */
/* x [M][F], W_split [N*d][F] -> ns [M][N*d] (= [M][N][d]).                    */
int orc_auto_split(const float *x, long M, int F, const float *W_split, int Nd, double *ns)
{
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (int j = 0; j < Nd; ++j) {
            double acc = 0.0;
            for (int k = 0; k < F; ++k) acc += (double)x[m * F + k] * W_split[(long)j * F + k];
            ns[m * Nd + j] = acc;
        }
    return 0;
}

/* Embedding gather: out[i] = table[ids[i]]; ids out of range -> error. */
int orc_embed_gather(const float *table, long rows, int d, const long long *ids, long n, double *out)
{
    for (long i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= rows) return 1;
    for (long i = 0; i < n; ++i)
        for (int k = 0; k < d; ++k) out[i * d + k] = table[ids[i] * d + k];
    return 0;
}

int orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
