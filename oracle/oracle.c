/*
 * oracle.c -- plain, slow CPU oracle of one sparse latent-MoE decode layer step.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU-baseline leg
 * may load this library.  It shares no code, header, table or helper with the CUDA path
 * and never calls it.  Every floating-point accumulation is in double; fp32 appears only
 * where the layer's definition rounds to fp32 (router logits, sigmoid scores, routing
 * weights).
 *
 * What the step computes.  The layer is Kimi K3's "Stable LatentMoE": 896 routed experts
 * with 16 active per token and MXFP4 weights ("快是可以生成的，可信只能证明（vLLM 重写
 * Kimi K3 解码路径…）", section 为什么一条请求会慢; "NVIDIA uses a 12,000-line Megakernel
 * to optimize Kimi K3 inference…", section 一个工程师、1.2万行代码、AI辅助开发).  Router
 * scoring, the latent projection and a shared expert are named as separate parts of the
 * step (same jetabc page, section 他们换掉了什么).  The pages give no formulas; the
 * layer's definition used here is the workload's:
 *
 *   logit[b,e] = fp32( sum_j R[e,j] x[b,j] )      products exact, summed in double (j asc)
 *   s[b,e]     = fp32( 1 / (1 + exp(-logit)) )     computed in double, libm exp
 *   top-k      = the k largest s, the lower expert index first among equal s
 *   w[b,r]     = s_r / S,  S = fp32 sum of the k selected s in rank order, fp32 divide
 *   h          = W_dn x                            (latent down-projection, H -> L)
 *   y_e        = D_e ( silu(G_e h) * (U_e h) ),    silu(z) = z / (1 + exp(-z))
 *   ylat       = sum over selected e (ascending e) of w_e y_e
 *   sh         = SD ( silu(SG x) * (SU x) )        (shared expert, acting on H)
 *   out        = W_up ylat + sh                    (returned in double, before any rounding)
 *
 * Readings where the pages are silent: the router and the shared expert see x (width H),
 * the routed experts see h = W_dn x (width L), the combine happens in the latent space and
 * one L -> H projection follows; there is no routed scaling factor, no router bias and no
 * group-limited routing.
 *
 * MXFP4 (OCP Microscaling Formats MX v1.0): a matrix [N, K] is codes uint8 [N][K/2] (element
 * 2j in the low nibble of byte j, 2j+1 in the high nibble) plus one E8M0 scale byte per
 * 32-element block along K, uint8 [N][K/32].  Element value = E2M1(code) * 2^(scale - 127).
 *
 * Rows of a matrix-vector product are independent, so an OpenMP row loop gives results
 * identical to one thread.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int hidden, latent, n_experts, top_k, expert_inter, shared_inter, n_shared;
} oracle_dims;

typedef struct {
    const uint16_t *router;     /* [E][H] bf16 */
    const uint16_t *w_down_lat; /* [L][H] bf16 */
    const uint16_t *w_up_lat;   /* [H][L] bf16 */
    const uint8_t *gate_q, *gate_s, *up_q, *up_s; /* [E][I][L/2], [E][I][L/32] */
    const uint8_t *down_q, *down_s;               /* [E][L][I/2], [E][L][I/32] */
    const uint8_t *sh_gate_q, *sh_gate_s, *sh_up_q, *sh_up_s; /* [Is][H/2], [Is][H/32] */
    const uint8_t *sh_down_q, *sh_down_s;                     /* [H][Is/2], [H][Is/32] */
} oracle_weights;

/* ---- number formats ---------------------------------------------------------------- */

/* bf16 bits -> value (bf16 is the top half of an IEEE binary32). */
double oracle_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* E2M1 (OCP MX v1.0): sign = bit 3; magnitudes of codes 0..7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1(unsigned code) {
    static const double magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = magnitude[code & 7u];
    return (code & 8u) ? -v : v;
}

/* E8M0 (OCP MX v1.0): 2^(s - 127); 0xFF is NaN. */
double oracle_e8m0(unsigned s) {
    if (s == 255u) return NAN;
    return ldexp(1.0, (int)s - 127);
}

/* Element (n, k) of an MXFP4 matrix with K columns. */
double oracle_mxfp4_element(const uint8_t *q, const uint8_t *s, int K, int n, int k) {
    uint8_t byte = q[(size_t)n * (size_t)(K / 2) + (size_t)(k / 2)];
    unsigned code = (k & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
    return oracle_e2m1(code) * oracle_e8m0(s[(size_t)n * (size_t)(K / 32) + (size_t)(k / 32)]);
}

/* ---- matrix-vector products ------------------------------------------------------------ */

/* out[n] = sum_k W[n][k] v[k], W bf16 [N][K], ascending k, double. */
void oracle_bf16_matvec(const uint16_t *W, int N, int K, const double *v, double *out) {
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const uint16_t *row = W + (size_t)n * (size_t)K;
        double acc = 0.0;
        for (int k = 0; k < K; ++k) acc += oracle_bf16(row[k]) * v[k];
        out[n] = acc;
    }
}

/* out[n] = sum_k W[n][k] v[k], W MXFP4 [N][K], ascending k, double. */
void oracle_mxfp4_matvec(const uint8_t *q, const uint8_t *s, int N, int K, const double *v, double *out) {
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int k = 0; k < K; ++k) acc += oracle_mxfp4_element(q, s, K, n, k) * v[k];
        out[n] = acc;
    }
}

double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* ---- routing --------------------------------------------------------------------------- */

/* logits[b][e] = fp32(sum_j R[e][j] x[b][j]): exact bf16 products summed in double, j ascending. */
void oracle_router_logits(const uint16_t *R, const uint16_t *x, int B, int E, int H, float *logits) {
    for (int b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < H; ++j)
                acc += oracle_bf16(R[(size_t)e * H + j]) * oracle_bf16(x[(size_t)b * H + j]);
            logits[(size_t)b * E + e] = (float)acc;
        }
    }
}

/* score = fp32(1 / (1 + exp(-logit))) evaluated in double. */
float oracle_score(float logit) { return (float)(1.0 / (1.0 + exp(-(double)logit))); }

typedef struct {
    float s;
    int e;
} oracle_cand;

static int cand_order(const void *pa, const void *pb) {
    const oracle_cand *a = (const oracle_cand *)pa, *b = (const oracle_cand *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->e < b->e) ? -1 : (a->e > b->e);
}

/*
 * Top-k of one token's E scores: rank by score descending, lower index first among equal
 * scores; keep the first k.  idx[r], w[r] in rank order; w_r = s_r / S with S the fp32 sum of
 * the kept scores in rank order and an fp32 divide.
 */
void oracle_topk(const float *scores, int E, int k, int32_t *idx, float *w) {
    oracle_cand *c = (oracle_cand *)malloc(sizeof(oracle_cand) * (size_t)E);
    for (int e = 0; e < E; ++e) {
        c[e].s = scores[e];
        c[e].e = e;
    }
    qsort(c, (size_t)E, sizeof(oracle_cand), cand_order);
    float S = 0.0f;
    for (int r = 0; r < k; ++r) S += c[r].s;
    for (int r = 0; r < k; ++r) {
        idx[r] = c[r].e;
        w[r] = c[r].s / S;
    }
    free(c);
}

/* Routing of B tokens: logits, then scores and top-k per token. */
void oracle_route(const uint16_t *R, const uint16_t *x, int B, int E, int H, int k, float *logits,
                  int32_t *idx, float *w) {
    oracle_router_logits(R, x, B, E, H, logits);
    float *s = (float *)malloc(sizeof(float) * (size_t)E);
    for (int b = 0; b < B; ++b) {
        for (int e = 0; e < E; ++e) s[e] = oracle_score(logits[(size_t)b * E + e]);
        oracle_topk(s, E, k, idx + (size_t)b * k, w + (size_t)b * k);
    }
    free(s);
}

/* ---- one routed expert and the shared expert ------------------------------------------ */

/* y = D_e( silu(G_e h) * (U_e h) ) for expert e; h has L entries, y has L entries. */
void oracle_expert(const oracle_dims *d, const oracle_weights *W, int e, const double *h, double *y) {
    int L = d->latent, I = d->expert_inter;
    size_t gq = (size_t)e * I * (L / 2), gs = (size_t)e * I * (L / 32);
    size_t dq = (size_t)e * L * (I / 2), ds = (size_t)e * L * (I / 32);
    double *g = (double *)malloc(sizeof(double) * I), *u = (double *)malloc(sizeof(double) * I);
    oracle_mxfp4_matvec(W->gate_q + gq, W->gate_s + gs, I, L, h, g);
    oracle_mxfp4_matvec(W->up_q + gq, W->up_s + gs, I, L, h, u);
    for (int i = 0; i < I; ++i) g[i] = oracle_silu(g[i]) * u[i];
    oracle_mxfp4_matvec(W->down_q + dq, W->down_s + ds, L, I, g, y);
    free(g);
    free(u);
}

/* sh = SD( silu(SG x) * (SU x) ); x has H entries (double), sh has H entries. */
void oracle_shared_expert(const oracle_dims *d, const oracle_weights *W, const double *x, double *sh) {
    int H = d->hidden, Is = d->shared_inter;
    if (d->n_shared == 0) {
        for (int j = 0; j < H; ++j) sh[j] = 0.0;
        return;
    }
    double *g = (double *)malloc(sizeof(double) * Is), *u = (double *)malloc(sizeof(double) * Is);
    oracle_mxfp4_matvec(W->sh_gate_q, W->sh_gate_s, Is, H, x, g);
    oracle_mxfp4_matvec(W->sh_up_q, W->sh_up_s, Is, H, x, u);
    for (int i = 0; i < Is; ++i) g[i] = oracle_silu(g[i]) * u[i];
    oracle_mxfp4_matvec(W->sh_down_q, W->sh_down_s, H, Is, g, sh);
    free(g);
    free(u);
}

/* ---- the step -------------------------------------------------------------------------- */

static int int_cmp(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/*
 * One decode layer step for the tokens [b0, b0 + nb) of x[B][H] (bf16 bits).  Routing is
 * computed for those tokens only.  Outputs are indexed from token b0 (row 0 = token b0):
 * out, sh [nb][H]; h, ylat [nb][L]; logits [nb][E]; idx, w [nb][k].  Any output pointer may
 * be NULL except out.  dense_masked = 1 evaluates all E experts and weights the unselected
 * ones by exact zeros (a check of the sparse path; the sums are identical).
 */
int oracle_step_tokens(const oracle_dims *d, const oracle_weights *W, const uint16_t *x, int b0, int nb,
                       int dense_masked, double *out, double *h_tap, double *ylat_tap, double *sh_tap,
                       float *logits_out, int32_t *idx_out, float *w_out) {
    int H = d->hidden, L = d->latent, E = d->n_experts, k = d->top_k;
    if (H % 32 || L % 32 || d->expert_inter % 32 || d->shared_inter % 32 || k < 1 || k > E) return -1;
    double *xd = (double *)malloc(sizeof(double) * H);
    double *h = (double *)malloc(sizeof(double) * L);
    double *y = (double *)malloc(sizeof(double) * L);
    double *ylat = (double *)malloc(sizeof(double) * L);
    double *sh = (double *)malloc(sizeof(double) * H);
    double *up = (double *)malloc(sizeof(double) * H);
    float *logits = (float *)malloc(sizeof(float) * E);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * k);
    float *w = (float *)malloc(sizeof(float) * k);
    int *order = (int *)malloc(sizeof(int) * k);
    for (int t = 0; t < nb; ++t) {
        const uint16_t *xb = x + (size_t)(b0 + t) * H;
        for (int j = 0; j < H; ++j) xd[j] = oracle_bf16(xb[j]);
        oracle_route(W->router, xb, 1, E, H, k, logits, idx, w);
        oracle_bf16_matvec(W->w_down_lat, L, H, xd, h);
        for (int l = 0; l < L; ++l) ylat[l] = 0.0;
        if (!dense_masked) {
            /* selected experts in ascending expert order */
            for (int r = 0; r < k; ++r) order[r] = idx[r];
            qsort(order, (size_t)k, sizeof(int), int_cmp);
            for (int i = 0; i < k; ++i) {
                int e = order[i];
                double we = 0.0;
                for (int r = 0; r < k; ++r)
                    if (idx[r] == e) we = (double)w[r];
                oracle_expert(d, W, e, h, y);
                for (int l = 0; l < L; ++l) ylat[l] += we * y[l];
            }
        } else {
            for (int e = 0; e < E; ++e) {
                double we = 0.0;
                for (int r = 0; r < k; ++r)
                    if (idx[r] == e) we = (double)w[r];
                oracle_expert(d, W, e, h, y);
                for (int l = 0; l < L; ++l) ylat[l] += we * y[l];
            }
        }
        oracle_shared_expert(d, W, xd, sh);
        oracle_bf16_matvec(W->w_up_lat, H, L, ylat, up);
        for (int j = 0; j < H; ++j) out[(size_t)t * H + j] = up[j] + sh[j];
        if (h_tap) memcpy(h_tap + (size_t)t * L, h, sizeof(double) * L);
        if (ylat_tap) memcpy(ylat_tap + (size_t)t * L, ylat, sizeof(double) * L);
        if (sh_tap) memcpy(sh_tap + (size_t)t * H, sh, sizeof(double) * H);
        if (logits_out) memcpy(logits_out + (size_t)t * E, logits, sizeof(float) * E);
        if (idx_out) memcpy(idx_out + (size_t)t * k, idx, sizeof(int32_t) * k);
        if (w_out) memcpy(w_out + (size_t)t * k, w, sizeof(float) * k);
    }
    free(xd); free(h); free(y); free(ylat); free(sh); free(up);
    free(logits); free(idx); free(w); free(order);
    return 0;
}

int oracle_step(const oracle_dims *d, const oracle_weights *W, const uint16_t *x, int B, double *out,
                double *h_tap, double *ylat_tap, double *sh_tap, float *logits, int32_t *idx, float *w) {
    return oracle_step_tokens(d, W, x, 0, B, 0, out, h_tap, ylat_tap, sh_tap, logits, idx, w);
}

int oracle_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
