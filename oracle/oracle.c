/*
 * oracle.c -- fp64 CPU oracle of the mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, link or run
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or constant with the CUDA
 * library and includes nothing from it.
 *
 * What it computes.  The pages ("Cursor åpner megakernelen som ga 41 prosent
 * flere tokens i sekundet", last paragraph; "Cursor veröffentlicht
 * MoE-Megakernel Mixture-of-Kittens als Open Source", introduction) say only
 * that the kernel implements a DeepSeek-V3-type MoE layer, forward and
 * backward, in BF16 and MXFP8 ("Megakernels are dead and back…", section
 * "Números de MoK").  They print no formula.  The layer below is the plain
 * DeepSeek-V3 definition:
 *   router   logits = x . Wr^T (+ an optional additive logit term), fp64
 *   scoring  softmax top-k, or sigmoid + selection bias with group-limited
 *            top-k (group score = sum of the group's two best biased scores)
 *   weights  selected probabilities (softmax) or unbiased sigmoid scores,
 *            renormalised over the selected experts, times routed_scale
 *   experts  SwiGLU: h = silu(x Wg^T) * (x Wu^T), o = h Wd^T
 *   combine  y = sum_j w_j o_j (j ascending) + sum_s o_s (shared experts)
 *   backward the closed-form chain rule of the above.
 * Selection sorts (score descending, expert index ascending), so ties go to
 * the lower expert index; groups likewise go to the lower group id.
 *
 * Rounding mirrors.  Unless cfg->pure is set, the oracle rounds to bf16
 * (round-to-nearest-even, computed directly from fp64) exactly where the
 * layer stores a tensor in bf16: h, y, the saved gate/up pre-activations read
 * by the backward, the weighted h used by the down-projection weight
 * gradient, dGU, dx and the weight gradients.  The per-(token, slot) rows of
 * the forward (o) and of the backward (per-slot dx) are stored in fp32, so
 * they are not rounded.  In MXFP8 mode x and h are quantised with the 1x32 ue8m0
 * block rule below; weights are fake-quantised by the caller with
 * orc_mx_fakequant_bf16 before use.
 *
 * MXFP8 backward (not claimed by the pages; the plain reading of "MXFP8
 * training" applied to this layer): the two data-gradient products run on
 * MXFP8 operands quantised along their own contraction axis -- dy along H for
 * dy . W_down, and dGU along 2I (blocks of 32 inside the gate and the up half)
 * for dGU . W_gate_up, with weight copies that the caller fake-quantises along
 * that axis (orc_mx_fakequant_cols_bf16: W_down along H, W_gate_up along 2I).
 * dGU is quantised from its unrounded value.  The slot gradient is read off the
 * same product, G_j = <Q(dy) . W_down, Q(h_j)>, as the layer's fused epilogue
 * does.  The weight gradients stay BF16 products: dW_gate_up from the stored
 * bf16 dGU and the quantised x the forward used, dW_down from the bf16 dy and
 * bf16(w Q(h)).
 *
 * Pins.  Every function here is checked by tests that do not call it to
 * produce their own expected values: brute-force top-k, closed forms of the
 * weights, permutation invariants, a dense SwiGLU MLP via library matmuls,
 * torch's bf16/e4m3 conversions, hand-derived MX blocks and central finite
 * differences of the pure fp64 forward.  The DeepSeek-V3 routing reading
 * itself has no printed source on the pages ("parity unpinned" for the
 * reading, not for the arithmetic).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element kinds of an input array */
enum { ORC_BF16 = 0, ORC_F32 = 1, ORC_F64 = 2 };

typedef struct {
    int T, H, E, k, I, S, Is;     /* tokens, hidden, experts, top-k, expert inter, shared count, shared inter */
    int score_fn;                 /* 0 softmax, 1 sigmoid + selection bias */
    int n_group, topk_group;      /* group-limited selection; 1,1 = none */
    double routed_scale;
    int mx;                       /* 1: MXFP8 forward (x and h quantised) */
    int pure;                     /* 1: no rounding mirrors at all */
    int act_kind;                 /* kind of x and dy */
    int w_kind;                   /* kind of the expert weights */
    int r_kind;                   /* kind of router_w, e_bias, logit_bias */
} orc_cfg;

/* ---------------------------------------------------------------- scalars */

static double bf16_bits_to_d(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static inline double ld(const void *p, int64_t i, int kind)
{
    if (kind == ORC_BF16) return bf16_bits_to_d(((const uint16_t *)p)[i]);
    if (kind == ORC_F32) return (double)((const float *)p)[i];
    return ((const double *)p)[i];
}

/* Round a double to the nearest bf16 value (ties to even), in one rounding. */
double orc_round_bf16(double v)
{
    if (v == 0.0 || !isfinite(v)) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int q = (e - 1) - 7;          /* 8 significant bits */
    if (e - 1 < -126) q = -133;   /* subnormal spacing */
    double r = ldexp(nearbyint(ldexp(a, -q)), q);
    if (r > 3.3895313892515355e38) r = INFINITY;
    return copysign(r, v);
}

/* bf16 bit pattern of a value already representable in bf16 */
uint16_t orc_bf16_bits(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* Round to the nearest OCP e4m3 (fn) value, ties to even, saturating to +-448. */
double orc_round_e4m3(double v)
{
    if (v == 0.0) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);
    int p = e - 1;                /* a in [2^p, 2^(p+1)) */
    if (p < -6) p = -6;           /* subnormals share the spacing of the first binade */
    int q = p - 3;                /* 3 mantissa bits */
    double r = ldexp(nearbyint(ldexp(a, -q)), q);
    if (r > 448.0) r = 448.0;
    return copysign(r, v);
}

/* e4m3 code of a value that is exactly an e4m3 value (sign kept for zero) */
uint8_t orc_e4m3_bits(double r)
{
    uint8_t s = signbit(r) ? 0x80 : 0x00;
    double a = fabs(r);
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int p = e - 1;
    if (p < -6) return (uint8_t)(s | (uint8_t)ldexp(a, 9));        /* subnormal: a = m * 2^-9 */
    int mant = (int)ldexp(a, 3 - p) - 8;                           /* a = (1 + mant/8) 2^p */
    return (uint8_t)(s | ((p + 7) << 3) | mant);
}

double orc_e4m3_value(uint8_t b)
{
    int s = b >> 7, ex = (b >> 3) & 15, m = b & 7;
    if (ex == 15 && m == 7) return NAN;
    double a = ex == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, ex - 7);
    return s ? -a : a;
}

/* MX block exponent: the smallest integer e with amax <= 448 * 2^e, clamped to
 * [-127, 127]; an all-zero block takes -127.  The stored ue8m0 byte is e+127. */
int orc_mx_scale_exp(double amax)
{
    if (!(amax > 0.0)) return -127;
    int p;
    frexp(amax, &p);
    p -= 1;                       /* amax in [2^p, 2^(p+1)) */
    int e = p - 9;                /* 448 * 2^(p-9) < 2^p <= amax: too small */
    while (amax > ldexp(448.0, e)) e++;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Quantise one block of n (<= 32) values in place to their MX-dequantised
 * values; optionally emit codes and the scale byte. */
static void mx_block(double *v, int n, uint8_t *codes, uint8_t *scale)
{
    double amax = 0.0;
    for (int i = 0; i < n; i++) if (fabs(v[i]) > amax) amax = fabs(v[i]);
    int e = orc_mx_scale_exp(amax);
    for (int i = 0; i < n; i++) {
        double q = orc_round_e4m3(ldexp(v[i], -e));
        if (codes) codes[i] = orc_e4m3_bits(q);
        v[i] = ldexp(q, e);
    }
    if (scale) *scale = (uint8_t)(e + 127);
}

/* MXFP8 quantisation of a bf16 matrix [rows, K] along K: e4m3 codes [rows, K]
 * and ue8m0 scales [rows, K/32]. */
int orc_mx_quantize(const uint16_t *src, int64_t rows, int64_t K, uint8_t *q, uint8_t *sc)
{
    if (K % 32) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        double v[32];
        for (int64_t b = 0; b < K / 32; b++) {
            for (int i = 0; i < 32; i++) v[i] = bf16_bits_to_d(src[r * K + b * 32 + i]);
            mx_block(v, 32, q + r * K + b * 32, sc + r * (K / 32) + b);
        }
    }
    return 0;
}

/* Replace a bf16 matrix [rows, K] in place by its MXFP8-dequantised values
 * (exactly representable in bf16). */
int orc_mx_fakequant_bf16(uint16_t *data, int64_t rows, int64_t K)
{
    if (K % 32) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        double v[32];
        for (int64_t b = 0; b < K / 32; b++) {
            for (int i = 0; i < 32; i++) v[i] = bf16_bits_to_d(data[r * K + b * 32 + i]);
            mx_block(v, 32, NULL, NULL);
            for (int i = 0; i < 32; i++) data[r * K + b * 32 + i] = orc_bf16_bits(v[i]);
        }
    }
    return 0;
}

/* Replace a bf16 tensor [batch, R, C] in place by its MXFP8-dequantised values
 * with blocks of 32 consecutive rows of each column (quantisation along R, the
 * axis a product with the transposed matrix contracts over). */
int orc_mx_fakequant_cols_bf16(uint16_t *data, int64_t batch, int64_t R, int64_t C)
{
    if (R % 32) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < batch; b++)
        for (int64_t c = 0; c < C; c++) {
            double v[32];
            uint16_t *m = data + b * R * C + c;
            for (int64_t r0 = 0; r0 < R; r0 += 32) {
                for (int i = 0; i < 32; i++) v[i] = bf16_bits_to_d(m[(r0 + i) * C]);
                mx_block(v, 32, NULL, NULL);
                for (int i = 0; i < 32; i++) m[(r0 + i) * C] = orc_bf16_bits(v[i]);
            }
        }
    return 0;
}

static inline double mirror(const orc_cfg *c, double v) { return c->pure ? v : orc_round_bf16(v); }

/* ---------------------------------------------------------------- routing */

/* sort helper: indices by (key descending, index ascending) -- insertion sort */
static void order_desc(const double *key, int *idx, int n)
{
    for (int i = 0; i < n; i++) idx[i] = i;
    for (int i = 1; i < n; i++) {
        int v = idx[i], j = i - 1;
        while (j >= 0 && (key[idx[j]] < key[v] || (key[idx[j]] == key[v] && idx[j] > v))) {
            idx[j + 1] = idx[j];
            j--;
        }
        idx[j + 1] = v;
    }
}

/* Route one token.  Outputs: idx[k], w[k] (slot order = selection order),
 * sel[k] = the selection score of each slot, dlogit helpers are not needed
 * here.  Returns the smallest adjacent gap among the top k+1 selection scores
 * (and, with group limiting, among the top topk_group+1 group scores). */
static double route_token(const orc_cfg *c, const void *x, const void *Wr, const void *bias,
                          const void *lbias, int t, int *idx, double *w, double *logit_out,
                          double *score_out)
{
    const int E = c->E, H = c->H, k = c->k;
    double *lg = (double *)malloc(sizeof(double) * E * 4);
    double *sc = lg + E, *prob = lg + 2 * E, *tmp = lg + 3 * E;
    int *ord = (int *)malloc(sizeof(int) * (E + 2));
    for (int e = 0; e < E; e++) {
        double s = 0.0;
        for (int h = 0; h < H; h++) s += ld(x, (int64_t)t * H + h, c->act_kind) * ld(Wr, (int64_t)e * H + h, c->r_kind);
        if (lbias) s += ld(lbias, e, c->r_kind);
        lg[e] = s;
    }
    if (c->score_fn == 0) {
        /* a NaN logit (non-finite input) stays NaN and is left out of the
         * normaliser, so the other experts' probabilities do not depend on it */
        double mx = -INFINITY;
        for (int e = 0; e < E; e++) if (lg[e] > mx) mx = lg[e];
        double z = 0.0;
        for (int e = 0; e < E; e++) { prob[e] = exp(lg[e] - mx); if (!isnan(prob[e])) z += prob[e]; }
        for (int e = 0; e < E; e++) { prob[e] /= z; sc[e] = prob[e]; }
    } else {
        for (int e = 0; e < E; e++) {
            prob[e] = 1.0 / (1.0 + exp(-lg[e]));
            sc[e] = prob[e] + (bias ? ld(bias, e, c->r_kind) : 0.0);
        }
    }
    /* a NaN selection score (non-finite input) ranks below every other score,
     * like -inf; the order (score descending, index ascending) stays total */
    for (int e = 0; e < E; e++) if (isnan(sc[e])) sc[e] = -INFINITY;
    double gap = INFINITY;
    /* group limiting: keep the topk_group groups with the best top-2 sums */
    int G = c->n_group, gs = E / G;
    unsigned char *keep = (unsigned char *)malloc(E);
    if (G > 1 && c->topk_group < G) {
        double *gsc = (double *)malloc(sizeof(double) * G);
        int *gord = (int *)malloc(sizeof(int) * G);
        int *wo = (int *)malloc(sizeof(int) * gs);
        for (int g = 0; g < G; g++) {
            order_desc(sc + g * gs, wo, gs);
            gsc[g] = sc[g * gs + wo[0]] + (gs > 1 ? sc[g * gs + wo[1]] : 0.0);
            if (isnan(gsc[g])) gsc[g] = -INFINITY;      /* -inf + inf */
        }
        order_desc(gsc, gord, G);
        memset(keep, 0, E);
        for (int i = 0; i < c->topk_group; i++)
            for (int e = 0; e < gs; e++) keep[gord[i] * gs + e] = 1;
        for (int i = 0; i < c->topk_group && i + 1 < G; i++) {
            double d = gsc[gord[i]] - gsc[gord[i + 1]];
            if (d < gap) gap = d;
        }
        free(gsc); free(gord); free(wo);
    } else {
        memset(keep, 1, E);
    }
    for (int e = 0; e < E; e++) tmp[e] = keep[e] ? sc[e] : -INFINITY;
    order_desc(tmp, ord, E);
    double tot = 0.0;
    for (int j = 0; j < k; j++) tot += prob[ord[j]];
    for (int j = 0; j < k; j++) {
        idx[j] = ord[j];
        w[j] = c->routed_scale * prob[ord[j]] / tot;
    }
    int ncand = 0;
    for (int e = 0; e < E; e++) ncand += keep[e];
    for (int j = 0; j < k && j + 1 < ncand; j++) {
        double d = tmp[ord[j]] - tmp[ord[j + 1]];
        if (d < gap) gap = d;
    }
    if (logit_out) memcpy(logit_out, lg, sizeof(double) * E);
    if (score_out) memcpy(score_out, prob, sizeof(double) * E);
    free(keep); free(ord); free(lg);
    return gap;
}

/* Route the tokens tokens[0..n) (all T tokens when tokens is NULL).
 * idx, w: [T, k]; gap: [T]; logits, probs: [T, E] or NULL; rows of tokens not
 * routed are left untouched. */
int orc_route(const orc_cfg *c, const void *x, const void *Wr, const void *bias, const void *lbias,
              const int32_t *tokens, int n, int32_t *idx, double *w, double *gap, double *logits,
              double *probs)
{
    if (c->E % c->n_group || c->k > c->E || c->k > 256) return -1;
    if (!tokens) n = c->T;
#pragma omp parallel for schedule(dynamic, 4)
    for (int ti = 0; ti < n; ti++) {
        int t = tokens ? tokens[ti] : ti;
        int id[256];
        double g = route_token(c, x, Wr, bias, lbias, t, id, w + (int64_t)t * c->k,
                               logits ? logits + (int64_t)t * c->E : NULL,
                               probs ? probs + (int64_t)t * c->E : NULL);
        for (int j = 0; j < c->k; j++) idx[(int64_t)t * c->k + j] = id[j];
        if (gap) gap[t] = g;
    }
    return 0;
}

/* Stable counting sort of the T*k (token, slot) pairs by expert. */
int orc_dispatch(const orc_cfg *c, const int32_t *idx, int32_t *counts, int32_t *offsets,
                 int32_t *perm, int32_t *inv_perm)
{
    const int T = c->T, E = c->E, k = c->k;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int64_t i = 0; i < (int64_t)T * k; i++) {
        if (idx[i] < 0 || idx[i] >= E) return -1;
        counts[idx[i]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * E);
    memcpy(fill, offsets, sizeof(int32_t) * E);
    for (int t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int64_t s = (int64_t)t * k + j;
            int32_t pos = fill[idx[s]]++;
            perm[pos] = (int32_t)s;
            inv_perm[s] = pos;
        }
    free(fill);
    return 0;
}

/* ---------------------------------------------------------------- experts */

typedef struct {
    const void *x, *Wr, *bias, *lbias, *Wgu, *Wdn, *Wgu_s, *Wdn_s, *dy;
    /* MXFP8 backward: the weight copies quantised along the data-gradient
     * contraction axis (same layouts as Wgu, Wdn, Wgu_s, Wdn_s) */
    const void *Wgu_b, *Wdn_b, *Wgu_sb, *Wdn_sb;
} orc_inputs;

/* the weights of slot j of a token: routed expert idx[j] for j < k, shared
 * expert j-k otherwise (Wgu_b, Wdn_b: the MXFP8 backward's copies) */
typedef struct { const void *Wgu, *Wdn, *Wgu_b, *Wdn_b; int64_t gu_off, dn_off; int I; } slot_w;

static slot_w slot_weights(const orc_cfg *c, const orc_inputs *in, int e_or_shared, int shared)
{
    slot_w s;
    if (!shared) {
        s.Wgu = in->Wgu; s.Wdn = in->Wdn; s.I = c->I;
        s.Wgu_b = in->Wgu_b; s.Wdn_b = in->Wdn_b;
        s.gu_off = (int64_t)e_or_shared * 2 * c->I * c->H;
        s.dn_off = (int64_t)e_or_shared * c->H * c->I;
    } else {
        s.Wgu = in->Wgu_s; s.Wdn = in->Wdn_s; s.I = c->Is;
        s.Wgu_b = in->Wgu_sb; s.Wdn_b = in->Wdn_sb;
        s.gu_off = (int64_t)e_or_shared * 2 * c->Is * c->H;
        s.dn_off = (int64_t)e_or_shared * c->H * c->Is;
    }
    return s;
}

/* x row of token t as doubles (MX-quantised in MXFP8 mode) */
static void load_x(const orc_cfg *c, const void *x, int t, double *xd)
{
    for (int h = 0; h < c->H; h++) xd[h] = ld(x, (int64_t)t * c->H + h, c->act_kind);
    if (c->mx)
        for (int b = 0; b < c->H; b += 32) mx_block(xd + b, 32, NULL, NULL);
}

/* gate/up pre-activations g, u [I] of one (token, expert) pair */
static void gate_up(const orc_cfg *c, const slot_w *s, const double *xd, double *g, double *u)
{
    const int H = c->H;
    for (int i = 0; i < s->I; i++) {
        double a = 0.0, b = 0.0;
        for (int h = 0; h < H; h++) {
            a += xd[h] * ld(s->Wgu, s->gu_off + (int64_t)i * H + h, c->w_kind);
            b += xd[h] * ld(s->Wgu, s->gu_off + (int64_t)(s->I + i) * H + h, c->w_kind);
        }
        g[i] = a;
        u[i] = b;
    }
}

static inline double silu(double g) { return g / (1.0 + exp(-g)); }

/* h = silu(g) * u with the stored-h mirror (bf16, or MX blocks along I) */
static void swiglu_h(const orc_cfg *c, const double *g, const double *u, int I, double *h)
{
    for (int i = 0; i < I; i++) h[i] = silu(g[i]) * u[i];
    if (c->mx) {
        for (int b = 0; b < I; b += 32) mx_block(h + b, 32, NULL, NULL);
    } else {
        for (int i = 0; i < I; i++) h[i] = mirror(c, h[i]);
    }
}

/* o = h Wd^T (the per-(token, slot) rows are stored in fp32: no bf16 mirror) */
static void down(const orc_cfg *c, const slot_w *s, const double *h, double *o)
{
    for (int n = 0; n < c->H; n++) {
        double a = 0.0;
        for (int i = 0; i < s->I; i++) a += h[i] * ld(s->Wdn, s->dn_off + (int64_t)n * s->I + i, c->w_kind);
        o[n] = a;
    }
}

/* Forward of n tokens.  idx/w: routing of all T tokens (from orc_route).
 * y: [n, H]; O: [n, k+S, H] or NULL; h: [n, k+S, max(I,Is)] or NULL. */
int orc_fwd_tokens(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const double *w,
                   const int32_t *tokens, int n, double *y, double *O, double *hout)
{
    const int H = c->H, k = c->k, kk = c->k + c->S;
    const int Im = c->I > c->Is ? c->I : c->Is;
#pragma omp parallel for schedule(dynamic, 1)
    for (int ti = 0; ti < n; ti++) {
        int t = tokens[ti];
        double *xd = (double *)malloc(sizeof(double) * (H * 2 + Im * 3));
        double *acc = xd + H, *g = acc + H, *u = g + Im, *h = u + Im;
        double *o = (double *)malloc(sizeof(double) * H);
        load_x(c, in->x, t, xd);
        for (int n2 = 0; n2 < H; n2++) acc[n2] = 0.0;
        for (int j = 0; j < kk; j++) {
            int shared = j >= k;
            slot_w s = slot_weights(c, in, shared ? j - k : idx[(int64_t)t * k + j], shared);
            double wj = shared ? 1.0 : w[(int64_t)t * k + j];
            gate_up(c, &s, xd, g, u);
            swiglu_h(c, g, u, s.I, h);
            down(c, &s, h, o);
            for (int n2 = 0; n2 < H; n2++) acc[n2] += wj * o[n2];
            if (O) memcpy(O + ((int64_t)ti * kk + j) * H, o, sizeof(double) * H);
            if (hout) memcpy(hout + ((int64_t)ti * kk + j) * Im, h, sizeof(double) * s.I);
        }
        for (int n2 = 0; n2 < H; n2++) y[(int64_t)ti * H + n2] = mirror(c, acc[n2]);
        free(o);
        free(xd);
    }
    return 0;
}

/* MXFP8 mode: the quantised h of each (token, slot) of n tokens, as the down
 * projection reads it.  hraw: [n, k+S, max(I,Is)] the unrounded h = silu(g) u
 * (fp64); hq: e4m3 codes, same shape; hs: [n, k+S, max(I,Is)/32] ue8m0 scale
 * bytes.  Any output may be NULL. */
int orc_h_mx(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const int32_t *tokens, int n,
             double *hraw, uint8_t *hq, uint8_t *hs)
{
    const int H = c->H, k = c->k, kk = c->k + c->S;
    const int Im = c->I > c->Is ? c->I : c->Is;
    if (!c->mx || (c->I % 32) || (c->S && (c->Is % 32))) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int ti = 0; ti < n; ti++) {
        int t = tokens[ti];
        double *xd = (double *)malloc(sizeof(double) * (H + 3 * Im));
        double *g = xd + H, *u = g + Im, *h = u + Im;
        load_x(c, in->x, t, xd);
        for (int j = 0; j < kk; j++) {
            int shared = j >= k;
            slot_w s = slot_weights(c, in, shared ? j - k : idx[(int64_t)t * k + j], shared);
            gate_up(c, &s, xd, g, u);
            for (int i = 0; i < s.I; i++) h[i] = silu(g[i]) * u[i];
            int64_t row = (int64_t)ti * kk + j;
            if (hraw) memcpy(hraw + row * Im, h, sizeof(double) * s.I);
            for (int b = 0; b < s.I; b += 32)
                mx_block(h + b, 32, hq ? hq + row * Im + b : NULL, hs ? hs + row * (Im / 32) + b / 32 : NULL);
        }
        free(xd);
    }
    return 0;
}

/* ---------------------------------------------------------------- backward */

/* d loss / d logits of the k selected experts of token t, given G_j = <dy, o_j>.
 * Softmax: w_j = rho q_j with q the softmax over the selected logits, so
 *   dl_j = w_j (G_j - sum_i q_i G_i).
 * Sigmoid: w_j = rho s_j / S with S = sum of selected s, so
 *   ds_j = rho/S (G_j - sum_i (s_i/S) G_i),  dl_j = ds_j s_j (1 - s_j). */
static void dlogits_token(const orc_cfg *c, const double *prob, const int *idx, const double *w,
                          const double *G, double *dl)
{
    const int k = c->k;
    const double rho = c->routed_scale;
    double gbar = 0.0;
    for (int j = 0; j < k; j++) gbar += (w[j] / rho) * G[j];
    if (c->score_fn == 0) {
        for (int j = 0; j < k; j++) dl[j] = w[j] * (G[j] - gbar);
    } else {
        double S = 0.0;
        for (int j = 0; j < k; j++) S += prob[idx[j]];
        for (int j = 0; j < k; j++) {
            double s = prob[idx[j]];
            dl[j] = rho / S * (G[j] - gbar) * s * (1.0 - s);
        }
    }
}

/* SwiGLU backward of one row: dh given, g/u as stored (mirrored to bf16).
 * dg = dh u sig(g) (1 + g (1 - sig(g))), du = dh silu(g); both stored bf16.
 * raw (or NULL): the same two halves before the bf16 mirror. */
static void swiglu_bwd(const orc_cfg *c, const double *g, const double *u, const double *dh, int I,
                       double *dgu, double *raw)
{
    for (int i = 0; i < I; i++) {
        double gb = mirror(c, g[i]), ub = mirror(c, u[i]);
        double sg = 1.0 / (1.0 + exp(-gb));
        double dg = dh[i] * ub * sg * (1.0 + gb * (1.0 - sg)), du = dh[i] * gb * sg;
        dgu[i] = mirror(c, dg);
        dgu[I + i] = mirror(c, du);
        if (raw) { raw[i] = dg; raw[I + i] = du; }
    }
}

/* dh = dO Wd where dO = wj dy (row of H) */
static void down_dgrad(const orc_cfg *c, const slot_w *s, const double *dO, double *dh)
{
    for (int i = 0; i < s->I; i++) dh[i] = 0.0;
    for (int n = 0; n < c->H; n++) {
        double d = dO[n];
        for (int i = 0; i < s->I; i++) dh[i] += d * ld(s->Wdn, s->dn_off + (int64_t)n * s->I + i, c->w_kind);
    }
}

/* MXFP8 backward: a = Q(dy) W_down with the copy quantised along H (dyq is the
 * row already quantised per 1x32 block) */
static void down_dgrad_mx(const orc_cfg *c, const slot_w *s, const double *dyq, double *a)
{
    for (int i = 0; i < s->I; i++) a[i] = 0.0;
    for (int n = 0; n < c->H; n++) {
        double d = dyq[n];
        for (int i = 0; i < s->I; i++) a[i] += d * ld(s->Wdn_b, s->dn_off + (int64_t)n * s->I + i, c->w_kind);
    }
}

/* dy row of token t: dyd as stored (bf16), dyq quantised per 1x32 block along H
 * in MXFP8 mode (the operand of the MXFP8 down dgrad), else a copy */
static void load_dy(const orc_cfg *c, const void *dy, int t, double *dyd, double *dyq)
{
    for (int q = 0; q < c->H; q++) dyd[q] = dyq[q] = ld(dy, (int64_t)t * c->H + q, c->act_kind);
    if (c->mx)
        for (int b = 0; b < c->H; b += 32) mx_block(dyq + b, 32, NULL, NULL);
}

/* MXFP8 backward inputs present (the weight copies of the data gradients) */
static int mx_bwd_ready(const orc_cfg *c, const orc_inputs *in)
{
    if (!c->mx) return 1;
    if (c->I % 32 || !in->Wgu_b || !in->Wdn_b) return 0;
    if (c->S && (c->Is % 32 || !in->Wgu_sb || !in->Wdn_sb)) return 0;
    return 1;
}

/* One slot's data gradients.  h: the slot's h as the forward stored it (for G);
 * dyd/dyq: the token's dy row (as stored / quantised); wj: routing weight.
 * Writes dgu [2I] (stored bf16 values), the per-slot dx row dxs [H] (fp32 on the
 * layer: unrounded) and, when G is given, G = <dy, o_j> (BF16: o_j = h Wd^T;
 * MXFP8: <Q(dy) Wd, Q(h)> from the quantised product, the fused epilogue's value). */
static void slot_backward(const orc_cfg *c, const slot_w *s, const double *g, const double *u, const double *h,
                          const double *dyd, const double *dyq, double wj, double *dh, double *dgu,
                          double *raw, double *dxs, double *G)
{
    const int H = c->H, I = s->I;
    if (!c->mx) {
        if (G) {
            double a = 0.0;
            for (int n = 0; n < H; n++) {
                double o = 0.0;
                for (int i = 0; i < I; i++) o += h[i] * ld(s->Wdn, s->dn_off + (int64_t)n * I + i, c->w_kind);
                a += dyd[n] * o;
            }
            *G = a;
        }
        for (int q = 0; q < H; q++) dxs[q] = wj * dyd[q];          /* dO, reused as scratch */
        down_dgrad(c, s, dxs, dh);
    } else {
        down_dgrad_mx(c, s, dyq, dh);
        if (G) {
            double a = 0.0;
            for (int i = 0; i < I; i++) a += dh[i] * h[i];
            *G = a;
        }
        for (int i = 0; i < I; i++) dh[i] *= wj;
    }
    swiglu_bwd(c, g, u, dh, I, dgu, raw);
    const void *Wg = c->mx ? s->Wgu_b : s->Wgu;
    const double *op = dgu;
    if (c->mx) {                                   /* Q(dGU) per 1x32 block of each half */
        for (int b = 0; b < 2 * I; b += 32) mx_block(raw + b, 32, NULL, NULL);
        op = raw;
    }
    for (int q = 0; q < H; q++) {
        double a = 0.0;
        for (int i = 0; i < 2 * I; i++) a += op[i] * ld(Wg, s->gu_off + (int64_t)i * H + q, c->w_kind);
        dxs[q] = a;
    }
}

/* per-token backward: dx [n, H], dlogit [n, k], G [n, k] (any may be NULL but dx) */
int orc_bwd_tokens(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const double *w,
                   const int32_t *tokens, int n, double *dx, double *dlogit, double *Gout)
{
    const int H = c->H, k = c->k, kk = c->k + c->S, E = c->E;
    const int Im = c->I > c->Is ? c->I : c->Is;
    if (!mx_bwd_ready(c, in)) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int ti = 0; ti < n; ti++) {
        int t = tokens[ti];
        double *xd = (double *)malloc(sizeof(double) * (5 * H + 8 * Im + 2 * E + 2 * k));
        double *dyd = xd + H, *dyq = dyd + H, *acc = dyq + H, *dxs = acc + H;
        double *g = dxs + H, *u = g + Im, *h = u + Im, *dh = h + Im, *dgu = dh + Im, *raw = dgu + 2 * Im;
        double *lgt = raw + 2 * Im, *prob = lgt + E, *G = prob + E, *dl = G + k;
        int id[256];
        double ww[256];
        load_x(c, in->x, t, xd);
        load_dy(c, in->dy, t, dyd, dyq);
        for (int q = 0; q < H; q++) acc[q] = 0.0;
        route_token(c, in->x, in->Wr, in->bias, in->lbias, t, id, ww, lgt, prob);
        for (int j = 0; j < k; j++) {
            id[j] = idx[(int64_t)t * k + j];
            ww[j] = w[(int64_t)t * k + j];
        }
        for (int j = 0; j < kk; j++) {
            int shared = j >= k;
            slot_w s = slot_weights(c, in, shared ? j - k : id[j], shared);
            double wj = shared ? 1.0 : ww[j];
            gate_up(c, &s, xd, g, u);
            swiglu_h(c, g, u, s.I, h);
            slot_backward(c, &s, g, u, h, dyd, dyq, wj, dh, dgu, raw, dxs, shared ? NULL : &G[j]);
            for (int q = 0; q < H; q++) acc[q] += dxs[q];     /* per-slot dx rows are stored in fp32 */
        }
        dlogits_token(c, prob, id, ww, G, dl);
        for (int q = 0; q < H; q++) {
            double r = 0.0;
            for (int j = 0; j < k; j++) r += dl[j] * ld(in->Wr, (int64_t)id[j] * H + q, c->r_kind);
            dx[(int64_t)ti * H + q] = mirror(c, acc[q] + r);
        }
        if (dlogit) for (int j = 0; j < k; j++) dlogit[(int64_t)ti * k + j] = dl[j];
        if (Gout) for (int j = 0; j < k; j++) Gout[(int64_t)ti * k + j] = G[j];
        free(xd);
    }
    return 0;
}

/* Router weight gradient rows: dWr[e, :] = sum over tokens t routed to e
 * (ascending t) of dlogit[t, e] x[t, :].  experts: list of ne experts; out [ne, H]
 * (fp32 output on the layer, so no bf16 mirror). */
int orc_drouter(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const double *w,
                const int32_t *experts, int ne, double *out)
{
    const int T = c->T, H = c->H, k = c->k;
    for (int ei = 0; ei < ne; ei++) {
        int e = experts[ei];
        int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (T + 1));
        int32_t *slot = (int32_t *)malloc(sizeof(int32_t) * (T + 1));
        int n = 0;
        for (int t = 0; t < T; t++)
            for (int j = 0; j < k; j++)
                if (idx[(int64_t)t * k + j] == e) { tok[n] = t; slot[n] = j; n++; }
        double *dxs = (double *)malloc(sizeof(double) * ((int64_t)n * H + 1));
        double *dl = (double *)malloc(sizeof(double) * ((int64_t)n * k + 1));
        if (n) orc_bwd_tokens(c, in, idx, w, tok, n, dxs, dl, NULL);
        for (int q = 0; q < H; q++) {
            double a = 0.0;
            for (int r = 0; r < n; r++)
                a += dl[(int64_t)r * k + slot[r]] * ld(in->x, (int64_t)tok[r] * H + q, c->act_kind);
            out[(int64_t)ei * H + q] = a;
        }
        free(tok); free(slot); free(dxs); free(dl);
    }
    return 0;
}

/* Rows of one group: routed expert e (rows = tokens routed to e, ascending,
 * weights w) or shared expert s (all tokens, weight 1). */
static int group_rows(const orc_cfg *c, const int32_t *idx, const double *w, int grp, int shared,
                      int32_t *tok, double *wr)
{
    int n = 0;
    for (int t = 0; t < c->T; t++) {
        if (shared) { tok[n] = t; wr[n] = 1.0; n++; continue; }
        for (int j = 0; j < c->k; j++)
            if (idx[(int64_t)t * c->k + j] == grp) { tok[n] = t; wr[n] = w[(int64_t)t * c->k + j]; n++; }
    }
    return n;
}

/* Selected entries of one group's weight gradients.
 *   which = 0: dW_gate_up[n, q] = sum_r dGU_r[n] x[tok_r, q]          (n < 2I)
 *   which = 1: dW_down[q, i]    = sum_r dy[tok_r, q] hw_r[i],  hw = bf16(w_r h_r)
 * Rows r ascending in token.  rows/cols: ne entry coordinates; out: ne values
 * (bf16-mirrored like the layer's outputs).  MXFP8 mode: x and h as the forward
 * quantised them, dGU from the MXFP8 down dgrad (Q(dy) with the copy of W_down
 * quantised along H). */
int orc_dw_entries(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const double *w,
                   int grp, int shared, int which, const int32_t *rows, const int32_t *cols, int ne,
                   double *out)
{
    const int H = c->H;
    if (!mx_bwd_ready(c, in)) return -1;
    slot_w s = slot_weights(c, in, grp, shared);
    const int I = s.I;
    int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (c->T + 1));
    double *wr = (double *)malloc(sizeof(double) * (c->T + 1));
    int m = group_rows(c, idx, w, grp, shared, tok, wr);
    /* the per-row scalars each entry needs, over all rows of the group */
#pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < ne; q++) {
        int a = rows[q], b = cols[q];
        int i = which == 0 ? (a % I) : b;            /* the inter index involved */
        int i0 = c->mx ? i / 32 * 32 : i, nb = c->mx ? 32 : 1;   /* MX: the whole block of i */
        double sum = 0.0;
        double *xd = (double *)malloc(sizeof(double) * (3 * H + 64));
        double *dyd = xd + H, *dyq = dyd + H, *hb = dyq + H;
        for (int r = 0; r < m; r++) {
            int t = tok[r];
            load_x(c, in->x, t, xd);
            double g = 0.0, u = 0.0;
            for (int v = 0; v < nb; v++) {
                int iv = i0 + v;
                double gv = 0.0, uv = 0.0;
                for (int h = 0; h < H; h++) {
                    gv += xd[h] * ld(s.Wgu, s.gu_off + (int64_t)iv * H + h, c->w_kind);
                    uv += xd[h] * ld(s.Wgu, s.gu_off + (int64_t)(I + iv) * H + h, c->w_kind);
                }
                hb[v] = silu(gv) * uv;
                if (iv == i) { g = gv; u = uv; }
            }
            if (which == 1) {
                double hh;
                if (c->mx) {
                    mx_block(hb, 32, NULL, NULL);
                    hh = hb[i - i0];
                } else {
                    hh = mirror(c, hb[0]);
                }
                double hw = mirror(c, wr[r] * hh);
                sum += ld(in->dy, (int64_t)t * H + a, c->act_kind) * hw;
            } else {
                double dh = 0.0;
                if (c->mx) {
                    load_dy(c, in->dy, t, dyd, dyq);
                    for (int n = 0; n < H; n++) dh += dyq[n] * ld(s.Wdn_b, s.dn_off + (int64_t)n * I + i, c->w_kind);
                    dh *= wr[r];
                } else {
                    for (int n = 0; n < H; n++)
                        dh += wr[r] * ld(in->dy, (int64_t)t * H + n, c->act_kind) *
                              ld(s.Wdn, s.dn_off + (int64_t)n * I + i, c->w_kind);
                }
                double gb = mirror(c, g), ub = mirror(c, u);
                double sg = 1.0 / (1.0 + exp(-gb));
                double d = a < I ? dh * ub * sg * (1.0 + gb * (1.0 - sg)) : dh * gb * sg;
                sum += mirror(c, d) * xd[b];
            }
        }
        out[q] = mirror(c, sum);
        free(xd);
    }
    free(tok);
    free(wr);
    return m;
}

/* Full weight gradients of one group (small shapes): dWgu [2I, H], dWdn [H, I]. */
int orc_dw_full(const orc_cfg *c, const orc_inputs *in, const int32_t *idx, const double *w, int grp,
                int shared, double *dWgu, double *dWdn)
{
    const int H = c->H;
    if (!mx_bwd_ready(c, in)) return -1;
    slot_w s = slot_weights(c, in, grp, shared);
    const int I = s.I;
    int32_t *tok = (int32_t *)malloc(sizeof(int32_t) * (c->T + 1));
    double *wr = (double *)malloc(sizeof(double) * (c->T + 1));
    int m = group_rows(c, idx, w, grp, shared, tok, wr);
    double *X = (double *)malloc(sizeof(double) * ((int64_t)m * H + 1));
    double *DGU = (double *)malloc(sizeof(double) * ((int64_t)m * 2 * I + 1));
    double *HW = (double *)malloc(sizeof(double) * ((int64_t)m * I + 1));
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < m; r++) {
        double *g = (double *)malloc(sizeof(double) * (4 * I + 3 * H));
        double *u = g + I, *h = u + I, *dh = h + I, *dyd = dh + I, *dyq = dyd + H, *dO = dyq + H;
        int t = tok[r];
        load_x(c, in->x, t, X + (int64_t)r * H);
        gate_up(c, &s, X + (int64_t)r * H, g, u);
        swiglu_h(c, g, u, I, h);                  /* stored h: bf16, or MX blocks */
        for (int i = 0; i < I; i++) HW[(int64_t)r * I + i] = mirror(c, wr[r] * h[i]);
        load_dy(c, in->dy, t, dyd, dyq);
        if (c->mx) {
            down_dgrad_mx(c, &s, dyq, dh);
            for (int i = 0; i < I; i++) dh[i] *= wr[r];
        } else {
            for (int q = 0; q < H; q++) dO[q] = wr[r] * dyd[q];
            down_dgrad(c, &s, dO, dh);
        }
        swiglu_bwd(c, g, u, dh, I, DGU + (int64_t)r * 2 * I, NULL);
        free(g);
    }
#pragma omp parallel for schedule(static)
    for (int n = 0; n < 2 * I; n++)
        for (int q = 0; q < H; q++) {
            double a = 0.0;
            for (int r = 0; r < m; r++) a += DGU[(int64_t)r * 2 * I + n] * X[(int64_t)r * H + q];
            dWgu[(int64_t)n * H + q] = mirror(c, a);
        }
#pragma omp parallel for schedule(static)
    for (int q = 0; q < H; q++)
        for (int i = 0; i < I; i++) {
            double a = 0.0;
            for (int r = 0; r < m; r++) a += ld(in->dy, (int64_t)tok[r] * H + q, c->act_kind) * HW[(int64_t)r * I + i];
            dWdn[(int64_t)q * I + i] = mirror(c, a);
        }
    free(tok); free(wr); free(X); free(DGU); free(HW);
    return m;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
