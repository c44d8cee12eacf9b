/*
 * mmoe_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow CPU oracle of the fused MoE feed-forward layer of
 * "MobileMoE: Scaling On-Device Mixture of Experts" (paper-archivist reading,
 * section "MoE preliminaries and three design factors", Eq. (*)):
 *
 *     y = sum_{i in Top-k} router_i(x) * FFN_i(x) + FFN^(s)(x)
 *
 * with 60 fine-grained routed SwiGLU experts, top-4 and one always-on shared
 * expert (same page, "Finding 3" and "final MobileMoE architecture"), an FP32
 * router ("MoE training stability techniques": all router computation in FP32),
 * symmetric group-32 INT4 weights (Eq. (6), section "QAT") and dynamic
 * per-token INT8 activations (same section).
 *
 * It computes the plain definition token by token: no permutation, no tiling,
 * no fusion.  Only tests/, the package's smoke() entry and the CPU-baseline leg
 * of bench.py may load it.  It shares no code with the CUDA library.
 *
 * Precision choices (the pages fix INT4 / INT8 / FP32-router and nothing
 * more; where a float decides an integer both implementations decide in FP32):
 *   - router logits: exact FP32 products summed in FP64, rounded to FP32,
 *     then the bias added in FP32; softmax in FP64, rounded to FP32;
 *   - quantisation divisions are IEEE FP32 divisions, rounding is
 *     round-half-to-even (rintf in the default rounding mode);
 *   - INT8 x INT4 group partials are exact 32-bit integers;
 *   - promotion of the group partials: acc = fmaf((float)P_j, s_j, acc) for
 *     j ascending, then one FP32 multiply by the activation scale;
 *   - silu(g) = g / (1 + expf(-g)) in FP32;
 *   - combine: y = FFN_s, then y = y + gate_j * FFN_j for j = 0..k-1 (the
 *     product and the sum rounded separately).
 * Build with -ffp-contract=off so that no other multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GROUP 32

typedef struct {
    int64_t d;        /* d_model */
    int64_t h;        /* hidden size of a routed expert */
    int64_t hs;       /* hidden size of the shared expert */
    int64_t E;        /* routed experts (60) */
    int64_t k;        /* experts per token (4) */
    int64_t gating;   /* 0: softmax over E, no renormalisation; 1: sigmoid, top-k normalised;
                         2: as 1 with the bias added to the scores for the selection only */
    const float* w_router;     /* [d, E] row-major */
    const float* router_bias;  /* [E] or NULL */
    const uint8_t* w_gate_up;  /* expert g at byte g*2h*d/2: [2*hid][d/2], rows 0..hid-1 gate, then up */
    const float* s_gate_up;    /* expert g at g*2h*d/32:      [2*hid][d/32] */
    const uint8_t* w_down;     /* expert g at byte g*d*h/2:    [d][hid/2] */
    const float* s_down;       /* expert g at g*d*h/32:        [d][hid/32] */
} oracle_layer;

/* Optional per-stage outputs; every pointer may be NULL.  "slot" s in [0, k]
 * is the s-th selected expert of a token, slot k is the shared expert.
 * hmax = max(h, hs). */
typedef struct {
    float* logits;   /* [T, E] */
    float* probs;    /* [T, E] */
    int32_t* idx;    /* [T, k] */
    float* gate;     /* [T, k] */
    int8_t* xq;      /* [T, d] */
    float* sx;       /* [T] */
    int32_t* pg;     /* [T, k+1, hmax, d/32] gate group partials */
    int32_t* pu;     /* [T, k+1, hmax, d/32] up group partials */
    int8_t* hq;      /* [T, k+1, hmax] */
    float* sh;       /* [T, k+1] */
    int32_t* pd;     /* [T, k+1, d, hmax/32] down group partials */
    float* o;        /* [T, k+1, d] expert outputs (before gating) */
} oracle_dumps;

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Signed 4-bit value k of a packed row (two per byte, low nibble = even index). */
static int int4_at(const uint8_t* row, int64_t k)
{
    int v = (row[k >> 1] >> ((k & 1) * 4)) & 15;
    return v >= 8 ? v - 16 : v;
}

/* ---------------------------------------------------------------------------
 * Eq. (6), section "QAT": symmetric group quantisation with b = 4 bits,
 * group size 32 along K, s_g = 2 max|W_g| / (2^b - 1),
 * q = clamp(round(W / s_g), -2^(b-1), 2^(b-1) - 1).
 * An all-zero group gets s = 0 and q = 0.
 * W is [rows, K] row-major; packed is [rows, K/2]; scales is [rows, K/32].
 * ------------------------------------------------------------------------- */
int oracle_quantize_int4(const float* W, int64_t rows, int64_t K, uint8_t* packed, float* scales)
{
    if (K % ORACLE_GROUP) return -1;
    int64_t ng = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* w = W + r * K;
        uint8_t* p = packed + r * (K / 2);
        memset(p, 0, (size_t)(K / 2));
        for (int64_t j = 0; j < ng; ++j) {
            float m = 0.0f;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                float a = fabsf(w[j * ORACLE_GROUP + i]);
                if (a > m) m = a;
            }
            float s = (2.0f * m) / 15.0f;
            scales[r * ng + j] = s;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                int64_t kk = j * ORACLE_GROUP + i;
                int q = 0;
                if (s > 0.0f) {
                    float v = rintf(w[kk] / s);
                    q = v > 7.0f ? 7 : (v < -8.0f ? -8 : (int)v);
                }
                p[kk >> 1] |= (uint8_t)((q & 15) << ((kk & 1) * 4));
            }
        }
    }
    return 0;
}

/* Dynamic per-token INT8 activation quantisation (section "QAT": activations
 * quantised to INT8 on the fly; the benchmark table fixes s = absmax / 127).
 * Codes are symmetric in [-127, 127]; an all-zero row gets s = 0, codes 0. */
static void quantize_row_int8_f32(const float* a, int64_t n, int8_t* q, float* s_out)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(a[i]);
        if (v > m) m = v;
    }
    float s = m / 127.0f;
    *s_out = s;
    for (int64_t i = 0; i < n; ++i) {
        int c = 0;
        if (s > 0.0f) {
            float v = rintf(a[i] / s);
            c = v > 127.0f ? 127 : (v < -127.0f ? -127 : (int)v);
        }
        q[i] = (int8_t)c;
    }
}

int oracle_quantize_act(const uint16_t* x, int64_t T, int64_t d, int8_t* xq, float* sx)
{
    float* row = (float*)malloc((size_t)d * sizeof(float));
    if (!row) return -1;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < d; ++i) row[i] = bf16_to_f32(x[t * d + i]);
        quantize_row_int8_f32(row, d, xq + t * d, sx + t);
    }
    free(row);
    return 0;
}

/* ---------------------------------------------------------------------------
 * FP32 router of one token ("MoE training stability techniques": router in
 * FP32; Eq. (*): top-k by router score).
 *   gating 0: l_e = fp32( sum_i x_i * W_r[i, e] ) + b_e,
 *             p = softmax over all E, gate_j = p[idx_j] (no renormalisation),
 *             idx = the k largest l_e;
 *   gating 1: l_e as for gating 0, p_e = sigmoid(l_e),
 *             gate_j = p[idx_j] / sum_j' p[idx_j'], idx = the k largest l_e;
 *   gating 2: the auxiliary-loss-free balancing bias ("MoE training stability
 *             techniques": a per-expert bias, adjusted from the load
 *             imbalance, with no extra loss): l_e = fp32( sum_i x_i W_r[i, e] )
 *             without the bias, p_e = sigmoid(l_e), idx = the k largest of the
 *             FP32 sums p_e + b_e, gate_j = p[idx_j] / sum_j' p[idx_j'] -- the
 *             bias moves the selection but never enters a gate.
 * Among equal keys the lower expert index comes first.
 * ------------------------------------------------------------------------- */
static void router_token(const oracle_layer* L, const float* xf, float* logits, float* probs,
                         int32_t* idx, float* gate)
{
    const int64_t d = L->d, E = L->E, k = L->k;
    float key[64];
    for (int64_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += (double)xf[i] * (double)L->w_router[i * E + e];
        float l = (float)acc;
        if (L->router_bias && L->gating != 2) l = l + L->router_bias[e];
        logits[e] = l;
    }
    if (L->gating == 0) {
        double mx = logits[0];
        for (int64_t e = 1; e < E; ++e)
            if (logits[e] > mx) mx = logits[e];
        double sum = 0.0;
        for (int64_t e = 0; e < E; ++e) sum += exp((double)logits[e] - mx);
        for (int64_t e = 0; e < E; ++e) probs[e] = (float)(exp((double)logits[e] - mx) / sum);
    } else {
        for (int64_t e = 0; e < E; ++e) probs[e] = (float)(1.0 / (1.0 + exp(-(double)logits[e])));
    }
    for (int64_t e = 0; e < E; ++e)
        key[e] = L->gating == 2 ? (L->router_bias ? probs[e] + L->router_bias[e] : probs[e]) : logits[e];
    for (int64_t j = 0; j < k; ++j) {
        int64_t best = -1;
        for (int64_t e = 0; e < E; ++e) {
            int taken = 0;
            for (int64_t jj = 0; jj < j; ++jj)
                if (idx[jj] == e) taken = 1;
            if (taken) continue;
            if (best < 0 || key[e] > key[best]) best = e;
        }
        idx[j] = (int32_t)best;
    }
    if (L->gating == 0) {
        for (int64_t j = 0; j < k; ++j) gate[j] = probs[idx[j]];
    } else {
        double s = 0.0;
        for (int64_t j = 0; j < k; ++j) s += (double)probs[idx[j]];
        for (int64_t j = 0; j < k; ++j) gate[j] = (float)((double)probs[idx[j]] / s);
    }
}

static int check_layer(const oracle_layer* L);

int oracle_router(const oracle_layer* L, const uint16_t* x, int64_t T, float* logits, float* probs,
                  int32_t* idx, float* gate)
{
    if (check_layer(L) || T < 0) return -1;
    int err = 0;
#pragma omp parallel reduction(| : err)
    {
        float* xf = (float*)malloc((size_t)L->d * sizeof(float));
        if (!xf) err |= 1;
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            if (!xf) continue;
            for (int64_t i = 0; i < L->d; ++i) xf[i] = bf16_to_f32(x[t * L->d + i]);
            router_token(L, xf, logits + t * L->E, probs + t * L->E, idx + t * L->k, gate + t * L->k);
        }
        free(xf);
    }
    return err ? -1 : 0;
}

/* Byte / element offsets of expert g's blocks (expert E is the shared one and
 * follows the E routed experts, so the same formula locates it). */
static int64_t hid_of(const oracle_layer* L, int64_t g) { return g < L->E ? L->h : L->hs; }
static const uint8_t* gu_w(const oracle_layer* L, int64_t g) { return L->w_gate_up + g * 2 * L->h * (L->d / 2); }
static const float* gu_s(const oracle_layer* L, int64_t g) { return L->s_gate_up + g * 2 * L->h * (L->d / ORACLE_GROUP); }
static const uint8_t* dn_w(const oracle_layer* L, int64_t g) { return L->w_down + g * L->d * (L->h / 2); }
static const float* dn_s(const oracle_layer* L, int64_t g) { return L->s_down + g * L->d * (L->h / ORACLE_GROUP); }

/* Exact INT32 partial of group j of (INT8 row) . (INT4 row). */
static int32_t group_partial(const int8_t* a, const uint8_t* wrow, int64_t j)
{
    int32_t p = 0;
    for (int i = 0; i < ORACLE_GROUP; ++i) {
        int64_t kk = j * ORACLE_GROUP + i;
        p += (int32_t)a[kk] * (int32_t)int4_at(wrow, kk);
    }
    return p;
}

/* Gate/up half of one SwiGLU expert ("base architecture": SwiGLU FFN;
 * "custom MoE kernel": gate and up projections, then the SwiGLU activation):
 *   g_n = s_x * sum_j s_gate[n, j] * P_gate[n, j],   u_n likewise,
 *   a_n = silu(g_n) * u_n,
 * then a is requantised per row to INT8 like the activations.
 * pg, pu (optional) receive [hid, d/32] partials. */
int oracle_expert_gate_up(const oracle_layer* L, int64_t g, const int8_t* xq, float sx, int32_t* pg,
                          int32_t* pu, int8_t* hq, float* sh)
{
    const int64_t d = L->d, hid = hid_of(L, g), ng = d / ORACLE_GROUP;
    const uint8_t* W = gu_w(L, g);
    const float* S = gu_s(L, g);
    float* a = (float*)malloc((size_t)hid * sizeof(float));
    if (!a) return -1;
    for (int64_t n = 0; n < hid; ++n) {
        const uint8_t* wg = W + n * (d / 2);
        const uint8_t* wu = W + (hid + n) * (d / 2);
        float ga = 0.0f, ua = 0.0f;
        for (int64_t j = 0; j < ng; ++j) {
            int32_t p_g = group_partial(xq, wg, j);
            int32_t p_u = group_partial(xq, wu, j);
            if (pg) pg[n * ng + j] = p_g;
            if (pu) pu[n * ng + j] = p_u;
            ga = fmaf((float)p_g, S[n * ng + j], ga);
            ua = fmaf((float)p_u, S[(hid + n) * ng + j], ua);
        }
        float gv = ga * sx;
        float uv = ua * sx;
        float silu = gv / (1.0f + expf(-gv));
        a[n] = silu * uv;
    }
    quantize_row_int8_f32(a, hid, hq, sh);
    free(a);
    return 0;
}

/* Down projection of one expert: o_m = s_h * sum_j s_down[m, j] * P_down[m, j].
 * pd (optional) receives [d, hid/32] partials. */
int oracle_expert_down(const oracle_layer* L, int64_t g, const int8_t* hq, float sh, int32_t* pd, float* o)
{
    const int64_t d = L->d, hid = hid_of(L, g), ng = hid / ORACLE_GROUP;
    const uint8_t* W = dn_w(L, g);
    const float* S = dn_s(L, g);
    for (int64_t m = 0; m < d; ++m) {
        const uint8_t* wr = W + m * (hid / 2);
        float acc = 0.0f;
        for (int64_t j = 0; j < ng; ++j) {
            int32_t p = group_partial(hq, wr, j);
            if (pd) pd[m * ng + j] = p;
            acc = fmaf((float)p, S[m * ng + j], acc);
        }
        o[m] = acc * sh;
    }
    return 0;
}

static int64_t hmax_of(const oracle_layer* L) { return L->h > L->hs ? L->h : L->hs; }

/* The whole layer for one token t (Eq. (*)). */
static int layer_token(const oracle_layer* L, const uint16_t* xrow, int64_t t, float* yrow,
                       const oracle_dumps* D)
{
    const int64_t d = L->d, E = L->E, k = L->k, hm = hmax_of(L);
    const int64_t slots = k + 1;
    int rc = -1;
    float* xf = (float*)malloc((size_t)d * sizeof(float));
    float* logits = (float*)malloc((size_t)E * sizeof(float));
    float* probs = (float*)malloc((size_t)E * sizeof(float));
    int32_t* idx = (int32_t*)malloc((size_t)k * sizeof(int32_t));
    float* gate = (float*)malloc((size_t)k * sizeof(float));
    int8_t* xq = (int8_t*)malloc((size_t)d);
    int8_t* hq = (int8_t*)malloc((size_t)hm);
    float* o = (float*)malloc((size_t)d * sizeof(float));
    if (!xf || !logits || !probs || !idx || !gate || !xq || !hq || !o) goto done;

    for (int64_t i = 0; i < d; ++i) xf[i] = bf16_to_f32(xrow[i]);
    router_token(L, xf, logits, probs, idx, gate);
    float sx;
    quantize_row_int8_f32(xf, d, xq, &sx);
    if (D) {
        if (D->logits) memcpy(D->logits + t * E, logits, (size_t)E * sizeof(float));
        if (D->probs) memcpy(D->probs + t * E, probs, (size_t)E * sizeof(float));
        if (D->idx) memcpy(D->idx + t * k, idx, (size_t)k * sizeof(int32_t));
        if (D->gate) memcpy(D->gate + t * k, gate, (size_t)k * sizeof(float));
        if (D->xq) memcpy(D->xq + t * d, xq, (size_t)d);
        if (D->sx) D->sx[t] = sx;
    }
    /* slot k, the shared expert, first: y = FFN_s(x); then slots j = 0..k-1:
     * y = y + gate_j * FFN_{idx_j}(x), in that order */
    for (int64_t step = 0; step <= k; ++step) {
        int64_t s = (step == 0) ? k : step - 1;
        int64_t g = (s == k) ? E : idx[s];
        int64_t hid = hid_of(L, g);
        int64_t base = t * slots + s;
        int32_t* pg = (D && D->pg) ? D->pg + base * hm * (d / ORACLE_GROUP) : NULL;
        int32_t* pu = (D && D->pu) ? D->pu + base * hm * (d / ORACLE_GROUP) : NULL;
        int32_t* pd = (D && D->pd) ? D->pd + base * d * (hm / ORACLE_GROUP) : NULL;
        float sh;
        if (oracle_expert_gate_up(L, g, xq, sx, pg, pu, hq, &sh)) goto done;
        if (oracle_expert_down(L, g, hq, sh, pd, o)) goto done;
        if (D) {
            if (D->hq) memcpy(D->hq + base * hm, hq, (size_t)hid);
            if (D->sh) D->sh[base] = sh;
            if (D->o) memcpy(D->o + base * d, o, (size_t)d * sizeof(float));
        }
        if (s == k) {
            for (int64_t m = 0; m < d; ++m) yrow[m] = o[m];
        } else {
            for (int64_t m = 0; m < d; ++m) {
                float prod = gate[s] * o[m];
                yrow[m] = yrow[m] + prod;
            }
        }
    }
    rc = 0;
done:
    free(xf); free(logits); free(probs); free(idx); free(gate); free(xq); free(hq); free(o);
    return rc;
}

static int check_layer(const oracle_layer* L)
{
    if (!L || L->d <= 0 || L->h <= 0 || L->hs <= 0 || L->E <= 0 || L->E > 64 || L->k <= 0 || L->k > L->E) return -1;
    if (L->d % ORACLE_GROUP || L->h % ORACLE_GROUP || L->hs % ORACLE_GROUP) return -1;
    if (L->gating < 0 || L->gating > 2) return -1;
    return 0;
}

/* y[T, d] for all tokens; threads (OpenMP, if built with it) split the tokens. */
int oracle_moe_layer(const oracle_layer* L, const uint16_t* x, int64_t T, float* y, const oracle_dumps* D)
{
    if (check_layer(L) || T < 0) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t t = 0; t < T; ++t) err |= layer_token(L, x + t * L->d, t, y + t * L->d, D) != 0;
    return err ? -1 : 0;
}

/* y rows for a list of token ids only (sampled checks of large inputs):
 * y_rows[i] = layer output of token toks[i]. */
int oracle_moe_tokens(const oracle_layer* L, const uint16_t* x, int64_t T, const int64_t* toks, int64_t n,
                      float* y_rows)
{
    if (check_layer(L)) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t i = 0; i < n; ++i) {
        if (toks[i] < 0 || toks[i] >= T) { err |= 1; continue; }
        err |= layer_token(L, x + toks[i] * L->d, 0, y_rows + i * L->d, NULL) != 0;
    }
    return err ? -1 : 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the following calls (the CPU baseline is timed on one core and on all of them). */
int oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
