/*
 * Float64 CPU oracle of the DeepSeekMoE feed-forward layer (noaux_tc routing).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library, and it is deliberately plain: single-threaded, no BLAS, no blocking,
 * no fast-math, every sum taken in float64 in index order.
 *
 * Inputs are the same stored bits the GPU reads: x and expert weights as bf16
 * (passed as uint16 bit patterns), router weight and correction bias as fp32.
 * Each is widened to double exactly.
 *
 * Sources for what is computed:
 *  - "DeepSeekV3.2-Tiered-Implementations" README, § Architecture: sigmoid
 *    routing with a per-expert correction bias (topk_method "noaux_tc"),
 *    group-based routing with n_group groups of which topk_group are kept,
 *    256 routed experts, top-8.
 *  - "The Evolving Transformer · 07 — DeepSeek V2 & V3", § 02 DeepSeekMoE and
 *    § 03 Shared Expert: router(x) -> (weights, indices); routed outputs are
 *    added with their weights; the shared expert runs for every token; the
 *    layer returns shared + routed.  § 06: the bias only steers selection
 *    (nudged by load); weights come from the unbiased score.
 *  - Points the pages leave open follow the DeepSeek-V3 noaux_tc definition:
 *    the group score is the sum of the two largest biased scores of the group;
 *    groups are contiguous blocks of E / n_group experts; experts of dropped
 *    groups are excluded from the top-k (not given a score of 0); the lower
 *    index wins ties; the weights are normalised (when norm_topk_prob) and then
 *    multiplied by routed_scaling_factor.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t hidden_size;
    int32_t n_routed_experts;
    int32_t num_experts_per_tok;
    int32_t n_group;
    int32_t topk_group;
    int32_t moe_intermediate_size;
    int32_t n_shared_experts;
    int32_t norm_topk_prob;
    double routed_scaling_factor;
} oracle_cfg;

static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* sigma(z) = 1 / (1 + e^-z), the router's score function. */
static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* silu(z) = z * sigma(z), the SwiGLU gate activation. */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* "a beats b": larger value wins; on equal values the lower index wins. */
static int beats(double va, int ia, double vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

/*
 * Route T tokens (steps 1-7 of the layer definition).
 *   idx    [T,k]  chosen experts, in descending biased score
 *   w      [T,k]  routing weights (unbiased sigmoid, normalised, scaled)
 *   margin [T]    min(group-score gap at the keep boundary,
 *                     biased-score gap at the top-k boundary); +inf if none
 *   scores [T,E]  optional: unbiased sigmoid scores
 * Returns 0, or -1 on an invalid configuration or allocation failure.
 */
int oracle_route(const oracle_cfg *c, int64_t T, const uint16_t *x, const float *router_w,
                 const float *e_bias, int32_t *idx, double *w, double *margin, double *scores)
{
    const int H = c->hidden_size, E = c->n_routed_experts, G = c->n_group;
    const int TG = c->topk_group, K = c->num_experts_per_tok;
    if (H <= 0 || E <= 0 || G <= 0 || E % G != 0 || TG < 1 || TG > G || K < 1 ||
        K > TG * (E / G))
        return -1;
    const int gsize = E / G;

    double *xs = malloc(sizeof(double) * H);
    double *s = malloc(sizeof(double) * E);
    double *b = malloc(sizeof(double) * E);
    double *gs = malloc(sizeof(double) * G);
    int *kept = malloc(sizeof(int) * G);
    int *taken = malloc(sizeof(int) * E);
    if (!xs || !s || !b || !gs || !kept || !taken) {
        free(xs); free(s); free(b); free(gs); free(kept); free(taken);
        return -1;
    }

    for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) xs[h] = widen_bf16(x[t * H + h]);

        /* 1-3: logits, sigmoid scores, biased scores. */
        for (int e = 0; e < E; ++e) {
            double l = 0.0;
            for (int h = 0; h < H; ++h) l += xs[h] * (double)router_w[(int64_t)e * H + h];
            s[e] = sigmoid(l);
            b[e] = s[e] + (double)e_bias[e];
            if (scores) scores[t * E + e] = s[e];
        }

        /* 4: group score = largest + second-largest biased score in the group
         * (a one-expert group scores its only member). */
        for (int g = 0; g < G; ++g) {
            int i1 = -1, i2 = -1;
            for (int e = g * gsize; e < (g + 1) * gsize; ++e) {
                if (i1 < 0 || beats(b[e], e, b[i1], i1)) { i2 = i1; i1 = e; }
                else if (i2 < 0 || beats(b[e], e, b[i2], i2)) { i2 = e; }
            }
            gs[g] = b[i1] + (i2 >= 0 ? b[i2] : 0.0);
        }

        /* 5: keep the topk_group best groups (repeated arg-max, lower g on ties). */
        for (int g = 0; g < G; ++g) kept[g] = 0;
        double last_kept_gs = 0.0;
        for (int r = 0; r < TG; ++r) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!kept[g] && (best < 0 || beats(gs[g], g, gs[best], best))) best = g;
            kept[best] = 1;
            last_kept_gs = gs[best];
        }
        double group_gap = INFINITY;
        for (int g = 0; g < G; ++g)
            if (!kept[g] && last_kept_gs - gs[g] < group_gap) group_gap = last_kept_gs - gs[g];

        /* 6: top-k experts among the kept groups only (others are excluded, not
         * zeroed), by repeated arg-max of the biased score, lower index on ties. */
        for (int e = 0; e < E; ++e) taken[e] = 0;
        double last_b = 0.0;
        for (int j = 0; j < K; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e] || !kept[e / gsize]) continue;
                if (best < 0 || beats(b[e], e, b[best], best)) best = e;
            }
            taken[best] = 1;
            idx[t * K + j] = best;
            last_b = b[best];
        }
        double expert_gap = INFINITY;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && kept[e / gsize] && last_b - b[e] < expert_gap)
                expert_gap = last_b - b[e];
        margin[t] = group_gap < expert_gap ? group_gap : expert_gap;

        /* 7: weights from the unbiased scores, normalised, then scaled. */
        double sum = 0.0;
        for (int j = 0; j < K; ++j) sum += s[idx[t * K + j]];
        for (int j = 0; j < K; ++j) {
            double wj = s[idx[t * K + j]];
            if (c->norm_topk_prob) wj = wj / sum;
            w[t * K + j] = wj * c->routed_scaling_factor;
        }
    }
    free(xs); free(s); free(b); free(gs); free(kept); free(taken);
    return 0;
}

/*
 * One SwiGLU expert, down(silu(gate x) * up x), over n rows.
 *   x  [n,H] bf16 bits; w_gate, w_up [I,H] and w_down [H,I] bf16 bits in the
 *   nn.Linear (out, in) layout; out [n,H] float64.
 * Returns 0, or -1 on allocation failure.
 */
int oracle_swiglu(int64_t n, int64_t H, int64_t I, const uint16_t *x, const uint16_t *w_gate,
                  const uint16_t *w_up, const uint16_t *w_down, double *out)
{
    double *xs = malloc(sizeof(double) * H);
    double *hmid = malloc(sizeof(double) * I);
    if (!xs || !hmid) { free(xs); free(hmid); return -1; }
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t h = 0; h < H; ++h) xs[h] = widen_bf16(x[r * H + h]);
        for (int64_t i = 0; i < I; ++i) {
            double u = 0.0, v = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                u += widen_bf16(w_gate[i * H + h]) * xs[h];
                v += widen_bf16(w_up[i * H + h]) * xs[h];
            }
            hmid[i] = silu(u) * v;
        }
        for (int64_t o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int64_t i = 0; i < I; ++i) acc += widen_bf16(w_down[o * I + i]) * hmid[i];
            out[r * H + o] = acc;
        }
    }
    free(xs); free(hmid);
    return 0;
}

/*
 * Auxiliary-loss-free bias update ("The Evolving Transformer · 07", § 06: the
 * per-expert bias is nudged down when the expert is overloaded and up when it
 * is underloaded; knlb.dev DeepSeek-V3 notes, § architecture).  Load of expert
 * e = number of the batch's (token, slot) pairs routed to e; the reference load
 * is the mean T*k/E.  The step is gamma: bias_e <- bias_e - gamma if load_e is
 * above the mean, + gamma if below, unchanged if equal.  The bias is fp32 state,
 * so the sum is rounded to fp32 (the float64 sum of two floats, rounded once).
 *   idx [T,k] chosen experts; bias [E] updated in place; load [E] (output).
 */
void oracle_bias_update(int64_t T, int32_t K, int32_t E, const int32_t *idx, float *bias, float gamma,
                        int64_t *load)
{
    for (int e = 0; e < E; ++e) load[e] = 0;
    for (int64_t q = 0; q < T * K; ++q) load[idx[q]] += 1;
    for (int e = 0; e < E; ++e) {
        /* load_e vs T*K/E compared exactly as load_e * E vs T * K */
        const int64_t lhs = load[e] * (int64_t)E, rhs = T * (int64_t)K;
        double step = 0.0;
        if (lhs > rhs) step = -(double)gamma;
        else if (lhs < rhs) step = (double)gamma;
        bias[e] = (float)((double)bias[e] + step);
    }
}

/*
 * MXFP8 quantisation ("DeepSeek-V3 notes" (knlb.dev), § fp8: fine-grained
 * block-wise quantisation, E4M3 throughout, scales derived online from the
 * block's maximum; "DeepSeekV3.2-Tiered-Implementations", § DeepGEMM: FP8 grouped
 * GEMM for the MoE experts).  Written from the format definitions:
 *
 *  - E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinities;
 *    normal values (1 + m/8) 2^(e-7) for e = 1..15 (e = 15, m = 7 is NaN), so the
 *    largest finite value is 448; subnormals (m/8) 2^-6, i.e. multiples of 2^-9.
 *  - One scale per block of 32 consecutive elements along the contraction axis,
 *    a power of two stored as an 8-bit biased exponent (scale = 2^(code - 127)).
 *
 * The scale of a block is the smallest power of two that brings its largest
 * magnitude within the E4M3 range, so no element saturates.
 */

/* Nearest E4M3 value to v, ties to the even significand.  |v| > 448 saturates to
 * 448 (the quantiser never produces such inputs).  NaN passes through. */
double oracle_e4m3_round(double v)
{
    if (v != v) return v;
    const double a = fabs(v);
    if (a == 0.0) return v;
    double step;
    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);                 /* subnormal spacing */
    } else {
        int p;
        frexp(a, &p);                          /* a in [2^(p-1), 2^p) */
        step = ldexp(1.0, (p - 1) - 3);        /* 3 mantissa bits */
    }
    double q = nearbyint(a / step) * step;     /* a / step is exact; default mode: ties to even */
    if (q > 448.0) q = 448.0;
    return v < 0 ? -q : q;
}

/* E4M3 bit pattern of a value already on the E4M3 grid (|q| <= 448). */
uint8_t oracle_e4m3_bits(double q)
{
    uint8_t sign = (q < 0 || (q == 0 && signbit(q))) ? 0x80 : 0x00;
    double a = fabs(q);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -6)) return sign | (uint8_t)(a / ldexp(1.0, -9));      /* exponent field 0 */
    int p;
    frexp(a, &p);
    const int e = (p - 1) + 7;                                                /* biased exponent */
    const int m = (int)(a / ldexp(1.0, p - 1) * 8.0) - 8;                      /* 0..7 */
    return sign | (uint8_t)(e << 3) | (uint8_t)m;
}

/* Scale code of a block whose largest magnitude is amax: 127 + e for the smallest
 * integer e with amax <= 448 * 2^e, clamped to [0, 254]; an all-zero block gets 0. */
int oracle_mx_scale_code(double amax)
{
    if (!(amax > 0.0)) return 0;
    int p;
    const double m = frexp(amax, &p);          /* amax = m 2^p, m in [0.5, 1); 448 = 0.875 * 2^9 */
    const int e = (m <= 0.875) ? p - 9 : p - 8;
    const int code = 127 + e;
    return code < 0 ? 0 : (code > 254 ? 254 : code);
}

/*
 * Quantise rows [rows, K] (K a multiple of 32) in blocks of 32 along K.
 *   q     [rows, K]    the E4M3 element values (on the E4M3 grid, unscaled)
 *   codes [rows, K/32] the blocks' scale codes
 *   deq   [rows, K]    q * 2^(code - 127), the value the GEMM multiplies with
 * Any output pointer may be NULL.
 */
void oracle_mx_quantize(int64_t rows, int64_t K, const double *src, double *q, uint8_t *codes,
                        double *deq)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < K / 32; ++b) {
            const double *v = src + r * K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i)
                if (fabs(v[i]) > amax) amax = fabs(v[i]);
            const int code = oracle_mx_scale_code(amax);
            const double scale = ldexp(1.0, code - 127);
            if (codes) codes[r * (K / 32) + b] = (uint8_t)code;
            for (int i = 0; i < 32; ++i) {
                const double e = oracle_e4m3_round(v[i] / scale);   /* division by 2^k is exact */
                if (q) q[r * K + b * 32 + i] = e;
                if (deq) deq[r * K + b * 32 + i] = e * scale;
            }
        }
    }
}

/* Element-wise forms of the two E4M3 helpers above, over n values. */
void oracle_e4m3_round_n(int64_t n, const double *v, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_round(v[i]);
}

void oracle_e4m3_bits_n(int64_t n, const double *q, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_bits(q[i]);
}
