/*
 * moe_oracle.c -- the CPU oracle of the fused MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's CPU-baseline leg
 * are the only code that may load this library; the product path (the CUDA library and its
 * Python binding) never links, imports or calls it, and shares no code with it.
 *
 * Plain, slow and direct: every floating-point step is carried out in IEEE double on inputs
 * that are bf16 values (passed as their raw 16-bit patterns and widened exactly). No step is
 * blocked, fused or reordered beyond what the definitions below state. The only parallelism
 * is an OpenMP loop over independent tokens.
 *
 * Sources (page title, then the section or figure):
 *  - Layer equation and SwiGLU: Mixture-of-Kittens blog, section "Overlapping compute and
 *    communication in MoE":  x' = W_shared(x) + sum_{e in top-k} w_e W_down^e SwiGLU(W_up^e x,
 *    W_gate^e x),  SwiGLU(u, g) = SiLU(u) (.) g  -- SiLU sits on the *up* projection.
 *  - Router projection and top-k: Weave blog, section 1.1 (a router picks top-k experts per
 *    token); vLLM MoE execution analysis, table "Per-decode-step kernel launches"
 *    (topk_softmax); FlashMoE review, "core formulas" (gate affinities G_phi).
 *  - Align: vLLM PR #53280 summary, "implementation breakdown" items 1-2 and the reviewer's
 *    all-blocks alternative (per-expert counts, exclusive cumsum, token ids written into
 *    per-expert segments padded to a multiple of the block size, one block id per block);
 *    vLLM MoE execution analysis, moe_align_block_size and BLOCK_SIZE_M.
 *  - Capacity: FlashMoE review, "core formulas" (routing table T_phi with capacity C per
 *    expert) and the FlashMoE experimental setup (capacity factor 1.0).
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *  - top-k ties: the lower expert index wins; selection compares logits, not rounded
 *    probabilities.
 *  - gating weights: softmax over all E experts, then the k selected probabilities are
 *    renormalised to sum to 1.
 *  - align order inside an expert segment: ascending slot id s = t*k + j (stable).
 *  - padding sentinel: S = T*k; unused expert_ids entries: -1.
 *  - capacity C = ceil(cf * S / E); a slot whose stable rank inside its expert is >= C is
 *    dropped (contributes nothing) and the other weights are not renormalised again.
 *  - a router bias, when given, is added to the logits before softmax and selection.
 *  - the shared expert is an ungated SwiGLU FFN with weight 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Router projection: logits[t][e] = sum_h x[t][h] * W_router[e][h] (+ bias[e]), summed in
 * ascending h.  absdot[t][e] = sum_h |x[t][h] * W_router[e][h]| (nullable): the quantity
 * that bounds the rounding error of any fp32 evaluation of the same dot product. */
ORACLE_API void moe_oracle_router_logits(const uint16_t *x, const uint16_t *w_router,
                                         const float *bias, int64_t T, int64_t H, int64_t E,
                                         double *logits, double *absdot)
{
    double *wr = (double *)malloc(sizeof(double) * (size_t)(E * H));
    for (int64_t i = 0; i < E * H; ++i) wr[i] = bf16_to_double(w_router[i]);
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t h = 0; h < H; ++h) xt[h] = bf16_to_double(x[t * H + h]);
            for (int64_t e = 0; e < E; ++e) {
                const double *w = wr + e * H;
                double s = 0.0, a = 0.0;
                for (int64_t h = 0; h < H; ++h) {
                    s += xt[h] * w[h];
                    a += fabs(xt[h] * w[h]);
                }
                if (bias) s += (double)bias[e];
                logits[t * E + e] = s;
                if (absdot) absdot[t * E + e] = a;
            }
        }
        free(xt);
    }
    free(wr);
}

/* Top-k selection and renormalised softmax for each token.
 * Selection: k rounds, each taking the largest remaining logit (ties to the lower index).
 * Weights: p = softmax(logits[t]) over all E experts; w_j = p_{ids_j} / sum_i p_{ids_i}.
 * ids are written in selection order (descending logit). */
ORACLE_API void moe_oracle_topk_softmax(const double *logits, int64_t T, int64_t E, int64_t k,
                                        int32_t *topk_ids, double *topk_w)
{
#pragma omp parallel
    {
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const double *v = logits + t * E;
            memset(taken, 0, (size_t)E);
            for (int64_t j = 0; j < k; ++j) {
                int64_t best = -1;
                for (int64_t e = 0; e < E; ++e) {
                    if (taken[e]) continue;
                    if (best < 0 || v[e] > v[best]) best = e; /* equal value: keep lower index */
                }
                taken[best] = 1;
                topk_ids[t * k + j] = (int32_t)best;
            }
            /* softmax over all experts (shifted by the max for range, which cancels) */
            double m = v[0];
            for (int64_t e = 1; e < E; ++e) if (v[e] > m) m = v[e];
            double z = 0.0;
            for (int64_t e = 0; e < E; ++e) { p[e] = exp(v[e] - m); z += p[e]; }
            for (int64_t e = 0; e < E; ++e) p[e] /= z;
            double s = 0.0;
            for (int64_t j = 0; j < k; ++j) s += p[topk_ids[t * k + j]];
            for (int64_t j = 0; j < k; ++j) topk_w[t * k + j] = p[topk_ids[t * k + j]] / s;
        }
        free(p);
        free(taken);
    }
}

/* Align (moe_align_block_size semantics).
 * Inputs: topk_ids [T*k] (slot s = t*k + j), E experts, block size block_m, capacity
 * (<= 0 means dropless).
 * Outputs:
 *   kept[s]          1 if slot s survives the capacity limit
 *   sorted_ids[i]    slot ids grouped by expert in ascending slot order, each expert's
 *                    segment padded with the sentinel S up to a multiple of block_m; every
 *                    entry from P to sorted_len-1 is the sentinel too
 *   expert_ids[b]    expert owning block b (b < P/block_m); -1 for b >= P/block_m
 *   *num_post_padded P = sum_e ceil(kept_e / block_m) * block_m
 * Returns P, or -1 if sorted_len or blocks_len is too small. */
ORACLE_API int64_t moe_oracle_align(const int32_t *topk_ids, int64_t T, int64_t k, int64_t E,
                                    int64_t block_m, int64_t capacity, int32_t *sorted_ids,
                                    int64_t sorted_len, int32_t *expert_ids, int64_t blocks_len,
                                    int32_t *num_post_padded, uint8_t *kept)
{
    const int64_t S = T * k;
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *kept_n = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *offset = (int64_t *)calloc((size_t)E + 1, sizeof(int64_t));
    int64_t *fill = (int64_t *)calloc((size_t)E, sizeof(int64_t));

    /* per-expert histogram, with the capacity decision taken by stable rank */
    for (int64_t s = 0; s < S; ++s) {
        int64_t e = topk_ids[s];
        int64_t rank = count[e]++;
        int keep = (capacity <= 0) || (rank < capacity);
        kept[s] = (uint8_t)keep;
        if (keep) kept_n[e]++;
    }
    /* exclusive scan of the padded segment lengths */
    for (int64_t e = 0; e < E; ++e) {
        int64_t padded = (kept_n[e] + block_m - 1) / block_m * block_m;
        offset[e + 1] = offset[e] + padded;
    }
    const int64_t P = offset[E];
    if (P > sorted_len || P / block_m > blocks_len) {
        free(count); free(kept_n); free(offset); free(fill);
        return -1;
    }
    for (int64_t i = 0; i < sorted_len; ++i) sorted_ids[i] = (int32_t)S;
    for (int64_t s = 0; s < S; ++s) {
        if (!kept[s]) continue;
        int64_t e = topk_ids[s];
        sorted_ids[offset[e] + fill[e]++] = (int32_t)s;
    }
    for (int64_t b = 0; b < blocks_len; ++b) expert_ids[b] = -1;
    for (int64_t e = 0; e < E; ++e)
        for (int64_t i = offset[e]; i < offset[e + 1]; i += block_m) expert_ids[i / block_m] = (int32_t)e;
    *num_post_padded = (int32_t)P;
    free(count); free(kept_n); free(offset); free(fill);
    return P;
}

/* First half of one expert FFN on one token (the SwiGLU of the layer equation):
 *   a[d] = SiLU(u_d) * g_d,  u_d = sum_h W_up[d][h] x[h],  g_d = sum_h W_gate[d][h] x[h],
 * SiLU(u) = u / (1 + e^-u), sums in ascending h. Optional outputs (nullable): uo[d] = u_d,
 * go[d] = g_d, and au[d] = sum_h |W_up[d][h] x[h]|, ag[d] likewise, which bound the rounding
 * error of any fp32 evaluation of u_d and g_d. w_up, w_gate: [D][H]. */
static void swiglu_row(const double *x, const uint16_t *w_up, const uint16_t *w_gate, int64_t H,
                       int64_t D, double *a, double *uo, double *go, double *au, double *ag)
{
    for (int64_t d = 0; d < D; ++d) {
        const uint16_t *ru = w_up + d * H, *rg = w_gate + d * H;
        double u = 0.0, g = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            u += bf16_to_double(ru[h]) * x[h];
            g += bf16_to_double(rg[h]) * x[h];
        }
        a[d] = (u / (1.0 + exp(-u))) * g;
        if (uo) uo[d] = u;
        if (go) go[d] = g;
        if (au) {
            double m = 0.0;
            for (int64_t h = 0; h < H; ++h) m += fabs(bf16_to_double(ru[h]) * x[h]);
            au[d] = m;
        }
        if (ag) {
            double m = 0.0;
            for (int64_t h = 0; h < H; ++h) m += fabs(bf16_to_double(rg[h]) * x[h]);
            ag[d] = m;
        }
    }
}

/* Second half: y[h] = sum_d W_down[h][d] a[d] (ascending d); ay[h] = sum_d |W_down[h][d] a[d]|
 * (nullable). w_down: [H][D]. */
static void down_row(const double *a, const uint16_t *w_down, int64_t H, int64_t D, double *y,
                     double *ay)
{
    for (int64_t h = 0; h < H; ++h) {
        const uint16_t *rd = w_down + h * D;
        double s = 0.0;
        for (int64_t d = 0; d < D; ++d) s += bf16_to_double(rd[d]) * a[d];
        y[h] = s;
        if (ay) {
            double m = 0.0;
            for (int64_t d = 0; d < D; ++d) m += fabs(bf16_to_double(rd[d]) * a[d]);
            ay[h] = m;
        }
    }
}

/* One expert FFN on one token: y = W_down . SwiGLU(W_up x, W_gate x).
 * w_up, w_gate: [D][H]; w_down: [H][D]; a: scratch [D]. */
static void expert_ffn(const double *x, const uint16_t *w_up, const uint16_t *w_gate,
                       const uint16_t *w_down, int64_t H, int64_t D, double *a, double *y)
{
    swiglu_row(x, w_up, w_gate, H, D, a, NULL, NULL, NULL, NULL);
    down_row(a, w_down, H, D, y, NULL);
}

/* The layer output for a list of tokens:
 *   out[i] = W_shared(x_t) + sum_{j: kept} w[t*k+j] * W_down^e SwiGLU(W_up^e x_t, W_gate^e x_t)
 * with t = tokens[i], e = topk_ids[t*k+j]; the shared term first, then j ascending.
 * W_up, W_gate: [E][D][H]; W_down: [E][H][D]; shared weights [Ds][H], [Ds][H], [H][Ds]
 * (ignored when Ds == 0). out: [n_tokens][H]. */
ORACLE_API void moe_oracle_layer(const uint16_t *x, int64_t T, int64_t H, int64_t D, int64_t E,
                                 int64_t k, const int32_t *topk_ids, const double *topk_w,
                                 const uint8_t *kept, const uint16_t *w_up,
                                 const uint16_t *w_gate, const uint16_t *w_down, int64_t Ds,
                                 const uint16_t *ws_up, const uint16_t *ws_gate,
                                 const uint16_t *ws_down, const int64_t *tokens,
                                 int64_t n_tokens, double *out)
{
    (void)T; (void)E;
    const int64_t Dmax = Ds > D ? Ds : D;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
        double *a = (double *)malloc(sizeof(double) * (size_t)Dmax);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_tokens; ++i) {
            const int64_t t = tokens[i];
            double *o = out + i * H;
            for (int64_t h = 0; h < H; ++h) xt[h] = bf16_to_double(x[t * H + h]);
            for (int64_t h = 0; h < H; ++h) o[h] = 0.0;
            if (Ds > 0) {
                expert_ffn(xt, ws_up, ws_gate, ws_down, H, Ds, a, y);
                for (int64_t h = 0; h < H; ++h) o[h] += y[h];
            }
            for (int64_t j = 0; j < k; ++j) {
                const int64_t s = t * k + j;
                if (!kept[s]) continue;
                const int64_t e = topk_ids[s];
                expert_ffn(xt, w_up + e * D * H, w_gate + e * D * H, w_down + e * H * D, H, D, a, y);
                for (int64_t h = 0; h < H; ++h) o[h] += topk_w[s] * y[h];
            }
        }
        free(y);
        free(a);
        free(xt);
    }
}

/* ---------------------------------------------------------------------------------------
 * The layer equation stage by stage, for checking the GPU path's intermediates one step at a
 * time (each stage is fed the GPU's own output of the stage before it).
 * ------------------------------------------------------------------------------------- */

/* GEMM1 + SwiGLU for n (token, expert) pairs: h[i][0..Dt) = SwiGLU(W_up^e x_t, W_gate^e x_t),
 * t = tokens[i], e = experts[i]; e == E selects the shared expert (ws_up, ws_gate, Dt = Ds),
 * else Dt = D. u, g, au, ag (nullable) as uo, go, au, ag of swiglu_row. Every output is
 * [n][ld] (ld >= max(D, Ds)). */
ORACLE_API void moe_oracle_expert_h(const uint16_t *x, int64_t H, int64_t D, int64_t E,
                                    const uint16_t *w_up, const uint16_t *w_gate, int64_t Ds,
                                    const uint16_t *ws_up, const uint16_t *ws_gate,
                                    const int64_t *tokens, const int32_t *experts, int64_t n,
                                    int64_t ld, double *h, double *u, double *g, double *au,
                                    double *ag)
{
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n; ++i) {
            const int64_t t = tokens[i], e = experts[i];
            double *ui = u ? u + i * ld : NULL, *gi = g ? g + i * ld : NULL;
            double *aui = au ? au + i * ld : NULL, *agi = ag ? ag + i * ld : NULL;
            for (int64_t c = 0; c < H; ++c) xt[c] = bf16_to_double(x[t * H + c]);
            if (e == E)
                swiglu_row(xt, ws_up, ws_gate, H, Ds, h + i * ld, ui, gi, aui, agi);
            else
                swiglu_row(xt, w_up + e * D * H, w_gate + e * D * H, H, D, h + i * ld, ui, gi, aui, agi);
        }
        free(xt);
    }
}

/* GEMM2 with the router weight for n rows: y[i][c] = wts[i] * sum_d W_down^e[c][d] a[i][d],
 * e = experts[i] (E selects the shared expert, ws_down [H][Ds]); a: [n][lda], its first Dt
 * entries used. ay[i][c] = |wts[i]| * sum_d |W_down^e[c][d] a[i][d]| (nullable). y, ay: [n][H]. */
ORACLE_API void moe_oracle_expert_down(const double *a, int64_t lda, int64_t H, int64_t D, int64_t E,
                                       const uint16_t *w_down, int64_t Ds, const uint16_t *ws_down,
                                       const int32_t *experts, const double *wts, int64_t n, double *y,
                                       double *ay)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t e = experts[i];
        double *yi = y + i * H, *ai = ay ? ay + i * H : NULL;
        if (e == E)
            down_row(a + i * lda, ws_down, H, Ds, yi, ai);
        else
            down_row(a + i * lda, w_down + e * H * D, H, D, yi, ai);
        for (int64_t c = 0; c < H; ++c) {
            yi[c] = wts[i] * yi[c];
            if (ai) ai[c] = fabs(wts[i]) * ai[c];
        }
    }
}

/* Combine: out[i] = sum_{j < m, idx[i][j] >= 0} rows[idx[i][j]], summed in j order (the shared
 * expert's row first, then the token's slots j = 0..k-1, as in moe_oracle_layer).
 * rows: [*][H]; idx: [n][m]; out: [n][H]. */
ORACLE_API void moe_oracle_combine(const double *rows, int64_t H, const int64_t *idx, int64_t n,
                                   int64_t m, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double *o = out + i * H;
        for (int64_t c = 0; c < H; ++c) o[c] = 0.0;
        for (int64_t j = 0; j < m; ++j) {
            const int64_t r = idx[i * m + j];
            if (r < 0) continue;
            for (int64_t c = 0; c < H; ++c) o[c] += rows[r * H + c];
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * MXFP8 experts.  The pages name MXFP8 support (Mixture-of-Kittens blog, introduction and its
 * MXFP8 section heading; FlashMoE review, "future directions": FP8 and lower precisions) but do
 * not define the format; the reading taken is the OCP Microscaling (MX) format, MXFP8 with E4M3
 * elements:
 *  - a block is 32 consecutive elements along the contraction dimension; it shares one E8M0
 *    scale X = 2^s (code s + 127, s in [-127, 127]);
 *  - s = floor(log2(max |v|)) - 8 (8 = the exponent of E4M3's largest normal, 448 = 1.75 * 2^8),
 *    clamped to [-127, 127]; an all-zero block takes s = -127;
 *  - each element is v / X rounded to E4M3, to nearest with ties to even, magnitudes above 448
 *    clamped to 448 (saturating conversion);
 *  - the value of an element is its E4M3 value times X.
 * In the layer, x (along H), h (along D or Ds) and every expert weight matrix (along its
 * contraction dimension) are quantised this way; the products, SwiGLU, the router weights and
 * the combine stay exact (double). h is quantised from its value rounded to fp32, the
 * precision in which the GPU path takes the same decision.
 * ------------------------------------------------------------------------------------- */

/* E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 holds the
 * subnormals m * 2^-9; S.1111.111 is NaN (there is no infinity). */
ORACLE_API double moe_oracle_e4m3_value(uint8_t c)
{
    const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* Nearest E4M3 code to v, ties to the even code, |v| > 448 clamped to 448. */
ORACLE_API uint8_t moe_oracle_e4m3_encode(double v)
{
    const uint8_t sgn = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (a > 448.0) a = 448.0;
    /* spacing of the representable values around a: 2^-9 below 2^-6, else 2^(floor(log2 a) - 3) */
    int ex;
    double q;
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);
    } else {
        frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1 */
        q = ldexp(1.0, ex - 1 - 3);
    }
    const double r = a / q; /* exact: q is a power of two */
    double n = floor(r);
    const double frac = r - n;
    if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0)) n += 1.0;
    const double val = n * q; /* a representable magnitude (may be the next binade's first) */
    uint8_t code;
    if (val < ldexp(1.0, -6)) {
        code = (uint8_t)(val / ldexp(1.0, -9)); /* subnormal: m = val / 2^-9 */
    } else {
        frexp(val, &ex);
        const int e = ex - 1;                                   /* val = 2^e * (1 + m/8) */
        const int m = (int)(ldexp(val, -e) * 8.0 - 8.0);
        code = (uint8_t)(((e + 7) << 3) | m);
    }
    return (uint8_t)(sgn | code);
}

/* Quantise n values (n a multiple of 32) block by block: codes[n] and the E8M0 scale codes
 * scales[n / 32]. */
ORACLE_API void moe_oracle_mx_quantize(const double *v, int64_t n, uint8_t *codes, uint8_t *scales)
{
    for (int64_t b = 0; b < n / 32; ++b) {
        const double *blk = v + b * 32;
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
        int s = -127;
        if (amax > 0.0) {
            int ex;
            frexp(amax, &ex);
            s = (ex - 1) - 8;
            if (s < -127) s = -127;
            if (s > 127) s = 127;
        }
        scales[b] = (uint8_t)(s + 127);
        for (int i = 0; i < 32; ++i) codes[b * 32 + i] = moe_oracle_e4m3_encode(ldexp(blk[i], -s));
    }
}

/* Value of element i of a quantised vector. */
static double mx_value(const uint8_t *codes, const uint8_t *scales, int64_t i)
{
    return ldexp(moe_oracle_e4m3_value(codes[i]), (int)scales[i / 32] - 127);
}

/* v <- the values of its MX quantisation (n a multiple of 32); scratch: n + n/32 bytes. */
static void mx_round_trip(double *v, int64_t n, uint8_t *scratch)
{
    uint8_t *codes = scratch, *scales = scratch + n;
    moe_oracle_mx_quantize(v, n, codes, scales);
    for (int64_t i = 0; i < n; ++i) v[i] = mx_value(codes, scales, i);
}

/* Quantise the rows of a bf16 matrix [R][K] (K a multiple of 32): codes [R][K], scale codes
 * [R][K/32]. */
ORACLE_API void moe_oracle_mx_quantize_bf16_rows(const uint16_t *src, int64_t R, int64_t K,
                                                 uint8_t *codes, uint8_t *scales)
{
#pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < R; ++r) {
            for (int64_t i = 0; i < K; ++i) row[i] = bf16_to_double(src[r * K + i]);
            moe_oracle_mx_quantize(row, K, codes + r * K, scales + r * (K / 32));
        }
        free(row);
    }
}

/* xq[i] = the values of the MX quantisation of token row x[tokens[i]] (along H), i < n. */
static void mx_token_rows(const uint16_t *x, int64_t H, const int64_t *tokens, int64_t n, double *xq)
{
#pragma omp parallel
    {
        uint8_t *scratch = (uint8_t *)malloc((size_t)(H + H / 32));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < n; ++i) {
            for (int64_t h = 0; h < H; ++h) xq[i * H + h] = bf16_to_double(x[tokens[i] * H + h]);
            mx_round_trip(xq + i * H, H, scratch);
        }
        free(scratch);
    }
}

/* One expert's FFN on n MX-quantised token rows (values; row l is xq + rows[l] * H):
 *   a_l = SwiGLU(Wq_up xq_l, Wq_gate xq_l) rounded to fp32 and quantised along Dt,
 *   y_l = Wq_down a_l,
 * where every weight row is quantised along its contraction dimension -- once, and used for
 * all n rows. w_up, w_gate: [Dt][H]; w_down: [H][Dt] (NULL: stop after a); a: [n][Dt];
 * y: [n][H]. Optional outputs ([n][Dt], nullable): a_pre = a before its quantisation, uo / go
 * = the up / gate projections, au / ag = their sums of |Wq xq| (rounding-error bounds). */
static void expert_rows_mx(const double *xq, const int64_t *rows, int64_t n, int64_t H, int64_t Dt,
                           const uint16_t *w_up, const uint16_t *w_gate, const uint16_t *w_down,
                           double *a, double *y, double *a_pre, double *uo, double *go, double *au,
                           double *ag)
{
    const int64_t W = H > Dt ? H : Dt;
#pragma omp parallel
    {
        double *wu = (double *)malloc(sizeof(double) * (size_t)W);
        double *wg = (double *)malloc(sizeof(double) * (size_t)W);
        double *wd = (double *)malloc(sizeof(double) * (size_t)W);
        uint8_t *scratch = (uint8_t *)malloc((size_t)(W + W / 32));
#pragma omp for schedule(dynamic, 4)
        for (int64_t d = 0; d < Dt; ++d) {
            for (int64_t h = 0; h < H; ++h) wu[h] = bf16_to_double(w_up[d * H + h]);
            mx_round_trip(wu, H, scratch);
            for (int64_t h = 0; h < H; ++h) wg[h] = bf16_to_double(w_gate[d * H + h]);
            mx_round_trip(wg, H, scratch);
            for (int64_t l = 0; l < n; ++l) {
                const double *xl = xq + rows[l] * H;
                double u = 0.0, g = 0.0;
                for (int64_t h = 0; h < H; ++h) u += wu[h] * xl[h];
                for (int64_t h = 0; h < H; ++h) g += wg[h] * xl[h];
                a[l * Dt + d] = (double)(float)((u / (1.0 + exp(-u))) * g);
                if (a_pre) a_pre[l * Dt + d] = a[l * Dt + d];
                if (uo) uo[l * Dt + d] = u;
                if (go) go[l * Dt + d] = g;
                if (au) {
                    double m = 0.0;
                    for (int64_t h = 0; h < H; ++h) m += fabs(wu[h] * xl[h]);
                    au[l * Dt + d] = m;
                }
                if (ag) {
                    double m = 0.0;
                    for (int64_t h = 0; h < H; ++h) m += fabs(wg[h] * xl[h]);
                    ag[l * Dt + d] = m;
                }
            }
        }
#pragma omp for schedule(static)
        for (int64_t l = 0; l < n; ++l) mx_round_trip(a + l * Dt, Dt, scratch);
#pragma omp for schedule(dynamic, 4)
        for (int64_t h = 0; h < (w_down ? H : 0); ++h) {
            for (int64_t d = 0; d < Dt; ++d) wd[d] = bf16_to_double(w_down[h * Dt + d]);
            mx_round_trip(wd, Dt, scratch);
            for (int64_t l = 0; l < n; ++l) {
                double s = 0.0;
                for (int64_t d = 0; d < Dt; ++d) s += wd[d] * a[l * Dt + d];
                y[l * H + h] = s;
            }
        }
        free(scratch);
        free(wd);
        free(wg);
        free(wu);
    }
}

/* The MXFP8 layer's GEMM1 + SwiGLU for n (token, expert) pairs (expert E = the shared expert):
 * h[i] = SwiGLU(Wq_up^e xq_t, Wq_gate^e xq_t) rounded to fp32, i.e. the values that the layer then
 * quantises, with the projections u, g and their magnitude sums au, ag (each nullable). Every
 * output is [n][ld], ld >= max(D, Ds). */
ORACLE_API void moe_oracle_expert_h_mxfp8(const uint16_t *x, int64_t H, int64_t D, int64_t E,
                                          const uint16_t *w_up, const uint16_t *w_gate, int64_t Ds,
                                          const uint16_t *ws_up, const uint16_t *ws_gate,
                                          const int64_t *tokens, const int32_t *experts, int64_t n,
                                          int64_t ld, double *h, double *u, double *g, double *au,
                                          double *ag)
{
    const int64_t Dmax = Ds > D ? Ds : D;
    double *xq = (double *)malloc(sizeof(double) * (size_t)(n * H));
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
    int64_t *dest = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
    double *abuf = (double *)malloc(sizeof(double) * (size_t)(n * Dmax));
    double *part[5];
    for (int q = 0; q < 5; ++q) part[q] = (double *)malloc(sizeof(double) * (size_t)(n * Dmax));
    double *outs[5] = {h, u, g, au, ag};
    mx_token_rows(x, H, tokens, n, xq);
    for (int64_t e = 0; e <= E; ++e) {
        int64_t m = 0;
        for (int64_t i = 0; i < n; ++i)
            if (experts[i] == e) {
                rows[m] = i;
                dest[m++] = i;
            }
        if (m == 0) continue;
        const int64_t Dt = (e == E) ? Ds : D;
        if (e == E)
            expert_rows_mx(xq, rows, m, H, Dt, ws_up, ws_gate, NULL, abuf, NULL, part[0], part[1], part[2],
                           au ? part[3] : NULL, ag ? part[4] : NULL);
        else
            expert_rows_mx(xq, rows, m, H, Dt, w_up + e * D * H, w_gate + e * D * H, NULL, abuf, NULL, part[0],
                           part[1], part[2], au ? part[3] : NULL, ag ? part[4] : NULL);
        for (int64_t l = 0; l < m; ++l)
            for (int q = 0; q < 5; ++q)
                if (outs[q]) memcpy(outs[q] + dest[l] * ld, part[q] + l * Dt, sizeof(double) * (size_t)Dt);
    }
    for (int q = 0; q < 5; ++q) free(part[q]);
    free(abuf);
    free(dest);
    free(rows);
    free(xq);
}

/* moe_oracle_layer with MXFP8 experts (H, D and Ds multiples of 32): x, every expert weight
 * row and h are quantised as above; per token the shared expert's row first, then the kept
 * slots j = 0..k-1 weighted by topk_w, as in moe_oracle_layer. The experts are taken one at a
 * time (each weight row is quantised once per call); each slot's result is kept until the
 * per-token sums, which run in the order just stated. */
ORACLE_API void moe_oracle_layer_mxfp8(const uint16_t *x, int64_t T, int64_t H, int64_t D, int64_t E,
                                       int64_t k, const int32_t *topk_ids, const double *topk_w,
                                       const uint8_t *kept, const uint16_t *w_up,
                                       const uint16_t *w_gate, const uint16_t *w_down, int64_t Ds,
                                       const uint16_t *ws_up, const uint16_t *ws_gate,
                                       const uint16_t *ws_down, const int64_t *tokens,
                                       int64_t n_tokens, double *out)
{
    (void)T;
    const int64_t m = k + 1; /* per token: slots 0..k-1, then the shared expert */
    const int64_t Dmax = Ds > D ? Ds : D;
    double *xq = (double *)malloc(sizeof(double) * (size_t)(n_tokens * H));
    double *ys = (double *)calloc((size_t)(n_tokens * m * H), sizeof(double));
    double *a = (double *)malloc(sizeof(double) * (size_t)(n_tokens * Dmax));
    double *ye = (double *)malloc(sizeof(double) * (size_t)(n_tokens * H));
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_tokens);
    int64_t *dest = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_tokens);
    mx_token_rows(x, H, tokens, n_tokens, xq);
    for (int64_t e = 0; e <= E; ++e) {
        const int shared = (e == E);
        if (shared && Ds == 0) break;
        int64_t n = 0;
        for (int64_t i = 0; i < n_tokens; ++i) {
            if (shared) {
                rows[n] = i;
                dest[n++] = i * m + k;
                continue;
            }
            for (int64_t j = 0; j < k; ++j) {
                const int64_t s = tokens[i] * k + j;
                if (kept[s] && topk_ids[s] == e) {
                    rows[n] = i;
                    dest[n++] = i * m + j;
                }
            }
        }
        if (n == 0) continue;
        if (shared)
            expert_rows_mx(xq, rows, n, H, Ds, ws_up, ws_gate, ws_down, a, ye, NULL, NULL, NULL, NULL, NULL);
        else
            expert_rows_mx(xq, rows, n, H, D, w_up + e * D * H, w_gate + e * D * H, w_down + e * H * D, a, ye,
                           NULL, NULL, NULL, NULL, NULL);
        for (int64_t l = 0; l < n; ++l) memcpy(ys + dest[l] * H, ye + l * H, sizeof(double) * (size_t)H);
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_tokens; ++i) {
        const int64_t t = tokens[i];
        double *o = out + i * H;
        for (int64_t h = 0; h < H; ++h) o[h] = 0.0;
        if (Ds > 0)
            for (int64_t h = 0; h < H; ++h) o[h] += ys[(i * m + k) * H + h];
        for (int64_t j = 0; j < k; ++j) {
            const int64_t s = t * k + j;
            if (!kept[s]) continue;
            for (int64_t h = 0; h < H; ++h) o[h] += topk_w[s] * ys[(i * m + j) * H + h];
        }
    }
    free(dest);
    free(rows);
    free(ye);
    free(a);
    free(ys);
    free(xq);
}

/* Threads the OpenMP loops above use (1 when built without OpenMP). */
ORACLE_API int moe_oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
