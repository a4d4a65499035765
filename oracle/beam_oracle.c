/*
 * Beam MoE block forward pass: plain, slow CPU oracle in FP64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline /
 * reference arm may load this library.  It shares no code, header or constant with the CUDA
 * library; it is built separately (oracle/build.py) with gcc.
 *
 * What it computes, step by step, in the order of the Beam launch post ("Welcome Beam" page,
 * section "Mixture of Experts"; the same text in the Hugging Face post flattened on the
 * reducer.xgoose.org digest page; the Chinese digest on that page adds "sigmoid scoring, 8 experts,
 * x2.5"):
 *   1. score every expert with a sigmoid of the router projection, computed in FP32 by the model
 *      ("Welcome Beam" page, section "Residual Stream": the router computes in FP32);
 *   2. split the experts into n_groups contiguous groups; rank groups by the sum of each group's
 *      top group_topn scores; keep the topk_groups best groups;
 *   3. pick the topk experts with the largest scores inside the kept groups;
 *   4. combine the experts' outputs with router weights normalised to sum 1, then scale by
 *      routed_scale (2.5);
 *   5. each expert is a SwiGLU MLP: Wd (SiLU(Wg x) * (Wu x)).
 *
 * Readings where the pages are silent (all listed in the design notes of this repository):
 *   - an optional per-expert selection bias b is added to the scores for group and expert
 *     selection only; the weights use the unbiased sigmoid scores (DeepSeek-V3's scheme, which the
 *     pages name); b = 0 unless a workload sets it;
 *   - groups are contiguous index ranges;
 *   - ties go to the lower group / expert index; slots are in descending selected score;
 *   - the selection decision is taken on scores rounded to FP32 (the router's precision on the
 *     pages); the FP64 scores give the decision margins used to exclude near-ties from bit-exact
 *     comparison.
 *
 * Arithmetic: logits, sigmoid, weights, expert MLP and the weighted sum in FP64 on the exact bf16
 * inputs.  bf16 values arrive as their raw 16-bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Evaluation order of the dot products below.  Every output is one sum over the reduction index
 * taken in increasing order, acc = ((0 + a_0 b_0) + a_1 b_1) + ..., exactly as a plain loop per
 * output computes it.  Rows of activations are taken RB at a time, stored transposed (xb[h*RB + r]),
 * so the RB independent sums of one weight row advance together; no sum is split or reordered, so
 * every value is the one the plain per-output loop gives.
 */
#define RB 8

/* acc[r] = sum_{h=0}^{K-1} xb[h*RB + r] * w[h] for r < RB, each sum in increasing h. */
static void dot_rows(int K, const double *xb, const double *w, double *acc)
{
    double a[RB] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    for (int h = 0; h < K; ++h)
        for (int r = 0; r < RB; ++r) a[r] += xb[(int64_t)h * RB + r] * w[h];
    for (int r = 0; r < RB; ++r) acc[r] = a[r];
}

/* Rows [r0, r0 + nr) of a [*,K] bf16-bit matrix, widened to FP64 (exact) and transposed into
 * xb[k*RB + r]; rows nr..RB-1 are zero. */
static void bf16_rows_to_block(const uint16_t *rows, int64_t r0, int nr, int K, double *xb)
{
    for (int k = 0; k < K; ++k)
        for (int r = 0; r < RB; ++r)
            xb[(int64_t)k * RB + r] = r < nr ? bf16_bits_to_double(rows[(r0 + r) * K + k]) : 0.0;
}

static int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

/*
 * Step 1 (section "Mixture of Experts": "scores all 256 experts with a sigmoid"):
 * logit[t,e] = sum_h x[t,h] * W_r[e,h] in FP64, score = 1 / (1 + exp(-logit)).
 * x: [T,H] bf16 bits; w_router: [E,H] fp32; logit, score: [T,E] fp64.
 */
void oracle_router_scores(int64_t T, int H, int E, const uint16_t *x, const float *w_router,
                          double *logit, double *score)
{
    double *wr = (double *)malloc(sizeof(double) * (size_t)E * (size_t)H);
    for (int64_t q = 0; q < (int64_t)E * H; ++q) wr[q] = (double)w_router[q];
    const int64_t nb = (T + RB - 1) / RB;
    #pragma omp parallel
    {
        double *xb = (double *)malloc(sizeof(double) * (size_t)H * RB);
        #pragma omp for schedule(static)
        for (int64_t b = 0; b < nb; ++b) {
            const int nr = (int)min64(RB, T - b * RB);
            bf16_rows_to_block(x, b * RB, nr, H, xb);
            for (int e = 0; e < E; ++e) {
                double acc[RB];
                dot_rows(H, xb, wr + (int64_t)e * H, acc);
                for (int r = 0; r < nr; ++r) {
                    const int64_t t = b * RB + r;
                    if (logit) logit[t * E + e] = acc[r];
                    score[t * E + e] = 1.0 / (1.0 + exp(-acc[r]));
                }
            }
        }
        free(xb);
    }
    free(wr);
}

/* Index of the largest v[i] among alive[i] != 0; ties go to the lower index.  -1 if none. */
static int argmax_alive(const double *v, const unsigned char *alive, int n)
{
    int best = -1;
    for (int i = 0; i < n; ++i) {
        if (!alive[i]) continue;
        if (best < 0 || v[i] > v[best]) best = i;
    }
    return best;
}

/*
 * Group-limited selection for one token (steps 2 and 3).  `sel` holds the selection values of the
 * E experts (score + bias).  When `fp32` is set, every selection value and every group-score sum
 * is rounded to FP32 (the decision precision of the model's router); otherwise FP64.
 * Outputs the kept groups' mask and the topk expert ids in pick order (descending value).
 * Returns the sorted group scores and selected values so the caller can take margins.
 */
static void select_one(int E, int G, int topk_groups, int topk, int group_topn, const double *sel_in,
                       int fp32, unsigned char *group_kept, int32_t *ids, double *gs_sorted,
                       double *sel_sorted_kept, int *n_kept_experts)
{
    const int per = E / G;
    double sel[1024];
    unsigned char alive[1024];
    double gs[1024];
    for (int e = 0; e < E; ++e) sel[e] = fp32 ? (double)(float)sel_in[e] : sel_in[e];

    /* group score = sum of the group's top group_topn selection values, summed in pick order */
    for (int g = 0; g < G; ++g) {
        for (int i = 0; i < per; ++i) alive[i] = 1;
        double s64 = 0.0;
        float s32 = 0.0f;
        for (int r = 0; r < group_topn; ++r) {
            int i = argmax_alive(sel + g * per, alive, per);
            alive[i] = 0;
            if (fp32) s32 = s32 + (float)sel[g * per + i];
            else s64 += sel[g * per + i];
        }
        gs[g] = fp32 ? (double)s32 : s64;
    }
    /* keep the topk_groups best groups (lower group index on ties) */
    unsigned char galive[1024];
    for (int g = 0; g < G; ++g) { galive[g] = 1; group_kept[g] = 0; }
    for (int r = 0; r < G; ++r) {
        int g = argmax_alive(gs, galive, G);
        galive[g] = 0;
        gs_sorted[r] = gs[g];
        if (r < topk_groups) group_kept[g] = 1;
    }
    /* topk experts inside the kept groups (lower expert index on ties), in pick order */
    for (int e = 0; e < E; ++e) alive[e] = group_kept[e / per];
    int n = 0;
    for (int e = 0; e < E; ++e) n += alive[e];
    *n_kept_experts = n;
    for (int r = 0; r < n; ++r) {
        int e = argmax_alive(sel, alive, E);
        alive[e] = 0;
        sel_sorted_kept[r] = sel[e];
        if (r < topk) ids[r] = e;
    }
}

/*
 * Steps 2-4 for T tokens.  score: [T,E] fp64 (from oracle_router_scores); bias: [E] fp32 or NULL.
 * Outputs:
 *   ids     [T,topk] int32  the decision taken on FP32-rounded values (the model's router precision)
 *   ids64   [T,topk] int32  the same decision in FP64 (nullable)
 *   weight  [T,topk] fp64   score[id] / sum of the selected scores (unbiased scores)
 *   margin  [T,3]    fp64   FP64 decision margins (nullable):
 *                           [0] group: 4th-best minus 5th-best group score (topk_groups-th vs next)
 *                           [1] expert: topk-th minus next selection value inside the kept groups
 *                           [2] order: smallest gap between consecutive selected values
 *                           (+inf where no such comparison exists)
 * Returns 0, or -1 for a configuration this plain implementation does not accept.
 */
int oracle_select(int64_t T, int E, int G, int topk_groups, int topk, int group_topn,
                  const double *score, const float *bias, int32_t *ids, int32_t *ids64,
                  double *weight, double *margin)
{
    if (E <= 0 || E > 1024 || G <= 0 || E % G || topk_groups < 1 || topk_groups > G ||
        group_topn < 1 || group_topn > E / G || topk < 1 || topk > topk_groups * (E / G))
        return -1;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(+:bad)
    for (int64_t t = 0; t < T; ++t) {
        double sel[1024], gs_sorted[1024], sel_sorted[1024];
        unsigned char kept[1024];
        int32_t id32[1024], id64[1024];
        int nk = 0;
        const double *s = score + t * E;
        /* the biased value in FP32 is the FP32 sum of the FP32 score and the FP32 bias */
        for (int e = 0; e < E; ++e) {
            float s32 = (float)s[e];
            sel[e] = bias ? (double)(s32 + bias[e]) : (double)s32;
        }
        select_one(E, G, topk_groups, topk, group_topn, sel, 1, kept, id32, gs_sorted, sel_sorted, &nk);
        for (int e = 0; e < E; ++e) sel[e] = s[e] + (bias ? (double)bias[e] : 0.0);
        select_one(E, G, topk_groups, topk, group_topn, sel, 0, kept, id64, gs_sorted, sel_sorted, &nk);
        for (int j = 0; j < topk; ++j) {
            ids[t * topk + j] = id32[j];
            if (ids64) ids64[t * topk + j] = id64[j];
        }
        double den = 0.0;
        for (int j = 0; j < topk; ++j) den += s[id32[j]];
        if (!(den > 0.0)) bad++;
        for (int j = 0; j < topk; ++j) weight[t * topk + j] = s[id32[j]] / den;
        if (margin) {
            margin[t * 3 + 0] = topk_groups < G ? gs_sorted[topk_groups - 1] - gs_sorted[topk_groups] : INFINITY;
            margin[t * 3 + 1] = topk < nk ? sel_sorted[topk - 1] - sel_sorted[topk] : INFINITY;
            double mo = INFINITY;
            for (int j = 0; j + 1 < topk; ++j) {
                double d = sel_sorted[j] - sel_sorted[j + 1];
                if (d < mo) mo = d;
            }
            margin[t * 3 + 2] = mo;
        }
    }
    return bad ? -2 : 0;
}

/*
 * Token -> expert dispatch (the pages only say each token runs on its 8 experts; this is the plain
 * stable grouping of the T*topk (token, slot) pairs by expert).  Rows are ordered by
 * (expert ascending, token ascending); q = t*topk + j.
 *   counts[e]   number of pairs routed to e
 *   offsets[e]  exclusive prefix sum of counts (offsets[E] = T*topk)
 *   row_src[r]  the pair q placed in row r
 *   dest_row[q] the row of pair q
 * Returns 0, or -1 if an id is outside [0, E).
 */
int oracle_permute(int64_t T, int topk, int E, const int32_t *ids, int32_t *counts, int64_t *offsets,
                   int32_t *row_src, int32_t *dest_row)
{
    const int64_t n = T * topk;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t q = 0; q < n; ++q) {
        if (ids[q] < 0 || ids[q] >= E) return -1;
        counts[ids[q]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t r = 0;
    for (int e = 0; e < E; ++e)
        for (int64_t q = 0; q < n; ++q)
            if (ids[q] == e) {
                row_src[r] = (int32_t)q;
                dest_row[q] = (int32_t)r;
                ++r;
            }
    return 0;
}

/*
 * One SwiGLU expert ("each a SwiGLU MLP with an intermediate size of 2,560"; the SwiGLU product in
 * FP32 on the model, here FP64) applied to n rows:
 *   g = Wg x, u = Wu x, h = SiLU(g) * u with SiLU(z) = z / (1 + exp(-z)), out = Wd h.
 * x_rows [n,H] bf16 bits; wg, wu [I,H] bf16 bits; wd [H,I] bf16 bits; out [n,H] fp64.
 */
void oracle_expert_mlp(int64_t n, int H, int I, const uint16_t *x_rows, const uint16_t *wg,
                       const uint16_t *wu, const uint16_t *wd, double *out)
{
    const int64_t nb = (n + RB - 1) / RB;
    double *xb = (double *)malloc(sizeof(double) * (size_t)(nb * H * RB));  /* x, RB rows per block */
    double *hb = (double *)malloc(sizeof(double) * (size_t)(nb * I * RB));  /* h, same blocking */
    for (int64_t b = 0; b < nb; ++b) bf16_rows_to_block(x_rows, b * RB, (int)min64(RB, n - b * RB), H, xb + b * H * RB);

    /* g = Wg x, u = Wu x, h = SiLU(g) * u */
    #pragma omp parallel
    {
        double *wgr = (double *)malloc(sizeof(double) * (size_t)H);
        double *wur = (double *)malloc(sizeof(double) * (size_t)H);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < nb; ++b)
            for (int i = 0; i < I; ++i) {
                for (int h = 0; h < H; ++h) {
                    wgr[h] = bf16_bits_to_double(wg[(int64_t)i * H + h]);
                    wur[h] = bf16_bits_to_double(wu[(int64_t)i * H + h]);
                }
                double g[RB], u[RB];
                dot_rows(H, xb + b * H * RB, wgr, g);
                dot_rows(H, xb + b * H * RB, wur, u);
                for (int r = 0; r < RB; ++r) {
                    double silu = g[r] / (1.0 + exp(-g[r]));
                    hb[(b * I + i) * RB + r] = silu * u[r];
                }
            }
        free(wgr);
        free(wur);
    }

    /* out = Wd h */
    #pragma omp parallel
    {
        double *wdr = (double *)malloc(sizeof(double) * (size_t)I);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < nb; ++b)
            for (int o = 0; o < H; ++o) {
                for (int i = 0; i < I; ++i) wdr[i] = bf16_bits_to_double(wd[(int64_t)o * I + i]);
                double acc[RB];
                dot_rows(I, hb + b * I * RB, wdr, acc);
                for (int r = 0; r < RB && b * RB + r < n; ++r) out[(b * RB + r) * H + o] = acc[r];
            }
        free(wdr);
    }
    free(xb);
    free(hb);
}

/*
 * Step 4 ("Expert outputs are combined with normalized router weights and scaled by 2.5"):
 * y[t] = routed_scale * sum_j weight[t,j] * expert_out[t,j], summed over j = 0..topk-1.
 * expert_out [T,topk,H] fp64; weight [T,topk] fp64; y [T,H] fp64.
 */
void oracle_combine(int64_t T, int topk, int H, double routed_scale, const double *expert_out,
                    const double *weight, double *y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < topk; ++j)
                acc += weight[t * topk + j] * expert_out[(t * topk + j) * H + h];
            y[t * H + h] = routed_scale * acc;
        }
}

/*
 * Sublayer normalisation ("Welcome Beam" page, section "Residual Stream": every sublayer is
 * normalised before and after; the norms compute in FP32 on the model, here FP64).  Reading: RMSNorm
 * with a learned per-channel scale,
 *   out[t,h] = x[t,h] / sqrt(mean_h x[t,h]^2 + eps) * g[h].
 * x, out [T,H] fp64; g [H] fp64.
 */
void oracle_rmsnorm(int64_t T, int H, const double *x, const double *g, double eps, double *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += x[t * H + h] * x[t * H + h];
        const double inv = 1.0 / sqrt(ss / H + eps);
        for (int h = 0; h < H; ++h) out[t * H + h] = x[t * H + h] * inv * g[h];
    }
}

/*
 * Scaled residual update (same section): the input embedding is step 1; at step k the sublayer
 * output z is added with weight 1/sqrt(k) and the stream kept with weight sqrt((k-1)/k).
 *   out = sqrt((k-1)/k) * stream + z / sqrt(k).
 * Returns -1 for k < 2.
 */
int oracle_scaled_residual(int64_t T, int H, const double *stream, const double *z, int k, double *out)
{
    if (k < 2) return -1;
    const double keep = sqrt((double)(k - 1) / (double)k), add = 1.0 / sqrt((double)k);
    for (int64_t q = 0; q < T * (int64_t)H; ++q) out[q] = keep * stream[q] + add * z[q];
    return 0;
}

/*
 * FP8 expert weights ("Checkpoint formats: BF16, FP8, and NVFP4": "Welcome Beam" page, TL;DR; the
 * pages give no recipe).  Reading: the OCP MXFP8 layout, E4M3 elements with one power-of-two
 * (UE8M0) scale per 32 consecutive K elements of a weight row; the scales are stored
 * K-block-major, scale[kb][row].
 *   E4M3: sign s, exponent e (4 bits, bias 7), mantissa m (3 bits); e = 15 with m = 7 is NaN;
 *         e = 0 is subnormal, m * 2^-9; otherwise (1 + m/8) * 2^(e-7).
 *   UE8M0: 2^(c - 127); c = 255 is NaN.
 * w[row][k] = e4m3(q[row][k]) * 2^(scale[k/32][row] - 127), returned as bf16 bits.  Every such
 * product has at most 4 significant bits, so it is exact in bf16 whenever it lies in bf16's range;
 * returns -1 for a NaN code or a product that bf16 cannot hold exactly.
 * q [rows,K] uint8; scale [K/32, rows] uint8; out [rows,K] bf16 bits.
 */
static double e4m3_value(uint8_t b)
{
    const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

int oracle_dequant_mxfp8(int64_t rows, int K, const uint8_t *q, const uint8_t *scale, uint16_t *out)
{
    if (K % 32) return -1;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) {
            const uint8_t c = scale[(int64_t)(k / 32) * rows + r];
            const double v = e4m3_value(q[r * K + k]);
            if (c == 255 || isnan(v)) { bad = 1; out[r * K + k] = 0; continue; }
            const double w = ldexp(v, (int)c - 127);
            const float f = (float)w;
            uint32_t u;
            memcpy(&u, &f, sizeof u);
            if ((double)f != w || (u & 0xffffu)) { bad = 1; out[r * K + k] = 0; continue; }
            out[r * K + k] = (uint16_t)(u >> 16);
        }
    return bad ? -1 : 0;
}

/*
 * NVFP4 expert weights ("Checkpoint formats: BF16, FP8, and NVFP4": "Welcome Beam" page, TL;DR;
 * section "Hardware Requirements": the NVFP4 checkpoint keeps most parameters in 4 bits for
 * Blackwell; the pages give no recipe).  Reading: NVIDIA's NVFP4 layout,
 *   E2M1 elements: sign s, exponent e (2 bits, bias 1), mantissa m (1 bit); e = 0 is subnormal,
 *                  m * 0.5; otherwise (1 + m/2) * 2^(e-1).  The 8 magnitudes: 0, 0.5, 1, 1.5, 2,
 *                  3, 4, 6.
 *   one E4M3 scale per 16 consecutive K elements of a weight row (a non-negative, finite code),
 *   one FP32 scale per weight matrix.
 * w[row][k] = e2m1(code(row, k)) * e4m3(scale[k/16][row]) * global, with two codes per byte:
 * element k of a row is the low nibble of byte k/2 when k is even, the high nibble when k is odd.
 * q [rows, K/2] uint8; scale [K/16, rows] uint8; out [rows, K] fp64.  Returns -1 (out undefined)
 * when any scale code has the sign bit set or is NaN.
 */
static double e2m1_value(uint8_t nibble)
{
    const int s = (nibble >> 3) & 1, e = (nibble >> 1) & 3, m = nibble & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + m / 2.0, e - 1);
    return s ? -mag : mag;
}

int oracle_dequant_nvfp4(int64_t rows, int K, const uint8_t *q, const uint8_t *scale, double global,
                         double *out)
{
    if (K % 16) return -1;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) {
            const uint8_t c = scale[(int64_t)(k / 16) * rows + r];
            const double sv = e4m3_value(c);
            if ((c & 0x80) || isnan(sv)) { bad = 1; out[r * K + k] = 0.0; continue; }
            const uint8_t byte = q[r * (K / 2) + k / 2];
            const uint8_t nib = (k & 1) ? (byte >> 4) : (byte & 15);
            out[r * K + k] = e2m1_value(nib) * sv * global;
        }
    return bad ? -1 : 0;
}

/*
 * The SwiGLU expert of oracle_expert_mlp with FP64 weights (for checkpoint formats whose
 * dequantised weights are not bf16 values): out = Wd (SiLU(Wg x) * (Wu x)) per row, FP64.
 * x_rows [n,H] bf16 bits; wg, wu [I,H] fp64; wd [H,I] fp64; out [n,H] fp64.
 */
void oracle_expert_mlp_f64(int64_t n, int H, int I, const uint16_t *x_rows, const double *wg,
                           const double *wu, const double *wd, double *out)
{
    const int64_t nb = (n + RB - 1) / RB;
    double *xb = (double *)malloc(sizeof(double) * (size_t)(nb * H * RB));
    double *hb = (double *)malloc(sizeof(double) * (size_t)(nb * I * RB));
    for (int64_t b = 0; b < nb; ++b) bf16_rows_to_block(x_rows, b * RB, (int)min64(RB, n - b * RB), H, xb + b * H * RB);

    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        for (int i = 0; i < I; ++i) {
            double g[RB], u[RB];
            dot_rows(H, xb + b * H * RB, wg + (int64_t)i * H, g);
            dot_rows(H, xb + b * H * RB, wu + (int64_t)i * H, u);
            for (int r = 0; r < RB; ++r) {
                const double act = g[r] / (1.0 + exp(-g[r]));  /* SiLU(g) */
                hb[(b * I + i) * RB + r] = act * u[r];
            }
        }

    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        for (int o = 0; o < H; ++o) {
            double acc[RB];
            dot_rows(I, hb + b * I * RB, wd + (int64_t)o * I, acc);
            for (int r = 0; r < RB && b * RB + r < n; ++r) out[(b * RB + r) * H + o] = acc[r];
        }
    free(xb);
    free(hb);
}

/*
 * MXFP8 activations for the block-scaled FP8 path (reading; the pages name FP8 checkpoints but
 * give no recipe, and a tensor-core product of FP8 weights needs FP8 activations too).  OCP MXFP8
 * applied to activation rows: every block of 32 consecutive K elements of a row shares one UE8M0
 * scale 2^(c - 127), c = 127 + the smallest integer e with amax <= 448 * 2^e (amax = the block's
 * largest magnitude; c = 0 for an all-zero block), and each element becomes the E4M3 value nearest
 * to v * 2^(127 - c), ties to even.  The layer then computes on the dequantised values.
 */
static uint8_t e4m3_round_code(double a)  /* |a| <= 448: nearest E4M3 value, ties to even */
{
    const int s = signbit(a) ? 1 : 0;
    const double m = fabs(a);
    const int e = m >= ldexp(1.0, -6) ? ilogb(m) : -6;   /* subnormals share the quantum 2^-9 */
    const double quantum = ldexp(1.0, e - 3);
    const double r = nearbyint(m / quantum) * quantum;    /* default rounding mode: half to even */
    if (r == 0.0) return (uint8_t)(s << 7);
    const int re = ilogb(r);
    if (re < -6) return (uint8_t)((s << 7) | (int)ldexp(r, 9));            /* subnormal: r = m 2^-9 */
    const int mant = (int)(ldexp(r, -re) * 8.0) - 8;
    return (uint8_t)((s << 7) | ((re + 7) << 3) | mant);
}

/* The UE8M0 scale code of a block with largest magnitude amax (finite). */
static int mx_scale_code(double amax)
{
    if (amax == 0.0) return 0;
    int e = ilogb(amax) - 8;
    if (amax > ldexp(448.0, e)) e += 1;
    return e + 127;
}

/*
 * rows x K activations v (fp64) -> E4M3 codes q [rows,K], scale codes scale [rows,K/32] and the
 * dequantised values deq [rows,K] (fp64; any of q, scale may be NULL).  Returns -1 if K % 32 or a
 * scale code falls outside 1..254 (an exponent UE8M0 cannot hold).
 */
int oracle_quant_mxfp8_rows(int64_t rows, int K, const double *v, uint8_t *q, uint8_t *scale, double *deq)
{
    if (K % 32) return -1;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t r = 0; r < rows; ++r)
        for (int kb = 0; kb < K / 32; ++kb) {
            const double *blk = v + r * K + kb * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(blk[i]));
            const int c = mx_scale_code(amax);
            if (amax != 0.0 && (c < 1 || c > 254)) { bad = 1; continue; }
            if (scale) scale[r * (K / 32) + kb] = (uint8_t)c;
            for (int i = 0; i < 32; ++i) {
                const uint8_t code = amax == 0.0 ? 0 : e4m3_round_code(ldexp(blk[i], 127 - c));
                if (q) q[r * K + kb * 32 + i] = code;
                deq[r * K + kb * 32 + i] = amax == 0.0 ? 0.0 : ldexp(e4m3_value(code), c - 127);
            }
        }
    return bad ? -1 : 0;
}

/*
 * The SwiGLU expert of the block-scaled FP8 path on n rows: x~ = MXFP8(x) per row, g = Wg x~,
 * u = Wu x~, h = SiLU(g) * u, h~ = MXFP8(h) per row (blocks of 32 along the intermediate axis),
 * out = Wd h~, all in FP64 on the dequantised values.  Weights are bf16 bits (an MXFP8 checkpoint's
 * dequantised weights are bf16 values).  x_rows [n,H] bf16 bits; wg, wu [I,H]; wd [H,I]; out [n,H].
 * Returns -1 for an activation block whose scale UE8M0 cannot hold.
 */
int oracle_expert_mlp_mx8(int64_t n, int H, int I, const uint16_t *x_rows, const uint16_t *wg,
                          const uint16_t *wu, const uint16_t *wd, double *out)
{
    if (H % 32 || I % 32) return -1;
    const int64_t nb = (n + RB - 1) / RB;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(n * H));
    double *xq = (double *)malloc(sizeof(double) * (size_t)(n * H));
    double *hd = (double *)malloc(sizeof(double) * (size_t)(n * I));
    double *hq = (double *)malloc(sizeof(double) * (size_t)(n * I));
    double *xb = (double *)malloc(sizeof(double) * (size_t)(nb * H * RB));
    double *hb = (double *)malloc(sizeof(double) * (size_t)(nb * I * RB));
    int rc = 0;
    for (int64_t q = 0; q < n * H; ++q) xd[q] = bf16_bits_to_double(x_rows[q]);
    if (oracle_quant_mxfp8_rows(n, H, xd, NULL, NULL, xq)) { rc = -1; goto done; }
    /* x~ in the blocked layout of dot_rows */
    for (int64_t b = 0; b < nb; ++b)
        for (int h = 0; h < H; ++h)
            for (int r = 0; r < RB; ++r)
                xb[(b * H + h) * RB + r] = b * RB + r < n ? xq[(b * RB + r) * H + h] : 0.0;

    #pragma omp parallel
    {
        double *wgr = (double *)malloc(sizeof(double) * (size_t)H);
        double *wur = (double *)malloc(sizeof(double) * (size_t)H);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < nb; ++b)
            for (int i = 0; i < I; ++i) {
                for (int h = 0; h < H; ++h) {
                    wgr[h] = bf16_bits_to_double(wg[(int64_t)i * H + h]);
                    wur[h] = bf16_bits_to_double(wu[(int64_t)i * H + h]);
                }
                double g[RB], u[RB];
                dot_rows(H, xb + b * H * RB, wgr, g);
                dot_rows(H, xb + b * H * RB, wur, u);
                for (int r = 0; r < RB && b * RB + r < n; ++r) {
                    const double silu_g = g[r] / (1.0 + exp(-g[r]));
                    hd[(b * RB + r) * I + i] = silu_g * u[r];
                }
            }
        free(wgr);
        free(wur);
    }
    if (oracle_quant_mxfp8_rows(n, I, hd, NULL, NULL, hq)) { rc = -1; goto done; }
    for (int64_t b = 0; b < nb; ++b)
        for (int i = 0; i < I; ++i)
            for (int r = 0; r < RB; ++r)
                hb[(b * I + i) * RB + r] = b * RB + r < n ? hq[(b * RB + r) * I + i] : 0.0;

    #pragma omp parallel
    {
        double *wdr = (double *)malloc(sizeof(double) * (size_t)I);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < nb; ++b)
            for (int o = 0; o < H; ++o) {
                const uint16_t *wd_row = wd + (int64_t)o * I;  /* W_down row o */
                for (int i = 0; i < I; ++i) wdr[i] = bf16_bits_to_double(wd_row[i]);
                double acc[RB];
                dot_rows(I, hb + b * I * RB, wdr, acc);
                for (int r = 0; r < RB && b * RB + r < n; ++r) out[(b * RB + r) * H + o] = acc[r];
            }
        free(wdr);
    }
done:
    free(xd);
    free(xq);
    free(hd);
    free(hq);
    free(xb);
    free(hb);
    return rc;
}

/*
 * NVFP4 activations for the 4-bit tensor-core path (reading; the pages name NVFP4 checkpoints
 * "for Blackwell" but give no recipe; a native FP4 product needs FP4 activations).  NVFP4 applied to
 * activation rows: a row scale g (a power of two), one E4M3 scale code per 16 consecutive K elements
 * and E2M1 elements:
 *   g = 2^e with e the smallest integer such that amax_row <= 2688 g (2688 = 6 x 448), when the row
 *       scale is per row; g = 1 otherwise (the caller's choice);
 *   s = the E4M3 value nearest to amax_block / (6 g) (ties to even, at most 448);
 *   q = the E2M1 value nearest to v / (s g) (ties to even, magnitudes above 6 become 6; 0 if s = 0);
 *   dequantised value q s g.
 * v [rows,K] fp64; codes [rows,K] (one E2M1 code per element, 0..15) and scale codes
 * [rows,K/16] (any may be NULL); g [rows] (out); deq [rows,K].  Returns -1 if K % 16.
 */
static double e2m1_round(double m)  /* m >= 0: nearest E2M1 magnitude, ties to even, at most 6 */
{
    if (m >= 6.0) return 6.0;
    const double quantum = m < 2.0 ? 0.5 : (m < 4.0 ? 1.0 : 2.0);
    const double rounded = nearbyint(m / quantum) * quantum;  /* half to even */
    return rounded > 6.0 ? 6.0 : rounded;
}

static uint8_t e2m1_code_of(double v)  /* v already on the E2M1 grid */
{
    const double m = fabs(v);
    const int s = signbit(v) ? 8 : 0;
    if (m < 1.0) return (uint8_t)(s | (m == 0.5 ? 1 : 0));
    const int e = ilogb(m);                        /* 0, 1 or 2 */
    const int mant = ldexp(m, -e) > 1.0 ? 1 : 0;
    return (uint8_t)(s | ((e + 1) << 1) | mant);
}

/*
 * alt (nullable): for each element, the largest change of its dequantised value that a decision taken
 * on a value off by at most eps (relative) could make: the block's E4M3 scale rounded the other way
 * (amax / (6 g) within eps of a rounding boundary) or the element's E2M1 code rounded the other way
 * (v / (s g) within 6 eps of a boundary; the decision variable's error is relative to the block's
 * largest element, 6 s g), or both at once: under the other scale c the element's code is again
 * either rounding within the same absolute window (6 eps max(s, a) / c in units of c g).  0 where no
 * such decision is that close.  It bounds what a quantiser working on values within eps of these
 * (FP32 ones, say) may legitimately give.
 */
static void nvfp4_block_alt(const double *blk, double g, double a, double s, double eps, double *alt)
{
    for (int i = 0; i < 16; ++i) {
        const double m = s > 0.0 ? fabs(blk[i]) / (s * g) : 0.0;
        const double q = s > 0.0 ? e2m1_round(m) : 0.0;
        double d = 0.0;
        if (s > 0.0) {
            const double lo = e2m1_round(fmax(0.0, m - 6.0 * eps)), hi = e2m1_round(m + 6.0 * eps);
            d = fmax(fabs(lo - q), fabs(hi - q)) * s * g;
        }
        /* the other scale: both E4M3 roundings of a within eps */
        const double cand[2] = {e4m3_value(e4m3_round_code(fmin(a * (1.0 - eps), 448.0))),
                                e4m3_value(e4m3_round_code(fmin(a * (1.0 + eps), 448.0)))};
        for (int c = 0; c < 2; ++c) {
            if (cand[c] == s) continue;
            double lo2 = 0.0, hi2 = 0.0;
            if (cand[c] > 0.0) {
                const double m2 = fabs(blk[i]) / (cand[c] * g), w2 = 6.0 * eps * fmax(s, a) / cand[c];
                lo2 = e2m1_round(fmax(0.0, m2 - w2));
                hi2 = e2m1_round(m2 + w2);
            }
            /* the change is convex in the new code, so the two ends of the window bound it */
            d = fmax(d, fmax(fabs(lo2 * cand[c] - q * s), fabs(hi2 * cand[c] - q * s)) * g);
        }
        alt[i] = d;
    }
}

int oracle_quant_nvfp4_rows_alt(int64_t rows, int K, const double *v, int per_row_scale, uint8_t *codes,
                                uint8_t *scale, double *g_out, double *deq, double eps, double *alt);

int oracle_quant_nvfp4_rows(int64_t rows, int K, const double *v, int per_row_scale, uint8_t *codes,
                            uint8_t *scale, double *g_out, double *deq)
{
    return oracle_quant_nvfp4_rows_alt(rows, K, v, per_row_scale, codes, scale, g_out, deq, 0.0, NULL);
}

int oracle_quant_nvfp4_rows_alt(int64_t rows, int K, const double *v, int per_row_scale, uint8_t *codes,
                                uint8_t *scale, double *g_out, double *deq, double eps, double *alt)
{
    if (K % 16) return -1;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *row = v + r * K;
        double g = 1.0;
        if (per_row_scale) {
            double amax = 0.0;
            for (int k = 0; k < K; ++k) amax = fmax(amax, fabs(row[k]));
            if (amax > 0.0) {
                int e = ilogb(amax / 2688.0);
                if (amax > ldexp(2688.0, e)) e += 1;
                while (e > -1074 && amax <= ldexp(2688.0, e - 1)) e -= 1;
                g = ldexp(1.0, e);
            }
        }
        g_out[r] = g;
        for (int kb = 0; kb < K / 16; ++kb) {
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) amax = fmax(amax, fabs(row[kb * 16 + i]));
            double a = amax / (6.0 * g);
            if (a > 448.0) a = 448.0;
            const uint8_t sc = e4m3_round_code(a);
            const double s = e4m3_value(sc);
            if (scale) scale[r * (K / 16) + kb] = sc;
            for (int i = 0; i < 16; ++i) {
                const double x = row[kb * 16 + i];
                double q = 0.0;
                if (s > 0.0) {
                    q = e2m1_round(fabs(x) / (s * g));
                    if (signbit(x)) q = -q;
                }
                if (codes) codes[r * K + kb * 16 + i] = e2m1_code_of(q);
                deq[r * K + kb * 16 + i] = q * s * g;
            }
            if (alt) nvfp4_block_alt(row + kb * 16, g, a, s, eps, alt + r * K + kb * 16);
        }
    }
    return 0;
}

/*
 * The SwiGLU expert of the 4-bit path on n rows: x~ = NVFP4(x) with a per-row power-of-two scale,
 * g = Wg x~, u = Wu x~, h = SiLU(g) * u, h~ = NVFP4(h) with row scale 1 (the h tiles are produced
 * a slice of the intermediate axis at a time, so no row-wide scale is known when they are
 * quantised), out = Wd h~, FP64 on the dequantised values; weights FP64 (NVFP4 dequantised).
 * x_rows [n,H] bf16 bits; wg, wu [I,H]; wd [H,I]; out [n,H].
 */
int oracle_expert_mlp_w4a4_env(int64_t n, int H, int I, const uint16_t *x_rows, const double *wg, const double *wu,
                               const double *wd, double eps, double *out, double *env);

int oracle_expert_mlp_w4a4(int64_t n, int H, int I, const uint16_t *x_rows, const double *wg, const double *wu,
                           const double *wd, double *out)
{
    return oracle_expert_mlp_w4a4_env(n, H, I, x_rows, wg, wu, wd, 0.0, out, NULL);
}

/*
 * The same with the envelope env [n,H] (nullable): env[r][o] = sum_i |Wd[o,i]| alt_i, alt the largest
 * legitimate change of h~_i (see oracle_quant_nvfp4_rows_alt) for decisions on values within eps.
 */
int oracle_expert_mlp_w4a4_env(int64_t n, int H, int I, const uint16_t *x_rows, const double *wg, const double *wu,
                               const double *wd, double eps, double *out, double *env)
{
    if (H % 16 || I % 16) return -1;
    const int64_t nb = (n + RB - 1) / RB;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(n * H));
    double *x4 = (double *)malloc(sizeof(double) * (size_t)(n * H));
    double *gx = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *hd = (double *)malloc(sizeof(double) * (size_t)(n * I));
    double *h4 = (double *)malloc(sizeof(double) * (size_t)(n * I));
    double *gh = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *xb = (double *)malloc(sizeof(double) * (size_t)(nb * H * RB));
    double *hb = (double *)malloc(sizeof(double) * (size_t)(nb * I * RB));
    for (int64_t q = 0; q < n * H; ++q) xd[q] = bf16_bits_to_double(x_rows[q]);
    oracle_quant_nvfp4_rows(n, H, xd, 1, NULL, NULL, gx, x4);
    for (int64_t b = 0; b < nb; ++b)
        for (int h = 0; h < H; ++h)
            for (int r = 0; r < RB; ++r)
                xb[(b * H + h) * RB + r] = b * RB + r < n ? x4[(b * RB + r) * H + h] : 0.0;

    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < nb; ++b)
        for (int i = 0; i < I; ++i) {
            double g[RB], u[RB];
            dot_rows(H, xb + b * H * RB, wg + (int64_t)i * H, g);
            dot_rows(H, xb + b * H * RB, wu + (int64_t)i * H, u);
            for (int r = 0; r < RB && b * RB + r < n; ++r) {
                const double silu4 = g[r] / (1.0 + exp(-g[r]));
                hd[(b * RB + r) * I + i] = silu4 * u[r];
            }
        }
    double *halt = env ? (double *)malloc(sizeof(double) * (size_t)(n * I)) : NULL;
    double *ab = env ? (double *)malloc(sizeof(double) * (size_t)(nb * I * RB)) : NULL;
    oracle_quant_nvfp4_rows_alt(n, I, hd, 0, NULL, NULL, gh, h4, eps, halt);
    if (env)
        for (int64_t b = 0; b < nb; ++b)
            for (int i = 0; i < I; ++i)
                for (int r = 0; r < RB; ++r)
                    ab[(b * I + i) * RB + r] = b * RB + r < n ? halt[(b * RB + r) * I + i] : 0.0;
    for (int64_t b = 0; b < nb; ++b)
        for (int i = 0; i < I; ++i)
            for (int r = 0; r < RB; ++r)
                hb[(b * I + i) * RB + r] = b * RB + r < n ? h4[(b * RB + r) * I + i] : 0.0;

    #pragma omp parallel
    {
        double *wabs = env ? (double *)malloc(sizeof(double) * (size_t)I) : NULL;
        #pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < nb; ++b)
            for (int o = 0; o < H; ++o) {
                double acc[RB];
                dot_rows(I, hb + b * I * RB, wd + (int64_t)o * I, acc);
                for (int r = 0; r < RB && b * RB + r < n; ++r) out[(b * RB + r) * H + o] = acc[r];
                if (env) {
                    for (int i = 0; i < I; ++i) wabs[i] = fabs(wd[(int64_t)o * I + i]);
                    dot_rows(I, ab + b * I * RB, wabs, acc);
                    for (int r = 0; r < RB && b * RB + r < n; ++r) env[(b * RB + r) * H + o] = acc[r];
                }
            }
        free(wabs);
    }
    free(halt);
    free(ab);
    free(xd);
    free(x4);
    free(gx);
    free(hd);
    free(h4);
    free(gh);
    free(xb);
    free(hb);
    return 0;
}
