/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU reference of the forward
 * pass of one DeepSeekMoE layer whose expert FFNs run as FP8 (E4M3) GEMMs with
 * fine-grained scaling.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant generator with the CUDA library.
 *
 * Arithmetic is IEEE double unless a step is defined in FP32 (the FP8 scale
 * S = amax/448 and the quotient x/S that decides the E4M3 code, the routing
 * decision value s+b, and the bias update).  Build with -ffp-contract=off and
 * without -ffast-math so that every float operation rounds exactly once.
 *
 * Sources (page title, section):
 *  [P4] "DeepSeek-V3 Technischer Bericht" (xyznot.com/de), "Kernideen" FP8
 *       bullet (E4M3 for all tensors, 1x128 activation tiles, 128x128 weight
 *       blocks, FP32 promotion every N_c = 128 accumulation steps) and
 *       "Methode" section 2 "DeepSeekMoE mit Auxiliary-Loss-Free Balancing"
 *       (layer output equation, sigmoid affinity, biased top-K_r gating
 *       equation, normalisation of g', bias step gamma = 0.001).
 *  [P1] "DeepSeek-V3 技術報告書：MLAと極小スパースMoEがもたらす超低コストフロンティアモデル"
 *       (singularity-lens.com), formula paragraph: X_FP8 = clip(round(X/S),
 *       -448, 448) with S = max|X|/448, and b <- b + gamma*sign(mean_f - f_i).
 *  [P2] "DeepSeek-V3 Technical Report" slides (slideify.app), "FP8
 *       Quantization Logic" box: 1x128 tiles, 128x128 blocks.
 *  [P3] "DeepSeek-V3 MoE 2024" glossary (jisaku.com), feature list: 256
 *       routed experts + 1 shared expert, top-8 per token.
 *
 * Parity pins: every function below is pinned by a CPU test (tests/test_oracle_*.py)
 * except the group-limited pre-selection, whose group-score rule the pages do
 * not state ("parity unpinned" by the pages; its implementation is pinned by
 * brute force against the stated reading only).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QBLK 128 /* N_c and the tile edge of [P4] "Kernideen" */

/* ---------------------------------------------------------------- helpers */

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bf16 with round-to-nearest-even: bf16 keeps 8
 * significant bits, so scale the value until its last kept bit is the units
 * place, round to an integer (ties to even) and scale back. */
static uint16_t double_to_bf16_rne(double v)
{
    float f;
    uint32_t u;
    if (v == 0.0 || !isfinite(v)) {
        f = (float)v;
    } else {
        int e;
        frexp(v, &e);           /* |v| in [2^(e-1), 2^e) */
        int lsb = e - 8;        /* weight of the last kept bit */
        if (lsb < -133) lsb = -133; /* bf16 subnormal grid */
        f = (float)ldexp(nearbyint(ldexp(v, -lsb)), lsb); /* exact in float */
    }
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ E4M3 */
/* OCP FP8 E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits, no
 * infinities, S.1111.111 is NaN, largest finite 448 (the clip bound of [P1]),
 * subnormals m/8 * 2^-6. */

double moe_oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a float to the nearest E4M3 value, ties to even, saturating at +-448
 * ("clip(round(X/S), -448, 448)" of [P1]). */
uint8_t moe_oracle_e4m3_encode(float xf)
{
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid: multiples of 2^-9 */
        double q = a * 512.0;          /* exact: power-of-two scaling */
        int m = (int)nearbyint(q);     /* default rounding mode: ties to even */
        if (m == 8) return (uint8_t)(sign | 0x08);
        return (uint8_t)(sign | m);
    }
    int ex;
    double fr = frexp(a, &ex);         /* a = fr * 2^ex, fr in [0.5, 1) */
    int e = ex - 1;                    /* a = (2 fr) * 2^e */
    double mant = (2.0 * fr - 1.0) * 8.0; /* exact */
    int m = (int)nearbyint(mant);
    if (m == 8) { m = 0; e += 1; }
    int be = e + 7;
    if (be > 15 || (be == 15 && m > 6)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (be << 3) | m);
}

/* Shared step of both quantizers: with S = amax/448 in FP32 ([P1]), each
 * element's code is E4M3(x/S) with x/S an IEEE FP32 quotient.  amax == 0 gives
 * S = 0 and all codes 0x00.
 *
 * Scale mode 1 (not on the pages: the variant whose scales a tensor core can
 * apply itself, power-of-two "E8M0" scale factors): S = 2^e with e the
 * smallest integer for which amax <= 448 * 2^e, so the tile's largest
 * magnitude still fits the E4M3 range and x/S is an exact power-of-two
 * scaling; e is held at -127 or above (the smallest such scale factor).
 * amax == 0 again gives S = 0. */
static float scale_pow2(float amax)
{
    if (amax == 0.0f) return 0.0f;
    const double a = (double)amax;
    int e = ilogb(a) - 9;                  /* 448 * 2^e < a here */
    while (ldexp(448.0, e) < a) ++e;       /* exact comparisons in double: the first e that fits */
    if (e < -127) e = -127;
    return (float)ldexp(1.0, e);           /* exact: 2^e >= 2^-127 is a float */
}

static float scale_for(float amax, int mode) { return mode ? scale_pow2(amax) : amax / 448.0f; }

static uint8_t code_of(float x, float S)
{
    if (S == 0.0f) return 0x00;
    float q = x / S;
    return moe_oracle_e4m3_encode(q);
}

/* 1x128 activation tiles ([P4] "Kernideen", [P2]): one FP32 scale per row per
 * 128 consecutive columns.  x is bf16 [rows, ldx], q [rows, cols], s [rows,
 * cols/128]. */
void moe_oracle_quant_1x128_bf16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx,
                                 uint8_t *q, float *s, int mode)
{
    int64_t ng = cols / QBLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const uint16_t *xr = x + r * ldx + g * QBLK;
            float amax = 0.0f;
            for (int j = 0; j < QBLK; ++j) {
                float a = fabsf(bf16_to_float(xr[j]));
                if (a > amax) amax = a;
            }
            float S = scale_for(amax, mode);
            s[r * ng + g] = S;
            for (int j = 0; j < QBLK; ++j)
                q[r * cols + g * QBLK + j] = code_of(bf16_to_float(xr[j]), S);
        }
    }
}

/* Same tiling for an FP32 input (the SwiGLU output h before the down
 * projection, re-quantized along the intermediate dimension). */
void moe_oracle_quant_1x128_f32(const float *x, int64_t rows, int64_t cols, uint8_t *q, float *s, int mode)
{
    int64_t ng = cols / QBLK;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < ng; ++g) {
            const float *xr = x + r * cols + g * QBLK;
            float amax = 0.0f;
            for (int j = 0; j < QBLK; ++j) {
                float a = fabsf(xr[j]);
                if (a > amax) amax = a;
            }
            float S = scale_for(amax, mode);
            s[r * ng + g] = S;
            for (int j = 0; j < QBLK; ++j) q[r * cols + g * QBLK + j] = code_of(xr[j], S);
        }
    }
}

/* 128x128 weight blocks ([P4] "Kernideen", [P2]): w bf16 [n, k] (rows = output
 * features, k contiguous), q [n, k], s [n/128, k/128]. */
void moe_oracle_quant_128x128(const uint16_t *w, int64_t n, int64_t k, uint8_t *q, float *s, int mode)
{
    int64_t nb = n / QBLK, kb = k / QBLK;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bi = 0; bi < nb; ++bi) {
        for (int64_t bj = 0; bj < kb; ++bj) {
            float amax = 0.0f;
            for (int i = 0; i < QBLK; ++i)
                for (int j = 0; j < QBLK; ++j) {
                    float a = fabsf(bf16_to_float(w[(bi * QBLK + i) * k + bj * QBLK + j]));
                    if (a > amax) amax = a;
                }
            float S = scale_for(amax, mode);
            s[bi * kb + bj] = S;
            for (int i = 0; i < QBLK; ++i)
                for (int j = 0; j < QBLK; ++j) {
                    int64_t o = (bi * QBLK + i) * k + bj * QBLK + j;
                    q[o] = code_of(bf16_to_float(w[o]), S);
                }
        }
    }
}

/* ------------------------------------------------- block-scaled FP8 GEMM */
/* C[m][n] = sum over 128-wide K blocks kb of sA[m][kb] * sB[n/128][kb] * P,
 * P = sum_{k in kb} dec(A[m][k]) * dec(B[n][k]).  This is the definition of
 * the fine-grained-scaled product with promotion every N_c = 128 steps
 * ([P4] "Kernideen"): each 128-long partial is formed first, then scaled and
 * accumulated.  In double, P is exact (a product of two E4M3 values has at
 * most 8 significant bits and exponents within [-18, 17], so 128 of them sum
 * exactly in 53 bits).  A [M, K] (1x128 scales sA [M, K/128]); B [N, K]
 * (128x128 scales sB [N/128, K/128]); C [M, N] in double. */

static double g_dec[256];
static int g_dec_ready = 0;

static void init_dec(void)
{
    if (g_dec_ready) return;
    for (int c = 0; c < 256; ++c) g_dec[c] = moe_oracle_e4m3_decode((uint8_t)c);
    g_dec_ready = 1;
}

static double block_dot(const uint8_t *a, const uint8_t *b)
{
    double p = 0.0;
    for (int k = 0; k < QBLK; ++k) p += g_dec[a[k]] * g_dec[b[k]];
    return p;
}

static double scaled_row_dot(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb_row, int64_t K)
{
    double acc = 0.0;
    for (int64_t kb = 0; kb < K / QBLK; ++kb)
        acc += ((double)sa[kb] * (double)sb_row[kb]) * block_dot(a + kb * QBLK, b + kb * QBLK);
    return acc;
}

void moe_oracle_blockscaled_gemm(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                 int64_t M, int64_t N, int64_t K, double *C)
{
    init_dec();
    int64_t kbn = K / QBLK;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            C[m * N + n] = scaled_row_dot(A + m * K, sA + m * kbn, B + n * K, sB + (n / QBLK) * kbn, K);
}

/* --------------------------------------------------------------- routing */
/* [P4] Methode 2: s_{i,t} = Sigmoid(u_t^T e_i); an expert is selected when
 * s_{i,t} + b_i is among the K_r largest of {s_{j,t} + b_j}; g'_{i,t} = s_{i,t}
 * for selected experts, else 0; g = g' normalised over the selected set.
 *
 * Readings where the pages are silent:
 *  - the logit is summed in double over the bf16 products; s is a double;
 *  - the selection decision compares c_i = fp32(s_i) + b_i in FP32, the
 *    precision the GPU takes it in; equal c: lower expert index first;
 *  - optional group-limited pre-selection: experts [g*N_r/G, (g+1)*N_r/G)
 *    form group g, score(g) = sum (FP32) of the two largest c in the group,
 *    the top `topk_groups` groups (ties: lower index) stay eligible;
 *  - g = route_scale * s_i / sum_selected s_j (route_scale = 1 by default).
 * gap[t] is min over the decision boundaries taken for token t of (last
 * chosen - first rejected) score, so near-ties can be recognised. */
typedef struct {
    int32_t H, I, Nr, Kr, Ns, n_groups, topk_groups;
    int32_t scale_mode; /* 0: S = amax/448 (the pages); 1: power-of-two S (see scale_pow2) */
    double route_scale;
} moe_oracle_cfg;

static void route_token(const uint16_t *xr, const uint16_t *Wr, const float *bias, const moe_oracle_cfg *cf,
                        int32_t *idx, double *gate, float *gap, double *s_buf, float *c_buf, unsigned char *ok)
{
    int Nr = cf->Nr, H = cf->H;
    for (int i = 0; i < Nr; ++i) {
        double z = 0.0;
        const uint16_t *w = Wr + (int64_t)i * H;
        for (int h = 0; h < H; ++h) z += (double)bf16_to_float(xr[h]) * (double)bf16_to_float(w[h]);
        s_buf[i] = 1.0 / (1.0 + exp(-z));
        c_buf[i] = (float)s_buf[i] + bias[i];
        ok[i] = 1;
    }
    float g_gap = INFINITY;
    if (cf->n_groups > 0) {
        int G = cf->n_groups, gs = Nr / G;
        float score[64];
        for (int g = 0; g < G; ++g) {
            float b1 = -INFINITY, b2 = -INFINITY;
            for (int j = g * gs; j < (g + 1) * gs; ++j) {
                float c = c_buf[j];
                if (c > b1) { b2 = b1; b1 = c; }
                else if (c > b2) b2 = c;
            }
            score[g] = b1 + b2;
        }
        unsigned char keep[64] = {0};
        float last = INFINITY;
        for (int r = 0; r < cf->topk_groups; ++r) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!keep[g] && (best < 0 || score[g] > score[best])) best = g;
            keep[best] = 1;
            last = score[best];
        }
        float next = -INFINITY;
        for (int g = 0; g < G; ++g)
            if (!keep[g] && score[g] > next) next = score[g];
        if (cf->topk_groups < G) g_gap = last - next;
        for (int j = 0; j < Nr; ++j) ok[j] = keep[j / gs];
    }
    float last = INFINITY;
    double ssum = 0.0;
    for (int r = 0; r < cf->Kr; ++r) {
        int best = -1;
        for (int j = 0; j < Nr; ++j)
            if (ok[j] && (best < 0 || c_buf[j] > c_buf[best])) best = j;
        ok[best] = 0; /* taken */
        idx[r] = best;
        last = c_buf[best];
        ssum += s_buf[best];
    }
    float next = -INFINITY;
    for (int j = 0; j < Nr; ++j)
        if (ok[j] && c_buf[j] > next) next = c_buf[j];
    float e_gap = (next == -INFINITY) ? INFINITY : last - next;
    *gap = e_gap < g_gap ? e_gap : g_gap;
    for (int r = 0; r < cf->Kr; ++r) gate[r] = cf->route_scale * s_buf[idx[r]] / ssum;
}

/* x bf16 [T, H]; Wr bf16 [Nr, H]; bias f32 [Nr]; idx i32 [T, Kr] in
 * descending-score order; gate f64 [T, Kr]; gap f32 [T]; s_out (nullable) f64
 * [T, Nr] sigmoid affinities. */
void moe_oracle_route(const moe_oracle_cfg *cf, const uint16_t *x, int64_t T, const uint16_t *Wr,
                      const float *bias, int32_t *idx, double *gate, float *gap, double *s_out)
{
    int Nr = cf->Nr;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * Nr);
        float *c_buf = (float *)malloc(sizeof(float) * Nr);
        unsigned char *ok = (unsigned char *)malloc((size_t)Nr);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            route_token(x + t * cf->H, Wr, bias, cf, idx + t * cf->Kr, gate + t * cf->Kr, gap + t, s_buf, c_buf, ok);
            if (s_out) memcpy(s_out + t * Nr, s_buf, sizeof(double) * Nr);
        }
        free(s_buf);
        free(c_buf);
        free(ok);
    }
}

/* ------------------------------------------------------------ expert FFN */
/* One expert applied to one token, SwiGLU form W2(silu(W1 u) * (W3 u)):
 *   xq, xs   : the token's 1x128-quantized input (H codes, H/128 scales);
 *   W13q,s13 : [2I, H] codes, rows 0..I-1 = W1 (gate), I..2I-1 = W3 (up),
 *              128x128 scales [2I/128, H/128];
 *   W2q, s2  : [H, I] codes, scales [H/128, I/128];
 * Steps: G, U by the block-scaled product above, rounded to FP32 (the FP32
 * accumulator of [P4] "Kernideen"); h = silu(G) * U in double, rounded to FP32;
 * h re-quantized 1x128 along I ("E4M3 for all tensors"); y = block-scaled
 * product with W2, left in double.  Optional outputs: h (f32 [I]), hq/hs. */
static void expert_ffn(const moe_oracle_cfg *cf, const uint8_t *xq, const float *xs, const uint8_t *W13q,
                       const float *s13, const uint8_t *W2q, const float *s2, double *y, float *h_buf,
                       uint8_t *hq_buf, float *hs_buf)
{
    int H = cf->H, I = cf->I;
    int hk = H / QBLK, ik = I / QBLK;
    for (int j = 0; j < I; ++j) {
        float G = (float)scaled_row_dot(xq, xs, W13q + (int64_t)j * H, s13 + (int64_t)(j / QBLK) * hk, H);
        float U = (float)scaled_row_dot(xq, xs, W13q + (int64_t)(I + j) * H, s13 + (int64_t)((I + j) / QBLK) * hk, H);
        double g = (double)G;
        double silu = g / (1.0 + exp(-g));
        h_buf[j] = (float)(silu * (double)U);
    }
    moe_oracle_quant_1x128_f32(h_buf, 1, I, hq_buf, hs_buf, cf->scale_mode);
    for (int n = 0; n < H; ++n)
        y[n] = scaled_row_dot(hq_buf, hs_buf, W2q + (int64_t)n * I, s2 + (int64_t)(n / QBLK) * ik, I);
}

/* Single expert applied to several token rows (used by the GEMM/FFN pins and
 * by tests that check one expert in isolation).  xq [n, H], xs [n, H/128];
 * y [n, H] double; h (nullable) f32 [n, I]; hq (nullable) [n, I]; hs
 * (nullable) [n, I/128]. */
void moe_oracle_expert_ffn(const moe_oracle_cfg *cf, const uint8_t *xq, const float *xs, int64_t n,
                           const uint8_t *W13q, const float *s13, const uint8_t *W2q, const float *s2,
                           double *y, float *h, uint8_t *hq, float *hs)
{
    init_dec();
    int H = cf->H, I = cf->I;
#pragma omp parallel
    {
        float *hb = (float *)malloc(sizeof(float) * I);
        uint8_t *qb = (uint8_t *)malloc((size_t)I);
        float *sb = (float *)malloc(sizeof(float) * (I / QBLK));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < n; ++r) {
            expert_ffn(cf, xq + r * H, xs + r * (H / QBLK), W13q, s13, W2q, s2, y + r * H, hb, qb, sb);
            if (h) memcpy(h + r * I, hb, sizeof(float) * I);
            if (hq) memcpy(hq + r * I, qb, (size_t)I);
            if (hs) memcpy(hs + r * (I / QBLK), sb, sizeof(float) * (I / QBLK));
        }
        free(hb);
        free(qb);
        free(sb);
    }
}

/* ------------------------------------------------------------ full layer */
/* [P4] Methode 2: h'_t = u_t + sum_{i<=N_s} FFN^(s)_i(u_t) + sum_i g_{i,t} FFN^(r)_i(u_t).
 * Per listed token: quantize u_t (1x128), route it (using the same u_t in
 * bf16), apply the shared expert(s) and the K_r selected routed experts to
 * the quantized u_t, and sum in double.
 *   tokens  : indices into x of the rows to compute (n_tok of them);
 *   W13q[e], s13[e], W2q[e], s2[e] : per-expert pointers, e in [0, Nr) routed,
 *             e in [Nr, Nr+Ns) shared; a pointer may be NULL for an expert no
 *             listed token selects (returns -1 if one is needed);
 *   out     : [n_tok, H] double, unrounded layer output;
 *   out_bf16: (nullable) [n_tok, H] bf16 RNE of out;
 *   idx, gate, gap : routing of the listed tokens (as moe_oracle_route).
 * Returns 0 on success, -1 if a needed expert pointer is NULL. */
int moe_oracle_forward(const moe_oracle_cfg *cf, const uint16_t *x, const int64_t *tokens, int64_t n_tok,
                       const uint16_t *Wr, const float *bias, const uint8_t *const *W13q,
                       const float *const *s13, const uint8_t *const *W2q, const float *const *s2,
                       double *out, uint16_t *out_bf16, int32_t *idx, double *gate, float *gap)
{
    init_dec();
    int H = cf->H, I = cf->I, Nr = cf->Nr, Kr = cf->Kr, Ns = cf->Ns;
    int missing = 0;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * Nr);
        float *c_buf = (float *)malloc(sizeof(float) * Nr);
        unsigned char *ok = (unsigned char *)malloc((size_t)Nr);
        uint8_t *xq = (uint8_t *)malloc((size_t)H);
        float *xs = (float *)malloc(sizeof(float) * (H / QBLK));
        double *y = (double *)malloc(sizeof(double) * H);
        float *hb = (float *)malloc(sizeof(float) * I);
        uint8_t *qb = (uint8_t *)malloc((size_t)I);
        float *sb = (float *)malloc(sizeof(float) * (I / QBLK));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_tok; ++r) {
            const uint16_t *u = x + tokens[r] * H;
            double *o = out + r * H;
            moe_oracle_quant_1x128_bf16(u, 1, H, H, xq, xs, cf->scale_mode);
            route_token(u, Wr, bias, cf, idx + r * Kr, gate + r * Kr, gap + r, s_buf, c_buf, ok);
            for (int n = 0; n < H; ++n) o[n] = (double)bf16_to_float(u[n]);
            for (int e = Nr; e < Nr + Ns; ++e) {
                if (!W13q[e] || !W2q[e]) { missing = 1; continue; }
                expert_ffn(cf, xq, xs, W13q[e], s13[e], W2q[e], s2[e], y, hb, qb, sb);
                for (int n = 0; n < H; ++n) o[n] += y[n];
            }
            for (int k = 0; k < Kr; ++k) {
                int e = idx[r * Kr + k];
                if (!W13q[e] || !W2q[e]) { missing = 1; continue; }
                expert_ffn(cf, xq, xs, W13q[e], s13[e], W2q[e], s2[e], y, hb, qb, sb);
                double g = gate[r * Kr + k];
                for (int n = 0; n < H; ++n) o[n] += g * y[n];
            }
            if (out_bf16)
                for (int n = 0; n < H; ++n) out_bf16[r * H + n] = double_to_bf16_rne(o[n]);
        }
        free(s_buf); free(c_buf); free(ok); free(xq); free(xs); free(y); free(hb); free(qb); free(sb);
    }
    return missing ? -1 : 0;
}

/* ---------------------------------------------------------- bias update */
/* [P4] Methode 2: at the end of a step an overloaded expert gets b_i -= gamma,
 * an underloaded one b_i += gamma (gamma = 0.001); [P1] writes the same rule
 * as b_i += gamma * sign(mean_f - f_i).  load_i = counts[i] assignments,
 * mean = total / Nr; the comparison is done exactly in integers
 * (counts[i] * Nr vs total) and the step in FP32. */
void moe_oracle_bias_update(float *bias, const int32_t *counts, int Nr, int64_t total, float gamma)
{
    for (int i = 0; i < Nr; ++i) {
        int64_t d = (int64_t)counts[i] * Nr - total;
        if (d > 0) bias[i] = bias[i] - gamma;
        else if (d < 0) bias[i] = bias[i] + gamma;
    }
}

/* bf16 RNE of doubles (exported for tests that compare rounded outputs). */
void moe_oracle_round_bf16(const double *v, int64_t n, uint16_t *o)
{
    for (int64_t i = 0; i < n; ++i) o[i] = double_to_bf16_rne(v[i]);
}

int moe_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the following parallel regions started from the calling thread
 * (timing of the oracle with a chosen thread count). */
void moe_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
