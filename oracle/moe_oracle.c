/*
 * moe_oracle.c -- plain, slow, double-precision CPU reference of one step of
 * the top-k mixture-of-experts FFN layer with FP8 (e4m3) block-scaled weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA product path; the product never
 * calls it and must fail loudly if its own CUDA library is missing.
 *
 * What it follows (the reference pages):
 *  - "Qwen3.6-35B-A3B-FP8 on NVIDIA GB10" blueprint page, "Kernels" table:
 *    the per-layer MoE chain is a bf16 router GEMV (gemv::dense_gemv_bf16),
 *    top-k softmax (moe_topk::moe_topk_softmax), the routed+shared expert
 *    gate/up product over FP8 weights (moe_expert_gate_up_shared_fp8), the
 *    SiLU-times-up then down product (moe_expert_silu_down_shared_fp8) and
 *    the weighted blend (moe_expert_gemv::moe_weighted_sum_blend).
 *  - same page, "Precision" table: weights fp8/block128x128, read against
 *    bf16 activations (gate/up) and f32 activations (down); top-k node
 *    output f32,i32.
 *  - "colibri #1992" PR page, description of frame A2: the shared expert is
 *    applied together with its gate.
 *  - "Neurarch Qwen3-8B" page, exported PyTorch, swiglu block: gate_proj and
 *    up_proj are [I,H], down_proj is [H,I] (LLaMA-style SwiGLU).
 *  - OCP 8-bit Floating Point specification, E4M3: exponent bias 7, three
 *    mantissa bits, subnormals, no infinities, S.1111.111 is NaN, max 448.
 *  - "The Config That Launched a Thousand GPUs: Inspecting
 *    Qwen3.5-397B-A17B-NVFP4" page: the 397B checkpoint's experts are stored
 *    in NVFP4 (modelopt).  The format (not on the pages; its public
 *    definition): OCP MX E2M1 codes (one sign bit, two exponent bits with
 *    bias 1, one mantissa bit, no infinities or NaN: 0, 0.5, 1, 1.5, 2, 3,
 *    4, 6), one E4M3 scale per 16 consecutive elements along the reduction
 *    dimension, one fp32 scale per tensor.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - top-k ties go to the lower expert index; output order is by descending
 *    logit;
 *  - "softmax then renormalise" over the k selected logits equals a softmax
 *    restricted to those k logits (closed form used here);
 *  - the shared expert gate is sigmoid(g . x) with g a length-H vector, and
 *    it scales only the shared expert's output;
 *  - dequantised weight = e4m3(q) * s(block), s an fp32 per 128x128 block;
 *  - the optional router bias (one value per expert) is added to the logits
 *    before selection; the optional residual is added before the final
 *    rounding to bf16.
 *
 * Everything is computed in double from the exact values of the bf16 and
 * e4m3 inputs.  No blocking, fusion or reordering beyond the definitions.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t hidden;       /* H  */
    int32_t n_experts;    /* E  */
    int32_t top_k;        /* k  */
    int32_t inter;        /* I  : routed expert intermediate size */
    int32_t shared_inter; /* Is : shared expert intermediate size */
} oracle_dims;

/* ------------------------------------------------------------------ bf16 */

/* bf16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), directly from the
 * double (no intermediate float rounding).  Overflow goes to +-inf. */
uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    int e;
    (void)frexp(fabs(v), &e); /* |v| = m * 2^e with m in [0.5, 1) */
    /* bf16 keeps 8 significant bits; the smallest exponent of the last
     * place is 2^-133 (subnormal step). */
    int lsb_exp = e - 8;
    if (lsb_exp < -133) lsb_exp = -133;
    double q = nearbyint(ldexp(fabs(v), -lsb_exp)); /* default mode: ties to even */
    double r = ldexp(q, lsb_exp);
    if (r > 3.3895313892515355e38) { /* above the largest finite bf16 */
        return signbit(v) ? 0xFF80 : 0x7F80;
    }
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    return signbit(v) ? (uint16_t)(b | 0x8000) : b;
}

/* ------------------------------------------------------------------ e4m3 */

/* OCP E4M3: s eeee mmm, bias 7.  e == 0: subnormal m/8 * 2^-6.
 * e == 15 and m == 7: NaN.  No infinities.  Largest finite 1.75 * 2^8. */
double oracle_e4m3_decode(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest e4m3 value, ties to the even code (even mantissa), saturating
 * finite values beyond 448 to +-448; NaN maps to 0x7F.  Codes 0x00..0x7E
 * have strictly increasing values, so a binary search over them is the
 * plain definition of "nearest". */
uint8_t oracle_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E; /* invariant: decode(lo) <= a < decode(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (oracle_e4m3_decode((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dl = a - oracle_e4m3_decode((uint8_t)lo);
    double dh = oracle_e4m3_decode((uint8_t)hi) - a;
    int c;
    if (dl < dh)
        c = lo;
    else if (dh < dl)
        c = hi;
    else
        c = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | c);
}

/* Block quantiser for a row-major fp32 matrix [rows, cols], both multiples
 * of 128: per 128x128 block, s = amax / 448 in fp32 (an all-zero block gets
 * s = 1), q = e4m3(w / s) with the quotient formed in fp32.  scales is
 * [rows/128, cols/128] row-major. */
int oracle_quantize_blocks(const float *w, int64_t rows, int64_t cols,
                           uint8_t *q, float *scales)
{
    if (rows % 128 || cols % 128) return -2;
    int64_t br = rows / 128, bc = cols / 128;
    for (int64_t bi = 0; bi < br; ++bi) {
        for (int64_t bj = 0; bj < bc; ++bj) {
            float amax = 0.0f;
            for (int64_t r = bi * 128; r < bi * 128 + 128; ++r)
                for (int64_t c = bj * 128; c < bj * 128 + 128; ++c) {
                    float a = fabsf(w[r * cols + c]);
                    if (a > amax) amax = a;
                }
            float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
            scales[bi * bc + bj] = s;
            for (int64_t r = bi * 128; r < bi * 128 + 128; ++r)
                for (int64_t c = bj * 128; c < bj * 128 + 128; ++c) {
                    float qv = w[r * cols + c] / s;
                    q[r * cols + c] = oracle_e4m3_encode((double)qv);
                }
        }
    }
    return 0;
}

/* Dequantised weight of a [rows, cols] e4m3 matrix with [rows/128, cols/128]
 * fp32 block scales: e4m3(q[r, c]) * s[r/128, c/128]. */
static double dq(const uint8_t *q, const float *s, int64_t cols, int64_t r, int64_t c)
{
    return oracle_e4m3_decode(q[r * cols + c]) * (double)s[(r / 128) * (cols / 128) + (c / 128)];
}

/* ------------------------------------------------------------- NVFP4 */

/* OCP MX E2M1: code = s.ee.m, exponent bias 1; e = 0 is subnormal (m * 0.5). */
double oracle_e2m1_decode(uint8_t code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return s ? -v : v;
}

/* Nearest e2m1 value, ties to the even code (even mantissa), saturating to
 * +-6; codes 0..7 have strictly increasing values (binary search, as for
 * e4m3).  NaN maps to 0. */
uint8_t oracle_e2m1_encode(double v)
{
    if (isnan(v)) return 0;
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    if (a >= 6.0) return (uint8_t)(sign | 0x7);
    int lo = 0, hi = 7; /* invariant: decode(lo) <= a < decode(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (oracle_e2m1_decode((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dl = a - oracle_e2m1_decode((uint8_t)lo);
    double dh = oracle_e2m1_decode((uint8_t)hi) - a;
    int c;
    if (dl < dh)
        c = lo;
    else if (dh < dl)
        c = hi;
    else
        c = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | c);
}

/* NVFP4 quantiser for a row-major fp32 matrix [rows, cols], cols a multiple
 * of 16 (reading of the format: the tensor scale maps the largest magnitude
 * to the largest e4m3 scale times the largest e2m1 value):
 *   gs = amax / (448 * 6) in fp32 (1 for an all-zero matrix);
 *   per 16 consecutive elements of a row: sf = e4m3(amax16 / (6 * gs)),
 *     quotient in fp32;
 *   code = e2m1(w / (e4m3(sf) * gs)), divisor and quotient in fp32 (a zero
 *     block scale gives code 0);
 * codes packed two to a byte, element 2j in the low nibble of byte j:
 * q4 [rows, cols/2], sf [rows, cols/16] e4m3 codes, *gs. */
int oracle_quantize_nvfp4(const float *w, int64_t rows, int64_t cols, uint8_t *q4, uint8_t *sf, float *gs)
{
    if (cols % 16) return -2;
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * cols; ++i)
        if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
    const float g = (amax == 0.0f) ? 1.0f : amax / (448.0f * 6.0f);
    *gs = g;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 16; ++b) {
            float bmax = 0.0f;
            for (int64_t c = b * 16; c < b * 16 + 16; ++c)
                if (fabsf(w[r * cols + c]) > bmax) bmax = fabsf(w[r * cols + c]);
            const float sq = bmax / (6.0f * g);
            const uint8_t sc = oracle_e4m3_encode((double)sq);
            sf[r * (cols / 16) + b] = sc;
            const float div = (float)oracle_e4m3_decode(sc) * g;
            for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
                uint8_t code = 0;
                if (div != 0.0f) {
                    const float qv = w[r * cols + c] / div;
                    code = oracle_e2m1_encode((double)qv);
                }
                uint8_t *byte = &q4[r * (cols / 2) + c / 2];
                if (c % 2 == 0)
                    *byte = (uint8_t)((*byte & 0xF0) | code);
                else
                    *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
            }
        }
    }
    return 0;
}

/* Dequantised weight of a [rows, cols] NVFP4 matrix: e2m1(code) * e4m3(sf)
 * * gs. */
static double dq4(const uint8_t *q4, const uint8_t *sf, double gs, int64_t cols, int64_t r, int64_t c)
{
    const uint8_t byte = q4[r * (cols / 2) + c / 2];
    const uint8_t code = (c % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    return oracle_e2m1_decode(code) * oracle_e4m3_decode(sf[r * (cols / 16) + c / 16]) * gs;
}

/* ------------------------------------------------------------- RMSNorm */

/* The norm in front of the MoE block ("Qwen3.6-35B-A3B-FP8 on NVIDIA GB10"
 * blueprint page, Kernels table: norm::rms_norm and
 * norm::residual_add_rms_norm, whose bf16 output feeds the router GEMV;
 * "Neurarch Qwen3-8B" page: RMSNorm over the hidden size before each SwiGLU
 * block).  For each row r of the residual stream (bf16 [rows, H]):
 *   ms = sum_h r_h^2 / H,  inv = 1 / sqrt(ms + eps),  x_h = (r_h * inv) * w_h,
 * in double; xd (nullable) receives x before rounding, x_bf16 the nearest
 * bf16 (ties to even) of each x_h. */
int oracle_rmsnorm(int32_t H, int32_t rows, const uint16_t *resid, const uint16_t *norm_w, double eps,
                   double *xd, uint16_t *x_bf16)
{
    if (H <= 0 || rows < 0 || !resid || !norm_w || !x_bf16 || !(eps >= 0.0)) return -1;
    for (int t = 0; t < rows; ++t) {
        const uint16_t *r = resid + (int64_t)t * H;
        double ss = 0.0;
        for (int h = 0; h < H; ++h) {
            double v = oracle_bf16_to_f64(r[h]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int h = 0; h < H; ++h) {
            double v = (oracle_bf16_to_f64(r[h]) * inv) * oracle_bf16_to_f64(norm_w[h]);
            if (xd) xd[(int64_t)t * H + h] = v;
            x_bf16[(int64_t)t * H + h] = oracle_f64_to_bf16(v);
        }
    }
    return 0;
}

/* ------------------------------------------------------------ the layer */

static double sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

/* Router logits and shared-gate pre-activation for one row:
 * l[e] = sum_h x[h] * Wr[e, h] (+ bias[e]),  z = sum_h x[h] * g[h]. */
static void router_row(const oracle_dims *d, const uint16_t *x, const uint16_t *router_w,
                       const float *router_bias, const uint16_t *shared_gate,
                       double *l, double *z)
{
    const int H = d->hidden, E = d->n_experts;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h)
            acc += oracle_bf16_to_f64(x[h]) * oracle_bf16_to_f64(router_w[(int64_t)e * H + h]);
        if (router_bias) acc += (double)router_bias[e];
        l[e] = acc;
    }
    double acc = 0.0;
    for (int h = 0; h < H; ++h)
        acc += oracle_bf16_to_f64(x[h]) * oracle_bf16_to_f64(shared_gate[h]);
    *z = acc;
}

/* Top-k by (logit descending, expert index ascending), then the softmax
 * restricted to the k chosen logits: w_r = exp(l_r - l_0) / sum_j exp(l_j - l_0). */
int oracle_topk(const double *l, int32_t E, int32_t k, int32_t *idx, double *w)
{
    if (k < 1 || k > E) return -2;
    char *taken = (char *)calloc((size_t)E, 1);
    if (!taken) return -1;
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep the lower index */
        }
        taken[best] = 1;
        idx[r] = best;
    }
    free(taken);
    double sum = 0.0;
    for (int r = 0; r < k; ++r) sum += exp(l[idx[r]] - l[idx[0]]);
    for (int r = 0; r < k; ++r) w[r] = exp(l[idx[r]] - l[idx[0]]) / sum;
    return 0;
}

/* Router step alone for `rows` rows: logits [rows, E], top-k idx/w [rows, k]
 * and sigmoid(g . x) [rows], by the same definitions as the layer below. */
int oracle_router_topk(const oracle_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                       const float *router_bias, const uint16_t *shared_gate, double *logits,
                       int32_t *idx, double *w, double *gate_sig)
{
    if (!d || !x || !router_w || !shared_gate || !logits || !idx || !w || !gate_sig || rows < 0) return -1;
    const int E = d->n_experts, K = d->top_k;
    if (K < 1 || K > E) return -2;
    for (int t = 0; t < rows; ++t) {
        double z;
        router_row(d, x + (int64_t)t * d->hidden, router_w, router_bias, shared_gate,
                   logits + (int64_t)t * E, &z);
        int st = oracle_topk(logits + (int64_t)t * E, E, K, idx + (int64_t)t * K, w + (int64_t)t * K);
        if (st) return st;
        gate_sig[t] = sigmoid(z);
    }
    return 0;
}

/* One SwiGLU expert on one row, from its slab [W13: 2I x H | W2: H x I]
 * (e4m3 codes) and scales [s13: 2I/128 x H/128 | s2: H/128 x I/128]:
 *   gu = W13 x;  h_j = silu(gu_j) * gu_{I+j};  y = W2 h. */
int oracle_expert_ffn(const uint8_t *w8, const float *scales, int32_t H, int32_t I,
                      const double *x, double *y)
{
    const uint8_t *w13 = w8;
    const uint8_t *w2 = w8 + (int64_t)2 * I * H;
    const float *s13 = scales;
    const float *s2 = scales + (int64_t)(2 * I / 128) * (H / 128);
    double *gu = (double *)malloc(sizeof(double) * 2 * (size_t)I);
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    if (!gu || !hv) { free(gu); free(hv); return -1; }
    for (int j = 0; j < 2 * I; ++j) {
        double acc = 0.0;
        for (int k = 0; k < H; ++k) acc += dq(w13, s13, H, j, k) * x[k];
        gu[j] = acc;
    }
    for (int j = 0; j < I; ++j) {
        double g = gu[j];
        hv[j] = g * sigmoid(g) * gu[I + j];
    }
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int j = 0; j < I; ++j) acc += dq(w2, s2, I, n, j) * hv[j];
        y[n] = acc;
    }
    free(gu);
    free(hv);
    return 0;
}

/* The SwiGLU expert with NVFP4 weights: the same formulas as
 * oracle_expert_ffn with each weight e2m1(code) * e4m3(sf) * gs.  Slab
 * layout: w4 = [W13 (2I x H/2) | W2 (H x I/2)] packed codes, sf = [W13
 * (2I x H/16) | W2 (H x I/16)] e4m3 codes, gs = [gs13, gs2]. */
int oracle_expert_ffn_nvfp4(const uint8_t *w4, const uint8_t *sf, const float *gs, int32_t H, int32_t I,
                            const double *x, double *y)
{
    const uint8_t *w13 = w4;
    const uint8_t *w2 = w4 + (int64_t)2 * I * H / 2;
    const uint8_t *f13 = sf;
    const uint8_t *f2 = sf + (int64_t)2 * I * H / 16;
    double *gu = (double *)malloc(sizeof(double) * 2 * (size_t)I);
    double *hv = (double *)malloc(sizeof(double) * (size_t)I);
    if (!gu || !hv) { free(gu); free(hv); return -1; }
    for (int j = 0; j < 2 * I; ++j) {
        double acc = 0.0;
        for (int k = 0; k < H; ++k) acc += dq4(w13, f13, (double)gs[0], H, j, k) * x[k];
        gu[j] = acc;
    }
    for (int j = 0; j < I; ++j) {
        double g = gu[j];
        hv[j] = g * sigmoid(g) * gu[I + j];
    }
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int j = 0; j < I; ++j) acc += dq4(w2, f2, (double)gs[1], I, n, j) * hv[j];
        y[n] = acc;
    }
    free(gu);
    free(hv);
    return 0;
}

typedef struct {
    const oracle_dims *d;
    const uint16_t *x;
    int32_t rows;
    const uint16_t *router_w;
    const uint8_t *expert_w8;
    const float *expert_scales;
    const uint8_t *shared_w8;
    const float *shared_scales;
    const uint16_t *shared_gate;
    const uint16_t *residual;
    const float *router_bias;
    const int32_t *forced_idx;
    int dense;
    int nvfp4;                  /* expert_w8/shared_w8 hold packed e2m1 codes */
    const uint8_t *expert_sf;   /* NVFP4: e4m3 block scales, per expert */
    const float *expert_gs;     /* NVFP4: [E][2] tensor scales */
    const uint8_t *shared_sf;
    const float *shared_gs;
    double *out;
    int32_t *idx;
    double *w;
    double *gate_sig;
    double *logits;
    int32_t row_begin, row_end;
    int status;
} fwd_job;

static int64_t expert_bytes(const oracle_dims *d, int32_t I) { return (int64_t)3 * I * d->hidden; }
static int64_t expert_nscales(const oracle_dims *d, int32_t I)
{
    return (int64_t)(2 * I / 128) * (d->hidden / 128) + (int64_t)(d->hidden / 128) * (I / 128);
}

/* Expert e (-1: shared) of a job applied to xr. */
static int job_expert(const fwd_job *j, int e, const double *xr, double *y)
{
    const oracle_dims *d = j->d;
    const int H = d->hidden;
    if (j->nvfp4) {
        const int32_t I = e < 0 ? d->shared_inter : d->inter;
        if (e < 0) return oracle_expert_ffn_nvfp4(j->shared_w8, j->shared_sf, j->shared_gs, H, I, xr, y);
        return oracle_expert_ffn_nvfp4(j->expert_w8 + (int64_t)e * 3 * I * H / 2,
                                       j->expert_sf + (int64_t)e * 3 * I * H / 16, j->expert_gs + 2 * (int64_t)e,
                                       H, I, xr, y);
    }
    if (e < 0) return oracle_expert_ffn(j->shared_w8, j->shared_scales, H, d->shared_inter, xr, y);
    return oracle_expert_ffn(j->expert_w8 + (int64_t)e * expert_bytes(d, d->inter),
                             j->expert_scales + (int64_t)e * expert_nscales(d, d->inter), H, d->inter, xr, y);
}

static void *fwd_worker(void *arg)
{
    fwd_job *j = (fwd_job *)arg;
    const oracle_dims *d = j->d;
    const int H = d->hidden, E = d->n_experts, K = d->top_k;
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    double *xr = (double *)malloc(sizeof(double) * (size_t)H);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    int32_t *ix = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *wv = (double *)malloc(sizeof(double) * (size_t)K);
    double *mask = (double *)malloc(sizeof(double) * (size_t)E);
    if (!l || !xr || !y || !acc || !ix || !wv || !mask) { j->status = -1; goto done; }
    for (int t = j->row_begin; t < j->row_end; ++t) {
        const uint16_t *xt = j->x + (int64_t)t * H;
        double z;
        router_row(d, xt, j->router_w, j->router_bias, j->shared_gate, l, &z);
        if (j->logits) memcpy(j->logits + (int64_t)t * E, l, sizeof(double) * (size_t)E);
        if (j->forced_idx) {
            /* Given routing: weights are the softmax over the given k logits
             * (relative to the first given one, which is the largest only
             * when the given order is by descending logit; the result does
             * not depend on which logit is subtracted). */
            double sum = 0.0;
            for (int r = 0; r < K; ++r) ix[r] = j->forced_idx[(int64_t)t * K + r];
            for (int r = 0; r < K; ++r) {
                if (ix[r] < 0 || ix[r] >= E) { j->status = -2; goto done; }
                sum += exp(l[ix[r]] - l[ix[0]]);
            }
            for (int r = 0; r < K; ++r) wv[r] = exp(l[ix[r]] - l[ix[0]]) / sum;
        } else {
            if (oracle_topk(l, E, K, ix, wv)) { j->status = -2; goto done; }
        }
        for (int r = 0; r < K; ++r) {
            j->idx[(int64_t)t * K + r] = ix[r];
            j->w[(int64_t)t * K + r] = wv[r];
        }
        double gs = sigmoid(z);
        j->gate_sig[t] = gs;
        for (int h = 0; h < H; ++h) xr[h] = oracle_bf16_to_f64(xt[h]);
        for (int h = 0; h < H; ++h) acc[h] = 0.0;
        if (!j->dense) {
            /* routed: the k selected experts, in rank order */
            for (int r = 0; r < K; ++r) {
                if (job_expert(j, ix[r], xr, y)) { j->status = -1; goto done; }
                for (int h = 0; h < H; ++h) acc[h] += wv[r] * y[h];
            }
        } else {
            /* dense brute force: every expert evaluated, weighted by the
             * top-k mask (w_r for a selected expert, 0 otherwise) */
            for (int e = 0; e < E; ++e) mask[e] = 0.0;
            for (int r = 0; r < K; ++r) mask[ix[r]] = wv[r];
            for (int e = 0; e < E; ++e) {
                if (job_expert(j, e, xr, y)) { j->status = -1; goto done; }
                for (int h = 0; h < H; ++h) acc[h] += mask[e] * y[h];
            }
        }
        /* shared expert, scaled by its sigmoid gate */
        if (job_expert(j, -1, xr, y)) {
            j->status = -1;
            goto done;
        }
        for (int h = 0; h < H; ++h) acc[h] += gs * y[h];
        if (j->residual)
            for (int h = 0; h < H; ++h) acc[h] += oracle_bf16_to_f64(j->residual[(int64_t)t * H + h]);
        memcpy(j->out + (int64_t)t * H, acc, sizeof(double) * (size_t)H);
    }
done:
    free(l); free(xr); free(y); free(acc); free(ix); free(wv); free(mask);
    return NULL;
}

static int check_dims(const oracle_dims *d)
{
    if (!d) return -1;
    if (d->hidden <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->inter <= 0 || d->shared_inter <= 0) return -2;
    if (d->hidden % 128 || d->inter % 128 || d->shared_inter % 128) return -2;
    if (d->top_k > d->n_experts) return -2;
    return 0;
}

typedef struct {
    const uint8_t *expert_sf;
    const float *expert_gs;
    const uint8_t *shared_sf;
    const float *shared_gs;
} nvfp4_scales;

static int run_forward(const oracle_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                       const uint8_t *expert_w8, const float *expert_scales,
                       const uint8_t *shared_w8, const float *shared_scales,
                       const uint16_t *shared_gate, const uint16_t *residual,
                       const float *router_bias, const int32_t *forced_idx, int dense,
                       double *out, int32_t *idx, double *w, double *gate_sig, double *logits,
                       int32_t nthreads, const nvfp4_scales *f4)
{
    int st = check_dims(d);
    if (st) return st;
    if (!x || !router_w || !expert_w8 || !shared_w8 || !shared_gate || !out || !idx || !w || !gate_sig || rows < 0)
        return -1;
    if (f4 ? (!f4->expert_sf || !f4->expert_gs || !f4->shared_sf || !f4->shared_gs)
           : (!expert_scales || !shared_scales))
        return -1;
    if (f4 && (d->hidden % 16 || d->inter % 16 || d->shared_inter % 16)) return -2;
    if (rows == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = rows;
    fwd_job *jobs = (fwd_job *)calloc((size_t)nthreads, sizeof(fwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -1; }
    for (int i = 0; i < nthreads; ++i) {
        fwd_job *j = &jobs[i];
        j->d = d; j->x = x; j->rows = rows; j->router_w = router_w;
        j->expert_w8 = expert_w8; j->expert_scales = expert_scales;
        j->shared_w8 = shared_w8; j->shared_scales = shared_scales;
        j->shared_gate = shared_gate; j->residual = residual; j->router_bias = router_bias;
        j->forced_idx = forced_idx; j->dense = dense;
        if (f4) {
            j->nvfp4 = 1;
            j->expert_sf = f4->expert_sf; j->expert_gs = f4->expert_gs;
            j->shared_sf = f4->shared_sf; j->shared_gs = f4->shared_gs;
        }
        j->out = out; j->idx = idx; j->w = w; j->gate_sig = gate_sig; j->logits = logits;
        j->row_begin = (int32_t)((int64_t)rows * i / nthreads);
        j->row_end = (int32_t)((int64_t)rows * (i + 1) / nthreads);
    }
    char *created = (char *)calloc((size_t)nthreads, 1);
    if (!created) { free(jobs); free(th); return -1; }
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, fwd_worker, &jobs[i]) == 0)
            created[i] = 1;
        else
            fwd_worker(&jobs[i]); /* could not start a thread: run it here */
    }
    fwd_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i)
        if (created[i]) pthread_join(th[i], NULL);
    free(created);
    int rc = 0;
    for (int i = 0; i < nthreads; ++i)
        if (jobs[i].status) rc = jobs[i].status;
    free(jobs);
    free(th);
    return rc;
}

/* The layer, routed: out[t] = sum_r w[t,r] * expert_{idx[t,r]}(x_t)
 *                            + sigmoid(g . x_t) * shared(x_t) (+ residual_t),
 * in double, before any rounding to bf16.  forced_idx (nullable, [rows, k])
 * replaces the top-k selection by a given routing.  logits (nullable) is
 * [rows, E]. */
int oracle_moe_forward(const oracle_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                       const uint8_t *expert_w8, const float *expert_scales,
                       const uint8_t *shared_w8, const float *shared_scales,
                       const uint16_t *shared_gate, const uint16_t *residual,
                       const float *router_bias, const int32_t *forced_idx,
                       double *out, int32_t *idx, double *w, double *gate_sig, double *logits,
                       int32_t nthreads)
{
    return run_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                       shared_gate, residual, router_bias, forced_idx, 0, out, idx, w, gate_sig,
                       logits, nthreads, NULL);
}

/* The same layer by brute force: all E experts evaluated for every row and
 * summed in expert-index order with the top-k mask as weights. */
int oracle_moe_forward_dense(const oracle_dims *d, const uint16_t *x, int32_t rows,
                             const uint16_t *router_w, const uint8_t *expert_w8,
                             const float *expert_scales, const uint8_t *shared_w8,
                             const float *shared_scales, const uint16_t *shared_gate,
                             const uint16_t *residual, const float *router_bias,
                             double *out, int32_t *idx, double *w, double *gate_sig,
                             int32_t nthreads)
{
    return run_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                       shared_gate, residual, router_bias, NULL, 1, out, idx, w, gate_sig, NULL,
                       nthreads, NULL);
}

/* The layer with NVFP4 experts (routed, or dense brute force when dense is
 * non-zero): oracle_moe_forward's formulas with each weight e2m1(code) *
 * e4m3(sf) * gs.  expert_w4 [E][3*I*H/2] packed codes, expert_sf
 * [E][3*I*H/16] e4m3 scale codes, expert_gs [E][2] (W13, W2); the shared
 * expert likewise with Is. */
int oracle_moe_forward_nvfp4(const oracle_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                             const uint8_t *expert_w4, const uint8_t *expert_sf, const float *expert_gs,
                             const uint8_t *shared_w4, const uint8_t *shared_sf, const float *shared_gs,
                             const uint16_t *shared_gate, const uint16_t *residual,
                             const float *router_bias, const int32_t *forced_idx, int32_t dense,
                             double *out, int32_t *idx, double *w, double *gate_sig, double *logits,
                             int32_t nthreads)
{
    nvfp4_scales f4 = {expert_sf, expert_gs, shared_sf, shared_gs};
    return run_forward(d, x, rows, router_w, expert_w4, NULL, shared_w4, NULL, shared_gate, residual,
                       router_bias, dense ? NULL : forced_idx, dense ? 1 : 0, out, idx, w, gate_sig,
                       dense ? NULL : logits, nthreads, &f4);
}
