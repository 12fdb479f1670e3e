/*
 * DeltaQuant W4A4 linear layer -- CPU ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * statement of what the layer computes.  Only the tests, the smoke check and
 * the bench's CPU-baseline leg may load it.  It shares no code, header,
 * table or helper with the CUDA library, and nothing in the library calls it.
 *
 * Source: papernotes.org, "DeltaQuant: 4-bit Video Diffusion Models with
 * Spatiotemporal Delta Smoothing" (CVPR 2026 note), section "Key designs":
 *   design 2  cube partition of the (t,h,w) token lattice,
 *   design 3  Eq. 1: kernel token = cube mean, delta token = token - mean,
 *   design 4  Eq. 2 / Eq. 3: Y = Q8(mean) Q4(R) + Q4(delta) Q4(R) + X L1 L2,
 *             Eq. 4: Q(X) = round(X/s) s, s = max|X| / q_max, q_max = 6 (FP4),
 *   "Loss / training strategy" section: NVFP4 for the linear layers, FP8
 *             kernel tokens, SVD low-rank branch from SVDQuant.
 * Readings where the page is silent (each also listed in the design notes):
 *   - FP4 = E2M1 with one E4M3 scale per 16 channels and one fp32 per-tensor
 *     scale S = amax / (6 * 448) (the two-level form of Eq. 4); S = 1 if amax = 0.
 *   - FP8 = E4M3 with one fp32 scale per kernel token, s8 = amax / 448.
 *   - rounding is round-to-nearest-even with saturation to the largest finite
 *     value; a negative value that rounds to zero keeps its sign.
 *   - the cube mean is an fp32 running sum over the cube's tokens in (t,h,w)
 *     order, divided by the token count; edge cubes that the lattice cuts
 *     short average the tokens they hold.
 *   - every fp32 step is a single IEEE operation; this file is compiled with
 *     -ffp-contract=off so no multiply-add is fused.
 * Options beside the default (each pinned on its own): one kernel scale per 64
 * channels (or_fp8_kernel_tokens), a power-of-two per-tensor delta scale
 * (or_quantize_activations_opt), restricted weight scales with an exact FP8
 * form (or_fp4_quantize_c2, or_c2_fp8_operand), an additive bias (Python side),
 * and the step between the two layers of a feed-forward block (or_gelu_erf).
 *   - the feed-forward activation, which the note does not name, is GELU in its
 *     exact form y * Phi(y), evaluated in fp64 on the producer layer's output.
 * Parity pins: see tests/test_oracle_*.py.  Parity unpinned: nothing in this
 * file; the GPU's tensor-core accumulation order is covered only by the Y
 * tolerance.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* BF16 bits -> fp32 value (exact: BF16 is the top half of an fp32). */
float or_bf16_value(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp64 -> nearest BF16, ties to even, by search over the two neighbours. */
uint16_t or_bf16_round(double v) {
    /* truncate toward zero in fp32 bit space, then compare both candidates */
    float f = (float)v;                       /* only used to get near */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t lo = (uint16_t)(u >> 16);
    uint16_t best = lo;
    double bestd = INFINITY;
    for (int d = -2; d <= 2; d++) {
        uint16_t c = (uint16_t)(lo + d);
        float cv = or_bf16_value(c);
        if (isnan(cv)) continue;
        double dist = fabs((double)cv - v);
        if (dist < bestd || (dist == bestd && (c & 1) == 0)) { bestd = dist; best = c; }
    }
    return best;
}

/* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit.
 * Magnitudes by the low three code bits. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double or_e2m1_value(int code) {
    double m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 (FP8, the "fn" variant: no infinities, NaN = S.1111.111, max 448).
 * 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent field 0 is subnormal. */
double or_e4m3_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                 /* m/8 * 2^-6 */
    else
        v = ldexp(8.0 + (double)m, e - 10);       /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Nearest code among the non-negative codes 0..ncodes-1 whose values increase
 * with the code; ties go to the even code; beyond the top value saturate. */
static int nearest_code(double a, double (*val)(int), int ncodes) {
    if (!(a > 0.0)) return 0;                          /* +0 (and -0 handled by caller) */
    double top = val(ncodes - 1);
    if (a >= top) return ncodes - 1;
    int lo = 0, hi = ncodes - 1;                       /* val(lo) <= a < val(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (val(mid) <= a) lo = mid; else hi = mid;
    }
    double vl = val(lo), vh = val(lo + 1);
    double dl = a - vl, dh = vh - a;
    if (dl < dh) return lo;
    if (dh < dl) return lo + 1;
    return (lo % 2 == 0) ? lo : lo + 1;
}

/* fp32 -> E2M1 code, round to nearest even, saturate at +-6. */
int or_e2m1_encode(float v) {
    int sign = signbit(v) ? 8 : 0;
    int c = nearest_code(fabs((double)v), or_e2m1_value, 8);
    return sign | c;
}

/* fp32 -> E4M3 code, round to nearest even, saturate at +-448. */
int or_e4m3_encode(float v) {
    int sign = signbit(v) ? 0x80 : 0;
    int c = nearest_code(fabs((double)v), or_e4m3_value, 127);
    return sign | c;
}

/* ------------------------------------------------------------------------ */
/* Cube partition (key design 2)                                             */
/* ------------------------------------------------------------------------ */

static int cdiv(int a, int b) { return (a + b - 1) / b; }

long long or_num_cubes(int T, int H, int W, int t, int h, int w) {
    return (long long)cdiv(T, t) * cdiv(H, h) * cdiv(W, w);
}

/*
 * Enumerate the cubes in order k = (kt*KH + kh)*KW + kw and, inside each cube,
 * its tokens in (t,h,w) order.  The j-th token visited overall gets
 * cube-major row j.  Outputs (any may be NULL):
 *   row_of_n[n]  cube-major row of natural token n = (t*H + h)*W + w
 *   cube_of_n[n] cube index of token n
 *   n_of_row[j]  natural token of cube-major row j
 *   count[k]     tokens in cube k
 *   first[k]     first cube-major row of cube k
 */
void or_cube_order(int T, int H, int W, int t, int h, int w, int* row_of_n, int* cube_of_n,
                   int* n_of_row, int* count, int* first) {
    int KT = cdiv(T, t), KH = cdiv(H, h), KW = cdiv(W, w);
    int j = 0;
    for (int kt = 0; kt < KT; kt++)
        for (int kh = 0; kh < KH; kh++)
            for (int kw = 0; kw < KW; kw++) {
                int k = (kt * KH + kh) * KW + kw;
                if (first) first[k] = j;
                int cnt = 0;
                for (int tt = kt * t; tt < kt * t + t && tt < T; tt++)
                    for (int hh = kh * h; hh < kh * h + h && hh < H; hh++)
                        for (int ww = kw * w; ww < kw * w + w && ww < W; ww++) {
                            int n = (tt * H + hh) * W + ww;
                            if (row_of_n) row_of_n[n] = j;
                            if (cube_of_n) cube_of_n[n] = k;
                            if (n_of_row) n_of_row[j] = n;
                            j++;
                            cnt++;
                        }
                if (count) count[k] = cnt;
            }
}

/* ------------------------------------------------------------------------ */
/* Kernel tokens and delta tokens (key design 3, Eq. 1)                      */
/* ------------------------------------------------------------------------ */

typedef struct {
    int T, H, W, t, h, w, Ci;
    long long K;
    int* n_of_row;  /* N */
    int* count;     /* K */
    int* first;     /* K */
} geom_t;

static int geom_init(geom_t* g, int T, int H, int W, int t, int h, int w, int Ci) {
    g->T = T; g->H = H; g->W = W; g->t = t; g->h = h; g->w = w; g->Ci = Ci;
    g->K = or_num_cubes(T, H, W, t, h, w);
    long long N = (long long)T * H * W;
    g->n_of_row = (int*)malloc(sizeof(int) * (size_t)N);
    g->count = (int*)malloc(sizeof(int) * (size_t)g->K);
    g->first = (int*)malloc(sizeof(int) * (size_t)g->K);
    if (!g->n_of_row || !g->count || !g->first) return 2;
    or_cube_order(T, H, W, t, h, w, NULL, NULL, g->n_of_row, g->count, g->first);
    return 0;
}

static void geom_free(geom_t* g) {
    free(g->n_of_row); free(g->count); free(g->first);
}

/*
 * Eq. 1, kernel token: the fp32 mean of the cube's tokens per channel,
 * summed one token at a time in (t,h,w) order and divided by the count.
 * m is K x Ci.
 */
static void cube_means(const uint16_t* X, const geom_t* g, float* m) {
    int Ci = g->Ci;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long k = 0; k < g->K; k++) {
        float* mk = m + (size_t)k * Ci;
        for (int c = 0; c < Ci; c++) mk[c] = 0.0f;
        for (int j = 0; j < g->count[k]; j++) {
            const uint16_t* x = X + (size_t)g->n_of_row[g->first[k] + j] * Ci;
            for (int c = 0; c < Ci; c++) mk[c] = mk[c] + or_bf16_value(x[c]);
        }
        float cnt = (float)g->count[k];
        for (int c = 0; c < Ci; c++) mk[c] = mk[c] / cnt;
    }
}

int or_cube_means(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w, float* m) {
    geom_t g;
    if (geom_init(&g, T, H, W, t, h, w, Ci)) { geom_free(&g); return 2; }
    cube_means(X, &g, m);
    geom_free(&g);
    return 0;
}

/* The same mean and delta carried out in fp64 (no quantisation, no fp32
 * rounding): used to check that Eq. 1 splits X exactly. */
int or_cube_split_f64(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w,
                      double* mean /*K x Ci*/, double* delta /*N x Ci, natural order*/) {
    geom_t g;
    if (geom_init(&g, T, H, W, t, h, w, Ci)) { geom_free(&g); return 2; }
#pragma omp parallel for schedule(dynamic, 16)
    for (long long k = 0; k < g.K; k++) {
        double* mk = mean + (size_t)k * Ci;
        for (int c = 0; c < Ci; c++) mk[c] = 0.0;
        for (int j = 0; j < g.count[k]; j++) {
            const uint16_t* x = X + (size_t)g.n_of_row[g.first[k] + j] * Ci;
            for (int c = 0; c < Ci; c++) mk[c] += (double)or_bf16_value(x[c]);
        }
        for (int c = 0; c < Ci; c++) mk[c] /= (double)g.count[k];
        for (int j = 0; j < g.count[k]; j++) {
            int n = g.n_of_row[g.first[k] + j];
            const uint16_t* x = X + (size_t)n * Ci;
            for (int c = 0; c < Ci; c++) delta[(size_t)n * Ci + c] = (double)or_bf16_value(x[c]) - mk[c];
        }
    }
    geom_free(&g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Quantisers (key design 4, Eq. 4, with the NVFP4 / FP8 readings)           */
/* ------------------------------------------------------------------------ */

/* Per-tensor scale of the two-level FP4 form: amax / (6 * 448). */
float or_tensor_scale(float amax) {
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;
}

/* The smallest power of two >= v (v > 0), exactly: v = m 2^e with m in [0.5, 1). */
float or_pow2_ceil(float v) {
    int e;
    const float m = frexpf(v, &e);
    return (m == 0.5f) ? v : ldexpf(1.0f, e);
}

/*
 * One row of FP4 with E4M3 group-16 scales and the per-tensor scale S:
 *   s_b = E4M3(amax_b / (6 S)),  q = E2M1(z / (s_b S))   (Eq. 4 per group).
 * codes: cols/2 bytes, channel 2i in the low nibble of byte i.
 * scales: cols/16 bytes.
 */
static void fp4_row(const float* z, int cols, float S, uint8_t* codes, uint8_t* scales) {
    float denom = 6.0f * S;
    for (int b = 0; b < cols / 16; b++) {
        float amax = 0.0f;
        for (int i = 0; i < 16; i++) {
            float a = fabsf(z[b * 16 + i]);
            if (a > amax) amax = a;
        }
        int sb = or_e4m3_encode(amax / denom);
        float eff = (float)or_e4m3_value(sb) * S;
        scales[b] = (uint8_t)sb;
        for (int i = 0; i < 16; i += 2) {
            int q0 = (eff == 0.0f) ? 0 : or_e2m1_encode(z[b * 16 + i] / eff);
            int q1 = (eff == 0.0f) ? 0 : or_e2m1_encode(z[b * 16 + i + 1] / eff);
            codes[(b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* C2: restricted weight scales for an exact FP8-rate kernel-token product   */
/* ------------------------------------------------------------------------ */

/*
 * The restricted group scale of C2 weights: the member of
 *   A = {0} U { m 2^e : m in {1, 1.25, 1.5}, m 2^e an E4M3 value, m 2^e <= 384 }
 * nearest to v >= 0 (ties to the larger member).  The product of a member with
 * an E2M1 value has at most three fraction bits (1.5 x 1.25 = 1.875,
 * 1.5 x 1.5 = 1.125 x 2), so it is an E4M3 value times a power of two; m = 1.75
 * is left out because 1.5 x 1.75 needs four.  Below 2^-6 the E4M3 members are
 * k 2^-9 with k in {1, 2, 3, 4, 5, 6} (5 2^-9 = 1.25 x 2^-7; 7 2^-9 is not of
 * the form).  Found by search over A.
 */
static int c2_member(double c) {
    if (c == 0.0) return 1;
    if (c > 384.0) return 0;
    int e;
    const double m = 2.0 * frexp(c, &e);          /* c = m 2^(e-1), m in [1, 2) */
    if (m != 1.0 && m != 1.25 && m != 1.5) return 0;
    return or_e4m3_value(or_e4m3_encode((float)c)) == c;
}

/* The smallest member of A that is >= v > 0. */
static double c2_member_at_least(double v) {
    double best = 1e300;
    for (int e = -9; e <= 9; e++)
        for (int i = 0; i < 3; i++) {
            const double c = ldexp(i == 0 ? 1.0 : (i == 1 ? 1.25 : 1.5), e);
            if (c2_member(c) && c >= v && c < best) best = c;
        }
    return best;
}

float or_c2_scale_nearest(float v) {
    if (!(v > 0.0f)) return 0.0f;
    double best = 0.0, bd = (double)v;
    for (int e = -9; e <= 9; e++)
        for (int i = 0; i < 3; i++) {
            const double c = ldexp(i == 0 ? 1.0 : (i == 1 ? 1.25 : 1.5), e);
            if (!c2_member(c)) continue;
            const double d = fabs(c - (double)v);
            if (d < bd || (d == bd && c > best)) {
                best = c;
                bd = d;
            }
        }
    return (float)best;
}

/*
 * C2 weight quantiser (the restricted-scale reading, an option; the default is
 * fp4_row's Eq. 4 form).  Per-tensor S = amax / (6 * 384) (384 = 1.5 x 2^8,
 * the largest member), group-16 scales s_b = or_c2_scale_nearest(amax_b /
 * (6 S)), then, per 32 channels, a nonzero smaller scale raised to the
 * smallest member >= 2^-9 times the larger, so that the block's values q s_b
 * span at most 2^14 and fit E4M3's normal range under one power-of-two
 * exponent; q = E2M1(z / (s_b S)) (nearest even, saturating at 6).  Returns
 * the number of raised scales.
 */
long long or_fp4_quantize_c2(const float* Z, long long rows, int cols, uint8_t* codes, uint8_t* scales,
                             float* S_out) {
    if (cols % 32) return -1;
    float amax = 0.0f;
    for (long long i = 0; i < rows * (long long)cols; i++) {
        float a = fabsf(Z[i]);
        if (a > amax) amax = a;
    }
    const float S = (amax == 0.0f) ? 1.0f : amax / 2304.0f;
    const float denom = 6.0f * S;
    long long raised = 0;
#pragma omp parallel for schedule(static) reduction(+ : raised)
    for (long long r = 0; r < rows; r++) {
        const float* z = Z + (size_t)r * cols;
        for (int b2 = 0; b2 < cols / 32; b2++) {
            float sb[2];
            for (int h = 0; h < 2; h++) {
                const int b = 2 * b2 + h;
                float am = 0.0f;
                for (int i = 0; i < 16; i++) {
                    float a = fabsf(z[b * 16 + i]);
                    if (a > am) am = a;
                }
                sb[h] = or_c2_scale_nearest(am / denom);
            }
            const float big = sb[0] > sb[1] ? sb[0] : sb[1];
            for (int h = 0; h < 2; h++) {
                if (sb[h] > 0.0f && sb[h] < ldexpf(big, -9)) {
                    sb[h] = (float)c2_member_at_least(ldexp((double)big, -9));
                    raised++;
                }
            }
            for (int h = 0; h < 2; h++) {
                const int b = 2 * b2 + h;
                scales[(size_t)r * (cols / 16) + b] = (uint8_t)or_e4m3_encode(sb[h]);
                const float eff = sb[h] * S;
                for (int i = 0; i < 16; i += 2) {
                    int q0 = (eff == 0.0f) ? 0 : or_e2m1_encode(z[b * 16 + i] / eff);
                    int q1 = (eff == 0.0f) ? 0 : or_e2m1_encode(z[b * 16 + i + 1] / eff);
                    codes[(size_t)r * (cols / 2) + (b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
                }
            }
        }
    }
    if (S_out) *S_out = S;
    return raised;
}

/*
 * The FP8 form of C2 weights for a kind::mxf8f6f4 product: per 32 channels one
 * UE8M0 exponent u (biased by 127) and E4M3 codes of q s_b / 2^u, with u chosen
 * so that the block's largest |q s_b| lands in [128, 256) (a significand of
 * 1.875 in [256, 512) would exceed E4M3's 448).  Returns the number of elements
 * whose E4M3 code does not reproduce q s_b exactly (0 for weights from
 * or_fp4_quantize_c2).
 */
long long or_c2_fp8_operand(const uint8_t* codes, const uint8_t* scales, long long rows, int cols, uint8_t* fp8,
                            uint8_t* ue8m0) {
    long long inexact = 0;
#pragma omp parallel for schedule(static) reduction(+ : inexact)
    for (long long r = 0; r < rows; r++) {
        for (int b2 = 0; b2 < cols / 32; b2++) {
            double w[32], wmax = 0.0;
            for (int i = 0; i < 32; i++) {
                const int c = b2 * 32 + i;
                const int code = (codes[(size_t)r * (cols / 2) + c / 2] >> (4 * (c & 1))) & 15;
                w[i] = or_e2m1_value(code) * or_e4m3_value(scales[(size_t)r * (cols / 16) + c / 16]);
                if (fabs(w[i]) > wmax) wmax = fabs(w[i]);
            }
            int u = 0;
            if (wmax > 0.0) {
                int e;
                frexp(wmax, &e);          /* wmax in [2^(e-1), 2^e) */
                u = e - 1 - 7;
            }
            ue8m0[(size_t)r * (cols / 32) + b2] = (uint8_t)(u + 127);
            for (int i = 0; i < 32; i++) {
                const double v = ldexp(w[i], -u);
                const int q = or_e4m3_encode((float)v);
                fp8[(size_t)r * cols + b2 * 32 + i] = (uint8_t)q;
                if (or_e4m3_value(q) != v) inexact++;
            }
        }
    }
    return inexact;
}

/* FP4-quantise a rows x cols fp32 matrix with its own per-tensor scale
 * (computed from its amax) or with the given S when S_in > 0. */
int or_fp4_quantize(const float* Z, long long rows, int cols, float S_in, uint8_t* codes,
                    uint8_t* scales, float* S_out) {
    if (cols % 16) return 1;
    float S = S_in;
    if (!(S_in > 0.0f)) {
        float amax = 0.0f;
#pragma omp parallel for reduction(max : amax)
        for (long long i = 0; i < rows * (long long)cols; i++) {
            float a = fabsf(Z[i]);
            if (a > amax) amax = a;
        }
        S = or_tensor_scale(amax);
    }
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; r++)
        fp4_row(Z + (size_t)r * cols, cols, S, codes + (size_t)r * (cols / 2), scales + (size_t)r * (cols / 16));
    if (S_out) *S_out = S;
    return 0;
}

/* FP8 kernel tokens: s8 = max_c |m_c| / 448, q8 = E4M3(m / s8), 0 if s8 = 0
 * (over the Ci channels of a token, or over one group of channels). */
static void fp8_token(const float* m, int Ci, uint8_t* q8, float* s8) {
    float amax = 0.0f;
    for (int c = 0; c < Ci; c++) {
        float a = fabsf(m[c]);
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    *s8 = s;
    for (int c = 0; c < Ci; c++) q8[c] = (uint8_t)((s == 0.0f) ? 0 : or_e4m3_encode(m[c] / s));
}


/*
 * FP8 kernel tokens with one scale per `group` consecutive channels (the
 * note's per-group-64 kernel quantisation; group = Ci is one scale per token):
 * s8[k][j] = max |m[k][c]| over channels c of group j, / 448;
 * q8[k][c] = E4M3(m[k][c] / s8[k][c / group]), 0 where that scale is 0.
 * means: K x Ci fp32; q8: K x Ci; s8: K x Ci/group.
 */
int or_fp8_kernel_tokens(const float* means, long long K, int Ci, int group, uint8_t* q8, float* s8) {
    if (group <= 0 || Ci % group) return 1;
    const int ng = Ci / group;
#pragma omp parallel for schedule(static)
    for (long long k = 0; k < K; k++)
        for (int j = 0; j < ng; j++)
            fp8_token(means + (size_t)k * Ci + (size_t)j * group, group, q8 + (size_t)k * Ci + (size_t)j * group,
                      s8 + (size_t)k * ng + j);
    return 0;
}

/* The global max |x - m| over every delta of the tensor (Eq. 1 deltas in fp32):
 * the amax behind the per-tensor delta scale. */
static float delta_amax(const uint16_t* X, const geom_t* g, const float* m) {
    const int Ci = g->Ci;
    float amax = 0.0f;
#pragma omp parallel for reduction(max : amax) schedule(dynamic, 16)
    for (long long k = 0; k < g->K; k++) {
        const float* mk = m + (size_t)k * Ci;
        for (int j = 0; j < g->count[k]; j++) {
            const uint16_t* x = X + (size_t)g->n_of_row[g->first[k] + j] * Ci;
            for (int c = 0; c < Ci; c++) {
                float d = fabsf(or_bf16_value(x[c]) - mk[c]);
                if (d > amax) amax = d;
            }
        }
    }
    return amax;
}

/*
 * The activation side of Eq. 2/3 for a whole X (N x Ci, natural order):
 *   dcodes  N x Ci/2   FP4 delta codes, rows in cube-major order
 *   dscales N x Ci/16  E4M3 group scales, same row order
 *   S_delta           per-tensor scale from the amax of every delta
 *   q8      K x Ci     E4M3 kernel tokens;  s8  K fp32 scales
 *   means   K x Ci     fp32 kernel tokens before quantisation (optional)
 *   amax_delta        the global max |delta| (optional)
 */
/*
 * As or_quantize_activations, with pow2 != 0 taking a power-of-two per-tensor
 * delta scale: S = the smallest power of two >= amax / 2688 (1 if amax = 0).
 * A block encoded under another power-of-two scale then keeps its codes and
 * only its E4M3 scale's exponent moves (unless that scale leaves E4M3's normal
 * range): the property a single-read encoder with a scale fix-up pass relies
 * on.  A deviation from the two-level form of Eq. 4.  The kernel-token scales
 * keep max |m| / 448, which represents each token's largest element exactly.
 */
int or_quantize_activations_opt(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w,
                                uint8_t* dcodes, uint8_t* dscales, float* S_delta, uint8_t* q8, float* s8,
                                float* means, float* amax_delta, int pow2);

int or_quantize_activations(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w,
                            uint8_t* dcodes, uint8_t* dscales, float* S_delta, uint8_t* q8, float* s8,
                            float* means, float* amax_delta) {
    return or_quantize_activations_opt(X, T, H, W, Ci, t, h, w, dcodes, dscales, S_delta, q8, s8, means, amax_delta, 0);
}

int or_quantize_activations_opt(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w,
                                uint8_t* dcodes, uint8_t* dscales, float* S_delta, uint8_t* q8, float* s8,
                                float* means, float* amax_delta, int pow2) {
    if (Ci % 16) return 1;
    geom_t g;
    if (geom_init(&g, T, H, W, t, h, w, Ci)) { geom_free(&g); return 2; }
    float* m = means ? means : (float*)malloc(sizeof(float) * (size_t)g.K * Ci);
    if (!m) { geom_free(&g); return 2; }
    cube_means(X, &g, m);
    float amax = delta_amax(X, &g, m);
    float S = or_tensor_scale(amax);
    if (pow2 && amax != 0.0f) S = or_pow2_ceil(amax / 2688.0f);
    if (S_delta) *S_delta = S;
    if (amax_delta) *amax_delta = amax;

#pragma omp parallel for schedule(dynamic, 16)
    for (long long k = 0; k < g.K; k++) {
        const float* mk = m + (size_t)k * Ci;
        if (q8) fp8_token(mk, Ci, q8 + (size_t)k * Ci, s8 + k);
        float* z = (float*)malloc(sizeof(float) * (size_t)Ci);
        for (int j = 0; j < g.count[k]; j++) {
            long long row = g.first[k] + j;
            const uint16_t* x = X + (size_t)g.n_of_row[row] * Ci;
            for (int c = 0; c < Ci; c++) z[c] = or_bf16_value(x[c]) - mk[c];
            if (dcodes) fp4_row(z, Ci, S, dcodes + (size_t)row * (Ci / 2), dscales + (size_t)row * (Ci / 16));
        }
        free(z);
    }
    if (!means) free(m);
    geom_free(&g);
    return 0;
}

/*
 * The statistics half of the activation side over the whole tensor: the cube
 * means (Eq. 1) and the global max |delta|, from which the per-tensor delta
 * scale follows.  Used with or_quantize_cubes to quantise a sample of cubes
 * exactly as the whole tensor would be.
 */
int or_delta_amax(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w, float* amax_delta) {
    geom_t g;
    if (geom_init(&g, T, H, W, t, h, w, Ci)) { geom_free(&g); return 2; }
    float* m = (float*)malloc(sizeof(float) * (size_t)g.K * Ci);
    if (!m) { geom_free(&g); return 2; }
    cube_means(X, &g, m);
    *amax_delta = delta_amax(X, &g, m);
    free(m);
    geom_free(&g);
    return 0;
}

/*
 * The activation side for the listed cubes only, under a given per-tensor
 * delta scale S (the whole tensor's): for list entry i = cube k = cubes[i],
 * its mean, its FP8 kernel token q8[i] / s8[i] (per-token scale), and its
 * tokens' FP4 delta rows, written in list order and, inside a cube, in
 * (t,h,w) order; first_row[i] = the first of cube i's rows in that order.
 * The same arithmetic as or_quantize_activations row for row.
 */
int or_quantize_cubes(const uint16_t* X, int T, int H, int W, int Ci, int t, int h, int w, const long long* cubes,
                      long long ncubes, float S, uint8_t* dcodes, uint8_t* dscales, uint8_t* q8, float* s8,
                      long long* first_row) {
    if (Ci % 16) return 1;
    geom_t g;
    if (geom_init(&g, T, H, W, t, h, w, Ci)) { geom_free(&g); return 2; }
    long long row = 0;
    for (long long i = 0; i < ncubes; i++) {
        if (cubes[i] < 0 || cubes[i] >= g.K) { geom_free(&g); return 1; }
        first_row[i] = row;
        row += g.count[cubes[i]];
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = 0; i < ncubes; i++) {
        const long long k = cubes[i];
        float* mk = (float*)malloc(sizeof(float) * (size_t)Ci);
        float* z = (float*)malloc(sizeof(float) * (size_t)Ci);
        for (int c = 0; c < Ci; c++) mk[c] = 0.0f;
        for (int j = 0; j < g.count[k]; j++) {
            const uint16_t* x = X + (size_t)g.n_of_row[g.first[k] + j] * Ci;
            for (int c = 0; c < Ci; c++) mk[c] = mk[c] + or_bf16_value(x[c]);
        }
        const float cnt = (float)g.count[k];
        for (int c = 0; c < Ci; c++) mk[c] = mk[c] / cnt;
        fp8_token(mk, Ci, q8 + (size_t)i * Ci, s8 + i);
        for (int j = 0; j < g.count[k]; j++) {
            const uint16_t* x = X + (size_t)g.n_of_row[g.first[k] + j] * Ci;
            const long long r = first_row[i] + j;
            for (int c = 0; c < Ci; c++) z[c] = or_bf16_value(x[c]) - mk[c];
            fp4_row(z, Ci, S, dcodes + (size_t)r * (Ci / 2), dscales + (size_t)r * (Ci / 16));
        }
        free(mk);
        free(z);
    }
    geom_free(&g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Weight side (key design 4, Eq. 3: R = W - L1 L2, quantised to FP4)        */
/* ------------------------------------------------------------------------ */

/*
 * Residual R[o][i] = fl32( W[o][i] - sum_j L1[i][j] L2[j][o] ), the sum in
 * fp64 over ascending j.  W: Co x Ci (y = x W^T), L1: Ci x r, L2: r x Co.
 */
int or_residual(const uint16_t* Wt, const uint16_t* L1, const uint16_t* L2, int Co, int Ci, int r, float* R) {
#pragma omp parallel for schedule(static)
    for (long long o = 0; o < Co; o++) {
        for (int i = 0; i < Ci; i++) {
            double s = 0.0;
            for (int j = 0; j < r; j++)
                s = s + (double)or_bf16_value(L1[(size_t)i * r + j]) * (double)or_bf16_value(L2[(size_t)j * Co + o]);
            R[(size_t)o * Ci + i] = (float)((double)or_bf16_value(Wt[(size_t)o * Ci + i]) - s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Output (Eq. 3), fp64                                                      */
/* ------------------------------------------------------------------------ */

/*
 * Y rows in fp64 from the dequantised operands:
 *   Y[n][o] =  sum_c dqA[a(n)][c] dqR[o][c]                    (low-bit term)
 *            + sum_c s8[k(n)][c / s8_group] q8[k(n)][c] dqR[o][c] (single-token term)
 *            + sum_j (sum_c x[n][c] L1[c][j]) L2[j][o]           (low-rank term)
 * acodes/ascales: FP4 activation rows with per-tensor S_a; a(n) = arow_of_n[n]
 * (identity when NULL).  q8 == NULL drops the single-token term; L1 == NULL
 * drops the low-rank term.  rows[]: natural token indices to evaluate.
 */
int or_output_rows(const uint8_t* acodes, const uint8_t* ascales, float S_a, const int* arow_of_n,
                   const uint8_t* q8, const float* s8, int s8_group, const int* cube_of_n,
                   const uint8_t* wcodes, const uint8_t* wscales, float S_w, int Co, int Ci,
                   const uint16_t* X, const uint16_t* L1, const uint16_t* L2, int r,
                   const long long* rows, long long nrows, double* Y) {
    double* dqR = (double*)malloc(sizeof(double) * (size_t)Co * Ci);
    if (!dqR) return 2;
#pragma omp parallel for schedule(static)
    for (long long o = 0; o < Co; o++)
        for (int c = 0; c < Ci; c++) {
            int code = (wcodes[(size_t)o * (Ci / 2) + c / 2] >> (4 * (c & 1))) & 15;
            dqR[(size_t)o * Ci + c] =
                or_e2m1_value(code) * or_e4m3_value(wscales[(size_t)o * (Ci / 16) + c / 16]) * (double)S_w;
        }
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = 0; i < nrows; i++) {
        long long n = rows[i];
        long long a = arow_of_n ? arow_of_n[n] : n;
        double* dqA = (double*)malloc(sizeof(double) * (size_t)Ci);
        double* dqK = (double*)malloc(sizeof(double) * (size_t)Ci);
        double* U = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        for (int c = 0; c < Ci; c++) {
            int code = (acodes[(size_t)a * (Ci / 2) + c / 2] >> (4 * (c & 1))) & 15;
            dqA[c] = or_e2m1_value(code) * or_e4m3_value(ascales[(size_t)a * (Ci / 16) + c / 16]) * (double)S_a;
        }
        if (q8) {
            long long k = cube_of_n[n];
            const int ng = Ci / s8_group;
            for (int c = 0; c < Ci; c++)
                dqK[c] = or_e4m3_value(q8[(size_t)k * Ci + c]) * (double)s8[(size_t)k * ng + c / s8_group];
        }
        if (L1) {
            for (int j = 0; j < r; j++) {
                double s = 0.0;
                for (int c = 0; c < Ci; c++)
                    s += (double)or_bf16_value(X[(size_t)n * Ci + c]) * (double)or_bf16_value(L1[(size_t)c * r + j]);
                U[j] = s;
            }
        }
        for (int o = 0; o < Co; o++) {
            const double* wr = dqR + (size_t)o * Ci;
            double t1 = 0.0, t2 = 0.0, t3 = 0.0;
            for (int c = 0; c < Ci; c++) t1 += dqA[c] * wr[c];
            if (q8)
                for (int c = 0; c < Ci; c++) t2 += dqK[c] * wr[c];
            if (L1)
                for (int j = 0; j < r; j++) t3 += U[j] * (double)or_bf16_value(L2[(size_t)j * Co + o]);
            Y[(size_t)i * Co + o] = t1 + t2 + t3;
        }
        free(dqA); free(dqK); free(U);
    }
    free(dqR);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the element encoders (for exhaustive format checks)        */
/* ------------------------------------------------------------------------ */

void or_e2m1_encode_array(const float* v, long long n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++) out[i] = (uint8_t)or_e2m1_encode(v[i]);
}

void or_e4m3_encode_array(const float* v, long long n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++) out[i] = (uint8_t)or_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Feed-forward block: the activation between the up- and down-projection     */
/* ------------------------------------------------------------------------ */

/* GELU in its exact form: GELU(y) = y * Phi(y), Phi the standard normal CDF,
 * Phi(y) = erfc(-y / sqrt 2) / 2 (erfc keeps Phi accurate for large negative
 * y, where 1 + erf would cancel).  fp64, element by element. */
void or_gelu_erf(const double* y, long long n, double* out) {
    for (long long i = 0; i < n; i++) out[i] = 0.5 * y[i] * erfc(-y[i] / sqrt(2.0));
}

/* Threads an OpenMP loop of this file uses (for reporting the CPU baseline). */
int or_num_threads(void) { return omp_get_max_threads(); }
