/*
 * Seeded synthetic inputs for the DeltaQuant W4A4 linear layer.
 *
 * This module only draws random numbers and shapes them into activation and
 * weight tensors with the structure the DeltaQuant page describes for video
 * diffusion activations (papernotes.org, "DeltaQuant: 4-bit Video Diffusion
 * Models with Spatiotemporal Delta Smoothing", key design 1: neighbouring
 * tokens in time and space are highly similar while outlier channels move
 * with the denoising step).  It holds none of the method's arithmetic: no
 * means, no deltas, no quantisers.  Both the CUDA path's tests and the CPU
 * oracle read the same tensors from here.
 *
 * Random numbers: a counter-based generator.  Each value is addressed by
 * (seed, stream, index) and made by the SplitMix64 finaliser (Steele, Lea and
 * Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014), so
 * any element can be generated independently and in parallel.  Normals come
 * from the Box-Muller transform in fp64.  BF16 casts round to nearest even
 * from the fp32 value.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

static inline uint64_t sm64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

static inline uint64_t key_of(uint64_t seed, uint64_t stream) {
    return sm64(sm64(seed) ^ (stream * 0xD1B54A32D192ED03ull));
}

static inline uint64_t draw(uint64_t key, uint64_t idx) { return sm64(key + sm64(idx)); }

/* uniform on the open interval (0, 1) */
static inline double unif(uint64_t key, uint64_t idx) {
    return ((double)(draw(key, idx) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double gauss(uint64_t key, uint64_t idx) {
    double u1 = unif(key, 2 * idx), u2 = unif(key, 2 * idx + 1);
    return sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);
}

static inline uint16_t to_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Pick round(frac * n) distinct indices (partial Fisher-Yates); mark[i] = 1. */
static void pick_subset(uint64_t key, int n, double frac, unsigned char* mark) {
    if (n <= 0) return;
    int cnt = (int)floor(frac * n + 0.5);
    int* perm = (int*)malloc(sizeof(int) * (size_t)n);
    for (int i = 0; i < n; i++) perm[i] = i;
    for (int i = 0; i < cnt && i < n; i++) {
        int j = i + (int)(draw(key, (uint64_t)i) % (uint64_t)(n - i));
        int t = perm[i]; perm[i] = perm[j]; perm[j] = t;
    }
    memset(mark, 0, (size_t)n);
    for (int i = 0; i < cnt && i < n; i++) mark[perm[i]] = 1;
    free(perm);
}

/* align-corners coordinate of sample i of n on a grid of g points */
static inline void corner(int i, int n, int g, int* i0, int* i1, double* f) {
    double u = (g > 1 && n > 1) ? (double)i * (double)(g - 1) / (double)(n - 1) : 0.0;
    int a = (int)floor(u);
    if (a > g - 1) a = g - 1;
    *i0 = a;
    *i1 = (a + 1 < g) ? a + 1 : a;
    *f = u - (double)a;
}

enum { S_SCALE = 1, S_BIAS = 2, S_OUTLIER = 3, S_GRID = 4, S_NOISE = 5, S_W = 10, S_WOUT = 11 };

/*
 * Activations X, N = T*H*W rows in (t,h,w) row-major order, Ci channels, BF16.
 *   field G_c(t,h,w): N(0,1) values on a gT x gH x gW grid per channel,
 *                     trilinearly interpolated (align-corners) to T x H x W.
 *   gelu == 0: x = s_c * (b_c + G_c + 0.1 eps),  s_c ~ LogNormal(0,1),
 *              b_c ~ N(0,1); outlier channels have s_c multiplied by out_factor.
 *   gelu != 0: x = GELU_erf(G_c + 0.1 eps); outlier channels multiplied by
 *              out_factor after the GELU.
 * The outlier channel set is drawn from stream (S_OUTLIER, tau): a different
 * tau models a different denoising step.
 */
int synth_activations(uint16_t* X, int T, int H, int W, int Ci, int gT, int gH, int gW,
                      int gelu, double out_frac, double out_factor, uint64_t seed, uint64_t tau) {
    if (!X || T <= 0 || H <= 0 || W <= 0 || Ci <= 0 || gT <= 0 || gH <= 0 || gW <= 0) return 1;
    double* sc = (double*)malloc(sizeof(double) * (size_t)Ci);
    double* bc = (double*)malloc(sizeof(double) * (size_t)Ci);
    unsigned char* outl = (unsigned char*)malloc((size_t)Ci);
    size_t gsz = (size_t)gT * gH * gW * Ci;
    double* G = (double*)malloc(sizeof(double) * gsz);
    if (!sc || !bc || !outl || !G) { free(sc); free(bc); free(outl); free(G); return 2; }
    uint64_t k_scale = key_of(seed, S_SCALE), k_bias = key_of(seed, S_BIAS);
    uint64_t k_out = key_of(seed ^ (tau * 0x9E3779B97F4A7C15ull), S_OUTLIER);
    uint64_t k_grid = key_of(seed, S_GRID), k_noise = key_of(seed, S_NOISE);
    pick_subset(k_out, Ci, out_frac, outl);
    for (int c = 0; c < Ci; c++) {
        sc[c] = exp(gauss(k_scale, (uint64_t)c));
        bc[c] = gauss(k_bias, (uint64_t)c);
    }
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)gsz; i++) G[i] = gauss(k_grid, (uint64_t)i);

    long long rowsTH = (long long)T * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long th = 0; th < rowsTH; th++) {
        int t = (int)(th / H), h = (int)(th % H);
        int t0, t1, h0, h1;
        double ft, fh;
        corner(t, T, gT, &t0, &t1, &ft);
        corner(h, H, gH, &h0, &h1, &fh);
        for (int w = 0; w < W; w++) {
            int w0, w1;
            double fw;
            corner(w, W, gW, &w0, &w1, &fw);
            size_t n = ((size_t)th) * W + w;
            const double* g000 = G + (((size_t)t0 * gH + h0) * gW + w0) * Ci;
            const double* g001 = G + (((size_t)t0 * gH + h0) * gW + w1) * Ci;
            const double* g010 = G + (((size_t)t0 * gH + h1) * gW + w0) * Ci;
            const double* g011 = G + (((size_t)t0 * gH + h1) * gW + w1) * Ci;
            const double* g100 = G + (((size_t)t1 * gH + h0) * gW + w0) * Ci;
            const double* g101 = G + (((size_t)t1 * gH + h0) * gW + w1) * Ci;
            const double* g110 = G + (((size_t)t1 * gH + h1) * gW + w0) * Ci;
            const double* g111 = G + (((size_t)t1 * gH + h1) * gW + w1) * Ci;
            double a000 = (1 - ft) * (1 - fh) * (1 - fw), a001 = (1 - ft) * (1 - fh) * fw;
            double a010 = (1 - ft) * fh * (1 - fw), a011 = (1 - ft) * fh * fw;
            double a100 = ft * (1 - fh) * (1 - fw), a101 = ft * (1 - fh) * fw;
            double a110 = ft * fh * (1 - fw), a111 = ft * fh * fw;
            uint16_t* xr = X + n * (size_t)Ci;
            for (int c = 0; c < Ci; c++) {
                double g = a000 * g000[c] + a001 * g001[c] + a010 * g010[c] + a011 * g011[c] +
                           a100 * g100[c] + a101 * g101[c] + a110 * g110[c] + a111 * g111[c];
                double e = gauss(k_noise, (uint64_t)(n * (size_t)Ci + (size_t)c));
                double v;
                if (gelu) {
                    double z = g + 0.1 * e;
                    v = 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
                    if (outl[c]) v *= out_factor;
                } else {
                    double s = outl[c] ? sc[c] * out_factor : sc[c];
                    v = s * (bc[c] + g + 0.1 * e);
                }
                xr[c] = to_bf16(v);
            }
        }
    }
    free(sc); free(bc); free(outl); free(G);
    return 0;
}

/*
 * Weight W (Co x Ci, BF16, y = x W^T): N(0, 1/Ci) entries; a round(out_frac*Ci)
 * subset of input columns is multiplied by out_factor (out_frac = 0: none).
 */
int synth_weight(uint16_t* Wt, int Co, int Ci, double out_frac, double out_factor, uint64_t seed) {
    if (!Wt || Co <= 0 || Ci <= 0) return 1;
    unsigned char* outl = (unsigned char*)malloc((size_t)Ci);
    if (!outl) return 2;
    pick_subset(key_of(seed, S_WOUT), Ci, out_frac, outl);
    uint64_t kw = key_of(seed, S_W);
    double sd = 1.0 / sqrt((double)Ci);
#pragma omp parallel for schedule(static)
    for (long long o = 0; o < Co; o++) {
        for (int i = 0; i < Ci; i++) {
            double v = gauss(kw, (uint64_t)(o * (long long)Ci + i)) * sd;
            if (outl[i]) v *= out_factor;
            Wt[(size_t)o * Ci + i] = to_bf16(v);
        }
    }
    free(outl);
    return 0;
}

/* Plain seeded N(0, sd^2) BF16 values, for operands of stage-level tests. */
int synth_normal_bf16(uint16_t* out, long long n, double sd, uint64_t seed, uint64_t stream) {
    if (!out || n < 0) return 1;
    uint64_t k = key_of(seed, 100 + stream);
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++) out[i] = to_bf16(sd * gauss(k, (uint64_t)i));
    return 0;
}

/* Seeded fp32 values uniform in [lo, hi). */
int synth_uniform_f32(float* out, long long n, double lo, double hi, uint64_t seed, uint64_t stream) {
    if (!out || n < 0) return 1;
    uint64_t k = key_of(seed, 200 + stream);
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++) out[i] = (float)(lo + (hi - lo) * unif(k, (uint64_t)i));
    return 0;
}
