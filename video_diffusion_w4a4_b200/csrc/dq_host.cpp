// Host side of libdeltaquant: status strings, layout maps and the offline
// weight packer (truncated SVD, residual, FP4 quantisation, tensor-core
// layouts).
//
// The packer follows the DeltaQuant note (papernotes.org, "DeltaQuant:
// 4-bit Video Diffusion Models with Spatiotemporal Delta Smoothing"), key
// design 4, Eq. 3 (W ~ L1 L2 + R with R quantised to FP4, after SVDQuant) and
// Eq. 4 (s = max|X| / q_max per group), in the NVFP4 two-level form: one
// fp32 per-tensor scale S = amax / (6 * 448) and one E4M3 scale per 16 input
// channels.  All fp32 steps are single IEEE operations (compiled with
// -ffp-contract=off).
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "../../include/deltaquant.h"
#include "dq_common.h"

namespace {

// ------------------------------------------------------------------ formats

inline float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

// fp64 -> BF16 round-to-nearest-even, computed on the integer grid of the
// value's binade (so there is no intermediate fp32 rounding).
inline uint16_t double_to_bf16(double v) {
    if (v != v) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                          // a in [2^(e-1), 2^e)
    int eu = e - 1;
    if (eu < -126) eu = -126;              // subnormal spacing 2^-133
    double q = ldexp(a, 7 - eu);           // significand on an integer grid [128, 256)
    double r = nearbyint(q);               // ties to even
    if (r >= 256.0) { r = 128.0; eu += 1; }
    if (eu > 127) return sign | 0x7F80;    // overflow -> inf
    uint32_t mant = (uint32_t)r;
    uint16_t bits;
    if (mant < 128)
        bits = (uint16_t)mant;             // subnormal
    else
        bits = (uint16_t)(((uint32_t)(eu + 127) << 7) | (mant - 128));
    return sign | bits;
}

// fp32 -> E4M3 (max 448, no infinities), round to nearest even, saturating.
inline uint8_t float_to_e4m3(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0;
    float a = fabsf(v);
    if (a != a) return sign | 0x7F;
    if (a > 448.0f) return sign | 0x7E;
    if (a == 0.0f) return sign;
    int e;
    frexpf(a, &e);
    int eu = e - 1;                        // a in [2^eu, 2^(eu+1))
    if (eu < -6) eu = -6;                  // subnormals share the spacing 2^-9
    float q = ldexpf(a, 3 - eu);           // exact: power-of-two scaling
    float r = rintf(q);                    // ties to even
    uint32_t m = (uint32_t)r;
    if (m >= 16) { m = 8; eu += 1; }
    if (m < 8) return sign | (uint8_t)m;   // subnormal (eu == -6)
    return sign | (uint8_t)(((eu + 7) << 3) | (m - 8));
}

inline float e4m3_to_float(uint8_t c) {
    int e = (c >> 3) & 15, m = c & 7;
    float v = (e == 0) ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    return (c & 0x80) ? -v : v;
}

// fp32 -> E2M1, round to nearest even, saturating at 6.  The thresholds are
// the midpoints of {0, .5, 1, 1.5, 2, 3, 4, 6}; a value on a midpoint goes to
// the level with the even code.
inline uint8_t float_to_e2m1(float v) {
    uint8_t sign = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    uint8_t c;
    if (a <= 0.25f) c = 0;
    else if (a < 0.75f) c = 1;
    else if (a <= 1.25f) c = 2;
    else if (a < 1.75f) c = 3;
    else if (a <= 2.5f) c = 4;
    else if (a < 3.5f) c = 5;
    else if (a <= 5.0f) c = 6;
    else c = 7;
    return sign | c;
}

inline float e2m1_to_float(uint8_t c) {
    static const float mag[8] = {0.f, .5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
    float v = mag[c & 7];
    return (c & 8) ? -v : v;
}

// Restricted group scales of C2 weights: 0 and the values m 2^e (m in {1, 1.25, 1.5}) that E4M3
// holds, up to 384, in increasing order.  Their products with E2M1 values have at most three
// fraction bits, so each product is an E4M3 value times a power of two.  Built from the E4M3
// code table: normal codes whose 3-bit mantissa is 0, 2 or 4, and subnormal codes 1..6 (k 2^-9,
// each of the form m 2^e; 7 2^-9 = 1.75 x 2^-7 is not).
const std::vector<float>& c2_scale_set() {
    static const std::vector<float> set = [] {
        std::vector<float> v{0.0f};
        for (int code = 1; code < 0x7F; code++) {
            const int e = code >> 3, m = code & 7;
            const bool ok = e == 0 ? m <= 6 : (m == 0 || m == 2 || m == 4);
            const float val = e4m3_to_float((uint8_t)code);
            if (ok && val <= 384.0f) v.push_back(val);
        }
        std::sort(v.begin(), v.end());
        return v;
    }();
    return set;
}

// The member nearest to v >= 0, ties to the larger.
inline float c2_scale_nearest(float v) {
    const std::vector<float>& S = c2_scale_set();
    const auto it = std::lower_bound(S.begin(), S.end(), v);   // first member >= v
    if (it == S.end()) return S.back();
    if (it == S.begin()) return *it;
    const float hi = *it, lo = *(it - 1);
    return ((double)hi - v <= (double)v - lo) ? hi : lo;
}

// The smallest member >= v (v > 0, at most the largest member).
inline float c2_scale_at_least(double v) {
    const std::vector<float>& S = c2_scale_set();
    for (float c : S)
        if ((double)c >= v) return c;
    return S.back();
}

// ------------------------------------------------------------------ small dense linear algebra (fp64)

// Y (m x l) = A (m x n, row-major) * B (n x l, row-major)
void matmul_nn(const double* A, const double* B, double* Y, long m, long n, int l) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < m; i++) {
        double* y = Y + (size_t)i * l;
        for (int j = 0; j < l; j++) y[j] = 0.0;
        const double* a = A + (size_t)i * n;
        for (long k = 0; k < n; k++) {
            double av = a[k];
            const double* b = B + (size_t)k * l;
            for (int j = 0; j < l; j++) y[j] += av * b[j];
        }
    }
}

// Z (n x l) = A^T (A: m x n row-major) * Y (m x l)
void matmul_tn(const double* A, const double* Y, double* Z, long m, long n, int l) {
    const long blk = 64;
#pragma omp parallel for schedule(dynamic, 1)
    for (long i0 = 0; i0 < n; i0 += blk) {
        long i1 = std::min(n, i0 + blk);
        for (long i = i0; i < i1; i++)
            for (int j = 0; j < l; j++) Z[(size_t)i * l + j] = 0.0;
        for (long k = 0; k < m; k++) {
            const double* a = A + (size_t)k * n;
            const double* y = Y + (size_t)k * l;
            for (long i = i0; i < i1; i++) {
                double av = a[i];
                double* z = Z + (size_t)i * l;
                for (int j = 0; j < l; j++) z[j] += av * y[j];
            }
        }
    }
}

// Orthonormalise the l columns of Q (m x l, row-major) by Cholesky QR applied
// twice: G = Q^T Q, G = L L^T, Q <- Q L^-T.  A column whose Cholesky pivot
// vanishes (linearly dependent on earlier ones) is set to zero.
void orthonormalise(double* Q, long m, int l) {
    std::vector<double> G((size_t)l * l), Lc((size_t)l * l);
    std::vector<char> dead(l);
    for (int pass = 0; pass < 2; pass++) {
        std::fill(G.begin(), G.end(), 0.0);
#pragma omp parallel
        {
            std::vector<double> g((size_t)l * l, 0.0);
#pragma omp for schedule(static) nowait
            for (long r = 0; r < m; r++) {
                const double* q = Q + (size_t)r * l;
                for (int a = 0; a < l; a++) {
                    double qa = q[a];
                    double* ga = &g[(size_t)a * l];
                    for (int b = a; b < l; b++) ga[b] += qa * q[b];
                }
            }
#pragma omp critical
            for (size_t i = 0; i < g.size(); i++) G[i] += g[i];
        }
        double dmax = 0.0;
        for (int a = 0; a < l; a++) dmax = std::max(dmax, G[(size_t)a * l + a]);
        std::fill(Lc.begin(), Lc.end(), 0.0);
        for (int j = 0; j < l; j++) {
            double d = G[(size_t)j * l + j];
            for (int k = 0; k < j; k++) d -= Lc[(size_t)j * l + k] * Lc[(size_t)j * l + k];
            dead[j] = !(d > 1e-13 * dmax) || dead[j];
            double ljj = dead[j] ? 0.0 : sqrt(d);
            Lc[(size_t)j * l + j] = ljj;
            for (int i = j + 1; i < l; i++) {
                double v = G[(size_t)j * l + i];   // upper triangle holds G[j][i]
                for (int k = 0; k < j; k++) v -= Lc[(size_t)i * l + k] * Lc[(size_t)j * l + k];
                Lc[(size_t)i * l + j] = dead[j] ? 0.0 : v / ljj;
            }
        }
#pragma omp parallel for schedule(static)
        for (long r = 0; r < m; r++) {
            double* q = Q + (size_t)r * l;
            for (int j = 0; j < l; j++) {
                if (dead[j]) {
                    q[j] = 0.0;
                    continue;
                }
                double v = q[j];
                for (int k = 0; k < j; k++) v -= q[k] * Lc[(size_t)j * l + k];
                q[j] = v / Lc[(size_t)j * l + j];
            }
        }
    }
}

// Symmetric eigen-decomposition of G (l x l) by cyclic Jacobi rotations.
// On return G's diagonal holds the eigenvalues and V (row-major, columns =
// eigenvectors) the vectors.
void jacobi_eigen(std::vector<double>& G, std::vector<double>& V, int l) {
    V.assign((size_t)l * l, 0.0);
    for (int i = 0; i < l; i++) V[(size_t)i * l + i] = 1.0;
    for (int sweep = 0; sweep < 100; sweep++) {
        double off = 0.0, tot = 0.0;
        for (int i = 0; i < l; i++)
            for (int j = 0; j < l; j++) {
                double g2 = G[(size_t)i * l + j] * G[(size_t)i * l + j];
                tot += g2;
                if (i != j) off += g2;
            }
        if (off <= 1e-30 * tot || off == 0.0) break;
        for (int p = 0; p < l - 1; p++)
            for (int q = p + 1; q < l; q++) {
                double apq = G[(size_t)p * l + q];
                if (fabs(apq) < 1e-300) continue;
                double app = G[(size_t)p * l + p], aqq = G[(size_t)q * l + q];
                double theta = (aqq - app) / (2.0 * apq);
                double tt = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                double c = 1.0 / sqrt(tt * tt + 1.0), s = tt * c;
                for (int k = 0; k < l; k++) {
                    double gkp = G[(size_t)k * l + p], gkq = G[(size_t)k * l + q];
                    G[(size_t)k * l + p] = c * gkp - s * gkq;
                    G[(size_t)k * l + q] = s * gkp + c * gkq;
                }
                for (int k = 0; k < l; k++) {
                    double gpk = G[(size_t)p * l + k], gqk = G[(size_t)q * l + k];
                    G[(size_t)p * l + k] = c * gpk - s * gqk;
                    G[(size_t)q * l + k] = s * gpk + c * gqk;
                }
                for (int k = 0; k < l; k++) {
                    double vkp = V[(size_t)k * l + p], vkq = V[(size_t)k * l + q];
                    V[(size_t)k * l + p] = c * vkp - s * vkq;
                    V[(size_t)k * l + q] = s * vkp + c * vkq;
                }
            }
    }
}

inline uint64_t mix64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

inline double sketch_normal(uint64_t seed, uint64_t i) {
    double u1 = ((double)(mix64(seed ^ mix64(2 * i)) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    double u2 = ((double)(mix64(seed ^ mix64(2 * i + 1)) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

bool shape_ok(int Co, int Ci, int rank) {
    return Co >= 256 && Ci >= 256 && Co % 256 == 0 && Ci % 256 == 0 && rank >= 16 && rank <= 128 &&
           rank % 16 == 0 && rank <= std::min(Co, Ci);
}

}  // namespace

extern "C" {

const char* dq_status_string(int status) {
    switch (status) {
        case DQ_OK: return "ok";
        case DQ_ERR_INVALID_ARG: return "invalid argument";
        case DQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case DQ_ERR_ALIGNMENT: return "device pointer not 256-byte aligned";
        case DQ_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case DQ_ERR_CUDA: return "CUDA runtime error";
        case DQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case DQ_ERR_BAD_PACKED_WEIGHT: return "packed weight header mismatch";
        case DQ_ERR_NO_DEVICE: return "no usable sm_100 device";
        case DQ_ERR_ALLOC: return "allocation failed";
        default: return "unknown status";
    }
}

int dq_abi_version(void) { return DQ_ABI_VERSION; }

int dq_cube_count(int T, int H, int W, int t, int h, int w, long long* K) {
    if (!K || T <= 0 || H <= 0 || W <= 0 || t <= 0 || h <= 0 || w <= 0 || t > T || h > H || w > W)
        return DQ_ERR_INVALID_ARG;
    *K = dq::make_geom(T, H, W, t, h, w).K;
    return DQ_OK;
}

int dq_cube_major_row(int T, int H, int W, int t, int h, int w, long long n, long long* row, long long* cube) {
    if (!row || !cube || T <= 0 || H <= 0 || W <= 0 || t <= 0 || h <= 0 || w <= 0 || t > T || h > H || w > W)
        return DQ_ERR_INVALID_ARG;
    dq::Geom g = dq::make_geom(T, H, W, t, h, w);
    if (n < 0 || n >= g.N) return DQ_ERR_INVALID_ARG;
    dq::token_to_row(g, n, row, cube);
    return DQ_OK;
}

int dq_sf_offset(long long row, int block, int cols, size_t* offset) {
    if (!offset || row < 0 || cols <= 0 || cols % 64 || block < 0 || block >= cols / 16) return DQ_ERR_INVALID_ARG;
    *offset = dq::sf_offset(row, block, cols);
    return DQ_OK;
}

int dq_sf_bytes(long long rows, int cols, size_t* bytes) {
    if (!bytes || rows < 0 || cols <= 0 || cols % 64) return DQ_ERR_INVALID_ARG;
    *bytes = dq::sf_bytes(rows, cols);
    return DQ_OK;
}

int dq_sfa_offset(long long row, int block, int cols, size_t* offset) {
    if (!offset || row < 0 || cols <= 0 || cols % 256 || block < 0 || block >= cols / 16) return DQ_ERR_INVALID_ARG;
    *offset = dq::sfa_offset(row, block, cols);
    return DQ_OK;
}

int dq_sfa_bytes(long long rows, int cols, size_t* bytes) {
    if (!bytes || rows < 0 || cols <= 0 || cols % 256) return DQ_ERR_INVALID_ARG;
    *bytes = dq::sfa_bytes(rows, cols);
    return DQ_OK;
}

int dq_sfb_offset(long long row, int block, int cols, size_t* offset) {
    if (!offset || row < 0 || cols <= 0 || cols % 64 || block < 0 || block >= cols / 16) return DQ_ERR_INVALID_ARG;
    *offset = dq::sfb_offset(row, block, cols);
    return DQ_OK;
}

int dq_sfb_bytes(long long rows, int cols, size_t* bytes) {
    if (!bytes || rows < 0 || cols <= 0 || cols % 64) return DQ_ERR_INVALID_ARG;
    *bytes = dq::sfb_bytes(rows, cols);
    return DQ_OK;
}

int dq_lowrank_slab_width(int rank) { return (rank > 0) ? dq::slab_width(rank) : 0; }

int dq_packed_weight_layout(int Co, int Ci, int rank, dq_packed_layout* out) {
    if (!out) return DQ_ERR_INVALID_ARG;
    if (!shape_ok(Co, Ci, rank)) return DQ_ERR_UNSUPPORTED_SHAPE;
    dq::PackedLayout L = dq::packed_layout(Co, Ci, rank);
    out->total_bytes = L.total;
    out->off_codes = L.off_codes;
    out->off_scales = L.off_scales;
    out->off_dqw = L.off_dqw;
    out->off_bias = L.off_bias;
    out->Co = Co; out->Ci = Ci; out->rank = rank; out->slab = L.slab;
    return DQ_OK;
}

int dq_packed_weight_bytes(int Co, int Ci, int rank, size_t* bytes) {
    if (!bytes) return DQ_ERR_INVALID_ARG;
    dq_packed_layout L;
    int rc = dq_packed_weight_layout(Co, Ci, rank, &L);
    if (rc) return rc;
    *bytes = L.total_bytes;
    return DQ_OK;
}

int dq_lowrank_factors(const uint16_t* Wb, int Co, int Ci, int rank, uint64_t seed, uint16_t* L1, uint16_t* L2) {
    if (!Wb || !L1 || !L2) return DQ_ERR_INVALID_ARG;
    if (!shape_ok(Co, Ci, rank)) return DQ_ERR_UNSUPPORTED_SHAPE;
    const long m = Co, n = Ci;
    // oversampling max(32, r) and 16 power iterations: within 1e-4 of the
    // optimal rank-r error on the spectra used here (outlier columns over a
    // Marchenko-Pastur bulk), which has no gap at r
    const int l = std::min<int>(std::min(Co, Ci), rank + std::max(32, rank));
    const int iters = 16;
    std::vector<double> W((size_t)m * n), Om((size_t)n * l), Y((size_t)m * l), Z((size_t)n * l);
#pragma omp parallel for schedule(static)
    for (long i = 0; i < m * n; i++) W[i] = (double)bf16_to_float(Wb[i]);
    uint64_t key = mix64(seed ^ 0xC0FFEE1234567ull);
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n * l; i++) Om[i] = sketch_normal(key, (uint64_t)i);
    // range finder with power iterations: Y = (W W^T)^q W Omega
    matmul_nn(W.data(), Om.data(), Y.data(), m, n, l);
    orthonormalise(Y.data(), m, l);
    for (int it = 0; it < iters; it++) {
        matmul_tn(W.data(), Y.data(), Z.data(), m, n, l);
        orthonormalise(Z.data(), n, l);
        matmul_nn(W.data(), Z.data(), Y.data(), m, n, l);
        orthonormalise(Y.data(), m, l);
    }
    // B^T = W^T Q (n x l); G = B B^T (l x l)
    std::vector<double> Bt((size_t)n * l);
    matmul_tn(W.data(), Y.data(), Bt.data(), m, n, l);
    std::vector<double> G((size_t)l * l, 0.0), V;
    for (int a = 0; a < l; a++)
        for (int b = a; b < l; b++) {
            double s = 0.0;
            for (long i = 0; i < n; i++) s += Bt[(size_t)i * l + a] * Bt[(size_t)i * l + b];
            G[(size_t)a * l + b] = s;
            G[(size_t)b * l + a] = s;
        }
    jacobi_eigen(G, V, l);
    std::vector<int> order(l);
    for (int a = 0; a < l; a++) order[a] = a;
    std::sort(order.begin(), order.end(),
              [&](int x, int y) { return G[(size_t)x * l + x] > G[(size_t)y * l + y]; });
    // sigma_a, left vectors U = Q V_a, right vectors v_a = B^T V_a / sigma_a
    for (int a = 0; a < rank; a++) {
        int e = order[a];
        double lam = std::max(0.0, G[(size_t)e * l + e]);
        double sig = sqrt(lam);
        double rs = sqrt(sig);
        for (long o = 0; o < m; o++) {
            double u = 0.0;
            for (int b = 0; b < l; b++) u += Y[(size_t)o * l + b] * V[(size_t)b * l + e];
            L2[(size_t)a * Co + o] = double_to_bf16(rs * u);
        }
        for (long i = 0; i < n; i++) {
            double v = 0.0;
            for (int b = 0; b < l; b++) v += Bt[(size_t)i * l + b] * V[(size_t)b * l + e];
            L1[(size_t)i * rank + a] = double_to_bf16(sig > 0 ? v / rs : 0.0);
        }
    }
    return DQ_OK;
}

int dq_pack_weight_factors_ex(const uint16_t* Wb, const uint16_t* L1, const uint16_t* L2, int Co, int Ci, int rank,
                              int pack_flags, void* packed, size_t packed_bytes, uint16_t* L1_mma, uint16_t* L2_slab,
                              float* S_W_out) {
    if (!Wb || !L1 || !L2 || !packed) return DQ_ERR_INVALID_ARG;
    if (pack_flags & ~DQ_PACK_C2) return DQ_ERR_INVALID_ARG;
    const bool c2 = (pack_flags & DQ_PACK_C2) != 0;
    if (!shape_ok(Co, Ci, rank)) return DQ_ERR_UNSUPPORTED_SHAPE;
    dq::PackedLayout L = dq::packed_layout(Co, Ci, rank);
    if (packed_bytes < L.total) return DQ_ERR_INVALID_ARG;
    const int r = rank;
    // residual R = W - L1 L2 (fp64 sum over ascending j, rounded once to fp32)
    std::vector<float> R((size_t)Co * Ci);
    std::vector<double> l2t((size_t)Co * r), l1d((size_t)Ci * r);
    for (int j = 0; j < r; j++)
        for (int o = 0; o < Co; o++) l2t[(size_t)o * r + j] = (double)bf16_to_float(L2[(size_t)j * Co + o]);
    for (size_t i = 0; i < (size_t)Ci * r; i++) l1d[i] = (double)bf16_to_float(L1[i]);
    float amax = 0.0f;
#pragma omp parallel for schedule(static) reduction(max : amax)
    for (long o = 0; o < Co; o++) {
        const double* b = &l2t[(size_t)o * r];
        for (int i = 0; i < Ci; i++) {
            const double* a = &l1d[(size_t)i * r];
            double s = 0.0;
            for (int j = 0; j < r; j++) s = s + a[j] * b[j];
            float v = (float)((double)bf16_to_float(Wb[(size_t)o * Ci + i]) - s);
            R[(size_t)o * Ci + i] = v;
            amax = std::max(amax, fabsf(v));
        }
    }
    // per-tensor scale: amax / (6 q_max) with q_max the largest group scale (448; 384 = 1.5 x 2^8 for C2)
    const float S = (amax == 0.0f) ? 1.0f : amax / (c2 ? 2304.0f : 2688.0f);
    const float denom = 6.0f * S;
    uint8_t* base = (uint8_t*)packed;
    memset(base, 0, L.total);
    uint8_t* codes = base + L.off_codes;
    uint8_t* scales = base + L.off_scales;
    uint16_t* dqw = (uint16_t*)(base + L.off_dqw);
    if (c2) {
        // C2: per 32 channels, two restricted group scales (a nonzero smaller one raised to the smallest
        // member >= 2^-9 of the larger, so the 32 values q s_b fit E4M3 exactly under one UE8M0 exponent),
        // E2M1 codes, and the FP8 form: E4M3 codes of q s_b / 2^u with the block's largest |q s_b| / 2^u in
        // [128, 256) (E4M3 stops at 448, below 1.875 x 256)
        uint8_t* fp8 = base + L.off_dqw;
        uint8_t* ue = fp8 + (size_t)Co * Ci;
#pragma omp parallel for schedule(static)
        for (long o = 0; o < Co; o++) {
            const float* z = &R[(size_t)o * Ci];
            for (int j = 0; j < Ci / 32; j++) {
                float sb[2];
                for (int hh = 0; hh < 2; hh++) {
                    float am = 0.0f;
                    for (int i = 0; i < 16; i++) am = std::max(am, fabsf(z[32 * j + 16 * hh + i]));
                    sb[hh] = c2_scale_nearest(am / denom);
                }
                const double floor_s = ldexp((double)std::max(sb[0], sb[1]), -9);
                float w[32], wmax = 0.0f;
                for (int hh = 0; hh < 2; hh++) {
                    const float sbv = (sb[hh] > 0.0f && sb[hh] < floor_s) ? c2_scale_at_least(floor_s) : sb[hh];
                    const uint8_t code = float_to_e4m3(sbv);   // exact: a restricted scale is an E4M3 value
                    const int b = 2 * j + hh;
                    const size_t so = dq::sfb_offset(o, b, Ci);
                    for (int q = 0; q < 4; q++) scales[so + 1024 * q] = code;
                    const float eff = sbv * S;
                    for (int i = 0; i < 16; i += 2) {
                        const uint8_t q0 = (eff == 0.0f) ? 0 : float_to_e2m1(z[b * 16 + i] / eff);
                        const uint8_t q1 = (eff == 0.0f) ? 0 : float_to_e2m1(z[b * 16 + i + 1] / eff);
                        codes[(size_t)o * (Ci / 2) + (b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
                        w[16 * hh + i] = e2m1_to_float(q0) * sbv;       // exact products
                        w[16 * hh + i + 1] = e2m1_to_float(q1) * sbv;
                    }
                }
                for (int i = 0; i < 32; i++) wmax = std::max(wmax, fabsf(w[i]));
                int u = 0;
                if (wmax > 0.0f) {
                    int e;
                    frexpf(wmax, &e);    // wmax in [2^(e-1), 2^e)
                    u = e - 8;
                }
                for (int i = 0; i < 32; i++) fp8[(size_t)o * Ci + 32 * j + i] = float_to_e4m3(ldexpf(w[i], -u));
                const size_t uo = dq::c2_sf_offset(o, j, Ci);
                for (int q = 0; q < 4; q++) ue[uo + 1024 * q] = (uint8_t)(u + 127);
            }
        }
    }
#pragma omp parallel for schedule(static)
    for (long o = 0; o < (c2 ? 0 : Co); o++) {
        const float* z = &R[(size_t)o * Ci];
        for (int b = 0; b < Ci / 16; b++) {
            float am = 0.0f;
            for (int i = 0; i < 16; i++) am = std::max(am, fabsf(z[b * 16 + i]));
            uint8_t sb = float_to_e4m3(am / denom);
            float sbv = e4m3_to_float(sb);
            float eff = sbv * S;
            const size_t so = dq::sfb_offset(o, b, Ci);
            for (int q = 0; q < 4; q++) scales[so + 1024 * q] = sb;   // one copy per tensor-memory quadrant
            for (int i = 0; i < 16; i += 2) {
                uint8_t q0 = (eff == 0.0f) ? 0 : float_to_e2m1(z[b * 16 + i] / eff);
                uint8_t q1 = (eff == 0.0f) ? 0 : float_to_e2m1(z[b * 16 + i + 1] / eff);
                codes[(size_t)o * (Ci / 2) + (b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
                // q * s_b has at most 6 significant bits: exact in BF16
                dqw[(size_t)o * Ci + b * 16 + i] = double_to_bf16((double)e2m1_to_float(q0) * sbv);
                dqw[(size_t)o * Ci + b * 16 + i + 1] = double_to_bf16((double)e2m1_to_float(q1) * sbv);
            }
        }
    }
    dq::PackedHeader hdr;
    memset(&hdr, 0, sizeof(hdr));
    hdr.magic = DQ_PACK_MAGIC;
    hdr.version = DQ_PACK_FORMAT_VERSION;
    hdr.Co = Co; hdr.Ci = Ci; hdr.rank = r; hdr.slab = L.slab;
    hdr.S_W = S;
    hdr.off_codes = L.off_codes; hdr.off_scales = L.off_scales; hdr.off_dqw = L.off_dqw; hdr.total = L.total;
    hdr.off_bias = L.off_bias;
    hdr.flags = c2 ? dq::kPackedC2 : 0u;
    memcpy(base, &hdr, sizeof(hdr));
    if (L1_mma)
        for (int i = 0; i < Ci; i++)
            for (int j = 0; j < r; j++) L1_mma[(size_t)j * Ci + i] = L1[(size_t)i * r + j];
    if (L2_slab)
        for (int o = 0; o < Co; o++)
            for (int c = 0; c < L.slab; c++)
                L2_slab[(size_t)o * L.slab + c] = (c < 2 * r) ? L2[(size_t)(c % r) * Co + o] : (uint16_t)0;
    if (S_W_out) *S_W_out = S;
    return DQ_OK;
}

int dq_pack_weight_factors(const uint16_t* Wb, const uint16_t* L1, const uint16_t* L2, int Co, int Ci, int rank,
                           void* packed, size_t packed_bytes, uint16_t* L1_mma, uint16_t* L2_slab, float* S_W_out) {
    return dq_pack_weight_factors_ex(Wb, L1, L2, Co, Ci, rank, 0, packed, packed_bytes, L1_mma, L2_slab, S_W_out);
}

int dq_pack_bias(const uint16_t* bias, int Co, void* packed, size_t packed_bytes) {
    if (!packed || packed_bytes < sizeof(dq::PackedHeader)) return DQ_ERR_INVALID_ARG;
    dq::PackedHeader hdr;
    memcpy(&hdr, packed, sizeof(hdr));
    if (hdr.magic != DQ_PACK_MAGIC || hdr.version != DQ_PACK_FORMAT_VERSION || hdr.Co != Co ||
        !shape_ok(hdr.Co, hdr.Ci, hdr.rank))
        return DQ_ERR_BAD_PACKED_WEIGHT;
    const dq::PackedLayout L = dq::packed_layout(hdr.Co, hdr.Ci, hdr.rank);
    if (hdr.total != L.total || hdr.off_bias != L.off_bias) return DQ_ERR_BAD_PACKED_WEIGHT;
    if (packed_bytes < L.total) return DQ_ERR_INVALID_ARG;
    float* b = (float*)((uint8_t*)packed + L.off_bias);
    for (int o = 0; o < Co; o++) b[o] = bias ? bf16_to_float(bias[o]) : 0.0f;
    hdr.flags = bias ? (hdr.flags | dq::kPackedHasBias) : (hdr.flags & ~dq::kPackedHasBias);
    memcpy(packed, &hdr, sizeof(hdr));
    return DQ_OK;
}

int dq_pack_weight(const uint16_t* Wb, int Co, int Ci, int rank, void* packed, size_t packed_bytes, uint16_t* L1_mma,
                   uint16_t* L2_slab) {
    if (!Wb || !packed) return DQ_ERR_INVALID_ARG;
    if (!shape_ok(Co, Ci, rank)) return DQ_ERR_UNSUPPORTED_SHAPE;
    std::vector<uint16_t> L1((size_t)Ci * rank), L2((size_t)rank * Co);
    int rc = dq_lowrank_factors(Wb, Co, Ci, rank, 0, L1.data(), L2.data());
    if (rc) return rc;
    return dq_pack_weight_factors(Wb, L1.data(), L2.data(), Co, Ci, rank, packed, packed_bytes, L1_mma, L2_slab,
                                  nullptr);
}

}  // extern "C"
