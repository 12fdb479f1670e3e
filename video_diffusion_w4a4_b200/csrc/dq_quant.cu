// Cube-quantise kernels (DeltaQuant note, papernotes.org, key designs 2-4).
//
//   a1  k_cube_stats:  per cube the fp32 mean of its tokens (Eq. 1), the
//       max |mean| over channels (the FP8 kernel-token scale), the global
//       max |token - mean| (the FP4 per-tensor scale), and X L1 (the SVD
//       low-rank down-projection of Eq. 3) on the tensor cores.
//       It stores the means (K x Ci fp32) for the second pass.
//   a2  k_cube_encode: reads X and the means again, writes the FP8 E4M3 kernel
//       tokens, the FP4 E2M1 delta codes with their E4M3 group-16 scales (Eq. 4
//       per group), and U' = (X L1) / (S_delta S_W) as BF16 hi+lo.
//
// Both stream X through 4-D TMA boxes of t x h x (nw w) tokens by 64
// channels straight from the flattened (t,h,w) layout, so that every box
// holds nw whole cubes.  The two passes exist because the per-tensor delta
// scale needs the amax of every delta before any delta can be encoded.
//
// Work item = (box, channel split): the box's tokens over Ci / splits
// channels (chunks of 64).  The kernels are persistent: each CTA walks items
// it = blockIdx.x + n * gridDim.x and one producer thread streams all their
// chunks through one TMA ring.  In a1 a thread owns one (cube, 8 channels)
// task.  In a2 the box's tokens are listed in cube-major order and every
// compute warp owns 16 consecutive rows of that list (two lanes per row, 32
// channels each), with the box's kernel tokens streamed in next to X, so the
// compute warps never wait on one another.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/deltaquant.h"
#include "dq_common.h"
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

namespace {

constexpr int kQStages = 4;
constexpr int kQWarps = 8;                 // compute warps
constexpr int kQCompute = 32 * kQWarps;

struct QSmem {
    // offsets in bytes from the 1024-aligned dynamic smem base
    uint32_t x, x_stride, l1, mt, mt_stride, ms, ms_stride, red2, eff, bars, misc, total;
};

// m_rows: rows of the per-stage tile of kernel tokens (encode kernel; 0 for the statistics kernel)
// x_rows: tokens per TMA box (rows of the X stages; 128 at most)
// single: the single-read statistics kernel, which also keeps the means of two chunks (m_rows cube
// slots x 64 fp32 each) and their per-warp delta maxima
__host__ __device__ inline QSmem q_smem_layout(int rank, bool with_l1, int m_rows, int x_rows = 128,
                                               bool single = false) {
    QSmem L;
    uint32_t off = 0;
    L.x = off;
    L.x_stride = (uint32_t)align_up((size_t)x_rows * 128, 1024);
    off += kQStages * L.x_stride;
    L.l1 = off;
    if (with_l1) off += kQStages * (uint32_t)align_up((size_t)rank * 128, 1024);
    L.mt = off;
    L.mt_stride = single ? 0u : (uint32_t)align_up((size_t)m_rows * 256, 128);
    off += kQStages * L.mt_stride;
    L.ms = off;
    L.ms_stride = single ? (uint32_t)align_up((size_t)m_rows * 256, 128) : 0u;
    off += 2 * L.ms_stride;
    L.red2 = off;
    if (single) off += 2 * kQWarps * 4;
    L.eff = off;                 // 128 (eff, 1/eff) pairs, one per non-negative E4M3 scale code
    off += 128 * 8;
    L.bars = off;
    off += (2 * kQStages + 8) * 8;
    L.misc = off;
    off += 64;
    L.total = off;
    return L;
}

// 8 channels [8q, 8q+8) of a row as one 16-byte vector.
__device__ __forceinline__ uint4 ld_x8_swz(const uint8_t* xs, int row, int q) {
    uint32_t off = (uint32_t)row * 128u + ((((uint32_t)q) ^ ((uint32_t)row & 7u)) << 4);
    return *reinterpret_cast<const uint4*>(xs + off);
}

struct BoxPos {
    int bkt, bkh, bkw;
    int t0, h0, w0;
    int dt0, dh0, dw0;   // big cubes: position of the box's first token inside its cube
};

__device__ __forceinline__ BoxPos box_pos(const QuantParams& p, int b) {
    BoxPos B;
    if (p.big) {
        // box b = (token row (tt, hh), cube column kw, segment of up to 128 tokens)
        const int th = b / p.nbw, rem = b % p.nbw;
        const int kw = rem / p.nseg, seg = rem % p.nseg;
        const int tt = th / p.g.H, hh = th % p.g.H;
        B.bkt = tt / p.g.t;
        B.bkh = hh / p.g.h;
        B.bkw = kw;
        B.t0 = tt;
        B.h0 = hh;
        B.dt0 = tt - B.bkt * p.g.t;
        B.dh0 = hh - B.bkh * p.g.h;
        B.dw0 = 128 * seg;
        B.w0 = kw * p.g.w + B.dw0;
        return B;
    }
    B.dt0 = B.dh0 = B.dw0 = 0;
    B.bkw = b % p.nbw;
    int r = b / p.nbw;
    B.bkh = r % p.g.KH;
    B.bkt = r / p.g.KH;
    B.t0 = B.bkt * p.g.t;
    B.h0 = B.bkh * p.g.h;
    B.w0 = B.bkw * p.nw * p.g.w;
    return B;
}

// Row `row` of a box -> validity, cube-major row rho.
__device__ __forceinline__ bool box_row(const QuantParams& p, const BoxPos& B, int row, long long* rho) {
    const Geom& g = p.g;
    if (p.big) {
        const int kw = B.bkw, dw = B.dw0 + row;
        const int sh = imin(g.h, g.H - B.bkh * g.h), sw = imin(g.w, g.W - kw * g.w);
        if (row >= p.bw || dw >= sw) return false;
        *rho = cube_first_row(g, B.bkt, B.bkh, kw) + ((long long)B.dt0 * sh + B.dh0) * sw + dw;
        return true;
    }
    int nrow = p.bt * p.bh * p.bw;
    if (row >= nrow) return false;
    int dt = row / (p.bh * p.bw);
    int dh = (row / p.bw) % p.bh;
    int x = row % p.bw;
    int jj = x / g.w, dw = x % g.w;
    int kw = B.bkw * p.nw + jj;
    if (kw >= g.KW || B.t0 + dt >= g.T || B.h0 + dh >= g.H || B.w0 + x >= g.W) return false;
    int sh = imin(g.h, g.H - B.h0), sw = imin(g.w, g.W - kw * g.w);
    *rho = cube_first_row(g, B.bkt, B.bkh, kw) + ((long long)dt * sh + dh) * sw + dw;
    return true;
}

// The box's tokens as a cube-major row list.  Small cubes: the box's nv valid
// cube slots share kt, kh (so st, sh); only the last one can be cut by the
// lattice edge in w; cube j owns rows [j n, j n + n_j).  Big cubes: one cube,
// the box's R valid rows.
struct BoxRows {
    int nv, n, R;
    int st, sh, sw_last;
    long long k0;        // cube index of slot 0
    long long rho0;      // big cubes: cube-major row of box row 0
};

__device__ __forceinline__ BoxRows box_rows(const QuantParams& p, const BoxPos& B) {
    const Geom& g = p.g;
    BoxRows R;
    R.k0 = ((long long)B.bkt * g.KH + B.bkh) * g.KW + (p.big ? B.bkw : B.bkw * p.nw);
    if (p.big) {
        const int sh = imin(g.h, g.H - B.bkh * g.h), sw = imin(g.w, g.W - B.bkw * g.w);
        R.nv = 1;
        R.R = imin(p.bw, sw - B.dw0);
        R.n = R.R;
        R.st = R.sh = 1;
        R.sw_last = R.R;
        R.rho0 = cube_first_row(g, B.bkt, B.bkh, B.bkw) + ((long long)B.dt0 * sh + B.dh0) * sw + B.dw0;
        return R;
    }
    R.nv = imin(p.nw, g.KW - B.bkw * p.nw);
    R.st = imin(g.t, g.T - B.t0);
    R.sh = imin(g.h, g.H - B.h0);
    R.sw_last = imin(g.w, g.W - (B.bkw * p.nw + R.nv - 1) * g.w);
    R.n = R.st * R.sh * g.w;
    R.R = (R.nv - 1) * R.n + R.st * R.sh * R.sw_last;
    R.rho0 = 0;
    return R;
}

__device__ __forceinline__ int cube_of_row(const BoxRows& R, int r) { return imin(r / R.n, R.nv - 1); }

// Row r of the list -> box row (shared-memory row of the TMA box) and cube-major row.
__device__ __forceinline__ void list_row(const QuantParams& p, const BoxPos& B, const BoxRows& R, int r, int* row,
                                         long long* rho) {
    if (p.big) {
        *row = r;
        *rho = R.rho0 + r;
        return;
    }
    const int j = cube_of_row(R, r), i = r - j * R.n;
    const int sw = (j == R.nv - 1) ? R.sw_last : p.g.w;
    const int dw = i % sw, q = i / sw;
    const int dh = q % R.sh, dt = q / R.sh;
    *row = (dt * p.bh + dh) * p.bw + j * p.g.w + dw;
    // cube-major rows of one cube are its tokens in (t,h,w) order
    *rho = cube_first_row(p.g, B.bkt, B.bkh, B.bkw * p.nw + j) + i;
}

// Eight fp32 values as four packed pairs (16-byte aligned).
__device__ __forceinline__ void load8(const float* src, uint64_t (&m)[4]) {
    const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(src);
    const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(src + 4);
    m[0] = a.x; m[1] = a.y; m[2] = b.x; m[3] = b.y;
}

// max |x - m| over 8 channels: x as four BF16 words, m as four fp32 pairs
__device__ __forceinline__ float max_abs_diff8(const uint4 x, const uint64_t (&m)[4]) {
    float d[8];
    f2_unpack(f2_sub(f2_from_bf16x2(x.x), m[0]), d[0], d[1]);
    f2_unpack(f2_sub(f2_from_bf16x2(x.y), m[1]), d[2], d[3]);
    f2_unpack(f2_sub(f2_from_bf16x2(x.z), m[2]), d[4], d[5]);
    f2_unpack(f2_sub(f2_from_bf16x2(x.w), m[3]), d[6], d[7]);
    return fmaxf(max3_abs(d[0], d[1], d[2]), fmaxf(max3_abs(d[3], d[4], d[5]), max3_abs(d[6], d[7], 0.f)));
}

// This warp's rows [r_lo, r_hi) of the list and the cube slots they touch.
struct WarpRows {
    int r_lo, r_hi, j_lo, ncub;
};

__device__ __forceinline__ WarpRows warp_rows(const BoxRows& R, int warp) {
    WarpRows W;
    W.r_lo = 16 * warp;
    W.r_hi = imin(W.r_lo + 16, R.R);
    if (W.r_lo >= W.r_hi) {
        W.j_lo = 0;
        W.ncub = 0;
        return W;
    }
    W.j_lo = cube_of_row(R, W.r_lo);
    W.ncub = cube_of_row(R, W.r_hi - 1) - W.j_lo + 1;
    return W;
}

// The smallest power of two >= v (v > 0) and its exponent: v = m 2^e with m in [0.5, 1).
__device__ __forceinline__ float pow2_ceil(float v, int* exp2) {
    int e;
    const float m = frexpf(v, &e);
    *exp2 = (m == 0.5f) ? e - 1 : e;
    return (m == 0.5f) ? v : ldexpf(1.0f, e);
}

__device__ __forceinline__ void mean_from_sum(const uint64_t (&acc)[4], int cnt, uint64_t (&m)[4]) {
    if ((cnt & (cnt - 1)) == 0) {
        const float inv = inv_pow2(cnt);
        const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
        for (int e = 0; e < 4; e++) m[e] = f2_mul(acc[e], inv2);
    } else {
#pragma unroll
        for (int e = 0; e < 4; e++) {
            float a, b;
            f2_unpack(acc[e], a, b);
            m[e] = f2_pack(__fdiv_rn(a, (float)cnt), __fdiv_rn(b, (float)cnt));
        }
    }
}

// Element-wise max / min of two BF16 pairs (exact: no rounding involved).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Statistics task of a1: unit u (cube slot, or token row for big cubes) x
// channel group g8 of the box, with the shared-memory offsets of the unit's
// tokens when it has at most 8 (fixed for all chunks of the item).
struct StatTask {
    bool valid;
    int u, g8, ntok;
    uint32_t off[8];
};

__device__ __forceinline__ StatTask stat_task(const QuantParams& p, const BoxRows& R, int q) {
    StatTask T;
    T.u = q >> 3;
    T.g8 = q & 7;
    T.valid = T.u < (p.big ? R.R : R.nv);
    T.ntok = 0;
    if (!T.valid) return T;
    if (p.big) {
        T.ntok = 1;
        const uint32_t row = (uint32_t)T.u;
        T.off[0] = row * 128u + ((((uint32_t)T.g8) ^ (row & 7u)) << 4);
        return T;
    }
    const int sw = (T.u == R.nv - 1) ? R.sw_last : p.g.w;
    T.ntok = R.st * R.sh * sw;
    int dt = 0, dh = 0, dw = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t row = (uint32_t)((dt * p.bh + dh) * p.bw + T.u * p.g.w + dw);
        T.off[i] = row * 128u + ((((uint32_t)T.g8) ^ (row & 7u)) << 4);
        if (i + 1 < T.ntok && ++dw == sw) {
            dw = 0;
            if (++dh == R.sh) {
                dh = 0;
                ++dt;
            }
        }
    }
    return T;
}

// One token of a statistics task: running fp32 sum (pairs) and element-wise BF16 max / min.
__device__ __forceinline__ void stat_token(const uint4 v, uint64_t (&acc)[4], uint32_t (&hi)[4], uint32_t (&lo)[4]) {
    acc[0] = f2_add(acc[0], f2_from_bf16x2(v.x));
    acc[1] = f2_add(acc[1], f2_from_bf16x2(v.y));
    acc[2] = f2_add(acc[2], f2_from_bf16x2(v.z));
    acc[3] = f2_add(acc[3], f2_from_bf16x2(v.w));
    hi[0] = bf16x2_max(hi[0], v.x); lo[0] = bf16x2_min(lo[0], v.x);
    hi[1] = bf16x2_max(hi[1], v.y); lo[1] = bf16x2_min(lo[1], v.y);
    hi[2] = bf16x2_max(hi[2], v.z); lo[2] = bf16x2_min(lo[2], v.z);
    hi[3] = bf16x2_max(hi[3], v.w); lo[3] = bf16x2_min(lo[3], v.w);
}

template <int N>
__device__ __forceinline__ void stat_tokens(const uint8_t* xs, const uint32_t (&off)[8], uint64_t (&acc)[4],
                                            uint32_t (&hi)[4], uint32_t (&lo)[4]) {
#pragma unroll
    for (int i = 1; i < N; i++) stat_token(*reinterpret_cast<const uint4*>(xs + off[i]), acc, hi, lo);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// 32 channels of one delta row (Eq. 1 delta, Eq. 4 per 16-channel group): z = x - m in fp32 from
// four 16-byte X pieces of the box in shared memory (swizzled offsets xoff) and the 32 fp32 means at
// mrow; per group the E4M3 scale code s_b = E4M3(max|z| / (6 S)) (denom = 6 S, rdenom = fl(1/denom)),
// eff = s_b S from the table efft of (eff, 1/eff) per code, and the E2M1 codes of z / eff (+0 where
// eff = 0).  kPow2: efft holds the codes' values at S = 1 and S = sc, a power of two with
// reciprocal rsc, scales them exactly.  codes: 16 bytes, channel 2i in the low nibble of byte i;
// scw: the two scale codes, the first group's in the low byte.
template <bool kPow2>
__device__ __forceinline__ void encode_delta32(const uint8_t* xs, const uint32_t (&xoff)[4], const float* mrow,
                                               float denom, float rdenom, const float2* efft, float sc, float rsc,
                                               uint32_t (&codes)[4], uint32_t& scw) {
    scw = 0;
#pragma unroll
    for (int b = 0; b < 2; b++) {
        uint64_t z[8];
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xs + xoff[2 * b + hh]);
            uint64_t m[4];
            load8(mrow + 16 * b + 8 * hh, m);
            z[4 * hh + 0] = f2_sub(f2_from_bf16x2(xv.x), m[0]);
            z[4 * hh + 1] = f2_sub(f2_from_bf16x2(xv.y), m[1]);
            z[4 * hh + 2] = f2_sub(f2_from_bf16x2(xv.z), m[2]);
            z[4 * hh + 3] = f2_sub(f2_from_bf16x2(xv.w), m[3]);
        }
        float zf[16];
#pragma unroll
        for (int e = 0; e < 8; e++) f2_unpack(z[e], zf[2 * e], zf[2 * e + 1]);
        const float am = fmaxf(fmaxf(max3_abs(zf[0], zf[1], zf[2]), max3_abs(zf[3], zf[4], zf[5])),
                               fmaxf(fmaxf(max3_abs(zf[6], zf[7], zf[8]), max3_abs(zf[9], zf[10], zf[11])),
                                     fmaxf(max3_abs(zf[12], zf[13], zf[14]), fabsf(zf[15]))));
        // am >= 0, so the code is one of 0x00..0x7E
        const uint32_t sb = cvt_e4m3x2(div_pos(am, denom, rdenom), 0.f) & 0x7Fu;
        const float2 er = efft[sb];
        const float eff = kPow2 ? __fmul_rn(er.x, sc) : er.x;
        scw |= sb << (8 * b);
        uint32_t w0 = 0, w1 = 0;
        if (eff != 0.f) {
            // codes of the negated quotients, then every nibble's sign bit flipped
            // (E2M1 is sign-magnitude: code(-v) = code(v) ^ 8, signed zeros included)
            const float reff = kPow2 ? __fmul_rn(er.y, rsc) : er.y;
            const uint64_t b2 = f2_pack(eff, eff), nrb2 = f2_pack(-reff, -reff);
            float n[16];
#pragma unroll
            for (int e = 0; e < 8; e++) f2_unpack(f2_div_neg(z[e], b2, nrb2), n[2 * e], n[2 * e + 1]);
            w0 = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(&n[0])) ^ 0x88888888u;
            w1 = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(&n[8])) ^ 0x88888888u;
        }
        codes[2 * b] = w0;
        codes[2 * b + 1] = w1;
    }
}

}  // namespace

// ------------------------------------------------------------------ a1: statistics + X L1
//
// Warps 0-7 compute, warp 8 loads, warp 9 owns tensor memory and issues the
// X L1 MMAs (M = 128 box rows, N = rank, K = 64 per chunk) into one of two
// tensor-memory accumulators per item, which the compute warps drain to the
// item's partial sums after its last chunk.

//
// kSingle (the single-read quantiser, power-of-two S_delta): each chunk's means also go to shared
// memory, the compute warps exchange the chunk's max |delta| (a bounded mbarrier per chunk), and
// then encode the chunk's delta rows as the encode kernel would, under the chunk's own power-of-two
// scale S_c = pow2(max|delta of the chunk| / 2688) <= S_delta; the exponent of S_c goes to p.prov
// for the fix-up pass (k_single_finish), which also encodes the kernel tokens.

template <bool kPairs, bool kSingle>
__global__ void __launch_bounds__(kQCompute + 64, 2) k_cube_stats(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_l1,
                                                                  QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QSmem L = q_smem_layout(p.rank, true, kSingle ? p.m_rows : 0, 128, kSingle);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kQStages;
    uint64_t* accf = empty + kQStages;   // [2]
    uint64_t* acce = accf + 2;           // [2]
    uint64_t* done = acce + 2;
    uint64_t* sdone = done + 1;          // [2], kSingle: a chunk's statistics are in shared memory
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);
    float* red = (float*)(sm + L.misc + 16);  // 8 floats

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nchunks = p.chunks_per_split;
    const uint32_t l1_bytes = (uint32_t)p.rank * 128u;
    const uint32_t l1_stride = (uint32_t)align_up(l1_bytes, 1024);
    const uint32_t x_bytes = (uint32_t)p.bt * p.bh * p.bw * 128u;
    uint32_t tcols = 32;
    while (tcols < (uint32_t)p.rank) tcols <<= 1;

    if (tid == 0) {
        for (int s = 0; s < kQStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQWarps + 1);   // the compute warps + the MMA commit
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], kQWarps);
        }
        mbar_init(done, 1);
        mbar_init(&sdone[0], kQWarps);
        mbar_init(&sdone[1], kQWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    float2* efft = (float2*)(sm + L.eff);
    if (kSingle && tid < 128) {
        // E4M3 code -> (value, 1 / value) at S = 1; a chunk's power-of-two scale multiplies both exactly
        const float e = e4m3_to_f32((uint32_t)tid);
        efft[tid] = make_float2(e, (e != 0.f) ? __frcp_rn(e) : 0.f);
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 2 * tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ---------------- producer: all chunks of all this CTA's items through one ring
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_l1);
            long long g = 0;
            bool alive = true;
            for (int it = p.item0 + blockIdx.x; alive && it < p.item1; it += gridDim.x) {
                const BoxPos B = box_pos(p, it / p.splits);
                const int c_base = (it % p.splits) * nchunks * 64;
                for (int i = 0; i < nchunks; i++, g++) {
                    const int s = (int)(g % kQStages);
                    if (g >= kQStages &&
                        !mbar_wait(&empty[s], (uint32_t)((g / kQStages) - 1) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], x_bytes + l1_bytes);
                    const int c0 = c_base + i * 64;
                    tma_load_4d(sm + L.x + s * 16384, &tm_x, &full[s], c0, B.w0, B.h0, B.t0);
                    tma_load_2d(sm + L.l1 + s * l1_stride, &tm_l1, &full[s], c0, 0);
                }
            }
            // drain: every issued load lands before shared memory is released
            for (long long q = (g > kQStages ? g - kQStages : 0); q < g; q++)
                mbar_wait(&full[q % kQStages], (uint32_t)(q / kQStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 9) {
        // ---------------- MMA issuer: U_item = sum over its chunks of X_chunk L1_chunk^T
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, p.rank);
            long long g = 0;
            int n = 0;
            bool alive = true;
            for (int it = p.item0 + blockIdx.x; alive && it < p.item1; it += gridDim.x, n++) {
                const int buf = n & 1, use = n >> 1;
                const uint32_t acc = tmem + (uint32_t)buf * tcols;
                if (use > 0 && !mbar_wait(&acce[buf], (uint32_t)(use - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                tc_fence_after();
                for (int i = 0; i < nchunks; i++, g++) {
                    const int s = (int)(g % kQStages);
                    if (!mbar_wait(&full[s], (uint32_t)(g / kQStages) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xa = smem_u32(sm + L.x + s * 16384), la = smem_u32(sm + L.l1 + s * l1_stride);
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        mma_bf16(acc, desc_k_sw128(xa + 32 * k), desc_k_sw128(la + 32 * k), idesc, (i | k) != 0);
                    tc_commit(&empty[s]);
                }
                if (alive) tc_commit(&accf[buf]);
            }
            tc_commit(done);
            // every MMA has retired before tensor memory is released
            mbar_wait(done, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // ---------------- compute warps 0-7: thread = statistics task (unit x 8 channels).
        // The largest |token - mean| of a cube and channel is |x_max - mean| or |x_min - mean|
        // (fl(x - m) is monotone in x), so a cube's tokens are visited once: fp32 sum for the
        // mean, BF16 max and min for the delta bound.
        const int ntask = (int)cdiv((long long)(p.big ? p.bw : p.nw) * 8, kQCompute);
        float damax = 0.f;
        long long g = 0;
        int n = 0;
        bool ok = true;
        for (int it = p.item0 + blockIdx.x; ok && it < p.item1; it += gridDim.x, n++) {
            const BoxPos B = box_pos(p, it / p.splits);
            const int split = it % p.splits;
            const int c_base = split * nchunks * 64;
            const BoxRows R = box_rows(p, B);
            const StatTask T0 = stat_task(p, R, tid);
            float kam[4] = {0.f, 0.f, 0.f, 0.f};   // max |mean| of this thread's cube tasks
            // kSingle: the delta rows this warp encodes, as in the encode kernel (16 consecutive rows
            // of the box's cube-major list, two lanes per row, 32 channels each)
            const WarpRows W = warp_rows(R, warp);
            const int er = W.r_lo + (lane >> 1), ehalf = lane & 1;
            const bool has_row = kSingle && er < W.r_hi;
            int erow = 0;
            long long erho = 0;
            if (has_row) list_row(p, B, R, er, &erow, &erho);
            uint32_t xoff[4];
#pragma unroll
            for (int v = 0; v < 4; v++)
                xoff[v] = (uint32_t)erow * 128u + ((((uint32_t)(4 * ehalf + v)) ^ ((uint32_t)erow & 7u)) << 4);
            const uint32_t moff = (uint32_t)(has_row ? cube_of_row(R, er) : 0) * 256u + 128u * ehalf;
            // channel-pair mode: with fewer cubes than warps, the warps form kQWarps / nv groups
            // that take turns over the chunks, so that several stages of the ring are worked on at once
            const int ngrp = kPairs ? kQWarps / R.nv : 1;
            const int grp = kPairs ? warp / R.nv : 0, u_pair = kPairs ? warp - grp * R.nv : 0;
            int phase = 0;
            for (int i = 0; i < nchunks; i++, g++) {
                const int s = (int)(g % kQStages);
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(g / kQStages) & 1, abort_flag, p.status,
                                                       p.budget_ns));
                if (!ok) break;
                const uint8_t* xs = sm + L.x + s * 16384;
                const int c0 = c_base + i * 64;
                const int par = (int)(g & 1);
                float* mts = (float*)(sm + L.ms + (uint32_t)par * L.ms_stride);   // kSingle: this chunk's means
                float dch = 0.f;                                                 // this chunk's max |delta|
                if (kPairs) {
                    // cubes of 16 or more tokens (at most 8 per box): warp = cube slot, lane = channel
                    // pair (2 lane, 2 lane + 1)
                    const bool mine = grp < ngrp && phase == grp;
                    if (++phase == ngrp) phase = 0;
                    if (mine) {
                        const int u = u_pair;
                        const int sw = (u == R.nv - 1) ? R.sw_last : p.g.w;
                        uint64_t acc = 0ull;                          // (+0, +0)
                        uint32_t hi = 0xFF80FF80u, lo = 0x7F807F80u;  // BF16 -inf / +inf pairs
                        for (int dt = 0; dt < R.st; dt++)
                            for (int dh = 0; dh < R.sh; dh++) {
                                const int row0 = (dt * p.bh + dh) * p.bw + u * p.g.w;
                                for (int dw = 0; dw < sw; dw++) {
                                    const uint32_t row = (uint32_t)(row0 + dw);
                                    const uint32_t v = *reinterpret_cast<const uint32_t*>(
                                        xs + row * 128u + ((((uint32_t)lane >> 2) ^ (row & 7u)) << 4) + ((uint32_t)lane & 3u) * 4u);
                                    acc = f2_add(acc, f2_from_bf16x2(v));
                                    hi = bf16x2_max(hi, v);
                                    lo = bf16x2_min(lo, v);
                                }
                            }
                        const int cnt = R.st * R.sh * sw;
                        float a0, a1, m0, m1;
                        f2_unpack(acc, a0, a1);
                        if ((cnt & (cnt - 1)) == 0) {
                            const float inv = inv_pow2(cnt);
                            m0 = __fmul_rn(a0, inv);
                            m1 = __fmul_rn(a1, inv);
                        } else {
                            m0 = __fdiv_rn(a0, (float)cnt);
                            m1 = __fdiv_rn(a1, (float)cnt);
                        }
                        *reinterpret_cast<float2*>(p.means + (size_t)(R.k0 + u) * p.Ci + c0 + 2 * lane) = make_float2(m0, m1);
                        if (kSingle) *reinterpret_cast<float2*>(mts + u * 64 + 2 * lane) = make_float2(m0, m1);
                        kam[0] = fmaxf(kam[0], fmaxf(fabsf(m0), fabsf(m1)));
                        dch = fmaxf(dch, fmaxf(fmaxf(fabsf(__fsub_rn(bf16_lo(hi), m0)), fabsf(__fsub_rn(bf16_hi(hi), m1))),
                                               fmaxf(fabsf(__fsub_rn(bf16_lo(lo), m0)), fabsf(__fsub_rn(bf16_hi(lo), m1)))));
                    }
                }
#pragma unroll
                for (int t = 0; t < 4; t++) {
                    if (kPairs || t >= ntask) break;
                    const StatTask T = t == 0 ? T0 : stat_task(p, R, tid + kQCompute * t);
                    if (!T.valid) continue;
                    uint64_t m[4];
                    if (p.big) {
                        load8(p.means + (size_t)R.k0 * p.Ci + c0 + 8 * T.g8, m);
                        dch = fmaxf(dch, max_abs_diff8(*reinterpret_cast<const uint4*>(xs + T.off[0]), m));
                        continue;
                    }
                    // fp32 running sum from +0 in (t,h,w) order (Eq. 1; +0 + x keeps the sign of
                    // an all-zero sum as the sequential definition has it)
                    uint64_t acc[4];
                    uint32_t hi[4], lo[4];
                    if (T.ntok <= 8) {
                        const uint4 v0 = *reinterpret_cast<const uint4*>(xs + T.off[0]);
                        acc[0] = f2_add(0ull, f2_from_bf16x2(v0.x));
                        acc[1] = f2_add(0ull, f2_from_bf16x2(v0.y));
                        acc[2] = f2_add(0ull, f2_from_bf16x2(v0.z));
                        acc[3] = f2_add(0ull, f2_from_bf16x2(v0.w));
                        hi[0] = lo[0] = v0.x; hi[1] = lo[1] = v0.y; hi[2] = lo[2] = v0.z; hi[3] = lo[3] = v0.w;
                        switch (T.ntok) {
                            case 1: break;
                            case 2: stat_tokens<2>(xs, T.off, acc, hi, lo); break;
                            case 4: stat_tokens<4>(xs, T.off, acc, hi, lo); break;
                            case 8: stat_tokens<8>(xs, T.off, acc, hi, lo); break;
                            default:
#pragma unroll
                                for (int k = 1; k < 8; k++) {
                                    if (k >= T.ntok) break;
                                    stat_token(*reinterpret_cast<const uint4*>(xs + T.off[k]), acc, hi, lo);
                                }
                        }
                    } else {
                        // larger cubes: walk the tokens in (t,h,w) order
                        const int sw = (T.u == R.nv - 1) ? R.sw_last : p.g.w;
                        bool first = true;
                        for (int dt = 0; dt < R.st; dt++)
                            for (int dh = 0; dh < R.sh; dh++) {
                                const int row0 = (dt * p.bh + dh) * p.bw + T.u * p.g.w;
                                for (int dw = 0; dw < sw; dw++) {
                                    const uint4 v = ld_x8_swz(xs, row0 + dw, T.g8);
                                    if (first) {
                                        acc[0] = f2_add(0ull, f2_from_bf16x2(v.x));
                                        acc[1] = f2_add(0ull, f2_from_bf16x2(v.y));
                                        acc[2] = f2_add(0ull, f2_from_bf16x2(v.z));
                                        acc[3] = f2_add(0ull, f2_from_bf16x2(v.w));
                                        hi[0] = lo[0] = v.x; hi[1] = lo[1] = v.y; hi[2] = lo[2] = v.z; hi[3] = lo[3] = v.w;
                                        first = false;
                                    } else {
                                        stat_token(v, acc, hi, lo);
                                    }
                                }
                            }
                    }
                    mean_from_sum(acc, T.ntok, m);
                    {
                        const uint32_t mw[8] = {(uint32_t)m[0], (uint32_t)(m[0] >> 32), (uint32_t)m[1],
                                                (uint32_t)(m[1] >> 32), (uint32_t)m[2], (uint32_t)(m[2] >> 32),
                                                (uint32_t)m[3], (uint32_t)(m[3] >> 32)};
                        st_global_v8(p.means + (size_t)(R.k0 + T.u) * p.Ci + c0 + 8 * T.g8, mw);
                        if (kSingle) {
                            float4* md = reinterpret_cast<float4*>(mts + T.u * 64 + 8 * T.g8);
                            md[0] = make_float4(__uint_as_float(mw[0]), __uint_as_float(mw[1]), __uint_as_float(mw[2]),
                                                __uint_as_float(mw[3]));
                            md[1] = make_float4(__uint_as_float(mw[4]), __uint_as_float(mw[5]), __uint_as_float(mw[6]),
                                                __uint_as_float(mw[7]));
                        }
                    }
                    float mf[8];
#pragma unroll
                    for (int e = 0; e < 4; e++) f2_unpack(m[e], mf[2 * e], mf[2 * e + 1]);
                    kam[t] = fmaxf(kam[t], fmaxf(max3_abs(mf[0], mf[1], mf[2]),
                                                 fmaxf(max3_abs(mf[3], mf[4], mf[5]), max3_abs(mf[6], mf[7], 0.f))));
                    dch = fmaxf(dch, fmaxf(max_abs_diff8(make_uint4(hi[0], hi[1], hi[2], hi[3]), m),
                                           max_abs_diff8(make_uint4(lo[0], lo[1], lo[2], lo[3]), m)));
                }
                damax = fmaxf(damax, dch);
                if (kSingle) {
                    // big cubes: the chunk's means, formed by the means kernel, into shared memory
                    if (p.big && tid < 16)
                        reinterpret_cast<float4*>(mts)[tid] =
                            *reinterpret_cast<const float4*>(p.means + (size_t)R.k0 * p.Ci + c0 + 4 * tid);
                    // the chunk's max |delta| over all compute warps, then its power-of-two scale
                    const float wmx = warp_max(dch);
                    float* red = (float*)(sm + L.red2) + par * kQWarps;
                    __syncwarp();
                    if (lane == 0) {
                        red[warp] = wmx;
                        mbar_arrive(&sdone[par]);
                    }
                    ok = __all_sync(0xffffffffu, mbar_wait(&sdone[par], (uint32_t)(g >> 1) & 1, abort_flag, p.status,
                                                           p.budget_ns));
                    if (!ok) break;
                    float amc = 0.f;
#pragma unroll
                    for (int w = 0; w < kQWarps; w++) amc = fmaxf(amc, red[w]);
                    int ec = -128;   // an all-zero chunk: its codes and scales are 0 under any scale
                    float Sc = 1.f;
                    if (amc > 0.f) Sc = pow2_ceil(__fdiv_rn(amc, 2688.f), &ec);
                    const float den = __fmul_rn(6.f, Sc), rden = __frcp_rn(den), rSc = __frcp_rn(Sc);
                    if (has_row) {
                        uint32_t codes[4], scw;
                        encode_delta32<true>(xs, xoff, (const float*)((const uint8_t*)mts + moff), den, rden, efft,
                                             Sc, rSc, codes, scw);
                        *reinterpret_cast<uint4*>(p.dcodes + (size_t)erho * (p.Ci / 2) + 16 * ehalf + c0 / 2) =
                            make_uint4(codes[0], codes[1], codes[2], codes[3]);
                        *reinterpret_cast<uint16_t*>(p.dscales + sfa_offset(erho, c0 / 16 + 2 * ehalf, p.Ci)) =
                            (uint16_t)scw;
                        if (ehalf == 0) p.prov[(size_t)erho * (p.Ci / 64) + c0 / 64] = (int8_t)ec;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            // per-cube max |mean| over this item's channels -> kamax (small cubes; the means
            // kernel has done it for big ones); the eight threads of a cube are consecutive lanes,
            // or a whole warp in the channel-pair mode
            if (kPairs) {
                const float v = warp_max(kam[0]);
                if (lane == 0 && grp < ngrp) atomicMax(&p.kamax[R.k0 + u_pair], __float_as_uint(v));
            } else if (!p.big) {
#pragma unroll
                for (int t = 0; t < 4; t++) {
                    if (t >= ntask) break;
                    const int q = tid + kQCompute * t;
                    if ((q >> 3) < R.nv) {
                        const uint32_t gm = 0xFFu << (lane & 24);
                        float v = kam[t];
                        v = fmaxf(v, __shfl_xor_sync(gm, v, 1));
                        v = fmaxf(v, __shfl_xor_sync(gm, v, 2));
                        v = fmaxf(v, __shfl_xor_sync(gm, v, 4));
                        if ((q & 7) == 0) atomicMax(&p.kamax[R.k0 + (q >> 3)], __float_as_uint(v));
                    }
                }
            }
            // U partial rows of this item out of tensor memory (sub-partition warp % 4, column half warp / 4)
            const int buf = n & 1, use = n >> 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], (uint32_t)use & 1, abort_flag, p.status, p.budget_ns));
            if (!ok) break;
            tc_fence_after();
            const int urow_i = (warp & 3) * 32 + lane, uhalf = warp >> 2;
            long long urho = 0;
            const bool urow_ok = box_row(p, B, urow_i, &urho);
            float* urow = p.u_part + ((size_t)split * p.g.N + (size_t)urho) * p.rank;
            for (int c = 16 * uhalf; c < p.rank; c += 32) {
                uint32_t rr[16];
                tmem_ld_x16(tmem + (uint32_t)buf * tcols + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c, rr);
                tmem_ld_wait();
                if (urow_ok) {
#pragma unroll
                    for (int v = 0; v < 16; v += 4)
                        *reinterpret_cast<float4*>(urow + c + v) =
                            make_float4(__uint_as_float(rr[v]), __uint_as_float(rr[v + 1]), __uint_as_float(rr[v + 2]),
                                        __uint_as_float(rr[v + 3]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[buf]);
        }
        float wm = warp_max(damax);
        if (lane == 0) red[warp] = wm;
        bar_sync(1, kQCompute);
        if (tid == 0) {
            float bm = 0.f;
            for (int w = 0; w < kQWarps; w++) bm = fmaxf(bm, red[w]);
            atomicMax(&p.scalars[0], __float_as_uint(bm));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * tcols);
    }
}

// ------------------------------------------------------------------ a2: encode
//
// Warps 0-7 compute, warp 8 loads.

template <bool kLR>
__global__ void __launch_bounds__(kQCompute + (kLR ? 64 : 32), 2)
    k_cube_encode(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_m,
                  const __grid_constant__ CUtensorMap tm_l1, QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QSmem L = q_smem_layout(p.rank, kLR, p.m_rows, p.bt * p.bh * p.bw);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kQStages;
    uint64_t* accf = empty + kQStages;   // [2], kLR
    uint64_t* acce = accf + 2;           // [2], kLR
    uint64_t* done = acce + 2;           // kLR
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nchunks = p.chunks_per_split;
    const int n_items = p.n_boxes * p.splits;
    const uint32_t x_bytes = (uint32_t)p.bt * p.bh * p.bw * 128u;
    const uint32_t m_bytes = (uint32_t)p.m_rows * 256u;   // the box's kernel tokens for 64 channels
    const uint32_t l1_bytes = kLR ? (uint32_t)p.rank * 128u : 0u;
    const uint32_t l1_stride = (uint32_t)align_up(l1_bytes, 1024);
    uint32_t tcols = 32;
    while (tcols < (uint32_t)p.rank) tcols <<= 1;
    const int Ci = p.Ci;

    const PackedHeader* hdr = reinterpret_cast<const PackedHeader*>(p.packed_w);
    if (tid == 0) {
        for (int s = 0; s < kQStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQWarps + (kLR ? 1 : 0));   // the compute warps (+ the MMA commit)
        }
        if (kLR) {
            for (int b = 0; b < 2; b++) {
                mbar_init(&accf[b], 1);
                mbar_init(&acce[b], kQWarps);
            }
            mbar_init(done, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        if (blockIdx.x == 0 &&
            (hdr->magic != DQ_PACK_MAGIC || hdr->version != DQ_PACK_FORMAT_VERSION || hdr->Ci != p.Ci ||
             hdr->rank != p.rank || hdr->slab != p.slab || ((hdr->flags & kPackedC2) != 0) != (p.fp8_product != 0)))
            atomicCAS(p.status, 0, kStatusBadWeight);
    }
    // per-tensor delta scale S = amax / (6*448) (1 if amax = 0); S_W from the packed weight
    const float damax = __uint_as_float(p.scalars[0]);
    const float S = (damax == 0.f) ? 1.f : __fdiv_rn(damax, 2688.f);
    const float denom = __fmul_rn(6.f, S);
    const float rdenom = __frcp_rn(denom);
    if (blockIdx.x == 0 && tid == 0) p.scalars[1] = __float_as_uint(S);
    // group scale s_b (E4M3 code c) -> effective scale eff = fl(s_b S) and fl(1 / eff), for every
    // code a group's amax can produce (non-negative, finite)
    float2* efft = (float2*)(sm + L.eff);
    if (tid < 128) {
        const float e = __fmul_rn(e4m3_to_f32((uint32_t)tid), S);
        efft[tid] = make_float2(e, (e != 0.f) ? __frcp_rn(e) : 0.f);
    }
    if (kLR && warp == 9) {
        tmem_alloc(tmem_slot, 2 * tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = kLR ? *tmem_slot : 0u;

    if (warp == 8) {
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_m);
            if (kLR) prefetch_tmap(&tm_l1);
            long long g = 0;
            bool alive = true;
            for (int it = blockIdx.x; alive && it < n_items; it += gridDim.x) {
                const BoxPos B = box_pos(p, it / p.splits);
                const int k0 = (int)box_rows(p, B).k0;
                const int c_base = (it % p.splits) * nchunks * 64;
                for (int i = 0; i < nchunks; i++, g++) {
                    const int s = (int)(g % kQStages);
                    if (g >= kQStages &&
                        !mbar_wait(&empty[s], (uint32_t)((g / kQStages) - 1) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], x_bytes + m_bytes + l1_bytes);
                    tma_load_4d(sm + L.x + s * L.x_stride, &tm_x, &full[s], c_base + i * 64, B.w0, B.h0, B.t0);
                    tma_load_2d(sm + L.mt + s * L.mt_stride, &tm_m, &full[s], c_base + i * 64, k0);
                    if (kLR) tma_load_2d(sm + L.l1 + s * l1_stride, &tm_l1, &full[s], c_base + i * 64, 0);
                }
            }
            for (long long q = (g > kQStages ? g - kQStages : 0); q < g; q++)
                mbar_wait(&full[q % kQStages], (uint32_t)(q / kQStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 9) {
        // ---------------- kLR: X L1 on the tensor cores, the statistics kernel's MMAs in its order
        if (kLR && lane == 0) {
            const uint32_t idesc = idesc_bf16(128, p.rank);
            long long g = 0;
            int n = 0;
            bool alive = true;
            for (int it = blockIdx.x; alive && it < n_items; it += gridDim.x, n++) {
                const int buf = n & 1, use = n >> 1;
                const uint32_t acc = tmem + (uint32_t)buf * tcols;
                if (use > 0 && !mbar_wait(&acce[buf], (uint32_t)(use - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                tc_fence_after();
                for (int i = 0; i < nchunks; i++, g++) {
                    const int s = (int)(g % kQStages);
                    if (!mbar_wait(&full[s], (uint32_t)(g / kQStages) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xa = smem_u32(sm + L.x + s * L.x_stride), la = smem_u32(sm + L.l1 + s * l1_stride);
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        mma_bf16(acc, desc_k_sw128(xa + 32 * k), desc_k_sw128(la + 32 * k), idesc, (i | k) != 0);
                    tc_commit(&empty[s]);
                }
                if (alive) tc_commit(&accf[buf]);
            }
            tc_commit(done);
            // every MMA has retired before tensor memory is released
            mbar_wait(done, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        const float SS = __fmul_rn(S, hdr->S_W);
        long long g = 0;
        int n_it = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, n_it++) {
            const BoxPos B = box_pos(p, it / p.splits);
            const int split = it % p.splits;
            const int c_base = split * nchunks * 64;
            const BoxRows R = box_rows(p, B);
            const WarpRows W = warp_rows(R, warp);
            const int r = W.r_lo + (lane >> 1), half = lane & 1;
            const bool has_row = r < W.r_hi;
            int row = 0;
            long long rho = 0;
            if (has_row) list_row(p, B, R, r, &row, &rho);
            // the row's kernel tokens in the stage's tile (row = cube slot of the box, 64 fp32)
            const uint32_t moff = (uint32_t)(has_row ? cube_of_row(R, r) : 0) * 256u + 128u * half;
            uint32_t xoff[4];
#pragma unroll
            for (int v = 0; v < 4; v++) xoff[v] = (uint32_t)row * 128u + ((((uint32_t)(4 * half + v)) ^ ((uint32_t)row & 7u)) << 4);
            uint8_t* dcode_row = p.dcodes + (size_t)rho * (Ci / 2) + 16 * half;
            // the kernel tokens of a cube are encoded by the warp that holds the cube's
            // first row (big cubes: by warp 0 of the cube's first box)
            const int j_own = p.big ? ((B.dt0 == 0 && B.dh0 == 0 && B.dw0 == 0 && warp == 0) ? 0 : 1)
                                    : (W.ncub > 0 && W.j_lo * R.n < W.r_lo ? 1 : 0);
            // s8 = max|mean| / 448 of the first kernel-token task of this lane (others, which only
            // very small cubes have, are formed where they are used)
            const int q_first = lane + 8 * j_own;
            float s8_first = 0.f, rs8_first = 0.f;
            if (!p.kgroup && q_first < W.ncub * 8) {
                const long long k = R.k0 + W.j_lo + (q_first >> 3);
                s8_first = __fdiv_rn(__uint_as_float(p.kamax[k]), 448.f);
                rs8_first = (s8_first != 0.f) ? __frcp_rn(s8_first) : 0.f;
                if (split == 0 && (q_first & 7) == 0) p.s8[k] = s8_first;
            }
            for (int i = 0; i < nchunks; i++, g++) {
                const int s = (int)(g % kQStages);
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(g / kQStages) & 1, abort_flag, p.status,
                                                       p.budget_ns));
                if (!ok) break;
                const uint8_t* xs = sm + L.x + s * L.x_stride;
                const float* mt = (const float*)(sm + L.mt + s * L.mt_stride);
                const int c0 = c_base + i * 64;
                // kernel tokens: FP8 E4M3 codes under s8 = max|mean| / 448 (over the token, or over
                // this stage's 64 channels), and their BF16 form for the kernel-token product
                for (int q = q_first; q < W.ncub * 8; q += 32) {
                    const int jj = q >> 3, g8 = q & 7;
                    const long long k = R.k0 + W.j_lo + jj;
                    uint64_t m[4];
                    load8(mt + (W.j_lo + jj) * 64 + 8 * g8, m);
                    float s8 = s8_first, rs8 = rs8_first;
                    if (p.kgroup) {
                        // the cube's 64 channels of this stage are held by eight consecutive lanes
                        float a = 0.f;
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            float lo, hi;
                            f2_unpack(m[e], lo, hi);
                            a = fmaxf(a, fmaxf(fabsf(lo), fabsf(hi)));
                        }
                        const uint32_t gm = 0xFFu << (lane & 24);
                        a = fmaxf(a, __shfl_xor_sync(gm, a, 1));
                        a = fmaxf(a, __shfl_xor_sync(gm, a, 2));
                        a = fmaxf(a, __shfl_xor_sync(gm, a, 4));
                        s8 = __fdiv_rn(a, 448.f);
                        rs8 = (s8 != 0.f) ? __frcp_rn(s8) : 0.f;
                        if (g8 == 0) p.s8[k * (Ci / 64) + (c0 >> 6)] = s8;
                    } else if (q != q_first) {
                        s8 = __fdiv_rn(__uint_as_float(p.kamax[k]), 448.f);
                        rs8 = (s8 != 0.f) ? __frcp_rn(s8) : 0.f;
                        if (split == 0 && i == 0 && g8 == 0) p.s8[k] = s8;
                    }
                    uint32_t c[4] = {0u, 0u, 0u, 0u};
                    if (s8 != 0.f) {
                        // codes of the negated quotients with the sign bit of each byte flipped
                        // (E4M3 is sign-magnitude, saturation symmetric)
                        const uint64_t b2 = f2_pack(s8, s8), nrb2 = f2_pack(-rs8, -rs8);
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            float lo, hi;
                            f2_unpack(f2_div_neg(m[e], b2, nrb2), lo, hi);
                            c[e] = cvt_e4m3x2(lo, hi) ^ 0x8080u;
                        }
                    }
                    *reinterpret_cast<uint2*>(p.q8 + (size_t)k * Ci + c0 + 8 * g8) =
                        make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
                    if (p.kgroup) {
                        // q8 s8 as BF16 hi + lo: hi in columns [0, Ci), lo in [Ci, 2 Ci) of row k
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const float v0 = __fmul_rn(e4m3_to_f32(c[e] & 0xFF), s8);
                            const float v1 = __fmul_rn(e4m3_to_f32(c[e] >> 8), s8);
                            const uint16_t h0 = f32_to_bf16_rn(v0), h1 = f32_to_bf16_rn(v1);
                            const uint16_t l0 = f32_to_bf16_rn(__fsub_rn(v0, __uint_as_float((uint32_t)h0 << 16)));
                            const uint16_t l1 = f32_to_bf16_rn(__fsub_rn(v1, __uint_as_float((uint32_t)h1 << 16)));
                            hw[e] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                            lw[e] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                        }
                        uint16_t* arow = p.q8_bf16 + (size_t)k * (2 * Ci) + c0 + 8 * g8;
                        *reinterpret_cast<uint4*>(arow) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        *reinterpret_cast<uint4*>(arow + Ci) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    } else if (!p.fp8_product) {
                        // exact: E4M3 values have four significant bits
                        uint32_t bfw[4];
#pragma unroll
                        for (int e = 0; e < 4; e++) bfw[e] = e4m3x2_to_bf16x2(c[e]);
                        *reinterpret_cast<uint4*>(p.q8_bf16 + (size_t)k * Ci + c0 + 8 * g8) =
                            make_uint4(bfw[0], bfw[1], bfw[2], bfw[3]);
                    }
                }
                // delta tokens: FP4 E2M1 with E4M3 group-16 scales under S (two groups per lane)
                if (has_row) {
                    const float* mrow = (const float*)((const uint8_t*)mt + moff);
                    uint32_t codes[4];
                    uint32_t sc = 0;
                    encode_delta32<false>(xs, xoff, mrow, denom, rdenom, efft, 1.f, 1.f, codes, sc);
                    *reinterpret_cast<uint4*>(dcode_row + c0 / 2) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                    *reinterpret_cast<uint16_t*>(p.dscales + sfa_offset(rho, c0 / 16 + 2 * half, Ci)) = (uint16_t)sc;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            if (kLR) {
                // this item's X L1 partial sums out of tensor memory (sub-partition warp % 4, column half
                // warp / 4), as the statistics kernel stores them; U' follows in k_u_hilo
                const int buf = n_it & 1, use = n_it >> 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], (uint32_t)use & 1, abort_flag, p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                const int urow_i = (warp & 3) * 32 + lane, uhalf = warp >> 2;
                long long urho = 0;
                const bool urow_ok = box_row(p, B, urow_i, &urho);
                float* urow = p.u_part + ((size_t)split * p.g.N + (size_t)urho) * p.rank;
                for (int c = 16 * uhalf; c < p.rank; c += 32) {
                    uint32_t rr[16];
                    tmem_ld_x16(tmem + (uint32_t)buf * tcols + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c, rr);
                    tmem_ld_wait();
                    if (urow_ok) {
#pragma unroll
                        for (int v = 0; v < 16; v += 4)
                            *reinterpret_cast<float4*>(urow + c + v) =
                                make_float4(__uint_as_float(rr[v]), __uint_as_float(rr[v + 1]), __uint_as_float(rr[v + 2]),
                                            __uint_as_float(rr[v + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[buf]);
                continue;
            }
            // U' = (X L1) / (S_delta S_W) as BF16 hi + lo for this item's slice of the rank columns
            // (thread = box row x column half), the slab's zero padding by split 0
            const int urow_i = tid & 127, uhalf = tid >> 7;
            long long urho = 0;
            if (box_row(p, B, urow_i, &urho)) {
                uint16_t* dst = p.u_hilo + (size_t)urho * p.slab;
                const int cps = 2 * (int)cdiv(p.rank, 2 * p.splits);
                const int c_lo = imin(split * cps, p.rank), c_hi = imin(c_lo + cps, p.rank);
                for (int c = c_lo + 2 * uhalf; c < c_hi; c += 4) {
                    float u0 = 0.f, u1 = 0.f;
                    for (int sp = 0; sp < p.splits; sp++) {
                        const float2 v = *reinterpret_cast<const float2*>(
                            p.u_part + ((size_t)sp * p.g.N + (size_t)urho) * p.rank + c);
                        u0 = __fadd_rn(u0, v.x);
                        u1 = __fadd_rn(u1, v.y);
                    }
                    float a0 = __fdiv_rn(u0, SS), a1 = __fdiv_rn(u1, SS);
                    uint16_t h0 = f32_to_bf16_rn(a0), h1 = f32_to_bf16_rn(a1);
                    uint16_t l0 = f32_to_bf16_rn(__fsub_rn(a0, __uint_as_float((uint32_t)h0 << 16)));
                    uint16_t l1 = f32_to_bf16_rn(__fsub_rn(a1, __uint_as_float((uint32_t)h1 << 16)));
                    *reinterpret_cast<uint32_t*>(dst + c) = (uint32_t)h0 | ((uint32_t)h1 << 16);
                    *reinterpret_cast<uint32_t*>(dst + p.rank + c) = (uint32_t)l0 | ((uint32_t)l1 << 16);
                }
                if (split == 0) {
                    const int zb = 2 * p.rank, zl = (p.slab - zb) / 2;
                    for (int c = zb + uhalf * zl; c < zb + (uhalf + 1) * zl; c += 2)
                        *reinterpret_cast<uint32_t*>(dst + c) = 0u;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (kLR && warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * tcols);
    }
}

// U' = (X L1) / (S_delta S_W) as BF16 hi + lo from the X L1 partial sums, summed in split order (the
// arithmetic of k_cube_encode's own U' step), and the slab's zero padding: thread = (row, column pair).
__global__ void __launch_bounds__(256) k_u_hilo(QuantParams p) {
    const PackedHeader* hdr = reinterpret_cast<const PackedHeader*>(p.packed_w);
    const float SS = __fmul_rn(__uint_as_float(p.scalars[1]), hdr->S_W);
    const int pairs = p.slab / 2;
    const long long total = p.g.N * pairs;
    for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < total; q += (long long)gridDim.x * blockDim.x) {
        const long long rho = q / pairs;
        const int c2 = (int)(q - rho * pairs) * 2;
        uint16_t* dst = p.u_hilo + (size_t)rho * p.slab;
        if (c2 >= 2 * p.rank) {
            *reinterpret_cast<uint32_t*>(dst + c2) = 0u;
            continue;
        }
        if (c2 >= p.rank) continue;   // the lo half of the slab, written with its hi pair below
        float u0 = 0.f, u1 = 0.f;
        for (int sp = 0; sp < p.splits; sp++) {
            const float2 v = *reinterpret_cast<const float2*>(p.u_part + ((size_t)sp * p.g.N + (size_t)rho) * p.rank + c2);
            u0 = __fadd_rn(u0, v.x);
            u1 = __fadd_rn(u1, v.y);
        }
        const float a0 = __fdiv_rn(u0, SS), a1 = __fdiv_rn(u1, SS);
        const uint16_t h0 = f32_to_bf16_rn(a0), h1 = f32_to_bf16_rn(a1);
        const uint16_t l0 = f32_to_bf16_rn(__fsub_rn(a0, __uint_as_float((uint32_t)h0 << 16)));
        const uint16_t l1 = f32_to_bf16_rn(__fsub_rn(a1, __uint_as_float((uint32_t)h1 << 16)));
        *reinterpret_cast<uint32_t*>(dst + c2) = (uint32_t)h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t*>(dst + p.rank + c2) = (uint32_t)l0 | ((uint32_t)l1 << 16);
    }
}

// ------------------------------------------------------------------ kernel tokens of big cubes
//
// Cubes of more than 128 tokens (up to one global cube over the whole lattice).
// CTA = 64 channels of one cube: warp 1 streams the cube's rows through a TMA
// ring of row-segment boxes (the same boxes as the quantise kernels; stages
// sized to the box so that about 110 KB are in flight), and each lane of
// warp 0 keeps the fp32 running sums of two channels (a packed pair) over the
// tokens in (t,h,w) order (Eq. 1, the same arithmetic as the statistics
// kernel), then divides by the count; the per-cube max |mean| goes to kamax.
// The sums are dependent chains of one add per token, so the rows of a box
// are visited in groups of eight whose swizzled offsets are fixed.

constexpr int kMStagesMax = 32;

__host__ __device__ inline uint32_t means_stage_bytes(int bw) { return (uint32_t)align_up((size_t)bw * 128, 1024); }
__host__ __device__ inline int means_stages(int bw) {
    const int n = (int)(110u * 1024u / means_stage_bytes(bw));
    return n < 2 ? 2 : (n > kMStagesMax ? kMStagesMax : n);
}

__global__ void __launch_bounds__(64) k_cube_means_big(const __grid_constant__ CUtensorMap tm_x, QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t stage_bytes = means_stage_bytes(p.bw);
    const int S = means_stages(p.bw);
    uint64_t* full = (uint64_t*)(sm + (size_t)S * stage_bytes);
    uint64_t* empty = full + kMStagesMax;
    volatile int* abort_flag = (volatile int*)(empty + kMStagesMax);
    const Geom& g = p.g;
    const long long k = blockIdx.x;
    const int c0 = blockIdx.y * 64;
    const int kw = (int)(k % g.KW), kh = (int)((k / g.KW) % g.KH), kt = (int)(k / ((long long)g.KW * g.KH));
    const int st = imin(g.t, g.T - kt * g.t), sh = imin(g.h, g.H - kh * g.h), sw = imin(g.w, g.W - kw * g.w);
    const int nbox = st * sh * p.nseg;
    const uint32_t box_bytes = (uint32_t)p.bw * 128u;
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (tid >= 32) {
        if (tid == 32) {
            int issued = 0;
            prefetch_tmap(&tm_x);
            for (int b = 0; b < nbox; b++) {
                const int s = b % S;
                if (b >= S && !mbar_wait(&empty[s], ((b / S) - 1) & 1, abort_flag, p.status, p.budget_ns)) break;
                const int seg = b % p.nseg, dh = (b / p.nseg) % sh, dt = b / (p.nseg * sh);
                mbar_arrive_expect_tx(&full[s], box_bytes);
                tma_load_4d(sm + (size_t)s * stage_bytes, &tm_x, &full[s], c0, kw * g.w + 128 * seg, kh * g.h + dh,
                            kt * g.t + dt);
                issued = b + 1;
            }
            for (int b = (issued > S ? issued - S : 0); b < issued; b++)
                mbar_wait(&full[b % S], (b / S) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else {
        // lane l: channels 2l, 2l+1 = bytes 4 (l % 4) of 16-byte chunk l / 4 of each 128-byte row
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; i++) o[i] = (uint32_t)i * 128u + ((((uint32_t)lane >> 2) ^ (uint32_t)i) << 4) + ((uint32_t)lane & 3u) * 4u;
        uint64_t acc = 0ull;   // (+0, +0)
        bool ok = true;
        for (int b = 0; b < nbox; b++) {
            const int s = b % S;
            ok = ok && __all_sync(0xffffffffu, mbar_wait(&full[s], (b / S) & 1, abort_flag, p.status, p.budget_ns));
            if (ok) {
                const int seg = b % p.nseg;
                const int rows = imin(p.bw, sw - 128 * seg);
                const uint8_t* xs = sm + (size_t)s * stage_bytes;
                int r = 0;
                for (; r + 8 <= rows; r += 8) {
                    const uint8_t* x8 = xs + r * 128;
#pragma unroll
                    for (int i = 0; i < 8; i++) acc = f2_add(acc, f2_from_bf16x2(*reinterpret_cast<const uint32_t*>(x8 + o[i])));
                }
                for (; r < rows; r++) {
                    const uint32_t off = (uint32_t)r * 128u + ((((uint32_t)lane >> 2) ^ ((uint32_t)r & 7u)) << 4) +
                                         ((uint32_t)lane & 3u) * 4u;
                    acc = f2_add(acc, f2_from_bf16x2(*reinterpret_cast<const uint32_t*>(xs + off)));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        const int cnt = st * sh * sw;
        float a0, a1;
        f2_unpack(acc, a0, a1);
        float m0, m1;
        if ((cnt & (cnt - 1)) == 0) {
            const float inv = __frcp_rn((float)cnt);
            m0 = __fmul_rn(a0, inv);
            m1 = __fmul_rn(a1, inv);
        } else {
            m0 = __fdiv_rn(a0, (float)cnt);
            m1 = __fdiv_rn(a1, (float)cnt);
        }
        *reinterpret_cast<float2*>(p.means + k * p.Ci + c0 + 2 * lane) = make_float2(m0, m1);
        const float am = warp_max(fmaxf(fabsf(m0), fabsf(m1)));
        if (lane == 0) atomicMax(&p.kamax[k], __float_as_uint(am));
    }
    __syncthreads();
}

// ------------------------------------------------------------------ single-read quantiser: fix-up pass
//
// After k_cube_stats<., true> every delta group is encoded under its chunk's power-of-two scale
// S_c = 2^e_c, and the global max |delta| gives S_delta = 2^e = pow2(amax / 2688) >= S_c.  Under
// S_delta a group keeps its E2M1 codes and its E4M3 scale code drops by 8 j (j = e - e_c) exactly
// when the code's exponent field is at least j + 1; the other groups are encoded again under
// S_delta from X and their cube's mean.  Part 1 (blockIdx.y == 0) does that per (row, 64-channel
// chunk); part 2 encodes the FP8 kernel tokens from the stored means and the per-cube max |mean|;
// part 3 forms U' = (X L1) / (S_delta S_W) as BF16 hi + lo and the slab's zero padding.

// One 16-channel delta group of cube-major row rho under the power-of-two scale S (exponent e_s),
// from X and the cube's means in global memory: the encode kernels' arithmetic.  Returns the scale
// code; writes the 8 code bytes.
__device__ uint32_t reencode_group(const QuantParams& p, const uint16_t* X, long long rho, int blk, float S,
                                   uint8_t* code_out) {
    long long n = 0, k = 0;
    row_to_token(p.g, rho, &n, &k);
    const uint16_t* x = X + (size_t)n * p.Ci + 16 * blk;
    const float* m = p.means + (size_t)k * p.Ci + 16 * blk;
    float z[16], am = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        z[i] = __fsub_rn(__uint_as_float((uint32_t)x[i] << 16), m[i]);
        am = fmaxf(am, fabsf(z[i]));
    }
    const float den = __fmul_rn(6.f, S);
    const uint32_t sb = cvt_e4m3x2(div_pos(am, den, __frcp_rn(den)), 0.f) & 0x7Fu;
    const float eff = __fmul_rn(e4m3_to_f32(sb), S);
    uint32_t w[2] = {0u, 0u};
    if (eff != 0.f) {
        const float reff = __frcp_rn(eff);
        float q[16];
#pragma unroll
        for (int i = 0; i < 16; i++) q[i] = div_neg(z[i], eff, reff);
        w[0] = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(&q[0])) ^ 0x88888888u;
        w[1] = cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(&q[8])) ^ 0x88888888u;
    }
    *reinterpret_cast<uint2*>(code_out) = make_uint2(w[0], w[1]);
    return sb;
}

__global__ void __launch_bounds__(256) k_single_finish(const uint16_t* X, QuantParams p) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        const PackedHeader* hdr = reinterpret_cast<const PackedHeader*>(p.packed_w);
        if (hdr->magic != DQ_PACK_MAGIC || hdr->version != DQ_PACK_FORMAT_VERSION || hdr->Ci != p.Ci ||
            hdr->rank != p.rank || hdr->slab != p.slab || ((hdr->flags & kPackedC2) != 0) != (p.fp8_product != 0))
            atomicCAS(p.status, 0, kStatusBadWeight);
    }
    const float amax = __uint_as_float(p.scalars[0]);
    int es = 0;
    const float S = (amax == 0.f) ? 1.f : pow2_ceil(__fdiv_rn(amax, 2688.f), &es);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) p.scalars[1] = __float_as_uint(S);
    const int Ci = p.Ci, chunks = Ci / 64;
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    if (blockIdx.y == 0) {
        // scale codes: a warp per cube-major row, a lane per 64-channel chunk, whose four group scale
        // codes sit in one 32-bit word of the A-operand scale layout; shift each by the chunk's exponent
        // difference, or encode the group again
        for (long long rho = warp0; rho < p.g.N; rho += nwarps) {
            const int8_t* prow = p.prov + (size_t)rho * chunks;
            for (int ch = lane; ch < chunks; ch += 32) {
                const int ec = prow[ch];
                if (ec == -128 || ec == es) continue;   // an all-zero chunk, or no shift
                const int j = es - ec;
                uint32_t* sp = reinterpret_cast<uint32_t*>(p.dscales + sfa_offset(rho, 4 * ch, Ci));
                const uint32_t scw = *sp;
                uint32_t out = 0;
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const uint32_t c = (scw >> (8 * h)) & 0xFFu;
                    uint32_t nc;
                    if (c == 0u)
                        nc = 0u;                              // a zero scale stays zero, its codes +0
                    else if ((int)((c >> 3) & 15u) >= j + 1)
                        nc = c - 8u * (uint32_t)j;            // same codes, scale j binades lower
                    else
                        nc = reencode_group(p, X, rho, 4 * ch + h, S, p.dcodes + (size_t)rho * (Ci / 2) + 32 * ch + 8 * h);
                    out |= nc << (8 * h);
                }
                if (out != scw) *sp = out;
            }
        }
    } else if (blockIdx.y == 1) {
        // FP8 kernel tokens under s8 = max |mean| / 448 (and their BF16 copy for the exact product):
        // a warp per cube, a lane per 8 channels
        for (long long k = warp0; k < p.g.K; k += nwarps) {
            const float s8 = __fdiv_rn(__uint_as_float(p.kamax[k]), 448.f);
            if (lane == 0) p.s8[k] = s8;
            const float rs8 = (s8 != 0.f) ? __frcp_rn(s8) : 0.f;
            const uint64_t b2 = f2_pack(s8, s8), nrb2 = f2_pack(-rs8, -rs8);
            for (int c0 = 8 * lane; c0 < Ci; c0 += 256) {
                uint32_t c[4] = {0u, 0u, 0u, 0u};
                if (s8 != 0.f) {
                    uint64_t m[4];
                    load8(p.means + (size_t)k * Ci + c0, m);
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        float lo, hi;
                        f2_unpack(f2_div_neg(m[e], b2, nrb2), lo, hi);
                        c[e] = cvt_e4m3x2(lo, hi) ^ 0x8080u;
                    }
                }
                *reinterpret_cast<uint2*>(p.q8 + (size_t)k * Ci + c0) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
                if (!p.fp8_product) {
                    uint32_t bfw[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) bfw[e] = e4m3x2_to_bf16x2(c[e]);
                    *reinterpret_cast<uint4*>(p.q8_bf16 + (size_t)k * Ci + c0) = make_uint4(bfw[0], bfw[1], bfw[2], bfw[3]);
                }
            }
        }
    } else {
        // U' = (X L1) / (S_delta S_W) as BF16 hi + lo, the partial sums added in split order
        const float SS = __fmul_rn(S, reinterpret_cast<const PackedHeader*>(p.packed_w)->S_W);
        // a warp per row, a lane per two columns of the slab row
        for (long long rho = warp0; rho < p.g.N; rho += nwarps)
        for (int c = 2 * lane; c < p.slab; c += 64) {
            uint16_t* dst = p.u_hilo + (size_t)rho * p.slab;
            if (c >= p.rank) {
                if (c >= 2 * p.rank) *reinterpret_cast<uint32_t*>(dst + c) = 0u;   // padding
                continue;
            }
            float u0 = 0.f, u1 = 0.f;
            for (int sp = 0; sp < p.splits; sp++) {
                const float2 v = *reinterpret_cast<const float2*>(p.u_part + ((size_t)sp * p.g.N + (size_t)rho) * p.rank + c);
                u0 = __fadd_rn(u0, v.x);
                u1 = __fadd_rn(u1, v.y);
            }
            const float a0 = __fdiv_rn(u0, SS), a1 = __fdiv_rn(u1, SS);
            const uint16_t h0 = f32_to_bf16_rn(a0), h1 = f32_to_bf16_rn(a1);
            const uint16_t l0 = f32_to_bf16_rn(__fsub_rn(a0, __uint_as_float((uint32_t)h0 << 16)));
            const uint16_t l1 = f32_to_bf16_rn(__fsub_rn(a1, __uint_as_float((uint32_t)h1 << 16)));
            *reinterpret_cast<uint32_t*>(dst + c) = (uint32_t)h0 | ((uint32_t)h1 << 16);
            *reinterpret_cast<uint32_t*>(dst + p.rank + c) = (uint32_t)l0 | ((uint32_t)l1 << 16);
        }
    }
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_cube_means_big(const CUtensorMap& tm_x, const QuantParams& p, cudaStream_t st) {
    const size_t smem = (size_t)means_stages(p.bw) * means_stage_bytes(p.bw) + 2 * kMStagesMax * 8 + 16 + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_cube_means_big, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.g.K, (unsigned)(p.Ci / 64));
    k_cube_means_big<<<grid, 64, smem, st>>>(tm_x, p);
    return cudaGetLastError();
}

cudaError_t launch_single_finish(const void* X, const QuantParams& p, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    k_single_finish<<<dim3((unsigned)(4 * (sms > 0 ? sms : 148)), 3), 256, 0, st>>>((const uint16_t*)X, p);
    return cudaGetLastError();
}

size_t quant_smem_bytes(int rank, bool stats, int m_rows, int x_rows) {
    return q_smem_layout(rank, stats, m_rows, x_rows).total + 1024;
}

namespace {
// CTAs of a persistent quantise kernel: as many as can be resident at once,
// from the kernel's registers and shared memory (the runtime's occupancy
// query answers one CTA per SM for k_cube_stats where two fit and run).
int resident_grid(const void* fn, int threads, size_t smem, int items) {
    int dev = 0, sms = 148, smem_sm = 233472, reserved = 1024;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaFuncAttributes fa;
    int per_sm = 1;
    if (cudaFuncGetAttributes(&fa, fn) == cudaSuccess && sms > 0) {
        const int warps = (threads + 31) / 32;
        const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
        per_sm = 2048 / (warps * 32);
        // the four sub-partitions of an SM each hold 16384 registers and a quarter of its warps
        while (per_sm > 1 && ((per_sm * warps + 3) / 4) * regs_warp > 16384) per_sm--;
        while (per_sm > 1 && (size_t)per_sm * (smem + fa.sharedSizeBytes + (size_t)reserved) > (size_t)smem_sm)
            per_sm--;
    }
    return imin(items, (sms > 0 ? sms : 148) * per_sm);
}
}  // namespace

template <bool kPairs, bool kSingle>
cudaError_t launch_stats(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p, cudaStream_t st) {
    size_t smem = q_smem_layout(p.rank, true, kSingle ? p.m_rows : 0, 128, kSingle).total + 1024;
    auto fn = k_cube_stats<kPairs, kSingle>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int grid = resident_grid((const void*)fn, kQCompute + 64, smem, p.item1 - p.item0);
    fn<<<grid, kQCompute + 64, smem, st>>>(tm_x, tm_l1, p);
    return cudaGetLastError();
}

cudaError_t launch_cube_stats(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p,
                              cudaStream_t st) {
    return p.stat_pairs ? launch_stats<true, false>(tm_x, tm_l1, p, st) : launch_stats<false, false>(tm_x, tm_l1, p, st);
}

cudaError_t launch_cube_single(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p,
                               cudaStream_t st) {
    return p.stat_pairs ? launch_stats<true, true>(tm_x, tm_l1, p, st) : launch_stats<false, true>(tm_x, tm_l1, p, st);
}

cudaError_t launch_cube_encode(const CUtensorMap& tm_x, const CUtensorMap& tm_m, const QuantParams& p,
                               cudaStream_t st) {
    size_t smem = quant_smem_bytes(p.rank, false, p.m_rows, p.bt * p.bh * p.bw);
    cudaError_t e = cudaFuncSetAttribute(k_cube_encode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_cube_encode<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int grid = resident_grid((const void*)k_cube_encode<false>, kQCompute + 32, smem, p.n_boxes * p.splits);
    k_cube_encode<false><<<grid, kQCompute + 32, smem, st>>>(tm_x, tm_m, tm_m, p);
    return cudaGetLastError();
}

cudaError_t launch_cube_encode_lowrank(const CUtensorMap& tm_x, const CUtensorMap& tm_m, const CUtensorMap& tm_l1,
                                       const QuantParams& p, cudaStream_t st) {
    size_t smem = quant_smem_bytes(p.rank, true, p.m_rows, p.bt * p.bh * p.bw);
    cudaError_t e = cudaFuncSetAttribute(k_cube_encode<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_cube_encode<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int grid = resident_grid((const void*)k_cube_encode<true>, kQCompute + 64, smem, p.n_boxes * p.splits);
    k_cube_encode<true><<<grid, kQCompute + 64, smem, st>>>(tm_x, tm_m, tm_l1, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long work = p.g.N * (p.slab / 2);
    k_u_hilo<<<(int)imin((int)cdiv(work, 256), 8 * sms), 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace dq
