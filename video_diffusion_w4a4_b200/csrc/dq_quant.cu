// Cube-quantise kernels (DeltaQuant note, papernotes.org, key designs 2-4).
//
//   a1  k_cube_stats:  per cube the fp32 mean of its tokens (Eq. 1), the
//       max |mean| over channels (the FP8 kernel-token scale), the global
//       max |token - mean| (the FP4 per-tensor scale), and X L1 (the SVD
//       low-rank down-projection of Eq. 3) on the tensor cores.
//   a2  k_cube_encode: recomputes the same means bit for bit, writes the FP8
//       E4M3 kernel tokens, the FP4 E2M1 delta codes with their E4M3 group-16
//       scales (Eq. 4 per group), and U' = (X L1) / (S_delta S_W) as BF16 hi+lo.
//
// Both stream X through 4-D TMA boxes of t x h x (nw w) tokens by 64
// channels straight from the flattened (t,h,w) layout, so that every box
// holds nw whole cubes.  The two passes exist because the per-tensor delta
// scale needs the amax of every delta before any delta can be encoded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dq_common.h"
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

namespace {

constexpr int kQStages = 4;
constexpr int kMeanStride = 68;  // floats per cube row of the means table (bank spread)

struct QSmem {
    // offsets in bytes from the 1024-aligned dynamic smem base
    uint32_t x, l1, means, kmax, s8, bars, misc, total;  // means: 2 slots of nw x kMeanStride floats
};

__host__ __device__ inline QSmem q_smem_layout(int nw, int rank, bool with_l1) {
    QSmem L;
    uint32_t off = 0;
    L.x = off;
    off += kQStages * 16384;
    L.l1 = off;
    if (with_l1) off += kQStages * (uint32_t)align_up((size_t)rank * 128, 1024);
    L.means = off;
    off += 2u * (uint32_t)nw * kMeanStride * 4;   // one table per chunk group
    L.kmax = off;
    off += (uint32_t)nw * 4;
    L.s8 = off;
    off += (uint32_t)nw * 4;
    off = (uint32_t)align_up(off, 16);
    L.bars = off;
    off += (2 * kQStages + 2) * 8;
    L.misc = off;
    off += 64;
    L.total = off;
    return L;
}

__device__ __forceinline__ float ld_x_swz(const uint8_t* xs, int row, int c) {
    uint32_t off = (uint32_t)row * 128u + ((((uint32_t)c >> 3) ^ ((uint32_t)row & 7u)) << 4) + (((uint32_t)c & 7u) << 1);
    uint16_t v = *reinterpret_cast<const uint16_t*>(xs + off);
    return __uint_as_float((uint32_t)v << 16);
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

// Row `row` of a box -> validity, cube slot j, cube-major row rho, cube index k.
__device__ __forceinline__ bool box_row(const QuantParams& p, const BoxPos& B, int row, int* j, long long* rho,
                                        long long* k) {
    const Geom& g = p.g;
    if (p.big) {
        const int kw = B.bkw, dw = B.dw0 + row;
        const int sh = imin(g.h, g.H - B.bkh * g.h), sw = imin(g.w, g.W - kw * g.w);
        if (row >= p.bw || dw >= sw) return false;
        *j = 0;
        *rho = cube_first_row(g, B.bkt, B.bkh, kw) + ((long long)B.dt0 * sh + B.dh0) * sw + dw;
        *k = ((long long)B.bkt * g.KH + B.bkh) * g.KW + kw;
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
    *j = jj;
    *rho = cube_first_row(g, B.bkt, B.bkh, kw) + ((long long)dt * sh + dh) * sw + dw;
    *k = ((long long)B.bkt * g.KH + B.bkh) * g.KW + kw;
    return true;
}

// Kernel tokens (Eq. 1) of cube slot j for channels [8g, 8g+8) of the chunk:
// an fp32 running sum over the cube's tokens in (t,h,w) order, then the
// division by the token count (a product with the exact reciprocal when the
// count is a power of two, which gives the identical rounding).  Returns
// false for cube slots past the end of the lattice.
__device__ __forceinline__ bool cube_mean8(const QuantParams& p, const BoxPos& B, const uint8_t* xs, int j, int g,
                                           int st, int sh, float (&m)[8]) {
    const Geom& g_ = p.g;
    const int kw = B.bkw * p.nw + j;
    if (kw >= g_.KW) return false;
    const int sw = imin(g_.w, g_.W - kw * g_.w);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; e++) acc[e] = 0.f;
    for (int dt = 0; dt < st; dt++)
        for (int dh = 0; dh < sh; dh++) {
            const int row0 = (dt * p.bh + dh) * p.bw + j * g_.w;
            for (int dw = 0; dw < sw; dw++) {
                uint4 v = ld_x8_swz(xs, row0 + dw, g);
                acc[0] = __fadd_rn(acc[0], bf16_lo(v.x));
                acc[1] = __fadd_rn(acc[1], bf16_hi(v.x));
                acc[2] = __fadd_rn(acc[2], bf16_lo(v.y));
                acc[3] = __fadd_rn(acc[3], bf16_hi(v.y));
                acc[4] = __fadd_rn(acc[4], bf16_lo(v.z));
                acc[5] = __fadd_rn(acc[5], bf16_hi(v.z));
                acc[6] = __fadd_rn(acc[6], bf16_lo(v.w));
                acc[7] = __fadd_rn(acc[7], bf16_hi(v.w));
            }
        }
    const int cnt = st * sh * sw;
    if ((cnt & (cnt - 1)) == 0) {
        const float inv = __frcp_rn((float)cnt);
#pragma unroll
        for (int e = 0; e < 8; e++) m[e] = __fmul_rn(acc[e], inv);
    } else {
#pragma unroll
        for (int e = 0; e < 8; e++) m[e] = __fdiv_rn(acc[e], (float)cnt);
    }
    return true;
}

// Named barrier of one chunk group (constant barrier ids keep the CTA's barrier count at 3).
__device__ __forceinline__ void group_sync(int grp) {
    if (grp == 0)
        bar_sync(1, 128);
    else
        bar_sync(2, 128);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace

// ------------------------------------------------------------------ a1: statistics + X L1
//
// Warps 0-7 compute (thread t: token row t % 128, channel half t / 128 of each
// 64-channel chunk), warp 8 loads, warp 9 owns tensor memory and issues the
// X L1 MMAs.  One named barrier per chunk: the means table is double-buffered.

constexpr int kQCompute = 256;
constexpr int kQGroup = 128;   // compute threads per chunk group

__global__ void __launch_bounds__(kQCompute + 64, 2) k_cube_stats(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_l1,
                                                                  QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QSmem L = q_smem_layout(p.nw, p.rank, true);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kQStages;
    uint64_t* done = empty + kQStages;
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);
    float* red = (float*)(sm + L.misc + 16);  // 8 floats
    uint32_t* kmax = (uint32_t*)(sm + L.kmax);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int box = blockIdx.x, split = blockIdx.y;
    const BoxPos B = box_pos(p, box);
    const int nchunks = p.chunks_per_split;
    const int c_base = split * nchunks * 64;
    const uint32_t l1_bytes = (uint32_t)p.rank * 128u;
    const uint32_t l1_stride = (uint32_t)align_up(l1_bytes, 1024);
    const uint32_t x_bytes = (uint32_t)p.bt * p.bh * p.bw * 128u;
    uint32_t tmem_cols = 32;
    while (tmem_cols < (uint32_t)p.rank) tmem_cols <<= 1;

    if (tid == 0) {
        for (int s = 0; s < kQStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQGroup + 1);   // the chunk's group + the MMA commit
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    for (int j = tid; j < p.nw; j += blockDim.x) kmax[j] = 0u;
    if (warp == 9) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ---------------- producer
        if (lane == 0) {
            int issued = 0;
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_l1);
            for (int i = 0; i < nchunks; i++) {
                int s = i % kQStages;
                if (i >= kQStages && !mbar_wait(&empty[s], ((i / kQStages) - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                mbar_arrive_expect_tx(&full[s], x_bytes + l1_bytes);
                int c0 = c_base + i * 64;
                tma_load_4d(sm + L.x + s * 16384, &tm_x, &full[s], c0, B.w0, B.h0, B.t0);
                tma_load_2d(sm + L.l1 + s * l1_stride, &tm_l1, &full[s], c0, 0);
                issued = i + 1;
            }
            // drain: every issued load lands before shared memory is released
            for (int i = (issued > kQStages ? issued - kQStages : 0); i < issued; i++)
                mbar_wait(&full[i % kQStages], (i / kQStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 9) {
        // ---------------- MMA issuer: U += X_chunk L1_chunk^T (M = 128 rows, N = rank, K = 64)
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, p.rank);
            for (int i = 0; i < nchunks; i++) {
                int s = i % kQStages;
                if (!mbar_wait(&full[s], (i / kQStages) & 1, abort_flag, p.status, p.budget_ns)) break;
                tc_fence_after();
                uint32_t xa = smem_u32(sm + L.x + s * 16384), la = smem_u32(sm + L.l1 + s * l1_stride);
#pragma unroll
                for (int k = 0; k < 4; k++)
                    mma_bf16(tmem, desc_k_sw128(xa + 32 * k), desc_k_sw128(la + 32 * k), idesc, (i | k) != 0);
                tc_commit(&empty[s]);
            }
            tc_commit(done);
            // every MMA has retired before tensor memory is released
            mbar_wait(done, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // ---------------- compute warps 0-7: two groups of four warps take alternate chunks
        // (group g: chunks i = g, g+2, ...), each with its own means table and named barrier,
        // so that one group's waits overlap the other's work.  Thread = one token row.
        const int grp = tid >> 7, row = tid & 127, half = grp;
        float damax = 0.f;
        int myj = -1;
        long long myrho = 0, myk = 0;
        const bool row_ok = box_row(p, B, row, &myj, &myrho, &myk);
        const int st = imin(p.g.t, p.g.T - B.t0), sh = imin(p.g.h, p.g.H - B.h0);
        float* means = (float*)(sm + L.means) + grp * p.nw * kMeanStride;
        for (int i = grp; i < nchunks; i += 2) {
            const int s = i % kQStages;
            // a failed wait skips the work but keeps the barrier protocol
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / kQStages) & 1, abort_flag, p.status,
                                                              p.budget_ns));
            const uint8_t* xs = sm + L.x + s * 16384;
            if (!p.big) {
                // kernel tokens of the box's cubes for these 64 channels
                for (int q = row; ok && q < p.nw * 8; q += kQGroup) {
                    const int j = q >> 3, g8 = q & 7;
                    float m[8];
                    if (!cube_mean8(p, B, xs, j, g8, st, sh, m)) continue;
                    float* dst = means + j * kMeanStride + 8 * g8;
                    *reinterpret_cast<float4*>(dst) = make_float4(m[0], m[1], m[2], m[3]);
                    *reinterpret_cast<float4*>(dst + 4) = make_float4(m[4], m[5], m[6], m[7]);
                    float am = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; e++) am = fmaxf(am, fabsf(m[e]));
                    atomicMax(&kmax[j], __float_as_uint(am));
                }
                group_sync(grp);
            }
            // delta amax of this thread's token row (64 channels)
            if (ok && row_ok) {
                const float* mj = p.big ? p.means + (size_t)myk * p.Ci + c_base + i * 64 : means + myj * kMeanStride;
#pragma unroll
                for (int q8 = 0; q8 < 8; q8++) {
                    uint4 xv = ld_x8_swz(xs, row, q8);
                    float4 m0 = *reinterpret_cast<const float4*>(mj + q8 * 8);
                    float4 m1 = *reinterpret_cast<const float4*>(mj + q8 * 8 + 4);
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_lo(xv.x), m0.x)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_hi(xv.x), m0.y)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_lo(xv.y), m0.z)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_hi(xv.y), m0.w)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_lo(xv.z), m1.x)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_hi(xv.z), m1.y)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_lo(xv.w), m1.z)));
                    damax = fmaxf(damax, fabsf(__fsub_rn(bf16_hi(xv.w), m1.w)));
                }
            }
            if (!p.big) group_sync(grp);   // this group's means table is rewritten next chunk
            mbar_arrive(&empty[s]);
        }
        // epilogue: U partial rows out of tensor memory (sub-partition warp % 4; this warp's column half)
        const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, p.status, p.budget_ns));
        tc_fence_after();
        if (ok) {
            float* urow = p.u_part + ((size_t)split * p.g.N + (size_t)myrho) * p.rank;
            for (int c = 16 * half; c < p.rank; c += 32) {
                uint32_t r[16];
                tmem_ld_x16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)c, r);
                tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int v = 0; v < 16; v += 4)
                        *reinterpret_cast<float4*>(urow + c + v) =
                            make_float4(__uint_as_float(r[v]), __uint_as_float(r[v + 1]), __uint_as_float(r[v + 2]),
                                        __uint_as_float(r[v + 3]));
                }
            }
        }
        float wm = warp_max(damax);
        if (lane == 0) red[warp] = wm;
        // barrier 3: ids 1 and 2 belong to the chunk groups, and one group may still be in
        // its loop when the other gets here (a barrier must not see two thread counts at once)
        bar_sync(3, kQCompute);
        if (tid == 0) {
            float bm = 0.f;
            for (int w = 0; w < 8; w++) bm = fmaxf(bm, red[w]);
            atomicMax(&p.scalars[0], __float_as_uint(bm));
        }
        for (int j = tid; j < p.nw; j += kQCompute) {
            int kw = B.bkw * p.nw + j;
            if (kw < p.g.KW) {
                long long k = ((long long)B.bkt * p.g.KH + B.bkh) * p.g.KW + kw;
                atomicMax(&p.kamax[k], kmax[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

// ------------------------------------------------------------------ a2: encode
//
// Warps 0-7 compute (thread t: token row t % 128, channel half t / 128 of each
// 64-channel chunk, i.e. two FP4 groups of 16), warp 8 loads.

__global__ void __launch_bounds__(kQCompute + 32, 2) k_cube_encode(const __grid_constant__ CUtensorMap tm_x,
                                                                  QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const QSmem L = q_smem_layout(p.nw, p.rank, false);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kQStages;
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);
    float* s8s = (float*)(sm + L.s8);
    float* rs8s = (float*)(sm + L.kmax);   // reciprocals of s8 (the kmax slot is unused in this kernel)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int box = blockIdx.x, split = blockIdx.y;
    const BoxPos B = box_pos(p, box);
    const int nchunks = p.chunks_per_split;
    const int c_base = split * nchunks * 64;
    const uint32_t x_bytes = (uint32_t)p.bt * p.bh * p.bw * 128u;
    const int Ci = p.Ci;

    const PackedHeader* hdr = reinterpret_cast<const PackedHeader*>(p.packed_w);
    if (tid == 0) {
        for (int s = 0; s < kQStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQGroup);   // the chunk's group
        }
        *abort_flag = 0;
        fence_barrier_init();
        if (box == 0 && split == 0 &&
            (hdr->magic != 0x31575144u || hdr->Ci != p.Ci || hdr->rank != p.rank || hdr->slab != p.slab))
            atomicCAS(p.status, 0, kStatusBadWeight);
    }
    // per-tensor delta scale S = amax / (6*448) (1 if amax = 0); S_W from the packed weight
    const float damax = __uint_as_float(p.scalars[0]);
    const float S = (damax == 0.f) ? 1.f : __fdiv_rn(damax, 2688.f);
    const float denom = __fmul_rn(6.f, S);
    for (int j = tid; j < p.nw; j += blockDim.x) {
        int kw = B.bkw * p.nw + j;
        float s = 0.f;
        if (kw < p.g.KW) {
            long long k = ((long long)B.bkt * p.g.KH + B.bkh) * p.g.KW + kw;
            s = __fdiv_rn(__uint_as_float(p.kamax[k]), 448.f);
            if (split == 0) p.s8[k] = s;
        }
        s8s[j] = s;
        rs8s[j] = (s != 0.f) ? __frcp_rn(s) : 0.f;
    }
    if (box == 0 && split == 0 && tid == 0) p.scalars[1] = __float_as_uint(S);
    __syncthreads();

    if (warp == 8) {
        if (lane == 0) {
            int issued = 0;
            prefetch_tmap(&tm_x);
            for (int i = 0; i < nchunks; i++) {
                int s = i % kQStages;
                if (i >= kQStages && !mbar_wait(&empty[s], ((i / kQStages) - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                mbar_arrive_expect_tx(&full[s], x_bytes);
                tma_load_4d(sm + L.x + s * 16384, &tm_x, &full[s], c_base + i * 64, B.w0, B.h0, B.t0);
                issued = i + 1;
            }
            for (int i = (issued > kQStages ? issued - kQStages : 0); i < issued; i++)
                mbar_wait(&full[i % kQStages], (i / kQStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else {
        // two groups of four warps take alternate chunks (see k_cube_stats); thread = token row
        const int grp = tid >> 7, row = tid & 127, half = grp;
        int myj = -1;
        long long myrho = 0, myk = 0;
        const bool row_ok = box_row(p, B, row, &myj, &myrho, &myk);
        const int st = imin(p.g.t, p.g.T - B.t0), sh = imin(p.g.h, p.g.H - B.h0);
        float* means = (float*)(sm + L.means) + grp * p.nw * kMeanStride;
        for (int i = grp; i < nchunks; i += 2) {
            const int s = i % kQStages;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / kQStages) & 1, abort_flag, p.status,
                                                              p.budget_ns));
            const uint8_t* xs = sm + L.x + s * 16384;
            const int c0 = c_base + i * 64;
            // kernel tokens: means, FP8 E4M3 codes with the per-token scale s8 = max|mean| / 448
            // (big cubes: means from the means kernel, encoded once per cube by its first box)
            const bool enc_q8 = !p.big || (B.dt0 == 0 && B.dh0 == 0 && B.dw0 == 0);
            for (int q = row; ok && enc_q8 && q < p.nw * 8; q += kQGroup) {
                const int j = q >> 3, g8 = q & 7;
                float m[8];
                if (p.big) {
                    const float* src = p.means + (size_t)(((long long)B.bkt * p.g.KH + B.bkh) * p.g.KW + B.bkw) * Ci +
                                       c0 + 8 * g8;
                    const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
                    m[0] = a.x; m[1] = a.y; m[2] = a.z; m[3] = a.w; m[4] = b.x; m[5] = b.y; m[6] = b.z; m[7] = b.w;
                } else {
                    if (!cube_mean8(p, B, xs, j, g8, st, sh, m)) continue;
                    float* dst = means + j * kMeanStride + 8 * g8;
                    *reinterpret_cast<float4*>(dst) = make_float4(m[0], m[1], m[2], m[3]);
                    *reinterpret_cast<float4*>(dst + 4) = make_float4(m[4], m[5], m[6], m[7]);
                }
                const long long k = ((long long)B.bkt * p.g.KH + B.bkh) * p.g.KW + (B.bkw * p.nw + j);
                const float s8 = s8s[j], rs8 = rs8s[j];
                uint32_t c[4] = {0u, 0u, 0u, 0u};
                if (s8 != 0.f) {
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        c[e] = cvt_e4m3x2(div_pos(m[2 * e], s8, rs8), div_pos(m[2 * e + 1], s8, rs8));
                }
                *reinterpret_cast<uint2*>(p.q8 + (size_t)k * Ci + c0 + 8 * g8) =
                    make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
                uint32_t bfw[4];
#pragma unroll
                for (int e = 0; e < 4; e++)
                    bfw[e] = (uint32_t)f32_to_bf16_rn(e4m3_to_f32(c[e] & 0xFF)) |
                             ((uint32_t)f32_to_bf16_rn(e4m3_to_f32(c[e] >> 8)) << 16);
                *reinterpret_cast<uint4*>(p.q8_bf16 + (size_t)k * Ci + c0 + 8 * g8) =
                    make_uint4(bfw[0], bfw[1], bfw[2], bfw[3]);
            }
            if (!p.big) group_sync(grp);
            // delta tokens: FP4 E2M1 with E4M3 group-16 scales under S (four groups per thread)
            if (ok && row_ok) {
                const float* mj = p.big ? p.means + (size_t)myk * Ci + c0 : means + myj * kMeanStride;
                uint32_t codes[8];
                uint32_t sc = 0;
#pragma unroll
                for (int b = 0; b < 4; b++) {
                    float z[16];
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        uint4 xv = ld_x8_swz(xs, row, 2 * b + h);
                        float4 m0 = *reinterpret_cast<const float4*>(mj + 16 * b + 8 * h);
                        float4 m1 = *reinterpret_cast<const float4*>(mj + 16 * b + 8 * h + 4);
                        z[8 * h + 0] = __fsub_rn(bf16_lo(xv.x), m0.x);
                        z[8 * h + 1] = __fsub_rn(bf16_hi(xv.x), m0.y);
                        z[8 * h + 2] = __fsub_rn(bf16_lo(xv.y), m0.z);
                        z[8 * h + 3] = __fsub_rn(bf16_hi(xv.y), m0.w);
                        z[8 * h + 4] = __fsub_rn(bf16_lo(xv.z), m1.x);
                        z[8 * h + 5] = __fsub_rn(bf16_hi(xv.z), m1.y);
                        z[8 * h + 6] = __fsub_rn(bf16_lo(xv.w), m1.z);
                        z[8 * h + 7] = __fsub_rn(bf16_hi(xv.w), m1.w);
                    }
                    float am = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; e++) am = fmaxf(am, fabsf(z[e]));
                    uint32_t sb = cvt_e4m3x2(__fdiv_rn(am, denom), 0.f) & 0xFFu;
                    float eff = __fmul_rn(e4m3_to_f32(sb), S);
                    sc |= sb << (8 * b);
                    const float reff = (eff != 0.f) ? __frcp_rn(eff) : 0.f;
#pragma unroll
                    for (int e = 0; e < 16; e += 8) {
                        uint32_t wv = 0;
                        if (eff != 0.f) {
#pragma unroll
                            for (int u = 0; u < 8; u += 2)
                                wv |= cvt_e2m1x2(div_pos(z[e + u], eff, reff), div_pos(z[e + u + 1], eff, reff))
                                      << (4 * u);
                        }
                        codes[2 * b + e / 8] = wv;
                    }
                }
                uint8_t* dst = p.dcodes + (size_t)myrho * (Ci / 2) + c0 / 2;
                reinterpret_cast<uint4*>(dst)[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                reinterpret_cast<uint4*>(dst)[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                *reinterpret_cast<uint32_t*>(p.dscales + sf_offset(myrho, c0 / 16, Ci)) = sc;
            }
            if (!p.big) group_sync(grp);   // this group's means table is rewritten next chunk
            mbar_arrive(&empty[s]);
        }
        // U' = (X L1) / (S_delta S_W) as BF16 hi + lo, slab zero-padded (split 0 only; half the columns each)
        if (split == 0 && row_ok) {
            const float SS = __fmul_rn(S, hdr->S_W);
            uint16_t* dst = p.u_hilo + (size_t)myrho * p.slab;
            const int cpb = p.rank / 2;
            for (int c = half * cpb; c < (half + 1) * cpb; c += 2) {
                float u0 = 0.f, u1 = 0.f;
                for (int sp = 0; sp < p.splits; sp++) {
                    const float* src = p.u_part + ((size_t)sp * p.g.N + (size_t)myrho) * p.rank + c;
                    u0 = __fadd_rn(u0, src[0]);
                    u1 = __fadd_rn(u1, src[1]);
                }
                float a0 = __fdiv_rn(u0, SS), a1 = __fdiv_rn(u1, SS);
                uint16_t h0 = f32_to_bf16_rn(a0), h1 = f32_to_bf16_rn(a1);
                uint16_t l0 = f32_to_bf16_rn(__fsub_rn(a0, __uint_as_float((uint32_t)h0 << 16)));
                uint16_t l1 = f32_to_bf16_rn(__fsub_rn(a1, __uint_as_float((uint32_t)h1 << 16)));
                *reinterpret_cast<uint32_t*>(dst + c) = (uint32_t)h0 | ((uint32_t)h1 << 16);
                *reinterpret_cast<uint32_t*>(dst + p.rank + c) = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            const int zb = 2 * p.rank, zl = (p.slab - zb) / 2;
            for (int c = zb + half * zl; c < zb + (half + 1) * zl; c += 2) *reinterpret_cast<uint32_t*>(dst + c) = 0u;
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------ kernel tokens of big cubes
//
// Cubes of more than 128 tokens (up to one global cube over the whole lattice).
// CTA = 64 channels of one cube: warp 2 streams the cube's rows through an
// 8-stage TMA ring (the same row-segment boxes as the quantise kernels) and
// threads 0-63 each keep one channel's fp32 running sum over the tokens in
// (t,h,w) order (Eq. 1, the same arithmetic as cube_mean8), then divide by the
// count; the per-cube max |mean| goes to kamax.

constexpr int kMStages = 8;

__global__ void __launch_bounds__(96) k_cube_means_big(const __grid_constant__ CUtensorMap tm_x, QuantParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(sm + kMStages * 16384);
    uint64_t* empty = full + kMStages;
    volatile int* abort_flag = (volatile int*)(empty + kMStages);
    const Geom& g = p.g;
    const long long k = blockIdx.x;
    const int c0 = blockIdx.y * 64;
    const int kw = (int)(k % g.KW), kh = (int)((k / g.KW) % g.KH), kt = (int)(k / ((long long)g.KW * g.KH));
    const int st = imin(g.t, g.T - kt * g.t), sh = imin(g.h, g.H - kh * g.h), sw = imin(g.w, g.W - kw * g.w);
    const int nbox = st * sh * p.nseg;
    const uint32_t box_bytes = (uint32_t)p.bw * 128u;
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kMStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 64);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (tid >= 64) {
        if (tid == 64) {
            int issued = 0;
            prefetch_tmap(&tm_x);
            for (int b = 0; b < nbox; b++) {
                const int s = b % kMStages;
                if (b >= kMStages && !mbar_wait(&empty[s], ((b / kMStages) - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                const int seg = b % p.nseg, dh = (b / p.nseg) % sh, dt = b / (p.nseg * sh);
                mbar_arrive_expect_tx(&full[s], box_bytes);
                tma_load_4d(sm + s * 16384, &tm_x, &full[s], c0, kw * g.w + 128 * seg, kh * g.h + dh, kt * g.t + dt);
                issued = b + 1;
            }
            for (int b = (issued > kMStages ? issued - kMStages : 0); b < issued; b++)
                mbar_wait(&full[b % kMStages], (b / kMStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else {
        float acc = 0.f;
        bool ok = true;
        for (int b = 0; b < nbox; b++) {
            const int s = b % kMStages;
            ok = ok && mbar_wait(&full[s], (b / kMStages) & 1, abort_flag, p.status, p.budget_ns);
            if (ok) {
                const int seg = b % p.nseg;
                const int rows = imin(p.bw, sw - 128 * seg);
                const uint8_t* xs = sm + s * 16384;
                for (int r = 0; r < rows; r++) acc = __fadd_rn(acc, ld_x_swz(xs, r, tid));
            }
            mbar_arrive(&empty[s]);
        }
        const int cnt = st * sh * sw;
        const float m = ((cnt & (cnt - 1)) == 0) ? __fmul_rn(acc, __frcp_rn((float)cnt)) : __fdiv_rn(acc, (float)cnt);
        p.means[k * p.Ci + c0 + tid] = m;
        const float am = warp_max(fabsf(m));
        if ((tid & 31) == 0) atomicMax(&p.kamax[k], __float_as_uint(am));
    }
    __syncthreads();
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_cube_means_big(const CUtensorMap& tm_x, const QuantParams& p, cudaStream_t st) {
    const size_t smem = kMStages * 16384 + 2 * kMStages * 8 + 16 + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_cube_means_big, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.g.K, (unsigned)(p.Ci / 64));
    k_cube_means_big<<<grid, 96, smem, st>>>(tm_x, p);
    return cudaGetLastError();
}

size_t quant_smem_bytes(int nw, int rank, bool stats) {
    return q_smem_layout(nw, rank, stats).total + 1024;
}

cudaError_t launch_cube_stats(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p,
                              cudaStream_t st) {
    size_t smem = quant_smem_bytes(p.nw, p.rank, true);
    cudaError_t e = cudaFuncSetAttribute(k_cube_stats, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_boxes, p.splits);
    k_cube_stats<<<grid, kQCompute + 64, smem, st>>>(tm_x, tm_l1, p);
    return cudaGetLastError();
}

cudaError_t launch_cube_encode(const CUtensorMap& tm_x, const QuantParams& p, cudaStream_t st) {
    size_t smem = quant_smem_bytes(p.nw, p.rank, false);
    cudaError_t e = cudaFuncSetAttribute(k_cube_encode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_boxes, p.splits);
    k_cube_encode<<<grid, kQCompute + 32, smem, st>>>(tm_x, p);
    return cudaGetLastError();
}

}  // namespace dq
