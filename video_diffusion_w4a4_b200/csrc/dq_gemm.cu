// Tensor-core products of the DeltaQuant layer on tcgen05 (sm_100a).
//
// DeltaQuant note (papernotes.org), key design 4, Eq. 2/3:
//   Y = Q4(delta) Q4(R)  +  broadcast_cube(Q8(kernel) Q4(R))  +  X L1 L2
//
//   (c) kernel-token product: P'[k][o] = s8_k S_W sum_c q8[k][c] (q s_b)[o][c].
//       Both operands (the E4M3 kernel tokens and the dequantised weight
//       q*s_b) are exact in BF16, so it runs as kind::f16 (BF16 x BF16 -> fp32).
//       No FP8 tensor-core kind takes E4M3 group-16 weight scales.
//   (b) main product: acc[rho][o] = sum_c (q s)_delta (q s)_R with
//       kind::mxf4nvf4 block-16 scaled FP4 MMAs, then the low-rank
//       up-projection as extra BF16 K-steps [U_hi | U_lo] x [L2^T | L2^T] into
//       the same tensor-memory accumulator; the epilogue forms
//       Y[n(rho)][o] = S_delta S_W acc + P'[k(rho)][o] and scatters each
//       cube-major row back to its (t,h,w) position.
//
// One persistent kernel template serves both: one CTA per SM walks the
// 128 x 256 output tiles tile = blockIdx.x + i * gridDim.x.  Warp 0 streams
// operand tiles with TMA into a 4-stage shared-memory ring that runs on across
// tiles; warp 1 owns tensor memory and issues the MMAs from one thread; warp 2
// copies the block scale factors into tensor memory (main product); warps
// 3-10 drain the fp32 accumulator, two warps per 32-lane sub-partition, each
// half of the columns.  The kernel-token product double-buffers its
// accumulator in tensor memory so the epilogue of one tile overlaps the MMAs
// of the next; the main product needs tensor-memory columns for the block
// scale factors (a 48-column slot per ring stage), so it keeps one
// accumulator: its epilogue warps copy their slice of it into registers,
// release tensor memory, and then fetch P' and write Y while the next tile's
// MMAs run.
#include "dq_common.h"
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

namespace {

constexpr int kStages = 4;
constexpr int kTileM = 128, kTileN = 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 96 + 32 * kEpiWarps;   // producer, MMA, scale-factor copies, epilogue
constexpr uint32_t kABytes = kTileM * 128;  // 128 rows x 128 bytes
constexpr uint32_t kBBytes = kTileN * 128;  // 256 rows x 128 bytes
constexpr uint32_t kSFABytes = 4 * 512;     // 128 rows x 4 k-steps of 64
constexpr uint32_t kSFBBytes = 2 * 4 * 512; // 256 rows x 4 k-steps

struct GSmem {
    uint32_t a, b, sfa, sfb, bars, misc, total;
};

__host__ __device__ constexpr GSmem g_smem_layout(bool scaled) {
    GSmem L{};
    uint32_t off = 0;
    L.a = off;
    off += kStages * kABytes;
    L.b = off;
    off += kStages * kBBytes;
    L.sfa = off;
    if (scaled) off += kStages * kSFABytes;
    L.sfb = off;
    if (scaled) off += kStages * kSFBBytes;
    L.bars = off;
    off += (3 * kStages + 6) * 8;
    L.misc = off;
    off += 64;
    L.total = off;
    return L;
}

__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

}  // namespace

template <bool kMain>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_sa, const __grid_constant__ CUtensorMap tm_sb, GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr GSmem L = g_smem_layout(kMain);
    constexpr int kBufs = kMain ? 1 : 2;
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kStages;
    uint64_t* accf = empty + kStages;   // [2]
    uint64_t* acce = accf + 2;          // [2]
    uint64_t* drain = acce + 2;
    uint64_t* drain_sf = drain + 1;
    uint64_t* sfready = drain_sf + 1;   // [kStages]: block scales of a stage are in tensor memory
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int num_n = p.Nout / kTileN;
    const int num_tiles = (int)cdiv(p.M, kTileM) * num_n;
    const int nk = p.k_stages, ntot = p.k_stages + p.slab_stages;

    if (tid == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kMain ? 2 : 1);   // main: MMA commit + scale-copy commit
            mbar_init(&sfready[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 32 * kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(drain_sf, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
            if (kMain) {
                prefetch_tmap(&tm_sa);
                prefetch_tmap(&tm_sb);
            }
            const int kgroups = p.Ci / 64;
            long long g = 0;
            bool alive = true;
            for (int tile = blockIdx.x; alive && tile < num_tiles; tile += gridDim.x) {
                const int m0 = (tile / num_n) * kTileM, n0 = (tile % num_n) * kTileN;
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % kStages);
                    if (g >= kStages &&
                        !mbar_wait(&empty[s], (uint32_t)((g / kStages) - 1) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    if (!kMain) {
                        mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
                        tma_load_2d(sm + L.a + s * kABytes, &tm_a, &full[s], i * 64, m0);
                        tma_load_2d(sm + L.b + s * kBBytes, &tm_b, &full[s], i * 64, n0);
                    } else if (i < nk) {
                        mbar_arrive_expect_tx(&full[s], kABytes + kBBytes + kSFABytes + kSFBBytes);
                        tma_load_2d(sm + L.a + s * kABytes, &tm_a, &full[s], i * 128, m0);
                        tma_load_2d(sm + L.b + s * kBBytes, &tm_b, &full[s], i * 128, n0);
                        bulk_load(sm + L.sfa + s * kSFABytes, p.sfa + ((size_t)(m0 >> 7) * kgroups + 4 * i) * 512,
                                  kSFABytes, &full[s]);
#pragma unroll
                        for (int h = 0; h < 2; h++)
                            bulk_load(sm + L.sfb + s * kSFBBytes + h * (kSFBBytes / 2),
                                      p.sfb + ((size_t)((n0 >> 7) + h) * kgroups + 4 * i) * 512, kSFBBytes / 2,
                                      &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
                        tma_load_2d(sm + L.a + s * kABytes, &tm_sa, &full[s], (i - nk) * 64, m0);
                        tma_load_2d(sm + L.b + s * kBBytes, &tm_sb, &full[s], (i - nk) * 64, n0);
                    }
                }
            }
            // every issued load lands before shared memory is released
            for (long long q = (g > kStages ? g - kStages : 0); q < g; q++)
                mbar_wait(&full[q % kStages], (uint32_t)(q / kStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_main = kMain ? idesc_nvfp4(kTileM, kTileN) : idesc_bf16(kTileM, kTileN);
            const uint32_t id_slab = idesc_bf16(kTileM, kTileN);
            // block scales: one 48-column slot per ring stage (16 SFA + 32 SFB columns),
            // so the copies for one stage never wait on the MMAs still reading another
            const uint32_t t_sf0 = tmem + 256;
            long long g = 0;
            int it = 0;
            bool alive = true;
            for (int tile = blockIdx.x; alive && tile < num_tiles; tile += gridDim.x, it++) {
                const int buf = it % kBufs, use = it / kBufs;
                const uint32_t acc = tmem + (uint32_t)(buf * 256);
                if (use > 0 && !mbar_wait(&acce[buf], (uint32_t)(use - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                tc_fence_after();
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % kStages);
                    if (!mbar_wait(&full[s], (uint32_t)(g / kStages) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aa = smem_u32(sm + L.a + s * kABytes), bb = smem_u32(sm + L.b + s * kBBytes);
                    if (kMain && i < nk) {
                        const uint32_t t_sfa = t_sf0 + (uint32_t)(s * 48), t_sfb = t_sfa + 16;
                        if (!mbar_wait(&sfready[s], (uint32_t)(g / kStages) & 1, abort_flag, p.status, p.budget_ns)) {
                            alive = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; k++)
                            mma_nvfp4(acc, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), id_main,
                                      t_sfa + 4 * k, t_sfb + 8 * k, (i | k) != 0);
                    } else {
                        const uint32_t id = kMain ? id_slab : id_main;
#pragma unroll
                        for (int k = 0; k < 4; k++)
                            mma_bf16(acc, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), id,
                                     (kMain || (i | k) != 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (alive) tc_commit(&accf[buf]);
            }
            // no MMA may still run when tensor memory is released
            tc_commit(drain);
            mbar_wait(drain, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ block-scale copies (main product)
        // Copies each stage's scale factors from shared into tensor memory (its own
        // 48-column slot) from a thread of its own, so the copies run ahead of the
        // MMAs instead of sitting in the MMA thread's in-order stream.
        if (kMain && lane == 0) {
            const uint32_t t_sf0 = tmem + 256;
            long long g = 0;
            bool alive = true;
            for (int tile = blockIdx.x; alive && tile < num_tiles; tile += gridDim.x) {
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % kStages);
                    if (!mbar_wait(&full[s], (uint32_t)(g / kStages) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    if (i < nk) {
                        const uint32_t t_sfa = t_sf0 + (uint32_t)(s * 48), t_sfb = t_sfa + 16;
                        const uint32_t fa = smem_u32(sm + L.sfa + s * kSFABytes);
                        const uint32_t fb = smem_u32(sm + L.sfb + s * kSFBBytes);
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            tmem_cp_32x128b_x4(t_sfa + 4 * k, desc_sf(fa + 512 * k));
                            tmem_cp_32x128b_x4(t_sfb + 8 * k, desc_sf(fb + 512 * k));
                            tmem_cp_32x128b_x4(t_sfb + 8 * k + 4, desc_sf(fb + kSFBBytes / 2 + 512 * k));
                        }
                    }
                    tc_commit(&sfready[s]);
                    tc_commit(&empty[s]);
                }
            }
            // no copy may still run when tensor memory is released
            tc_commit(drain_sf);
            mbar_wait(drain_sf, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue warps
        const int quad = warp & 3, half = (warp - 3) >> 2;
        const float S_W = reinterpret_cast<const PackedHeader*>(p.packed_w)->S_W;
        const float SS = kMain ? __fmul_rn(__uint_as_float(p.scalars[1]), S_W) : 0.f;
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, it++) {
            const int buf = it % kBufs, use = it / kBufs;
            const int m0 = (tile / num_n) * kTileM, n0 = (tile % num_n) * kTileN;
            const long long rho = (long long)m0 + quad * 32 + lane;
            const bool row_ok = rho < p.M;
            const int c_base = n0 + half * 128;
            const uint32_t tacc = tmem + (uint32_t)(buf * 256) + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * 128);
            if (kMain) {
                // Pull this warp's 128-column slice of the accumulator into registers and
                // release tensor memory at once, so the next tile's MMAs start while this
                // tile's P' rows are fetched and its Y rows are written.
                long long n = 0, k = 0;
                if (row_ok) row_to_token(p.g, rho, &n, &k);
                const bool ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], (uint32_t)use & 1, abort_flag,
                                                                  p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                uint32_t acc[128];
#pragma unroll
                for (int c = 0; c < 128; c += 16)
                    tmem_ld_x16(tacc + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(&acc[c]));
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acce[buf]);
                if (row_ok) {
                    const float4* prow = reinterpret_cast<const float4*>(p.p + (size_t)k * p.Nout + c_base);
                    uint16_t* yrow = p.Y + (size_t)n * p.Nout + c_base;
                    float4 pa[8], pb[8];
#pragma unroll
                    for (int v = 0; v < 8; v++) pa[v] = __ldg(prow + v);
#pragma unroll
                    for (int c = 0; c < 128; c += 32) {
                        // software pipeline: the next 32 columns of P' are in flight while these are used
                        if (c + 32 < 128) {
#pragma unroll
                            for (int v = 0; v < 8; v++) pb[v] = __ldg(prow + (c + 32) / 4 + v);
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int v = 0; v < 32; v += 2) {
                            const float4 q = pa[v / 4];
                            const float a0 = (v & 2) ? q.z : q.x, a1 = (v & 2) ? q.w : q.y;
                            pk[v / 2] = (uint32_t)f32_to_bf16_rn(fmaf(SS, __uint_as_float(acc[c + v]), a0)) |
                                        ((uint32_t)f32_to_bf16_rn(fmaf(SS, __uint_as_float(acc[c + v + 1]), a1))
                                         << 16);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(yrow + c);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
                        dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
#pragma unroll
                        for (int v = 0; v < 8; v++) pa[v] = pb[v];
                    }
                }
                continue;   // tensor memory already released
            } else {
                const float scale = row_ok ? __fmul_rn(p.s8[rho], S_W) : 0.f;
                const bool ok = __all_sync(0xffffffffu, mbar_wait(&accf[buf], (uint32_t)use & 1, abort_flag,
                                                                  p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                float* dst = p.pout + (size_t)rho * p.Nout + c_base;
#pragma unroll
                for (int c = 0; c < 128; c += 32) {
                    uint32_t r0[16], r1[16];
                    tmem_ld_x16(tacc + (uint32_t)c, r0);
                    tmem_ld_x16(tacc + (uint32_t)c + 16, r1);
                    tmem_ld_wait();
                    if (row_ok) {
#pragma unroll
                        for (int v = 0; v < 16; v += 4) {
                            *reinterpret_cast<float4*>(dst + c + v) =
                                make_float4(__uint_as_float(r0[v]) * scale, __uint_as_float(r0[v + 1]) * scale,
                                            __uint_as_float(r0[v + 2]) * scale, __uint_as_float(r0[v + 3]) * scale);
                            *reinterpret_cast<float4*>(dst + c + 16 + v) =
                                make_float4(__uint_as_float(r1[v]) * scale, __uint_as_float(r1[v + 1]) * scale,
                                            __uint_as_float(r1[v + 2]) * scale, __uint_as_float(r1[v + 3]) * scale);
                        }
                    }
                }
            }
            // tensor-memory buffer free for the next tile
            tc_fence_before();
            mbar_arrive(&acce[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ launchers

namespace {
int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}
}  // namespace

cudaError_t launch_kernel_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmParams& p,
                               cudaStream_t st) {
    constexpr size_t smem = g_smem_layout(false).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (int)cdiv(p.M, kTileM) * (p.Nout / kTileN);
    k_gemm<false><<<imin(tiles, sm_count()), kThreads, smem, st>>>(tm_a, tm_b, tm_a, tm_b, p);
    return cudaGetLastError();
}

cudaError_t launch_main_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                             const CUtensorMap& tm_sb, const GemmParams& p, cudaStream_t st) {
    constexpr size_t smem = g_smem_layout(true).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (int)cdiv(p.M, kTileM) * (p.Nout / kTileN);
    k_gemm<true><<<imin(tiles, sm_count()), kThreads, smem, st>>>(tm_a, tm_b, tm_sa, tm_sb, p);
    return cudaGetLastError();
}

}  // namespace dq
