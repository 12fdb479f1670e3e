// Tensor-core products of the DeltaQuant layer on tcgen05 (sm_100a).
//
// DeltaQuant note (papernotes.org), key design 4, Eq. 2/3:
//   Y = Q4(delta) Q4(R)  +  broadcast_cube(Q8(kernel) Q4(R))  +  X L1 L2
//
//   (c) k_kernel_gemm: P'[k][o] = s8_k S_W sum_c q8[k][c] (q s_b)[o][c].  The
//       operands are the E4M3 kernel tokens and the dequantised weight q*s_b,
//       both exact in BF16, so the product runs as kind::f16 (BF16 x BF16 ->
//       fp32).  (No FP8 tensor-core kind takes E4M3 group-16 weight scales.)
//   (b) k_main_gemm: acc[rho][o] = sum_c (q s)_delta (q s)_R with
//       kind::mxf4nvf4 block-16 scaled FP4 MMAs, then the low-rank
//       up-projection as extra BF16 K-steps [U_hi | U_lo] x [L2^T | L2^T] into
//       the same tensor-memory accumulator; the epilogue forms
//       Y[n(rho)][o] = S_delta S_W acc + P'[k(rho)][o] and scatters each
//       cube-major row back to its (t,h,w) position.
//
// Structure (both): one 128 x 256 output tile per CTA; warp 0 issues TMA
// loads into a 4-stage shared-memory ring, warp 1 owns tensor memory and
// issues the MMAs from one thread, warps 2-5 drain the fp32 accumulator from
// tensor memory (each warp its 32-lane sub-partition).  All waits are bounded.
#include "dq_common.h"
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

namespace {

constexpr int kStages = 4;
constexpr int kTileM = 128, kTileN = 256;
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
    off += (2 * kStages + 2) * 8;
    L.misc = off;
    off += 64;
    L.total = off;
    return L;
}

__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

}  // namespace

// ------------------------------------------------------------------ (c) kernel-token product

__global__ void __launch_bounds__(192, 1) k_kernel_gemm(const __grid_constant__ CUtensorMap tm_a,
                                                         const __grid_constant__ CUtensorMap tm_b, GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr GSmem L = g_smem_layout(false);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kStages;
    uint64_t* accf = empty + kStages;
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * kTileN, m0 = blockIdx.y * kTileM;
    const int nk = p.k_stages;

    if (tid == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
            int issued = 0;
            for (int i = 0; i < nk; i++) {
                int s = i % kStages;
                if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
                tma_load_2d(sm + L.a + s * kABytes, &tm_a, &full[s], i * 64, m0);
                tma_load_2d(sm + L.b + s * kBBytes, &tm_b, &full[s], i * 64, n0);
                issued = i + 1;
            }
            for (int i = (issued > kStages ? issued - kStages : 0); i < issued; i++)
                mbar_wait(&full[i % kStages], (i / kStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kTileM, kTileN);
            for (int i = 0; i < nk; i++) {
                int s = i % kStages;
                if (!mbar_wait(&full[s], (i / kStages) & 1, abort_flag, p.status, p.budget_ns)) break;
                tc_fence_after();
                uint32_t aa = smem_u32(sm + L.a + s * kABytes), bb = smem_u32(sm + L.b + s * kBBytes);
#pragma unroll
                for (int k = 0; k < 4; k++)
                    mma_bf16(tmem, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), idesc, (i | k) != 0);
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
            mbar_wait(accf, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // epilogue: P'[m][n] = s8[m] S_W acc
        const int quad = warp & 3;
        const int row = m0 + quad * 32 + lane;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag, p.status, p.budget_ns));
        tc_fence_after();
        if (ok) {
            const float sw = reinterpret_cast<const PackedHeader*>(p.packed_w)->S_W;
            const float scale = (row < p.M) ? __fmul_rn(p.s8[row], sw) : 0.f;
            float* dst = p.pout + (size_t)row * p.Nout + n0;
            for (int c = 0; c < kTileN; c += 16) {
                uint32_t r[16];
                tmem_ld_x16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c, r);
                tmem_ld_wait();
                if (row < p.M) {
#pragma unroll
                    for (int v = 0; v < 16; v += 4)
                        *reinterpret_cast<float4*>(dst + c + v) =
                            make_float4(__uint_as_float(r[v]) * scale, __uint_as_float(r[v + 1]) * scale,
                                        __uint_as_float(r[v + 2]) * scale, __uint_as_float(r[v + 3]) * scale);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ (b) main product

__global__ void __launch_bounds__(192, 1) k_main_gemm(const __grid_constant__ CUtensorMap tm_a,
                                                       const __grid_constant__ CUtensorMap tm_b,
                                                       const __grid_constant__ CUtensorMap tm_sa,
                                                       const __grid_constant__ CUtensorMap tm_sb, GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr GSmem L = g_smem_layout(true);
    uint64_t* full = (uint64_t*)(sm + L.bars);
    uint64_t* empty = full + kStages;
    uint64_t* accf = empty + kStages;
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * kTileN, m0 = blockIdx.y * kTileM;
    const int nk = p.k_stages, ntot = p.k_stages + p.slab_stages;
    const int kgroups = p.Ci / 64;

    if (tid == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
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
    const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 272;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
            prefetch_tmap(&tm_sa);
            prefetch_tmap(&tm_sb);
            int issued = 0;
            for (int i = 0; i < ntot; i++) {
                int s = i % kStages;
                if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                if (i < nk) {
                    mbar_arrive_expect_tx(&full[s], kABytes + kBBytes + kSFABytes + kSFBBytes);
                    tma_load_2d(sm + L.a + s * kABytes, &tm_a, &full[s], i * 128, m0);
                    tma_load_2d(sm + L.b + s * kBBytes, &tm_b, &full[s], i * 128, n0);
                    const uint8_t* sa = p.sfa + ((size_t)(m0 >> 7) * kgroups + 4 * i) * 512;
                    bulk_load(sm + L.sfa + s * kSFABytes, sa, kSFABytes, &full[s]);
#pragma unroll
                    for (int g = 0; g < 2; g++) {
                        const uint8_t* sb = p.sfb + ((size_t)((n0 >> 7) + g) * kgroups + 4 * i) * 512;
                        bulk_load(sm + L.sfb + s * kSFBBytes + g * (kSFBBytes / 2), sb, kSFBBytes / 2, &full[s]);
                    }
                } else {
                    mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
                    tma_load_2d(sm + L.a + s * kABytes, &tm_sa, &full[s], (i - nk) * 64, m0);
                    tma_load_2d(sm + L.b + s * kBBytes, &tm_sb, &full[s], (i - nk) * 64, n0);
                }
                issued = i + 1;
            }
            for (int i = (issued > kStages ? issued - kStages : 0); i < issued; i++)
                mbar_wait(&full[i % kStages], (i / kStages) & 1, abort_flag, nullptr, p.budget_ns, false);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id4 = idesc_nvfp4(kTileM, kTileN), id16 = idesc_bf16(kTileM, kTileN);
            for (int i = 0; i < ntot; i++) {
                int s = i % kStages;
                if (!mbar_wait(&full[s], (i / kStages) & 1, abort_flag, p.status, p.budget_ns)) break;
                tc_fence_after();
                uint32_t aa = smem_u32(sm + L.a + s * kABytes), bb = smem_u32(sm + L.b + s * kBBytes);
                if (i < nk) {
                    uint32_t fa = smem_u32(sm + L.sfa + s * kSFABytes), fb = smem_u32(sm + L.sfb + s * kSFBBytes);
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        tmem_cp_32x128b_x4(t_sfa + 4 * k, desc_sf(fa + 512 * k));
                        tmem_cp_32x128b_x4(t_sfb + 8 * k, desc_sf(fb + 512 * k));
                        tmem_cp_32x128b_x4(t_sfb + 8 * k + 4, desc_sf(fb + kSFBBytes / 2 + 512 * k));
                    }
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        mma_nvfp4(tmem, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), id4, t_sfa + 4 * k,
                                  t_sfb + 8 * k, (i | k) != 0);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; k++)
                        mma_bf16(tmem, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), id16, 1u);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
            mbar_wait(accf, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // epilogue: Y[n][o] = bf16(S_delta S_W acc + P'[k][o]), row scattered to (t,h,w) order
        const int quad = warp & 3;
        const long long rho = (long long)m0 + quad * 32 + lane;
        const bool row_ok = rho < p.M;
        long long n = 0, k = 0;
        if (row_ok) row_to_token(p.g, rho, &n, &k);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, abort_flag, p.status, p.budget_ns));
        tc_fence_after();
        if (ok) {
            const float SS =
                __fmul_rn(__uint_as_float(p.scalars[1]), reinterpret_cast<const PackedHeader*>(p.packed_w)->S_W);
            const float* prow = p.p + (size_t)k * p.Nout + n0;
            uint16_t* yrow = p.Y + (size_t)n * p.Nout + n0;
            for (int c = 0; c < kTileN; c += 16) {
                uint32_t r[16];
                tmem_ld_x16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c, r);
                tmem_ld_wait();
                if (row_ok) {
                    uint32_t packed[8];
#pragma unroll
                    for (int v = 0; v < 16; v += 4) {
                        float4 pv = *reinterpret_cast<const float4*>(prow + c + v);
                        float y0 = fmaf(SS, __uint_as_float(r[v]), pv.x);
                        float y1 = fmaf(SS, __uint_as_float(r[v + 1]), pv.y);
                        float y2 = fmaf(SS, __uint_as_float(r[v + 2]), pv.z);
                        float y3 = fmaf(SS, __uint_as_float(r[v + 3]), pv.w);
                        packed[v / 2] = (uint32_t)f32_to_bf16_rn(y0) | ((uint32_t)f32_to_bf16_rn(y1) << 16);
                        packed[v / 2 + 1] = (uint32_t)f32_to_bf16_rn(y2) | ((uint32_t)f32_to_bf16_rn(y3) << 16);
                    }
                    reinterpret_cast<uint4*>(yrow + c)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    reinterpret_cast<uint4*>(yrow + c)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                }
            }
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

cudaError_t launch_kernel_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmParams& p,
                               cudaStream_t st) {
    constexpr size_t smem = g_smem_layout(false).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_kernel_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.Nout / kTileN, (unsigned)cdiv(p.M, kTileM));
    k_kernel_gemm<<<grid, 192, smem, st>>>(tm_a, tm_b, p);
    return cudaGetLastError();
}

cudaError_t launch_main_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                             const CUtensorMap& tm_sb, const GemmParams& p, cudaStream_t st) {
    constexpr size_t smem = g_smem_layout(true).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_main_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.Nout / kTileN, (unsigned)cdiv(p.M, kTileM));
    k_main_gemm<<<grid, 192, smem, st>>>(tm_a, tm_b, tm_sa, tm_sb, p);
    return cudaGetLastError();
}

}  // namespace dq
