// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor/bulk copies,
// tcgen05 tensor-memory allocation, MMA, copies and loads, and the format
// conversions the quantisers use.  Every wait on an mbarrier is bounded: when
// the budget (in ns of %globaltimer) runs out the wait records
// DQ_ERR_DEVICE_TIMEOUT in the caller's status word, raises the CTA's abort
// flag and returns false, so that no kernel of this library can spin forever.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dq {

constexpr int kStatusTimeout = 6;     // DQ_ERR_DEVICE_TIMEOUT
constexpr int kStatusBadWeight = 7;   // DQ_ERR_BAD_PACKED_WEIGHT

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may sleep up to `suspend_ns` for the phase
// to complete (it wakes as soon as it does), instead of returning at once and
// spending issue slots on polling.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t suspend_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(suspend_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of `bar`.  Returns false on timeout or, when
// check_abort is set, as soon as another role of the CTA has given up (abort
// flag raised).  Drain waits at teardown pass check_abort = false so that
// copies already in flight land before shared memory is released.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t budget_ns, bool check_abort = true) {
    uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
        if (check_abort && *abort_flag) return false;
        if (globaltimer() - t0 > budget_ns) {
            *abort_flag = 1;
            if (status) atomicCAS(status, 0, kStatusTimeout);
            return false;
        }
    }
}

// Bounded wait that polls without a suspend hint, for the products' stage and accumulator
// hand-offs, where the wake-up of a suspended wait showed in the step time (about 1 %).
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                               uint64_t budget_ns) {
    uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    uint64_t t0 = globaltimer();
    for (uint32_t n = 1;; n++) {
        if (mbar_try_wait(b, parity)) return true;
        if ((n & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > budget_ns) {
                *abort_flag = 1;
                if (status) atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Commit all prior tcgen05 async operations of this thread to an mbarrier.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format).
//   start address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29,
//   stride byte offset >> 4 in 32-45, version 1 in bits 46-47,
//   layout (swizzle) type in bits 61-63: 0 none, 2 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7) << 61;
    return d;
}

// K-major operand tile with 128-byte rows and the 128-byte swizzle
// (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }

// Instruction descriptor, kind::f16: BF16 x BF16 -> fp32, K-major A and B.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                    // D = fp32
           | (1u << 7)                  // A = BF16
           | (1u << 10)                 // B = BF16
           | ((uint32_t)(N >> 3) << 17) //
           | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor, kind::mxf4nvf4 with block-16 E4M3 scales:
// E2M1 x E2M1 -> fp32, K-major, scale-factor ids 0.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N) {
    return (1u << 7)                    // A = E2M1
           | (1u << 10)                 // B = E2M1
           | ((uint32_t)(N >> 3) << 17) //
           | (0u << 23)                 // scale format E4M3
           | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ CTA pairs (cluster of two)
//
// The paired products run one tile per cluster of two CTAs: both CTAs stage
// half of the operands in their own shared memory, the even CTA (rank 0)
// issues the tcgen05 instructions for both, and the operand copies of both
// CTAs signal barriers that live in rank 0.

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address in the shared::cluster window of the variable at shared address
// `saddr` in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Tensor copies into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (given by its shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

// L2 eviction policies for cache-hinted copies: operands reused by many tiles
// (the weights) are kept, operands streamed once are evicted first.
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d_pair_hint(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                      int y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Tensor-memory allocation shared by the pair: the same warp of both CTAs
// issues it and both receive the same columns.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Completion of this thread's paired tcgen05 operations: one arrival on the
// barrier at `bar` in this CTA ...
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// ... or one arrival on the barrier at the same shared-memory offset in each CTA of `cta_mask`.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// 128 rows x 256 bits (8 columns per lane, no replication) from each CTA's
// shared memory at `sdesc` to its own tensor memory at `taddr`.
__device__ __forceinline__ void tmem_cp_pair_128x256b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Paired MMAs: M = 256 rows, 128 in each CTA's tensor memory; A and B are read
// at the same shared-memory offsets in both CTAs (each holds half of B's rows).
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_nvfp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Paired block-scaled FP8 MMA (kind::mxf8f6f4, E4M3 x E4M3, one UE8M0 scale per 32 K of each row;
// the instruction descriptor's scale-factor ids pick the byte of the 32-bit tensor-memory word).
__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Instruction descriptor, kind::mxf8f6f4: E4M3 x E4M3 -> fp32, K-major, K = 32, UE8M0 scales; the
// MMA reads byte sf_a / sf_b of each scale word.
__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, uint32_t sf_a, uint32_t sf_b) {
    return ((sf_b & 3u) << 4)           // B scale-factor byte
           | (0u << 7)                  // A = E4M3
           | (0u << 10)                 // B = E4M3
           | ((uint32_t)(N >> 3) << 17) //
           | (1u << 23)                 // scale format UE8M0
           | ((uint32_t)(M >> 4) << 24) //
           | ((sf_a & 3u) << 29);       // A scale-factor byte
}

// Each thread of the warp writes four consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v0), "r"(v1),
                 "r"(v2), "r"(v3)
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ 256-bit global access (sm_100)

// Eight fp32 from 32-byte aligned global memory through the non-coherent path.
__device__ __forceinline__ void ld_global_nc_v8(const float* src, float (&v)[8]) {
    asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(src));
}

__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t (&v)[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Streaming store (evict-first in the caches): results no kernel re-reads soon.
__device__ __forceinline__ void st_global_cs_v8(void* dst, const uint32_t (&v)[8]) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// ------------------------------------------------------------------ named barriers

__device__ __forceinline__ void bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ formats

// Two fp32 -> two E4M3 codes, round to nearest even, saturating; `lo` lands in
// the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> two E2M1 codes in one byte, round to nearest even, saturating;
// `lo` lands in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// E4M3 code -> fp32 value (exact) through the half-precision pair conversion.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t c = (uint16_t)(code & 0xFF);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    __half_raw hr;
    hr.x = (uint16_t)(h2 & 0xFFFF);
    return __half2float(__half(hr));
}

// Two E4M3 codes (the low byte of `codes` first) -> their values as a BF16 pair
// (low code in the low half).  Exact: E4M3 values have at most four significant
// bits and lie in BF16's range; f16 holds them exactly on the way.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t codes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(codes & 0xFFFFu)));
    __half_raw lo, hi;
    lo.x = (uint16_t)(h2 & 0xFFFFu);
    hi.x = (uint16_t)(h2 >> 16);
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__half2float(__half(hi))), "f"(__half2float(__half(lo))));
    return r;
}

// fl32(a / b) for b > 0 from rb = fl32(1 / b): one product and one FMA
// correction step (Markstein), which returns the correctly rounded quotient
// when rb is the correctly rounded reciprocal; the result takes a's sign, as
// IEEE division by a positive b does (also for a = -0 and for underflow).
__device__ __forceinline__ float div_pos(float a, float b, float rb) {
    float q = __fmul_rn(a, rb);
    float r = __fmaf_rn(-q, b, a);
    q = __fmaf_rn(r, rb, q);
    return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(a) & 0x80000000u));
}

// -fl32(a / b) for b > 0 from rb = fl32(1 / b): the same Markstein step as
// div_pos with every operand of the correction negated, which returns the
// correctly rounded quotient negated, zero quotients included (-(+0) for
// a = +0, -(-0) for a = -0) without a sign fix-up.  Valid while the quotient
// does not underflow.
__device__ __forceinline__ float div_neg(float a, float b, float rb) {
    const float q = __fmul_rn(a, rb);
    const float r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(-r, rb, -q);
}

// ------------------------------------------------------------------ packed fp32 pairs
//
// sm_100 executes add / sub / mul / fma on two fp32 values held in one 64-bit
// register pair, each correctly rounded as the scalar instruction would be.

__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// a * b + c, one rounding per element
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// The two BF16 values of a 32-bit word (low half first) as an exact fp32 pair.
__device__ __forceinline__ uint64_t f2_from_bf16x2(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// -fl32(a / b) for both elements of the pair a, b > 0 the same for both,
// b2 = (b, b), nrb2 = (-rb, -rb) with rb = fl32(1 / b).  With p = a (-rb) =
// -fl32(a rb), r = p b + a (exact) and p + r (-rb), every rounding is the one
// of div_neg, so the result is div_neg's bit for bit (zero quotients keep
// their sign the same way).
__device__ __forceinline__ uint64_t f2_div_neg(uint64_t a, uint64_t b2, uint64_t nrb2) {
    const uint64_t p = f2_mul(a, nrb2);
    const uint64_t r = f2_fma(p, b2, a);
    return f2_fma(r, nrb2, p);
}

// max(|a|, |b|, |c|)
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

// Eight fp32 -> eight E2M1 codes in one word (value 2i in the low nibble of
// byte i), round to nearest even, saturating.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// 1 / cnt for a power of two cnt (exact)
__device__ __forceinline__ float inv_pow2(int cnt) { return __int_as_float((127 - (31 - __clz(cnt))) << 23); }

// The cube mean from its fp32 running sum (Eq. 1): the sum divided by the token count, the
// division being an exact multiplication when the count is a power of two.
__device__ __forceinline__ float mean_of_sum(float s, int cnt) {
    return (cnt & (cnt - 1)) == 0 ? __fmul_rn(s, inv_pow2(cnt)) : __fdiv_rn(s, (float)cnt);
}

// GELU(y) = y Phi(y), Phi(y) = 1 - erfc(y / sqrt 2) / 2 for y >= 0 and erfc(-y / sqrt 2) / 2 for y < 0, with
// erfc(x) = t (a1 + a2 t + a3 t^2 + a4 t^3 + a5 t^4) exp(-x^2), t = 1 / (1 + p x), x >= 0: the rational
// approximation of Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26 (absolute error
// at most 1.5e-7), in fp32 with the hardware's approximate reciprocal and base-2 exponential:
// |GELU error| <= 3e-7 max(1, |y|), far below the BF16 rounding of the result.  Two values at once in
// packed f32x2 arithmetic.
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ uint64_t gelu_erf2(uint64_t y2) {
    float y0, y1, d0, d1, q0, q1, a0, a1, b0, b1;
    f2_unpack(y2, y0, y1);
    const uint64_t x2 = f2_mul(f2_pack(fabsf(y0), fabsf(y1)), f2_pack(0.70710678118654752f, 0.70710678118654752f));
    f2_unpack(f2_fma(f2_pack(0.3275911f, 0.3275911f), x2, f2_pack(1.0f, 1.0f)), d0, d1);
    const uint64_t t2 = f2_pack(rcp_approx(d0), rcp_approx(d1));
    uint64_t P = f2_fma(f2_pack(1.061405429f, 1.061405429f), t2, f2_pack(-1.453152027f, -1.453152027f));
    P = f2_fma(P, t2, f2_pack(1.421413741f, 1.421413741f));
    P = f2_fma(P, t2, f2_pack(-0.284496736f, -0.284496736f));
    P = f2_fma(P, t2, f2_pack(0.254829592f, 0.254829592f));
    // exp(-x^2) = 2^(-x^2 log2 e)
    f2_unpack(f2_mul(f2_mul(x2, x2), f2_pack(-1.4426950408889634f, -1.4426950408889634f)), q0, q1);
    const uint64_t e2 = f2_mul(f2_mul(t2, P), f2_pack(ex2_approx(q0), ex2_approx(q1)));   // erfc(x)
    f2_unpack(f2_fma(f2_pack(-0.5f, -0.5f), e2, f2_pack(1.0f, 1.0f)), a0, a1);             // 1 - erfc / 2
    f2_unpack(f2_mul(f2_pack(0.5f, 0.5f), e2), b0, b1);                                      // erfc / 2
    return f2_mul(y2, f2_pack(y0 >= 0.f ? a0 : b0, y1 >= 0.f ? a1 : b1));
}

// Two fp32 -> BF16 (round to nearest even) in one word, the first in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

}  // namespace dq
