// Tensor-core products of the DeltaQuant layer on tcgen05 (sm_100a).
//
// DeltaQuant note (papernotes.org), key design 4, Eq. 2/3:
//   Y = Q4(delta) Q4(R)  +  broadcast_cube(Q8(kernel) Q4(R))  +  X L1 L2
//
//   (c) kernel-token product: P'[k][o] = s8_k S_W sum_c q8[k][c] (q s_b)[o][c] (+ b[o] when the
//       packed weight holds a bias).
//       Both operands (the E4M3 kernel tokens and the dequantised weight
//       q*s_b) are exact in BF16, so it runs as kind::f16 (BF16 x BF16 -> fp32).
//       No FP8 tensor-core kind takes E4M3 group-16 weight scales.
//       With one kernel scale per 64 channels the scale varies along K, so the
//       A operand is q8 s8 itself as BF16 hi + lo (2 Ci columns: every weight
//       k-block is read twice) and P' = S_W acc.
//   (b) main product: acc[rho][o] = sum_c (q s)_delta (q s)_R with
//       kind::mxf4nvf4 block-16 scaled FP4 MMAs, then the low-rank
//       up-projection as extra BF16 K-steps [U_hi | U_lo] x [L2^T | L2^T] into
//       the same tensor-memory accumulator; the epilogue forms
//       Y[n(rho)][o] = S_delta S_W acc + P'[k(rho)][o] and scatters each
//       cube-major row back to its (t,h,w) position.
//
// One persistent kernel template serves both.  A cluster of two CTAs (one per
// SM) owns a 256 x 256 output tile at a time, walking tiles
// tile = cluster + i * clusters.  Each CTA stages 128 rows of A and 128 rows of
// B (half the tile's columns) per K step with TMA into its own shared-memory
// ring, so every operand byte crosses from L2 once per 256 x 256 tile (a
// third less traffic per FLOP than 128 x 256 tiles on one SM).  The even CTA
// issues the paired (cta_group::2) MMAs, which read A and B from both CTAs
// and leave 128 rows of fp32 accumulator in each CTA's tensor memory.  Roles:
// warp 0 of each CTA streams its operand halves; warp 1 of the even CTA issues
// the MMAs; warp 2 of the even CTA copies the block scale factors of both CTAs
// into tensor memory (main product); warps 3-10 of each CTA drain that CTA's
// accumulator rows, two warps per 32-lane sub-partition, each half of the
// columns (warps 3-18, four per sub-partition and a quarter of the columns
// each, for the feed-forward epilogue).  The operand copies of both CTAs count on the even CTA's
// "stage full" barriers; the MMA thread's commits arrive on the "stage empty"
// and "accumulator full" barriers of both CTAs; the epilogue warps of both
// CTAs arrive on the even CTA's "accumulator empty" barrier.
//
//   (c') FP8 kernel-token product (weights packed with DQ_PACK_C2): the same P'
//       from q8 (E4M3) and the FP8 form of q s_b (E4M3 codes times one UE8M0
//       exponent per 32 channels) with kind::mxf8f6f4 MMAs at twice the BF16
//       rate.  Every product q8 * (q s_b) is exact in fp32 either way; the A
//       operand's scales are a constant 1 (UE8M0 127) written to tensor memory
//       once, the B operand's exponents are copied in per 256-channel stage
//       (two 4 KB copies).
//
//   (b') main product with the feed-forward epilogue (kGemmMainFfn, the up-projection of a
//       transformer feed-forward block): Y = BF16(GELU(y)), and optionally the statistics pass of
//       the down-projection over that Y (cube means, max |mean| per cube, max |Y - mean|), so that
//       the down-projection's statistics kernel only forms Y L1.
//
// The BF16 kernel-token product double-buffers its accumulator in tensor memory so
// the epilogue of one tile overlaps the MMAs of the next; the main product
// needs tensor-memory columns for the block scale factors (a 48-column slot
// per ring stage), so it keeps one accumulator: its epilogue warps copy their
// slice into registers, release tensor memory, and then fetch P' and write Y
// while the next tile's MMAs run.  The FP8 kernel-token product does the same
// (a 16-column exponent slot per stage next to one accumulator).
#include <atomic>

#include "dq_common.h"
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

namespace {

constexpr int kTileM = 128;                     // accumulator rows per CTA (256 per pair)
constexpr int kTileN = 256;                     // output columns per pair tile
// Epilogue warps: two per 32-lane sub-partition of tensor memory (128 columns each), four (64 columns
// each) for the feed-forward epilogue, whose GELU and statistics want more warps to hide their latency.
__host__ __device__ constexpr int epi_warps(int kind) { return kind == kGemmMainFfn ? 16 : 8; }
__host__ __device__ constexpr int g_threads(int kind) { return 96 + 32 * epi_warps(kind); }   // + producer, MMA, copies
constexpr uint32_t kABytes = kTileM * 128;      // 128 rows x 128 bytes
constexpr uint32_t kBBytes = (kTileN / 2) * 128;  // this CTA's 128 rows of B x 128 bytes
constexpr uint32_t kSFABytes = 2 * 4096;        // 128 rows x 4 k-blocks of 64, A-operand scale layout
constexpr uint32_t kSFBBytes = 4 * 4096;        // all 256 columns x 4 k-blocks, B-operand scale layout (each CTA)
constexpr uint32_t kSFB8Bytes = 4096;           // FP8 product: UE8M0 exponents of 256 columns x 4 blocks of 32 (per 128 channels)
constexpr uint16_t kPairMask = 0x3;
constexpr uint32_t kFp8SfaCol = 256;            // FP8 product: tensor-memory columns of the constant A scales
constexpr uint32_t kFp8SfbCol = 264;            //   and of the first B-exponent slot (16 columns per stage)

__host__ __device__ constexpr bool is_main(int kind) { return kind == kGemmMain || kind == kGemmMainFfn; }

__host__ __device__ constexpr int g_stages(int kind) {
    return is_main(kind) ? 4 : 3;
}
// Operand tiles per stage: the kernel-token products stage two 128-byte-row boxes of each operand
// (128 channels of BF16, 256 of FP8; eight MMAs) between barrier hand-offs, measured 6-8 % faster
// than one box per stage with twice the stages; the main product keeps one (its scale copies and
// TMEM slots are per box).
__host__ __device__ constexpr uint32_t stage_mul(int kind) { return is_main(kind) ? 1u : 2u; }

// Output tile -> (row tile, column tile).  group <= 1: row-major, which suits a weight that stays
// in L2 while the row tiles stream.  Otherwise groups of `group` row tiles walked column by column:
// a wave of CTA pairs then touches `group` row tiles and a few column tiles, and each group reads
// the weight once (the host picks this for weights too large to stay in L2 beside the rows).
struct TileRC {
    int m, n;
};

__device__ __forceinline__ TileRC tile_rc(int tile, int num_m, int num_n, int group) {
    if (group <= 1) return TileRC{tile / num_n, tile % num_n};
    const int grp = tile / (group * num_n), in = tile - grp * (group * num_n);
    const int gm = min(group, num_m - grp * group);
    return TileRC{grp * group + in % gm, in / gm};
}

struct GSmem {
    uint32_t a, b, sfa, sfb, bars, misc, total;
};

__host__ __device__ constexpr GSmem g_smem_layout(int kind) {
    GSmem L{};
    const int S = g_stages(kind);
    uint32_t off = 0;
    L.a = off;
    off += S * kABytes * stage_mul(kind);
    L.b = off;
    off += S * kBBytes * stage_mul(kind);
    L.sfa = off;
    if (is_main(kind)) off += S * kSFABytes;
    L.sfb = off;
    if (is_main(kind)) off += S * kSFBBytes;
    if (kind == kGemmKernelFp8) off += S * 2 * kSFB8Bytes;
    L.bars = off;
    off += (3 * S + 6) * 8;
    L.misc = off;
    off += 64;
    L.total = off;
    return L;
}


// Consumer statistics of the feed-forward epilogue (see k_gemm<kGemmMainFfn>) over one warp's 64-column
// slice, held as 32 BF16 pairs pk per lane (lane = row).  Cubes of S tokens on S aligned consecutive lanes,
// rows in cube order: lane li of a cube gathers the 32/S pairs li*32/S.. of every row of its cube (S - 1
// exchange rounds with lane li ^ r, each lane sending the chunk its partner gathers), sums the rows in cube
// order from +0 (the statistics kernel's order), and keeps max |mean| and max |x - mean| of its columns;
// `valid` lanes store their 64/S means at mrow (the slice's first column of the cube's row of means).
template <int S>
__device__ __forceinline__ void ffn_stats_aligned(const uint32_t (&pk)[32], int li, bool valid, float* mrow,
                                                  float& kam, float& dmx) {
    constexpr int W = 32 / S;
    const float inv = inv_pow2(S);
    uint32_t mw[8];
#pragma unroll
    for (int q = 0; q < W; q++) {
        uint32_t v[S];   // v[r]: pair li * W + q of the row li ^ r
#pragma unroll
        for (int r = 0; r < S; r++) {
            const int c = li ^ r;
            uint32_t send = pk[q];
#pragma unroll
            for (int cc = 1; cc < S; cc++) send = (c == cc) ? pk[cc * W + q] : send;
            v[r] = r ? __shfl_xor_sync(0xffffffffu, send, r) : send;
        }
        uint64_t s2 = 0ull;   // (+0, +0)
#pragma unroll
        for (int j = 0; j < S; j++) {
            // row j arrived in round li ^ j
            const int r = li ^ j;
            uint32_t x = v[0];
#pragma unroll
            for (int rr = 1; rr < S; rr++) x = (r == rr) ? v[rr] : x;
            s2 = f2_add(s2, f2_from_bf16x2(x));
        }
        const uint64_t m2 = f2_mul(s2, f2_pack(inv, inv));
        float m0, m1;
        f2_unpack(m2, m0, m1);
        if (valid) {
            kam = max3_abs(m0, m1, kam);
#pragma unroll
            for (int r = 0; r < S; r++) {
                float d0, d1;
                f2_unpack(f2_sub(f2_from_bf16x2(v[r]), m2), d0, d1);
                dmx = max3_abs(d0, d1, dmx);
            }
        }
        mw[(2 * q) & 7] = __float_as_uint(m0);
        mw[(2 * q + 1) & 7] = __float_as_uint(m1);
        if ((q & 3) == 3 && valid) st_global_v8(mrow + 2 * li * W + 2 * (q - 3), mw);
    }
}

}  // namespace

template <int kKind>
__global__ void __launch_bounds__(g_threads(kKind), 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
           const __grid_constant__ CUtensorMap tm_sa, const __grid_constant__ CUtensorMap tm_sb,
           const __grid_constant__ CUtensorMap tm_fa, const __grid_constant__ CUtensorMap tm_fb, GemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr bool kMain = is_main(kKind);          // the main product, with either epilogue
    constexpr bool kFfn = kKind == kGemmMainFfn;    // its feed-forward epilogue
    constexpr bool kFp8 = kKind == kGemmKernelFp8;
    constexpr bool kScaled = kMain || kFp8;      // block scales copied into tensor memory, one accumulator
    constexpr GSmem L = g_smem_layout(kKind);
    constexpr int S = g_stages(kKind);
    constexpr int kBufs = kScaled ? 1 : 2;
    uint64_t* full = (uint64_t*)(sm + L.bars);   // [S], used in the even CTA
    uint64_t* empty = full + S;                  // [S], both CTAs
    uint64_t* sfready = empty + S;               // [S], even CTA: block scales of a stage are in tensor memory
    uint64_t* accf = sfready + S;                // [2], both CTAs
    uint64_t* acce = accf + 2;                   // [2], even CTA
    uint64_t* drain = acce + 2;
    uint64_t* drain_sf = drain + 1;
    uint32_t* tmem_slot = (uint32_t*)(sm + L.misc);
    volatile int* abort_flag = (volatile int*)(sm + L.misc + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();     // 0: issues the MMAs; 1: its peer
    const bool lead = rank == 0;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int num_n = p.Nout / kTileN;
    const int m_lo = p.tile_m0, num_m = p.tile_m1 - p.tile_m0;   // this launch's row tiles
    const int num_tiles = num_m * num_n;
    const int nk = p.k_stages, ntot = p.k_stages + p.slab_stages;

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kScaled ? 2 : 1);   // scaled kinds: MMA commit + scale-copy commit
            mbar_init(&sfready[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 2 * epi_warps(kKind));   // one arrival per epilogue warp of each CTA
        }
        mbar_init(drain, 1);
        mbar_init(drain_sf, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();   // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (kFp8) {
        // the A operand (q8) carries its scale in the epilogue: its MMA scales are 1 (UE8M0 127),
        // written once into four columns of every lane of both CTAs' tensor memory
        if (warp >= 3 && warp < 7) {
            const uint32_t v = 0x7F7F7F7Fu;
            tmem_st_x4(tmem + ((uint32_t)((warp & 3) * 32) << 16) + kFp8SfaCol, v, v, v, v);
            tmem_st_wait();
        }
        tc_fence_before();
        cluster_sync();
        tc_fence_after();
    }

    if (warp == 0) {
        // ------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
            if (kFp8) prefetch_tmap(&tm_fb);
            if (kMain) {
                prefetch_tmap(&tm_sa);
                prefetch_tmap(&tm_sb);
                prefetch_tmap(&tm_fa);
                prefetch_tmap(&tm_fb);
            }
            const uint32_t full0 = mapa_shared(smem_u32(full), 0);
            // the weight-side operands are read by every row tile: keep them in L2
            const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
            long long g = 0;
            bool alive = true;
            for (int tile = pair; alive && tile < num_tiles; tile += npairs) {
                const TileRC rc = tile_rc(tile, num_m, num_n, p.tile_group);
                const int m0 = (m_lo + rc.m) * (2 * kTileM) + (int)rank * kTileM;   // this CTA's A rows
                const int n0 = rc.n * kTileN;                               // the pair's columns
                const int nb = n0 + (int)rank * (kTileN / 2);                         // this CTA's B rows
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % S);
                    if (g >= S && !mbar_wait(&empty[s], (uint32_t)((g / S) - 1) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    const uint32_t fb = full0 + (uint32_t)(s * 8);
                    uint8_t* sa = sm + L.a + s * kABytes * stage_mul(kKind);
                    uint8_t* sb = sm + L.b + s * kBBytes * stage_mul(kKind);
                    if (kFp8) {
                        // 128 channels of q8 and of the FP8 weight, and the stage's 4 KB of exponents
                        if (lead) mbar_arrive_expect_tx(&full[s], 2 * (2 * kABytes + 2 * kBBytes + 2 * kSFB8Bytes));
                        tma_load_2d_pair_hint(sa, &tm_a, fb, i * 256, m0, stream);
                        tma_load_2d_pair_hint(sa + kABytes, &tm_a, fb, i * 256 + 128, m0, stream);
                        tma_load_2d_pair_hint(sb, &tm_b, fb, i * 256, nb, keep);
                        tma_load_2d_pair_hint(sb + kBBytes, &tm_b, fb, i * 256 + 128, nb, keep);
                        tma_load_3d_pair(sm + L.sfb + s * 2 * kSFB8Bytes, &tm_fb, fb, 0, 32 * i, n0 >> 8);
                    } else if (!kMain) {
                        // 128 channels of A (two 64-channel boxes); B's channels are A's modulo Ci
                        // (the grouped-scale operand repeats the weight for its hi and lo halves)
                        if (lead) mbar_arrive_expect_tx(&full[s], 2 * (2 * kABytes + 2 * kBBytes));
                        tma_load_2d_pair_hint(sa, &tm_a, fb, i * 128, m0, stream);
                        tma_load_2d_pair_hint(sa + kABytes, &tm_a, fb, i * 128 + 64, m0, stream);
                        tma_load_2d_pair_hint(sb, &tm_b, fb, (i * 128) % p.Ci, nb, keep);
                        tma_load_2d_pair_hint(sb + kBBytes, &tm_b, fb, (i * 128 + 64) % p.Ci, nb, keep);
                    } else if (i < nk) {
                        if (lead) mbar_arrive_expect_tx(&full[s], 2 * (kABytes + kBBytes + kSFABytes + kSFBBytes));
                        tma_load_2d_pair(sa, &tm_a, fb, i * 128, m0);
                        tma_load_2d_pair(sb, &tm_b, fb, i * 128, nb);
                        // scale factors: A 8192 B per 128-row group and K step (32 lines of 256 B),
                        // B 16384 B per 256-column tile and K step (64 lines)
                        tma_load_3d_pair(sm + L.sfa + s * kSFABytes, &tm_fa, fb, 0, 32 * i, m0 >> 7);
                        tma_load_3d_pair(sm + L.sfb + s * kSFBBytes, &tm_fb, fb, 0, 64 * i, n0 >> 8);
                    } else {
                        if (lead) mbar_arrive_expect_tx(&full[s], 2 * (kABytes + kBBytes));
                        tma_load_2d_pair(sa, &tm_sa, fb, (i - nk) * 64, m0);
                        tma_load_2d_pair(sb, &tm_sb, fb, (i - nk) * 64, nb);
                    }
                }
            }
            // every issued copy lands before shared memory is released: the even CTA
            // waits for its last stages to fill (they count both CTAs' bytes), the odd
            // CTA for the MMAs that consumed its last stages
            for (long long q = (g > S ? g - S : 0); q < g; q++) {
                if (lead)
                    mbar_wait(&full[q % S], (uint32_t)(q / S) & 1, abort_flag, nullptr, p.budget_ns, false);
                else
                    mbar_wait(&empty[q % S], (uint32_t)(q / S) & 1, abort_flag, nullptr, p.budget_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lead && lane == 0) {
            const uint32_t id_main = kMain ? idesc_nvfp4(2 * kTileM, kTileN) : idesc_bf16(2 * kTileM, kTileN);
            const uint32_t id_slab = idesc_bf16(2 * kTileM, kTileN);
            // block scales: one 48-column slot per ring stage (16 SFA + 32 SFB columns),
            // so the copies for one stage never wait on the MMAs still reading another
            const uint32_t t_sf0 = tmem + 256;
            long long g = 0;
            int it = 0;
            bool alive = true;
            for (int tile = pair; alive && tile < num_tiles; tile += npairs, it++) {
                const int buf = it % kBufs, use = it / kBufs;
                const uint32_t acc = tmem + (uint32_t)(buf * 256);
                if (use > 0 && !mbar_wait_spin(&acce[buf], (uint32_t)(use - 1) & 1, abort_flag, p.status, p.budget_ns))
                    break;
                tc_fence_after();
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % S);
                    if (!mbar_wait_spin(&full[s], (uint32_t)(g / S) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aa = smem_u32(sm + L.a + s * kABytes * stage_mul(kKind)), bb = smem_u32(sm + L.b + s * kBBytes * stage_mul(kKind));
                    if (kFp8) {
                        if (!mbar_wait_spin(&sfready[s], (uint32_t)(g / S) & 1, abort_flag, p.status, p.budget_ns)) {
                            alive = false;
                            break;
                        }
                        tc_fence_after();
                        // four MMAs of 32 channels; MMA k reads byte k of the stage's scale words
#pragma unroll
                        for (int k = 0; k < 8; k++)
                            mma_mxf8_pair(acc, desc_k_sw128(aa + (k / 4) * kABytes + 32 * (k % 4)),
                                          desc_k_sw128(bb + (k / 4) * kBBytes + 32 * (k % 4)),
                                          idesc_mxf8(2 * kTileM, kTileN, (uint32_t)(k % 4), (uint32_t)(k % 4)),
                                          tmem + kFp8SfaCol, tmem + kFp8SfbCol + (uint32_t)(16 * s + 8 * (k / 4)),
                                          (i | k) != 0);
                    } else if (kMain && i < nk) {
                        const uint32_t t_sfa = t_sf0 + (uint32_t)(s * 48), t_sfb = t_sfa + 16;
                        if (!mbar_wait_spin(&sfready[s], (uint32_t)(g / S) & 1, abort_flag, p.status, p.budget_ns)) {
                            alive = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; k++)
                            mma_nvfp4_pair(acc, desc_k_sw128(aa + 32 * k), desc_k_sw128(bb + 32 * k), id_main,
                                           t_sfa + 8 * (k >> 1) + 4 * (k & 1), t_sfb + 8 * k, (i | k) != 0);
                    } else {
                        const uint32_t id = kMain ? id_slab : id_main;
#pragma unroll
                        for (int k = 0; k < 4 * (int)stage_mul(kKind); k++)
                            mma_bf16_pair(acc, desc_k_sw128(aa + (k / 4) * kABytes + 32 * (k % 4)),
                                          desc_k_sw128(bb + (k / 4) * kBBytes + 32 * (k % 4)), id,
                                          (kMain || (i | k) != 0) ? 1u : 0u);
                    }
                    tc_commit_pair_both(&empty[s], kPairMask);
                }
                if (alive) tc_commit_pair_both(&accf[buf], kPairMask);
            }
            // no MMA may still run when tensor memory is released
            tc_commit_pair(drain);
            mbar_wait(drain, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ block-scale copies (main product, even CTA)
        // One copy instruction moves each CTA's scale factors from its own shared
        // memory into its own tensor memory; a thread of its own lets the copies
        // run ahead of the MMAs instead of sitting in the MMA thread's stream.
        if (kFp8 && lead && lane == 0) {
            long long g = 0;
            bool alive = true;
            for (int tile = pair; alive && tile < num_tiles; tile += npairs) {
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % S);
                    if (!mbar_wait_spin(&full[s], (uint32_t)(g / S) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    // one copy: lane i of every quadrant gets rows 32 c + i (c = 0..7) of the tile, four
                    // exponent bytes (the stage's four 32-channel blocks) per row
                    tmem_cp_pair_128x256b(tmem + kFp8SfbCol + (uint32_t)(16 * s),
                                          smem_desc(smem_u32(sm + L.sfb + s * 2 * kSFB8Bytes), 128, 256, 0));
                    tmem_cp_pair_128x256b(tmem + kFp8SfbCol + (uint32_t)(16 * s + 8),
                                          smem_desc(smem_u32(sm + L.sfb + s * 2 * kSFB8Bytes + kSFB8Bytes), 128, 256, 0));
                    tc_commit_pair(&sfready[s]);
                    tc_commit_pair_both(&empty[s], kPairMask);
                }
            }
            tc_commit_pair(drain_sf);
            mbar_wait(drain_sf, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        if (kMain && lead && lane == 0) {
            const uint32_t t_sf0 = tmem + 256;
            long long g = 0;
            bool alive = true;
            for (int tile = pair; alive && tile < num_tiles; tile += npairs) {
                for (int i = 0; i < ntot; i++, g++) {
                    const int s = (int)(g % S);
                    if (!mbar_wait_spin(&full[s], (uint32_t)(g / S) & 1, abort_flag, p.status, p.budget_ns)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    if (i < nk) {
                        const uint32_t t_sfa = t_sf0 + (uint32_t)(s * 48), t_sfb = t_sfa + 16;
                        const uint32_t fa = smem_u32(sm + L.sfa + s * kSFABytes);
                        const uint32_t fb = smem_u32(sm + L.sfb + s * kSFBBytes);
                        // A: lane r receives 8 columns per copy, of which the MMA of k-block k reads
                        // column 8 (k / 2) + 4 (k % 2) + r / 32; B: every quadrant needs every column's
                        // scales, and the packed weight holds them once per quadrant, so one copy per
                        // k-block fills all four
                        tmem_cp_pair_128x256b(t_sfa, smem_desc(fa, 128, 256, 0));
                        tmem_cp_pair_128x256b(t_sfa + 8, smem_desc(fa + 4096, 128, 256, 0));
#pragma unroll
                        for (int k = 0; k < 4; k++) tmem_cp_pair_128x256b(t_sfb + 8 * k, smem_desc(fb + 4096 * k, 128, 256, 0));
                    }
                    tc_commit_pair(&sfready[s]);
                    tc_commit_pair_both(&empty[s], kPairMask);
                }
            }
            // no copy may still run when tensor memory is released
            tc_commit_pair(drain_sf);
            mbar_wait(drain_sf, 0, abort_flag, nullptr, p.budget_ns, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue warps (both CTAs)
        constexpr int kSlice = 256 / (epi_warps(kKind) / 4);   // accumulator columns per epilogue warp
        const int quad = warp & 3, half = (warp - 3) >> 2;
        const float S_W = reinterpret_cast<const PackedHeader*>(p.packed_w)->S_W;
        const float SS = kMain ? __fmul_rn(__uint_as_float(p.scalars[1]), S_W) : 0.f;
        const uint32_t acce0 = mapa_shared(smem_u32(acce), 0);
        int it = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, it++) {
            const int buf = it % kBufs, use = it / kBufs;
            const TileRC rc = tile_rc(tile, num_m, num_n, p.tile_group);
            const int m0 = (m_lo + rc.m) * (2 * kTileM) + (int)rank * kTileM;
            const int n0 = rc.n * kTileN;
            const long long rho = (long long)m0 + quad * 32 + lane;
            const bool row_ok = rho < p.M;
            const int c_base = n0 + half * kSlice;
            const uint32_t tacc = tmem + (uint32_t)(buf * 256) + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * kSlice);
            if (kFfn) {
                // Feed-forward epilogue: Y = BF16(GELU(S_delta S_W acc + P')).  With c_means set, the
                // statistics pass of the consumer layer runs here over these BF16 values: per cube of
                // its partition the fp32 running sum from +0 in (t,h,w) order and the mean (as the
                // statistics kernel forms them), max |mean| over the channels, and max |Y - mean|.
                // Every consumer cube's rows are consecutive rows of one 32-row group (the host checks
                // this before it asks for the statistics), so the lanes of a cube form its sums from
                // one another's values by shuffles, each of them the same sums in the same order.
                const bool cst = p.c_means != nullptr;
                long long n = 0, k = 0, kc = 0;
                int c_first = lane, c_size = 0;
                if (row_ok) {
                    row_to_token(p.g, rho, &n, &k);
                    if (cst) {
                        int pos = 0;
                        cube_pos(p.cg, n, &kc, &pos, &c_size);
                        c_first = lane - pos;
                    }
                }
                const int c_span = (int)__reduce_max_sync(0xffffffffu, (uint32_t)c_size);
                const bool ok = __all_sync(0xffffffffu, mbar_wait_spin(&accf[buf], (uint32_t)use & 1, abort_flag,
                                                                  p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                uint32_t acc[kSlice];
#pragma unroll
                for (int c = 0; c < kSlice; c += 16)
                    tmem_ld_x16(tacc + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(&acc[c]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce0 + (uint32_t)(buf * 8));
                const float* prow = p.p + (size_t)k * p.Nout + c_base;
                uint16_t* yrow = p.Y + (size_t)n * p.Nout + c_base;
                float* mrow = cst ? p.c_means + (size_t)kc * p.Nout + c_base : nullptr;
                const bool writer = cst && row_ok && lane == c_first;   // stores the cube's means
                float kam = 0.f, dmx = 0.f;
                // y = S_delta S_W acc + P' in place over the whole slice first (the P' loads of all pieces
                // in flight together), then GELU, the BF16 rounding and the statistics piece by piece
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < kSlice; c += 8) {
                        float pv[8];
                        ld_global_nc_v8(prow + c, pv);
#pragma unroll
                        for (int e = 0; e < 8; e++)
                            acc[c + e] = __float_as_uint(fmaf(SS, __uint_as_float(acc[c + e]), pv[e]));
                    }
                }
                static_assert(!kFfn || kSlice == 64, "the feed-forward epilogue takes 64-column slices");
                uint32_t pk[32];   // the slice as BF16 pairs
#pragma unroll
                for (int v = 0; v < 32; v++) {
                    float h0, h1;
                    f2_unpack(gelu_erf2(f2_pack(__uint_as_float(acc[2 * v]), __uint_as_float(acc[2 * v + 1]))), h0,
                              h1);
                    pk[v] = bf16x2_rn(h0, h1);
                }
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < 4; c++) st_global_v8(yrow + 16 * c, *reinterpret_cast<const uint32_t(*)[8]>(&pk[8 * c]));
                }
                // statistics: the transposed form when every cube of the warp holds 2 or 4 tokens on aligned
                // lanes (the 720p feed-forward block's down-projection cubes), else one shuffle per row and pair
                const int aligned = cst ? (int)__reduce_min_sync(
                                              0xffffffffu, (uint32_t)(!row_ok ? 7 : (c_first == (lane & ~(c_size - 1)) &&
                                                                                      (c_size == 2 || c_size == 4))
                                                                                         ? c_size
                                                                                         : 0))
                                        : 0;
                const int span_all = cst ? (int)__reduce_max_sync(0xffffffffu, (uint32_t)(row_ok ? c_size : 0)) : 0;
                if (cst && aligned != 0 && aligned != 7 && aligned == span_all) {
                    float* mchunk = mrow;   // this cube's row of means at the slice's first column
                    if (aligned == 4)
                        ffn_stats_aligned<4>(pk, lane & 3, row_ok, mchunk, kam, dmx);
                    else
                        ffn_stats_aligned<2>(pk, lane & 1, row_ok, mchunk, kam, dmx);
                    // the cube's max |mean| over the lanes that hold its columns, to its first lane
                    kam = fmaxf(kam, __shfl_xor_sync(0xffffffffu, kam, 1));
                    if (aligned == 4) kam = fmaxf(kam, __shfl_xor_sync(0xffffffffu, kam, 2));
                } else if (cst) {
#pragma unroll
                    for (int c = 0; c < kSlice; c += 16) {
                        uint32_t mw[8];
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const uint32_t w = pk[c / 2 + j];
                            uint64_t s2 = 0ull;   // (+0, +0)
                            for (int i = 0; i < c_span; i++) {
                                const uint32_t o = __shfl_sync(0xffffffffu, w, (c_first + i) & 31);
                                if (i < c_size) s2 = f2_add(s2, f2_from_bf16x2(o));
                            }
                            float s0, s1, m0 = 0.f, m1 = 0.f;
                            f2_unpack(s2, s0, s1);
                            if (c_size > 0) {
                                m0 = mean_of_sum(s0, c_size);
                                m1 = mean_of_sum(s1, c_size);
                                float d0, d1;
                                f2_unpack(f2_sub(f2_from_bf16x2(w), f2_pack(m0, m1)), d0, d1);
                                kam = max3_abs(m0, m1, kam);
                                dmx = max3_abs(d0, d1, dmx);
                            }
                            mw[(2 * j) & 7] = __float_as_uint(m0);
                            mw[(2 * j + 1) & 7] = __float_as_uint(m1);
                            if ((j & 3) == 3 && writer) st_global_v8(mrow + c + 8 * (j >> 2), mw);
                        }
                    }
                }
                if (cst) {
                    if (writer) atomicMax(&p.c_kamax[kc], __float_as_uint(kam));
                    // non-negative floats order as their bit patterns
                    const uint32_t wd = __reduce_max_sync(0xffffffffu, __float_as_uint(dmx));
                    if (lane == 0) atomicMax(&p.c_scalars[0], wd);
                }
            } else if (kMain) {
                // Pull this warp's 128-column slice of the accumulator into registers and
                // release tensor memory at once, so the next tile's MMAs start while this
                // tile's P' rows are fetched and its Y rows are written.
                long long n = 0, k = 0;
                if (row_ok) row_to_token(p.g, rho, &n, &k);
                const bool ok = __all_sync(0xffffffffu, mbar_wait_spin(&accf[buf], (uint32_t)use & 1, abort_flag,
                                                                  p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                uint32_t acc[128];
#pragma unroll
                for (int c = 0; c < 128; c += 16)
                    tmem_ld_x16(tacc + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(&acc[c]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce0 + (uint32_t)(buf * 8));
                if (row_ok) {
                    // 32-byte accesses: P' in 8-float pieces, Y in 16-value pieces
                    const float* prow = p.p + (size_t)k * p.Nout + c_base;
                    uint16_t* yrow = p.Y + (size_t)n * p.Nout + c_base;
                    float pa[4][8], pb[4][8];
#pragma unroll
                    for (int v = 0; v < 4; v++) ld_global_nc_v8(prow + 8 * v, pa[v]);
#pragma unroll
                    for (int c = 0; c < 128; c += 32) {
                        // software pipeline: the next 32 columns of P' are in flight while these are used
                        if (c + 32 < 128) {
#pragma unroll
                            for (int v = 0; v < 4; v++) ld_global_nc_v8(prow + c + 32 + 8 * v, pb[v]);
                        }
                        uint32_t pk[2][8];
#pragma unroll
                        for (int v = 0; v < 32; v += 2) {
                            const float a0 = pa[v / 8][v % 8], a1 = pa[v / 8][v % 8 + 1];
                            pk[v / 16][(v % 16) / 2] =
                                (uint32_t)f32_to_bf16_rn(fmaf(SS, __uint_as_float(acc[c + v]), a0)) |
                                ((uint32_t)f32_to_bf16_rn(fmaf(SS, __uint_as_float(acc[c + v + 1]), a1)) << 16);
                        }
                        st_global_v8(yrow + c, pk[0]);
                        st_global_v8(yrow + c + 16, pk[1]);
#pragma unroll
                        for (int v = 0; v < 4; v++)
#pragma unroll
                            for (int e = 0; e < 8; e++) pa[v][e] = pb[v][e];
                    }
                }
            } else if (kFp8) {
                // the whole 128-column slice into registers, tensor memory released, then P'
                const float scale = row_ok ? __fmul_rn(p.s8[rho], S_W) : 0.f;
                const float* bias =
                    (reinterpret_cast<const PackedHeader*>(p.packed_w)->flags & kPackedHasBias) ? p.bias + c_base
                                                                                                 : nullptr;
                const bool ok = __all_sync(0xffffffffu, mbar_wait_spin(&accf[buf], (uint32_t)use & 1, abort_flag,
                                                                  p.status, p.budget_ns));
                if (!ok) break;
                tc_fence_after();
                uint32_t acc[128];
#pragma unroll
                for (int c = 0; c < 128; c += 16)
                    tmem_ld_x16(tacc + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(&acc[c]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce0 + (uint32_t)(buf * 8));
                if (row_ok) {
                    float* dst = p.pout + (size_t)rho * p.Nout + c_base;
#pragma unroll
                    for (int c = 0; c < 128; c += 8) {
                        float b0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (bias) ld_global_nc_v8(bias + c, b0);
                        uint32_t o0[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) o0[e] = __float_as_uint(fmaf(__uint_as_float(acc[c + e]), scale, b0[e]));
                        st_global_cs_v8(dst + c, o0);
                    }
                }
            } else {
                const float scale = row_ok ? (p.s8 ? __fmul_rn(p.s8[rho], S_W) : S_W) : 0.f;
                // the layer's bias, when the packed weight holds one, joins P' once per cube
                const float* bias =
                    (reinterpret_cast<const PackedHeader*>(p.packed_w)->flags & kPackedHasBias) ? p.bias + c_base
                                                                                                 : nullptr;
                const bool ok = __all_sync(0xffffffffu, mbar_wait_spin(&accf[buf], (uint32_t)use & 1, abort_flag,
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
                        // 32-byte stores
#pragma unroll
                        for (int v = 0; v < 16; v += 8) {
                            float b0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                            float b1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                            if (bias) {
                                ld_global_nc_v8(bias + c + v, b0);
                                ld_global_nc_v8(bias + c + 16 + v, b1);
                            }
                            uint32_t o0[8], o1[8];
#pragma unroll
                            for (int e = 0; e < 8; e++) {
                                o0[e] = __float_as_uint(fmaf(__uint_as_float(r0[v + e]), scale, b0[e]));
                                o1[e] = __float_as_uint(fmaf(__uint_as_float(r1[v + e]), scale, b1[e]));
                            }
                            st_global_cs_v8(dst + c + v, o0);
                            st_global_cs_v8(dst + c + 16 + v, o1);
                        }
                    }
                }
                // tensor-memory buffer free for the next tile
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce0 + (uint32_t)(buf * 8));
            }
        }
    }
    // Neither CTA leaves, nor frees tensor memory, while its peer may still
    // touch its shared memory, barriers or tensor memory.
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

// ------------------------------------------------------------------ launchers

namespace {

constexpr int kMaxDevices = 64;

template <int kKind>
cudaError_t launch_pairs(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                         const CUtensorMap& tm_sb, const CUtensorMap& tm_fa, const CUtensorMap& tm_fb,
                         const GemmParams& p, cudaStream_t st) {
    constexpr size_t smem = g_smem_layout(kKind).total + 1024;
    static_assert(smem <= 232448, "shared memory of a paired product");
    cudaError_t e = cudaFuncSetAttribute(k_gemm<kKind>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (p.tile_m1 - p.tile_m0) * (p.Nout / kTileN);
    if (tiles <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(g_threads(kKind));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once (one CTA per SM), queried once per
    // device (concurrent first calls may both query; they store the same answer)
    static std::atomic<int> resident[kMaxDevices];
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int mp = resident[dev].load(std::memory_order_relaxed);
    if (mp == 0) {
        cfg.gridDim = dim3(2 * tiles);
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, k_gemm<kKind>, &cfg);
        if (e != cudaSuccess) return e;
        if (n <= 0) return cudaErrorInvalidConfiguration;
        mp = n;
        resident[dev].store(mp, std::memory_order_relaxed);
    }
    cfg.gridDim = dim3(2 * imin(tiles, mp));
    return cudaLaunchKernelEx(&cfg, k_gemm<kKind>, tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb, p);
}

}  // namespace

cudaError_t launch_kernel_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmParams& p,
                               cudaStream_t st) {
    return launch_pairs<kGemmKernelBf16>(tm_a, tm_b, tm_a, tm_b, tm_a, tm_b, p, st);
}

cudaError_t launch_kernel_gemm_fp8(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_fb,
                                   const GemmParams& p, cudaStream_t st) {
    return launch_pairs<kGemmKernelFp8>(tm_a, tm_b, tm_a, tm_b, tm_a, tm_fb, p, st);
}

cudaError_t launch_main_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                             const CUtensorMap& tm_sb, const CUtensorMap& tm_fa, const CUtensorMap& tm_fb,
                             const GemmParams& p, cudaStream_t st) {
    return launch_pairs<kGemmMain>(tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb, p, st);
}

cudaError_t launch_main_gemm_ffn(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                                 const CUtensorMap& tm_sb, const CUtensorMap& tm_fa, const CUtensorMap& tm_fb,
                                 const GemmParams& p, cudaStream_t st) {
    return launch_pairs<kGemmMainFfn>(tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb, p, st);
}

}  // namespace dq
