// Kernel parameter blocks and launchers shared between the C-ABI layer
// (dq_api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dq_common.h"

namespace dq {

struct QuantParams {
    Geom g;
    int Ci, rank, slab, splits, chunks_per_split;
    int nw;             // whole cubes per box along w
    int bt, bh, bw;     // box extent in tokens: t x h x (nw w)
    int nbw;            // boxes along w
    int n_boxes;
    int item0, item1;   // the statistics kernel's work items [item0, item1) of n_boxes * splits (a T-slab)
    int m_rows;         // kernel tokens per box (rows of the encode kernel's per-stage tile)
    int stat_pairs;     // statistics kernel: one warp per cube, a channel pair per lane (cubes of 16+ tokens)
    int kgroup;         // 0: s8 per kernel token (K); 64: per 64 channels (K x Ci/64), q8_bf16 = [hi | lo]
    int fp8_product;    // the kernel-token product reads q8 (C2 weights): no q8_bf16, packed weight must be C2
    int pow2;           // single-read quantiser: power-of-two S_delta, provisional per-chunk scales, fix-up pass
    int8_t* prov;       //   N x Ci/64 provisional scale exponents (-128: a chunk whose deltas are all zero)
    int big;            // cubes of more than 128 tokens: boxes are row segments of one cube,
    int nseg;           //   nseg segments of up to 128 tokens per cube row; the kernel tokens
    float* means;       //   K x Ci fp32 kernel tokens: written by k_cube_stats (by k_cube_means_big for big cubes)
    int* status;
    uint32_t* scalars;  // [0] bits of max|delta|, [1] S_delta
    uint32_t* kamax;
    float* s8;
    uint8_t* q8;
    uint16_t* q8_bf16;
    uint8_t* dcodes;
    uint8_t* dscales;
    float* u_part;
    uint16_t* u_hilo;
    const uint8_t* packed_w;
    uint64_t budget_ns;
};

struct GemmParams {
    Geom g;
    int M;               // valid rows of A
    int Nout;            // output columns (Co)
    int Ci;
    int k_stages;        // main-operand K stages
    int slab_stages;     // extra BF16 K stages (low-rank slab), main product only
    int b_kblocks;       // kernel-token product: B k-blocks (Ci/64); A k-block i reads B k-block i mod this
    int tile_group;      // tile order: 1 row-major, else groups of this many row tiles walked column by column
    int tile_m0, tile_m1;  // the launch's row tiles [tile_m0, tile_m1) of 256 rows
    const float* p;      // per-cube kernel term, K x Co fp32 (main product)
    const uint32_t* scalars;
    const uint8_t* packed_w;
    const float* s8;     // per-row kernel-token scales (kernel-token product); null when A carries them
    float* pout;         // kernel-token product output, K x Co fp32
    const float* bias;   // Co fp32 bias section of the packed weight (read when its flag is set)
    uint16_t* Y;         // main product output, N x Co BF16 (t,h,w) order
    // feed-forward epilogue (kGemmMainFfn): Y = BF16(GELU(y)); with c_means set, also the statistics
    // pass of the consumer layer over that Y, for its cube partition cg of the same lattice: the fp32
    // cube means (K_c x Co), max |mean| per cube (atomic max into c_kamax) and max |Y - mean| (atomic
    // max into c_scalars[0]); every consumer cube's rows are consecutive rows of one 32-row group here
    Geom cg;
    float* c_means;
    uint32_t* c_kamax;
    uint32_t* c_scalars;
    int* status;
    uint64_t budget_ns;
};

// Paired-GEMM kinds: the exact kernel-token product (BF16, kind::f16), the main block-scaled FP4
// product, the FP8 kernel-token product on C2 weights (kind::mxf8f6f4, UE8M0 scales per 32).
// The main product with the feed-forward epilogue (GELU, consumer statistics) is a kind of its own
// so that the plain main product keeps its registers.
enum GemmKind { kGemmKernelBf16 = 0, kGemmMain = 1, kGemmKernelFp8 = 2, kGemmMainFfn = 3 };

size_t quant_smem_bytes(int rank, bool stats, int m_rows, int x_rows);
cudaError_t launch_cube_stats(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p,
                              cudaStream_t st);
cudaError_t launch_cube_encode(const CUtensorMap& tm_x, const CUtensorMap& tm_m, const QuantParams& p,
                               cudaStream_t st);
cudaError_t launch_cube_means_big(const CUtensorMap& tm_x, const QuantParams& p, cudaStream_t st);
// the encode pass with X L1 on the tensor cores (for a layer whose statistics a producer's epilogue
// formed, so that no statistics pass runs), then U' from the partial sums (k_u_hilo)
cudaError_t launch_cube_encode_lowrank(const CUtensorMap& tm_x, const CUtensorMap& tm_m, const CUtensorMap& tm_l1,
                                       const QuantParams& p, cudaStream_t st);
// single-read quantiser: statistics + provisional encode (one read of X), then the fix-up pass with
// the kernel tokens and U' (no read of X except for re-encoded groups)
cudaError_t launch_cube_single(const CUtensorMap& tm_x, const CUtensorMap& tm_l1, const QuantParams& p,
                               cudaStream_t st);
cudaError_t launch_single_finish(const void* X, const QuantParams& p, cudaStream_t st);

cudaError_t launch_kernel_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmParams& p,
                               cudaStream_t st);
cudaError_t launch_kernel_gemm_fp8(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_fb,
                                   const GemmParams& p, cudaStream_t st);
cudaError_t launch_main_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                             const CUtensorMap& tm_sb, const CUtensorMap& tm_fa, const CUtensorMap& tm_fb,
                             const GemmParams& p, cudaStream_t st);
// the main product with the feed-forward epilogue (kGemmMainFfn)
cudaError_t launch_main_gemm_ffn(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_sa,
                                 const CUtensorMap& tm_sb, const CUtensorMap& tm_fa, const CUtensorMap& tm_fb,
                                 const GemmParams& p, cudaStream_t st);

// Device address of the no-allocation entry point's fixed workspace on the
// current device (dq_noalloc.cu); a dq_status code.
int noalloc_workspace(void** out);

cudaError_t launch_selftest_wait(int* status, uint64_t budget_ns, cudaStream_t st);
cudaError_t launch_selftest_gelu(const float* in, long long n, float* out, cudaStream_t st);
cudaError_t launch_selftest_divide(long long n, uint64_t seed, unsigned long long* mismatches, float* first,
                                   cudaStream_t st);
cudaError_t launch_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* back,
                                    cudaStream_t st);

}  // namespace dq
