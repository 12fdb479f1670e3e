/*
 * deltaquant.h -- C ABI of the DeltaQuant W4A4 linear layer for B200 (sm_100a).
 *
 * The layer (papernotes.org, "DeltaQuant: 4-bit Video Diffusion Models with
 * Spatiotemporal Delta Smoothing", key designs 2-4):
 *   X (N = T*H*W tokens x Ci channels, BF16, rows in (t,h,w) row-major order)
 *   is viewed as T x H x W x Ci and cut into t x h x w cubes (design 2).  Each
 *   cube's fp32 mean is its kernel token, each token minus its cube's mean a
 *   delta token (Eq. 1).  Kernel tokens are quantised to FP8 E4M3 with one fp32
 *   scale per token (or per 64 channels, dq_linear_forward_grouped); delta
 *   tokens to FP4 E2M1 with one E4M3 scale per 16 channels and one fp32
 *   per-tensor scale (Eq. 4 with the NVFP4 reading).
 *   W (Co x Ci) is split offline into rank-r BF16 factors L1, L2 from its SVD
 *   and a residual R = W - L1 L2 quantised to the same FP4 format (Eq. 3):
 *     Y = dq(delta) dq(R)^T + broadcast_cube(dq(kernel) dq(R)^T) + (X L1) L2  [+ b]
 *   Y is N x Co BF16 in (t,h,w) order; b is an optional bias (dq_pack_bias).
 *
 * Conventions for every entry point:
 *   - The return value is a dq_status code; nothing aborts or exits.
 *   - Arguments are checked before anything is launched or written.
 *   - "host" pointers are ordinary CPU memory; "device" pointers are global
 *     memory of the current CUDA device.  The caller owns every buffer.
 *   - Online entry points are asynchronous on the given stream (a
 *     cudaStream_t passed as void*; NULL = legacy default stream).  Errors
 *     found by the device (bad packed-weight header, a bounded wait that ran
 *     out) are written to a status word inside the workspace; read it with
 *     dq_read_device_status after the stream has been synchronised.
 *   - Inputs are never modified; outputs are fully overwritten.
 *   - Shapes: Ci and Co multiples of 256; rank a multiple of 16 in [16, 128];
 *     1 <= t <= T, 1 <= h <= H, 1 <= w <= W (cubes of any size up to the whole
 *     lattice, which gives one global kernel token); N = T*H*W < 2^31.
 *     Anything else returns DQ_ERR_UNSUPPORTED_SHAPE.  Device pointers must be 256-byte aligned
 *     (DQ_ERR_ALIGNMENT otherwise).
 */
#ifndef DELTAQUANT_H
#define DELTAQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DQ_ABI_VERSION 4
#define DQ_PACK_FORMAT_VERSION 3
#define DQ_PACK_MAGIC 0x31575144u /* "DQW1" little-endian */

typedef enum dq_status {
    DQ_OK = 0,
    DQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad flag */
    DQ_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the conventions above */
    DQ_ERR_ALIGNMENT = 3,          /* a device pointer is not 256-byte aligned */
    DQ_ERR_WORKSPACE_TOO_SMALL = 4,
    DQ_ERR_CUDA = 5,               /* a CUDA runtime call failed */
    DQ_ERR_DEVICE_TIMEOUT = 6,     /* a bounded device-side wait ran out */
    DQ_ERR_BAD_PACKED_WEIGHT = 7,  /* packed-weight header does not match */
    DQ_ERR_NO_DEVICE = 8,          /* no usable sm_100 device */
    DQ_ERR_ALLOC = 9               /* host or device allocation failed */
} dq_status;

/* Text for a status code (static storage). */
const char* dq_status_string(int status);

/* Text of the CUDA runtime error behind the last DQ_ERR_CUDA that an entry
 * point returned on the calling thread ("" if none); static per-thread storage. */
const char* dq_last_cuda_error(void);

/* DQ_ABI_VERSION of the loaded library. */
int dq_abi_version(void);

/* ------------------------------------------------------------------------ */
/* Layout maps                                                               */
/* ------------------------------------------------------------------------ */

/*
 * Cube partition (key design 2): KT = ceil(T/t), KH = ceil(H/h), KW = ceil(W/w),
 * K = KT*KH*KW cubes, cube k = (kt*KH + kh)*KW + kw.  Edge cubes that the
 * lattice cuts short hold fewer tokens (their mean is over those tokens).
 * Cube-major order lists the cubes in k order and, inside a cube, its tokens
 * in (t,h,w) order.  dq_cube_major_row maps natural token n to its cube-major
 * row and cube.
 */
int dq_cube_count(int T, int H, int W, int t, int h, int w, long long* K);
int dq_cube_major_row(int T, int H, int W, int t, int h, int w, long long n, long long* row,
                      long long* cube);

/*
 * Scale-factor layout of an FP4 matrix with `rows` rows and `cols` columns
 * (one E4M3 scale per 16 consecutive columns of a row).  Rows are grouped by
 * 128 and columns by 64; each (row group, column group) owns 512 contiguous
 * bytes in which scale (row, block) sits at
 *   (row % 32) * 16 + ((row % 128) / 32) * 4 + (block % 4),
 * groups ordered row-group-major:
 *   offset = ((row/128) * (cols/64) + block/4) * 512 + (the above).
 * This is the order in which the tensor cores' block-scaled MMA reads scale
 * factors from tensor memory after a 32x128-bit copy, so tiles move with bulk
 * copies and no reshuffle.  Total size: ceil(rows/128) * (cols/64) * 512.
 */
int dq_sf_offset(long long row, int block, int cols, size_t* offset);
int dq_sf_bytes(long long rows, int cols, size_t* bytes);

/*
 * A-operand scale layout (the delta group scales in the workspace; cols a
 * multiple of 256).  The block-scaled MMA reads the scales of row r of a
 * 128-row tile from tensor-memory lane r, column (scale address + r / 32): the
 * 32-lane quadrant q of the tensor memory uses the q-th 32-bit column of each
 * 4-column group.  So one 128x256-bit copy per two 64-column blocks suffices
 * (instead of one replicating 32x128-bit copy per block), from this layout:
 * per 128-row group and 256-column K step, two 4096-byte blocks (one per pair
 * of 64-column blocks), each 128 rows x 32 bytes stored as 8-row x 16-byte
 * core matrices (row-group stride 256, column-half stride 128); row r holds
 * the four scales of 64-column block kb at 32-bit word 4 (kb % 2) + r / 32:
 *   offset = (((row/128) * (cols/256) + kb/4) * 2 + (kb/2) % 2) * 4096
 *            + ((row%128)/8) * 256 + (kb % 2) * 128 + (row % 8) * 16
 *            + ((row%128)/32) * 4 + block % 4,      kb = block / 4.
 * A quarter of the bytes hold scales; the rest are never read.  Total size:
 * ceil(rows/128) * (cols/256) * 8192.
 */
int dq_sfa_offset(long long row, int block, int cols, size_t* offset);
int dq_sfa_bytes(long long rows, int cols, size_t* bytes);

/*
 * B-operand scale layout (the weight group scales of the packed weight; rows
 * a multiple of 256).  Every 32-lane quadrant of the tensor memory needs the
 * scales of all 256 columns of an output tile, in lane i the scales of rows
 * 32 c + i and 128 + 32 c + i (c = 0..3) of the tile in its eight 32-bit
 * columns.  Stored so that one 128x256-bit copy per 64-column block writes
 * that (instead of two replicating 32x128-bit copies): per 256-row tile and
 * 64-column block one 4096-byte block of 128 lanes x 32 bytes in 8-row x
 * 16-byte core matrices (row-group stride 256, column-half stride 128), lanes
 * i, i + 32, i + 64 and i + 96 holding the same bytes.  dq_sfb_offset gives
 * the byte in lane row % 32; the copies in the other three lanes sit 1024,
 * 2048 and 3072 bytes further:
 *   n = row % 256, w = 4 (n / 128) + (n % 128) / 32, b = 4 w + block % 4,
 *   offset = ((row/256) * (cols/64) + block/4) * 4096
 *            + ((n%32)/8) * 256 + (b/16) * 128 + (n % 8) * 16 + b % 16.
 * Total size: ceil(rows/256) * (cols/64) * 4096.
 */
int dq_sfb_offset(long long row, int block, int cols, size_t* offset);
int dq_sfb_bytes(long long rows, int cols, size_t* bytes);

/* ------------------------------------------------------------------------ */
/* Offline weight packing (host only, synchronous)                           */
/* ------------------------------------------------------------------------ */

/*
 * Packed weight blob (device copy of what dq_pack_weight writes), all
 * sections 256-byte aligned:
 *   header  256 bytes: uint32 magic, uint32 version, int32 Co, Ci, rank,
 *           slab, float S_W, uint32 flags (bit 0: the layer has a bias),
 *           then uint64 byte offsets of codes, scales, dqw, the total size
 *           and the offset of the bias section.
 *   codes   Co x Ci/2 bytes, E2M1 codes of R, row o = output channel,
 *           channel 2i in the low nibble of byte i.
 *   scales  E4M3 group-16 scales of R in the B-operand scale layout above.
 *   dqw     Co x Ci BF16 values q * s_b of R (exact: at most 6 significant
 *           bits), the operand of the kernel-token product.
 *   bias    Co fp32, the layer's bias b (y = x W^T + b) widened exactly from
 *           BF16 by dq_pack_bias; zeros and flag bit 0 clear when unset.
 * S_W is R's per-tensor scale.  dq_packed_weight_bytes gives the size.
 */
typedef struct dq_packed_layout {
    size_t total_bytes;
    size_t off_codes, off_scales, off_dqw, off_bias;
    int Co, Ci, rank, slab;
} dq_packed_layout;

int dq_packed_weight_layout(int Co, int Ci, int rank, dq_packed_layout* out);
int dq_packed_weight_bytes(int Co, int Ci, int rank, size_t* bytes);

/*
 * Width of the low-rank slab: 2*rank rounded up to a multiple of 64.  The
 * up-projection runs as extra K-steps of the main product with A = [U_hi | U_lo]
 * and B = [L2^T | L2^T], zero-padded to this width.
 */
int dq_lowrank_slab_width(int rank);

/*
 * Rank-r factors from a truncated SVD of W (SVDQuant low-rank branch, Eq. 3):
 * W^T ~ V_r S_r U_r^T, L1 = V_r S_r^(1/2) (Ci x r), L2 = S_r^(1/2) U_r^T (r x Co),
 * both rounded to BF16 (nearest even).  Randomised subspace iteration in fp64
 * with the given seed.  W: host Co x Ci BF16 (y = x W^T).  Outputs: host, caller-owned.
 */
int dq_lowrank_factors(const uint16_t* W, int Co, int Ci, int rank, uint64_t seed, uint16_t* L1,
                       uint16_t* L2);

/*
 * Pack W with given BF16 factors L1 (Ci x r, host) and L2 (r x Co, host):
 *   R[o][i] = fl32(W[o][i] - sum_j L1[i][j] L2[j][o]) (fp64 sum, ascending j),
 *   S_W = amax(R)/2688 (1 if 0), s_b = E4M3(amax_b / (6 S_W)),
 *   q = E2M1(R / (s_b S_W))   (Eq. 4 per 16-channel group, nearest even, saturating).
 * Writes the packed blob (host, packed_bytes >= dq_packed_weight_bytes), the
 * tensor-core copies of the factors: L1_mma = L1^T (r x Ci BF16, host) and
 * L2_slab (Co x slab BF16, host, [L2^T | L2^T | 0]), and optionally S_W.
 */
int dq_pack_weight_factors(const uint16_t* W, const uint16_t* L1, const uint16_t* L2, int Co, int Ci,
                           int rank, void* packed, size_t packed_bytes, uint16_t* L1_mma,
                           uint16_t* L2_slab, float* S_W);

/*
 * Packing options (pack_flags of dq_pack_weight_factors_ex):
 *   DQ_PACK_C2  restricted group scales for an FP8-rate kernel-token product
 *               (DQ_KERNEL_PRODUCT_FP8).  The note runs the kernel-token product
 *               on FP8 tensor cores; with Eq. 4's E4M3 group-16 scales the
 *               product q s_b needs up to 6 significant bits, which no FP8
 *               operand holds.  C2 takes S_W = amax(R) / (6 * 384) and rounds
 *               each group scale to the nearest member (ties to the larger) of
 *               {0} and the E4M3 values m 2^e with m in {1, 1.25, 1.5}, up to
 *               384; per 32 channels a nonzero smaller scale is raised to the
 *               smallest member >= 2^-9 times the larger.  Then every q s_b of a
 *               32-channel block is an E4M3 value times one power of two 2^u.
 *               The blob's dqw section then holds, in place of BF16 q s_b:
 *               Co x Ci E4M3 codes of q s_b / 2^u (u such that the block's
 *               largest |q s_b| / 2^u lies in [128, 256)),
 *               followed by the exponents u + 127 (UE8M0) in the layout
 *               dq_sfb_offset gives for a Co x (Ci / 2) matrix, block j of that
 *               matrix standing for 32-channel block j (four copies, one per
 *               tensor-memory quadrant, as for the weight scales).  Header flag
 *               bit 1 marks such a blob.  The price is accuracy: three scale
 *               mantissas instead of E4M3's eight (weight error 1.06 to 1.14
 *               times Eq. 4's on the synthetic weights).
 */
#define DQ_PACK_C2 1

/* dq_pack_weight_factors with pack_flags (0 or DQ_PACK_C2; anything else:
 * DQ_ERR_INVALID_ARG). */
int dq_pack_weight_factors_ex(const uint16_t* W, const uint16_t* L1, const uint16_t* L2, int Co, int Ci, int rank,
                              int pack_flags, void* packed, size_t packed_bytes, uint16_t* L1_mma, uint16_t* L2_slab,
                              float* S_W);

/*
 * Set (bias != NULL) or clear (bias == NULL) the bias of a packed blob in
 * host memory: bias is host, Co BF16 values; Co must equal the blob's Co and
 * packed_bytes its total size.  The forward pass then returns x W^T + b: the
 * bias is added once per cube to the kernel-token product P', which every
 * token of the cube receives (no per-token cost).  Linear layers commonly
 * carry such a bias; the method's equations leave it out.
 * Returns DQ_ERR_BAD_PACKED_WEIGHT when the blob's header is not a packed
 * weight of this format.
 */
int dq_pack_bias(const uint16_t* bias, int Co, void* packed, size_t packed_bytes);

/* dq_lowrank_factors (seed 0) followed by dq_pack_weight_factors. */
int dq_pack_weight(const uint16_t* W, int Co, int Ci, int rank, void* packed, size_t packed_bytes,
                   uint16_t* L1_mma, uint16_t* L2_slab);

/* ------------------------------------------------------------------------ */
/* Online forward (device, asynchronous)                                      */
/* ------------------------------------------------------------------------ */

/*
 * Workspace carve-up (all offsets 256-byte aligned).  Tensors a test or a
 * profiler may read after a forward:
 *   status     int32 device status word (0 = ok, else a dq_status)
 *   scalars    uint32[4]: [0] bits of max|delta| (fp32), [1] S_delta (fp32)
 *   kamax      K uint32: bits of max_c |mean_k[c]| per cube (fp32)
 *   s8         K fp32 kernel-token scales (per-token), or K x Ci/64 (group 64)
 *   q8         K x Ci E4M3 kernel tokens
 *   q8_bf16    the kernel-token product's A operand: K_pad x Ci BF16 copy of q8
 *              (per-token), or K_pad x 2Ci BF16 q8*s8 split as hi (columns
 *              0..Ci-1) + lo (Ci..2Ci-1), |hi + lo - q8 s8| <= 2^-16 |q8 s8| (group 64);
 *              empty with DQ_KERNEL_PRODUCT_FP8, whose A operand is q8 itself
 *   dcodes     N x Ci/2 E2M1 delta codes, cube-major rows
 *   dscales    delta group scales, A-operand scale layout (dq_sfa_offset) over N rows
 *   u_part     splits x N x rank fp32 partial sums of X L1 (cube-major rows)
 *   u_hilo     N x slab BF16: U' = (X L1)/(S_delta S_W) split as hi + lo
 *   p          K x Co fp32: s8 S_W q8 dqw^T (the per-cube kernel term)
 *   means      K x Ci fp32 kernel tokens before quantisation
 *   prov       DQ_DELTA_SCALE_POW2 only: N x Ci/64 int8 exponents of the
 *              provisional per-chunk delta scales (-128: all deltas of the
 *              chunk are zero); empty otherwise
 */
typedef struct dq_workspace_layout {
    size_t total_bytes;
    size_t off_status, off_scalars, off_kamax, off_s8, off_q8, off_q8_bf16, off_dcodes, off_dscales,
        off_u_part, off_u_hilo, off_p, off_means;
    long long N, K, N_pad, K_pad;
    int splits, slab;
    int kernel_group;
    size_t off_prov;
} dq_workspace_layout;

/*
 * FP8 kernel-token scale granularity (argument kernel_group):
 *   DQ_KERNEL_SCALE_PER_TOKEN  s8[k] = max_c |mean_k[c]| / 448, one per kernel token
 *   DQ_KERNEL_SCALE_GROUP64    s8[k][j] = max |mean_k[c]| / 448 over channels
 *                              c in [64 j, 64 j + 64): the DeltaQuant note's
 *                              per-group-64 kernel quantisation (its section on
 *                              the training strategy).  The kernel-token product then reads
 *                              2 Ci BF16 columns per kernel token (hi + lo).
 * q8[k][c] = E4M3(mean_k[c] / scale), 0 where the scale is 0, in both.
 */
#define DQ_KERNEL_SCALE_PER_TOKEN 0
#define DQ_KERNEL_SCALE_GROUP64 64

/* Workspace carve-up of a forward call with per-token kernel scales. */
int dq_workspace_layout_get(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                            dq_workspace_layout* out);
int dq_workspace_bytes(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                       size_t* bytes);
/* The same for a kernel_group (DQ_KERNEL_SCALE_*; anything else: DQ_ERR_INVALID_ARG). */
int dq_workspace_layout_grouped(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                                int kernel_group, dq_workspace_layout* out);
int dq_workspace_bytes_grouped(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                               int kernel_group, size_t* bytes);

/* Stage selection for dq_linear_forward_ex. */
#define DQ_STAGE_QUANTIZE 1    /* cube statistics + cube encode (kernels a1, a2) */
#define DQ_STAGE_KERNEL_GEMM 2 /* kernel-token product P (kernel c) */
#define DQ_STAGE_MAIN_GEMM 4   /* block-scaled FP4 product + low-rank slab + epilogue (kernel b) */
#define DQ_STAGE_ALL 7
/*
 * The two halves of DQ_STAGE_QUANTIZE, for a layer sharded by cubes across
 * devices: after DQ_STAGE_STATS the workspace's scalars[0] holds this shard's
 * max |delta| (fp32 bits, non-negative); the caller replaces it with the
 * maximum over all shards (one all-reduce) before DQ_STAGE_ENCODE, which
 * derives S_delta from it.  Shards are slabs of whole cubes along T; every
 * other quantity of the layer is local to a cube.
 */
#define DQ_STAGE_STATS 8       /* a1: cube means, max |mean| per cube, max |delta|, X L1 partial sums */
#define DQ_STAGE_ENCODE 16     /* a2: FP8 kernel tokens, FP4 delta codes and scales, U' hi + lo */

/*
 * Y = DeltaQuant linear layer of X (see top of file), on `stream`.
 *   X        device, N x Ci BF16, (t,h,w) row-major
 *   packed_W device, the blob written by dq_pack_weight (copied to device)
 *   L1_mma   device, rank x Ci BF16;  L2_slab device, Co x slab BF16
 *   Y        device, N x Co BF16, (t,h,w) row-major
 * Uses a library-owned workspace on the current device, allocated on the
 * first call for the largest shape seen so far (a blocking cudaMalloc; make
 * that first call before any stream capture).  Calls that share the library
 * workspace must be ordered (same stream); use _ex for concurrent calls.
 */
int dq_linear_forward(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                      const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y, void* stream);

/*
 * As dq_linear_forward with a caller-owned device workspace of at least
 * dq_workspace_bytes bytes, a stage mask (DQ_STAGE_*; stages read what
 * earlier stages left in the same workspace), and optional timing events:
 * stage_events NULL or an array of 4 cudaEvent_t (as void*) recorded before
 * the first stage and after each of the three stages.
 */
int dq_linear_forward_ex(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                         const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y,
                         void* workspace, size_t workspace_bytes, int stage_mask, void* const* stage_events,
                         void* stream);

/*
 * As dq_linear_forward_ex with the kernel-token scale granularity kernel_group
 * (DQ_KERNEL_SCALE_*); the workspace is at least dq_workspace_bytes_grouped
 * for the same kernel_group.  dq_linear_forward_ex is this call with
 * DQ_KERNEL_SCALE_PER_TOKEN.
 */
int dq_linear_forward_grouped(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                              int kernel_group, const void* packed_W, const void* L1_mma, const void* L2_slab,
                              void* Y, void* workspace, size_t workspace_bytes, int stage_mask,
                              void* const* stage_events, void* stream);

/*
 * Forward options (dq_linear_forward_opts, dq_workspace_layout_opts):
 *   kernel_group    DQ_KERNEL_SCALE_PER_TOKEN or DQ_KERNEL_SCALE_GROUP64
 *   kernel_product  DQ_KERNEL_PRODUCT_BF16: the kernel-token product on exact
 *                   BF16 operands (q8 widened, q s_b), kind::f16; any packed weight
 *                   without DQ_PACK_C2.
 *                   DQ_KERNEL_PRODUCT_FP8: q8 (E4M3) times the FP8 form of
 *                   DQ_PACK_C2 weights with UE8M0 scales per 32 channels,
 *                   kind::mxf8f6f4, at twice the BF16 rate; per-token kernel
 *                   scales only.  The product is the same exact sum as with
 *                   BF16 operands of the same (C2) weights.
 *   delta_scale     DQ_DELTA_SCALE_AMAX: the per-tensor delta scale S = amax / 2688
 *                   (Eq. 4 with two levels); the quantise stage reads X twice, since
 *                   no delta can be encoded before every delta's amax is known.
 *                   DQ_DELTA_SCALE_POW2: S = the smallest power of two >= amax / 2688
 *                   (1 if amax = 0), a deviation from Eq. 4 that lets X be read once:
 *                   the statistics pass also encodes each 64-channel chunk under
 *                   the chunk's own power-of-two scale S_c <= S (its exponent kept in
 *                   the workspace section prov), and the encode stage then lowers
 *                   each group's E4M3 scale code by 8 log2(S / S_c), keeping its E2M1
 *                   codes, or encodes the group again under S when the code's
 *                   exponent field is below log2(S / S_c) + 1 (E4M3's subnormal
 *                   grid); the result equals encoding every group under S.  The
 *                   encode stage also forms the kernel tokens and U' from the stored
 *                   means and partial sums (no read of X apart from re-encoded
 *                   groups).  Per-token kernel scales only.
 *   epilogue        DQ_EPILOGUE_NONE: Y = BF16(y), y = S_delta S_W acc + P'[k(n)] in fp32.
 *                   DQ_EPILOGUE_GELU: Y = BF16(GELU(y)), GELU(y) = y Phi(y) =
 *                   y erfc(-y / sqrt 2) / 2 in fp32 (erfcf), one rounding to BF16:
 *                   the up-projection of a transformer feed-forward block with its
 *                   activation in the main product's epilogue (the note's
 *                   overall pipeline ends in a fused kernel; the activation itself
 *                   is not on the pages and is taken in its exact erf form).
 * A packed weight whose C2 flag does not match kernel_product is reported as
 * DQ_ERR_BAD_PACKED_WEIGHT in the device status word.
 */
#define DQ_KERNEL_PRODUCT_BF16 0
#define DQ_KERNEL_PRODUCT_FP8 1
#define DQ_DELTA_SCALE_AMAX 0
#define DQ_DELTA_SCALE_POW2 1
#define DQ_EPILOGUE_NONE 0
#define DQ_EPILOGUE_GELU 1

typedef struct dq_forward_options {
    int kernel_group;
    int kernel_product;
    int delta_scale;
    int epilogue;
} dq_forward_options;

int dq_workspace_layout_opts(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                             const dq_forward_options* opts, dq_workspace_layout* out);

/* dq_linear_forward_grouped with forward options (opts NULL: the defaults, all 0). */
int dq_linear_forward_opts(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                           const dq_forward_options* opts, const void* packed_W, const void* L1_mma,
                           const void* L2_slab, void* Y, void* workspace, size_t workspace_bytes, int stage_mask,
                           void* const* stage_events, void* stream);

/*
 * A transformer feed-forward block as two DeltaQuant layers with the producer
 * step fused (the note's overall pipeline, "fused kernel output"; its
 * training-strategy section fuses kernel-token generation into the activation
 * quantisation kernel):
 *   Hid = BF16(GELU(up(X)))        up:   T x H x W lattice, cube cube_up,   Ci -> Cf
 *   Y   = down(Hid)                down: the same lattice, cube cube_down, Cf -> Co
 * Each layer computes exactly what dq_linear_forward_opts computes for it (the
 * up-projection with DQ_EPILOGUE_GELU, both with the default options); Hid and Y
 * are bit-identical to those two calls.  The fusion: when every cube_down cube
 * of the lattice occupies consecutive cube-major rows of the cube_up partition,
 * in its own (t,h,w) order, inside one aligned group of 32 rows
 * (dq_ffn_fused_statistics; e.g. cube_down = (1, h, w) inside cube_up =
 * (t', h, w), or cube_down = cube_up, with at most 32 tokens), the
 * up-projection's main-product epilogue also forms the down-projection's
 * statistics pass over the BF16 Hid it writes: the fp32 cube means (K_down x Cf,
 * the running sum from +0 in (t,h,w) order divided by the count), max |mean| per
 * cube and max |Hid - mean|.  The down-projection then runs no statistics pass:
 * its encode pass also forms Hid L1_down on the tensor cores, so Hid is read once
 * instead of twice.  Otherwise, or with DQ_FFN_SEPARATE_STATISTICS, the
 * down-projection runs its own statistics pass.
 *
 *   X        device, N x Ci BF16, (t,h,w) order; read only
 *   cube_up, cube_down  host, 3 ints each (t, h, w)
 *   packed_up, L1_up, L2_up       the up-projection's (Co = Cf, rank_up) weight as
 *                                  dq_pack_weight makes it (no DQ_PACK_C2)
 *   packed_down, L1_down, L2_down the down-projection's (Ci = Cf, Co, rank_down)
 *   Hid      device, N x Cf BF16, (t,h,w) order; written (the hidden activation)
 *   Y        device, N x Co BF16, (t,h,w) order; written
 *   ws_up    device workspace of dq_workspace_bytes(T,H,W, cube_up, Ci, Cf, rank_up)
 *   ws_down  device workspace of dq_workspace_bytes(T,H,W, cube_down, Cf, Co, rank_down)
 *   ffn_flags      0 or DQ_FFN_SEPARATE_STATISTICS
 *   stage_events   NULL or 8 cudaEvent_t (as void*): the up-projection's 4 (before its
 *                  first stage and after each of its three stages) then the
 *                  down-projection's 4
 *   stream         the CUDA stream of every launch
 * All buffers are caller-owned; nothing is allocated.  Errors as
 * dq_linear_forward_ex (each layer's shape is checked as for that call); device
 * errors land in each layer's workspace status word (dq_read_device_status).
 */
#define DQ_FFN_SEPARATE_STATISTICS 1
int dq_ffn_forward(const void* X, int T, int H, int W, const int* cube_up, const int* cube_down, int Ci, int Cf,
                   int Co, int rank_up, int rank_down, const void* packed_up, const void* L1_up, const void* L2_up,
                   const void* packed_down, const void* L1_down, const void* L2_down, void* Hid, void* Y,
                   void* ws_up, size_t ws_up_bytes, void* ws_down, size_t ws_down_bytes, int ffn_flags,
                   void* const* stage_events, void* stream);

/*
 * dq_ffn_forward with forward options per layer (NULL: the defaults): kernel_group,
 * kernel_product and delta_scale as dq_linear_forward_opts takes them (an FP8
 * kernel-token product needs that layer's weight packed with DQ_PACK_C2, and
 * each workspace is sized by dq_workspace_layout_opts for its layer's options).
 * The up-projection's epilogue is GELU whatever opts_up->epilogue says; the
 * down-projection's must be DQ_EPILOGUE_NONE.  The statistics fuse only under the
 * two-pass delta scale (opts_down->delta_scale = DQ_DELTA_SCALE_AMAX).
 */
int dq_ffn_forward_opts(const void* X, int T, int H, int W, const int* cube_up, const int* cube_down, int Ci, int Cf,
                        int Co, int rank_up, int rank_down, const dq_forward_options* opts_up,
                        const dq_forward_options* opts_down, const void* packed_up, const void* L1_up,
                        const void* L2_up, const void* packed_down, const void* L1_down, const void* L2_down, void* Hid,
                        void* Y, void* ws_up, size_t ws_up_bytes, void* ws_down, size_t ws_down_bytes, int ffn_flags,
                        void* const* stage_events, void* stream);

/*
 * *fused = 1 when dq_ffn_forward forms the down-projection's statistics in the
 * up-projection's epilogue for this lattice and pair of cubes, else 0.  Host
 * only (no device call); O(T H W) the first time a pair of partitions is asked.
 */
int dq_ffn_fused_statistics(int T, int H, int W, const int* cube_up, const int* cube_down, int* fused);

/*
 * As dq_linear_forward_ex with HOST X and Y (pinned for asynchronous copies):
 * copies X to X_dev, runs the layer, copies Y_dev to Y, all on `stream`.
 * X_dev (N x Ci BF16) and Y_dev (N x Co BF16) are caller-owned device buffers.
 */
int dq_linear_forward_host(const void* X_host, int T, int H, int W, int t, int h, int w, int Ci, int Co,
                           int rank, const void* packed_W, const void* L1_mma, const void* L2_slab,
                           void* Y_host, void* X_dev, void* Y_dev, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * As dq_linear_forward_host with host_flags:
 *   DQ_HOST_OVERLAP_PREVIOUS  the copy of X into X_dev may start as soon as the
 *       previous call of this entry point on the device has read X_dev for the
 *       last time (its encode stage), instead of after all work enqueued on
 *       `stream` so far: the copy of one step's input then overlaps the previous
 *       step's products and copy out.  Work the caller enqueues on `stream`
 *       between two such calls must not touch X_dev.
 * dq_linear_forward_host is this call with host_flags = 0.  Both copy X in
 * T-slabs of whole cube layers, start each slab's statistics pass when its
 * rows have arrived, and copy the frames finished by each range of the main
 * product's row tiles back while the next range computes; the call's work
 * (copies included) ends on `stream`.  Copy streams and events are created on
 * the first call on a device and kept until exit.
 */
#define DQ_HOST_OVERLAP_PREVIOUS 1

int dq_linear_forward_host_ex(const void* X_host, int T, int H, int W, int t, int h, int w, int Ci, int Co,
                              int rank, const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y_host,
                              void* X_dev, void* Y_dev, void* workspace, size_t workspace_bytes, int host_flags,
                              void* stream);

/*
 * Forward pass for callers that cannot allocate device memory (code running
 * under a fixed memory plan such as CUDA-graph capture, processes whose
 * allocator owns all device memory, embedded callers that may not grow their
 * footprint).  The paper has no counterpart; this is a property of the library.
 * Same layer and arguments as dq_linear_forward; the caller still provides X,
 * the packed weight, the factors and Y.  The scratch workspace is a fixed
 * 32 MiB array in device memory that the library declares: every GPU that
 * loads the library holds it until the process exits.  Layers whose
 * dq_workspace_bytes exceeds 32 MiB are refused with
 * DQ_ERR_WORKSPACE_TOO_SMALL before anything is launched.  No cudaMalloc,
 * cudaFree or other allocating call is made.
 * The first call on a device looks up the array's device address (no stream
 * operation); make that first call before any stream capture all the same,
 * since the lookup may load the library's device code.  All calls share the
 * one array and it keeps the previous call's contents: each call clears the
 * status word and the accumulators it needs on its own stream, so calls
 * ordered on one stream are independent, but calls that may overlap on the GPU
 * (different streams without ordering) race on it.  Device-side errors (a
 * packed weight that does not match, a bounded wait that ran out) go to the
 * array's status word: read it with
 * dq_read_device_status(DQ_NOALLOC_WORKSPACE, stream, ...).
 */
int dq_linear_forward_noalloc(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                              const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y, void* stream);

/* The workspace argument of dq_read_device_status that names the fixed array
 * of dq_linear_forward_noalloc. */
#define DQ_NOALLOC_WORKSPACE ((const void*)1)

/*
 * Synchronises `stream`, reads the workspace status word into *status, and
 * clears it when `clear` is nonzero.  workspace: a caller workspace, NULL for
 * the library workspace of dq_linear_forward (DQ_OK when none exists yet), or
 * DQ_NOALLOC_WORKSPACE for the array of dq_linear_forward_noalloc.
 */
int dq_read_device_status(const void* workspace, void* stream, int* status, int clear);

/*
 * Failure-detection self test: launches one kernel that waits on an mbarrier
 * nothing arrives at, with a wait budget of budget_us microseconds.  It must
 * come back with DQ_ERR_DEVICE_TIMEOUT in *status (and the context usable).
 */
int dq_selftest_bounded_wait(int budget_us, void* stream, int* status);

/*
 * GELU self test: out[i] = the feed-forward epilogue's GELU of in[i] (DQ_EPILOGUE_GELU's
 * fp32 evaluation, two values at a time as the epilogue takes them), for n device fp32
 * values; asynchronous.
 */
int dq_selftest_gelu(const float* in, long long n, float* out, void* stream);

/*
 * Format self test: for each of the n fp32 values in `in` (device), writes the
 * E2M1 code (low nibble, round to nearest even, saturating), the E4M3 code
 * (same rules) and that E4M3 code's value, using the very conversions the
 * quantisers use.  All buffers are device memory of n elements; asynchronous.
 */
int dq_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* e4m3_value,
                        void* stream);

/*
 * Quotient self test: the quantisers compute fl32(a / b) (b > 0) from the
 * correctly rounded reciprocal of b with one product and one FMA correction
 * step.  This draws n operand pairs from a counter-based hash of `seed` on the
 * device and counts, into *mismatches (host), the pairs where that quotient
 * differs in any bit from IEEE division; first_ab (host, 2 floats) receives
 * the first mismatching pair.  Synchronous.
 */
int dq_selftest_divide(long long n, uint64_t seed, unsigned long long* mismatches, float* first_ab, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DELTAQUANT_H */
