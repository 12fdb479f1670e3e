// Internal layout arithmetic shared by the host packer/launcher and the
// kernels of libdeltaquant.  Everything here is index math: cube partition
// (DeltaQuant note, key design 2), the scale-factor layout of the
// block-scaled tensor-core product, and the workspace / packed-weight
// carve-up declared in include/deltaquant.h.
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define DQ_HD __host__ __device__ __forceinline__
#else
#define DQ_HD inline
#endif

namespace dq {

constexpr int kAlign = 256;

DQ_HD long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
DQ_HD size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
DQ_HD int imin(int a, int b) { return a < b ? a : b; }

// Cube partition of the T x H x W token lattice into t x h x w cubes.
struct Geom {
    int T, H, W, t, h, w;
    int KT, KH, KW;
    long long N, K;
};

DQ_HD Geom make_geom(int T, int H, int W, int t, int h, int w) {
    Geom g;
    g.T = T; g.H = H; g.W = W; g.t = t; g.h = h; g.w = w;
    g.KT = (int)cdiv(T, t); g.KH = (int)cdiv(H, h); g.KW = (int)cdiv(W, w);
    g.N = (long long)T * H * W;
    g.K = (long long)g.KT * g.KH * g.KW;
    return g;
}

// First cube-major row of cube (kt, kh, kw): all kt-slabs before it are full
// in t, all cube-rows before it in this slab are full in h, all cubes before
// it in this cube-row are full in w.
DQ_HD long long cube_first_row(const Geom& g, int kt, int kh, int kw) {
    int st = imin(g.t, g.T - kt * g.t);
    int sh = imin(g.h, g.H - kh * g.h);
    return (long long)kt * g.t * g.H * g.W + (long long)st * ((long long)kh * g.h * g.W + (long long)sh * kw * g.w);
}

// Natural token n = (tt*H + hh)*W + ww  ->  cube-major row and cube index.
DQ_HD void token_to_row(const Geom& g, long long n, long long* row, long long* cube) {
    int ww = (int)(n % g.W);
    int hh = (int)((n / g.W) % g.H);
    int tt = (int)(n / ((long long)g.W * g.H));
    int kt = tt / g.t, kh = hh / g.h, kw = ww / g.w;
    int sh = imin(g.h, g.H - kh * g.h), sw = imin(g.w, g.W - kw * g.w);
    int dt = tt - kt * g.t, dh = hh - kh * g.h, dw = ww - kw * g.w;
    *row = cube_first_row(g, kt, kh, kw) + ((long long)dt * sh + dh) * sw + dw;
    *cube = ((long long)kt * g.KH + kh) * g.KW + kw;
}

// Cube-major row -> natural token and cube index (inverse of token_to_row).
DQ_HD void row_to_token(const Geom& g, long long row, long long* n, long long* cube) {
    long long slab = (long long)g.t * g.H * g.W;
    int kt = (int)(row / slab);
    long long r1 = row - (long long)kt * slab;
    int st = imin(g.t, g.T - kt * g.t);
    long long crow = (long long)st * g.h * g.W;
    int kh = (int)(r1 / crow);
    long long r2 = r1 - (long long)kh * crow;
    int sh = imin(g.h, g.H - kh * g.h);
    long long csz = (long long)st * sh * g.w;
    int kw = (int)(r2 / csz);
    int r3 = (int)(r2 - (long long)kw * csz);
    int sw = imin(g.w, g.W - kw * g.w);
    int dt = r3 / (sh * sw);
    int rem = r3 - dt * sh * sw;
    int dh = rem / sw, dw = rem - dh * sw;
    *n = ((long long)(kt * g.t + dt) * g.H + (kh * g.h + dh)) * g.W + (kw * g.w + dw);
    *cube = ((long long)kt * g.KH + kh) * g.KW + kw;
}

// Natural token n -> its cube in the partition g, its place in the cube's (t,h,w) order and the
// cube's token count (edge cubes hold the tokens the lattice leaves them).
DQ_HD void cube_pos(const Geom& g, long long n, long long* cube, int* pos, int* count) {
    int ww = (int)(n % g.W);
    int hh = (int)((n / g.W) % g.H);
    int tt = (int)(n / ((long long)g.W * g.H));
    int kt = tt / g.t, kh = hh / g.h, kw = ww / g.w;
    int st = imin(g.t, g.T - kt * g.t), sh = imin(g.h, g.H - kh * g.h), sw = imin(g.w, g.W - kw * g.w);
    *pos = ((tt - kt * g.t) * sh + (hh - kh * g.h)) * sw + (ww - kw * g.w);
    *count = st * sh * sw;
    *cube = ((long long)kt * g.KH + kh) * g.KW + kw;
}

// Scale-factor layout (see include/deltaquant.h): byte offset of the scale of
// 16-column block `blk` in row `row` of a matrix with `cols` columns.
DQ_HD size_t sf_offset(long long row, int blk, int cols) {
    long long grp = (row >> 7) * (long long)(cols >> 6) + (blk >> 2);
    return (size_t)grp * 512 + (size_t)((row & 31) * 16 + ((row & 127) >> 5) * 4 + (blk & 3));
}

DQ_HD size_t sf_bytes(long long rows, int cols) { return (size_t)cdiv(rows, 128) * (size_t)(cols / 64) * 512; }

// A-operand scale layout (the delta scales; see include/deltaquant.h): per
// 128-row group and 256-column K step two 4 KB blocks, one per pair of
// 64-column blocks, each 128 rows x 32 bytes in 8-row x 16-byte core matrices;
// row r of the group holds the four scales of 64-column block kb at 32-bit
// word 4 (kb % 2) + r / 32 of its 32 bytes (the other six words are unused).
DQ_HD size_t sfa_offset(long long row, int blk, int cols) {
    const int kb = blk >> 2, r = (int)(row & 127);
    const long long block = ((row >> 7) * (long long)(cols >> 8) + (kb >> 2)) * 2 + ((kb >> 1) & 1);
    return (size_t)block * 4096 + (size_t)((r >> 3) * 256 + (kb & 1) * 128 + (r & 7) * 16 + (r >> 5) * 4 + (blk & 3));
}

DQ_HD size_t sfa_bytes(long long rows, int cols) { return (size_t)cdiv(rows, 128) * (size_t)(cols / 256) * 8192; }

// B-operand scale layout (the weight scales of the packed weight; see
// include/deltaquant.h): per 256-row tile and 64-column block one 4 KB block
// of 128 lanes x 32 bytes in 8-row x 16-byte core matrices, lane r holding the
// scales of rows 32 c + r % 32 (c = 0..3) and 128 + 32 c + r % 32 in its eight
// 32-bit words; lanes r, r + 32, r + 64, r + 96 hold the same bytes.  Returns
// the offset of the copy in lane r % 32; the copy in lane r % 32 + 32 q sits
// 1024 q bytes further.
DQ_HD size_t sfb_offset(long long row, int blk, int cols) {
    const int nl = (int)(row & 255), kb = blk >> 2;
    const int i = nl & 31, word = 4 * (nl >> 7) + ((nl >> 5) & 3), b = 4 * word + (blk & 3);
    const long long block = (row >> 8) * (long long)(cols >> 6) + kb;
    return (size_t)block * 4096 + (size_t)((i >> 3) * 256 + (b >> 4) * 128 + (i & 7) * 16 + (b & 15));
}

DQ_HD size_t sfb_bytes(long long rows, int cols) { return (size_t)cdiv(rows, 256) * (size_t)(cols / 64) * 4096; }

// Scale layout of the FP8 operand of C2 weights (one UE8M0 exponent per 32 channels, B operand of
// a kind::mxf8f6f4 product with one scale per 32 K): the four MMAs (K = 32 each) of a 128-channel
// stage read byte 0..3 of the same 32-bit tensor-memory word, so a stage's exponents of a 256-row
// tile fill one 4 KB block laid out as the B-operand layout above with four 32-channel blocks in
// place of four 16-channel blocks: block j of row o sits where sfb_offset puts 16-channel block j
// of a matrix with cols / 2 columns.
DQ_HD size_t c2_sf_offset(long long row, int blk32, int cols) { return sfb_offset(row, blk32, cols / 2); }
DQ_HD size_t c2_sf_bytes(long long rows, int cols) { return sfb_bytes(rows, cols / 2); }

DQ_HD int slab_width(int rank) { return (int)(cdiv(2 * rank, 64) * 64); }

// Packed weight blob header (first 256 bytes of the blob).
struct PackedHeader {
    uint32_t magic, version;
    int32_t Co, Ci, rank, slab;
    float S_W;
    uint32_t flags;      // kPackedHasBias: the bias section holds the layer's bias
    uint64_t off_codes, off_scales, off_dqw, total, off_bias;
};

constexpr uint32_t kPackedHasBias = 1u;
// Restricted-scale (C2) weights: group scales {1, 1.5} x 2^e, S_W = amax / (6 * 384), and the
// dqw section holding the FP8 form of q s_b (E4M3 codes, Co x Ci, then their UE8M0 exponents per
// 32 channels in the 1X scale layout c2_sf_offset) instead of BF16 q s_b.
constexpr uint32_t kPackedC2 = 2u;

struct PackedLayout {
    size_t total, off_codes, off_scales, off_dqw, off_bias;
    int Co, Ci, rank, slab;
};

DQ_HD PackedLayout packed_layout(int Co, int Ci, int rank) {
    PackedLayout L;
    L.Co = Co; L.Ci = Ci; L.rank = rank; L.slab = slab_width(rank);
    size_t off = kAlign;
    L.off_codes = off;
    off = align_up(off + (size_t)Co * (Ci / 2), kAlign);
    L.off_scales = off;
    off = align_up(off + sfb_bytes(Co, Ci), kAlign);
    L.off_dqw = off;
    off = align_up(off + (size_t)Co * Ci * 2, kAlign);
    L.off_bias = off;
    off = align_up(off + (size_t)Co * 4, kAlign);
    L.total = off;
    return L;
}

// Number of splits of the channel dimension in the cube-quantise kernels:
// work items are (box, split), so more splits even out the last wave of the
// persistent grid; each split leaves its own partial sums of X L1, reduced in
// a fixed order.
DQ_HD int quant_splits(int Ci) {
    int chunks = Ci / 64;
    int s = 8;
    while (s > 1 && chunks % s) s--;
    return s;
}

struct WsLayout {
    size_t total, off_status, off_scalars, off_kamax, off_s8, off_q8, off_q8_bf16, off_dcodes, off_dscales,
        off_u_part, off_u_hilo, off_p, off_means, off_prov;
    long long N, K, N_pad, K_pad;
    int splits, slab;
};

// kgroup: 0 = one FP8 scale per kernel token; 64 = one per 64 channels, whose
// kernel tokens enter the product as BF16 hi + lo (twice the columns)
// pow2_single: the single-read quantiser (power-of-two delta scale), which also keeps one provisional
// scale exponent per (row, 64-channel chunk)
DQ_HD WsLayout ws_layout(const Geom& g, int Ci, int Co, int rank, int kgroup = 0, bool fp8_product = false,
                         bool pow2_single = false) {
    WsLayout L;
    L.N = g.N; L.K = g.K;
    L.N_pad = cdiv(g.N, 128) * 128;
    L.K_pad = cdiv(g.K, 128) * 128;
    L.splits = quant_splits(Ci);
    L.slab = slab_width(rank);
    size_t off = 0;
    L.off_status = off;   off = align_up(off + 16, kAlign);
    L.off_scalars = off;  off = align_up(off + 16, kAlign);
    L.off_kamax = off;    off = align_up(off + (size_t)g.K * 4, kAlign);
    L.off_s8 = off;       off = align_up(off + (size_t)g.K * (kgroup ? Ci / kgroup : 1) * 4, kAlign);
    L.off_q8 = off;       off = align_up(off + (size_t)g.K * Ci, kAlign);
    // BF16 operand of the exact kernel-token product (the FP8 product reads q8 itself)
    L.off_q8_bf16 = off;  off = align_up(off + (fp8_product ? 0 : (size_t)L.K_pad * Ci * 2 * (kgroup ? 2 : 1)), kAlign);
    L.off_dcodes = off;   off = align_up(off + (size_t)g.N * (Ci / 2), kAlign);
    L.off_dscales = off;  off = align_up(off + sfa_bytes(g.N, Ci), kAlign);
    L.off_u_part = off;   off = align_up(off + (size_t)L.splits * g.N * rank * 4, kAlign);
    L.off_u_hilo = off;   off = align_up(off + (size_t)g.N * L.slab * 2, kAlign);
    L.off_p = off;        off = align_up(off + (size_t)g.K * Co * 4, kAlign);
    // fp32 kernel tokens (written by the statistics pass, read by the encode pass)
    L.off_means = off;    off = align_up(off + (size_t)g.K * Ci * 4, kAlign);
    L.off_prov = off;     off = align_up(off + (pow2_single ? (size_t)g.N * (Ci / 64) : 0), kAlign);
    L.total = off;
    return L;
}

}  // namespace dq
