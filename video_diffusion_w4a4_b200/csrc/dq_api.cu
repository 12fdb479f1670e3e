// Online entry points of libdeltaquant: argument checks, workspace carve-up,
// TMA tensor maps, and the launch sequence of the DeltaQuant layer
//   a1 cube statistics -> a2 cube encode -> (c) kernel-token product ->
//   (b) main FP4 product with low-rank slab and scatter epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <functional>
#include <map>
#include <mutex>
#include <vector>

#include "../../include/deltaquant.h"
#include "dq_common.h"
#include "dq_internal.h"

namespace {

using dq::Geom;

constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // 2 s per wait: far above any legitimate wait

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over a row-major matrix: inner = elements per row, outer = rows.
bool map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t outer,
            uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * (uint64_t)esize};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return f(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map over X viewed as T x H x W x Ci (BF16), boxes of 64 channels x bw x bh x bt tokens.
bool map_x(CUtensorMap* m, const void* X, const Geom& g, int Ci, int bw, int bh, int bt) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {(cuuint64_t)Ci, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T};
    cuuint64_t strides[3] = {(cuuint64_t)Ci * 2, (cuuint64_t)g.W * Ci * 2, (cuuint64_t)g.H * g.W * Ci * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)bw, (cuuint32_t)bh, (cuuint32_t)bt};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(X), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the A-operand scale layout (dq_sfa_offset): dim 0 the bytes of a
// 256-byte line, dim 1 the 32 (Ci/256) lines of one 128-row group (8192 bytes
// per K step of 256 channels), dim 2 the row groups.  Boxes of one K step.
bool map_sfa(CUtensorMap* m, const void* base, int Ci, uint64_t row_groups) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {256, (cuuint64_t)Ci / 256 * 32, row_groups};
    cuuint64_t strides[2] = {256, (cuuint64_t)Ci / 256 * 8192};
    cuuint32_t box[3] = {256, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over the K x Ci fp32 kernel tokens, boxes of 64 channels x `rows` consecutive cubes.
bool map_means(CUtensorMap* m, const void* base, int Ci, long long K, int rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {(cuuint64_t)Ci, (cuuint64_t)K};
    cuuint64_t strides[1] = {(cuuint64_t)Ci * 4};
    cuuint32_t box[2] = {64, (cuuint32_t)rows};
    cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the B-operand scale layout (dq_sfb_offset) of a matrix with `cols`
// 16-column blocks' worth of columns: dim 0 the bytes of a 256-byte line, dim 1 the
// 16 lines of each 4096-byte block (cols / 64 blocks per 256-row tile), dim 2 the
// 256-row tiles.  Boxes of `blocks` consecutive 4096-byte blocks: four (one K step
// of 256 channels) for the FP4 weight scales, one (a 128-channel stage) for the
// UE8M0 exponents of C2 weights (cols = Ci / 2).
bool map_sfb(CUtensorMap* m, const void* base, int cols, int Co, int blocks = 4) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {256, (cuuint64_t)cols / 64 * 16, (cuuint64_t)Co / 256};
    cuuint64_t strides[2] = {256, (cuuint64_t)cols / 64 * 4096};
    cuuint32_t box[3] = {256, (cuuint32_t)(16 * blocks), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p) { return ((uintptr_t)p & 255u) == 0; }

// Text of the last CUDA runtime error an entry point of this thread returned DQ_ERR_CUDA for.
thread_local char g_last_cuda_error[160] = "";

int map_fail(const char* which) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed for %s", which);
    return DQ_ERR_CUDA;
}

int cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", where, cudaGetErrorString(e));
    return DQ_ERR_CUDA;
}

int check_shape(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank) {
    if (T <= 0 || H <= 0 || W <= 0 || t <= 0 || h <= 0 || w <= 0) return DQ_ERR_INVALID_ARG;
    if (t > T || h > H || w > W) return DQ_ERR_UNSUPPORTED_SHAPE;
    if (Ci < 256 || Co < 256 || Ci % 256 || Co % 256) return DQ_ERR_UNSUPPORTED_SHAPE;
    if (rank < 16 || rank > 128 || rank % 16 || rank > Ci || rank > Co) return DQ_ERR_UNSUPPORTED_SHAPE;
    if ((long long)T * H * W >= (1ll << 31)) return DQ_ERR_UNSUPPORTED_SHAPE;
    return DQ_OK;
}

int check_options(const dq_forward_options& o) {
    if (o.kernel_group != DQ_KERNEL_SCALE_PER_TOKEN && o.kernel_group != DQ_KERNEL_SCALE_GROUP64)
        return DQ_ERR_INVALID_ARG;
    if (o.kernel_product != DQ_KERNEL_PRODUCT_BF16 && o.kernel_product != DQ_KERNEL_PRODUCT_FP8) return DQ_ERR_INVALID_ARG;
    // the FP8 product carries the kernel-token scale in its epilogue: one per token
    if (o.kernel_product == DQ_KERNEL_PRODUCT_FP8 && o.kernel_group != DQ_KERNEL_SCALE_PER_TOKEN)
        return DQ_ERR_INVALID_ARG;
    if (o.delta_scale != DQ_DELTA_SCALE_AMAX && o.delta_scale != DQ_DELTA_SCALE_POW2) return DQ_ERR_INVALID_ARG;
    // the single-read quantiser forms per-token kernel scales in its fix-up pass
    if (o.delta_scale == DQ_DELTA_SCALE_POW2 && o.kernel_group != DQ_KERNEL_SCALE_PER_TOKEN) return DQ_ERR_INVALID_ARG;
    if (o.epilogue != DQ_EPILOGUE_NONE && o.epilogue != DQ_EPILOGUE_GELU) return DQ_ERR_INVALID_ARG;
    return DQ_OK;
}

// Copy streams and events of the pipelined host-buffer entry point, one set per device, created on
// first use and kept until the process exits; one call at a time uses them.
constexpr int kHostSlabs = 8;    // T-slabs of X copied in (at most; whole cube layers)
constexpr int kHostChunks = 4;   // row-tile ranges of the main product whose frames are copied out
struct Aux {
    std::mutex mu;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev[2 + kHostSlabs + kHostChunks] = {};
    cudaEvent_t x_free = nullptr;   // recorded after a call's last read of X_dev (its encode pass)
    bool x_free_recorded = false;
};
std::mutex g_aux_mu;
std::map<int, Aux> g_aux;

int cuda_fail(cudaError_t e, const char* where);

int host_aux(Aux** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_aux_mu);
    Aux& A = g_aux[dev];
    if (!A.in) {
        cudaError_t e;
        if ((e = cudaStreamCreateWithFlags(&A.in, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&A.out, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "copy streams");
        for (cudaEvent_t& ev : A.ev)
            if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e, "events");
        if ((e = cudaEventCreateWithFlags(&A.x_free, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e, "events");
    }
    *out = &A;
    return DQ_OK;
}

struct LibWorkspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
std::mutex g_ws_mu;
std::map<int, LibWorkspace> g_ws;

int ensure_lib_workspace(size_t need, void** ws) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    LibWorkspace& L = g_ws[dev];
    if (L.bytes < need) {
        if (L.ptr) {
            cudaDeviceSynchronize();
            cudaFree(L.ptr);
            L.ptr = nullptr;
            L.bytes = 0;
        }
        if (cudaMalloc(&L.ptr, need) != cudaSuccess) {
            L.ptr = nullptr;
            return DQ_ERR_ALLOC;
        }
        cudaMemset(L.ptr, 0, 256);
        L.bytes = need;
    }
    *ws = L.ptr;
    return DQ_OK;
}

}  // namespace

extern "C" {

int dq_workspace_layout_opts(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                             const dq_forward_options* opts, dq_workspace_layout* out) {
    if (!out) return DQ_ERR_INVALID_ARG;
    int rc = check_shape(T, H, W, t, h, w, Ci, Co, rank);
    if (rc) return rc;
    const dq_forward_options o = opts ? *opts : dq_forward_options{};
    if ((rc = check_options(o))) return rc;
    const int kernel_group = o.kernel_group;
    dq::WsLayout L = dq::ws_layout(dq::make_geom(T, H, W, t, h, w), Ci, Co, rank, kernel_group,
                                   o.kernel_product == DQ_KERNEL_PRODUCT_FP8, o.delta_scale == DQ_DELTA_SCALE_POW2);
    out->total_bytes = L.total;
    out->off_status = L.off_status;
    out->off_scalars = L.off_scalars;
    out->off_kamax = L.off_kamax;
    out->off_s8 = L.off_s8;
    out->off_q8 = L.off_q8;
    out->off_q8_bf16 = L.off_q8_bf16;
    out->off_dcodes = L.off_dcodes;
    out->off_dscales = L.off_dscales;
    out->off_u_part = L.off_u_part;
    out->off_u_hilo = L.off_u_hilo;
    out->off_p = L.off_p;
    out->off_means = L.off_means;
    out->N = L.N;
    out->K = L.K;
    out->N_pad = L.N_pad;
    out->K_pad = L.K_pad;
    out->splits = L.splits;
    out->slab = L.slab;
    out->kernel_group = kernel_group;
    out->off_prov = L.off_prov;
    return DQ_OK;
}

int dq_workspace_layout_grouped(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank, int kernel_group,
                                dq_workspace_layout* out) {
    dq_forward_options o{};
    o.kernel_group = kernel_group;
    return dq_workspace_layout_opts(T, H, W, t, h, w, Ci, Co, rank, &o, out);
}

int dq_workspace_layout_get(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                            dq_workspace_layout* out) {
    return dq_workspace_layout_grouped(T, H, W, t, h, w, Ci, Co, rank, DQ_KERNEL_SCALE_PER_TOKEN, out);
}

int dq_workspace_bytes_grouped(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank, int kernel_group,
                               size_t* bytes) {
    if (!bytes) return DQ_ERR_INVALID_ARG;
    dq_workspace_layout L;
    int rc = dq_workspace_layout_grouped(T, H, W, t, h, w, Ci, Co, rank, kernel_group, &L);
    if (rc) return rc;
    *bytes = L.total_bytes;
    return DQ_OK;
}

int dq_workspace_bytes(int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank, size_t* bytes) {
    if (!bytes) return DQ_ERR_INVALID_ARG;
    dq_workspace_layout L;
    int rc = dq_workspace_layout_get(T, H, W, t, h, w, Ci, Co, rank, &L);
    if (rc) return rc;
    *bytes = L.total_bytes;
    return DQ_OK;
}

}  // extern "C"

namespace {

// A split of one forward into pieces for the host-buffer entry point: the statistics pass in T-slabs
// of whole cube layers (before_slab(i) runs before slab i's launch, e.g. to wait for its copy of X),
// the main product in ranges of 256-row tiles (after_chunk(k, last cube-major row done) after each).
struct Pipeline {
    std::vector<int> kt_cuts;    // cube-layer boundaries of the slabs: 0 = kt_cuts[0] < ... = KT
    std::vector<int> tile_cuts;  // row-tile boundaries of the main-product launches: 0 = ... = ceil(N / 256)
    std::function<int(int)> before_slab;
    std::function<int()> after_encode;
    std::function<int(int, long long)> after_chunk;
};

// The two halves of the producer-epilogue fusion of a feed-forward block: the up-projection's main
// product forms the down-projection's statistics pass (c_means set), and the down-projection's
// statistics kernel then only forms X L1 (stats_given).
struct FfnHooks {
    Geom cg{};
    float* c_means = nullptr;
    uint32_t* c_kamax = nullptr;
    uint32_t* c_scalars = nullptr;
    bool stats_given = false;
};

// Whether the down-projection's statistics pass can run in the up-projection's epilogue: every
// cube of the consumer partition gd must hold at most 32 tokens and occupy consecutive cube-major
// rows of the producer partition gu, in its own (t,h,w) order, inside one aligned group of 32 rows
// (the rows one epilogue warp holds).  O(N) on the host; the answer is kept per pair of partitions.
bool ffn_stats_fusable(const Geom& gu, const Geom& gd) {
    if ((long long)gd.t * gd.h * gd.w > 32) return false;
    static std::mutex mu;
    static std::map<std::vector<int>, bool> memo;
    const std::vector<int> key = {gu.T, gu.H, gu.W, gu.t, gu.h, gu.w, gd.t, gd.h, gd.w};
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = memo.find(key);
        if (it != memo.end()) return it->second;
    }
    std::vector<long long> base((size_t)gd.K, -1);
    bool ok = true;
    for (long long n = 0; ok && n < gu.N; n++) {
        long long ru = 0, ku = 0, kd = 0;
        int pos = 0, cnt = 0;
        dq::token_to_row(gu, n, &ru, &ku);
        dq::cube_pos(gd, n, &kd, &pos, &cnt);
        const long long b = ru - pos;
        if (base[(size_t)kd] < 0)
            base[(size_t)kd] = b;
        else if (base[(size_t)kd] != b)
            ok = false;
        if ((b >> 5) != ((b + cnt - 1) >> 5)) ok = false;
    }
    std::lock_guard<std::mutex> lk(mu);
    memo[key] = ok;
    return ok;
}

int forward_impl(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                 const dq_forward_options* opts, const void* packed_W, const void* L1_mma, const void* L2_slab,
                 void* Y, void* workspace, size_t workspace_bytes, int stage_mask, void* const* stage_events,
                 void* stream, const Pipeline* pipe, const FfnHooks* hk = nullptr) {
    int rc = check_shape(T, H, W, t, h, w, Ci, Co, rank);
    if (rc) return rc;
    const dq_forward_options o = opts ? *opts : dq_forward_options{};
    if ((rc = check_options(o))) return rc;
    const int kg = o.kernel_group;
    const bool fp8prod = o.kernel_product == DQ_KERNEL_PRODUCT_FP8;
    const bool pow2 = o.delta_scale == DQ_DELTA_SCALE_POW2;
    const bool stats_given = hk && hk->stats_given;
    if (stats_given && (pow2 || (long long)t * h * w > 32)) return DQ_ERR_INVALID_ARG;
    if (!X || !packed_W || !L1_mma || !L2_slab || !Y || !workspace) return DQ_ERR_INVALID_ARG;
    if (stage_mask <= 0 || (stage_mask & ~(DQ_STAGE_ALL | DQ_STAGE_STATS | DQ_STAGE_ENCODE))) return DQ_ERR_INVALID_ARG;
    const bool do_stats = stage_mask & (DQ_STAGE_QUANTIZE | DQ_STAGE_STATS);
    const bool do_encode = stage_mask & (DQ_STAGE_QUANTIZE | DQ_STAGE_ENCODE);
    if (!aligned(X) || !aligned(packed_W) || !aligned(L1_mma) || !aligned(L2_slab) || !aligned(Y) ||
        !aligned(workspace))
        return DQ_ERR_ALIGNMENT;
    const Geom g = dq::make_geom(T, H, W, t, h, w);
    const dq::WsLayout wl = dq::ws_layout(g, Ci, Co, rank, kg, fp8prod, pow2);
    if (workspace_bytes < wl.total) return DQ_ERR_WORKSPACE_TOO_SMALL;
    if (!encode_fn()) return DQ_ERR_NO_DEVICE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* ws = (uint8_t*)workspace;
    const dq::PackedLayout pl = dq::packed_layout(Co, Ci, rank);
    const uint8_t* pw = (const uint8_t*)packed_W;

    dq::QuantParams qp;
    memset(&qp, 0, sizeof(qp));
    qp.g = g;
    qp.Ci = Ci;
    qp.rank = rank;
    qp.slab = wl.slab;
    qp.splits = wl.splits;
    qp.kgroup = kg;
    qp.fp8_product = fp8prod;
    qp.pow2 = pow2;
    qp.chunks_per_split = Ci / 64 / wl.splits;
    qp.big = (long long)t * h * w > 128;
    if (!qp.big) {
        // boxes of t x h x (nw w) tokens: nw whole cubes side by side along w
        // (as many as fit in 128 tokens, then evened out over the boxes of a cube row)
        const int nw_max = dq::imin(128 / (t * h * w), g.KW);
        qp.nbw = (int)dq::cdiv(g.KW, nw_max);
        qp.nw = (int)dq::cdiv(g.KW, qp.nbw);
        qp.bt = t;
        qp.bh = h;
        qp.bw = qp.nw * w;
        qp.n_boxes = g.KT * g.KH * qp.nbw;
        qp.m_rows = qp.nw;
        qp.stat_pairs = t * h * w >= 16;   // then at most 8 cubes per box, one per compute warp
    } else {
        // boxes are segments of up to 128 tokens of one (t, h) row inside one cube
        qp.nw = 1;
        qp.bt = 1;
        qp.bh = 1;
        qp.bw = dq::imin(w, 128);
        qp.nseg = (int)dq::cdiv(w, 128);
        qp.nbw = g.KW * qp.nseg;
        qp.n_boxes = g.T * g.H * qp.nbw;
        qp.m_rows = 1;
    }
    qp.item0 = 0;
    qp.item1 = qp.n_boxes * qp.splits;
    qp.means = (float*)(ws + wl.off_means);
    qp.status = (int*)(ws + wl.off_status);
    qp.scalars = (uint32_t*)(ws + wl.off_scalars);
    qp.kamax = (uint32_t*)(ws + wl.off_kamax);
    qp.s8 = (float*)(ws + wl.off_s8);
    qp.q8 = ws + wl.off_q8;
    qp.q8_bf16 = (uint16_t*)(ws + wl.off_q8_bf16);
    qp.dcodes = ws + wl.off_dcodes;
    qp.dscales = ws + wl.off_dscales;
    qp.u_part = (float*)(ws + wl.off_u_part);
    qp.u_hilo = (uint16_t*)(ws + wl.off_u_hilo);
    qp.prov = (int8_t*)(ws + wl.off_prov);
    qp.packed_w = pw;
    qp.budget_ns = kWaitBudgetNs;

    dq::GemmParams gp;
    memset(&gp, 0, sizeof(gp));
    gp.g = g;
    gp.Nout = Co;
    gp.Ci = Ci;
    gp.scalars = qp.scalars;
    gp.packed_w = pw;
    gp.status = qp.status;
    gp.budget_ns = kWaitBudgetNs;

    auto rec = [&](int i) {
        if (stage_events && stage_events[i]) cudaEventRecord((cudaEvent_t)stage_events[i], st);
    };
    rec(0);
    if (do_stats || do_encode) {
        CUtensorMap tm_x, tm_l1, tm_m;
        cudaError_t e0;
        if (!map_x(&tm_x, X, g, Ci, qp.bw, qp.bh, qp.bt)) return map_fail("X");
        if (!map_means(&tm_m, ws + wl.off_means, Ci, g.K, qp.m_rows)) return map_fail("kernel tokens");
        if (!map_2d(&tm_l1, L1_mma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Ci, rank, 64, rank)) return map_fail("L1");
        cudaError_t e;
        if (do_stats && !stats_given) {
            if ((e0 = cudaMemsetAsync(ws + wl.off_scalars, 0, 16, st)) != cudaSuccess) return cuda_fail(e0, "memset");
            if ((e0 = cudaMemsetAsync(ws + wl.off_kamax, 0, (size_t)g.K * 4, st)) != cudaSuccess)
                return cuda_fail(e0, "memset");
        }
        // with the statistics given (a producer's epilogue formed them) no statistics pass runs: the
        // encode pass also forms X L1
        if (do_stats && !stats_given) {
            if (qp.big && (e = dq::launch_cube_means_big(tm_x, qp, st)) != cudaSuccess)
                return cuda_fail(e, "k_cube_means_big");
            // one launch over all work items, or one per T-slab (items of boxes in cube layers [kt0, kt1))
            const int items_per_layer = (qp.big ? g.t * g.H * qp.nbw : g.KH * qp.nbw) * qp.splits;
            const int nslab = pipe ? (int)pipe->kt_cuts.size() - 1 : 1;
            for (int sl = 0; sl < nslab; sl++) {
                dq::QuantParams qs = qp;
                if (pipe) {
                    if ((rc = pipe->before_slab(sl))) return rc;
                    qs.item0 = pipe->kt_cuts[sl] * items_per_layer;
                    qs.item1 = dq::imin(pipe->kt_cuts[sl + 1] * items_per_layer, qp.item1);
                }
                if (pow2) {
                    if ((e = dq::launch_cube_single(tm_x, tm_l1, qs, st)) != cudaSuccess)
                        return cuda_fail(e, "k_cube_stats (single read)");
                } else if ((e = dq::launch_cube_stats(tm_x, tm_l1, qs, st)) != cudaSuccess) {
                    return cuda_fail(e, "k_cube_stats");
                }
            }
        }
        if (do_encode && pow2) {
            if ((e = dq::launch_single_finish(X, qp, st)) != cudaSuccess) return cuda_fail(e, "k_single_finish");
        } else if (do_encode && stats_given) {
            if ((e = dq::launch_cube_encode_lowrank(tm_x, tm_m, tm_l1, qp, st)) != cudaSuccess)
                return cuda_fail(e, "k_cube_encode (with X L1)");
        } else if (do_encode && (e = dq::launch_cube_encode(tm_x, tm_m, qp, st)) != cudaSuccess) {
            return cuda_fail(e, "k_cube_encode");
        }
        if (pipe && pipe->after_encode && (rc = pipe->after_encode())) return rc;
    }
    rec(1);
    if ((stage_mask & DQ_STAGE_KERNEL_GEMM) && fp8prod) {
        // q8 (E4M3, K x Ci) times the FP8 form of C2 weights with their UE8M0 exponents per 32 channels
        CUtensorMap tm_a, tm_b, tm_fb;
        if (!map_2d(&tm_a, ws + wl.off_q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Ci, g.K, 128, 128))
            return map_fail("FP8 product A");
        if (!map_2d(&tm_b, pw + pl.off_dqw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Ci, Co, 128, 128))
            return map_fail("FP8 product B");
        if (!map_sfb(&tm_fb, pw + pl.off_dqw + (size_t)Co * Ci, Ci / 2, Co, 2)) return map_fail("FP8 product scales");
        dq::GemmParams p = gp;
        p.M = (int)g.K;
        p.tile_m0 = 0;
        p.tile_m1 = (int)dq::cdiv(g.K, 256);
        p.k_stages = Ci / 256;
        p.tile_group = 8;
        p.s8 = qp.s8;
        p.pout = (float*)(ws + wl.off_p);
        p.bias = (const float*)(pw + pl.off_bias);
        cudaError_t e = dq::launch_kernel_gemm_fp8(tm_a, tm_b, tm_fb, p, st);
        if (e != cudaSuccess) return cuda_fail(e, "FP8 kernel-token product");
    } else if (stage_mask & DQ_STAGE_KERNEL_GEMM) {
        CUtensorMap tm_a, tm_b;
        const int a_cols = kg ? 2 * Ci : Ci;   // grouped scales: [hi | lo]
        if (!map_2d(&tm_a, ws + wl.off_q8_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a_cols, g.K, 64, 128))
            return map_fail("product A");
        if (!map_2d(&tm_b, pw + pl.off_dqw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Ci, Co, 64, 128)) return map_fail("product B");
        dq::GemmParams p = gp;
        p.M = (int)g.K;
        p.tile_m0 = 0;
        p.tile_m1 = (int)dq::cdiv(g.K, 256);
        p.k_stages = a_cols / 128;
        p.b_kblocks = Ci / 64;
        p.tile_group = 8;   // the BF16 weight (Co x Ci x 2 bytes) does not stay in L2 beside the rows
        p.s8 = kg ? nullptr : qp.s8;
        p.pout = (float*)(ws + wl.off_p);
        p.bias = (const float*)(pw + pl.off_bias);
        cudaError_t e = dq::launch_kernel_gemm(tm_a, tm_b, p, st);
        if (e != cudaSuccess) return cuda_fail(e, "kernel-token product");
    }
    rec(2);
    if (stage_mask & DQ_STAGE_MAIN_GEMM) {
        CUtensorMap tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb;
        if (!map_2d(&tm_a, ws + wl.off_dcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Ci / 2, g.N, 128, 128))
            return map_fail("product A");
        if (!map_2d(&tm_b, pw + pl.off_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Ci / 2, Co, 128, 128))
            return map_fail("product B");
        if (!map_2d(&tm_sa, ws + wl.off_u_hilo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wl.slab, g.N, 64, 128))
            return map_fail("slab A");
        if (!map_2d(&tm_sb, L2_slab, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wl.slab, Co, 64, 128)) return map_fail("slab B");
        if (!map_sfa(&tm_fa, ws + wl.off_dscales, Ci, (uint64_t)dq::cdiv(g.N, 128))) return map_fail("delta scales");
        if (!map_sfb(&tm_fb, pw + pl.off_scales, Ci, Co)) return map_fail("weight scales");
        dq::GemmParams p = gp;
        p.M = (int)g.N;
        p.tile_m0 = 0;
        p.tile_m1 = (int)dq::cdiv(g.N, 256);
        p.k_stages = Ci / 256;
        p.slab_stages = wl.slab / 64;
        // weight codes and scales above 32 MB (the 720p FFN layers) are re-read by every wave of a
        // row-major walk; up to that size (the 480p projection, 20 MB) they stay in L2 and row-major wins
        p.tile_group = ((size_t)Co * (Ci / 2) + pl.off_dqw - pl.off_scales > ((size_t)32 << 20)) ? 8 : 1;
        p.p = (const float*)(ws + wl.off_p);
        p.Y = (uint16_t*)Y;
        // the feed-forward epilogue: GELU, and the consumer's statistics when a fused block asks for them
        const bool ffn = o.epilogue == DQ_EPILOGUE_GELU;
        if (ffn && hk && hk->c_means) {
            p.cg = hk->cg;
            p.c_means = hk->c_means;
            p.c_kamax = hk->c_kamax;
            p.c_scalars = hk->c_scalars;
        }
        const int nchunk = pipe ? (int)pipe->tile_cuts.size() - 1 : 1;
        for (int c = 0; c < nchunk; c++) {
            if (pipe) {
                p.tile_m0 = pipe->tile_cuts[c];
                p.tile_m1 = pipe->tile_cuts[c + 1];
            }
            cudaError_t e = ffn ? dq::launch_main_gemm_ffn(tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb, p, st)
                                : dq::launch_main_gemm(tm_a, tm_b, tm_sa, tm_sb, tm_fa, tm_fb, p, st);
            if (e != cudaSuccess) return cuda_fail(e, "main product");
            if (pipe && (rc = pipe->after_chunk(c, dq::imin(p.tile_m1 * 256, (int)g.N))))
                return rc;
        }
    }
    rec(3);
    return DQ_OK;
}

}  // namespace

extern "C" {

int dq_ffn_fused_statistics(int T, int H, int W, const int* cube_up, const int* cube_down, int* fused) {
    if (!cube_up || !cube_down || !fused) return DQ_ERR_INVALID_ARG;
    for (int i = 0; i < 3; i++)
        if (cube_up[i] <= 0 || cube_down[i] <= 0) return DQ_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || W <= 0) return DQ_ERR_INVALID_ARG;
    if (cube_up[0] > T || cube_up[1] > H || cube_up[2] > W || cube_down[0] > T || cube_down[1] > H ||
        cube_down[2] > W || (long long)T * H * W >= (1ll << 31))
        return DQ_ERR_UNSUPPORTED_SHAPE;
    *fused = ffn_stats_fusable(dq::make_geom(T, H, W, cube_up[0], cube_up[1], cube_up[2]),
                               dq::make_geom(T, H, W, cube_down[0], cube_down[1], cube_down[2]))
                 ? 1
                 : 0;
    return DQ_OK;
}

int dq_ffn_forward_opts(const void* X, int T, int H, int W, const int* cube_up, const int* cube_down, int Ci, int Cf,
                        int Co, int rank_up, int rank_down, const dq_forward_options* opts_up,
                        const dq_forward_options* opts_down, const void* packed_up, const void* L1_up,
                        const void* L2_up, const void* packed_down, const void* L1_down, const void* L2_down, void* Hid,
                        void* Y, void* ws_up, size_t ws_up_bytes, void* ws_down, size_t ws_down_bytes, int ffn_flags,
                        void* const* stage_events, void* stream) {
    if (!cube_up || !cube_down || (ffn_flags & ~DQ_FFN_SEPARATE_STATISTICS)) return DQ_ERR_INVALID_ARG;
    int rc = check_shape(T, H, W, cube_up[0], cube_up[1], cube_up[2], Ci, Cf, rank_up);
    if (rc) return rc;
    if ((rc = check_shape(T, H, W, cube_down[0], cube_down[1], cube_down[2], Cf, Co, rank_down))) return rc;
    // each layer's options; the up-projection's epilogue is GELU whatever opts_up says, the
    // down-projection's none
    dq_forward_options ou = opts_up ? *opts_up : dq_forward_options{};
    dq_forward_options od = opts_down ? *opts_down : dq_forward_options{};
    ou.epilogue = DQ_EPILOGUE_GELU;
    if (od.epilogue != DQ_EPILOGUE_NONE) return DQ_ERR_INVALID_ARG;
    if ((rc = check_options(ou)) || (rc = check_options(od))) return rc;
    // every argument is checked before the first device call, so a refused call changes nothing
    const void* ptrs[] = {X, packed_up, L1_up, L2_up, packed_down, L1_down, L2_down, Hid, Y, ws_up, ws_down};
    for (const void* q : ptrs) {
        if (!q) return DQ_ERR_INVALID_ARG;
        if (!aligned(q)) return DQ_ERR_ALIGNMENT;
    }
    const Geom gu = dq::make_geom(T, H, W, cube_up[0], cube_up[1], cube_up[2]);
    const Geom gd = dq::make_geom(T, H, W, cube_down[0], cube_down[1], cube_down[2]);
    const dq::WsLayout wu = dq::ws_layout(gu, Ci, Cf, rank_up, ou.kernel_group,
                                          ou.kernel_product == DQ_KERNEL_PRODUCT_FP8,
                                          ou.delta_scale == DQ_DELTA_SCALE_POW2);
    const dq::WsLayout wd = dq::ws_layout(gd, Cf, Co, rank_down, od.kernel_group,
                                          od.kernel_product == DQ_KERNEL_PRODUCT_FP8,
                                          od.delta_scale == DQ_DELTA_SCALE_POW2);
    if (ws_up_bytes < wu.total || ws_down_bytes < wd.total) return DQ_ERR_WORKSPACE_TOO_SMALL;
    // the fused statistics are those of the two-pass quantiser (S_delta = amax / 2688)
    const bool fuse = !(ffn_flags & DQ_FFN_SEPARATE_STATISTICS) && od.delta_scale == DQ_DELTA_SCALE_AMAX &&
                      ffn_stats_fusable(gu, gd);
    FfnHooks up, down;
    if (fuse) {
        // the up-projection's epilogue takes the maxima of the down-projection's statistics pass
        cudaStream_t st = (cudaStream_t)stream;
        uint8_t* wsd = (uint8_t*)ws_down;
        cudaError_t e;
        if ((e = cudaMemsetAsync(wsd + wd.off_scalars, 0, 16, st)) != cudaSuccess) return cuda_fail(e, "memset");
        if ((e = cudaMemsetAsync(wsd + wd.off_kamax, 0, (size_t)gd.K * 4, st)) != cudaSuccess)
            return cuda_fail(e, "memset");
        up.cg = gd;
        up.c_means = (float*)(wsd + wd.off_means);
        up.c_kamax = (uint32_t*)(wsd + wd.off_kamax);
        up.c_scalars = (uint32_t*)(wsd + wd.off_scalars);
        down.stats_given = true;
    }
    rc = forward_impl(X, T, H, W, cube_up[0], cube_up[1], cube_up[2], Ci, Cf, rank_up, &ou, packed_up, L1_up, L2_up,
                      Hid, ws_up, ws_up_bytes, DQ_STAGE_ALL, stage_events, stream, nullptr, &up);
    if (rc) return rc;
    return forward_impl(Hid, T, H, W, cube_down[0], cube_down[1], cube_down[2], Cf, Co, rank_down, &od,
                        packed_down, L1_down, L2_down, Y, ws_down, ws_down_bytes, DQ_STAGE_ALL,
                        stage_events ? stage_events + 4 : nullptr, stream, nullptr, &down);
}

int dq_ffn_forward(const void* X, int T, int H, int W, const int* cube_up, const int* cube_down, int Ci, int Cf,
                   int Co, int rank_up, int rank_down, const void* packed_up, const void* L1_up, const void* L2_up,
                   const void* packed_down, const void* L1_down, const void* L2_down, void* Hid, void* Y,
                   void* ws_up, size_t ws_up_bytes, void* ws_down, size_t ws_down_bytes, int ffn_flags,
                   void* const* stage_events, void* stream) {
    return dq_ffn_forward_opts(X, T, H, W, cube_up, cube_down, Ci, Cf, Co, rank_up, rank_down, nullptr, nullptr,
                               packed_up, L1_up, L2_up, packed_down, L1_down, L2_down, Hid, Y, ws_up, ws_up_bytes,
                               ws_down, ws_down_bytes, ffn_flags, stage_events, stream);
}

int dq_linear_forward_opts(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                           const dq_forward_options* opts, const void* packed_W, const void* L1_mma,
                           const void* L2_slab, void* Y, void* workspace, size_t workspace_bytes, int stage_mask,
                           void* const* stage_events, void* stream) {
    return forward_impl(X, T, H, W, t, h, w, Ci, Co, rank, opts, packed_W, L1_mma, L2_slab, Y, workspace,
                        workspace_bytes, stage_mask, stage_events, stream, nullptr);
}

int dq_linear_forward_grouped(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                              int kernel_group, const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y,
                              void* workspace, size_t workspace_bytes, int stage_mask, void* const* stage_events,
                              void* stream) {
    dq_forward_options o{};
    o.kernel_group = kernel_group;
    return dq_linear_forward_opts(X, T, H, W, t, h, w, Ci, Co, rank, &o, packed_W, L1_mma, L2_slab, Y, workspace,
                                  workspace_bytes, stage_mask, stage_events, stream);
}

int dq_linear_forward_ex(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                         const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y, void* workspace,
                         size_t workspace_bytes, int stage_mask, void* const* stage_events, void* stream) {
    return dq_linear_forward_grouped(X, T, H, W, t, h, w, Ci, Co, rank, DQ_KERNEL_SCALE_PER_TOKEN, packed_W, L1_mma,
                                     L2_slab, Y, workspace, workspace_bytes, stage_mask, stage_events, stream);
}

int dq_linear_forward(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                      const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y, void* stream) {
    size_t need = 0;
    int rc = dq_workspace_bytes(T, H, W, t, h, w, Ci, Co, rank, &need);
    if (rc) return rc;
    void* ws = nullptr;
    rc = ensure_lib_workspace(need, &ws);
    if (rc) return rc;
    return dq_linear_forward_ex(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, ws, need,
                                DQ_STAGE_ALL, nullptr, stream);
}

int dq_linear_forward_host(const void* X_host, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                           const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y_host, void* X_dev,
                           void* Y_dev, void* workspace, size_t workspace_bytes, void* stream) {
    return dq_linear_forward_host_ex(X_host, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y_host, X_dev,
                                     Y_dev, workspace, workspace_bytes, 0, stream);
}

int dq_linear_forward_host_ex(const void* X_host, int T, int H, int W, int t, int h, int w, int Ci, int Co, int rank,
                              const void* packed_W, const void* L1_mma, const void* L2_slab, void* Y_host, void* X_dev,
                              void* Y_dev, void* workspace, size_t workspace_bytes, int host_flags, void* stream) {
    int rc = check_shape(T, H, W, t, h, w, Ci, Co, rank);
    if (rc) return rc;
    if (!X_host || !Y_host || !X_dev || !Y_dev) return DQ_ERR_INVALID_ARG;
    if (host_flags & ~DQ_HOST_OVERLAP_PREVIOUS) return DQ_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const Geom g = dq::make_geom(T, H, W, t, h, w);
    const size_t HW = (size_t)H * W;
    if ((long long)t * h * w > 128 || g.KT < 2) {
        // one copy in, the layer, one copy out, all on `stream` (a later overlapping call then waits
        // for all of it)
        Aux* aux = nullptr;
        if ((rc = host_aux(&aux))) return rc;
        {
            std::lock_guard<std::mutex> lk(aux->mu);
            aux->x_free_recorded = false;
        }
        size_t N = (size_t)T * HW;
        cudaError_t e;
        if ((e = cudaMemcpyAsync(X_dev, X_host, N * Ci * 2, cudaMemcpyHostToDevice, st)) != cudaSuccess)
            return cuda_fail(e, "copy of X");
        rc = dq_linear_forward_ex(X_dev, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y_dev, workspace,
                                  workspace_bytes, DQ_STAGE_ALL, nullptr, stream);
        if (rc) return rc;
        if ((e = cudaMemcpyAsync(Y_host, Y_dev, N * Co * 2, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
            return cuda_fail(e, "copy of Y");
        return DQ_OK;
    }
    // Pipelined: X crosses in T-slabs of whole cube layers on a copy stream, and the statistics pass of
    // each slab starts as soon as its rows are on the device; the encode stage and the kernel-token
    // product need every slab's statistics (the per-tensor delta scale); the main product then runs in
    // ranges of row tiles, and the frames each range completes cross back on a second copy stream while
    // the next range computes.  `stream` waits for the last copy, so the call's work ends on `stream`.
    Aux* aux = nullptr;
    if ((rc = host_aux(&aux))) return rc;
    std::lock_guard<std::mutex> lk(aux->mu);
    const int nslab = dq::imin(g.KT, kHostSlabs);
    const int tiles = (int)dq::cdiv(g.N, 256);
    const int nchunk = dq::imin(tiles, kHostChunks);
    Pipeline pipe;
    for (int i = 0; i <= nslab; i++) pipe.kt_cuts.push_back((int)((long long)g.KT * i / nslab));
    for (int i = 0; i <= nchunk; i++) pipe.tile_cuts.push_back((int)((long long)tiles * i / nchunk));
    cudaError_t e;
    if ((host_flags & DQ_HOST_OVERLAP_PREVIOUS) && aux->x_free_recorded) {
        // the copies in wait only for the previous call's last read of X_dev, so that they overlap its
        // products and its copies out
        if ((e = cudaStreamWaitEvent(aux->in, aux->x_free, 0)) != cudaSuccess) return cuda_fail(e, "stream order");
    } else {
        // the copies in wait for earlier work on `stream` (which may still read X_dev)
        if ((e = cudaEventRecord(aux->ev[0], st)) != cudaSuccess || (e = cudaStreamWaitEvent(aux->in, aux->ev[0], 0)))
            return cuda_fail(e, "stream order");
    }
    for (int i = 0; i < nslab; i++) {
        const size_t f0 = (size_t)pipe.kt_cuts[i] * t, f1 = dq::imin(pipe.kt_cuts[i + 1] * t, T);
        const size_t off = f0 * HW * Ci * 2, bytes = (f1 - f0) * HW * Ci * 2;
        if ((e = cudaMemcpyAsync((uint8_t*)X_dev + off, (const uint8_t*)X_host + off, bytes, cudaMemcpyHostToDevice,
                                 aux->in)) != cudaSuccess ||
            (e = cudaEventRecord(aux->ev[1 + i], aux->in)) != cudaSuccess)
            return cuda_fail(e, "copy of X");
    }
    pipe.after_encode = [&]() {
        cudaError_t e1 = cudaEventRecord(aux->x_free, st);
        if (e1 != cudaSuccess) return cuda_fail(e1, "stream order");
        aux->x_free_recorded = true;
        return (int)DQ_OK;
    };
    pipe.before_slab = [&](int i) {
        cudaError_t e1 = cudaStreamWaitEvent(st, aux->ev[1 + i], 0);
        return e1 == cudaSuccess ? DQ_OK : cuda_fail(e1, "stream order");
    };
    // frames whose rows are complete after a range of row tiles: whole cube layers below the last row done
    size_t frames_out = 0;
    const long long layer_rows = (long long)t * H * W;
    pipe.after_chunk = [&](int c, long long rows_done) {
        const int last = c == nchunk - 1;
        const size_t f1 = last ? (size_t)T : dq::imin((int)(rows_done / layer_rows) * t, T);
        if (f1 <= frames_out) return (int)DQ_OK;
        cudaEvent_t ev = aux->ev[1 + kHostSlabs + c];
        cudaError_t e1;
        if ((e1 = cudaEventRecord(ev, st)) != cudaSuccess || (e1 = cudaStreamWaitEvent(aux->out, ev, 0)) != cudaSuccess)
            return cuda_fail(e1, "stream order");
        const size_t off = frames_out * HW * Co * 2, bytes = (f1 - frames_out) * HW * Co * 2;
        if ((e1 = cudaMemcpyAsync((uint8_t*)Y_host + off, (const uint8_t*)Y_dev + off, bytes, cudaMemcpyDeviceToHost,
                                  aux->out)) != cudaSuccess)
            return cuda_fail(e1, "copy of Y");
        frames_out = f1;
        return (int)DQ_OK;
    };
    rc = forward_impl(X_dev, T, H, W, t, h, w, Ci, Co, rank, nullptr, packed_W, L1_mma, L2_slab, Y_dev, workspace,
                      workspace_bytes, DQ_STAGE_ALL, nullptr, stream, &pipe);
    if (rc) return rc;
    cudaEvent_t done = aux->ev[1 + kHostSlabs + kHostChunks];
    if ((e = cudaEventRecord(done, aux->out)) != cudaSuccess || (e = cudaStreamWaitEvent(st, done, 0)) != cudaSuccess)
        return cuda_fail(e, "stream order");
    return DQ_OK;
}

int dq_read_device_status(const void* workspace, void* stream, int* status, int clear) {
    if (!status) return DQ_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const void* ws = workspace;
    if (ws == DQ_NOALLOC_WORKSPACE) {
        void* p = nullptr;
        const int rc = dq::noalloc_workspace(&p);
        if (rc) return rc;
        ws = p;
    } else if (!ws) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ERR_NO_DEVICE;
        std::lock_guard<std::mutex> lk(g_ws_mu);
        auto it = g_ws.find(dev);
        if (it == g_ws.end() || !it->second.ptr) {
            *status = DQ_OK;
            return DQ_OK;
        }
        ws = it->second.ptr;
    }
    int h = 0;
    if (cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DQ_ERR_CUDA;
    if (clear) {
        if (cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(int), st) != cudaSuccess) return DQ_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return DQ_ERR_CUDA;
    }
    *status = h;
    return DQ_OK;
}

const char* dq_last_cuda_error(void) { return g_last_cuda_error; }

int dq_selftest_bounded_wait(int budget_us, void* stream, int* status) {
    if (!status || budget_us <= 0) return DQ_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    int* d = nullptr;
    if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return DQ_ERR_ALLOC;
    int rc = DQ_OK;
    if (cudaMemsetAsync(d, 0, sizeof(int), st) != cudaSuccess ||
        dq::launch_selftest_wait(d, (uint64_t)budget_us * 1000ull, st) != cudaSuccess ||
        cudaMemcpyAsync(status, d, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        rc = DQ_ERR_CUDA;
    cudaFree(d);
    return rc;
}

int dq_selftest_gelu(const float* in, long long n, float* out, void* stream) {
    if (n < 0 || (n > 0 && (!in || !out))) return DQ_ERR_INVALID_ARG;
    if (dq::launch_selftest_gelu(in, n, out, (cudaStream_t)stream) != cudaSuccess) return DQ_ERR_CUDA;
    return DQ_OK;
}

int dq_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* e4m3_value,
                        void* stream) {
    if (n < 0 || (n > 0 && (!in || !e2m1 || !e4m3 || !e4m3_value))) return DQ_ERR_INVALID_ARG;
    if (dq::launch_selftest_convert(in, n, e2m1, e4m3, e4m3_value, (cudaStream_t)stream) != cudaSuccess)
        return DQ_ERR_CUDA;
    return DQ_OK;
}

int dq_selftest_divide(long long n, uint64_t seed, unsigned long long* mismatches, float* first_ab, void* stream) {
    if (n < 0 || !mismatches || !first_ab) return DQ_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned long long* d = nullptr;
    if (cudaMalloc(&d, 16) != cudaSuccess) return DQ_ERR_ALLOC;
    int rc = DQ_OK;
    if (cudaMemsetAsync(d, 0, 16, st) != cudaSuccess ||
        dq::launch_selftest_divide(n, seed, d, (float*)(d + 1), st) != cudaSuccess ||
        cudaMemcpyAsync(mismatches, d, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(first_ab, d + 1, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        rc = DQ_ERR_CUDA;
    cudaFree(d);
    return rc;
}

}  // extern "C"
