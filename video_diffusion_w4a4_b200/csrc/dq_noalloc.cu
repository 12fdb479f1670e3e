// Forward pass that allocates no device memory.
//
// Some callers cannot call cudaMalloc: code that runs while a CUDA graph is
// being captured or replayed into a fixed memory plan, allocators that own
// every device byte of the process, and embedded callers that are not allowed
// to grow their memory footprint after start-up.  For them the layer's scratch
// (the workspace that the other forward entry points take from the caller or
// from a library-owned cudaMalloc) lives in one fixed array in device memory
// that this file declares.  The array exists on every GPU where this library's
// module is loaded and stays there until the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/deltaquant.h"
#include "dq_internal.h"

namespace {

// Largest workspace this entry point accepts (dq_workspace_bytes of the call).
constexpr size_t kStaticWorkspaceBytes = (size_t)32 << 20;

static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

bool aligned256(const void* p) { return ((uintptr_t)p & 255u) == 0; }

}  // namespace

namespace dq {

// Device address of the array on the current device.  Host code may not use
// the symbol itself as a pointer (it names a host-side stand-in), so the
// address is looked up once per device, with that device current, and cached.
// The lookup is not a stream operation and writes nothing to the device.
int noalloc_workspace(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DQ_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return DQ_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return DQ_OK;
}

}  // namespace dq

extern "C" int dq_linear_forward_noalloc(const void* X, int T, int H, int W, int t, int h, int w, int Ci, int Co,
                                         int rank, const void* packed_W, const void* L1_mma, const void* L2_slab,
                                         void* Y, void* stream) {
    size_t need = 0;
    int rc = dq_workspace_bytes(T, H, W, t, h, w, Ci, Co, rank, &need);
    if (rc) return rc;
    if (need > kStaticWorkspaceBytes) return DQ_ERR_WORKSPACE_TOO_SMALL;
    if (!X || !packed_W || !L1_mma || !L2_slab || !Y) return DQ_ERR_INVALID_ARG;
    if (!aligned256(X) || !aligned256(packed_W) || !aligned256(L1_mma) || !aligned256(L2_slab) || !aligned256(Y))
        return DQ_ERR_ALIGNMENT;
    void* ws = nullptr;
    rc = dq::noalloc_workspace(&ws);
    if (rc) return rc;
    // The array keeps the previous call's contents.  Every scratch tensor of the
    // forward is fully rewritten by it, and the accumulators that must start at
    // zero (the amax words) are cleared by the forward's first stage; the status
    // word is cleared here, on the caller's stream, so that an earlier call's
    // error does not carry over (dq_read_device_status(DQ_NOALLOC_WORKSPACE, ...)
    // reads it after the call).
    if (cudaMemsetAsync(ws, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess) return DQ_ERR_CUDA;
    return dq_linear_forward_ex(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, ws,
                                kStaticWorkspaceBytes, DQ_STAGE_ALL, nullptr, stream);
}
