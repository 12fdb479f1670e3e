// Diagnostic kernels behind the self-test entry points: the bounded-wait
// failure path and the device format conversions used by the quantisers.
#include "dq_internal.h"
#include "dq_ptx.cuh"

namespace dq {

// Waits on an mbarrier that nothing arrives at; the bounded wait must give up
// with DQ_ERR_DEVICE_TIMEOUT in *status and the kernel must return.
__global__ void k_selftest_wait(int* status, uint64_t budget_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, (volatile int*)&abort_flag, status, budget_ns);
    __syncthreads();
}

// The same conversion helpers the quantisers use, element by element.
__global__ void k_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* e4m3_back) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float v = in[i];
    e2m1[i] = (uint8_t)(cvt_e2m1x2(v, 0.f) & 0xF);
    uint32_t c = cvt_e4m3x2(v, 0.f) & 0xFF;
    e4m3[i] = (uint8_t)c;
    e4m3_back[i] = e4m3_to_f32(c);
}

cudaError_t launch_selftest_wait(int* status, uint64_t budget_ns, cudaStream_t st) {
    k_selftest_wait<<<1, 32, 0, st>>>(status, budget_ns);
    return cudaGetLastError();
}

cudaError_t launch_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* back,
                                    cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    k_selftest_convert<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(in, n, e2m1, e4m3, back);
    return cudaGetLastError();
}

}  // namespace dq
