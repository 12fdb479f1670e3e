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

// The feed-forward epilogue's GELU (gelu_erf2, two values per call) on n fp32 values.
__global__ void k_selftest_gelu(const float* in, long long n, float* out) {
    const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float y0 = in[i], y1 = (i + 1 < n) ? in[i + 1] : 0.f;
    float h0, h1;
    f2_unpack(gelu_erf2(f2_pack(y0, y1)), h0, h1);
    out[i] = h0;
    if (i + 1 < n) out[i + 1] = h1;
}

__device__ __forceinline__ uint64_t mix64d(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

// Compares the quantisers' quotient paths (correctly rounded reciprocal, one
// product, one FMA correction; div_pos, the negated div_neg and its packed
// pair form f2_div_neg on (a, -a)) with IEEE division, bit for bit, on operand pairs drawn from a counter-based hash: a
// with exponent in [-40, 12] (and exact zeros of either sign), b > 0 with
// exponent in [-30, 12].  A pair counts once if either path differs.
__global__ void k_selftest_divide(long long n, uint64_t seed, unsigned long long* mismatches, float* first) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    unsigned long long bad = 0;
    for (; i < n; i += stride) {
        uint64_t h1 = mix64d(seed ^ (uint64_t)(2 * i)), h2 = mix64d(seed ^ (uint64_t)(2 * i + 1));
        uint32_t ma = (uint32_t)(h1 & 0x7FFFFFu), mb = (uint32_t)(h2 & 0x7FFFFFu);
        int ea = (int)((h1 >> 23) % 53) - 40, eb = (int)((h2 >> 23) % 43) - 30;
        uint32_t sa = (uint32_t)((h1 >> 40) & 1u) << 31;
        float a = __uint_as_float(sa | ((uint32_t)(ea + 127) << 23) | ma);
        if (((h1 >> 41) & 1023u) == 0) a = __uint_as_float(sa);          // signed zeros
        float b = __uint_as_float(((uint32_t)(eb + 127) << 23) | mb);
        float q0 = __fdiv_rn(a, b);
        const float rb = __frcp_rn(b);
        float q1 = div_pos(a, b, rb);
        float q2 = -div_neg(a, b, rb);
        float q3, q4;
        f2_unpack(f2_div_neg(f2_pack(a, -a), f2_pack(b, b), f2_pack(-rb, -rb)), q3, q4);
        q3 = -q3;
        const float q5 = __fdiv_rn(-a, b);
        if (__float_as_uint(q0) != __float_as_uint(q1) || __float_as_uint(q0) != __float_as_uint(q2) ||
            __float_as_uint(q0) != __float_as_uint(q3) || __float_as_uint(q5) != __float_as_uint(-q4)) {
            if (atomicAdd(mismatches, 1ull) == 0ull) {
                first[0] = a;
                first[1] = b;
            }
            bad++;
        }
    }
}

cudaError_t launch_selftest_divide(long long n, uint64_t seed, unsigned long long* mismatches, float* first,
                                   cudaStream_t st) {
    k_selftest_divide<<<148 * 8, 256, 0, st>>>(n, seed, mismatches, first);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int* status, uint64_t budget_ns, cudaStream_t st) {
    k_selftest_wait<<<1, 32, 0, st>>>(status, budget_ns);
    return cudaGetLastError();
}

cudaError_t launch_selftest_gelu(const float* in, long long n, float* out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    k_selftest_gelu<<<(unsigned)((n + 511) / 512), 256, 0, st>>>(in, n, out);
    return cudaGetLastError();
}

cudaError_t launch_selftest_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3, float* back,
                                    cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    k_selftest_convert<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(in, n, e2m1, e4m3, back);
    return cudaGetLastError();
}

}  // namespace dq
