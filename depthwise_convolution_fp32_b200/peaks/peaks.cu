// Roofline denominators measured on the GPU the benchmark runs on: the FP32
// CUDA-core FMA rate and the 5th-generation tensor-core MMA rates for the two
// operand kinds the implicit-GEMM convolution issues (kind::tf32 for the main
// term, kind::f16 with bf16 operands for the cross terms).
//
// Measurement tooling for the benchmark, not part of libgconv.so's C ABI.
// Each function launches its kernel once untimed (clocks ramp, code loads),
// then times one launch with CUDA events and returns the elapsed time and the
// floating-point operations it performed (2 per multiply-add).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../csrc/device_utils.cuh"
#include "peaks.h"

namespace {

using namespace gconv;

// ---- FP32 FMA -------------------------------------------------------------
// 16 independent accumulation chains per thread, each x = x * a + b with
// |a| < 1, so values stay finite; enough warps per SM to cover the FMA latency.
constexpr int kChains = 16;

__global__ void __launch_bounds__(256) ffma_kernel(float *out, int iters, float a, float b) {
    float x[kChains];
#pragma unroll
    for (int j = 0; j < kChains; ++j) x[j] = (float)(threadIdx.x + j) * 1e-3f;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int j = 0; j < kChains; ++j) x[j] = fmaf(x[j], a, b);
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kChains; ++j) s += x[j];
    if (s == 1234.5f) out[blockIdx.x * blockDim.x + threadIdx.x] = s;   // never true: keeps the loop live
}

// ---- tcgen05 MMA ----------------------------------------------------------
// One CTA per SM (the shared memory request keeps it alone); thread 0 issues
// `iters` back-to-back MMAs of M = 128, N = 256 into one TMEM accumulator,
// commits, and waits (bounded) for completion.  Operands are zeros in the
// K-major no-swizzle layout the convolution uses (8-row x 16-byte core
// matrices; the two 16-byte K halves 128 bytes apart, 8-row groups 256 bytes
// apart), so the rate is the pipe's, not the data's.
constexpr int kMmaM = 128, kMmaN = 256;
constexpr int kMmaSmem = 128 * 1024;   // > half of the SM's shared memory: one CTA per SM

template <bool TF32>
__global__ void __launch_bounds__(128, 1) mma_kernel(int iters, int *status) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + 8);
    unsigned char *A = smem + 1024;                    // 128 rows x 32 B
    unsigned char *B = A + kMmaM * 32;                 // 256 rows x 32 B
    for (int i = threadIdx.x; i < (kMmaM + kMmaN) * 32 / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(A)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        dev::mbar_init(bar, 1);
        dev::fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // operand zeros visible to the tensor core
    if (threadIdx.x < 32) {
        dev::tmem_alloc(tslot, kMmaN);
        dev::tmem_relinquish();
    }
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = *tslot;
    if (threadIdx.x == 0) {
        const uint64_t da = dev::smem_desc(A, 128, 256);
        const uint64_t db = dev::smem_desc(B, 128, 256);
        constexpr uint32_t idesc = TF32 ? dev::idesc_tf32(kMmaM, kMmaN) : dev::idesc_bf16(kMmaM, kMmaN);
        for (int i = 0; i < iters; ++i) {
            if constexpr (TF32) dev::mma_tf32(tmem, da, db, idesc, i > 0 ? 1u : 0u);
            else dev::mma_bf16(tmem, da, db, idesc, i > 0 ? 1u : 0u);
        }
        dev::mma_commit(bar);
        if (!dev::mbar_wait_bounded(bar, 0)) atomicExch(status, 1);
    }
    dev::tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) dev::tmem_dealloc(tmem, kMmaN);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

template <typename F>
int time_twice(F launch, double *ms) {
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return 1;
    int rc = 0;
    if (launch() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) rc = 2;
    if (!rc) {
        cudaEventRecord(e0);
        if (launch() != cudaSuccess) rc = 2;
        cudaEventRecord(e1);
        if (!rc && cudaEventSynchronize(e1) != cudaSuccess) rc = 3;
        float t = 0.f;
        if (!rc && cudaEventElapsedTime(&t, e0, e1) != cudaSuccess) rc = 3;
        *ms = t;
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return rc;
}

}  // namespace

extern "C" {

int gpeaks_ffma(int iters, double *ms, double *flops) {
    const int sms = sm_count();
    if (sms < 1 || iters < 1 || !ms || !flops) return 1;
    float *out = nullptr;
    const int blocks = sms * 8, threads = 256;
    if (cudaMalloc(&out, sizeof(float) * blocks * threads) != cudaSuccess) return 2;
    const int rc = time_twice([&] {
        ffma_kernel<<<blocks, threads>>>(out, iters, 0.9999f, 1e-4f);
        return cudaGetLastError();
    }, ms);
    cudaFree(out);
    *flops = 2.0 * kChains * 8.0 * iters * (double)blocks * threads;
    return rc;
}

static int mma_peak(bool tf32, int iters, double *ms, double *flops) {
    const int sms = sm_count();
    if (sms < 1 || iters < 1 || !ms || !flops) return 1;
    int *status = nullptr;
    if (cudaMalloc(&status, sizeof(int)) != cudaSuccess) return 2;
    cudaMemset(status, 0, sizeof(int));
    auto kern = tf32 ? mma_kernel<true> : mma_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMmaSmem) != cudaSuccess) {
        cudaFree(status);
        return 2;
    }
    int rc = time_twice([&] {
        kern<<<sms, 128, kMmaSmem>>>(iters, status);
        return cudaGetLastError();
    }, ms);
    int st = 0;
    cudaMemcpy(&st, status, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(status);
    if (!rc && st) rc = 4;   // a bounded wait gave up
    const double k = tf32 ? 8.0 : 16.0;   // K of one MMA: 32 bytes of each operand row
    *flops = 2.0 * kMmaM * kMmaN * k * (double)iters * sms;
    return rc;
}

int gpeaks_mma_tf32(int iters, double *ms, double *flops) { return mma_peak(true, iters, ms, flops); }
int gpeaks_mma_bf16(int iters, double *ms, double *flops) { return mma_peak(false, iters, ms, flops); }

}  // extern "C"
