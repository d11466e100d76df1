// Small device-side building blocks shared by the kernels: asynchronous
// copies (cp.async, TMA tensor loads), mbarrier waits with an iteration
// bound, and programmatic dependent launch control.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gconv {
namespace dev {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch --------------------------------------
// wait(): blocks until every grid this one depends on has completed and its
// memory is visible (a no-op when the launch had no programmatic edge).
// Every kernel calls it before its first global-memory access.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// launch_dependents(): lets the next grid in the stream start launching; its
// own wait() still holds it until this grid has completed.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---- cp.async (LDGSTS) -----------------------------------------------------
__device__ __forceinline__ void cp_async16(float *sdst, const float *gsrc, bool valid) {
    int nbytes = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr(sdst)), "l"(gsrc),
                 "r"(nbytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async4(float *sdst, const float *gsrc, bool valid) {
    int nbytes = valid ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_addr(sdst)), "l"(gsrc),
                 "r"(nbytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// ---- mbarrier ----------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase.  Each try_wait suspends the thread for a
// hardware-chosen interval; 1<<22 attempts is far beyond any legitimate wait
// (well over a second).  Returns false when the bound is hit.
constexpr uint32_t kMbarSpinLimit = 1u << 22;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kMbarSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// ---- TMA ---------------------------------------------------------------------
// 3-D tiled load of one box into shared memory; completion is signalled on
// `bar` as transaction bytes.  Out-of-bounds elements are zero-filled.  The
// innermost coordinate times 4 bytes must be a multiple of 16.
__device__ __forceinline__ void tma_load_3d(void *sdst, const void *tmap, uint64_t *bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(smem_addr(sdst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace dev
}  // namespace gconv
