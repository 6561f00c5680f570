// Thin inline-PTX wrappers for the sm_100a features both GEMM kernels use: bounded mbarrier
// waits, TMA loads (cp.async.bulk.tensor), programmatic dependent launch, cluster shared memory
// and LOP3. The tensor-memory kernel's own wrappers (tcgen05) are in tcgen05_ptx.cuh.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace lowbit {

// ---- status / bounded waits ------------------------------------------------------------
// A wait that has not completed after this many SM clocks (about 2 s at 1.9 GHz) gives up,
// records LOWBIT_DEVERR_TIMEOUT in the device status word and raises the CTA's abort flag.
constexpr long long kWaitLimitCycles = 4000000000LL;
constexpr unsigned kDevErrTimeout = 1u;   // a bounded wait gave up
constexpr unsigned kDevErrCheck = 2u;     // a device-side index check failed (debug builds)

// Device-side index checks of the debug build (LOWBIT_DEBUG_CHECKS): dcheck(ok, word) records
// kDevErrCheck in the status word when `ok` is false and returns `ok`, so the caller skips the
// access instead of trapping; release builds compile the checks away.
#ifdef LOWBIT_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
__device__ __forceinline__ bool dcheck(bool ok, unsigned* status_word) {
    if (!ok) atomicOr(status_word, kDevErrCheck);
    return ok;
}
#else
constexpr bool kDebugChecks = false;
__device__ __forceinline__ bool dcheck(bool, unsigned*) { return true; }
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with parity `parity` of `bar` to complete. Returns false if the CTA's
// abort flag is (or becomes) set or the wait exceeds kWaitLimitCycles; in the latter case the
// device status word gets kDevErrTimeout and the abort flag is raised.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* status_word, long long limit = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    uint32_t it = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++it & 63u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - t0 > limit) {
                atomicOr(status_word, kDevErrTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// ---- TMA ----------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2D tiled load of one box into this CTA's shared memory; completes `bar`'s transaction count.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 3D tiled load of one box into this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// ---- programmatic dependent launch ---------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}


// ---- clusters ---------------------------------------------------------------------------
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
// Store 16 bytes into the shared memory of a CTA of the cluster (`addr` from map_shared_rank).
__device__ __forceinline__ void st_shared_cluster_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

// ---- bit / fp16x2 helpers ------------------------------------------------------------------
template <uint32_t LUT>
__device__ __forceinline__ uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
    return d;
}
// (a & b) | c
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) { return lop3<0xEA>(a, b, c); }
// a ^ (~b & c)
__device__ __forceinline__ uint32_t xor_andnot(uint32_t a, uint32_t b, uint32_t c) { return lop3<0xD2>(a, b, c); }

}  // namespace lowbit
