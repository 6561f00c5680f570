// lowbit_gemm_noalloc: the GEMM for callers that must not allocate device memory.
//
// lowbit_gemm needs a workspace (the fp16 copy of X plus one factor per row) that the caller
// allocates. Some callers cannot allocate at the point where they run a linear: a plug-in
// inside a host engine that owns all device memory and forbids allocations after start-up,
// or a latency-critical loop where cudaMalloc would synchronise the device. This entry point
// runs the same two kernels with their scratch in a fixed array of static device memory
// instead, so it allocates nothing; in exchange, the problem size it accepts is capped.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "lowbit_internal.h"

#define LOWBIT_API extern "C" __attribute__((visibility("default")))

namespace lowbit {
namespace {

// The scratch: the fp16 copy of X ([M][K]) followed by M fp32 row factors, both rounded up to
// 256 bytes. Every call on a device shares it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LOWBIT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device. The
// array's name in host code is only a host-side handle, so it is never passed to a kernel.
lowbit_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LOWBIT_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LOWBIT_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LOWBIT_OK;
}

}  // namespace
}  // namespace lowbit

using namespace lowbit;

LOWBIT_API lowbit_status lowbit_gemm_noalloc(int64_t M, int64_t N, int64_t K, int bits, int group_size,
                                             const void* X, const uint32_t* Wp, const void* scales,
                                             const void* zeros, void* Y, void* stream) {
    GemmProblem g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.bits = bits;
    g.group_size = group_size;
    g.X = X;
    g.Wp = Wp;
    g.scales = scales;
    g.zeros = zeros;
    g.Y = Y;
    g.workspace = nullptr;
    g.workspace_bytes = LOWBIT_NOALLOC_SCRATCH_BYTES;
    // Shape and pointer checks first (with a stand-in address for the scratch), so that bad
    // arguments and oversized problems are rejected before any CUDA call.
    g.workspace = reinterpret_cast<void*>(uintptr_t(256));
    lowbit_status st = validate_gemm(g);
    if (st != LOWBIT_OK || M == 0 || N == 0) return st;
    if ((st = check_device()) != LOWBIT_OK) return st;
    if ((st = scratch_address(&g.workspace)) != LOWBIT_OK) return st;
    return gemm_launch(g, 0, 0, 0, static_cast<cudaStream_t>(stream));
}
