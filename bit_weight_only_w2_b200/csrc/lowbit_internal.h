// Declarations shared by the library's translation units (host side).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "lowbit.h"

namespace lowbit {

struct GemmProblem {
    int64_t M, N, K;
    int bits, group_size;
    const void* X;
    const uint32_t* Wp;
    const void* scales;
    const void* zeros;
    void* Y;
    void* workspace;
    size_t workspace_bytes;
};

// Workspace of one GEMM: the fp16 copy of X ([M][K]) then one fp32 factor per row of X.
struct WorkspaceLayout {
    size_t rowmul_offset;
    size_t total;
};
inline WorkspaceLayout workspace_layout(int64_t M, int64_t K) {
    const size_t xh = (static_cast<size_t>(M) * static_cast<size_t>(K) * 2 + 255) / 256 * 256;
    const size_t rm = (static_cast<size_t>(M) * 4 + 255) / 256 * 256;
    return WorkspaceLayout{xh, xh + rm};
}

// Validates one problem against the ABI's preconditions (no launch, no CUDA call).
lowbit_status validate_gemm(const GemmProblem& g);

// Launches the X conversion and the GEMM kernel for a validated problem. force_bt (tokens per
// tile), force_rows (weight rows per tile) and force_split (K slices): 0 = automatic.
lowbit_status gemm_launch(const GemmProblem& g, int force_bt, int force_rows, int force_split,
                          cudaStream_t stream);

// Reads (and optionally clears) the device status word. Synchronises the device.
lowbit_status read_device_status(int clear);

// Packing kernels (synchronous on `stream`); `bad` receives the number of invalid codes.
lowbit_status pack_launch(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed,
                          cudaStream_t stream, unsigned long long* bad);
lowbit_status unpack_launch(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes,
                            cudaStream_t stream, unsigned long long* bad);

// Launches the bounded-wait self-test kernel.
lowbit_status selftest_bounded_wait(long long limit_cycles, cudaStream_t stream);

// True when the current device can run the sm_100a kernels.
lowbit_status check_device();

}  // namespace lowbit
