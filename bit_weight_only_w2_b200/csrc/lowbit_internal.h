// Declarations shared by the library's translation units (host side).
#pragma once

#include <cuda.h>
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
// convert_x = false skips the conversion when the workspace already holds this X's fp16 copy
// and row factors (a batch whose previous linear read the same, unchanged X).
lowbit_status gemm_launch(const GemmProblem& g, int force_bt, int force_rows, int force_split,
                          cudaStream_t stream, bool convert_x = true);

// True if the problem runs on the tensor-memory kernel (and so through the X conversion pass)
// when its configuration is chosen automatically.
bool uses_x_copy(const GemmProblem& g);

// Launches the X -> fp16 conversion pass into the problem's workspace (programmatic dependent
// launch). The GEMM kernels read its output.
lowbit_status launch_convert_x(const GemmProblem& g, cudaStream_t stream);

// Small-M GEMM (M <= 16) on warp-level bf16 tensor-core MMAs, reading X directly (no
// conversion pass, no workspace). rows (weight rows per CTA, multiple of 8, <= 128) and ksplit
// (K slices per cluster, <= 8): 0 = automatic. swap: weights as the MMA's 16-row operand and up
// to 8 tokens as its n8 operand (M <= 8; rows a multiple of 16). smallm_supported: whether the
// shape fits the kernel at all.
bool smallm_supported(const GemmProblem& g);
lowbit_status smallm_launch(const GemmProblem& g, int rows, int ksplit, bool swap, cudaStream_t stream);

// Device address of the current device's status word (nullptr on failure).
unsigned* device_status_address();

// 2-D tiled tensor map (inner dimension contiguous) and the device's SM count.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz);
int num_sms();
bool make_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t (&dims)[3],
                 const uint64_t (&strides)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swz);

// Reads (and optionally clears) the device status word. Synchronises the device.
lowbit_status read_device_status(int clear);

// Reads and clears the device status word in the order of `stream`, waiting for that stream only.
lowbit_status read_stream_status(cudaStream_t stream);

// Packing kernels (synchronous on `stream`); `bad` receives the number of invalid codes.
lowbit_status pack_launch(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed,
                          cudaStream_t stream, unsigned long long* bad);
lowbit_status unpack_launch(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes,
                            cudaStream_t stream, unsigned long long* bad);

// Launches the bounded-wait self-test kernel.
lowbit_status selftest_bounded_wait(long long limit_cycles, cudaStream_t stream);

// Launches the index-check self-test kernel (debug builds; else LOWBIT_ERR_UNSUPPORTED).
lowbit_status selftest_index_check(cudaStream_t stream);

// True when the current device can run the sm_100a kernels.
lowbit_status check_device();

// Failure injection for tests of the error paths (lowbit_test_fail_next): true, once, if a
// failure of `kind` was requested; the call site then reports it as the real failure would.
enum InjectKind { kInjectEncode = 1, kInjectLaunch = 2 };
bool take_injected_failure(int kind);

}  // namespace lowbit
