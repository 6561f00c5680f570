// The C ABI of liblowbit.so (declared in include/lowbit.h): argument checks, the device
// probe, and dispatch to the packing and GEMM kernels. Every check runs before any launch.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "lowbit_internal.h"

#define LOWBIT_API extern "C" __attribute__((visibility("default")))

namespace lowbit {
namespace {

std::mutex g_pack_mutex;   // pack / unpack share one device-side error counter

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_bits(int bits) { return bits == 1 || bits == 2 || bits == 4; }

lowbit_status check_pack_args(const void* a, const void* b, int64_t N, int64_t K, int bits) {
    if (!valid_bits(bits) || N < 0 || K < 0) return LOWBIT_ERR_INVALID_ARG;
    if (K % (32 / bits) != 0) return LOWBIT_ERR_INVALID_ARG;
    if (N == 0 || K == 0) return LOWBIT_OK;
    if (!a || !b) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b)) return LOWBIT_ERR_ALIGNMENT;
    return LOWBIT_OK;
}

}  // namespace

lowbit_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    // the answer per device never changes: 1 = supported, 2 = not (0 = not yet asked)
    static std::atomic<int> known[64];
    if (dev >= 0 && dev < 64) {
        const int k = known[dev].load(std::memory_order_relaxed);
        if (k) return k == 1 ? LOWBIT_OK : LOWBIT_ERR_UNSUPPORTED_DEVICE;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    // The kernels are built for sm_100a only (tcgen05 / tensor memory).
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) known[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? LOWBIT_OK : LOWBIT_ERR_UNSUPPORTED_DEVICE;
}

namespace {
std::atomic<int> g_injected{0};   // InjectKind bits still to be consumed
}  // namespace

bool take_injected_failure(int kind) {
    int cur = g_injected.load(std::memory_order_relaxed);
    while (cur & kind)
        if (g_injected.compare_exchange_weak(cur, cur & ~kind, std::memory_order_acq_rel)) return true;
    return false;
}

lowbit_status validate_gemm(const GemmProblem& g) {
    if (!valid_bits(g.bits)) return LOWBIT_ERR_INVALID_ARG;
    if (g.M < 0 || g.N < 0 || g.K <= 0 || g.group_size <= 0) return LOWBIT_ERR_INVALID_ARG;
    if (g.K % g.group_size != 0 || g.group_size % (32 / g.bits) != 0) return LOWBIT_ERR_INVALID_ARG;
    if ((g.bits == 4) != (g.zeros != nullptr)) return LOWBIT_ERR_INVALID_ARG;
    if (g.M == 0 || g.N == 0) return LOWBIT_OK;
    if (!g.X || !g.Wp || !g.scales || !g.Y) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned16(g.X) || !aligned16(g.Wp) || !aligned16(g.scales) || !aligned16(g.Y) ||
        (g.zeros && !aligned16(g.zeros)))
        return LOWBIT_ERR_ALIGNMENT;
    // GPU path limits (TMA strides must be multiples of 16 bytes; supported tile configs).
    if (g.group_size != 64 && g.group_size != 128) return LOWBIT_ERR_UNSUPPORTED;
    if (g.bits == 1 && g.K % 128 != 0) return LOWBIT_ERR_UNSUPPORTED;
    if (g.N % 8 != 0) return LOWBIT_ERR_UNSUPPORTED;
    if (g.M >= (int64_t(1) << 31) || g.N >= (int64_t(1) << 31) || g.K >= (int64_t(1) << 31))
        return LOWBIT_ERR_UNSUPPORTED;
    if (!g.workspace || (reinterpret_cast<uintptr_t>(g.workspace) & 255u) != 0 ||
        g.workspace_bytes < workspace_layout(g.M, g.K).total)
        return LOWBIT_ERR_WORKSPACE;
    return LOWBIT_OK;
}

}  // namespace lowbit

using namespace lowbit;

LOWBIT_API const char* lowbit_status_string(lowbit_status s) {
    switch (s) {
        case LOWBIT_OK: return "LOWBIT_OK";
        case LOWBIT_ERR_INVALID_ARG: return "LOWBIT_ERR_INVALID_ARG";
        case LOWBIT_ERR_ALIGNMENT: return "LOWBIT_ERR_ALIGNMENT";
        case LOWBIT_ERR_UNSUPPORTED: return "LOWBIT_ERR_UNSUPPORTED";
        case LOWBIT_ERR_UNSUPPORTED_DEVICE: return "LOWBIT_ERR_UNSUPPORTED_DEVICE";
        case LOWBIT_ERR_BAD_CODE: return "LOWBIT_ERR_BAD_CODE";
        case LOWBIT_ERR_TIMEOUT: return "LOWBIT_ERR_TIMEOUT";
        case LOWBIT_ERR_CUDA: return "LOWBIT_ERR_CUDA";
        case LOWBIT_ERR_WORKSPACE: return "LOWBIT_ERR_WORKSPACE";
        case LOWBIT_ERR_DEVICE_CHECK: return "LOWBIT_ERR_DEVICE_CHECK";
    }
    return "LOWBIT_ERR_UNKNOWN";
}

LOWBIT_API int lowbit_version(void) { return 100; }

LOWBIT_API size_t lowbit_packed_words(int64_t N, int64_t K, int bits) {
    if (!valid_bits(bits) || N < 0 || K < 0 || K % (32 / bits) != 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K) * bits / 32;
}

LOWBIT_API lowbit_status lowbit_pack(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed,
                                     void* stream) {
    lowbit_status st = check_pack_args(codes, packed, N, K, bits);
    if (st != LOWBIT_OK || N == 0 || K == 0) return st;
    if ((st = check_device()) != LOWBIT_OK) return st;
    std::lock_guard<std::mutex> lock(g_pack_mutex);
    unsigned long long bad = 0;
    st = pack_launch(codes, N, K, bits, packed, static_cast<cudaStream_t>(stream), &bad);
    if (st != LOWBIT_OK) return st;
    return bad ? LOWBIT_ERR_BAD_CODE : LOWBIT_OK;
}

LOWBIT_API lowbit_status lowbit_unpack(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes,
                                       void* stream) {
    lowbit_status st = check_pack_args(packed, codes, N, K, bits);
    if (st != LOWBIT_OK || N == 0 || K == 0) return st;
    if ((st = check_device()) != LOWBIT_OK) return st;
    std::lock_guard<std::mutex> lock(g_pack_mutex);
    unsigned long long bad = 0;
    st = unpack_launch(packed, N, K, bits, codes, static_cast<cudaStream_t>(stream), &bad);
    if (st != LOWBIT_OK) return st;
    return bad ? LOWBIT_ERR_BAD_CODE : LOWBIT_OK;
}

static GemmProblem make_problem(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                                const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                                void* workspace, size_t workspace_bytes) {
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
    g.workspace = workspace;
    g.workspace_bytes = workspace_bytes;
    return g;
}

LOWBIT_API size_t lowbit_gemm_workspace_size(int64_t M, int64_t K) {
    if (M < 0 || K < 0) return 0;
    return workspace_layout(M, K).total;
}

LOWBIT_API lowbit_status lowbit_gemm(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                                     const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    const GemmProblem g = make_problem(M, N, K, bits, group_size, X, Wp, scales, zeros, Y, workspace, workspace_bytes);
    lowbit_status st = validate_gemm(g);
    if (st != LOWBIT_OK || M == 0 || N == 0) return st;
    if ((st = check_device()) != LOWBIT_OK) return st;
    return gemm_launch(g, 0, 0, 0, static_cast<cudaStream_t>(stream));
}

LOWBIT_API lowbit_status lowbit_gemm_ex(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                                        const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                                        void* workspace, size_t workspace_bytes, int tile_tokens, int tile_rows,
                                        int ksplit, void* stream) {
    const GemmProblem g = make_problem(M, N, K, bits, group_size, X, Wp, scales, zeros, Y, workspace, workspace_bytes);
    lowbit_status st = validate_gemm(g);
    if (st != LOWBIT_OK || M == 0 || N == 0) return st;
    if (tile_tokens != 0 && tile_tokens != 1 && tile_tokens != 8 && tile_tokens != 16 && tile_tokens != 32 &&
        tile_tokens != 64 && tile_tokens != 128 && tile_tokens != 256)
        return LOWBIT_ERR_UNSUPPORTED;
    if ((tile_tokens == 1 && M > 16) || (tile_tokens == 8 && M > 8)) return LOWBIT_ERR_UNSUPPORTED;
    if (tile_tokens == 8 && tile_rows % 16 != 0) return LOWBIT_ERR_UNSUPPORTED;
    if (ksplit < 0 || ksplit > 8) return LOWBIT_ERR_UNSUPPORTED;
    if (tile_rows < 0 || tile_rows % 8 != 0) return LOWBIT_ERR_UNSUPPORTED;
    if (tile_rows > 128 && !(tile_rows == 256 && (tile_tokens == 0 || tile_tokens == 256))) return LOWBIT_ERR_UNSUPPORTED;
    if ((st = check_device()) != LOWBIT_OK) return st;
    return gemm_launch(g, tile_tokens, tile_rows, ksplit, static_cast<cudaStream_t>(stream));
}

LOWBIT_API lowbit_status lowbit_gemm_batch(const lowbit_gemm_desc* descs, int count, void* workspace,
                                           size_t workspace_bytes, void* stream) {
    if (count < 0 || (count > 0 && !descs)) return LOWBIT_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const lowbit_gemm_desc& d = descs[i];
        const lowbit_status st = validate_gemm(make_problem(d.M, d.N, d.K, d.bits, d.group_size, d.X, d.Wp,
                                                            d.scales, d.zeros, d.Y, workspace, workspace_bytes));
        if (st != LOWBIT_OK) return st;
    }
    if (count == 0) return LOWBIT_OK;
    lowbit_status st = check_device();
    if (st != LOWBIT_OK) return st;
    // The fp16 copy of X in the workspace is reused by the next linear that reads the same X
    // (same pointer, M and K) when no output written since the copy was made overlaps that X:
    // e.g. separate Q, K and V projections of one input convert it once.
    const void* copied_x = nullptr;
    int64_t copied_m = -1, copied_k = -1;
    std::vector<std::pair<uintptr_t, uintptr_t>> written;   // Y byte ranges since the copy
    for (int i = 0; i < count; ++i) {
        const lowbit_gemm_desc& d = descs[i];
        if (d.M == 0 || d.N == 0) continue;
        const GemmProblem g = make_problem(d.M, d.N, d.K, d.bits, d.group_size, d.X, d.Wp, d.scales, d.zeros, d.Y,
                                           workspace, workspace_bytes);
        bool convert = true;
        if (uses_x_copy(g)) {
            const uintptr_t x0 = reinterpret_cast<uintptr_t>(d.X), x1 = x0 + static_cast<uintptr_t>(d.M * d.K * 2);
            bool clean = copied_x == d.X && copied_m == d.M && copied_k == d.K;
            for (size_t j = 0; clean && j < written.size(); ++j)
                if (written[j].first < x1 && x0 < written[j].second) clean = false;
            convert = !clean;
        }
        st = gemm_launch(g, 0, 0, 0, static_cast<cudaStream_t>(stream), convert);
        if (st != LOWBIT_OK) return st;
        if (uses_x_copy(g) && convert) {
            copied_x = d.X;
            copied_m = d.M;
            copied_k = d.K;
            written.clear();
        }
        const uintptr_t y0 = reinterpret_cast<uintptr_t>(d.Y);
        written.emplace_back(y0, y0 + static_cast<uintptr_t>(d.M * d.N * 2));
    }
    return LOWBIT_OK;
}

LOWBIT_API lowbit_status lowbit_device_status(int clear) { return read_device_status(clear); }

LOWBIT_API lowbit_status lowbit_last_device_status(void* stream) {
    const lowbit_status st = check_device();
    if (st != LOWBIT_OK) return st;
    return read_stream_status(static_cast<cudaStream_t>(stream));
}

LOWBIT_API lowbit_status lowbit_test_fail_next(int what) {
    if (what < 0 || what > (kInjectEncode | kInjectLaunch)) return LOWBIT_ERR_INVALID_ARG;
    if (what == 0) g_injected.store(0, std::memory_order_release);
    else g_injected.fetch_or(what, std::memory_order_acq_rel);
    return LOWBIT_OK;
}

LOWBIT_API int lowbit_debug_checks_enabled(void) {
#ifdef LOWBIT_DEBUG_CHECKS
    return 1;
#else
    return 0;
#endif
}

LOWBIT_API lowbit_status lowbit_selftest_index_check(void* stream) {
    if (!lowbit_debug_checks_enabled()) return LOWBIT_ERR_UNSUPPORTED;
    const lowbit_status st = check_device();
    if (st != LOWBIT_OK) return st;
    return selftest_index_check(static_cast<cudaStream_t>(stream));
}

LOWBIT_API lowbit_status lowbit_selftest_bounded_wait(long long limit_cycles, void* stream) {
    if (limit_cycles <= 0) return LOWBIT_ERR_INVALID_ARG;
    const lowbit_status st = check_device();
    if (st != LOWBIT_OK) return st;
    return selftest_bounded_wait(limit_cycles, static_cast<cudaStream_t>(stream));
}
