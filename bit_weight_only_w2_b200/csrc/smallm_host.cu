// Host side of the small-M kernel (smallm_kernel.cuh): orientation, tile choice, tensor maps and
// launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "lowbit_internal.h"
#include "smallm_kernel.cuh"

namespace lowbit {
namespace smallm {
namespace {

const void* kernel_for(int bits, int gs, int noct, bool swap) {
    switch (bits) {
        case 1: return kernel_b1(gs, noct, swap);
        case 2: return kernel_b2(gs, noct, swap);
        case 4: return kernel_b4(gs, noct, swap);
        default: return nullptr;
    }
}

std::mutex g_mu;

// Allows the kernel the full shared memory, once per entry point and device (the opt-in is a
// per-device function attribute).
bool prepare(const void* fn) {
    struct Done {
        const void* fn;
        int dev;
    };
    static Done done[8 * 3 * 2 * (kMaxOct + kMaxOct / 2)];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < used; ++i)
        if (done[i].fn == fn && done[i].dev == dev) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess) return false;
    if (used < static_cast<int>(sizeof(done) / sizeof(done[0]))) done[used++] = Done{fn, dev};
    return true;
}

// Clusters of `ks` CTAs that fit on the current device at once (one CTA per SM), cached per
// device and entry point family (all octet counts of a format share the occupancy of one CTA
// per SM).
int cluster_capacity(const void* fn, int bits, int gs, int ks, bool swap) {
    constexpr int kDevices = 16;
    static int cache[kDevices][3][2][2][9] = {};
    const int bi = bits == 1 ? 0 : bits == 2 ? 1 : 2, gi = gs == 64 ? 0 : 1, si = swap ? 1 : 0;
    int dev = 0;
    cudaGetDevice(&dev);
    const bool cached = dev >= 0 && dev < kDevices;
    if (cached) {
        std::lock_guard<std::mutex> lock(g_mu);
        if (cache[dev][bi][gi][si][ks] > 0) return cache[dev][bi][gi][si][ks];
    }
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = ks;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(1, ks, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 200 * 1024;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / ks;
    }
    if (n <= 0) n = 1;
    if (cached) {
        std::lock_guard<std::mutex> lock(g_mu);
        cache[dev][bi][gi][si][ks] = n;
    }
    return n;
}

struct Choice {
    int rows, ksplit, kslice, clusters;
};

// Time model of the kernel, fitted to B200 measurements at 16 tokens (microseconds): a 512-wide
// K step of a CTA costs a + b * rows (a: the step's fixed work -- waiting for the ring, the X
// fragments, group sums and scale table, the refill -- b: decode, MMAs and scaling per row), and
// summing K slices across a cluster about 2 us per row block. Long-K runs gave a = 0.64 /
// b = 0.0072 for uint4 and 0.41 / 0.0086 for ternary; binary uses the ternary figures.
double step_us(int bits, int rows) { return bits == 4 ? 0.64 + 0.0072 * rows : 0.41 + 0.0086 * rows; }
constexpr double kSplitUs = 2.0;

// Rows per CTA (a multiple of `align`: 8, or 16 with weights as the 16-row operand) and K slices
// with the smallest modelled time: waves x (steps per slice x step time + the split's reduction).
Choice choose(const void* probe, int bits, int gs, int N, int K, int force_rows, int force_split, bool swap) {
    const int align = swap ? 16 : 8;
    Choice best{0, 0, 0, 0};
    double best_cost = 0;
    for (int ks = 1; ks <= 8; ++ks) {
        if (force_split && ks != force_split) continue;
        const int kslice = ((K + ks * kStepK - 1) / (ks * kStepK)) * kStepK;
        const int ks_eff = (K + kslice - 1) / kslice;
        if (!force_split && ks_eff != ks) continue;
        const int cap = cluster_capacity(probe, bits, gs, ks_eff, swap);
        int fit = align * ((N + align * cap - 1) / (align * cap));   // rows that spread N over every cluster
        if (fit < align) fit = align;
        if (fit > kMaxRows) fit = kMaxRows;
        const int cands[5] = {force_rows ? force_rows : fit, 64, 96, 128, 48};
        for (int c = 0; c < (force_rows ? 1 : 5); ++c) {
            const int rows = cands[c];
            if (rows % align || rows > kMaxRows) continue;
            const int nb = (N + rows - 1) / rows;
            const int waves = (nb + cap - 1) / cap;
            const double cost = waves * ((kslice / kStepK) * step_us(bits, rows) + (ks_eff > 1 ? kSplitUs : 0.0));
            if (!best.rows || cost < best_cost) {
                best = Choice{rows, ks_eff, kslice, nb < cap ? nb : cap};
                best_cost = cost;
            }
        }
    }
    return best;
}

template <int BITS, int GS>
lowbit_status launch(const GemmProblem& g, int force_rows, int force_split, bool swap, cudaStream_t stream) {
    using F = Fmt<BITS, GS>;
    const int M = static_cast<int>(g.M), N = static_cast<int>(g.N), K = static_cast<int>(g.K);
    const void* probe = kernel_for(BITS, GS, 8, swap);
    if (!probe || !prepare(probe)) return LOWBIT_ERR_CUDA;
    const Choice ch = choose(probe, BITS, GS, N, K, force_rows, force_split, swap);
    const void* fn = kernel_for(BITS, GS, ch.rows / 8, swap);
    if (!fn || !prepare(fn)) return LOWBIT_ERR_CUDA;
    Params p;
    int smem = 0;
    if (!layout<BITS, GS>(ch.rows, ch.ksplit, swap, &p, &smem)) return LOWBIT_ERR_UNSUPPORTED;
    p.M = M;
    p.N = N;
    p.K = K;
    p.kslice = ch.kslice;
    p.ksplit = ch.ksplit;
    p.n_tiles = (N + ch.rows - 1) / ch.rows;
    p.Y = static_cast<__nv_bfloat16*>(g.Y);
    p.status = device_status_address();
    if (!p.status) return LOWBIT_ERR_CUDA;

    CUtensorMap mx, mw, ms, mz;
    const uint64_t xdims[3] = {64, static_cast<uint64_t>(M), static_cast<uint64_t>(K) / 64};
    const uint64_t xstr[2] = {static_cast<uint64_t>(K) * 2, 128};
    const uint32_t xbox[3] = {64, static_cast<uint32_t>(swap ? kSwapTokens : kTokens), kStepK / 64};
    bool ok = make_map_3d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.X, xdims, xstr, xbox, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, g.Wp, uint64_t(K) * BITS / 32, N,
                           uint64_t(K) * BITS / 8, F::kWBoxWords, ch.rows,
                           BITS == 1 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.scales, N, K / GS, uint64_t(N) * 2, ch.rows,
                           F::kGroups, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (BITS == 4)
        ok = ok && make_map_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.zeros, N, K / GS, uint64_t(N) * 2,
                               ch.rows, F::kGroups, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        mz = ms;
    if (!ok) return LOWBIT_ERR_CUDA;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (ch.ksplit > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = ch.ksplit;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.gridDim = dim3(ch.clusters, ch.ksplit, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    void* args[] = {&mx, &mw, &ms, &mz, &p};
    if (take_injected_failure(kInjectLaunch)) return LOWBIT_ERR_CUDA;
    return cudaLaunchKernelExC(&cfg, fn, args) == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace
}  // namespace smallm

bool smallm_supported(const GemmProblem& g) { return g.M >= 1 && g.M <= smallm::kTokens; }

lowbit_status smallm_launch(const GemmProblem& g, int rows, int ksplit, bool swap, cudaStream_t stream) {
    if (!smallm_supported(g) || (swap && g.M > smallm::kSwapTokens)) return LOWBIT_ERR_UNSUPPORTED;
    if (rows < 0 || rows > smallm::kMaxRows || rows % (swap ? 16 : 8) != 0 || ksplit < 0 || ksplit > 8)
        return LOWBIT_ERR_UNSUPPORTED;
    switch (g.bits * 1000 + g.group_size) {
        case 1064: return smallm::launch<1, 64>(g, rows, ksplit, swap, stream);
        case 1128: return smallm::launch<1, 128>(g, rows, ksplit, swap, stream);
        case 2064: return smallm::launch<2, 64>(g, rows, ksplit, swap, stream);
        case 2128: return smallm::launch<2, 128>(g, rows, ksplit, swap, stream);
        case 4064: return smallm::launch<4, 64>(g, rows, ksplit, swap, stream);
        case 4128: return smallm::launch<4, 128>(g, rows, ksplit, swap, stream);
        default: return LOWBIT_ERR_UNSUPPORTED;
    }
}

}  // namespace lowbit
