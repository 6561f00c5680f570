// Small-M weight-only low-bit GEMM (M <= 16 tokens) for sm_100a: the HBM-bound case, e.g. the
// Qwen3 text-encoder linears at 16 tokens (mlx-vlm Bonsai article, component architecture:
// bits=4, group_size=64) or a GEMV-like decode step.
//
// At 16 tokens the work is streaming the packed weights; the multiply-accumulates still exceed
// what CUDA-core FMAs can sustain at HBM speed, so they run on tensor cores. The warp-level
// mma.sync.m16n8k16 path suits this shape better than tcgen05.mma: measured on B200, a
// tcgen05.mma with M = 128 costs at least ~45 clocks however narrow N is (~45 weights per clock
// per SM at N = 16), while mma.sync sustains ~1000 MACs per clock per SM (~64 weights per clock
// at 16 tokens) and takes its B operand from registers, so decoded weights need no staging.
//
// Design:
//   * A CTA owns 64 weight rows (8 consumer warps x 8 rows) and one K slice; the K slices of a
//     row block run on the CTAs of a thread-block cluster and their fp32 partials are summed in
//     rank order through distributed shared memory.
//   * A producer warp streams the packed codes, scales (and zeros) of the CTA's rows through a
//     shared-memory ring with TMA (the first stages before waiting for the X conversion), and
//     copies the CTA's slice of the fp16 X into shared memory with bulk copies.
//   * Each consumer lane decodes, for every 16-wide K step, the two code pairs that form its B
//     fragment (row = lane / 4, k pairs 2q and 2q + 8 with q = lane % 4) straight to fp16x2, loads
//     the A fragment of X with ldmatrix, and issues mma.sync (fp32 accumulation).
//   * Decoding is the same exact fp16 arithmetic as the large-M kernel: binary / ternary weights
//     are exactly +-s or 0, uint4 weights (q - z) * s round once.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "lowbit_internal.h"
#include "sm100_ptx.cuh"

namespace lowbit {
namespace {

constexpr int kGvWarps = 8;                   // consumer warps, 8 weight rows each
constexpr int kGvRows = kGvWarps * 8;         // weight rows per CTA
constexpr int kGvThreads = (kGvWarps + 1) * 32;
constexpr int kGvK = 128;                     // K per weight stage
constexpr int kGvStages = 8;
constexpr int kGvMaxKSlice = 1280;            // K per CTA at most (bounds the X slice in smem)
constexpr int kGvTokens = 16;

template <int BITS, int GS>
struct GvCfg {
    static constexpr int kWords = kGvK * BITS / 32;          // packed words per row per stage
    static constexpr int kRowBytes = kWords * 4;              // 16 / 32 / 64
    static constexpr int kWBytes = kGvRows * kRowBytes;
    static constexpr int kGroups = kGvK / GS;                 // scale rows per stage
    static constexpr int kSBytes = kGroups * kGvRows * 2;
    static constexpr int kZBytes = (BITS == 4) ? kSBytes : 0;
    static constexpr int kSOff = kWBytes;
    static constexpr int kZOff = kSOff + kSBytes;
    static constexpr int kStageBytes = (kZOff + kZBytes + 1023) / 1024 * 1024;
    static constexpr int kXStride = (kGvMaxKSlice + 8) * 2;   // bytes per token row of the X slice
    static constexpr int kXBytes = kGvTokens * kXStride;
    static constexpr int kRingOff = (kXBytes + 1023) / 1024 * 1024;
    static constexpr int kPartOff = kRingOff + kGvStages * kStageBytes;
    static constexpr int kPartBytes = kGvWarps * 32 * 16;     // 4 fp32 per consumer lane
    static constexpr int kBarOff = kPartOff + kPartBytes;
    static constexpr int kSmemBytes = 1024 + kBarOff + 256;
};

struct GvParams {
    int M, N, K;
    int kslice;          // K per cluster rank (multiple of 128)
    int ksplit;
    const uint16_t* Xh;  // fp16 [M][K]
    const float* rowmul;
    __nv_bfloat16* Y;
    unsigned* status;    // the device status word (bounded waits record timeouts here)
};

// Decoders for one code pair (k, k + 1) at pair index c of a packed word, to fp16x2.
template <int BITS>
__device__ __forceinline__ uint32_t decode_pair(uint32_t v, int c, uint32_t s2, uint32_t c2) {
    if (BITS == 1) {
        return xor_andnot(s2, v << (15 - c), 0x80008000u);            // +-s by the code bit
    } else if (BITS == 2) {
        const uint32_t e = and_or(v >> (2 * c), 0x00030003u, 0x64006400u);  // 1024 + f, exact
        const uint32_t t = f16x2_fma(e, 0x3C003C00u, 0xE401E401u);         // f - 1, exact
        return f16x2_mul(t, s2);
    } else {
        const uint32_t e = and_or(v >> (4 * c), 0x000F000Fu, 0x64006400u);  // 1024 + q, exact
        const uint32_t q = f16x2_fma(e, 0x3C003C00u, 0xE400E400u);         // q, exact
        return f16x2_fma(q, s2, c2);                                       // q * s - z * s
    }
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int BITS, int GS>
__global__ void __launch_bounds__(kGvThreads, 2)
    lowbit_gemv_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_s,
                       const __grid_constant__ CUtensorMap map_z, const GvParams p) {
    using C = GvCfg<BITS, GS>;
    constexpr int S = kGvStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xs = smem;
    uint8_t* ring = smem + C::kRingOff;
    float* part = reinterpret_cast<float*>(smem + C::kPartOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + S;
    uint64_t* xbar = empty + S;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kGvRows;
    const int rank = static_cast<int>(blockIdx.y);
    const int k_begin = rank * p.kslice;
    const int k_len = min(p.kslice, p.K - k_begin);      // > 0 by construction, multiple of 64
    const int nchunks = (k_len + kGvK - 1) / kGvK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGvWarps);
        }
        mbar_init(xbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Zero the X slice (token rows past M and K past the slice stay zero; the copies fill the rest).
    for (int i = threadIdx.x; i < C::kXBytes / 16; i += kGvThreads)
        reinterpret_cast<uint4*>(xs)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    grid_launch_dependents();

    if (warp == kGvWarps) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&map_w);
            tma_prefetch_desc(&map_s);
            if (BITS == 4) tma_prefetch_desc(&map_z);
            const uint32_t tx = C::kWBytes + C::kSBytes + C::kZBytes;
            auto issue = [&](int c) {
                const int s = c % S;
                uint8_t* st = ring + s * C::kStageBytes;
                const int kk = k_begin + c * kGvK;
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_2d(&map_w, &full[s], st, kk * BITS / 32, n0);
                tma_load_2d(&map_s, &full[s], st + C::kSOff, n0, kk / GS);
                if (BITS == 4) tma_load_2d(&map_z, &full[s], st + C::kZOff, n0, kk / GS);
            };
            // Weights are not written by the X conversion just before this kernel (which itself
            // starts only after everything earlier in the stream has finished): fetch them now.
            const int pre = nchunks < S ? nchunks : S;
            for (int c = 0; c < pre; ++c) issue(c);
            grid_dependency_wait();
            const int mrows = min(p.M, kGvTokens);
            mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(mrows * k_len * 2));
            for (int m = 0; m < mrows; ++m)
                bulk_g2s(xs + m * C::kXStride, p.Xh + static_cast<size_t>(m) * p.K + k_begin,
                         static_cast<uint32_t>(k_len * 2), xbar);
            for (int c = pre; c < nchunks; ++c) {
                if (!mbar_wait(&empty[c % S], ((c / S) & 1u) ^ 1u, abort_flag, p.status)) break;
                issue(c);
            }
        }
    } else {
        // ---------------------------------------------------------------- consumer warps
        const int g = lane >> 2;                 // row within the warp's 8 = B column
        const int q = lane & 3;                  // k pair within a 16-wide step
        const int rl = warp * 8 + g;             // row within the CTA
        // ldmatrix addresses: lanes 0-15 rows 0-15 at k, lanes 16-31 rows 0-15 at k + 8
        const uint32_t xaddr = smem_u32(xs) + static_cast<uint32_t>((lane & 15) * C::kXStride + (lane >> 4) * 16);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        bool ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0, abort_flag, p.status));
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c % S;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (c / S) & 1u, abort_flag, p.status))) break;
            const uint8_t* st = ring + s * C::kStageBytes;
            // this row's words (swizzled like the TMA wrote them) and its group scales / zeros
            uint32_t w[C::kWords];
            const uint8_t* wrow = st + rl * C::kRowBytes;
#pragma unroll
            for (int ch = 0; ch < C::kRowBytes / 16; ++ch) {
                int pc = ch;
                if (C::kRowBytes == 32) pc = ch ^ ((rl >> 2) & 1);
                if (C::kRowBytes == 64) pc = ch ^ ((rl >> 1) & 3);
                const uint4 v = *reinterpret_cast<const uint4*>(wrow + pc * 16);
                w[4 * ch + 0] = v.x;
                w[4 * ch + 1] = v.y;
                w[4 * ch + 2] = v.z;
                w[4 * ch + 3] = v.w;
            }
            uint32_t s2[C::kGroups], c2[C::kGroups];
#pragma unroll
            for (int gi = 0; gi < C::kGroups; ++gi) {
                const uint32_t sb = reinterpret_cast<const uint16_t*>(st + C::kSOff)[gi * kGvRows + rl];
                s2[gi] = sb | (sb << 16);
                c2[gi] = 0;
                if (BITS == 4) {
                    const uint16_t zb = reinterpret_cast<const uint16_t*>(st + C::kZOff)[gi * kGvRows + rl];
                    const float cz = -__half2float(__ushort_as_half(zb)) *
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(sb)));
                    const uint32_t cb = __half_as_ushort(__float2half_rn(cz));
                    c2[gi] = cb | (cb << 16);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            const uint32_t kx = xaddr + static_cast<uint32_t>(c * kGvK * 2);
#pragma unroll
            for (int j = 0; j < kGvK / 16; ++j) {
                const int gi = (j * 16) / GS;
                uint32_t b0, b1;
                if (BITS == 1) {
                    const uint32_t v = w[j >> 1];
                    const int c0 = (j & 1) * 8 + q;
                    b0 = decode_pair<1>(v, c0, s2[gi], 0);
                    b1 = decode_pair<1>(v, c0 + 4, s2[gi], 0);
                } else if (BITS == 2) {
                    b0 = decode_pair<2>(w[j], q, s2[gi], 0);
                    b1 = decode_pair<2>(w[j], q + 4, s2[gi], 0);
                } else {
                    b0 = decode_pair<4>(w[2 * j], q, s2[gi], c2[gi]);
                    b1 = decode_pair<4>(w[2 * j + 1], q, s2[gi], c2[gi]);
                }
                uint32_t a[4];
                ldmatrix_x4(kx + j * 32, a);
                mma_16816(acc, a, b0, b1);
            }
        }
        // ---- epilogue: acc[0..1] = tokens g, rows 2q, 2q+1; acc[2..3] = token g + 8
        grid_dependency_wait();
        const int n = n0 + warp * 8 + 2 * q;
        if (p.ksplit == 1) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int m = g + 8 * h;
                if (m < p.M && n < p.N) {
                    const float mul = p.rowmul[m];
                    const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * h] * mul, acc[2 * h + 1] * mul);
                    *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<size_t>(m) * p.N + n) = v;
                }
            }
        } else {
            *reinterpret_cast<float4*>(part + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }

    if (p.ksplit > 1) {
        // Sum the K slices in rank order: rank r finishes the warps w with w % ksplit == r.
        __syncwarp();
        cluster_sync_all();
        if (warp < kGvWarps && !*abort_flag && warp % p.ksplit == rank) {
            const int g = lane >> 2, q = lane & 3;
            const uint32_t off = smem_u32(part + (warp * 32 + lane) * 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r = 0; r < p.ksplit; ++r) {
                const float4 v = ld_shared_cluster_v4(map_shared_rank(off, r));
                sum.x += v.x;
                sum.y += v.y;
                sum.z += v.z;
                sum.w += v.w;
            }
            const float a4[4] = {sum.x, sum.y, sum.z, sum.w};
            const int n = n0 + warp * 8 + 2 * q;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int m = g + 8 * h;
                if (m < p.M && n < p.N) {
                    const float mul = p.rowmul[m];
                    const __nv_bfloat162 v = __floats2bfloat162_rn(a4[2 * h] * mul, a4[2 * h + 1] * mul);
                    *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<size_t>(m) * p.N + n) = v;
                }
            }
        }
        cluster_sync_all();
    }
}

template <int BITS, int GS>
lowbit_status gv_launch(const GemmProblem& g, int ksplit_request, cudaStream_t stream) {
    using C = GvCfg<BITS, GS>;
    auto kernel = lowbit_gemv_kernel<BITS, GS>;
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return LOWBIT_ERR_CUDA;
        attr_done = true;
    }
    const int M = static_cast<int>(g.M), N = static_cast<int>(g.N), K = static_cast<int>(g.K);
    const CUtensorMapSwizzle wswz = C::kRowBytes == 16   ? CU_TENSOR_MAP_SWIZZLE_NONE
                                    : C::kRowBytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                         : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mw, ms, mz;
    bool ok = make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, g.Wp, uint64_t(K) * BITS / 32, N,
                          uint64_t(K) * BITS / 8, C::kWords, kGvRows, wswz);
    ok = ok && make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.scales, N, K / GS, uint64_t(N) * 2, kGvRows,
                           C::kGroups, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (BITS == 4)
        ok = ok && make_map_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.zeros, N, K / GS, uint64_t(N) * 2,
                               kGvRows, C::kGroups, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        mz = ms;
    if (!ok) return LOWBIT_ERR_CUDA;

    // K split: at most kGvMaxKSlice per CTA, and enough CTAs for about two per SM.
    const int nblocks = (N + kGvRows - 1) / kGvRows;
    const int nchunks = (K + kGvK - 1) / kGvK;
    int ksplit = ksplit_request;
    if (ksplit <= 0) {
        const int sms = num_sms();
        ksplit = (K + kGvMaxKSlice - 1) / kGvMaxKSlice;
        const int want = (2 * sms + nblocks - 1) / nblocks;
        if (want > ksplit) ksplit = want;
    }
    if (ksplit > 8) ksplit = 8;
    if (ksplit > nchunks) ksplit = nchunks;
    int per = (nchunks + ksplit - 1) / ksplit;
    if (per * kGvK > kGvMaxKSlice) return LOWBIT_ERR_UNSUPPORTED;   // K too large for one cluster
    ksplit = (nchunks + per - 1) / per;                              // every rank gets K
    const WorkspaceLayout ws = workspace_layout(g.M, g.K);
    GvParams p;
    p.M = M;
    p.N = N;
    p.K = K;
    p.kslice = per * kGvK;
    p.ksplit = ksplit;
    p.Xh = static_cast<const uint16_t*>(g.workspace);
    p.rowmul = reinterpret_cast<const float*>(static_cast<const uint8_t*>(g.workspace) + ws.rowmul_offset);
    p.Y = static_cast<__nv_bfloat16*>(g.Y);
    p.status = device_status_address();
    if (!p.status) return LOWBIT_ERR_CUDA;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (ksplit > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = ksplit;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.gridDim = dim3(nblocks, ksplit, 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, mw, ms, mz, p) == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

}  // namespace

bool gemv_supported(const GemmProblem& g) {
    const int64_t nchunks = (g.K + kGvK - 1) / kGvK;
    return g.M <= kGvTokens && (nchunks + 7) / 8 * kGvK <= kGvMaxKSlice;
}

lowbit_status gemv_launch(const GemmProblem& g, int ksplit, cudaStream_t stream) {
    if (!gemv_supported(g)) return LOWBIT_ERR_UNSUPPORTED;
    const lowbit_status st = launch_convert_x(g, stream);
    if (st != LOWBIT_OK) return st;
    switch (g.bits * 1000 + g.group_size) {
        case 1064: return gv_launch<1, 64>(g, ksplit, stream);
        case 1128: return gv_launch<1, 128>(g, ksplit, stream);
        case 2064: return gv_launch<2, 64>(g, ksplit, stream);
        case 2128: return gv_launch<2, 128>(g, ksplit, stream);
        case 4064: return gv_launch<4, 64>(g, ksplit, stream);
        case 4128: return gv_launch<4, 128>(g, ksplit, stream);
        default: return LOWBIT_ERR_UNSUPPORTED;
    }
}

}  // namespace lowbit
