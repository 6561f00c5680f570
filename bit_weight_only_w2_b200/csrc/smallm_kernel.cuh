// Small-M weight-only low-bit GEMM (M <= 16 tokens) for sm_100a: the HBM-bound case, e.g. the
// Qwen3 text-encoder linears at 16 tokens (mlx-vlm Bonsai article, component architecture:
// bits=4, group_size=64) or a GEMV-like decode step.
//
// At 16 tokens the work is streaming the packed weights; the multiply-accumulates still exceed
// what CUDA-core FMAs sustain at HBM speed, so they run on warp-level tensor-core MMAs
// (mma.sync m16n8k16, bf16 in, fp32 accumulate). tcgen05.mma is the wrong tool here: measured
// on B200 it costs at least ~45 clocks per instruction with M = 128 however narrow N is, while
// mma.sync sustains ~1000 MACs per clock per SM (one per ~8 clocks per SM sub-partition, also
// with the decode instructions interleaved) and takes its B operand from registers, so decoded
// weights need no staging. Its latency is long (~90 clocks when chains restart), so each warp
// keeps several independent accumulator chains (weight-row octets) in flight; the number of
// octets per CTA is a template parameter so that a step's chains form one straight-line block
// the compiler can interleave.
//
// Arithmetic. X is used as stored (bf16); codes are decoded WITHOUT their scale into exact bf16
// values and the group scale is applied to fp32 group sums afterwards:
//   binary   w = s * (+-1)                       -> decode +-1 exactly
//   ternary  w = s * (f - 1),     f = t + 1       -> decode 128 + f exactly, subtract 129 * s * Sx
//   uint4    w = s * (q - z)                     -> decode 128 + q exactly, subtract s * (128 + z) * Sx
// where Sx is the sum of the group's X entries per token (an MMA against a ones operand). Each
// product is exact in fp32, so the only roundings are the fp32 accumulations and the final bf16
// store; no X conversion pass is needed.
//
// Work decomposition. A CTA (one per SM) owns 8 * NOCT weight rows (<= 128) and one K slice; the
// K slices of a row block run on the CTAs of a thread-block cluster and are summed in rank
// order through distributed shared memory. Tiles are visited persistently when there are more
// row blocks than co-resident clusters. Inside a CTA:
//   * 512-wide K steps stream through a shared-memory ring with TMA: the X slice [16 tokens]
//     [512] (rows past M are zero-filled by the copy), the packed codes of the tile's rows and
//     the scales (and zeros) of the step's groups. There is no producer warp: thread 0 issues
//     the first ring's worth, and afterwards the last warp to finish with a slot refills it
//     (a shared-memory arrival counter), so no warp ever blocks on a slot being released;
//   * eight warps, each taking 64 of the step's 512 K (one group or half of one) for all the
//     tile's octets (kHalves = 2 instead runs sixteen warps of 128 registers, warps w and w + 8
//     sharing a K chunk with half the octets each). A warp turns its group's fp16 scales /
//     zeros for its rows into fp32 pairs (s, -s * c), loads its four X fragments once with
//     ldmatrix, forms Sx with four MMAs against ones, and runs the decode + MMA chains of its
//     octets, each lane loading one 32-bit code word per block of block-ordered codes;
//   * at the end of a tile the eight K-chunk partial sums of every octet are added in a fixed
//     order through shared memory, then across the cluster, so results do not depend on timing.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "lowbit_internal.h"
#include "sm100_ptx.cuh"

namespace lowbit {
namespace smallm {

constexpr int kKWarps = 8;                        // 64-wide K chunks per step
// Octet halves per K chunk: with 2, warps w and w + 8 take the same K chunk, each for half the
// octets (16 warps of 128 registers). Measured on B200 with block-ordered codes, 1 (8 warps)
// is as fast or faster on the 16-token text-encoder shapes, so it is the one built.
constexpr int kHalves = 1;
constexpr int kWarps = kKWarps * kHalves;
constexpr int kThreads = kWarps * 32;
constexpr int kStepK = 512;                       // K per ring step
constexpr int kTokens = 16;                       // tokens per MMA tile, X as the 16-row operand
constexpr int kSwapTokens = 8;                    // tokens per MMA tile, weights as the 16-row operand
constexpr int kMaxRows = 128;
constexpr int kMaxOct = kMaxRows / 8;
constexpr int kMaxChains = kHalves == 1 ? 12 : 5;  // accumulator chains interleaved per sub-batch
constexpr int kMaxStages = 8;
// X slice of one step: [tokens][512] bf16 (16 KB, or 8 KB with weights as the 16-row operand)
constexpr int x_bytes(bool swap) { return (swap ? kSwapTokens : kTokens) * kStepK * 2; }
constexpr int kSmemLimit = 227 * 1024;
constexpr int kBarBytes = 256;
constexpr uint32_t kBf16One2 = 0x3F803F80u;       // bf16 pair (1, 1)

template <int BITS, int GS>
struct Fmt {
    static constexpr int kGroups = kStepK / GS;              // scale rows per step
    static constexpr int kWBoxes = BITS == 4 ? 2 : 1;        // TMA boxes of codes per step
    static constexpr int kWRow = BITS == 1 ? 64 : 128;       // bytes per row per box
    static constexpr int kWBoxWords = kWRow / 4;
};

struct Params {
    int M, N, K;
    int kslice, ksplit;   // K per cluster rank (multiple of 512) and ranks per cluster
    int n_tiles;          // ceil(N / rows)
    int stages;
    uint32_t stage_bytes, w_off, s_off, z_off, tx_bytes;
    uint32_t scr_off, red_off, part_off, bar_off;
    __nv_bfloat16* Y;
    unsigned* status;     // the device status word (bounded waits record timeouts here)
};

// Shared-memory layout for `rows` weight rows per tile (a multiple of 16 when `swap`). Every TMA
// destination starts on a 128-byte boundary (1024 for the swizzled X and code boxes). Returns
// false if fewer than two ring stages fit. A tile's MMA units are its octets of rows, or with
// `swap` its pairs of octets (16 rows, the A operand's height).
template <int BITS, int GS>
bool layout(int rows, int ksplit, bool swap, Params* p, int* smem_bytes) {
    using F = Fmt<BITS, GS>;
    const int units = swap ? rows / 16 : rows / 8;
    const uint32_t xb = x_bytes(swap);
    const uint32_t w_bytes = F::kWBoxes * rows * F::kWRow;   // a multiple of 512
    const uint32_t s_raw = F::kGroups * rows * 2;
    const uint32_t s_bytes = (s_raw + 127) / 128 * 128;
    p->w_off = xb;
    p->s_off = p->w_off + w_bytes;
    p->z_off = p->s_off + s_bytes;
    const uint32_t end = p->z_off + (BITS == 4 ? s_bytes : 0);
    p->stage_bytes = (end + 1023) / 1024 * 1024;
    p->tx_bytes = xb + w_bytes + s_raw * (BITS == 4 ? 2 : 1);
    // per warp, fp32 (s, -s * c) of its rows: four float4 per octet (pairs of rows), or eight per
    // unit with `swap` (rows g and g + 8 of the unit for each g)
    const uint32_t scr = kWarps * (swap ? 8 : 4) * ((units + kHalves - 1) / kHalves) * 16;
    const uint32_t red = 4 * units * 512;
    // receive buffer of the units this rank finishes: [ksplit][ceil(units / ksplit)][32 lanes]
    const uint32_t part = ksplit > 1 ? ksplit * ((units + ksplit - 1) / ksplit) * 512 : 0;
    const int fixed = static_cast<int>(scr + red + part) + kBarBytes + 1024;
    int stages = (kSmemLimit - fixed) / static_cast<int>(p->stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    p->stages = stages;
    p->scr_off = stages * p->stage_bytes;
    p->red_off = p->scr_off + scr;
    p->part_off = p->red_off + red;
    p->bar_off = p->part_off + part;
    *smem_bytes = static_cast<int>(p->bar_off) + kBarBytes + 1024;
    return true;
}

// ---- device helpers -------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with a zero accumulator input (first K step of a group sum).
__device__ __forceinline__ void mma_bf16_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// (d0, d1) = (a0 * b0 + d0, a1 * b1 + d1): one packed fp32 FMA (each lane rounded once, as fmaf).
__device__ __forceinline__ void fma_f32x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 rd, ra, rb;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rd, {%0, %1};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void cta_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }

// Shared-memory counter increment with acquire-release ordering at CTA scope; returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}


// Exact bf16 pairs of two neighbouring codes (k, k + 1) at pair index c of a packed word (c a
// compile-time constant after unrolling, so pair 0 needs no shift).
__device__ __forceinline__ uint32_t dec_u4(uint32_t v, int c) {       // 128 + q
    return and_or(v >> (4 * c), 0x000F000Fu, 0x43004300u);
}
__device__ __forceinline__ uint32_t dec_t2(uint32_t v, int c) {       // 128 + f, f = t + 1
    return and_or(v >> (2 * c), 0x00030003u, 0x43004300u);
}
__device__ __forceinline__ uint32_t dec_b1(uint32_t v, int c) {       // +-1 by the code bit
    return xor_andnot(0x3F803F80u, v << (15 - c), 0x80008000u);
}

template <int BITS, int GS, int NOCT, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
    lowbit_smallm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                         const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_z,
                         const Params p) {
    using F = Fmt<BITS, GS>;
    static_assert(!SWAP || NOCT % 2 == 0, "weights as the 16-row operand take rows in pairs of octets");
    constexpr int R = 8 * NOCT;                       // weight rows per tile
    constexpr int NUT = SWAP ? NOCT / 2 : NOCT;       // MMA units per tile: octets, or 16-row pairs of octets
    constexpr int NH = (NUT + kHalves - 1) / kHalves; // units per warp (its half of the tile)
    constexpr int HP = (SWAP ? 8 : 4) * NH;           // scale-table entries of a warp
    constexpr int NB = (NH + kMaxChains - 1) / kMaxChains;
    constexpr int B = (NH + NB - 1) / NB;             // units per sub-batch
    constexpr int WPS = BITS == 4 ? 2 : BITS == 2 ? 1 : 2;   // code words per lane per octet per step
    constexpr int OPU = SWAP ? 2 : 1;                 // octets per unit
    constexpr uint32_t kAtomBytes = (SWAP ? kSwapTokens : kTokens) * 128;   // one 64-wide k-atom of X
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_s);
        if (BITS == 4) tma_prefetch_desc(&map_z);
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    uint8_t* ring = smem;
    float4* red = reinterpret_cast<float4*>(smem + p.red_off);
    float4* part = reinterpret_cast<float4*>(smem + p.part_off);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(full + kMaxStages);   // per slot: warps done, all rounds
    uint32_t* iss = cnt + kMaxStages;                         // per slot: fills issued
    volatile int* abort_flag = reinterpret_cast<volatile int*>(iss + kMaxStages);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ks = p.ksplit;
    const int rank = static_cast<int>(blockIdx.y);
    const int k_begin = rank * p.kslice;
    const int k_len = min(p.kslice, p.K - k_begin);   // > 0 by construction
    const int nst = (k_len + kStepK - 1) / kStepK;
    const int my_tiles = (p.n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                         static_cast<int>(gridDim.x);
    const int total = my_tiles * nst;                 // ring steps this CTA consumes

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            mbar_init(&full[i], 1);
            cnt[i] = 0;
            iss[i] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (ks > 1) cluster_sync_all();   // every CTA of the cluster has started (remote stores target it)
    grid_launch_dependents();

    // Ring step `gs` of this CTA: tile blockIdx.x + (gs / nst) * gridDim.x, K step gs % nst.
    // Every CTA of a slice reads the same X (only its weight rows differ). Walking the slice's K
    // steps from a different first step per CTA spreads those reads over the whole slice, instead
    // of every SM asking the same few L2 lines for the same 16 KB at the same moment. (Each CTA's
    // summation order is still fixed, so results stay run-to-run identical.)
    const int rot = static_cast<int>(blockIdx.x) % nst;
    auto issue = [&](int gs, bool codes, bool x) {
        const int s = gs % S;
        uint8_t* st = ring + s * p.stage_bytes;
        const int n0 = (static_cast<int>(blockIdx.x) + (gs / nst) * static_cast<int>(gridDim.x)) * R;
        int kc = gs % nst + rot;
        if (kc >= nst) kc -= nst;
        const int kk = k_begin + kc * kStepK;
        if (codes) {
            mbar_arrive_expect_tx(&full[s], p.tx_bytes);
#pragma unroll
            for (int b = 0; b < F::kWBoxes; ++b)
                tma_load_2d(&map_w, &full[s], st + p.w_off + b * R * F::kWRow, kk * BITS / 32 + b * F::kWBoxWords, n0);
            tma_load_2d(&map_s, &full[s], st + p.s_off, n0, kk / GS);
            if (BITS == 4) tma_load_2d(&map_z, &full[s], st + p.z_off, n0, kk / GS);
        }
        if (x) tma_load_3d(&map_x, &full[s], st, 0, 0, kk / 64);
    };
    // The codes, scales and zeros are not written by earlier kernels of the stream that this one
    // may overlap, X may be: thread 0 queues step 0's codes, waits for those kernels, then X of
    // step 0 and the rest of the first ring (the copy engine serves requests in order, so step 0
    // completes first). The ring runs `look` = S steps ahead: the last warp out of step it
    // queues step it + look. (Measured on the 16-token text-encoder shapes: looking 2, 3 or S
    // steps ahead gives the same time.)
    const int look = S;
    const int pre = min(look, total);
    if (threadIdx.x == 0) {
        if (pre > 0) issue(0, true, false);
        grid_dependency_wait();
        for (int gs = 0; gs < pre; ++gs) {
            if (gs > 0) issue(gs, true, false);
            issue(gs, false, true);
            iss[gs] = 1;
        }
    }

    const int w = warp & (kKWarps - 1);      // this warp's 64-wide K chunk of every step
    const int ob0 = (warp / kKWarps) * NH;   // first unit of this warp's half of the tile
    const int nh = (NUT % kHalves == 0) ? NH : min(NH, NUT - ob0);   // units it owns
    const int g = lane >> 2;                 // fragment row group: weight row in the octet (B / A rows)
    const int q = lane & 3;
    const int gi = (w * 64) / GS;            // this warp's group within a step
    // X fragments: with X as the 16-row A operand, lane supplies token lane & 15 of k half lane >> 4;
    // with weights as A, X is the n8 B operand and lane supplies token lane & 7 of 16-byte chunk
    // lane >> 3 (plus 4 for the second pair of K steps).
    const int tok = SWAP ? (lane & 7) : (lane & 15);
    const uint32_t xoff = static_cast<uint32_t>(w * kAtomBytes + tok * 128);
    const int xhalf = lane >> 4;
    // This lane's code bytes in row g of octet 0 of a step (swizzled as the TMA wrote them; the
    // swizzle depends on the row only through g, so octet o is at a fixed offset from it). 2- and
    // 4-bit codes are in block order: each 16-byte unit of a row is one block of four words, and
    // word q of a block is exactly lane q's codes for the block's columns, so a lane loads one
    // word per block: two blocks (uint4) or one (ternary) per 64-wide K chunk.
    uint32_t wb0, wb1;                       // the lane's word in each block (binary: 8 bytes)
    constexpr uint32_t kOctStride = BITS == 1 ? 512u : 1024u;
    if (BITS == 4) {
        const int c0 = 2 * (w & 3);
        wb0 = static_cast<uint32_t>((w >> 2) * R * 128 + g * 128 + ((c0 ^ g) << 4) + 4 * q);
        wb1 = static_cast<uint32_t>((w >> 2) * R * 128 + g * 128 + (((c0 + 1) ^ g) << 4) + 4 * q);
    } else if (BITS == 2) {
        wb0 = wb1 = static_cast<uint32_t>(g * 128 + ((w ^ g) << 4) + 4 * q);
    } else {
        wb0 = wb1 = static_cast<uint32_t>(g * 64 + (((w >> 1) ^ ((g >> 1) & 3)) << 4) + (w & 1) * 8);
    }
    float4* scr = reinterpret_cast<float4*>(smem + p.scr_off) + warp * HP;

    float acc[NH][4];
#pragma unroll
    for (int o = 0; o < NH; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.f;

    // ---- the phases of one ring step, shared by both loop drivers below ----
    // P1: this warp's group: fp32 (s, -s * c) of every row of its units, into `tab` (negated so
    // that the scale epilogue is two packed FMAs per pair of accumulators)
    auto build_table = [&](const uint8_t* st, float4* tab) {
        const __half* sh = reinterpret_cast<const __half*>(st + p.s_off) + gi * R;
        const __half* zh = reinterpret_cast<const __half*>(st + p.z_off) + gi * R;
        auto sc_of = [&](int r, float& sf, float& cf) {
            sf = __half2float(sh[r]);
            cf = BITS == 4 ? -(sf * (128.f + __half2float(zh[r]))) : BITS == 2 ? -(129.f * sf) : 0.f;
        };
        if constexpr (SWAP) {
            // entry 8u + g: rows 16u + g and 16u + g + 8 of the warp's units
#pragma unroll
            for (int i0 = 0; i0 < HP; i0 += 32) {
                const int i = i0 + lane;
                if (i < 8 * nh) {
                    const int r = 16 * (ob0 + (i >> 3)) + (i & 7);
                    float s0, c0, s1, c1;
                    sc_of(r, s0, c0);
                    sc_of(r + 8, s1, c1);
                    tab[i] = make_float4(s0, s1, c0, c1);
                }
            }
        } else {
            const __half2* sp = reinterpret_cast<const __half2*>(sh) + 4 * ob0;
            const __half2* zp = reinterpret_cast<const __half2*>(zh) + 4 * ob0;
#pragma unroll
            for (int i0 = 0; i0 < HP; i0 += 32) {
                const int i = i0 + lane;
                if (i < 4 * nh) {
                    const float2 sf = __half22float2(sp[i]);
                    float c0 = 0.f, c1 = 0.f;
                    if (BITS == 4) {
                        const float2 zf = __half22float2(zp[i]);
                        c0 = -(sf.x * (128.f + zf.x));
                        c1 = -(sf.y * (128.f + zf.y));
                    } else if (BITS == 2) {
                        c0 = -(129.f * sf.x);
                        c1 = -(129.f * sf.y);
                    }
                    tab[i] = make_float4(sf.x, sf.y, c0, c1);
                }
            }
        }
    };
    // P2: X fragments of this warp's four 16-wide K steps (128-byte swizzled rows): a[j] = the A
    // operand of step j, or with SWAP a[p] = the B operands of steps 2p, 2p + 1
    auto load_frags = [&](uint32_t st_u, uint32_t (&a)[4][4]) {
        if constexpr (SWAP) {
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                const int chunk = 4 * pp + (lane >> 3);
                ldmatrix_x4(st_u + xoff + static_cast<uint32_t>((chunk ^ tok) << 4), a[pp]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int chunk = (j << 1) | xhalf;
                ldmatrix_x4(st_u + xoff + static_cast<uint32_t>((chunk ^ (tok & 7)) << 4), a[j]);
            }
        }
    };
    // P3: group sums of X: tokens g (0) and g + 8 (2), or with SWAP tokens 2q (0) and 2q + 1 (1)
    auto group_sums = [&](const uint32_t (&a)[4][4], float (&tsx)[4]) {
        tsx[0] = tsx[1] = tsx[2] = tsx[3] = 0.f;
        if (BITS != 1) {
            if constexpr (SWAP) {
                const uint32_t ones[4] = {kBf16One2, kBf16One2, kBf16One2, kBf16One2};
                mma_bf16_z(tsx, ones, a[0][0], a[0][1]);
                mma_bf16(tsx, ones, a[0][2], a[0][3]);
                mma_bf16(tsx, ones, a[1][0], a[1][1]);
                mma_bf16(tsx, ones, a[1][2], a[1][3]);
            } else {
                mma_bf16_z(tsx, a[0], kBf16One2, kBf16One2);
#pragma unroll
                for (int j = 1; j < 4; ++j) mma_bf16(tsx, a[j], kBf16One2, kBf16One2);
            }
        }
    };
    // P4: code words of the sub-batch starting at unit ob, for this warp's 64 K
    auto load_codes = [&](const uint8_t* wst, int ob, uint32_t (&wd)[B][OPU][WPS]) {
#pragma unroll
        for (int u = 0; u < B; ++u) {
            if (ob + u < nh) {
#pragma unroll
                for (int h = 0; h < OPU; ++h) {
                    const uint8_t* rp = wst + (OPU * (ob0 + ob + u) + h) * kOctStride;
                    if (BITS == 4) {
                        wd[u][h][0] = *reinterpret_cast<const uint32_t*>(rp + wb0);
                        wd[u][h][1] = *reinterpret_cast<const uint32_t*>(rp + wb1);
                    } else if (BITS == 2) {
                        wd[u][h][0] = *reinterpret_cast<const uint32_t*>(rp + wb0);
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2*>(rp + wb0);
                        wd[u][h][0] = v.x; wd[u][h][1] = v.y;
                    }
                }
            }
        }
    };
    // P5: decode + MMA chains of the sub-batch: T[u] = the unscaled group sums of unit ob + u
    auto mma_units = [&](const uint32_t (&a)[4][4], const uint32_t (&wd)[B][OPU][WPS], int ob, float (&T)[B][4]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int u = 0; u < B; ++u) {
                if (ob + u < nh) {
                    // (b0, b1): row g's codes for k = 2q, 2q + 1 and 2q + 8, 2q + 9 of step j
                    uint32_t b0[OPU], b1[OPU];
#pragma unroll
                    for (int h = 0; h < OPU; ++h) {
                        if (BITS == 4) {           // block j / 2, pairs 2(j % 2) and + 1
                            b0[h] = dec_u4(wd[u][h][j >> 1], 2 * (j & 1));
                            b1[h] = dec_u4(wd[u][h][j >> 1], 2 * (j & 1) + 1);
                        } else if (BITS == 2) {    // the chunk's block, pairs 2j and 2j + 1
                            b0[h] = dec_t2(wd[u][h][0], 2 * j);
                            b1[h] = dec_t2(wd[u][h][0], 2 * j + 1);
                        } else {
                            const int pc = (j & 1) * 8 + q;
                            b0[h] = dec_b1(wd[u][h][j >> 1], pc);
                            b1[h] = dec_b1(wd[u][h][j >> 1], pc + 4);
                        }
                    }
                    if constexpr (SWAP) {
                        // A = rows g (octet 2u) and g + 8 (octet 2u + 1) of the unit
                        const uint32_t aw[4] = {b0[0], b0[OPU - 1], b1[0], b1[OPU - 1]};
                        const uint32_t x0 = a[j >> 1][2 * (j & 1)], x1 = a[j >> 1][2 * (j & 1) + 1];
                        if (j == 0) mma_bf16_z(T[u], aw, x0, x1);
                        else mma_bf16(T[u], aw, x0, x1);
                    } else {
                        if (j == 0) mma_bf16_z(T[u], a[0], b0[0], b1[0]);
                        else mma_bf16(T[u], a[j], b0[0], b1[0]);
                    }
                }
            }
        }
    };
    // P6: scale the group sums and add them to the accumulators, acc += s * T + (-s * c) * Sx, as
    // packed fp32 FMAs over pairs of accumulators (bit-identical to one fmaf per element)
    auto scale_units = [&](const float (&T)[B][4], const float (&tsx)[4], const float4* tab, int ob) {
#pragma unroll
        for (int u = 0; u < B; ++u) {
            if (ob + u < nh) {
                float* d = acc[ob + u];
                if constexpr (SWAP) {
                    // d: (row g, token 2q), (row g, 2q + 1), (row g + 8, 2q), (row g + 8, 2q + 1)
                    const float4 sc = tab[8 * (ob + u) + g];
                    fma_f32x2(d[0], d[1], sc.x, sc.x, T[u][0], T[u][1]);
                    fma_f32x2(d[2], d[3], sc.y, sc.y, T[u][2], T[u][3]);
                    if (BITS != 1) {
                        fma_f32x2(d[0], d[1], sc.z, sc.z, tsx[0], tsx[1]);
                        fma_f32x2(d[2], d[3], sc.w, sc.w, tsx[0], tsx[1]);
                    }
                } else {
                    // d: (token g, row 2q), (g, 2q + 1), (g + 8, 2q), (g + 8, 2q + 1)
                    const float4 sc = tab[4 * (ob + u) + q];
                    fma_f32x2(d[0], d[1], sc.x, sc.y, T[u][0], T[u][1]);
                    fma_f32x2(d[2], d[3], sc.x, sc.y, T[u][2], T[u][3]);
                    if (BITS != 1) {
                        fma_f32x2(d[0], d[1], sc.z, sc.w, tsx[0], tsx[0]);
                        fma_f32x2(d[2], d[3], sc.z, sc.w, tsx[2], tsx[2]);
                    }
                }
            }
        }
    };
    // Release a ring slot; the last warp out queues ring step it + look into it. Once no step is
    // left to queue, this slot (and every later step's) needs no count.
    auto release = [&](int it_done, int slot) {
        __syncwarp();
        if (lane == 0 && it_done + look < total) {
            const uint32_t prev = atom_add_acq_rel(&cnt[slot], 1);
            if ((prev & (kWarps - 1)) == kWarps - 1 && !*abort_flag) {
                issue(it_done + look, true, true);
                iss[slot] += 1;
            }
        }
    };

    int it = 0;
    int s = 0;                               // ring slot of step it, and its fill parity
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
        for (int c = 0; c < nst; ++c, ++it) {
            ok = ok && __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, p.status));
            bool released = false;
            if (ok) {
                const uint8_t* st = ring + s * p.stage_bytes;
                build_table(st, scr);         // (read back by the other lanes after the first sub-batch's MMAs)
                uint32_t a[4][4];
                load_frags(smem_u32(st), a);
                float tsx[4];
                group_sums(a, tsx);
#pragma unroll
                for (int ob = 0; ob < NH; ob += B) {
                    uint32_t wd[B][OPU][WPS];
                    load_codes(st + p.w_off, ob, wd);
                    float T[B][4];
                    mma_units(a, wd, ob, T);
                    if (ob + B >= NH) {
                        release(it, s);       // the last shared-memory read of this slot is done
                        released = true;
                    } else if (ob == 0) {
                        __syncwarp();         // the scale entries above are written
                    }
                    scale_units(T, tsx, scr, ob);
                }
            }
            if (!released) release(it, s);
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
        }

        // ---- tile end: every unit's eight K-chunk partials (one per warp of its half) are added
        // in a fixed order. On a CTA's only tile the drained ring holds all eight: one exchange,
        // ((((c0 + c1) + c2) + ...) + c7). Otherwise the ring already holds the next tile's steps
        // and `red` takes two rounds: (c + (c + 4)) for chunks c < 4, then ((0 + 1) + 2) + 3.
        grid_dependency_wait();   // Y may still be read by the kernel this one overlaps
        const bool one_round =
            my_tiles == 1 && static_cast<uint32_t>(S) * p.stage_bytes >= kKWarps * NUT * 512u;
        float4* rbuf = one_round ? reinterpret_cast<float4*>(ring) : red;
        const int nslot = one_round ? kKWarps : 4;
        cta_bar();                // the ring is drained / the previous tile's readers of `red` are done
        if (one_round || w >= 4) {
            const int slot = one_round ? w : w - 4;
#pragma unroll
            for (int o = 0; o < NH; ++o)
                if (o < nh)
                    rbuf[(slot * NUT + ob0 + o) * 32 + lane] = make_float4(acc[o][0], acc[o][1], acc[o][2], acc[o][3]);
        }
        cta_bar();
        if (!one_round) {
            if (w < 4) {
#pragma unroll
                for (int o = 0; o < NH; ++o) {
                    if (o < nh) {
                        const float4 v = red[(w * NUT + ob0 + o) * 32 + lane];
                        acc[o][0] += v.x;
                        acc[o][1] += v.y;
                        acc[o][2] += v.z;
                        acc[o][3] += v.w;
                    }
                }
            }
            cta_bar();
            if (w < 4) {
#pragma unroll
                for (int o = 0; o < NH; ++o)
                    if (o < nh)
                        red[(w * NUT + ob0 + o) * 32 + lane] = make_float4(acc[o][0], acc[o][1], acc[o][2], acc[o][3]);
            }
            cta_bar();
        }
#pragma unroll
        for (int o = 0; o < NH; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.f;

        const int n0 = t * R;
        auto store = [&](int o, float4 v) {
            if constexpr (SWAP) {
                // rows n and n + 8 of unit o, tokens 2q and 2q + 1
                const int n = n0 + 16 * o + g;
                const int t0 = 2 * q;
                if (dcheck(o < NUT && n >= 0, p.status)) {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int ne = n + (e >> 1) * 8, te = t0 + (e & 1);
                        if (ne < p.N && te < p.M) p.Y[static_cast<size_t>(te) * p.N + ne] = __float2bfloat16_rn(vv[e]);
                    }
                }
            } else {
                const int n = n0 + 8 * o + 2 * q;
                if (n < p.N && dcheck(n >= 0 && n + 1 < p.N && o < NUT, p.status)) {
                    if (g < p.M)
                        *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<size_t>(g) * p.N + n) =
                            __floats2bfloat162_rn(v.x, v.y);
                    if (g + 8 < p.M)
                        *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<size_t>(g + 8) * p.N + n) =
                            __floats2bfloat162_rn(v.z, v.w);
                }
            }
        };
        auto tile_sum = [&](int o) {
            float4 v = rbuf[o * 32 + lane];
#pragma unroll
            for (int r = 1; r < kKWarps; ++r) {
                if (r >= nslot) break;
                const float4 u = rbuf[(r * NUT + o) * 32 + lane];
                v.x += u.x;
                v.y += u.y;
                v.z += u.z;
                v.w += u.w;
            }
            return v;
        };
        if (ks == 1) {
            for (int o = warp; o < NUT; o += kWarps) store(o, tile_sum(o));
        } else {
            // Unit o is finished by rank o % ks: every rank stores its tile sum of o straight into
            // that rank's receive buffer (slot [own rank][o / ks]); after a cluster barrier the
            // finishing rank adds the slots in rank order; a second barrier keeps the buffers
            // (and every CTA) alive until all ranks have read them.
            const int per = (NUT + ks - 1) / ks;
            for (int o = warp; o < NUT; o += kWarps) {
                const uint32_t slot = smem_u32(part + ((rank * per + o / ks) * 32 + lane));
                st_shared_cluster_v4(map_shared_rank(slot, o % ks), tile_sum(o));
            }
            cluster_sync_all();
            for (int o = warp; o < NUT; o += kWarps) {
                if (o % ks != rank) continue;
                const int li = o / ks;
                float4 sum = part[li * 32 + lane];
#pragma unroll
                for (int r = 1; r < 8; ++r)
                    if (r < ks) {
                        const float4 v = part[(r * per + li) * 32 + lane];
                        sum.x += v.x;
                        sum.y += v.y;
                        sum.z += v.z;
                        sum.w += v.w;
                    }
                store(o, sum);
            }
            cluster_sync_all();
        }
    }
    // Leave no copy in flight into shared memory (only possible after an aborted wait).
    cta_bar();
    if (threadIdx.x == 0 && *abort_flag) {
        int zero = 0;
        for (int i = 0; i < S; ++i)
            if (iss[i]) mbar_wait(&full[i], (iss[i] - 1) & 1u, &zero, p.status, kWaitLimitCycles / 8);
    }
}

// Kernel entry for (BITS, GS), `noct` octets per tile (1..16) and the orientation (`swap`:
// weights as the 16-row operand, even `noct` only), or nullptr. One definition per code width
// lives in its own translation unit so the instantiations build in parallel.
const void* kernel_b1(int group_size, int noct, bool swap);
const void* kernel_b2(int group_size, int noct, bool swap);
const void* kernel_b4(int group_size, int noct, bool swap);

}  // namespace smallm
}  // namespace lowbit

// Defines kernel_b<BITS>: tables of the sixteen octet counts (and the eight even ones with weights
// as the 16-row operand) for both group sizes.
#define LOWBIT_SMALLM_TABLE(BITS)                                                                     \
    namespace lowbit {                                                                                \
    namespace smallm {                                                                                \
    template <int GS, int... Ns>                                                                      \
    static const void* pick_##BITS(int noct, std::integer_sequence<int, Ns...>) {                     \
        static const void* const table[] = {                                                          \
            reinterpret_cast<const void*>(&lowbit_smallm_kernel<BITS, GS, Ns + 1, false>)...};        \
        return (noct >= 1 && noct <= static_cast<int>(sizeof...(Ns))) ? table[noct - 1] : nullptr;    \
    }                                                                                                 \
    template <int GS, int... Ns>                                                                      \
    static const void* pick_swap_##BITS(int noct, std::integer_sequence<int, Ns...>) {                \
        static const void* const table[] = {                                                          \
            reinterpret_cast<const void*>(&lowbit_smallm_kernel<BITS, GS, 2 * (Ns + 1), true>)...};   \
        return (noct >= 2 && noct % 2 == 0 && noct / 2 <= static_cast<int>(sizeof...(Ns)))           \
                   ? table[noct / 2 - 1] : nullptr;                                                   \
    }                                                                                                 \
    const void* kernel_b##BITS(int group_size, int noct, bool swap) {                                 \
        if (swap) {                                                                                   \
            if (group_size == 64) return pick_swap_##BITS<64>(noct, std::make_integer_sequence<int, kMaxOct / 2>{}); \
            if (group_size == 128) return pick_swap_##BITS<128>(noct, std::make_integer_sequence<int, kMaxOct / 2>{}); \
            return nullptr;                                                                           \
        }                                                                                             \
        if (group_size == 64) return pick_##BITS<64>(noct, std::make_integer_sequence<int, kMaxOct>{}); \
        if (group_size == 128) return pick_##BITS<128>(noct, std::make_integer_sequence<int, kMaxOct>{}); \
        return nullptr;                                                                               \
    }                                                                                                 \
    }                                                                                                 \
    }
