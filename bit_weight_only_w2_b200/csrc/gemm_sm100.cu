// Weight-only low-bit GEMM for sm_100a:  Y[M][N] = X[M][K] * W^T,  W decoded from packed
// binary / ternary / uint4 codes and fp16 group scales (and zeros).
//
// The multiply behind the Bonsai Image (FLUX.2-Klein-4B) transformer linears: binary weights
// w = scale_g * b (bonsai-image-binary-4B-gemlite-1bit model card, "Binary Weight
// Representation: 1-bit g128"), ternary 2-bit weights (mlx-vlm Bonsai article, model
// overview) and the 4-bit group-64 text-encoder linears (same article, component
// architecture). After decoding it is a dense contraction, so it runs on the tcgen05 tensor
// cores.
//
// Precision: the tensor cores run in fp16 with fp32 accumulation. A pre-pass converts X from
// bf16 to fp16 (exact: every bf16 value in fp16's normal range is an fp16 value), with a
// per-row power-of-two scale so that rows whose magnitude exceeds fp16's range still convert
// exactly (the epilogue multiplies that row back). In fp16 a binary or ternary weight t * s is
// exactly +-s or 0 for the fp16 scale s, and a uint4 weight (q - z) * s is rounded once to fp16
// (2^-11 relative); rounding s to bf16 instead would cost up to 2^-8 per group, enough to
// break a 1e-2 tolerance in the tails.
//
// Kernel design ("swap AB", weights as the MMA's A operand):
//   * One CTA tile = up to 128 weight rows (MMA M) x BT tokens (MMA N), K in stages of 128.
//   * Warp 0 (one lane) is the TMA producer: per stage it loads two 64-wide, 128B-swizzled
//     boxes of the fp16 copy of X (the MMA's B operand, K-major), the packed code box of the
//     tile's rows and their group scales (and zeros) into a shared-memory ring. The first
//     stages' weight boxes are requested before waiting for the X conversion to finish.
//   * The dequant warps each own 32 weight rows (one per lane, matching the tensor-memory lane
//     quarter the warp may access): they read the row's packed words from shared memory,
//     decode codes x scale to fp16 pairs with a few integer / fp16x2 instructions per pair,
//     and store them straight into a tensor-memory ring with tcgen05.st. The decoded weights
//     never touch shared memory, which leaves its bandwidth to TMA and the MMA's B reads.
//   * Warp 1 (one lane) issues tcgen05.mma (kind::f16, A from tensor memory, B from shared
//     memory, fp32 accumulators in tensor memory) and frees ring slots with tcgen05.commit.
//   * Epilogue warps (8 for 128/256-token tiles) read the accumulators with tcgen05.ld, apply
//     the row's power-of-two factor, round to bf16 into registers and hand the accumulator
//     back before storing, so a tile's stores overlap the next tile's MMAs even with a single
//     accumulator buffer; neighbouring lanes swap halves so each store writes two outputs.
//   * Grids: persistent over 128-row tiles when there are many; for small M either "flat"
//     tiles of ceil(N / #SMs) rows with the whole K per CTA, or K split over the CTAs of a
//     thread-block cluster whose fp32 partial tiles are summed in rank order through
//     distributed shared memory.
//   * Every mbarrier wait is bounded (see sm100_ptx.cuh): a wait that gives up records
//     LOWBIT_ERR_TIMEOUT in the device status word and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include <cstdint>
#include <cstdio>

#include "lowbit_internal.h"
#include "sm100_ptx.cuh"
#include "tcgen05_ptx.cuh"

namespace lowbit {

__device__ unsigned g_device_status = 0;

constexpr int kBlockN = 128;        // weight rows per tile at most (MMA M)
constexpr int kBlockK = 128;        // K per pipeline stage
constexpr int kNumCtrlWarps = 2;    // warp 0: TMA producer, warp 1: MMA issuer + TMEM owner
constexpr int kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per block

// PAIR: a tile of 256 weight rows x BT tokens computed by a CTA pair on cta_group::2 MMAs. Each
// CTA decodes its 128 weight rows into its own tensor memory and loads half of the X tile (BT/2
// tokens); the even CTA issues the MMAs, which read both halves of X, so every X element read
// into shared memory serves 256 weight rows instead of 128.
template <int BITS, int GS, int BT, bool PAIR = false>
struct Cfg {
    static_assert(BITS == 1 || BITS == 2 || BITS == 4, "bits");
    static_assert(GS == 64 || GS == 128, "group size");
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N");
    static_assert(!PAIR || BT == 256, "pair tiles are 256 x 256");
    static constexpr int kCtasPerSm = (BT <= 64) ? 2 : 1;
    // Epilogue: warps e and e+4 cover the same 32 weight rows (TMEM lane quarter = warp % 4),
    // each half of the tile's token columns when there are 8.
    static constexpr int kNumEpiWarps = (BT >= 128) ? 8 : 4;
    static constexpr int kEpiParts = kNumEpiWarps / 4;
    static constexpr int kEpiCols = BT / kEpiParts;                 // accumulator columns per thread
    static constexpr int kNumDqWarps = (BITS == 4) ? 8 : 4;
    static constexpr int kParts = kNumDqWarps / 4;                  // dequant warps per row quarter
    static constexpr int kFirstEpiWarp = kNumCtrlWarps;
    static constexpr int kFirstDqWarp = kNumCtrlWarps + kNumEpiWarps;
    static constexpr int kThreads = 32 * (kNumCtrlWarps + kNumEpiWarps + kNumDqWarps);
    static constexpr int kNumAcc = (BT == 64 || BT == 256) ? 1 : 2;   // fit the tensor-memory budget
    static constexpr int kAccCols = kNumAcc * BT;
    static constexpr int kACol0 = (kAccCols + 31) / 32 * 32;
    static constexpr int kNumA = (kCtasPerSm == 2) ? 3 : 4;          // A ring stages (64 columns each)
    static constexpr int kColsUsed = kACol0 + kNumA * 64;
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                     : kColsUsed <= 256 ? 256 : 512;
    static_assert(kColsUsed <= 512 && kTmemCols * kCtasPerSm <= 512, "tensor memory");

    static constexpr int kWordsPerRow = kBlockK * BITS / 32;        // 4 / 8 / 16
    static constexpr int kWRowBytes = kWordsPerRow * 4;             // 16 / 32 / 64
    static constexpr int kXRows = PAIR ? BT / 2 : BT;               // token rows of X in this CTA
    static constexpr int kXHalfBytes = kXRows * 128;                // 64 fp16 per row
    static constexpr int kXBytes = 2 * kXHalfBytes;
    static constexpr int kWBytes = kBlockN * kWRowBytes;
    static constexpr int kGroupsPerStage = kBlockK / GS;            // 1 or 2
    static constexpr int kSBytes = kGroupsPerStage * kBlockN * 2;
    static constexpr int kZBytes = (BITS == 4) ? kSBytes : 0;
    // Two rings in shared memory: X stages (the MMA's B operand, freed by the MMA) and weight
    // stages (packed codes + scales + zeros, freed by the dequant warps). The weight ring runs
    // ahead of the X ring, so decoding never waits for X. One X stage is one 128-wide k-block,
    // fetched by a single TMA request (large requests stream from L2 faster than small ones).
    static constexpr int kXStageBytes = kXBytes;                    // a multiple of 2048
    static constexpr int kWOff = 0;
    static constexpr int kSOff = kWBytes;
    static constexpr int kZOff = kSOff + kSBytes;
    static constexpr int kWStageBytes = (kZOff + kZBytes + 1023) / 1024 * 1024;
    static constexpr int kWTxFixed = kSBytes + kZBytes;            // plus rows * kWRowBytes
    static constexpr int kBarBytes = 1024;
    static constexpr int kBudget = kSmemLimit / kCtasPerSm - 1024 /*align*/ - kBarBytes - 2048 /*reserve*/;
    static constexpr int kXStagesFit = (kBudget - 2 * kWStageBytes) / kXStageBytes;
    static constexpr int kXStages = kXStagesFit > 8 ? 8 : kXStagesFit;
    static constexpr int kWStagesFit = (kBudget - kXStages * kXStageBytes) / kWStageBytes;
    static constexpr int kWStages = kWStagesFit > 8 ? 8 : kWStagesFit;
    static_assert(kXStages >= 2 && kWStages >= 2, "shared memory");
    static constexpr int kWRingOff = kXStages * kXStageBytes;
    static constexpr int kBarOff = kWRingOff + kWStages * kWStageBytes;
    // Request enough shared memory that at most kCtasPerSm CTAs of these kernels share an SM:
    // tensor memory (512 columns per SM) is not a scheduling resource, so residency is capped
    // through shared memory instead (228 KB per SM).
    static constexpr int kSmemNeeded = 1024 + kBarOff + kBarBytes;
    static constexpr int kSmemFloor = (kCtasPerSm == 2) ? 80 * 1024 : 150 * 1024;
    static constexpr int kSmemBytes = kSmemNeeded > kSmemFloor ? kSmemNeeded : kSmemFloor;
    static_assert(kSmemBytes <= kSmemLimit, "shared memory");
    // split-K receive buffers (fp32 [ksplit][128 rows][odd number of 16-byte chunks]) reuse the
    // X ring: the largest over ksplit 2..8
    static constexpr int recv_bytes(int ks) {
        return ks * kBlockN * ((((BT + ks - 1) / ks + 3) / 4) | 1) * 16;
    }
    static constexpr int max_recv_bytes() {
        int m = 0;
        for (int ks = 2; ks <= 8; ++ks) m = recv_bytes(ks) > m ? recv_bytes(ks) : m;
        return m;
    }
    static_assert(PAIR || max_recv_bytes() <= kXStages * kXStageBytes, "split-K receive buffer");
    static constexpr uint32_t kIdesc = idesc_f16_f32(PAIR ? 2 * kBlockN : kBlockN, BT);
    // the last tile's bf16 Y box [BT][128 rows] is staged at the start of the (idle) X ring
    static constexpr int kYStageBytes = BT * kBlockN * 2;
    static_assert(kYStageBytes <= kXStages * kXStageBytes, "Y staging");
};

struct KernelParams {
    int M, N, K;
    int num_kb;          // k-blocks of 128
    int kb_per_split;    // k-blocks per cluster rank (split-K), else num_kb
    int rows;            // weight rows per tile: 128, or fewer (multiple of 8) for small M
    int m_tiles, n_tiles, num_tiles;
    int ksplit;          // cluster size along z (1 = no split)
    uint32_t wtx_bytes;  // bytes delivered into one weight stage
    __nv_bfloat16* Y;
    const float* rowmul; // per-row power-of-two factor written by the X conversion pass
};

// ---------------------------------------------------------------------------------------------
// Decoders: one 64-wide K half of one weight row -> 32 fp16x2 values (even k low, odd k high),
// out[i] holding columns 2i and 2i + 1 of the half. 2- and 4-bit words are in block order
// (word q of a four-word block holds, in pair p, columns 8p + 2q and 8p + 2q + 1 of the
// block), so pair p of word w lands in out[4p + q] of its block; binary words are in plain order.
// ---------------------------------------------------------------------------------------------

// Binary: bit 1 -> +s, 0 -> -s. Pair c of a word is (bit c, bit 16 + c); shifting the word
// left by 15 - c puts them on the two fp16 sign bits, and one LOP3 flips the sign of s where
// the bit is 0. Exact.
__device__ __forceinline__ void decode_half_b1(uint32_t w0, uint32_t w1, uint32_t s2, uint32_t (&out)[32]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) out[c] = xor_andnot(s2, w0 << (15 - c), 0x80008000u);
#pragma unroll
    for (int c = 0; c < 16; ++c) out[16 + c] = xor_andnot(s2, w1 << (15 - c), 0x80008000u);
}

// Ternary: field f = t + 1 in {0,1,2}. OR-ing the two fields of a pair, left at bit 2j of each
// half, into the mantissas of fp16 1024.0 gives e = 1024 + f * 4^j exactly (j <= 4 keeps the
// field inside the 10-bit mantissa). One fp16x2 FMA computes e * 4^-j - (1024 * 4^-j + 1) =
// f - 1 = t exactly (the exact result is representable, so nothing rounds) and a multiply by
// s gives t * s exactly. Pairs 0..4 are decoded in place, pairs 5..7 after one shift by 10.
// Word q of the half's only block: pair c goes to out[4c + q].
__device__ __forceinline__ void decode_word_b2(uint32_t v, uint32_t s2, uint32_t* out, int q) {
    constexpr uint32_t kMagic = 0x64006400u;                                           // 1024.0
    constexpr uint32_t kMul[5] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u, 0x1C001C00u};  // 4^-j
    constexpr uint32_t kAdd[5] = {0xE401E401u, 0xDC04DC04u, 0xD410D410u, 0xCC40CC40u, 0xC500C500u};  // -(1024*4^-j+1)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int shift = (c < 5) ? 0 : 10;
        const int j = (c < 5) ? c : c - 5;
        const uint32_t e = and_or(v >> shift, 0x00030003u << (2 * j), kMagic);
        const uint32_t t = f16x2_fma(e, kMul[j], kAdd[j]);
        out[4 * c + q] = f16x2_mul(t, s2);
    }
}

// uint4: the nibbles of a pair, left at bit 4j of each half (j <= 1), OR-ed into fp16 1024.0
// give 1024 + q * 16^j exactly, and one fp16x2 FMA recovers q exactly. Each weight is then
// (q - z) * s = q * s + cz with cz = -z * s in fp32 (exact: the product of two fp16 values has
// at most 22 significant bits), formed by one mixed-precision FMA (q * s is exact as well, so
// the only fp32 rounding is below 2^-24 relative) and rounded to fp16 once. A code equal or
// next to its zero point thus keeps the full fp16 precision of the small difference (q - z) * s;
// rounding -z * s to fp16 first would cost up to 2^-11 |z * s| per weight, which is most of
// such a weight. Word w of the half (block w / 4, word q = w % 4 of it): pair c goes to
// out[16 * (w / 4) + 4c + q].
__device__ __forceinline__ void decode_word_b4(uint32_t v, uint16_t s, float cz, uint32_t* out, int w) {
    constexpr uint32_t kMagic = 0x64006400u;
    constexpr uint32_t kMul[2] = {0x3C003C00u, 0x2C002C00u};   // 1, 1/16
    constexpr uint32_t kAdd[2] = {0xE400E400u, 0xD400D400u};   // -1024, -64
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int shift = (c < 2) ? 0 : 8;
        const int j = c & 1;
        const uint32_t e = and_or(v >> shift, 0x000F000Fu << (4 * j), kMagic);
        const uint32_t q = f16x2_fma(e, kMul[j], kAdd[j]);
        float lo, hi;
        fma_f16x2_f32(q, s, cz, lo, hi);
        out[16 * (w >> 2) + 4 * c + (w & 3)] = pack_f16x2(lo, hi);
    }
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
template <int BITS, int GS, int BT, bool PAIR>
__global__ void __launch_bounds__(Cfg<BITS, GS, BT, PAIR>::kThreads, Cfg<BITS, GS, BT, PAIR>::kCtasPerSm)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_z,
                       const __grid_constant__ CUtensorMap map_y, const KernelParams p) {
    using C = Cfg<BITS, GS, BT, PAIR>;
    constexpr int SX = C::kXStages;
    constexpr int SW = C::kWStages;
    constexpr int NA = C::kNumA;
    constexpr int NACC = C::kNumAcc;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* wring = smem + C::kWRingOff;
    uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* xempty = xfull + SX;
    uint64_t* wfull = xempty + SX;
    uint64_t* wempty = wfull + SW;
    uint64_t* afull = wempty + SW;
    uint64_t* aempty = afull + NA;
    uint64_t* accfull = aempty + NA;
    uint64_t* accempty = accfull + NACC;
    uint64_t* drain = accempty + NACC;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Pair mode: the CTA of cluster rank 0 issues the MMAs. The other CTA's X copies complete on
    // the issuer's X barrier, its dequant and epilogue warps arrive on the issuer's A-ready and
    // accumulator-free barriers, and the issuer's commits arrive on the empty / ready barriers of
    // both CTAs (same offsets).
    const uint32_t pair_rank = PAIR ? cluster_ctarank() : 0u;
    const bool issuer = pair_rank == 0;
    constexpr int kPairCtas = PAIR ? 2 : 1;
    auto on_issuer = [&](uint64_t* bar) { return map_shared_rank(smem_u32(bar), 0u); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; ++i) {
            mbar_init(&xfull[i], 1);
            mbar_init(&xempty[i], 1);
        }
        for (int i = 0; i < SW; ++i) {
            mbar_init(&wfull[i], 1);
            mbar_init(&wempty[i], C::kNumDqWarps);
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&afull[i], kPairCtas * C::kNumDqWarps);
            mbar_init(&aempty[i], 1);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], kPairCtas * C::kNumEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_s);
        if (BITS == 4) tma_prefetch_desc(&map_z);
        tma_prefetch_desc(&map_y);
    }
    if (warp == 1) {
        tmem_alloc<PAIR>(tmem_holder, C::kTmemCols);
        tmem_relinquish<PAIR>();
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync_all();   // both CTAs' barriers are initialised before either uses the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // Programmatic dependent launch: the next kernel in the stream may start its prologue now.
    // Threads that touch global memory wait for the previous kernel (the X conversion) first.
    grid_launch_dependents();

    const bool split = p.ksplit > 1;
    const int kb_begin = split ? static_cast<int>(blockIdx.z) * p.kb_per_split : 0;
    const int kb_end = split ? min(p.num_kb, kb_begin + p.kb_per_split) : p.num_kb;
    const int nkb = kb_end - kb_begin;
    // first tile and tile stride of this CTA (a pair's two CTAs, adjacent along x, share both)
    const int tile0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int tile_step = split ? p.num_tiles : static_cast<int>(PAIR ? gridDim.x >> 1 : gridDim.x);
    const int my_tiles = tile0 < p.num_tiles ? (p.num_tiles - 1 - tile0) / tile_step + 1 : 0;
    // first weight row of this CTA in tile t: pair tiles cover 2 * p.rows rows, this CTA's half
    // starting at pair_rank * p.rows
    const int n_stride = PAIR ? 2 * p.rows : p.rows;
    const int n_off = PAIR ? static_cast<int>(pair_rank) * p.rows : 0;
    unsigned* status = &g_device_status;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint32_t total = static_cast<uint32_t>(my_tiles * nkb);
            auto coords = [&](uint32_t it, int& m0, int& n0, int& kb) {
                const int tile = tile0 + static_cast<int>(it / nkb) * tile_step;
                kb = kb_begin + static_cast<int>(it % nkb);
                m0 = (tile / p.n_tiles) * BT;
                n0 = (tile % p.n_tiles) * n_stride + n_off;
            };
            auto issue_w = [&](uint32_t it) {
                int m0, n0, kb;
                coords(it, m0, n0, kb);
                const uint32_t s = it % SW;
                uint8_t* st = wring + s * C::kWStageBytes;
                mbar_arrive_expect_tx(&wfull[s], p.wtx_bytes);
                tma_load_2d(&map_w, &wfull[s], st + C::kWOff, kb * C::kWordsPerRow, n0);
                tma_load_2d(&map_s, &wfull[s], st + C::kSOff, n0, kb * C::kGroupsPerStage);
                if (BITS == 4) tma_load_2d(&map_z, &wfull[s], st + C::kZOff, n0, kb * C::kGroupsPerStage);
            };
            auto issue_x = [&](uint32_t it) {
                int m0, n0, kb;
                coords(it, m0, n0, kb);
                const uint32_t s = it % SX;
                uint8_t* st = smem + s * C::kXStageBytes;
                // box (64 k, kXRows tokens, 2 halves) = both 128-byte-swizzled K halves in one request
                if (!PAIR) {
                    mbar_arrive_expect_tx(&xfull[s], C::kXBytes);
                    tma_load_3d(&map_x, &xfull[s], st, 0, m0, kb * 2);
                } else {
                    // both halves complete on the issuer's barrier, which expects both
                    if (issuer) mbar_arrive_expect_tx(&xfull[s], 2 * C::kXBytes);
                    tma_load_3d_pair(&map_x, on_issuer(&xfull[s]), st, 0, m0 + static_cast<int>(pair_rank) * C::kXRows,
                                     kb * 2);
                }
            };
            // The packed weights and scales are not written by the kernel just before this one
            // (the X conversion, which itself starts only once everything earlier in the stream
            // has completed), so the first weight stages are requested before waiting for it.
            uint32_t itw = 0, itx = 0;
            const uint32_t wpre = total < static_cast<uint32_t>(SW) ? total : static_cast<uint32_t>(SW);
            for (; itw < wpre; ++itw) issue_w(itw);
            grid_dependency_wait();
            // Fill both rings as their slots free up, without blocking on either.
            bool ok = true;
            long long t_last = clock64();
            uint32_t idle = 0;
            while (itx < total || itw < total) {
                bool progress = false;
                if (itx < total && mbar_test_wait(&xempty[itx % SX], ((itx / SX) & 1u) ^ 1u)) {
                    issue_x(itx++);
                    progress = true;
                }
                if (itw < total && mbar_test_wait(&wempty[itw % SW], ((itw / SW) & 1u) ^ 1u)) {
                    issue_w(itw++);
                    progress = true;
                }
                if (progress) {
                    idle = 0;
                    t_last = clock64();
                } else if ((++idle & 63u) == 0) {
                    if (*abort_flag) { ok = false; break; }
                    if (clock64() - t_last > kWaitLimitCycles) {
                        atomicOr(status, kDevErrTimeout);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) {
                // Drain: wait (bounded) for the copies still in flight before the CTA exits. The
                // second CTA of a pair cannot wait on the issuer's barrier its X copies count on:
                // it gives them a fixed time instead (both CTAs meet again before either exits).
                if (PAIR && !issuer) {
                    const long long t0 = clock64();
                    while (clock64() - t0 < kWaitLimitCycles / 64) {
                    }
                } else {
                    for (uint32_t j = (itx > static_cast<uint32_t>(SX) ? itx - SX : 0u); j < itx; ++j) {
                        const long long t0 = clock64();
                        while (!mbar_try_wait(&xfull[j % SX], (j / SX) & 1u) && clock64() - t0 < kWaitLimitCycles) {
                        }
                    }
                }
                for (uint32_t j = (itw > static_cast<uint32_t>(SW) ? itw - SW : 0u); j < itw; ++j) {
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&wfull[j % SW], (j / SW) & 1u) && clock64() - t0 < kWaitLimitCycles) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0 && issuer) {
            uint32_t it = 0, ait = 0, tcount = 0;
            bool ok = true;
            bool issued = false;
            for (int t = 0; t < my_tiles && ok; ++t, ++tcount) {
                const uint32_t b = tcount % NACC, acc_ph = (tcount / NACC) & 1u;
                if (!mbar_wait(&accempty[b], acc_ph ^ 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BT;
                for (int kb = kb_begin; kb < kb_end; ++kb, ++it, ++ait) {
                    const uint32_t s = it % SX, ph = (it / SX) & 1u;
                    const uint32_t a = ait % NA, aph = (ait / NA) & 1u;
                    if (!mbar_wait(&xfull[s], ph, abort_flag, status)) { ok = false; break; }
                    if (!mbar_wait(&afull[a], aph, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t xs = smem_u32(smem + s * C::kXStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; ++kk) {
                        const uint32_t a_tmem = tmem_base + C::kACol0 + a * 64 + kk * 8;
                        const uint64_t bdesc =
                            smem_desc_k_sw128(xs + (kk >> 2) * C::kXHalfBytes + (kk & 3) * 32);
                        if (PAIR)
                            mma_f16_ts_pair(d_tmem, a_tmem, bdesc, C::kIdesc, (kb > kb_begin || kk > 0) ? 1u : 0u);
                        else
                            mma_f16_ts(d_tmem, a_tmem, bdesc, C::kIdesc, (kb > kb_begin || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    if (PAIR) {
                        mma_commit_pair_mc(&xempty[s], 0x3);
                        mma_commit_pair_mc(&aempty[a], 0x3);
                    } else {
                        mma_commit(&xempty[s]);
                        mma_commit(&aempty[a]);
                    }
                }
                if (!ok) break;
                if (PAIR)
                    mma_commit_pair_mc(&accfull[b], 0x3);
                else
                    mma_commit(&accfull[b]);
            }
            if (!ok && issued) {
                // Drain: make sure no MMA is still writing tensor memory before it is freed.
                if (PAIR)
                    mma_commit_pair(drain);
                else
                    mma_commit(drain);
                const long long t0 = clock64();
                while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles) {
                }
            }
        }
    } else if (warp >= C::kFirstDqWarp) {
        // ---------------------------------------------------------------- dequant warps
        const int dq = warp - C::kFirstDqWarp;
        const int quarter = warp & 3;
        const int part = dq >> 2;                    // which K part of the stage this warp decodes
        const int row = quarter * 32 + lane;         // weight row within the tile = TMEM lane
        const bool row_ok = row < p.rows;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        constexpr int kHalvesPerPart = 2 / C::kParts;   // 64-wide K halves decoded by this warp
        uint32_t it = 0, ait = 0;
        bool ok = true;
        for (int t = 0; t < my_tiles && ok; ++t) {
            for (int kb = kb_begin; kb < kb_end; ++kb, ++it, ++ait) {
                const uint32_t s = it % SW, ph = (it / SW) & 1u;
                const uint32_t a = ait % NA, aph = (ait / NA) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&wfull[s], ph, abort_flag, status))) { ok = false; break; }
                const uint8_t* st = wring + s * C::kWStageBytes;
                // --- this row's packed words and scales (rows past the tile decode to zero)
                uint32_t words[kHalvesPerPart][C::kWordsPerRow / 2];
                uint32_t s2[kHalvesPerPart];
                float cz[kHalvesPerPart];
                const uint8_t* wrow = st + C::kWOff + row * C::kWRowBytes;
#pragma unroll
                for (int hh = 0; hh < kHalvesPerPart; ++hh) {
                    const int h = part * kHalvesPerPart + hh;
                    const int gi = (GS == 64) ? h : 0;
#pragma unroll
                    for (int w = 0; w < C::kWordsPerRow / 2; ++w) words[hh][w] = 0;
                    s2[hh] = 0;
                    cz[hh] = 0.f;
                    if (row_ok) {
                        if (BITS == 1) {
                            const uint2 v = *reinterpret_cast<const uint2*>(wrow + h * 8);
                            words[hh][0] = v.x;
                            words[hh][1] = v.y;
                        } else if (BITS == 2) {
                            const int chunk = h ^ ((row >> 2) & 1);           // 32-byte swizzle
                            const uint4 v = *reinterpret_cast<const uint4*>(wrow + chunk * 16);
                            words[hh][0] = v.x; words[hh][1] = v.y; words[hh][2] = v.z; words[hh][3] = v.w;
                        } else {
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const int chunk = (2 * h + q) ^ ((row >> 1) & 3);  // 64-byte swizzle
                                const uint4 v = *reinterpret_cast<const uint4*>(wrow + chunk * 16);
                                words[hh][4 * q + 0] = v.x; words[hh][4 * q + 1] = v.y;
                                words[hh][4 * q + 2] = v.z; words[hh][4 * q + 3] = v.w;
                            }
                        }
                        const uint16_t* srow = reinterpret_cast<const uint16_t*>(st + C::kSOff) + gi * kBlockN;
                        const uint32_t sb = srow[row];
                        s2[hh] = sb | (sb << 16);
                        if (BITS == 4) {   // -z * s, exact in fp32
                            const __half* zrow = reinterpret_cast<const __half*>(st + C::kZOff) + gi * kBlockN;
                            cz[hh] = -__half2float(zrow[row]) *
                                     __half2float(__ushort_as_half(static_cast<unsigned short>(sb)));
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&wempty[s]);
                // --- decode into the tensor-memory A ring
                if (!__all_sync(0xffffffffu, mbar_wait(&aempty[a], aph ^ 1u, abort_flag, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < kHalvesPerPart; ++hh) {
                    const int h = part * kHalvesPerPart + hh;
                    uint32_t out[32];
                    if (BITS == 1) {
                        decode_half_b1(words[hh][0], words[hh][1], s2[hh], out);
                    } else if (BITS == 2) {
#pragma unroll
                        for (int w = 0; w < 4; ++w) decode_word_b2(words[hh][w], s2[hh], out, w);
                    } else {
#pragma unroll
                        for (int w = 0; w < 8; ++w)
                            decode_word_b4(words[hh][w], static_cast<uint16_t>(s2[hh]), cz[hh], out, w);
                    }
                    if (dcheck(C::kACol0 + a * 64 + h * 32 + 32 <= C::kTmemCols, status))
                        tmem_st32(lane_base + C::kACol0 + a * 64 + h * 32, out);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR && !issuer)
                        mbar_arrive_remote(on_issuer(&afull[a]));
                    else
                        mbar_arrive(&afull[a]);
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue warps
        const int e = warp - C::kFirstEpiWarp;
        const int quarter = warp & 3;
        const int epart = e >> 2;                    // which slice of the token columns
        const int col0 = epart * C::kEpiCols;
        const int row = quarter * 32 + lane;
        const bool row_ok = row < p.rows;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        grid_dependency_wait();                      // before the first global access
        constexpr int kChunk = (C::kEpiCols >= 32) ? 32 : 16;
        uint32_t tcount = 0;
        constexpr int kChunks = C::kEpiCols / kChunk;
        for (int t = 0; t < my_tiles; ++t, ++tcount) {
            const int tile = tile0 + t * tile_step;
            const uint32_t b = tcount % NACC, acc_ph = (tcount / NACC) & 1u;
            const int m0 = (tile / p.n_tiles) * BT + col0;   // first token of this thread's columns
            const int n = (tile % p.n_tiles) * n_stride + n_off + row;
            // Lane j of the warp holds the row factor of token m0 + c0 + j of every chunk c0,
            // requested before waiting for the accumulator so the loads overlap the MMAs.
            float mul[kChunks];
#pragma unroll
            for (int ci = 0; ci < kChunks; ++ci) {
                const int mj = m0 + ci * kChunk + lane;
                mul[ci] = (!split && lane < kChunk && mj < p.M && dcheck(mj >= 0, status)) ? p.rowmul[mj] : 1.0f;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&accfull[b], acc_ph, abort_flag, status))) break;
            tc_fence_after();
            if (!split && t + 1 == my_tiles) {
                // The CTA's last tile has nothing to overlap its stores with, and its X ring is
                // idle (the MMAs just completed consumed every stage, and no copy is in flight):
                // the tile goes, chunk by chunk, to the start of the X ring as the Y box [BT
                // tokens][p.rows rows] (one X stage, or two of a CTA pair's half-size stages) and
                // leaves in one TMA store, which clips the parts past M or N.
                uint32_t* stg = reinterpret_cast<uint32_t*>(smem);
                const bool even = (lane & 1) == 0;
                const int r_pair = row - (even ? 0 : 1);   // the pair's even row within the tile
#pragma unroll 1
                for (int c0 = 0; c0 < C::kEpiCols; c0 += kChunk) {
                    uint32_t v[32];
                    if (kChunk == 32) {
                        tmem_ld32(lane_base + b * BT + col0 + c0, v);
                    } else {
                        tmem_ld16(lane_base + b * BT + col0 + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
                    }
                    float mul_j = mul[0];
#pragma unroll
                    for (int ci = 1; ci < kChunks; ++ci)
                        if (ci == c0 / kChunk) mul_j = mul[ci];   // keeps mul[] in registers
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < kChunk; j += 2) {
                        const float f0 = __uint_as_float(v[j]) * __shfl_sync(0xffffffffu, mul_j, j);
                        const float f1 = __uint_as_float(v[j + 1]) * __shfl_sync(0xffffffffu, mul_j, j + 1);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(f0, f1);   // (token j, token j+1)
                        const uint32_t mine = *reinterpret_cast<const uint32_t*>(&h2);
                        // lanes 2i, 2i+1 (rows n, n+1) swap halves: (row n, row n+1) at one token
                        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                        const uint32_t outw =
                            even ? __byte_perm(mine, other, 0x5410) : __byte_perm(other, mine, 0x7632);
                        const int ml = col0 + c0 + j + (even ? 0 : 1);   // token within the tile
                        if (r_pair < p.rows && dcheck((ml * p.rows + r_pair) * 2 + 4 <= C::kYStageBytes, status))
                            stg[(ml * p.rows + r_pair) >> 1] = outw;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR && !issuer)
                        mbar_arrive_remote(on_issuer(&accempty[b]));
                    else
                        mbar_arrive(&accempty[b]);
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 32 * C::kNumEpiWarps);
                if (e == 0 && lane == 0) {
                    tma_store_2d(&map_y, smem, (tile % p.n_tiles) * n_stride + n_off, (tile / p.n_tiles) * BT);
                    bulk_commit_group();
                    bulk_wait_read_all();   // the shared memory may not be released before this
                }
            } else if (!split) {
                // Read the whole slice into registers (scaled, rounded to bf16), hand the
                // accumulator back to the MMA issuer, then store: the stores of this tile
                // overlap the next tile's MMAs.
                uint32_t packed[C::kEpiCols / 2];
#pragma unroll
                for (int c0 = 0; c0 < C::kEpiCols; c0 += kChunk) {
                    uint32_t v[32];
                    if (kChunk == 32) {
                        tmem_ld32(lane_base + b * BT + col0 + c0, v);
                    } else {
                        tmem_ld16(lane_base + b * BT + col0 + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
                    }
                    const float mul_j = mul[c0 / kChunk];
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < kChunk; j += 2) {
                        const float f0 = __uint_as_float(v[j]) * __shfl_sync(0xffffffffu, mul_j, j);
                        const float f1 = __uint_as_float(v[j + 1]) * __shfl_sync(0xffffffffu, mul_j, j + 1);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(f0, f1);   // (token j, token j+1)
                        packed[(c0 + j) / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR && !issuer)
                        mbar_arrive_remote(on_issuer(&accempty[b]));
                    else
                        mbar_arrive(&accempty[b]);
                }
                // Lanes 2i and 2i+1 hold rows n and n+1: one shuffle turns each lane's
                // (token m, token m+1) pair into a 4-byte (row n, row n+1) store at one token.
                const bool even = (lane & 1) == 0;
                const int n_pair = even ? n : n - 1;
                const bool pair_ok = row_ok && (n_pair + 1 < p.N + 1) && n_pair < p.N;
#pragma unroll
                for (int j = 0; j < C::kEpiCols; j += 2) {
                    const uint32_t mine = packed[j / 2];
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                    const uint32_t outw = even ? __byte_perm(mine, other, 0x5410) : __byte_perm(other, mine, 0x7632);
                    const int m = m0 + j + (even ? 0 : 1);
                    if (pair_ok && m < p.M &&
                        dcheck(m >= 0 && n_pair >= 0 && n_pair + 1 < p.N && (n_pair & 1) == 0, status))
                        *reinterpret_cast<uint32_t*>(p.Y + static_cast<size_t>(m) * p.N + n_pair) = outw;
                }
            } else {
                // split-K (one tile per CTA): the accumulator stays in tensor memory until every
                // rank of the cluster has finished its K slice, when it is pushed to the ranks
                // that reduce it (below). The row factors of the tile's tokens go to the weight
                // ring (every stage has been decoded by now), for the reduction to read from
                // shared memory instead of waiting on a global load behind each store.
                const int te = (warp - C::kFirstEpiWarp) * 32 + lane;
                const int mt = (tile / p.n_tiles) * BT;
                if (te < BT) reinterpret_cast<float*>(wring)[te] = (mt + te < p.M) ? p.rowmul[mt + te] : 1.0f;
            }
        }
    }

    __syncwarp();
    if (split) {
        // Sum the K slices of the cluster in rank order. Rank r owns a contiguous range of the
        // tile's token columns (a multiple of 4 wide). Once every rank has finished its slice
        // (barrier 1; their X rings are free), each rank pushes its fp32 partial of every range
        // into the owner's shared memory with remote stores, which do not wait for a reply;
        // after barrier 2 every owner adds the ranks' partials from its own shared memory,
        // scales them by the row factors and stores the bf16 result.
        // Receive buffer of an owner: [source rank][128 rows][P 16-byte chunks], P = its column
        // count / 4 made odd, so that 32 rows' chunks at one column fall in distinct banks.
        const int ks = p.ksplit;
        const int rank = static_cast<int>(cluster_ctarank());
        const int per_rank = ((BT + ks - 1) / ks + 3) / 4 * 4;
        const int chunks = per_rank / 4;
        const int P = chunks | 1;
        const uint32_t recv0 = smem_u32(smem);
        cluster_sync_all();   // barrier 1
        const bool epi = warp >= C::kFirstEpiWarp && warp < C::kFirstDqWarp;
        if (epi && !*abort_flag) {
            tc_fence_after();
            const int e = warp - C::kFirstEpiWarp;
            const int quarter = warp & 3;
            const int row = quarter * 32 + lane;
            const int col0 = (e >> 2) * C::kEpiCols;
            const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
            constexpr int kChunk = (C::kEpiCols >= 32) ? 32 : 16;
#pragma unroll
            for (int c0 = 0; c0 < C::kEpiCols; c0 += kChunk) {
                uint32_t v[32];
                if (kChunk == 32) {
                    tmem_ld32(lane_base + col0 + c0, v);
                } else {
                    tmem_ld16(lane_base + col0 + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < kChunk; j += 4) {
                    const int col = col0 + c0 + j;
                    const int owner = col / per_rank;
                    const int cl = (col - owner * per_rank) >> 2;
                    const uint32_t off = static_cast<uint32_t>(((rank * kBlockN + row) * P + cl) * 16);
                    if (dcheck(owner < ks && off + 16 <= static_cast<uint32_t>(C::kXStages * C::kXStageBytes), status))
                        st_shared_cluster_v4(map_shared_rank(recv0 + off, static_cast<uint32_t>(owner)),
                                             make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                         __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])));
                }
            }
        }
        cluster_sync_all();   // barrier 2: every push has landed
        if (epi && !*abort_flag) {
            const int e = warp - C::kFirstEpiWarp;
            const int quarter = warp & 3;
            const int epart = e >> 2;
            const int row = quarter * 32 + lane;
            const int tile = blockIdx.x;
            const int m0 = (tile / p.n_tiles) * BT;
            const int n = (tile % p.n_tiles) * p.rows + row;
            const int cb = rank * per_rank;
            const int cend = min(min(BT, cb + per_rank), p.M - m0);
            const float* fac = reinterpret_cast<const float*>(wring);
            const float4* recv = reinterpret_cast<const float4*>(smem);
            if (row < p.rows && n < p.N) {
                constexpr int kStep = 4 * C::kEpiParts;
                for (int c = cb + 4 * epart; c < cend; c += kStep) {
                    const int cl = (c - cb) >> 2;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int q = 0; q < ks; ++q) {
                        const float4 v = recv[(q * kBlockN + row) * P + cl];
                        acc.x += v.x;
                        acc.y += v.y;
                        acc.z += v.z;
                        acc.w += v.w;
                    }
                    const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int m = m0 + c + j;
                        if (m < p.M && dcheck(m >= 0 && n >= 0 && n < p.N && c + j < BT, status))
                            p.Y[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(a4[j] * fac[c + j]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // a pair's tensor memory is freed by both CTAs together, once neither uses it (and no
    // remote arrival or copy of one CTA targets the other after it has exited)
    if (PAIR) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<PAIR>(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// X conversion pass: bf16 [M][K] -> fp16 [M][K] with a power-of-two factor per row.
// ---------------------------------------------------------------------------------------------
// One CTA per row: finds the largest |x| of the row (from the bf16 bits), picks e so that the
// row's largest value scaled by 2^-e lies in [2^15, 2^16) -- inside fp16's range, with every value
// within 2^29 of it still an fp16 normal -- writes the row times 2^-e as fp16 (exact) and
// rowmul[row] = 2^e, which the GEMM epilogue multiplies back (exact). Rows that are all zero,
// or hold an infinity or NaN, keep e = 0 (non-finite values convert as they are).
__device__ __forceinline__ uint32_t absmax_bf16x8(const uint4& v, uint32_t m) {
    m = max(m, max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu));
    m = max(m, max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu));
    m = max(m, max(v.z & 0x7FFFu, (v.z >> 16) & 0x7FFFu));
    m = max(m, max(v.w & 0x7FFFu, (v.w >> 16) & 0x7FFFu));
    return m;
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float scale) {
    return pack_f16x2(__uint_as_float(w << 16) * scale, __uint_as_float(w & 0xFFFF0000u) * scale);
}

constexpr int kConvThreads = 256;

// One CTA per row of X. PER > 0: the row is held in registers (PER 16-byte chunks per thread,
// K <= 2048 * PER), so X is read from memory once; PER == 0: any K, the row is read twice.
template <int PER>
__global__ void __launch_bounds__(kConvThreads) convert_x_kernel(const uint4* __restrict__ X, int K8,
                                                                 uint4* __restrict__ Xh, float* __restrict__ rowmul) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int row = blockIdx.x;
    const uint4* src = X + static_cast<size_t>(row) * K8;
    uint4* dst = Xh + static_cast<size_t>(row) * K8;
    uint32_t mx = 0;
    uint4 v[PER > 0 ? PER : 1];
    if (PER > 0) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = threadIdx.x + j * kConvThreads;
            v[j] = i < K8 ? ldg_nc_v4(src + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < PER; ++j) mx = absmax_bf16x8(v[j], mx);
    } else {
        for (int i = threadIdx.x; i < K8; i += kConvThreads) mx = absmax_bf16x8(src[i], mx);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    __shared__ uint32_t warp_max[kConvThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = 0;
#pragma unroll
    for (int w = 0; w < kConvThreads / 32; ++w) mx = max(mx, warp_max[w]);
    const int E = static_cast<int>(mx >> 7);            // biased exponent of the largest |x|
    int e = (mx == 0 || E >= 255) ? 0 : E - 142;          // largest |x| * 2^-e in [2^15, 2^16)
    e = max(-100, min(112, e));
    const float scale = __int_as_float((127 - e) << 23);  // 2^-e
    auto cvt = [&](const uint4& a) {
        uint4 o;
        o.x = bf16x2_to_f16x2(a.x, scale);
        o.y = bf16x2_to_f16x2(a.y, scale);
        o.z = bf16x2_to_f16x2(a.z, scale);
        o.w = bf16x2_to_f16x2(a.w, scale);
        return o;
    };
    if (PER > 0) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = threadIdx.x + j * kConvThreads;
            if (i < K8) dst[i] = cvt(v[j]);
        }
    } else {
        for (int i = threadIdx.x; i < K8; i += kConvThreads) dst[i] = cvt(src[i]);
    }
    if (threadIdx.x == 0) rowmul[row] = __int_as_float((127 + e) << 23);   // 2^e
}

lowbit_status launch_convert_x(const GemmProblem& g, cudaStream_t stream) {
    const WorkspaceLayout ws = workspace_layout(g.M, g.K);
    cudaLaunchConfig_t ccfg = {};
    cudaLaunchAttribute cattr[1];
    cattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    cattr[0].val.programmaticStreamSerializationAllowed = 1;
    ccfg.gridDim = dim3(static_cast<unsigned>(g.M), 1, 1);
    ccfg.blockDim = dim3(kConvThreads, 1, 1);
    ccfg.stream = stream;
    ccfg.attrs = cattr;
    ccfg.numAttrs = 1;
    const int K8 = static_cast<int>(g.K / 8);
    if (take_injected_failure(kInjectLaunch)) return LOWBIT_ERR_CUDA;
    const uint4* x = static_cast<const uint4*>(g.X);
    uint4* xh = static_cast<uint4*>(g.workspace);
    float* rm = reinterpret_cast<float*>(static_cast<uint8_t*>(g.workspace) + ws.rowmul_offset);
    cudaError_t e;
    if (K8 <= kConvThreads) e = cudaLaunchKernelEx(&ccfg, convert_x_kernel<1>, x, K8, xh, rm);
    else if (K8 <= 2 * kConvThreads) e = cudaLaunchKernelEx(&ccfg, convert_x_kernel<2>, x, K8, xh, rm);
    else if (K8 <= 4 * kConvThreads) e = cudaLaunchKernelEx(&ccfg, convert_x_kernel<4>, x, K8, xh, rm);
    else if (K8 <= 8 * kConvThreads) e = cudaLaunchKernelEx(&ccfg, convert_x_kernel<8>, x, K8, xh, rm);
    else e = cudaLaunchKernelEx(&ccfg, convert_x_kernel<0>, x, K8, xh, rm);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// One CTA waits on a barrier that nothing arrives on, with the GEMM's bounded wait: the wait
// gives up after `limit` clocks and records the timeout in the device status word.
__global__ void bounded_wait_selftest_kernel(long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, &g_device_status, limit);
}

lowbit_status selftest_bounded_wait(long long limit_cycles, cudaStream_t stream) {
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_cycles);
    return cudaGetLastError() == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// One thread asks to store one element past a one-element array. The store happens only when
// the index is in range, so nothing is ever written out of bounds; in debug builds the index
// check in front of it records the failure in the status word, as the GEMM kernels' checks do.
__device__ unsigned g_selftest_cell[1];
__global__ void index_check_selftest_kernel(int index) {
    const bool ok = index >= 0 && index < 1;
    if (dcheck(ok, &g_device_status) && ok) g_selftest_cell[index] = 1u;
}

lowbit_status selftest_index_check(cudaStream_t stream) {
    if (!kDebugChecks) return LOWBIT_ERR_UNSUPPORTED;
    index_check_selftest_kernel<<<1, 1, 0, stream>>>(1);
    return cudaGetLastError() == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn();

// Tensor maps are a pure function of their arguments (address, geometry, box, swizzle), so
// encoded maps are kept in a small direct-mapped cache: a linear called again with the same
// buffers skips the driver's encode.
struct MapKey {
    uint64_t base;
    uint64_t dims[3];
    uint64_t strides[2];
    uint32_t box[3];
    int dtype, rank, swz;
    bool operator==(const MapKey& o) const {
        return base == o.base && dims[0] == o.dims[0] && dims[1] == o.dims[1] && dims[2] == o.dims[2] &&
               strides[0] == o.strides[0] && strides[1] == o.strides[1] && box[0] == o.box[0] &&
               box[1] == o.box[1] && box[2] == o.box[2] && dtype == o.dtype && rank == o.rank && swz == o.swz;
    }
};

bool encode_cached(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                   const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swz) {
    if (take_injected_failure(kInjectEncode)) return false;
    constexpr int kSlots = 1024;
    struct Slot {
        bool used;
        MapKey key;
        CUtensorMap map;
    };
    static Slot* slots = new Slot[kSlots]();
    static std::mutex mu;
    MapKey k = {};
    k.base = reinterpret_cast<uint64_t>(base);
    for (int i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
    k.dtype = static_cast<int>(dtype);
    k.rank = rank;
    k.swz = static_cast<int>(swz);
    uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
    for (int i = 0; i < 3; ++i) h ^= (k.dims[i] + 0x632BE59BD9B4E019ull * (k.box[i] + 1)) * (2 * i + 3);
    h ^= (k.strides[0] * 31 + k.strides[1]) ^ (static_cast<uint64_t>(k.dtype) << 40) ^
         (static_cast<uint64_t>(k.swz) << 48) ^ (static_cast<uint64_t>(rank) << 56);
    h ^= h >> 29;
    Slot& sl = slots[h % kSlots];
    {
        std::lock_guard<std::mutex> lock(mu);
        if (sl.used && sl.key == k) {
            *map = sl.map;
            return true;
        }
    }
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t d[3], st[2];
    cuuint32_t b[3], estr[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
    const CUresult r = fn(map, dtype, rank, const_cast<void*>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lock(mu);
    sl.used = true;
    sl.key = k;
    sl.map = *map;
    return true;
}

// The driver's tensor-map encoder, looked up once (a function-local static: initialised exactly
// once even when several host threads make their first call at the same time).
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        cudaGetLastError();
        return nullptr;
    }();
    return fn;
}

// X as a 3-D tensor (64 k, M rows, K/64 k-atoms) so that one box covers a whole 128-wide k-block
// of BT token rows in the 128-byte-swizzled layout [k half][row][64 k] the MMA reads.
bool make_map_x3d(CUtensorMap* map, const void* base, uint64_t M, uint64_t K, uint32_t box_rows) {
    const uint64_t dims[3] = {64, M, K / 64};
    const uint64_t strides[2] = {K * 2, 128};
    const uint32_t box[3] = {64, box_rows, 2};
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool make_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t (&dims)[3],
                 const uint64_t (&strides)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swz) {
    return encode_cached(map, dtype, 3, base, dims, strides, box, swz);
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
    (void)elem_bytes;
    const uint64_t dims[2] = {inner, outer};
    const uint64_t strides[1] = {row_bytes};
    const uint32_t box[2] = {box_inner, box_outer};
    return encode_cached(map, dtype, 2, base, dims, strides, box, swz);
}

int cluster_capacity(const void* kernel, int ks, int threads, int smem_bytes, bool along_x = false) {
    struct Entry {
        const void* fn;
        int dev, ks;
        bool x;
        int cap;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].fn == kernel && cache[i].dev == dev && cache[i].ks == ks && cache[i].x == along_x)
                return cache[i].cap;
    }
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = along_x ? ks : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = along_x ? 1 : ks;
    cfg.gridDim = along_x ? dim3(ks, 1, 1) : dim3(1, 1, ks);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / ks;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64) cache[used++] = Entry{kernel, dev, ks, along_x, n};
    return n;
}

// SM count of the current device (cached per device; 148 if the query fails).
int num_sms() {
    static std::atomic<int> sms[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int n = sms[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {

// rows: weight rows per CTA tile (0 = automatic: 128, or a CTA pair's 256 where that applies).
template <int BITS, int GS, int BT, bool PAIR = false>
lowbit_status launch(const GemmProblem& g, int rows, int ksplit_request, cudaStream_t stream, bool convert_x) {
    using C = Cfg<BITS, GS, BT, PAIR>;
    auto kernel = lowbit_gemm_kernel<BITS, GS, BT, PAIR>;
    const bool auto_rows = rows == 0;
    if (auto_rows || PAIR) rows = kBlockN;
    // the shared-memory opt-in is per device: one bit per device that has it
    static std::atomic<uint64_t> attr_devices{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(attr_devices.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return LOWBIT_ERR_CUDA;
        attr_devices.fetch_or(bit, std::memory_order_acq_rel);
    }
    CUtensorMap mx, mw, ms, mz;
    const int K = static_cast<int>(g.K), N = static_cast<int>(g.N), M = static_cast<int>(g.M);
    const CUtensorMapSwizzle wswz = C::kWRowBytes == 16   ? CU_TENSOR_MAP_SWIZZLE_NONE
                                    : C::kWRowBytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                          : CU_TENSOR_MAP_SWIZZLE_64B;
    const WorkspaceLayout ws = workspace_layout(g.M, g.K);
    void* xh = g.workspace;
    float* rowmul = reinterpret_cast<float*>(static_cast<uint8_t*>(g.workspace) + ws.rowmul_offset);
    bool ok = make_map_x3d(&mx, xh, M, K, C::kXRows);
    ok = ok && make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, g.Wp, uint64_t(K) * BITS / 32, N,
                           uint64_t(K) * BITS / 8, C::kWordsPerRow, rows, wswz);
    ok = ok && make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.scales, N, K / GS, uint64_t(N) * 2, kBlockN,
                           C::kGroupsPerStage, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (BITS == 4)
        ok = ok && make_map_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, g.zeros, N, K / GS, uint64_t(N) * 2,
                               kBlockN, C::kGroupsPerStage, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        mz = ms;
    // Y as (N, M) with a box of one tile, [BT tokens][rows]: the store of each CTA's last tile
    CUtensorMap my;
    ok = ok && make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.Y, N, M, uint64_t(N) * 2, rows, BT,
                           CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return LOWBIT_ERR_CUDA;

    KernelParams p;
    p.M = M;
    p.N = N;
    p.K = K;
    p.num_kb = (K + kBlockK - 1) / kBlockK;
    p.rows = rows;
    p.wtx_bytes = static_cast<uint32_t>(C::kWTxFixed + rows * C::kWRowBytes);
    p.m_tiles = (M + BT - 1) / BT;
    p.n_tiles = PAIR ? N / (2 * rows) : (N + rows - 1) / rows;
    p.num_tiles = p.m_tiles * p.n_tiles;
    p.Y = static_cast<__nv_bfloat16*>(g.Y);
    p.rowmul = rowmul;
    int ksplit = PAIR ? 1 : ksplit_request;
    if (ksplit < 0) {
        // Automatic: the largest split that leaves every rank at least 24 k-blocks (3072 of K)
        // and keeps all clusters resident at once (the split grid is not persistent, so a
        // second wave would double the time); cluster placement is limited by the GPC layout.
        ksplit = 1;
        const int slots = num_sms() * C::kCtasPerSm;
        for (int ks = 8; ks >= 2; --ks) {
            if (p.num_kb / ks < 24 || p.num_tiles * ks > slots) continue;
            if (p.num_tiles <= cluster_capacity(reinterpret_cast<const void*>(kernel), ks, C::kThreads,
                                                C::kSmemBytes)) {
                ksplit = ks;
                break;
            }
        }
    }
    if (ksplit < 1) ksplit = 1;
    if (ksplit > 8) ksplit = 8;
    // An unsplit grid of 256-token tiles over a multiple of 256 weight rows runs on CTA pairs.
    if constexpr (BT == 256 && !PAIR) {
        if (auto_rows && ksplit == 1 && N % (2 * kBlockN) == 0)
            return launch<BITS, GS, BT, true>(g, 0, 1, stream, convert_x);
    }
    if (ksplit > p.num_kb) ksplit = p.num_kb;
    int kbps = (p.num_kb + ksplit - 1) / ksplit;
    ksplit = (p.num_kb + kbps - 1) / kbps;     // every rank gets at least one k-block
    p.kb_per_split = ksplit > 1 ? kbps : p.num_kb;
    p.ksplit = ksplit;

    // X -> fp16 copy in the workspace, then the GEMM; both launched as programmatic dependents
    // of whatever precedes them on the stream.
    if (convert_x && launch_convert_x(g, stream) != LOWBIT_OK) return LOWBIT_ERR_CUDA;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (PAIR) {
        // persistent grid of CTA pairs, the two CTAs of a pair adjacent along x (clusters of 2)
        int pairs = cluster_capacity(reinterpret_cast<const void*>(kernel), 2, C::kThreads, C::kSmemBytes, true);
        if (pairs > num_sms() / 2) pairs = num_sms() / 2;
        if (pairs < 1) pairs = 1;
        cfg.gridDim = dim3(2 * (p.num_tiles < pairs ? p.num_tiles : pairs), 1, 1);
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 2;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    } else if (ksplit > 1) {
        cfg.gridDim = dim3(p.num_tiles, 1, ksplit);
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = ksplit;
        ++na;
    } else {
        const int slots = num_sms() * C::kCtasPerSm;
        cfg.gridDim = dim3(p.num_tiles < slots ? p.num_tiles : slots, 1, 1);
    }
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    if (take_injected_failure(kInjectLaunch)) return LOWBIT_ERR_CUDA;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, mx, mw, ms, mz, my, p);
    return e == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

// Token-tile width for M rows.
int pick_bt(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

int ctas_per_sm_for(int bt) { return bt <= 64 ? 2 : 1; }

template <int BITS, int GS>
lowbit_status launch_bits_gs(const GemmProblem& g, int bt, int rows, int ksplit, cudaStream_t s, bool cx) {
    switch (bt) {
        case 16: return launch<BITS, GS, 16>(g, rows, ksplit, s, cx);
        case 32: return launch<BITS, GS, 32>(g, rows, ksplit, s, cx);
        case 64: return launch<BITS, GS, 64>(g, rows, ksplit, s, cx);
        case 128: return launch<BITS, GS, 128>(g, rows, ksplit, s, cx);
        case 256:
            if (rows == 2 * kBlockN) return launch<BITS, GS, 256, true>(g, 0, 1, s, cx);
            return launch<BITS, GS, 256>(g, rows, ksplit, s, cx);
        default: return LOWBIT_ERR_UNSUPPORTED;
    }
}

}  // namespace

// Chooses the launch configuration (tile_tokens, tile_rows, ksplit), each 0 = automatic:
//   * one token tile and small M (weight streaming, HBM-bound): either "flat" tiles of
//     ceil(N / #SMs) rows (a multiple of 8) with the whole K per CTA and no reduction, or 128-row
//     tiles with K split over a cluster, whichever reads fewer X bytes per weight byte;
//   * few tiles otherwise: 128-row tiles with K split over a cluster;
//   * many tiles: 128-row tiles on a persistent grid.
bool uses_x_copy(const GemmProblem& g) { return !smallm_supported(g); }

lowbit_status gemm_launch(const GemmProblem& g, int force_bt, int force_rows, int force_split,
                          cudaStream_t stream, bool convert_x) {
    // tile_tokens == 1 selects the small-M warp-MMA kernel with X as the 16-row operand, 8 the
    // one with weights as the 16-row operand (M <= 8); automatic: 8 for M <= 8, else 1 up to 16
    if (force_bt == 1 || force_bt == 8) return smallm_launch(g, force_rows, force_split, force_bt == 8, stream);
    if (!force_bt && !force_rows && !force_split && smallm_supported(g))
        return smallm_launch(g, 0, 0, g.M <= 8, stream);
    const int bt = force_bt ? force_bt : pick_bt(g.M);
    const int sms = num_sms();
    const int64_t num_kb = (g.K + kBlockK - 1) / kBlockK;
    const int64_t m_tiles = (g.M + bt - 1) / bt;
    int rows = force_rows ? force_rows : kBlockN;
    int ksplit = force_split;
    if (!force_rows && !force_split) {
        const int64_t slots = static_cast<int64_t>(sms) * ctas_per_sm_for(bt);
        const int64_t tiles128 = m_tiles * ((g.N + kBlockN - 1) / kBlockN);
        int64_t flat_rows = ((g.N + sms - 1) / sms + 7) / 8 * 8;
        // X bytes read per packed-weight byte by one CTA: 2 * bt / (rows * bits / 8)
        const double x_per_w = (2.0 * bt) / (static_cast<double>(flat_rows) * g.bits / 8.0);
        ksplit = 1;
        if (bt <= 64 && m_tiles == 1 && flat_rows < kBlockN && x_per_w <= 1.25) {
            rows = static_cast<int>(flat_rows);
        } else if (bt <= 64 && m_tiles == 1) {
            if (tiles128 * 2 <= slots && num_kb >= 4) {
                int64_t s = sms / tiles128;   // small M: one CTA per SM
                if (s > 8) s = 8;
                if (s > num_kb / 2) s = num_kb / 2;
                ksplit = static_cast<int>(s < 1 ? 1 : s);
            }
        } else {
            ksplit = -1;   // chosen by the launch from the cluster capacity
        }
    }
    if (!ksplit) ksplit = 1;
    // 256 rows: one tile per CTA pair (256-token tiles, N a multiple of 256, no K split)
    const bool pair_rows = force_rows == 2 * kBlockN;
    if (pair_rows && (bt != 256 || g.N % (2 * kBlockN) != 0 || ksplit > 1)) return LOWBIT_ERR_UNSUPPORTED;
    if (!pair_rows && (rows < 8 || rows > kBlockN || rows % 8)) return LOWBIT_ERR_UNSUPPORTED;   // (ksplit -1: automatic)
    if (!force_rows && rows == kBlockN) rows = 0;   // automatic: the launch may use CTA pairs
    switch (g.bits * 1000 + g.group_size) {
        case 1064: return launch_bits_gs<1, 64>(g, bt, rows, ksplit, stream, convert_x);
        case 1128: return launch_bits_gs<1, 128>(g, bt, rows, ksplit, stream, convert_x);
        case 2064: return launch_bits_gs<2, 64>(g, bt, rows, ksplit, stream, convert_x);
        case 2128: return launch_bits_gs<2, 128>(g, bt, rows, ksplit, stream, convert_x);
        case 4064: return launch_bits_gs<4, 64>(g, bt, rows, ksplit, stream, convert_x);
        case 4128: return launch_bits_gs<4, 128>(g, bt, rows, ksplit, stream, convert_x);
        default: return LOWBIT_ERR_UNSUPPORTED;
    }
}

unsigned* device_status_address() {
    constexpr int kMaxDevices = 64;
    static std::atomic<unsigned*> ptrs[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned* p = ptrs[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(mu);
    p = ptrs[dev].load(std::memory_order_relaxed);
    if (!p) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) return nullptr;
        p = static_cast<unsigned*>(ptr);
        ptrs[dev].store(p, std::memory_order_release);
    }
    return p;
}

namespace {
lowbit_status status_of_word(unsigned v) {
    if (v & kDevErrTimeout) return LOWBIT_ERR_TIMEOUT;
    if (v & kDevErrCheck) return LOWBIT_ERR_DEVICE_CHECK;
    return LOWBIT_OK;
}
}  // namespace

lowbit_status read_device_status(int clear) {
    unsigned v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (clear && v) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return LOWBIT_ERR_CUDA;
    }
    return status_of_word(v);
}

// Stream-ordered read and clear: the copy of the word and the clearing store are queued on
// `stream`, so only the work queued there before them is waited for.
lowbit_status read_stream_status(cudaStream_t stream) {
    unsigned* word = device_status_address();
    if (!word) return LOWBIT_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaMemsetAsync(word, 0, sizeof(unsigned), stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return LOWBIT_ERR_CUDA;
    return status_of_word(v);
}

}  // namespace lowbit
