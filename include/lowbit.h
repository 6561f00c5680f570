/*
 * lowbit.h -- C ABI of liblowbit.so: weight-only low-bit GEMM for NVIDIA B200 (sm_100a).
 *
 *   Y[M][N] = X[M][K] * W^T,   W[N][K] decoded from packed low-bit codes and fp16 group scales.
 *
 * This is the matrix multiply behind the Q/K/V, output and MLP linears of the Bonsai Image
 * (FLUX.2-Klein-4B) transformer, whose weights are binary 1-bit with one FP16 scale per group
 * of 128 (bonsai-image-binary-4B-gemlite-1bit model card, "Binary Weight Representation:
 * 1-bit g128") or ternary 2-bit (mlx-vlm Bonsai article, model overview), and of the 4-bit
 * grouped text-encoder linears, group 64 (same article, component architecture).
 *
 * Formats (bits):
 *   1  binary   w = s * b,        b in {-1,+1}         code values -1 / +1
 *   2  ternary  w = s * t,        t in {-1, 0,+1}      code values -1 / 0 / +1
 *   4  uint4    w = (q - z) * s,  q in 0..15           code values 0..15, z = per-group zero
 * s and z are fp16, one per group of `group_size` consecutive K elements of one output row.
 *
 * Packed code layout (uint32 words, packed along K; produced by lowbit_pack):
 *   cpw = 32 / bits codes per word; row n of W owns words [n*K/cpw, (n+1)*K/cpw).
 *   Offset i of a word (0 .. cpw-1) occupies bits [pos, pos + bits) with
 *   pos = (i % 2) * 16 + (i / 2) * bits: offsets 2p and 2p + 1 ("pair p") fill the low and
 *   the high 16 bits, each half LSB-first. Which column an offset holds:
 *   - block order (2- and 4-bit rows, words taken in blocks of four, a block spanning
 *     4 * cpw columns: 32 for uint4, 64 for ternary): in word q (0..3) of block b, pair p
 *     holds columns 4*cpw*b + 8p + 2q (low half) and 4*cpw*b + 8p + 2q + 1 (high half);
 *   - plain order (every binary word, and the words after the last whole block of a 2- or
 *     4-bit row, i.e. when K is not a multiple of 4 * cpw): word j, offset i holds column
 *     cpw * j + i.
 *   Stored fields: binary +1 -> 1, -1 -> 0; ternary t -> t + 1 (3 is invalid); uint4 q -> q.
 *   (The pages pack codes along K into uint32 words -- Bonsai-Image-Demo PR #20, GemLite
 *   int2 layout note; image-studio backend.md, checkpoint layout -- but leave the order
 *   inside the words open. Pairs put two K-neighbours in the two 16-bit halves of one
 *   register, so one mask builds a bf16x2 / fp16x2 operand; block order makes word q of a
 *   block exactly the codes lane q of a warp-level m16n8k16 MMA needs from that block, so
 *   the small-M kernel loads one 32-bit word per lane per block.)
 *
 * Scale / zero layout: fp16, group-major [K/group_size][N]: s(n, k) = scales[(k/g)*N + n].
 * X: bf16 row-major [M][K]. Y: bf16 row-major [M][N].
 *
 * Arithmetic (M > 16): X is copied to fp16 in the caller's workspace (exactly: each row is first
 * scaled by a power of two that keeps it inside fp16's range, and the result is scaled back);
 * binary and ternary weights decode to exactly +-s or 0 in fp16; a uint4 weight (q - z) * s is
 * computed in fp32 (error below 2^-24 relative) and rounded once to fp16; products are summed in
 * fp32 on the tensor cores and Y is rounded to bf16 once. M <= 16: codes decode exactly without
 * their scale, X is used as stored (bf16), group sums are formed in fp32 and scaled there (see
 * lowbit_gemm_ex, tile_tokens = 1).
 *
 * Ownership: the caller owns every buffer (device memory unless stated), including the GEMM
 * workspace (see lowbit_gemm_workspace_size). The library allocates nothing; it holds a few
 * status words per device in static device memory.
 * Streams are CUDA stream handles (cudaStream_t) passed as void*; NULL = legacy stream.
 * Errors: argument / shape errors return before any launch and change nothing.
 */
#ifndef LOWBIT_H_
#define LOWBIT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lowbit_status {
    LOWBIT_OK = 0,
    LOWBIT_ERR_INVALID_ARG = 1,        /* NULL pointer, bad bits / group size, bad shape        */
    LOWBIT_ERR_ALIGNMENT = 2,          /* a pointer is not 16-byte aligned                      */
    LOWBIT_ERR_UNSUPPORTED = 3,        /* valid problem the GPU path does not take (see below)  */
    LOWBIT_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 (B200 class)             */
    LOWBIT_ERR_BAD_CODE = 5,           /* pack: a code outside its format; unpack: field 3       */
    LOWBIT_ERR_TIMEOUT = 6,            /* a bounded wait inside a kernel gave up (device status) */
    LOWBIT_ERR_CUDA = 7,               /* a CUDA runtime / driver call failed                    */
    LOWBIT_ERR_WORKSPACE = 8,          /* workspace NULL, misaligned or smaller than required    */
    LOWBIT_ERR_DEVICE_CHECK = 9        /* a device-side index check failed (debug builds only;   */
                                       /* see lowbit_debug_checks_enabled)                       */
} lowbit_status;

/* Human-readable name of a status. Never NULL. */
const char* lowbit_status_string(lowbit_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int lowbit_version(void);

/* Number of uint32 words of the packed codes of an [N][K] weight: N * K * bits / 32.
 * Returns 0 for invalid arguments (bits not 1/2/4, K not a multiple of 32/bits, N or K < 0). */
size_t lowbit_packed_words(int64_t N, int64_t K, int bits);

/* Pack int8 codes [N][K] (device, row-major) into `packed` [N][K*bits/32] uint32 (device),
 * in the layout above. Validates every code: on any invalid code returns
 * LOWBIT_ERR_BAD_CODE (the packed buffer is then unspecified). Synchronous: waits for the
 * work on `stream`. Requires K % (32/bits) == 0; codes 16-byte aligned when K > 0.
 * Calls are serialised inside the library (they share one device-side error counter). */
lowbit_status lowbit_pack(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed,
                          void* stream);

/* Inverse of lowbit_pack: packed [N][K*bits/32] -> int8 codes [N][K] (device). Returns
 * LOWBIT_ERR_BAD_CODE if a ternary field holds 3 (written as 0). Synchronous, serialised. */
lowbit_status lowbit_unpack(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes,
                            void* stream);

/* Bytes of device workspace lowbit_gemm needs for an X of [M][K]: the fp16 copy of X
 * (M*K*2 bytes, rounded up to 256) plus one float per row (rounded up to 256). 0 if M or K < 0. */
size_t lowbit_gemm_workspace_size(int64_t M, int64_t K);

/* Y = X * W^T on `stream` (asynchronous; never synchronises). For M > 16 two kernels run in
 * order on the stream: the X -> fp16 conversion into `workspace`, then the GEMM; for M <= 16 one
 * kernel reads X directly. Kernels are programmatic dependents of the work enqueued before
 * them: for M <= 16 the GEMM starts streaming Wp, scales and zeros before that work has
 * finished (X is read only after it), so Wp, scales and zeros must not be written by the
 * kernel enqueued immediately before the call (lowbit_pack returns only after its kernel has
 * completed, so packing right before is fine).
 *   X          [M][K]            bf16, device, 16-byte aligned
 *   Wp         [N][K*bits/32]    uint32 packed codes, device, 16-byte aligned
 *   scales     [K/group_size][N] fp16, device, 16-byte aligned
 *   zeros      [K/group_size][N] fp16 for bits == 4, NULL otherwise
 *   Y          [M][N]            bf16, device, 16-byte aligned; must not overlap the inputs
 *   workspace  device, 256-byte aligned, >= lowbit_gemm_workspace_size(M, K) bytes; owned by
 *              the caller, overwritten by the call, and must not be used by concurrently
 *              running work until the call's kernels have finished
 * GPU path preconditions (else LOWBIT_ERR_UNSUPPORTED): group_size 64 or 128,
 * K % group_size == 0, K % 128 == 0 when bits == 1, N % 8 == 0, M, N, K < 2^31.
 * M == 0 or N == 0 is a no-op. Kernel-side bounded waits that give up set the device
 * status word (see lowbit_device_status) instead of trapping. */
lowbit_status lowbit_gemm(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                          const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                          void* workspace, size_t workspace_bytes, void* stream);

/* lowbit_gemm with the kernel configuration fixed instead of chosen from the shape, for
 * tuning and tests (each 0 = automatic):
 *   tile_tokens  tokens per CTA tile of the tensor-memory kernel: 16, 32, 64, 128 or 256; or 1
 *                for the small-M kernel on warp-level MMAs (M <= 16 only; chosen automatically
 *                for M <= 16; it reads X directly and leaves the workspace untouched). That
 *                kernel sums unscaled codes times X in fp32 per group before applying the
 *                scale, so its results are exact only for |x| below about 2^114; the
 *                tensor-memory kernel (M > 16, or tile_tokens >= 16) covers the full bf16 range
 *   tile_rows    weight rows per CTA tile: a multiple of 8 up to 128 (128 unless the shape is
 *                small; fewer rows give more CTAs, each streaming the whole K), or 256: one
 *                256 x 256 tile per pair of CTAs on paired tensor-core MMAs (tile_tokens 0 or
 *                256, 256-token tiles, N % 256 == 0, no K split; chosen automatically for
 *                unsplit 256-token tiles when N % 256 == 0)
 *   ksplit       number of K slices summed across a thread-block cluster, 1..8 (1 = no split;
 *                the small-M kernel cuts K into slices of whole 512-wide steps, so a request
 *                may be served with fewer slices)
 * Other arguments and all checks are those of lowbit_gemm; values outside these sets return
 * LOWBIT_ERR_UNSUPPORTED. */
lowbit_status lowbit_gemm_ex(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                             const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                             void* workspace, size_t workspace_bytes, int tile_tokens, int tile_rows,
                             int ksplit, void* stream);

/* One linear of a chain, with the meaning and layout of lowbit_gemm's arguments. */
typedef struct lowbit_gemm_desc {
    int64_t M, N, K;
    int bits, group_size;
    const void* X;
    const uint32_t* Wp;
    const void* scales;
    const void* zeros;
    void* Y;
} lowbit_gemm_desc;

/* Run `count` GEMMs (host array of descriptors) in order on `stream`, as if lowbit_gemm were
 * called for each in turn with the same workspace: a descriptor may read an earlier one's Y.
 * This is the unit of one denoise step of the transformer: its 25 MMDiT blocks, 5 double-stream
 * and 20 single-stream (bonsai-image-binary-4B-gemlite-1bit model card, model overview /
 * specifications), each run their Q/K/V, output and MLP linears in order.
 * The workspace must hold the largest lowbit_gemm_workspace_size(M, K) of the descriptors.
 * All descriptors are validated first; on any invalid one nothing is launched and its error
 * is returned. Consecutive launches overlap their prologues with the previous kernel's tail
 * (programmatic dependent launch); results are the same as separate calls. A linear with more
 * than 16 tokens that reads the same X as the previous such linear (same pointer, M and K),
 * with no output written since then overlapping that X, reuses the fp16 copy of X already in
 * the workspace instead of converting it again (separate Q, K and V projections of one input
 * convert it once). A failure while launching returns at once; the linears before it have
 * been queued and will run. */
lowbit_status lowbit_gemm_batch(const lowbit_gemm_desc* descs, int count, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Read the current device's sticky status word, written by kernels whose bounded waits gave
 * up (LOWBIT_ERR_TIMEOUT) or, in debug builds, whose index checks failed
 * (LOWBIT_ERR_DEVICE_CHECK), and clear it when `clear` != 0. Synchronises the whole device. */
lowbit_status lowbit_device_status(int clear);

/* Debug: the same status word read in stream order -- the read and the clearing of the word are
 * queued on `stream` and only that stream is waited for, so other streams keep running. The
 * word is per device: it also reports kernels of other streams that finished before the read.
 * Returns LOWBIT_OK, LOWBIT_ERR_TIMEOUT or LOWBIT_ERR_DEVICE_CHECK (then clears the word), or
 * LOWBIT_ERR_CUDA if the copy could not be made. */
lowbit_status lowbit_last_device_status(void* stream);

/* Size of the static device scratch used by lowbit_gemm_noalloc: 32 MiB. */
#define LOWBIT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* lowbit_gemm for callers that cannot allocate device memory where they run a linear -- for
 * example a plug-in inside a host engine that owns all device memory and forbids allocations
 * after start-up, or a latency-critical loop in which cudaMalloc's device synchronisation is not
 * acceptable. It takes the same arguments as lowbit_gemm minus the workspace: its scratch (the
 * fp16 copy of X and the row factors) lives in a fixed array of static device memory of
 * LOWBIT_NOALLOC_SCRATCH_BYTES, which a device holds from the first use of this entry point
 * on it (or from library load, if CUDA modules are loaded eagerly) until the process exits.
 *  - Problems with lowbit_gemm_workspace_size(M, K) > LOWBIT_NOALLOC_SCRATCH_BYTES (for
 *    example M * K > about 16.7 million at small M) are rejected with LOWBIT_ERR_WORKSPACE
 *    before any launch; other argument errors are those of lowbit_gemm.
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *    with that device current; make that first call before any stream capture.
 *  - Nothing in the scratch has to start at zero: each call overwrites the part it reads.
 *  - All calls on a device share the one array, so calls whose kernels overlap on the GPU
 *    (different streams or host threads without ordering) race; order them on one stream, or
 *    use lowbit_gemm with separate workspaces.
 *  - Allocates nothing: no cudaMalloc / cudaFree and no allocating library routine.
 * The pages have no counterpart to this entry point; it is a deployment variant of lowbit_gemm. */
lowbit_status lowbit_gemm_noalloc(int64_t M, int64_t N, int64_t K, int bits, int group_size, const void* X,
                                  const uint32_t* Wp, const void* scales, const void* zeros, void* Y,
                                  void* stream);

/* Diagnostic for the kernels' failure detection: launches one CTA that waits on a
 * shared-memory barrier nothing ever completes, using the same bounded wait as the GEMM kernel
 * but giving up after `limit_cycles` SM clocks (> 0). The wait then records LOWBIT_ERR_TIMEOUT in
 * the device status word and the kernel returns normally, so the context stays usable; read it
 * with lowbit_device_status. Asynchronous. */
lowbit_status lowbit_selftest_bounded_wait(long long limit_cycles, void* stream);

/* Failure injection, for tests of the error paths: `what` = 1 makes the next tensor-map encode
 * fail, 2 the next kernel launch (either of the GEMM's two launches counts), 3 both; 0 cancels
 * what is still pending. Each injected failure fires once, in any thread of the process, at the
 * point where the real failure would be detected: the call then returns LOWBIT_ERR_CUDA before
 * launching the affected kernel, exactly as it does when the driver reports the failure. No
 * kernel is launched differently and no GPU fault is involved. Returns LOWBIT_ERR_INVALID_ARG
 * for other values. The paper has no counterpart; this is test support. */
lowbit_status lowbit_test_fail_next(int what);

/* 1 if this library was built with device-side index checks (LOWBIT_DEBUG_CHECKS, shipped as
 * liblowbit_debug.so), else 0. In such a build every global store of Y, every load of a row
 * factor and every tensor-memory store of decoded weights first checks its index against the
 * problem's bounds; a failed check records LOWBIT_ERR_DEVICE_CHECK in the device status word
 * and skips the access instead of trapping, so the context stays usable. */
int lowbit_debug_checks_enabled(void);

/* Diagnostic for the debug build's index checks: launches one thread whose store index is one
 * past its one-element target. The store is made only when the index is in range, so nothing is
 * written out of bounds in any build; a debug build also records LOWBIT_ERR_DEVICE_CHECK in the
 * device status word. Returns LOWBIT_ERR_UNSUPPORTED (launching nothing) in release builds.
 * Asynchronous. */
lowbit_status lowbit_selftest_index_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOWBIT_H_ */
