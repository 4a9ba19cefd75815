/*
 * dg.h — C ABI of the B200 (sm_100a) FP8 block-scaled NT GEMM library.
 *
 * The operation is D = C + A·Bᵀ in NT layout: A is [M,K] and B is [N,K], both K-contiguous
 * e4m3 (OCP E4M3FN). A carries one fp32 scale per 1×128 K-slice of each row, B one fp32
 * scale per 128×128 block, and C and D are bf16. Sources: the DeepGEMM write-ups —
 * likun.im/craft/deepgemm §一 (the D = C + A·Bᵀ NT convention; dense, M-grouped contiguous
 * and masked GEMMs) and §二 (the register_apis list: fp8_gemm_nt, m_grouped_*_contiguous with
 * grouped_layout, m_grouped_*_masked with masked_m / expected_m, transform_sf);
 * aitangshan.cn/news/1491278 技术原理 §4 (block-wise scaling, one scale per block, applied
 * after the multiplication); likun.im §五 (the LHS scales need a TMA-aligned, transposed
 * layout).
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library neither frees
 *    nor keeps them after the call returns; the memory must stay valid until the work queued
 *    on `stream` has finished.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every
 *    call is asynchronous with respect to the host and never synchronises the device.
 *  - Kb = K/128 and Nb = ceil(N/128). "pad4(x)" is x rounded up to a multiple of 4, so that
 *    every row of an MN-major fp32 scale array starts on a 16-byte boundary
 *    (dg_sf_ld(x) returns it).
 *  - Layout of the A scales ("sfa"): fp32 [Kb][pad4(M)], MN-major: sfa[kb*pad4(M) + m]
 *    scales A[m, kb*128 .. kb*128+127]. Entries m >= M are padding and never read.
 *  - Layout of the B scales ("sfb"): fp32 [G][Nb][Kb]: sfb[(g*Nb + nb)*Kb + kb] scales
 *    B[g, nb*128 .. nb*128+127, kb*128 .. kb*128+127] (G = 1 for the dense GEMM).
 *  - Argument errors are reported synchronously, before anything is queued:
 *      DG_ERR_INVALID_ARG (a size out of range, a NULL where a tensor is required),
 *      DG_ERR_ALIGNMENT (a base pointer not 16-byte aligned),
 *      DG_ERR_UNSUPPORTED (no device of compute capability 10.0 current).
 *    A failed launch returns DG_ERR_CUDA. Faults that only the device can see (an expert id
 *    in grouped_layout >= G, masked_m[g] > M_max, a pipeline wait that ran out of time) set a
 *    per-device error word that dg_get_device_error() returns. Nothing aborts the process
 *    and nothing throws across this ABI.
 *  - Preconditions of the GEMMs: K % 128 == 0, N % 8 == 0 (16-byte D rows), M >= 0.
 *    The results of the GEMMs satisfy |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref) against the
 *    exact fp64 value of the same block-scaled operands. Every GEMM is deterministic: the
 *    same inputs give the same bits, call after call.
 *  - Environment variables, each read once per process:
 *      DG_WAIT_TIMEOUT_MS  the limit of every pipeline wait inside a kernel (default 4000);
 *                          on expiry the kernel stops and DG_ERR_TIMEOUT is reported.
 *    For experiments and tests only (they change which kernel runs, never the result beyond
 *    the stated bound): DG_FORCE_PAIR=0|1 (CTA pairs for the tile GEMM), DG_FORCE_BN=128|256,
 *    DG_FORCE_SWAP=0|1 (few-row kernels off for M <= 128, or on for the masked layout),
 *    DG_FEW_ROW=streamk|cluster, DG_SPLITK_S=1|2|3|4|6|8|16 (cluster size). Debug only:
 *    DG_TEST_SKIP_RELEASE=1|2|3 makes one kernel withhold barrier arrives or partial flags,
 *    so that a wait runs out of time (failure tests).
 */
#ifndef DG_H
#define DG_H

#include <stdint.h>

#if defined(__GNUC__)
#define DG_API __attribute__((visibility("default")))
#else
#define DG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dg_status {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1,
    DG_ERR_ALIGNMENT = 2,
    DG_ERR_UNSUPPORTED = 3,
    DG_ERR_CUDA = 4,
    DG_ERR_TIMEOUT = 5,
    DG_ERR_DEVICE = 6
} dg_status;

/* Dense FP8 NT GEMM, D = C + A·Bᵀ (likun.im/craft/deepgemm §二, fp8_gemm_nt).
 *   a   e4m3 [M,K] row-major;          sfa fp32 [Kb][pad4(M)]
 *   b   e4m3 [N,K] row-major;          sfb fp32 [Nb][Kb]
 *   c   bf16 [M,N] row-major or NULL (then C = 0); may alias d
 *   d   bf16 [M,N] row-major, written in full.
 * M may be 0 (nothing is queued). For M <= 128 the K blocks are split over several SMs:
 *   - with few 128-column tiles (at most 64) and K <= 8192, over a thread-block cluster per
 *     tile, whose partial sums meet in distributed shared memory (no scratch at all);
 *   - otherwise over every SM (stream-K), whose partial sums meet in a library-owned
 *     workspace of the (device, stream) pair, allocated (cudaMalloc, sm_count x 64 KB) by
 *     the pair's first such call and kept until the process ends; a first call made under
 *     CUDA-graph capture cannot allocate and computes with the tile kernel instead.
 * Every choice gives the same result within the stated bound, and each is deterministic. */
DG_API dg_status dg_fp8_gemm_nt(const void *a, const float *sfa, const void *b, const float *sfb,
                         const void *c, void *d, int M, int N, int K, void *stream);

/* dg_fp8_gemm_nt's stream-K path for M <= 128 without any allocation, for callers that must
 * not call cudaMalloc (an allocator-owning runtime, a pre-planned memory arena, a decode loop
 * that must not add allocations). Same arguments, and the same result bit for bit as
 * dg_fp8_gemm_nt whenever that call takes the stream-K kernel (the same kernel and the same
 * split of the work), but the kernel's scratch (the fp32 partial sums, their flags and a launch
 * epoch) is a fixed static __device__ array of the library, 16 MB + 1 KB, instead of a
 * per-stream workspace; every GPU that loads the library holds it until the process exits.
 * The first call of any entry point on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before any stream
 * capture. The array is shared by every call on a device and keeps what the last call left:
 * calls that overlap on the GPU (on different streams, or replays of captured graphs that run
 * at the same time) race on it and must not be made. Flags left by a launch that stopped early
 * (after DG_ERR_TIMEOUT) are never taken for a later launch's: each launch waits for its own
 * ticket. The pages have no counterpart of this entry point.
 * Errors: those of dg_fp8_gemm_nt, plus DG_ERR_UNSUPPORTED (nothing queued) when M > 128 or
 * when the device has more than 256 SMs (the array's capacity). */
DG_API dg_status dg_fp8_gemm_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb,
                                        const void *c, void *d, int M, int N, int K, void *stream);

/* M-grouped "contiguous" FP8 NT GEMM for MoE prefill (likun.im §二,
 * m_grouped_*_gemm_nt_contiguous; zwt0204.github.io "DeepGEMM deep dive", the grouped-layout
 * constraint). The rows of A are the tokens of all G experts stacked, each expert's block
 * padded to a multiple of 128 rows.
 *   a   e4m3 [M_sum,K];                sfa fp32 [Kb][M_sum]   (M_sum % 128 == 0)
 *   b   e4m3 [G,N,K];                  sfb fp32 [G][Nb][Kb]
 *   grouped_layout  int32 [M_sum] on the device: the expert id of each row, -1 for a
 *       padding row. Every aligned 128-row block belongs to one expert; the block's expert is
 *       read from its first row. A block whose first row is -1 is skipped.
 *   c   bf16 [M_sum,N] or NULL;        d bf16 [M_sum,N].
 * D rows of padding rows have no defined value (they may be written). An id >= G sets the
 * device error word and its block is skipped. */
DG_API dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b,
                                              const float *sfb, const void *c, void *d,
                                              const int32_t *grouped_layout, int M_sum, int N,
                                              int K, int G, void *stream);

/* M-grouped "masked" FP8 NT GEMM for MoE decode (likun.im §二, m_grouped_*_gemm_nt_masked;
 * §四: it consumes the low-latency dispatch output). Expert g owns rows [0, masked_m[g]) of
 * its [M_max,K] slice of A.
 *   a   e4m3 [G,M_max,K];              sfa fp32 [G][Kb][pad4(M_max)]
 *   b   e4m3 [G,N,K];                  sfb fp32 [G][Nb][Kb]
 *   masked_m  int32 [G] on the device, read by the kernel (values > M_max are clamped to
 *       M_max and set the device error word; negative values count as 0).
 *   expected_m  host-side hint of the typical masked_m, used only to choose tile shapes.
 *   c   bf16 [G,M_max,N] or NULL;      d bf16 [G,M_max,N].
 * Rows r >= masked_m[g] of D are never written and their A rows never reach D. */
DG_API dg_status dg_m_grouped_fp8_gemm_nt_masked(const void *a, const float *sfa, const void *b,
                                          const float *sfb, const void *c, void *d,
                                          const int32_t *masked_m, int expected_m, int G,
                                          int M_max, int N, int K, void *stream);

/* Scale-layout transform (likun.im §二 transform_sf / get_mn_major_tma_aligned_tensor; §五:
 * LHS scales in a TMA-aligned transposed layout).
 *   sf_kmajor  fp32 [batch][MN][Kb] (one row of Kb scales per token)
 *   sf_mnmajor fp32 [batch][Kb][pad4(MN)]; the pad4 tail of every row is written with 0.
 * The two buffers must not overlap. */
DG_API dg_status dg_transform_sf(const float *sf_kmajor, float *sf_mnmajor, int batch, int MN, int Kb,
                          void *stream);

/* Per-token FP8 cast of activations (block-wise scaling, aitangshan.cn 技术原理 §4, at
 * 1×128 granularity). For every row m and K-slice kb: amax = max|x|, s = amax/448 (s = 1 when
 * amax = 0), q = e4m3(x/s) rounded to nearest-even and saturated to ±448.
 *   x   bf16 [batch,M,K];  q e4m3 [batch,M,K];  sfa fp32 [batch][Kb][pad4(M)] (padding
 *   entries are not written). K % 128 == 0. */
DG_API dg_status dg_cast_fp8_per_token(const void *x, void *q, float *sfa, int batch, int M, int K,
                                void *stream);

/* Per-block FP8 cast of weights, 128×128 blocks (same rule; a partial last block of rows
 * uses its valid rows only).
 *   x   bf16 [batch,N,K];  q e4m3 [batch,N,K];  sfb fp32 [batch][Nb][Kb]. K % 128 == 0. */
DG_API dg_status dg_cast_fp8_per_block(const void *x, void *q, float *sfb, int batch, int N, int K,
                                void *stream);

/* pad4(mn): the leading dimension of an MN-major scale array. */
DG_API int dg_sf_ld(int mn);

/* Waits for `stream`, then returns and clears the current device's error word
 * (DG_OK, DG_ERR_TIMEOUT or DG_ERR_DEVICE). */
DG_API dg_status dg_get_device_error(void *stream);

/* Static, human-readable name of a status code. */
DG_API const char *dg_status_string(dg_status status);

/* Name of the GEMM kernel that the calling thread's last GEMM call launched ("" before the
 * first): "gemm_kernel", "gemm_kernel (CTA pairs)", "gemm_swap_kernel (stream-K)" or
 * "gemm_splitk_kernel (cluster split-K)". For benchmarks and profiles; static storage. */
DG_API const char *dg_last_kernel(void);

/* Bytes of device memory the library has allocated with cudaMalloc so far, over all devices
 * (the few-row stream-K workspaces); the static arrays of the module are not counted. */
DG_API long long dg_allocated_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
