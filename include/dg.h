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
 *    DG_FEW_ROW=streamk|cluster, DG_SPLITK_S=1|2|3|4|6|8|16 (cluster size), DG_ONE_ISSUER=1
 *    (one MMA-issuing thread per CTA instead of two), DG_TAIL_SPLIT=0|2..64 (the dense tile
 *    GEMM's last-wave split off, or S pieces per last-wave tile). Debug only:
 *    DG_TEST_SKIP_RELEASE=1|2|3|4 makes one kernel withhold barrier arrives or partial flags,
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
 *     workspace of the (device, stream) pair, allocated (cudaMalloc, sm_count x 128 KB plus
 *     the flags) by the pair's first call that wants it and kept until the process ends; a
 *     first call made under CUDA-graph capture cannot allocate and computes with the tile
 *     kernel instead.
 * For M > 128 (the persistent tile kernel), when the tiles do not fill a whole number of
 * waves of resident CTAs, the last wave's tiles are cut along K into pieces run at once on
 * otherwise idle SMs, whose partial sums meet in the same workspace (in a fixed order); without
 * a workspace (a first call under graph capture) the last wave runs whole.
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

/* Dense FP8 NT GEMM with UE8M0 (power-of-two) scales, applied by the tensor core's
 * block-scaled MMA (likun.im §五: SM100 wants packed UE8M0 scales, four per 32-bit word; §二:
 * disable_ue8m0_cast). D = C + A·Bᵀ with the block scaling of dg_fp8_gemm_nt, every scale
 * being 2^(byte - 127):
 *   a   e4m3 [M,K];   sfa uint32 [ceil(Kb/4)][pad4(M)]: byte kb%4 of word (kb/4, m) scales
 *                     A[m, kb*128 .. kb*128+127]   (dg_cast_fp8_per_token_ue8m0 writes it)
 *   b   e4m3 [N,K];   sfb uint32 [Nb][ceil(Kb/4)]: byte kb%4 of word (nb, kb/4) scales the
 *                     128x128 block (nb, kb) of B   (dg_cast_fp8_per_block_ue8m0 writes it)
 *   c   bf16 [M,N] or NULL (may alias d);   d  bf16 [M,N].
 * Since every sfa·sfb is a power of two the hardware applies it exactly and accumulates all K
 * blocks in TMEM (fp32). Extra precondition: N % 16 == 0. Errors as for dg_fp8_gemm_nt. */
DG_API dg_status dg_fp8_gemm_nt_ue8m0(const void *a, const uint32_t *sfa, const void *b, const uint32_t *sfb,
                                      const void *c, void *d, int M, int N, int K, void *stream);

/* The dense GEMM in the other three storage layouts the pages name (likun.im §一,
 * "fp8_fp4_gemm_{nt,nn,tn,tt}"; §二, "同类: _nn / _tn / _tt"). The first letter is A's
 * storage, the second B's: A "n" = [M,K] (K contiguous), A "t" = [K,M] (M contiguous);
 * B "t" = [N,K] (K contiguous), B "n" = [K,N] (N contiguous). The product is the NT one,
 * D[m,n] = C[m,n] + sum_k A_log[m,k]·B_log[n,k], with the same scales:
 *   sfa fp32 [Kb][pad4(M)] (one per row m and 128-wide K slice), sfb fp32 [Nb][Kb] (one per
 *   128x128 block of B_log), c/d bf16 [M,N] row-major as for dg_fp8_gemm_nt.
 *   nn: a [M,K], b [K,N];   tn: a [K,M], b [K,N];   tt: a [K,M], b [N,K].
 * An MN-major operand reaches the tensor core through MN-major shared-memory descriptors, with
 * no transpose pass. Extra precondition: M % 16 == 0 when A is MN-major and N % 16 == 0 when B
 * is (16-byte rows for the tensor-map loads), else DG_ERR_INVALID_ARG. Every M takes the tile
 * kernel (no few-row split). Errors as for dg_fp8_gemm_nt. */
DG_API dg_status dg_fp8_gemm_nn(const void *a, const float *sfa, const void *b, const float *sfb,
                                const void *c, void *d, int M, int N, int K, void *stream);
DG_API dg_status dg_fp8_gemm_tn(const void *a, const float *sfa, const void *b, const float *sfb,
                                const void *c, void *d, int M, int N, int K, void *stream);
DG_API dg_status dg_fp8_gemm_tt(const void *a, const float *sfa, const void *b, const float *sfb,
                                const void *c, void *d, int M, int N, int K, void *stream);

/* K-grouped FP8 GEMM for the MoE weight gradient (likun.im §一, "沿 K 轴分组的
 * k_grouped_fp8_gemm_tn（MoE 反向）"; §二, k_grouped_fp8_gemm_tn_contiguous with ks_cpu and
 * recipe (1,1,128)). The K dimension (tokens) of both operands is cut into G consecutive groups
 * of ks[g] tokens; group g gives D[g] = C[g] + A_gᵀ·B_g:
 *   a   e4m3 [sum_K, M] (token-major, M contiguous: the "T" operand)
 *   sfa fp32 [sum_K/128][pad4(M)]: one scale per channel m per 128 tokens
 *   b   e4m3 [sum_K, N] (token-major, N contiguous: the "N" operand)
 *   sfb fp32 [sum_K/128][pad4(N)]: one scale per channel n per 128 tokens
 *   c   fp32 [G, M, N] or NULL (C = 0); may alias d.   d  fp32 [G, M, N], written in full.
 *   ks         host array [G] of the group sizes, each a multiple of 128 (0 allowed: D[g] = C[g])
 *   ks_device  the same G values in device memory (int32), read by the kernel.
 * D[g,m,n] = C[g,m,n] + sum_{kb in g} sfa[kb][m]·sfb[kb][n]·sum_{k in kb} A[k,m]·B[k,n].
 * Preconditions: 1 <= G <= 511, M % 16 == 0, N % 16 == 0, 16-byte aligned pointers. A device
 * value that is not a multiple of 128 or reaches past the host's sum sets the device error word
 * (DG_ERR_DEVICE) and its group is computed as empty. */
DG_API dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void *a, const float *sfa, const void *b,
                                                     const float *sfb, const float *c, float *d,
                                                     const int *ks, const int32_t *ks_device, int G,
                                                     int M, int N, void *stream);

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
 *   expected_m  host-side hint of the typical masked_m, used only to choose tile shapes:
 *       128-row tiles when expected_m <= 128, 256-row CTA-pair tiles above (0 = use M_max).
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

/* The per-token cast written straight into the M-grouped contiguous layout: the MoE dispatch
 * in front of dg_m_grouped_fp8_gemm_nt_contiguous (likun.im §二, m_grouped_*_contiguous with
 * grouped_layout; the pages' "fused cast + grouped GEMM"). Token t of x is quantised as by
 * dg_cast_fp8_per_token and written to row dst_rows[t] of q and sfa, in one pass, and the
 * GEMM that follows on the stream overlaps its prologue with this kernel (programmatic
 * dependent launch, as every kernel of the library).
 *   x         bf16 [T,K] (tokens in any order)
 *   dst_rows  int32 [T] on the device: the token's row in the contiguous layout, -1 to drop it;
 *             no two tokens may share a row. A row >= M_sum sets the device error word
 *             (DG_ERR_DEVICE) and the token is dropped.
 *   q         e4m3 [M_sum,K];  sfa fp32 [Kb][pad4(M_sum)] (the GEMM's layouts). Rows no token
 *             maps to (the padding of each expert's block) are not written.
 * K % 128 == 0. */
DG_API dg_status dg_cast_fp8_per_token_scatter(const void *x, const int32_t *dst_rows, void *q, float *sfa, int T,
                                               int M_sum, int K, void *stream);

/* Per-token and per-block FP8 casts with UE8M0 scales (likun.im §五: on SM100 the scales are
 * packed UE8M0, four per 32-bit word; §二: disable_ue8m0_cast). The scale of a block is the
 * smallest power of two s = 2^e >= amax/448 (the fp32 quotient), e clamped to [-127, 127]
 * (s = 1 when amax = 0), kept as the byte e + 127; q = e4m3(x/s) as for the fp32 casts (the
 * division by a power of two is exact). Scales are packed four K blocks per uint32 word, K
 * block kb in bits 8·(kb%4) .. 8·(kb%4)+7; bytes of K blocks >= Kb hold 127.
 *   per token: x bf16 [batch,M,K]; q e4m3 [batch,M,K];
 *              sfa uint32 [batch][ceil(Kb/4)][pad4(M)] (MN-major; padding entries m >= M
 *              are not written)
 *   per block: x bf16 [batch,N,K]; q e4m3 [batch,N,K]; sfb uint32 [batch][Nb][ceil(Kb/4)]
 * K % 128 == 0. */
DG_API dg_status dg_cast_fp8_per_token_ue8m0(const void *x, void *q, uint32_t *sfa, int batch, int M, int K,
                                             void *stream);
DG_API dg_status dg_cast_fp8_per_block_ue8m0(const void *x, void *q, uint32_t *sfb, int batch, int N, int K,
                                             void *stream);

/* Per-channel FP8 cast along the token dimension, the recipe (1,1,128) of the K-grouped GEMM's
 * operands (likun.im §二, k_grouped_fp8_gemm_tn_contiguous): for every 128-token block tb and
 * channel c, amax = max_t |x[t,c]| over the block's tokens, s = amax/448 (s = 1 when amax = 0),
 * q[t,c] = e4m3(x[t,c]/s), nearest-even, saturated to ±448 (the per-token cast's rule).
 *   x   bf16 [T,C] token-major;  q e4m3 [T,C];  sf fp32 [T/128][pad4(C)] (padding entries are
 *   not written). T % 128 == 0, C % 8 == 0, else DG_ERR_INVALID_ARG. */
DG_API dg_status dg_cast_fp8_per_channel(const void *x, void *q, float *sf, int T, int C, void *stream);

/* pad4(mn): the leading dimension of an MN-major scale array. */
DG_API int dg_sf_ld(int mn);

/* Waits for `stream`, then returns and clears the current device's error word
 * (DG_OK, DG_ERR_TIMEOUT or DG_ERR_DEVICE). */
DG_API dg_status dg_get_device_error(void *stream);

/* Static, human-readable name of a status code. */
DG_API const char *dg_status_string(dg_status status);

/* Name of the GEMM kernel that the calling thread's last GEMM call launched ("" before the
 * first): "gemm_kernel", "gemm_kernel (CTA pairs)", "gemm_kernel (last-wave split S)" or
 * "gemm_kernel (CTA pairs, last-wave split S)" when the last wave's tiles were cut into S K
 * pieces, "gemm_swap_kernel (stream-K)",
 * "gemm_splitk_kernel (cluster split-K)" or "gemm_bs_kernel (UE8M0 block-scaled MMA)". For
 * benchmarks and profiles; valid until the thread's next GEMM call. */
DG_API const char *dg_last_kernel(void);

/* Number of kernels the calling thread's last launching GEMM call launched (0 before the
 * first): 1, or 2 for a tile GEMM whose last-wave split ran behind a launch of the whole
 * waves. For benchmarks that count launches. */
DG_API int dg_last_launch_count(void);

/* Bytes of device memory the library has allocated with cudaMalloc so far, over all devices
 * (the few-row stream-K workspaces); the static arrays of the module are not counted. */
DG_API long long dg_allocated_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
