// dg_gemm_bs.cuh — FP8 NT GEMM with UE8M0 (power-of-two) block scales applied by the tensor
// core itself (tcgen05.mma kind::mxf8f6f4.block_scale), sm_100a.
//
// likun.im/craft/deepgemm §五: on SM100 the scales are packed UE8M0, four per 32-bit word; §二:
// the fp8 GEMM takes disable_ue8m0_cast. D = C + A·Bᵀ (§一) with the block scaling of
// aitangshan.cn/news/1491278 技术原理 §4, where every scale is a power of two: then
// sfa·sfb·S_kb is exact in fp32 and the hardware applies it inside the MMA, and the product
// accumulates in TMEM across all K blocks — no promotion through registers and no commit per
// K block for the math warps to wait on.
//
// Scales in global memory (packed, MN-major for A): sfa uint32 [ceil(Kb/4)][pad4(M)], byte kb%4
// of word (kb/4, m) = the UE8M0 of A[m, kb·128 ..]; sfb uint32 [Nb][ceil(Kb/4)] for the 128x128
// blocks of B. The MMA reads its scales from TMEM: per K block (four MMAs of K = 32, one scale
// per row of A and per row of B for each), row r of A's scale sits in TMEM lane r%32, column
// c + r/32, byte j (the scale-factor id of the instruction descriptor picks the byte), the same
// in all four lane quadrants, and B's likewise in columns c+4 .. c+11 (rows 0-127, 128-255) —
// the layout a tcgen05.cp .32x128b.warpx4 of a 512-byte scale atom gives. The scale warps write
// it directly from registers with tcgen05.st, each warp its own lane quadrant. With 1x128 and
// 128x128 scale blocks the four bytes of a word are equal, so every sub-block sees the same scale.
//
// Tiles: one CTA per 128 x BN tile (cta_group::1, M = 128, N = BN = 224), persistent. Two TMEM
// accumulators of 224 columns (448 of the 512) let a tile's epilogue overlap the next tile's
// MMAs; the last 64 columns hold four 16-column scale slots, a ring of its own beside the five
// operand stages.
//
// CTA layout (384 threads): warp 0 A producers and warp 2 B producers (lanes 0 and 16: even and
// odd K blocks, TMA into a 5-deep ring), warp 1 TMEM allocator and the MMA issuer (one thread:
// four block-scaled MMAs per K block, a commit of the stages every two K blocks and of the
// accumulator at the tile's end), warps 4-7 the scale writers (per K block, once the MMAs that
// last used the slot are done, they load the packed scale words, unpack the K block's byte and
// store the slot with tcgen05.st), warps 8-11 the epilogue (per tile, 64 columns at a time: C
// loads issued, the accumulator read with tcgen05.ld, released after its last columns, C
// added and D stored as bf16, rounded to nearest even, while the MMA already works on the next
// tile).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include <type_traits>

#include "dg_gemm.cuh"
#include "dg_ptx.cuh"

namespace dg {

constexpr int BS_BN = 224;                 // tile columns (two accumulators + scale slots fit 512 TMEM columns)
constexpr int BS_STAGES = 5;
constexpr int BS_SF_SLOTS = 4;             // TMEM scale slots, a ring of their own
constexpr int BS_THREADS = 384;
constexpr int BS_SF_COL0 = 2 * BS_BN;      // first TMEM column of the scale slots (448)
constexpr int BS_SF_SLOT_COLS = 16;        // per slot: SFA 4 columns, SFB 8 columns

struct BsParams {
    int M, N, K;
    int Kb, Nb, Kq;          // K/128, ceil(N/128), ceil(Kb/4)
    int ld_sfa;              // pad4(M)
    int m_blocks, n_blocks;  // ceil(M/128), ceil(N/BS_BN)
    int num_tiles;
    int has_c;
    const uint32_t *sfa;     // packed UE8M0 [Kq][ld_sfa]
    const uint32_t *sfb;     // packed UE8M0 [Nb][Kq]
    const __nv_bfloat16 *c;
    __nv_bfloat16 *d;
    int *err;
    uint64_t timeout_ns;
};

struct BsLayout {
    static constexpr int A_BYTES = BM * BK;                  // 16 KB
    static constexpr int B_BYTES = BS_BN * BK;               // 28 KB
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + BS_STAGES * A_BYTES;
    static constexpr int OFF_BAR = OFF_B + BS_STAGES * B_BYTES;
    // full, empty per stage; sf_full per scale slot; tfull, tempty per accumulator
    static constexpr int NUM_BARS = 2 * BS_STAGES + BS_SF_SLOTS + 4;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;
    static_assert(OFF_B % 1024 == 0, "1024-byte aligned operand tiles");
    static_assert(BS_SF_COL0 + BS_SF_SLOTS * BS_SF_SLOT_COLS <= 512, "TMEM columns");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

// Instruction descriptor of tcgen05.mma kind::mxf8f6f4.block_scale: A and B E4M3 (format 0 at
// bits 7-9 and 10-12), both K-major, N>>3 at bits 17-22, scale format UE8M0 (bit 23 = 1), M>>4
// at bits 24-28; scale-factor ids of B (bits 4-5) and A (bits 29-30) pick the byte of the TMEM
// scale word; accumulation is fp32.
template <int M_, int N_>
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3_ue8m0(uint32_t sf_id) {
    return (sf_id << 4) | (static_cast<uint32_t>(N_ >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(M_ >> 4) << 24) | (sf_id << 29);
}

// D[tmem] (+)= (A ⊙ sfa)·(B ⊙ sfb)ᵀ with the scales read from TMEM, one CTA, one thread.
__device__ __forceinline__ void umma_mxf8_bs(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
}

__global__ void __launch_bounds__(BS_THREADS, 1)
    gemm_bs_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const BsParams p) {
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    using L = BsLayout;
    constexpr int S = BS_STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *empty = full + S;
    uint64_t *sf_full = empty + S;            // [BS_SF_SLOTS]
    uint64_t *tfull = sf_full + BS_SF_SLOTS;
    uint64_t *tempty = tfull + 2;
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    volatile int *abort_flag = &ctx->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < BS_SF_SLOTS; ++j) mbar_init(&sf_full[j], 4);   // one arrive per scale warp
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);          // one arrive per epilogue warp
        }
        ctx->abort = 0;
        ctx->err = p.err;
        ctx->limit_ns = p.timeout_ns;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(&ctx->tmem_base, 512);
        tmem_relinquish();
    }
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;
    const int cid = static_cast<int>(blockIdx.x), ncid = static_cast<int>(gridDim.x);
    // tile t -> 128-row block and 224-column block, bands of 16 row blocks for L2 reuse of B
    auto tile_of = [&](int t, int &mb, int &nbk) { raster(t, p.m_blocks, p.n_blocks, RASTER_BLOCKS, mb, nbk); };

    if (warp < 4) {
        const int stream = (warp == 0 || warp == 2) && (lane & 15) == 0 ? warp >> 1 : -1;
        const uint32_t parity = static_cast<uint32_t>(lane >> 4);
        if (stream >= 0) {
            // TMA producers: A (warp 0) and B (warp 2), even and odd K blocks on lanes 0 / 16
            uint32_t it = 0;
            for (int t = cid; t < p.num_tiles && !*abort_flag; t += ncid) {
                int mb, nbk;
                tile_of(t, mb, nbk);
                for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                    if ((it & 1u) != parity) continue;
                    const int s = it % S;
                    if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, ctx)) break;
                    if (stream == 0) {
                        mbar_arrive_expect_tx(&full[s], L::STAGE_TX);
                        tma_load_2d(&tm_a, &full[s], smem + L::OFF_A + s * L::A_BYTES, kb * BK, mb * BM);
                    } else {
                        tma_load_2d(&tm_b, &full[s], smem + L::OFF_B + s * L::B_BYTES, kb * BK, nbk * BS_BN);
                    }
                }
            }
        } else if (warp == 1 && lane == 0) {
            // MMA issuer. Once the stage is loaded and its scale slot written, four MMAs of
            // K = 32; a commit releases two stages at a time (a commit holds back this thread's
            // later MMAs until the committed ones are done, so fewer commits keep the pipe full)
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int t = cid; t < p.num_tiles && ok; t += ncid, ++tcount) {
                const int b = tcount & 1;
                ok = mbar_wait(&tempty[b], ((tcount >> 1) & 1) ^ 1, ctx);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + static_cast<uint32_t>(b * BS_BN);
                int pending = 0;
                for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                    const int s = it % S;
                    const int j = it % BS_SF_SLOTS;
                    ok = mbar_wait(&full[s], (it / S) & 1, ctx) &&
                         mbar_wait(&sf_full[j], (it / BS_SF_SLOTS) & 1, ctx);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(BS_SF_COL0 + j * BS_SF_SLOT_COLS);
                    const uint64_t ad = sdesc_k_sw128(smem_u32(smem + L::OFF_A + s * L::A_BYTES));
                    const uint64_t bd = sdesc_k_sw128(smem_u32(smem + L::OFF_B + s * L::B_BYTES));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        umma_mxf8_bs(dt, ad + 2 * k, bd + 2 * k, idesc_mxf8_e4m3_ue8m0<128, BS_BN>(static_cast<uint32_t>(k)),
                                     sf_col, sf_col + 4, (kb > 0 || k > 0) ? 1u : 0u);
                    if (++pending == 2 || kb + 1 == p.Kb) {
                        for (uint32_t q = it + 1 - pending; q <= it; ++q) umma_commit(&empty[q % S]);
                        pending = 0;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[b]);
            }
        }
    } else if (warp < 8) {
        // ---------------- scales (warps 4-7) into the TMEM scale slots ----------------
        // Warp q (= warp % 4) writes TMEM lanes 32q..32q+31 of slot j = it % BS_SF_SLOTS, all four
        // quadrants alike (the layout a 32x128b.warpx4 copy of a scale atom would give): lane l,
        // column c + k holds the UE8M0 of A row 32k + l of the tile (its byte repeated for the
        // four K sub-blocks), column c + 4 + 4h + k that of B row 128h + 32k + l (the scale of its
        // 128x128 block). A slot is rewritten once the MMAs of the K block that last used it are
        // done (their stage's release; the ring of stages is longer than the ring of slots).
        const int q = warp & 3;
        uint32_t it = 0;
        bool ok = true;
        for (int t = cid; t < p.num_tiles && ok; t += ncid) {
            int mb, nbk;
            tile_of(t, mb, nbk);
            for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                const int j = it % BS_SF_SLOTS;
                if (it >= static_cast<uint32_t>(BS_SF_SLOTS)) {
                    const uint32_t prev = it - BS_SF_SLOTS;
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(&empty[prev % S], (prev / S) & 1, ctx));
                    if (!ok) break;
                    tc_fence_after();
                }
                const int shift = 8 * (kb & 3);
                uint32_t wa[4], wb[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int row = mb * BM + 32 * k + lane;
                    const uint32_t w = row < p.M ? __ldg(p.sfa + static_cast<size_t>(kb >> 2) * p.ld_sfa + row) : 0x7F7F7F7Fu;
                    wa[k] = ((w >> shift) & 0xFFu) * 0x01010101u;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int n = nbk * BS_BN + 128 * h + 32 * k + lane;   // rows past the tile's 224 are never read
                        const int nb = min(n, p.N - 1) >> 7;
                        const uint32_t w = __ldg(p.sfb + static_cast<size_t>(nb) * p.Kq + (kb >> 2));
                        wb[4 * h + k] = ((w >> shift) & 0xFFu) * 0x01010101u;
                    }
                const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                      static_cast<uint32_t>(BS_SF_COL0 + j * BS_SF_SLOT_COLS);
                tmem_st4(tcol, wa);
                tmem_st8(tcol + 4, wb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[j]);
            }
        }
    } else {
        // ---------------- epilogue (warps 8-11): lanes 32q.., all 224 columns ----------------
        // Per tile: this thread's row of C is prefetched into L2 before the accumulator is ready;
        // then 64 columns at a time (the last group 32): the C loads of the group are issued,
        // its TMEM loads issued and waited for, and the sums stored, so that every memory and
        // TMEM latency of a group overlaps the others of the same group.
        const int q = warp & 3;                    // TMEM lane quadrant
        uint32_t tcount = 0;
        bool ok = true;
        for (int t = cid; t < p.num_tiles && ok; t += ncid, ++tcount) {
            int mb, nbk;
            tile_of(t, mb, nbk);
            const int b = tcount & 1;
            const int row = mb * BM + q * 32 + lane;
            const int col0 = nbk * BS_BN;
            const size_t rbase = static_cast<size_t>(row < p.M ? row : 0) * p.N;

            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (tcount >> 1) & 1, ctx));
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BS_BN);
            // NC chunks of 16 columns starting at chunk c0 (N % 16 == 0: a chunk is all in or out)
            auto group = [&](auto nc_tag, int c0) {
                constexpr int NC = decltype(nc_tag)::value;
                uint4 cv[NC][2];
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const int col = col0 + (c0 + c) * 16;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        cv[c][hh] = p.has_c && row < p.M && col < p.N
                                        ? __ldg(reinterpret_cast<const uint4 *>(p.c + rbase + col + hh * 8))
                                        : make_uint4(0, 0, 0, 0);
                }
                uint32_t r16[NC][16];
#pragma unroll
                for (int c = 0; c < NC; ++c) tmem_ld16(taddr + (c0 + c) * 16, r16[c]);
#pragma unroll
                for (int c = 0; c < NC; ++c) tmem_ld_wait_regs16(r16[c]);
                if (c0 + NC == BS_BN / 16) {
                    // every column of the accumulator is in registers: the next tile may use it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[b]);
                }
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const int col = col0 + (c0 + c) * 16;
                    if (row < p.M && col < p.N) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t cw[4] = {cv[c][hh].x, cv[c][hh].y, cv[c][hh].z, cv[c][hh].w};
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float f0 = __uint_as_float(r16[c][hh * 8 + 2 * e]);
                                float f1 = __uint_as_float(r16[c][hh * 8 + 2 * e + 1]);
                                if (p.has_c) {
                                    f0 += __uint_as_float(cw[e] << 16);
                                    f1 += __uint_as_float(cw[e] & 0xFFFF0000u);
                                }
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(f0, f1);
                                w[e] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            *reinterpret_cast<uint4 *>(p.d + rbase + col + hh * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            };
            static_assert(BS_BN % 64 == 32, "three groups of 64 columns and one of 32");
#pragma unroll 1
            for (int g = 0; g < BS_BN / 64; ++g) group(std::integral_constant<int, 4>(), g * 4);
            group(std::integral_constant<int, 2>(), (BS_BN / 64) * 4);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
#endif
}

}  // namespace dg
