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
// per row of A and per row of B for each), the scales go to TMEM by tcgen05.cp from "scale
// atoms" in shared memory: 512 bytes for 128 rows x 4 K sub-blocks, row r's byte for sub-block
// j at 16·(r%32) + 4·(r/32) + j. tcgen05.cp .32x128b.warpx4 puts atom row l into TMEM lane l
// (columns c .. c+3) of all four lane quadrants; the MMA then finds row r's scale in lane r%32,
// column c + r/32, byte j (the scale-factor id of the instruction descriptor). With 1x128 and
// 128x128 scale blocks the four bytes of a row are equal, so every sub-block sees the same scale.
//
// Tiles: one CTA per 128 x BN tile (cta_group::1, M = 128, N = BN = 224), persistent. Two TMEM
// accumulators of 224 columns (448 of the 512) let a tile's epilogue overlap the next tile's
// MMAs; the last 64 columns hold four 16-column scale slots (SFA 4 columns, SFB 8 columns for
// the up to 256 B rows of two 128-row atoms), one per ring stage.
//
// CTA layout (384 threads): warp 0 A producers and warp 2 B producers (lanes 0 and 16: even and
// odd K blocks, TMA into a STAGES-deep ring), warp 1 TMEM allocator and the MMA issuer (one
// thread: copies the stage's scale atoms to TMEM, issues four block-scaled MMAs, commits the
// stage every two K blocks and the accumulator at the tile's end), warps 4-7 the scale-atom
// writers (per K block they unpack the stage's scale bytes into its atoms once the stage's
// previous MMAs are done, running up to the ring's depth ahead of the MMA), warps 8-11 the
// epilogue (per tile they read the accumulator with tcgen05.ld, release it, add C and store D
// as bf16, rounded to nearest even, while the MMA already works on the next tile).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_gemm.cuh"
#include "dg_ptx.cuh"

namespace dg {

constexpr int BS_BN = 224;                 // tile columns (two accumulators + scale slots fit 512 TMEM columns)
constexpr int BS_STAGES = 4;
constexpr int BS_THREADS = 384;
constexpr int BS_SF_COL0 = 2 * BS_BN;      // first TMEM column of the scale slots (448)
constexpr int BS_SF_SLOT_COLS = 16;        // per stage: SFA 4 columns, SFB 8 columns

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
    static constexpr int ATOM = 512;                         // 128 rows x 4 scale bytes
    static constexpr int SF_BYTES = 3 * ATOM;                // SFA + two SFB atoms per stage
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + BS_STAGES * A_BYTES;
    static constexpr int OFF_SF = OFF_B + BS_STAGES * B_BYTES;
    static constexpr int OFF_BAR = OFF_SF + BS_STAGES * SF_BYTES;
    // full, empty, sf_full per stage; tfull, tempty per accumulator
    static constexpr int NUM_BARS = 3 * BS_STAGES + 4;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;
    static_assert(OFF_B % 1024 == 0 && OFF_SF % 1024 == 0, "1024-byte aligned operand tiles");
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

// Shared-memory descriptor of a scale atom for tcgen05.cp: 32 rows of 16 bytes, no swizzle,
// K-major core matrices of 8 rows x 16 bytes (128 bytes) one after another (stride byte offset
// 128), version 1, layout type 0.
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(16 >> 4) << 16;
    d |= static_cast<uint64_t>(128 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;
}

// 32 lanes x 128 bits from shared memory into TMEM columns taddr .. taddr+3 of all four lane
// quadrants (the copy of a scale atom).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
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
    uint64_t *sf_full = empty + S;
    uint64_t *tfull = sf_full + S;
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
            mbar_init(&sf_full[s], 4);         // one arrive per atom-writing warp
        }
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
            // MMA issuer. The stage's scale atoms go to its TMEM scale slot, then four MMAs of
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
                    ok = mbar_wait(&full[s], (it / S) & 1, ctx) && mbar_wait(&sf_full[s], (it / S) & 1, ctx);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(BS_SF_COL0 + s * BS_SF_SLOT_COLS);
                    const uint32_t sf_smem = smem_u32(smem + L::OFF_SF + s * L::SF_BYTES);
                    tmem_cp_32x128b_x4(sf_col, sdesc_sf_atom(sf_smem));                      // SFA
                    tmem_cp_32x128b_x4(sf_col + 4, sdesc_sf_atom(sf_smem + L::ATOM));        // SFB rows 0-127
                    tmem_cp_32x128b_x4(sf_col + 8, sdesc_sf_atom(sf_smem + 2 * L::ATOM));    // SFB rows 128-255
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
        // ---------------- scale atoms (warps 4-7): thread r writes row r of every atom ----------------
        const int r = threadIdx.x - 128;           // 0..127
        uint32_t it = 0;
        bool ok = true;
        for (int t = cid; t < p.num_tiles && ok; t += ncid) {
            int mb, nbk;
            tile_of(t, mb, nbk);
            const int row = mb * BM + r;
            for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                const int s = it % S;
                // the stage's previous MMAs have read its atoms (their commit released the stage)
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], ((it / S) & 1) ^ 1, ctx));
                if (!ok) break;
                uint32_t *atoms = reinterpret_cast<uint32_t *>(smem + L::OFF_SF + s * L::SF_BYTES);
                const int shift = 8 * (kb & 3);
                const int slot = 4 * (r & 31) + (r >> 5);
                // SFA: row r's byte, replicated over the four K sub-blocks
                const uint32_t wa = row < p.M ? __ldg(p.sfa + static_cast<size_t>(kb >> 2) * p.ld_sfa + row) : 0x7F7F7F7Fu;
                atoms[slot] = ((wa >> shift) & 0xFFu) * 0x01010101u;
                // SFB: B rows r and 128 + r of the tile (rows past its 224 are never read) take
                // the scale of their 128x128 block
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = nbk * BS_BN + h * 128 + r;
                    const int nb = min(n, p.N - 1) >> 7;
                    const uint32_t wb = __ldg(p.sfb + static_cast<size_t>(nb) * p.Kq + (kb >> 2));
                    atoms[128 * (1 + h) + slot] = ((wb >> shift) & 0xFFu) * 0x01010101u;
                }
                fence_proxy_async_smem();          // generic writes -> the tensor core's copy
                __syncwarp();
                if ((r & 31) == 0) mbar_arrive(&sf_full[s]);
            }
        }
    } else {
        // ---------------- epilogue (warps 8-11): lanes 32q.., all 224 columns ----------------
        const int q = warp & 3;                    // TMEM lane quadrant
        uint32_t tcount = 0;
        bool ok = true;
        for (int t = cid; t < p.num_tiles && ok; t += ncid, ++tcount) {
            int mb, nbk;
            tile_of(t, mb, nbk);
            const int b = tcount & 1;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (tcount >> 1) & 1, ctx));
            if (!ok) break;
            tc_fence_after();
            const int row = mb * BM + q * 32 + lane;
            const int col0 = nbk * BS_BN;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BS_BN);
            const size_t rbase = static_cast<size_t>(row < p.M ? row : 0) * p.N;
#pragma unroll 1
            for (int c = 0; c < BS_BN / 16; ++c) {
                uint32_t r16[16];
                tmem_ld16(taddr + c * 16, r16);
                tmem_ld_wait();
                if (c + 1 == BS_BN / 16) {
                    // every column of the accumulator is in registers: the next tile may use it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[b]);
                }
                const int col = col0 + c * 16;
                if (row < p.M && col < p.N) {      // N % 16 == 0: a 16-column chunk is all in or out
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r16[hh * 8 + e]);
                        if (p.has_c) {
                            const uint4 cv = __ldg(reinterpret_cast<const uint4 *>(p.c + rbase + col + hh * 8));
                            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                f[2 * e] += __uint_as_float(cw[e] << 16);
                                f[2 * e + 1] += __uint_as_float(cw[e] & 0xFFFF0000u);
                            }
                        }
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
                            w[e] = *reinterpret_cast<uint32_t *>(&h2);
                        }
                        *reinterpret_cast<uint4 *>(p.d + rbase + col + hh * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
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
