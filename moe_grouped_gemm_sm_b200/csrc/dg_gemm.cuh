// dg_gemm.cuh — persistent, warp-specialised FP8 block-scaled NT GEMM for sm_100a.
//
// D = C + A·Bᵀ (likun.im/craft/deepgemm §一) with block-wise scales promoted per 128-wide
// K block (aitangshan.cn/news/1491278 技术原理 §4): for every K block kb the tensor core
// produces the unscaled partial P_kb = A[:, kb]·B[:, kb]ᵀ in TMEM, and the math warps fold it
// into fp32 registers as acc += P_kb · sfa[m,kb] · sfb[n/128,kb].
//
// CTA layout (384 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: A tile [128 x 128 B], B tile [BN x 128 B] into a STAGES-deep
//               ring (full/empty mbarriers), and the tile's 128 A scales into a separate,
//               deeper ring so that releasing an operand stage never waits for the promotion.
//   warp 1      TMEM allocator and the single thread that issues tcgen05.mma (kind::f8f6f4,
//               M=128, N=BN, four K=32 steps per K block) into one of two TMEM buffers.
//   warps 2-3   idle.
//   warps 4-11  two math warpgroups. Warp w reads TMEM lanes 32·(w%4)..+31 (its 32 rows);
//               warpgroup j owns columns [j·BN/2, (j+1)·BN/2). Each K block: wait for the
//               TMEM buffer, load the partial, release the buffer, FMA into registers.
//               Epilogue: C (prefetched by TMA into the warp's staging slab at tile start) is
//               added, the result converted to bf16 (round to nearest even), written to the
//               slab in the 128-byte-swizzled layout and stored by TMA.
//
// Tile order: dense and contiguous tiles are rasterised in bands of GROUP_M M-blocks so that
// concurrently resident CTAs share B tiles in L2. Contiguous: the expert of an M-block is
// grouped_layout[first row] (likun.im §二 grouped_layout; each expert's rows are padded to
// 128). Masked: tiles are enumerated per expert over ceil(masked_m[g]/128) M-blocks only
// (likun.im §二 masked_m), and rows >= masked_m[g] are never stored.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

enum GemmKind : int { KIND_DENSE = 0, KIND_CONTIGUOUS = 1, KIND_MASKED = 2 };

constexpr int BM = 128;          // rows of a tile (MMA M, one TMEM lane per row)
constexpr int BK = 128;          // K block = scale granularity = one 128-byte swizzle row
constexpr int GEMM_THREADS = 384;
constexpr int GROUP_M = 16;      // rasterisation band height, in M-blocks

struct GemmParams {
    int M;            // rows per group of D (dense: M, contiguous: M_sum, masked: M_max)
    int N, K, G;
    int Kb, Nb;       // K/128, ceil(N/128)
    int m_blocks;     // ceil(M/128)
    int n_blocks;     // ceil(N/BN)
    int num_tiles;    // dense / contiguous (masked: derived on the device from masked_m)
    int has_c;
    const float *sfb;
    const int32_t *grouped_layout;
    const int32_t *masked_m;
    __nv_bfloat16 *d;
    int *err;
    uint64_t timeout_ns;
};

template <int BN, int STAGES>
struct NormalLayout {
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
    static constexpr int HALF = BN / 2;                 // columns per math warpgroup
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int SLAB_BYTES = 32 * HALF * 2;    // 32 rows x HALF bf16 per math warp
    static constexpr int SFA_STAGES = STAGES + 4;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_D = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFA = OFF_D + 8 * SLAB_BYTES;
    static constexpr int OFF_BAR = OFF_SFA + SFA_STAGES * BM * 4;
    static constexpr int NBUF = 512 / BN;               // TMEM partial buffers (MMA run-ahead)
    static constexpr int NUM_BARS = 2 * STAGES + 2 * SFA_STAGES + 2 * NBUF + 8;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;          // slack to align the base to 1024 B
    static constexpr uint32_t TMEM_COLS = 512;          // NBUF partial buffers of BN columns
    static_assert(OFF_B % 1024 == 0 && OFF_D % 1024 == 0, "1024-byte aligned operand tiles");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

struct TileInfo {
    int m_blk, n_blk, g;
    bool valid;
};

__device__ __forceinline__ int clamp_masked(int v, int M) { return v < 0 ? 0 : (v > M ? M : v); }

// Number of tiles of the masked layout: sum over experts of ceil(masked_m[g]/128)·n_blocks.
__device__ __forceinline__ int masked_num_tiles(const GemmParams &p) {
    int total = 0;
    for (int g = 0; g < p.G; ++g) {
        const int mm = clamp_masked(__ldg(p.masked_m + g), p.M);
        total += (mm + BM - 1) / BM * p.n_blocks;
    }
    return total;
}

template <int KIND>
__device__ __forceinline__ TileInfo decode_tile(int t, const GemmParams &p) {
    TileInfo ti;
    ti.valid = true;
    ti.g = 0;
    if (KIND == KIND_MASKED) {
        int rem = t;
        for (int g = 0; g < p.G; ++g) {
            const int mt = (clamp_masked(__ldg(p.masked_m + g), p.M) + BM - 1) / BM;
            const int cnt = mt * p.n_blocks;
            if (rem < cnt) {
                ti.g = g;
                ti.m_blk = rem % mt;       // M-blocks of one expert are adjacent: B tile reuse
                ti.n_blk = rem / mt;
                return ti;
            }
            rem -= cnt;
        }
        ti.valid = false;
        ti.m_blk = ti.n_blk = 0;
        return ti;
    }
    const int per_band = GROUP_M * p.n_blocks;
    const int band = t / per_band;
    const int first_m = band * GROUP_M;
    const int band_m = min(GROUP_M, p.m_blocks - first_m);
    const int local = t - band * per_band;
    ti.m_blk = first_m + local % band_m;
    ti.n_blk = local / band_m;
    if (KIND == KIND_CONTIGUOUS) {
        const int g = __ldg(p.grouped_layout + ti.m_blk * BM);
        ti.g = g;
        ti.valid = (g >= 0 && g < p.G);
    }
    return ti;
}

// tcgen05.wait::ld with the loaded registers as in/out operands, so that no use of them can
// be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

// The same for one 32-register batch.
__device__ __forceinline__ void tmem_ld_wait_regs32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// The same for four 16-register groups (64 registers).
__device__ __forceinline__ void tmem_ld_wait_regs4(uint32_t (&r)[4][16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[0][4]), "+r"(r[0][5]),
                   "+r"(r[0][6]), "+r"(r[0][7]), "+r"(r[0][8]), "+r"(r[0][9]), "+r"(r[0][10]), "+r"(r[0][11]),
                   "+r"(r[0][12]), "+r"(r[0][13]), "+r"(r[0][14]), "+r"(r[0][15]),
                   "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[1][4]), "+r"(r[1][5]),
                   "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[1][8]), "+r"(r[1][9]), "+r"(r[1][10]), "+r"(r[1][11]),
                   "+r"(r[1][12]), "+r"(r[1][13]), "+r"(r[1][14]), "+r"(r[1][15]),
                   "+r"(r[2][0]), "+r"(r[2][1]), "+r"(r[2][2]), "+r"(r[2][3]), "+r"(r[2][4]), "+r"(r[2][5]),
                   "+r"(r[2][6]), "+r"(r[2][7]), "+r"(r[2][8]), "+r"(r[2][9]), "+r"(r[2][10]), "+r"(r[2][11]),
                   "+r"(r[2][12]), "+r"(r[2][13]), "+r"(r[2][14]), "+r"(r[2][15]),
                   "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3]), "+r"(r[3][4]), "+r"(r[3][5]),
                   "+r"(r[3][6]), "+r"(r[3][7]), "+r"(r[3][8]), "+r"(r[3][9]), "+r"(r[3][10]), "+r"(r[3][11]),
                   "+r"(r[3][12]), "+r"(r[3][13]), "+r"(r[3][14]), "+r"(r[3][15])
                 :
                 : "memory");
}

template <int BN, int STAGES, int KIND>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_normal_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_c,
                       const __grid_constant__ CUtensorMap tm_d, const GemmParams p) {
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    using L = NormalLayout<BN, STAGES>;
    constexpr int HALF = L::HALF;
    constexpr int SFS = L::SFA_STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *sfa_full = empty + STAGES;
    uint64_t *sfa_empty = sfa_full + SFS;
    uint64_t *tfull = sfa_empty + SFS;
    uint64_t *tempty = tfull + L::NBUF;
    uint64_t *cfull = tempty + L::NBUF;
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    volatile int *abort_flag = &ctx->abort;
    const float *sfa_ring = reinterpret_cast<const float *>(smem + L::OFF_SFA);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < SFS; ++j) {
            mbar_init(&sfa_full[j], 1);
            mbar_init(&sfa_empty[j], 8);
        }
        for (int b = 0; b < L::NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        for (int w = 0; w < 8; ++w) mbar_init(&cfull[w], 1);
        ctx->abort = 0;
        ctx->err = p.err;
        ctx->limit_ns = p.timeout_ns;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_sfa);
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_d);
    }
    if (warp == 1) {
        tmem_alloc(&ctx->tmem_base, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;

    const int num_tiles = (KIND == KIND_MASKED) ? masked_num_tiles(p) : p.num_tiles;
    if (KIND == KIND_MASKED && blockIdx.x == 0 && threadIdx.x == 0) {
        for (int g = 0; g < p.G; ++g)
            if (__ldg(p.masked_m + g) > p.M) report_error(p.err, ERR_DATA);
    }

    if (warp < 4) {
        reg_dealloc<56>();
        if (warp == 0 && lane == 0) {
            // ---------------- TMA producer ----------------
            uint32_t it = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile<KIND>(t, p);
                if (!ti.valid) {
                    if (KIND == KIND_CONTIGUOUS && ti.g >= p.G) report_error(p.err, ERR_DATA);
                    continue;
                }
                for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, ctx)) break;
                    const int j = it % SFS;
                    const uint32_t phj = (it / SFS) & 1;
                    if (!mbar_wait(&sfa_empty[j], phj ^ 1, ctx)) break;
                    mbar_arrive_expect_tx(&full[s], L::A_BYTES + L::B_BYTES);
                    uint8_t *sa = smem + L::OFF_A + s * L::A_BYTES;
                    uint8_t *sb = smem + L::OFF_B + s * L::B_BYTES;
                    if (KIND == KIND_MASKED)
                        tma_load_3d(&tm_a, &full[s], sa, kb * BK, ti.m_blk * BM, ti.g);
                    else
                        tma_load_2d(&tm_a, &full[s], sa, kb * BK, ti.m_blk * BM);
                    tma_load_3d(&tm_b, &full[s], sb, kb * BK, ti.n_blk * BN, ti.g);
                    mbar_arrive_expect_tx(&sfa_full[j], BM * 4);
                    float *sf = reinterpret_cast<float *>(smem + L::OFF_SFA) + j * BM;
                    if (KIND == KIND_MASKED)
                        tma_load_3d(&tm_sfa, &sfa_full[j], sf, ti.m_blk * BM, kb, ti.g);
                    else
                        tma_load_2d(&tm_sfa, &sfa_full[j], sf, ti.m_blk * BM, kb);
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t IDESC = idesc_f8_e4m3_f32<BM, BN>();
            uint32_t it = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile<KIND>(t, p);
                if (!ti.valid) continue;
                for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    const int b = it % L::NBUF;
                    const uint32_t phb = (it / L::NBUF) & 1;
                    if (!mbar_wait(&full[s], ph, ctx)) break;
                    if (!mbar_wait(&tempty[b], phb ^ 1, ctx)) break;
                    tc_fence_after();
                    const uint64_t ad = sdesc_k_sw128(smem_u32(smem + L::OFF_A + s * L::A_BYTES));
                    const uint64_t bd = sdesc_k_sw128(smem_u32(smem + L::OFF_B + s * L::B_BYTES));
                    const uint32_t dt = tmem_base + static_cast<uint32_t>(b * BN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        umma_f8(dt, ad + 2 * k, bd + 2 * k, IDESC, k > 0 ? 1u : 0u);
                    umma_commit(&empty[s]);
                    umma_commit(&tfull[b]);
                }
            }
        }
    } else {
        reg_alloc<224>();
        // ---------------- math warpgroups: promotion + epilogue ----------------
        const int mw = warp - 4;               // 0..7
        const int wg = mw >> 2;                // column half
        const int q = warp & 3;                // TMEM lane quadrant
        uint8_t *slab = smem + L::OFF_D + mw * L::SLAB_BYTES;
        uint32_t it = 0, ctile = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const TileInfo ti = decode_tile<KIND>(t, p);
            if (!ti.valid) continue;
            const int col0 = ti.n_blk * BN + wg * HALF;          // first column of this warp
            const int row0 = ti.m_blk * BM + q * 32;             // first row of this warp's slab
            const int nblk = min(col0 / 128, p.Nb - 1);
            const float *sfb_row = p.sfb + (static_cast<size_t>(ti.g) * p.Nb + nblk) * p.Kb;
            if (p.has_c && lane == 0) {
                bulk_wait_group_read0();                         // the slab's last store has read it
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&cfull[mw], L::SLAB_BYTES);
#pragma unroll
                for (int bx = 0; bx < HALF / 64; ++bx) {
                    if (KIND == KIND_MASKED)
                        tma_load_3d(&tm_c, &cfull[mw], slab + bx * 4096, col0 + bx * 64, row0, ti.g);
                    else
                        tma_load_2d(&tm_c, &cfull[mw], slab + bx * 4096, col0 + bx * 64, row0);
                }
            }
            float2 acc[HALF / 2];
#pragma unroll
            for (int i = 0; i < HALF / 2; ++i) acc[i] = make_float2(0.f, 0.f);
            // sfb of this warp's n-block for 32 consecutive K blocks, one per lane; the next
            // window is fetched a full window ahead and broadcast by shuffle
            float sb_win = lane < p.Kb ? __ldg(sfb_row + lane) : 0.f;
            float sb_nxt = 32 + lane < p.Kb ? __ldg(sfb_row + 32 + lane) : 0.f;
            for (int kb = 0; kb < p.Kb; ++kb, ++it) {
                const int b = it % L::NBUF;
                const uint32_t phb = (it / L::NBUF) & 1;
                const int j = it % SFS;
                const uint32_t phj = (it / SFS) & 1;
                if ((kb & 31) == 0 && kb > 0) {
                    sb_win = sb_nxt;
                    sb_nxt = kb + 32 + lane < p.Kb ? __ldg(sfb_row + kb + 32 + lane) : 0.f;
                }
                const float sb = __shfl_sync(0xFFFFFFFFu, sb_win, kb & 31);
                // every lane waits; the outcome is made warp-uniform before any .sync.aligned op
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sfa_full[j], phj, ctx));
                if (!ok) break;
                const float sa = sfa_ring[j * BM + q * 32 + lane];
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfa_empty[j]);
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], phb, ctx));
                if (!ok) break;
                tc_fence_after();
                const float scale = sa * sb;
                const float2 scale2 = make_float2(scale, scale);
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(b * BN + wg * HALF);
                // 32-column batches, double-buffered in registers: the TMEM load of batch c+1 is
                // in flight while batch c is folded into the accumulator (tcgen05.wait::ld waits
                // for every outstanding load, so at most one batch is in flight)
                uint32_t r[2][32];
                tmem_ld32(taddr, r[0]);
                tmem_ld_wait_regs32(r[0]);
#pragma unroll
                for (int c = 0; c < HALF / 32; ++c) {
                    if (c + 1 < HALF / 32) tmem_ld32(taddr + (c + 1) * 32, r[(c + 1) & 1]);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        acc[c * 16 + i] = __ffma2_rn(make_float2(__uint_as_float(r[c & 1][2 * i]),
                                                                 __uint_as_float(r[c & 1][2 * i + 1])),
                                                     scale2, acc[c * 16 + i]);
                    if (c + 1 < HALF / 32) tmem_ld_wait_regs32(r[(c + 1) & 1]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[b]);
            }
            if (!ok) break;
            if (p.has_c) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&cfull[mw], ctile & 1, ctx));
                if (!ok) break;
                ++ctile;
            } else {
                if (lane == 0) bulk_wait_group_read0();          // the slab's last store has read it
                __syncwarp();
            }
            // bf16 epilogue into the swizzled slab: row `lane`, 16-byte chunk ch of box bx lives
            // at bx*4096 + lane*128 + ((ch ^ (lane & 7)) * 16).
#pragma unroll
            for (int bx = 0; bx < HALF / 64; ++bx) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 *pchunk = reinterpret_cast<uint4 *>(slab + bx * 4096 + lane * 128 + ((ch ^ (lane & 7)) * 16));
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[2 * e] = acc[bx * 32 + ch * 4 + e].x;
                        v[2 * e + 1] = acc[bx * 32 + ch * 4 + e].y;
                    }
                    if (p.has_c) {
                        const uint4 cv = *pchunk;
                        const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 c2 = *reinterpret_cast<const __nv_bfloat162 *>(&cw[e]);
                            v[2 * e] += __bfloat162float(c2.x);
                            v[2 * e + 1] += __bfloat162float(c2.y);
                        }
                    }
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                        w[e] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    *pchunk = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (KIND == KIND_MASKED) {
                const int mm = clamp_masked(__ldg(p.masked_m + ti.g), p.M);
                const int valid_rows = max(0, min(32, mm - row0));
                if (valid_rows == 32) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
#pragma unroll
                        for (int bx = 0; bx < HALF / 64; ++bx)
                            tma_store_3d(&tm_d, slab + bx * 4096, col0 + bx * 64, row0, ti.g);
                        bulk_commit_group();
                    }
                } else if (lane < valid_rows) {
                    // partial slab: only rows below masked_m[g] are written, each by its owner
                    __nv_bfloat16 *drow = p.d + (static_cast<size_t>(ti.g) * p.M + row0 + lane) * p.N;
#pragma unroll
                    for (int bx = 0; bx < HALF / 64; ++bx)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            const int col = col0 + bx * 64 + ch * 8;
                            if (col < p.N)
                                *reinterpret_cast<uint4 *>(drow + col) =
                                    *reinterpret_cast<const uint4 *>(slab + bx * 4096 + lane * 128 + ((ch ^ (lane & 7)) * 16));
                        }
                }
                fence_proxy_async_smem();
                __syncwarp();
            } else {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int bx = 0; bx < HALF / 64; ++bx) tma_store_2d(&tm_d, slab + bx * 4096, col0 + bx * 64, row0);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
#endif
}

}  // namespace dg
