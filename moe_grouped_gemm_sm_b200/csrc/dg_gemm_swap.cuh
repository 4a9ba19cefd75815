// dg_gemm_swap.cuh — FP8 block-scaled NT GEMM for few rows (decode): swapped operands and
// split-K over a thread-block cluster, sm_100a.
//
// Same result as dg_gemm.cuh, D = C + A·Bᵀ with per-128-K-block promotion (likun.im/craft/
// deepgemm §一; aitangshan.cn/news/1491278 技术原理 §4), for layouts whose row count per group
// is small (the decode shapes and the masked MoE layout, likun.im §二 masked_m). With so
// few rows the GEMM streams the weights B from HBM, so the kernel is laid out for bandwidth:
//
//   * operands swapped: the tensor core computes P_kbᵀ = B_tile · A_kbᵀ with the 128 weight
//     rows of a tile on the MMA's M side (TMEM lanes) and the TN activation rows on its N side
//     (TMEM columns). A tile's 128 weight rows are one 128x128 scale block, so sfb is a single
//     scalar per (tile, K block), and sfa becomes a per-column factor read from shared memory;
//   * split-K: a cluster of S CTAs shares one tile, CTA r taking an even share of its K blocks;
//     the S fp32 partials meet in distributed shared memory, where CTA r reduces rows
//     [r·128/S, (r+1)·128/S) of the tile, adds C and writes D (bf16, round to nearest even).
//     No global workspace is used and the reduction order is fixed (deterministic);
//   * a deep TMA ring (6-8 stages of the 16 KB weight tile) keeps enough bytes in flight.
//
// CTA layout: warps 0, 2, 3 TMA producers (weights, activations, A scales), warp 1 TMEM
// allocator + single-thread tcgen05.mma issuer (kind::f8f6f4, M = 128, N = TN), warps 4.. TN/64
// math warpgroups (thread = weight row, registers = its warpgroup's 64 token columns).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_gemm.cuh"
#include "dg_ptx.cuh"

namespace dg {

struct SwapParams {
    int M;            // rows per group (dense: M <= TN; masked: M_max)
    int N, K, G;
    int Kb, Nb;       // K/128, ceil(N/128)
    int ld_sfa;       // pad4(M)
    int n_tiles;      // ceil(N/128)
    int m_tiles;      // ceil(M/TN): token tiles per group
    int num_tiles;    // (masked: G ·) m_tiles · n_tiles
    int splits;       // S: CTAs per cluster along K
    int has_c;
    const float *sfb;
    const int32_t *masked_m;   // masked layout only
    const __nv_bfloat16 *c;
    __nv_bfloat16 *d;
    int *err;
    uint64_t timeout_ns;
};

template <int TN, int STAGES>
struct SwapLayout {
    static_assert(TN == 64 || TN == 128, "token tile");
    static constexpr int NWG = TN / 64;                      // math warpgroups, 64 token columns each
    static constexpr int COLS = TN / NWG;                    // token columns per math warpgroup
    static constexpr int THREADS = 128 + 128 * NWG;
    static constexpr int W_BYTES = 128 * BK;                 // weight tile: 128 rows x 128 B
    static constexpr int X_BYTES = TN * BK;                  // activation tile: TN rows x 128 B
    static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
    static constexpr int NBUF = (512 / TN) > 4 ? 4 : (512 / TN);
    static constexpr int SFS = STAGES + NBUF + 1;            // A-scale ring (see dg_gemm.cuh)
    static constexpr int RED_BYTES = TN * 128 * 4;           // fp32 partial [TN][128], reuses the ring
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_SFA = OFF_X + STAGES * X_BYTES;
    static constexpr int OFF_C = OFF_SFA + SFS * TN * 4;        // C tile [TN][128] bf16 (S == 1 epilogue)
    static constexpr int C_BYTES = TN * 128 * 2;
    static constexpr int OFF_BAR = OFF_C + C_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + SFS + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = NBUF * TN <= 256 ? (NBUF * TN <= 128 ? 128 : 256) : 512;
    static_assert(OFF_X % 1024 == 0 && OFF_SFA % 16 == 0 && OFF_C % 128 == 0, "aligned tiles");
    static_assert(STAGES * STAGE_BYTES >= RED_BYTES, "the reduction buffer reuses the operand ring");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

template <int TN, int STAGES, int KIND>
__global__ void __launch_bounds__(SwapLayout<TN, STAGES>::THREADS, 1)
    gemm_swap_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_c,
                     const SwapParams p) {
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    using L = SwapLayout<TN, STAGES>;
    constexpr int NBUF = L::NBUF;
    constexpr int COLS = L::COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *sfa_full = tempty + NBUF;
    uint64_t *c_full = sfa_full + L::SFS;
    const __nv_bfloat16 *c_tile = reinterpret_cast<const __nv_bfloat16 *>(smem + L::OFF_C);
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    const float *sfa_ring = reinterpret_cast<const float *>(smem + L::OFF_SFA);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = p.splits;
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    // S == 1: persistent CTAs stride over the tiles; S > 1: one tile per cluster (grid = tiles·S)
    const int cid = S > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int ncid = S > 1 ? p.num_tiles : static_cast<int>(gridDim.x);
    const int per = (p.Kb + S - 1) / S;                      // K blocks per split
    const int kb0 = static_cast<int>(rank) * per;
    const int kb1 = min(p.Kb, kb0 + per);
    const int nkb = max(0, kb1 - kb0);

    // tile t = (g · m_tiles + mt) · n_tiles + nt: weight tile nt of expert g, token tile mt;
    // returns the number of token rows of the tile that exist (<= 0: nothing to do)
    auto tile_rows = [&](int t, int &g, int &m0, int &n0) {
        const int nt = t % p.n_tiles;
        const int mt = (t / p.n_tiles) % p.m_tiles;
        g = KIND == KIND_MASKED ? t / (p.n_tiles * p.m_tiles) : 0;
        n0 = nt * 128;
        m0 = mt * TN;
        int valid = p.M;
        if (KIND == KIND_MASKED) {
            const int mm = __ldg(p.masked_m + g);
            valid = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
        }
        return min(TN, valid - m0);
    };
    if (KIND == KIND_MASKED && blockIdx.x == 0 && threadIdx.x == 0) {
        for (int gg = 0; gg < p.G; ++gg)
            if (__ldg(p.masked_m + gg) > p.M) report_error(p.err, ERR_DATA);
    }
    if (S > 1) {                                           // every CTA of the cluster agrees
        int g_, m0_, n0_;
        if (tile_rows(cid, g_, m0_, n0_) <= 0) return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4 * L::NWG);
        }
        for (int j = 0; j < L::SFS; ++j) mbar_init(&sfa_full[j], 1);
        mbar_init(c_full, 1);
        ctx->abort = 0;
        ctx->err = p.err;
        ctx->limit_ns = p.timeout_ns;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_sfa);
        tma_prefetch_desc(&tm_c);
    }
    if (warp == 1) {
        tmem_alloc(&ctx->tmem_base, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;
    volatile int *abort_flag = &ctx->abort;

    float acc[COLS];
    int g = 0, m0 = 0, n0 = 0, rows = 0;                   // the last tile (split reduction)

    if (warp < 4) {
        // TMA producers, one thread per stream (one thread's bulk copies are served one after
        // another): warp 0 arms each stage and loads the weights, warp 2 the activations,
        // warp 3 the A scales. All wait on the ring's "empty" barriers.
        const int stream = warp == 0 ? 0 : (warp == 2 ? 1 : (warp == 3 ? 2 : -1));
        if (stream >= 0 && lane == 0) {
            uint32_t it = 0;
            for (int t = cid; t < p.num_tiles && !*abort_flag; t += ncid) {
                int tg, tm0, tn0;
                if (tile_rows(t, tg, tm0, tn0) <= 0) continue;
                for (int i = 0; i < nkb; ++i, ++it) {
                    const int kb = kb0 + i;
                    const int s = it % STAGES;
                    if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, ctx)) break;
                    if (stream == 2) {
                        const int j = it % L::SFS;
                        mbar_arrive_expect_tx(&sfa_full[j], TN * 4);
                        float *sf = reinterpret_cast<float *>(smem + L::OFF_SFA) + j * TN;
                        if (KIND == KIND_MASKED)
                            tma_load_3d(&tm_sfa, &sfa_full[j], sf, tm0, kb, tg);
                        else
                            tma_load_2d(&tm_sfa, &sfa_full[j], sf, tm0, kb);
                    } else if (stream == 0) {
                        mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
                        tma_load_3d(&tm_w, &full[s], smem + L::OFF_W + s * L::W_BYTES, kb * BK, tn0, tg);
                    } else if (KIND == KIND_MASKED) {
                        tma_load_3d(&tm_x, &full[s], smem + L::OFF_X + s * L::X_BYTES, kb * BK, tm0, tg);
                    } else {
                        tma_load_2d(&tm_x, &full[s], smem + L::OFF_X + s * L::X_BYTES, kb * BK, tm0);
                    }
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t IDESC = idesc_f8_e4m3_f32<128, TN>();
            uint32_t it = 0;
            for (int t = cid; t < p.num_tiles && !*abort_flag; t += ncid) {
                int tg, tm0, tn0;
                if (tile_rows(t, tg, tm0, tn0) <= 0) continue;
                for (int i = 0; i < nkb; ++i, ++it) {
                    const int s = it % STAGES;
                    const int b = it % NBUF;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, ctx)) break;
                    if (!mbar_wait(&tempty[b], ((it / NBUF) & 1) ^ 1, ctx)) break;
                    tc_fence_after();
                    const uint64_t wd = sdesc_k_sw128(smem_u32(smem + L::OFF_W + s * L::W_BYTES));
                    const uint64_t xd = sdesc_k_sw128(smem_u32(smem + L::OFF_X + s * L::X_BYTES));
                    const uint32_t dt = tmem_base + static_cast<uint32_t>(b * TN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) umma_f8(dt, wd + 2 * k, xd + 2 * k, IDESC, k > 0 ? 1u : 0u);
                    umma_commit(&empty[s]);
                    umma_commit(&tfull[b]);
                }
            }
        }
    } else {
        // ---------------- math warpgroups: promotion (+ the epilogue when S == 1) ----------------
        const int wg = (warp - 4) >> 2;                    // token columns [wg·64, wg·64 + 64)
        const int q = warp & 3;                            // TMEM lane quadrant = weight rows 32q..
        const int n = q * 32 + lane;                       // this thread's weight row in the tile
        uint32_t it = 0, ctile = 0;
        bool ok = true;
        for (int t = cid; t < p.num_tiles && ok; t += ncid) {
            rows = tile_rows(t, g, m0, n0);
            if (rows <= 0) continue;
            const int nt = n0 / 128;
            const bool do_c = S == 1 && p.has_c;
            if (do_c) {
                // the previous tile's C has been read by every math thread before it is replaced
                asm volatile("bar.sync 1, %0;" ::"n"(128 * L::NWG) : "memory");
                if (threadIdx.x == 128) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(c_full, L::C_BYTES);
                    if (KIND == KIND_MASKED)
                        tma_load_3d(&tm_c, c_full, smem + L::OFF_C, n0, m0, g);
                    else
                        tma_load_2d(&tm_c, c_full, smem + L::OFF_C, n0, m0);
                }
            }
#pragma unroll
            for (int i = 0; i < COLS; ++i) acc[i] = 0.f;
            const float *sfb_col = p.sfb + (static_cast<size_t>(g) * p.Nb + nt) * p.Kb;
            float sb_win = kb0 + lane < kb1 ? __ldg(sfb_col + kb0 + lane) : 0.f;
            float sb_nxt = kb0 + 32 + lane < kb1 ? __ldg(sfb_col + kb0 + 32 + lane) : 0.f;
            for (int i = 0; i < nkb; ++i, ++it) {
                const int b = it % NBUF;
                const int j = it % L::SFS;
                if ((i & 31) == 0 && i > 0) {
                    sb_win = sb_nxt;
                    sb_nxt = kb0 + i + 32 + lane < kb1 ? __ldg(sfb_col + kb0 + i + 32 + lane) : 0.f;
                }
                const float sb = __shfl_sync(0xFFFFFFFFu, sb_win, i & 31);
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (it / NBUF) & 1, ctx));
                if (!ok) break;
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sfa_full[j], (it / L::SFS) & 1, ctx));
                if (!ok) break;
                tc_fence_after();
                const float *sfa_row = sfa_ring + j * TN + wg * COLS;
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(b * TN + wg * COLS);
                uint32_t r[2][32];
                tmem_ld32(taddr, r[0]);
                tmem_ld_wait_regs32(r[0]);
#pragma unroll
                for (int c = 0; c < COLS / 32; ++c) {
                    if (c + 1 < COLS / 32) tmem_ld32(taddr + (c + 1) * 32, r[(c + 1) & 1]);
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        // four token columns: their A scales (broadcast from shared memory) times sb
                        const float4 sa4 = *reinterpret_cast<const float4 *>(sfa_row + c * 32 + v * 4);
                        const float2 s01 = __fmul2_rn(make_float2(sa4.x, sa4.y), make_float2(sb, sb));
                        const float2 s23 = __fmul2_rn(make_float2(sa4.z, sa4.w), make_float2(sb, sb));
                        const int e = c * 32 + v * 4;
                        const float2 a01 = __ffma2_rn(make_float2(__uint_as_float(r[c & 1][v * 4]),
                                                                  __uint_as_float(r[c & 1][v * 4 + 1])),
                                                      s01, make_float2(acc[e], acc[e + 1]));
                        const float2 a23 = __ffma2_rn(make_float2(__uint_as_float(r[c & 1][v * 4 + 2]),
                                                                  __uint_as_float(r[c & 1][v * 4 + 3])),
                                                      s23, make_float2(acc[e + 2], acc[e + 3]));
                        acc[e] = a01.x;
                        acc[e + 1] = a01.y;
                        acc[e + 2] = a23.x;
                        acc[e + 3] = a23.y;
                    }
                    if (c + 1 < COLS / 32) tmem_ld_wait_regs32(r[(c + 1) & 1]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_relaxed(&tempty[b]);
            }
            if (!ok) break;
            if (S == 1) {
                if (do_c) {
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(c_full, ctile & 1, ctx));
                    ++ctile;
                    if (!ok) break;
                }
                // direct epilogue: D[g][m0+m][n0+n] for the tile's token rows; a warp stores 32
                // consecutive columns of one token row per instruction; C comes from the tile
                // TMA prefetched at tile start ([m][n] in shared memory: conflict-free reads)
                if (n0 + n < p.N) {
                    const size_t base = (static_cast<size_t>(g) * p.M + m0) * p.N + n0 + n;
#pragma unroll
                    for (int e = 0; e < COLS; ++e) {
                        const int m = wg * COLS + e;
                        if (m < rows) {
                            const float cv = do_c ? __bfloat162float(c_tile[m * 128 + n]) : 0.f;
                            p.d[base + static_cast<size_t>(m) * p.N] = __float2bfloat16_rn(acc[e] + cv);
                        }
                    }
                }
            }
        }
    }

    if (S > 1) {
        // ---------------- split-K reduction through distributed shared memory ----------------
        // The cluster's one tile is done: the operand ring is reused for this CTA's fp32 partial,
        // laid out [TN token rows][128 weight rows] (each math thread owns one weight row).
        __syncwarp();
        tc_fence_before();
        __syncthreads();
        float *red = reinterpret_cast<float *>(smem + L::OFF_W);
        if (warp >= 4) {
            const int n = (warp & 3) * 32 + lane;
            const int wg = (warp - 4) >> 2;
#pragma unroll
            for (int i = 0; i < COLS; ++i) red[(wg * COLS + i) * 128 + n] = acc[i];
        }
        __syncwarp();
        cluster_sync();
        int g_, m0_, n0_;
        const int trows = tile_rows(cid, g_, m0_, n0_);
        // CTA `rank` owns weight rows [rank·R, rank·R + R) of the tile, R = 128/S: a thread sums
        // groups of 4 consecutive weight rows of one token row over the S partials; all loads
        // of a thread (up to 4 items) are issued before any is used.
        const int R = 128 / S;
        const int groups = R / 4;
        const int items = trows * groups;
        const uint32_t red_local = smem_u32(red);
        for (int base_it = 0; base_it < items; base_it += 4 * static_cast<int>(blockDim.x)) {
            float4 sum[4];
            float4 cvals[4];
            bool live[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int itm = base_it + u * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
                live[u] = itm < items;
                sum[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                cvals[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (!live[u]) continue;
                const int m = itm / groups;
                const int nn = static_cast<int>(rank) * R + (itm % groups) * 4;
                const uint32_t off = static_cast<uint32_t>((m * 128 + nn) * 4);
                for (int src = 0; src < S; ++src) {
                    const float4 v = ld_shared_cluster_v4(mapa_shared(red_local + off, src));
                    sum[u].x += v.x;
                    sum[u].y += v.y;
                    sum[u].z += v.z;
                    sum[u].w += v.w;
                }
                const int col = n0_ + nn;
                if (p.has_c && col < p.N) {
                    const size_t o = (static_cast<size_t>(g_) * p.M + m0_ + m) * p.N + col;
                    const uint2 cv = *reinterpret_cast<const uint2 *>(p.c + o);
                    const __nv_bfloat162 c01 = *reinterpret_cast<const __nv_bfloat162 *>(&cv.x);
                    const __nv_bfloat162 c23 = *reinterpret_cast<const __nv_bfloat162 *>(&cv.y);
                    cvals[u] = make_float4(__bfloat162float(c01.x), __bfloat162float(c01.y), __bfloat162float(c23.x),
                                           __bfloat162float(c23.y));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (!live[u]) continue;
                const int itm = base_it + u * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
                const int m = itm / groups;
                const int nn = static_cast<int>(rank) * R + (itm % groups) * 4;
                const int col = n0_ + nn;
                if (col >= p.N) continue;                      // N % 8 == 0: a group of 4 is in or out
                const size_t o = (static_cast<size_t>(g_) * p.M + m0_ + m) * p.N + col;
                __nv_bfloat162 h01 = __floats2bfloat162_rn(sum[u].x + cvals[u].x, sum[u].y + cvals[u].y);
                __nv_bfloat162 h23 = __floats2bfloat162_rn(sum[u].z + cvals[u].z, sum[u].w + cvals[u].w);
                uint2 w;
                w.x = *reinterpret_cast<uint32_t *>(&h01);
                w.y = *reinterpret_cast<uint32_t *>(&h23);
                *reinterpret_cast<uint2 *>(p.d + o) = w;
            }
        }
        __syncwarp();                                      // lanes left the loop at different trips
        cluster_sync();                                    // peers may still read this CTA's partial
    } else {
        __syncwarp();
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
#endif
}

}  // namespace dg
