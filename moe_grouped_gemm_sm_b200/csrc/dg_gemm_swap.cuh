// dg_gemm_swap.cuh — FP8 block-scaled NT GEMM for few rows (decode): swapped operands and a
// stream-K split of the work over every SM, sm_100a.
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
//   * stream-K: the (tile, K block) units of all active tiles, in order, are cut into
//     gridDim.x equal runs, one per CTA (one CTA per SM), so every SM streams the same number
//     of weight bytes whatever the tile count. A CTA's run is a sequence of segments, each
//     a range of K blocks of one tile. The CTA whose run holds a tile's first K block owns the
//     tile: the other CTAs that cover part of it (higher-numbered, and for each of them it is
//     the first segment of its run, done before anything else) leave fp32 partials in a
//     global workspace, and the owner, for which the tile is the last segment of its run,
//     adds them to its own in CTA order (a fixed order: results are deterministic), adds C and
//     writes D (bf16, round to nearest even). Flags in the workspace tell the owner when a
//     partial is complete. A flag holds the ticket of the launch that wrote it: every launch
//     reads the workspace's epoch word at its start and uses epoch + 1 as its ticket, and the
//     last CTA to finish stores that ticket back into the epoch word. A flag left over from an
//     earlier launch (one whose owner gave up after a bounded wait, say) therefore never
//     matches, no flag needs clearing, and CUDA-graph replays stay valid;
//   * a deep TMA ring (5-8 stages of the 16 KB weight tile) keeps enough bytes in flight.
//
// CTA layout: warps 0 and 2 TMA producers (weights and activations on two threads each, the A
// scales on four), warps 1 and 3 the tcgen05.mma issuers (kind::f8f6f4, M = 128, N = TN), one
// thread each for the even and the odd K blocks (warp 1 also allocates TMEM), warps 4-11 two
// math warpgroups (thread = weight row, registers = its warpgroup's TN/2 token columns).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_gemm.cuh"
#include "dg_ptx.cuh"

namespace dg {

struct SwapParams {
    int M;            // rows per group (dense: M; masked: M_max)
    int N, K, G;
    int Kb, Nb;       // K/128, ceil(N/128)
    int ld_sfa;       // pad4(M)
    int n_tiles;      // ceil(N/128)
    int m_tiles;      // ceil(M/TN): token tiles per group
    int has_c;
    const float *sfb;
    const int32_t *masked_m;   // masked layout only
    const __nv_bfloat16 *c;
    __nv_bfloat16 *d;
    float *ws;        // stream-K partials, [gridDim.x][TN][128] fp32
    int *flags;       // [gridDim.x] partial flags, each the ticket of the launch that wrote it
    unsigned *epoch;  // [2]: the last finished launch's ticket, and the count of finished CTAs
    int *err;
    uint64_t timeout_ns;
    // failure tests only: 2 = the cluster kernel's CTA 0, warp 4 withholds its first push
    // arrive; 3 = the stream-K kernel's odd-numbered CTAs withhold their partial flags
    int test_skip_release;
    int one_issuer;   // experiments: warp 1 issues every K block (no second issuer)
};

template <int TN, int STAGES>
struct SwapLayout {
    static_assert(TN == 64 || TN == 128, "token tile");
    static constexpr int NWG = 2;                            // math warpgroups: two warps per SM sub-partition
    static constexpr int COLS = TN / NWG;                    // token columns per math warpgroup (32 or 64)
    static constexpr int THREADS = 128 + 128 * NWG;
    static constexpr int W_BYTES = 128 * BK;                 // weight tile: 128 rows x 128 B
    static constexpr int X_BYTES = TN * BK;                  // activation tile: TN rows x 128 B
    static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
    static constexpr int NBUF = 512 / TN;                    // TMEM buffers of TN columns
    static constexpr int KG = 1;                             // K blocks per commit (see the MMA issuer)
    static constexpr int SFS = 16;                           // A-scale ring (a power of two), own barriers
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_SFA = OFF_X + STAGES * X_BYTES;
    static constexpr int OFF_C = OFF_SFA + SFS * TN * 4;        // C tile [TN][128] bf16 (tile owner)
    static constexpr int C_BYTES = TN * 128 * 2;
    static constexpr int OFF_BAR = OFF_C + C_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 2 * SFS + 2;
    static constexpr int PART_BYTES = TN * 128 * 4;          // one fp32 partial of a tile
    static constexpr int MAX_PARTS = STAGES * STAGE_BYTES / PART_BYTES;   // fit the idle ring
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(OFF_X % 1024 == 0 && OFF_SFA % 16 == 0 && OFF_C % 128 == 0, "aligned tiles");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

// The active tiles, in the order the stream-K units run through them: for each group g, its
// token tiles mt < ceil(rows_g / TN) (rows_g = M, or masked_m[g] clamped to [0, M]), and for
// each token tile the weight tiles nt, nt fastest (consecutive tiles share the activations).
template <int TN, int KIND>
struct SwapTiles {
    const SwapParams &p;
    int count;
    __device__ explicit SwapTiles(const SwapParams &pp) : p(pp) {
        if (KIND == KIND_MASKED) {
            count = 0;
            for (int g = 0; g < p.G; ++g) count += (rows_of(g) + TN - 1) / TN * p.n_tiles;
        } else {
            count = p.m_tiles * p.n_tiles;
        }
    }
    __device__ int rows_of(int g) const {
        if (KIND != KIND_MASKED) return p.M;
        const int mm = __ldg(p.masked_m + g);
        return mm < 0 ? 0 : (mm > p.M ? p.M : mm);
    }
    // tile a -> group g, first token row m0, first weight row n0; returns the token rows of the
    // tile that exist (>= 1 for a < count)
    __device__ int coords(int a, int &g, int &m0, int &n0) const {
        g = 0;
        if (KIND == KIND_MASKED) {
            while (g < p.G - 1) {
                const int cnt = (rows_of(g) + TN - 1) / TN * p.n_tiles;
                if (a < cnt) break;
                a -= cnt;
                ++g;
            }
        }
        n0 = (a % p.n_tiles) * 128;
        m0 = (a / p.n_tiles) * TN;
        return min(TN, rows_of(g) - m0);
    }
};

// A CTA's run of units [u0, u1) out of U = tiles · Kb (unit u = K block u % Kb of tile u / Kb);
// the CTA holding unit u is cta_of(u). The units are cut over the first P CTAs of the grid
// (the others get empty runs), P small enough that every run holds at least
// ceil((Kb - 1) / max_parts) units: then no tile is spread over more than max_parts + 1 runs,
// i.e. no owner has more than max_parts partials to add (and no run is empty, which the
// masked layout, with fewer units than the grid was sized for, would otherwise allow). Runs
// are walked segment by segment: segment() gives the tile and the K-block range
// [kb_begin, kb_end) of the segment starting at unit u.
struct StreamK {
    long long U, u0, u1;
    int Kb, P;
    __device__ StreamK(int tiles, int kb, int c, int grid, int max_parts) : Kb(kb) {
        U = static_cast<long long>(tiles) * kb;
        const long long min_run = kb > 1 ? (kb - 1 + max_parts - 1) / max_parts : 1;
        const long long pmax = U / min_run > 1 ? U / min_run : 1;
        P = pmax < grid ? static_cast<int>(pmax) : grid;
        u0 = c < P ? U * c / P : U;
        u1 = c < P ? U * (c + 1) / P : U;
    }
    __device__ int cta_of(long long u) const { return static_cast<int>(((u + 1) * P - 1) / U); }
    __device__ void segment(long long u, int &tile, int &kb_begin, int &kb_end) const {
        tile = static_cast<int>(u / Kb);
        kb_begin = static_cast<int>(u - static_cast<long long>(tile) * Kb);
        const long long rest = u1 - u;
        kb_end = rest < Kb - kb_begin ? kb_begin + static_cast<int>(rest) : Kb;
    }
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
    uint64_t *sfa_empty = sfa_full + L::SFS;
    uint64_t *c_full = sfa_empty + L::SFS;
    uint64_t *fix_full = c_full + 1;
    const __nv_bfloat16 *c_tile = reinterpret_cast<const __nv_bfloat16 *>(smem + L::OFF_C);
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    const float *sfa_ring = reinterpret_cast<const float *>(smem + L::OFF_SFA);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_launch_dependents();
    // prologue (overlaps the previous kernel's tail): barriers, descriptors, TMEM
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4 * L::NWG);
        }
        for (int j = 0; j < L::SFS; ++j) {
            mbar_init(&sfa_full[j], 1);
            mbar_init(&sfa_empty[j], 4 * L::NWG);   // one arrive per math warp
        }
        mbar_init(c_full, 1);
        mbar_init(fix_full, 1);
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
    pdl_wait();   // from here on global memory may be read and written
    __shared__ int ticket_smem;
    if (threadIdx.x == 0) ticket_smem = streamk_ticket(p.epoch);
    if (KIND == KIND_MASKED && blockIdx.x == 0 && threadIdx.x == 0) {
        for (int gg = 0; gg < p.G; ++gg)
            if (__ldg(p.masked_m + gg) > p.M) report_error(p.err, ERR_DATA);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;
    const int ticket = ticket_smem;
    volatile int *abort_flag = &ctx->abort;
    const SwapTiles<TN, KIND> tiles(p);
    const StreamK sk(tiles.count, p.Kb, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x), L::MAX_PARTS);

    if (warp < 4) {
        // TMA producers. One thread's bulk copies are served one after another, so the weights
        // and the activations each get two threads (lanes 0 and 16 of warps 0 and 2, even and
        // odd K blocks) and the small A-scale copies four (lanes 0, 8, 16, 24 of warp 3, K block
        // mod 4). The weight thread of a K block arms its stage. All wait on the ring's "empty"
        // barriers.
        const bool is_producer = (warp == 0 || warp == 2) && (lane & 7) == 0;
        const int stream = !is_producer ? -1 : ((lane & 15) == 0 ? warp >> 1 : 2);
        // weights/activations: K block parity = lane / 16; A scales (lanes 8 and 24 of warps 0
        // and 2): K block mod 4 = 2·(warp / 2) + lane / 16
        const uint32_t parity = static_cast<uint32_t>(stream == 2 ? 2 * (warp >> 1) + (lane >> 4) : lane >> 4);
        const uint32_t nlanes = stream == 2 ? 4u : 2u;
        if (stream >= 0) {
            // the weights are read once: evict them first; activations and A scales are read
            // again by the CTAs working on other weight tiles: keep them
            const uint64_t pol = stream == 0 ? l2_policy_evict_first() : l2_policy_evict_last();
            uint32_t it = 0;
            for (long long u = sk.u0; u < sk.u1 && !*abort_flag;) {
                int tile, kbs, kbe, tg, tm0, tn0;
                sk.segment(u, tile, kbs, kbe);
                u += kbe - kbs;
                tiles.coords(tile, tg, tm0, tn0);
                for (int kb = kbs; kb < kbe; ++kb, ++it) {
                    if (it % nlanes != parity) continue;
                    const int s = it % STAGES;
                    const int j = it % L::SFS;
                    if (!mbar_wait(stream == 2 ? &sfa_empty[j] : &empty[s],
                                   stream == 2 ? ((it / L::SFS) & 1) ^ 1 : ((it / STAGES) & 1) ^ 1, ctx))
                        break;
                    if (stream == 2) {
                        mbar_arrive_expect_tx(&sfa_full[j], TN * 4);
                        float *sf = reinterpret_cast<float *>(smem + L::OFF_SFA) + j * TN;
                        if (KIND == KIND_MASKED)
                            tma_load_3d_hint(&tm_sfa, &sfa_full[j], sf, tm0, kb, tg, pol);
                        else
                            tma_load_2d_hint(&tm_sfa, &sfa_full[j], sf, tm0, kb, pol);
                    } else if (stream == 0) {
                        mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
                        tma_load_3d_hint(&tm_w, &full[s], smem + L::OFF_W + s * L::W_BYTES, kb * BK, tn0, tg, pol);
                    } else if (KIND == KIND_MASKED) {
                        tma_load_3d_hint(&tm_x, &full[s], smem + L::OFF_X + s * L::X_BYTES, kb * BK, tm0, tg, pol);
                    } else {
                        tma_load_2d_hint(&tm_x, &full[s], smem + L::OFF_X + s * L::X_BYTES, kb * BK, tm0, pol);
                    }
                }
            }
        } else if ((warp == 1 || (warp == 3 && STAGES % 2 == 0 && NBUF % 2 == 0 && !p.one_issuer)) && lane == 0) {
            // ---------------- MMA issuers: warp 1 even K blocks, warp 3 odd ones ----------------
            // (a commit holds back only the MMAs its own thread issues after it, so the other
            // issuer keeps the tensor pipe busy while one waits; each has its own TMEM buffers)
            // two issuers need even stage and buffer counts (each issuer then owns its stages
            // and buffers and waits on their barriers phase after phase); odd counts keep one
            static_assert(L::KG == 1, "one commit per K block");
            const bool two = STAGES % 2 == 0 && NBUF % 2 == 0 && !p.one_issuer;
            const uint32_t mine = warp == 1 ? 0u : 1u;
            constexpr uint32_t IDESC = idesc_f8_e4m3_f32<128, TN>();
            // one commit per K block (KG = 1): grouping commits, which saves tensor-pipe drains,
            // measured slower here, where the run is bandwidth-bound and the tile tails matter
            uint32_t it = 0;
            bool ok = true;
            for (long long u = sk.u0; u < sk.u1 && ok;) {
                int tile, kbs, kbe;
                sk.segment(u, tile, kbs, kbe);
                u += kbe - kbs;
                int pending = 0;
                for (int kb = kbs; kb < kbe; ++kb, ++it) {
                    if (two && (it & 1u) != mine) continue;
                    const int s = it % STAGES;
                    const int b = it % NBUF;
                    ok = mbar_wait(&full[s], (it / STAGES) & 1, ctx) && mbar_wait(&tempty[b], ((it / NBUF) & 1) ^ 1, ctx);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t wd = sdesc_k_sw128(smem_u32(smem + L::OFF_W + s * L::W_BYTES));
                    const uint64_t xd = sdesc_k_sw128(smem_u32(smem + L::OFF_X + s * L::X_BYTES));
                    const uint32_t dt = tmem_base + static_cast<uint32_t>(b * TN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) umma_f8(dt, wd + 2 * k, xd + 2 * k, IDESC, k > 0 ? 1u : 0u);
                    if (++pending == L::KG || kb + 1 == kbe) {
                        for (uint32_t q = it + 1 - pending; q <= it; ++q) umma_commit(&empty[q % STAGES]);
                        for (uint32_t q = it + 1 - pending; q <= it; ++q) umma_commit(&tfull[q % NBUF]);
                        pending = 0;
                    }
                }
            }
        }
    } else {
        // ---------------- math warpgroups: promotion, partials, tile epilogue ----------------
        // Every math thread walks the same segments and meets the same named barriers, even
        // after a wait has given up (then the work is skipped), so no barrier is left waiting.
        const int wg = (warp - 4) >> 2;                    // token columns [wg·COLS, wg·COLS + COLS)
        const int q = warp & 3;                            // TMEM lane quadrant = weight rows 32q..
        const int n = q * 32 + lane;                       // this thread's weight row in the tile
        const int c_self = static_cast<int>(blockIdx.x);
        uint32_t it = 0, ctile = 0;
        bool ok = true;
        float acc[COLS];
        for (long long u = sk.u0; u < sk.u1;) {
            int tile, kbs, kbe, g, m0, n0;
            sk.segment(u, tile, kbs, kbe);
            u += kbe - kbs;
            const int rows = tiles.coords(tile, g, m0, n0);
            const bool owner = kbs == 0;                   // this CTA holds the tile's first K block
            const int nt = n0 / 128;
            const bool do_c = owner && p.has_c;
            if (do_c) {
                // the previous tile's C has been read by every math thread before it is replaced
                // by the next TMA write (each reader's proxy fence orders its generic reads
                // before that async-proxy write)
                fence_proxy_async_smem();
                asm volatile("bar.sync 1, %0;" ::"n"(128 * L::NWG) : "memory");
                if (threadIdx.x == 128 && ok) {
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
            float sb_win = kbs + lane < kbe ? __ldg(sfb_col + kbs + lane) : 0.f;
            float sb_nxt = kbs + 32 + lane < kbe ? __ldg(sfb_col + kbs + 32 + lane) : 0.f;
            const int nk = kbe - kbs;
            // fold one K block's partial (in registers rr) into acc: acc += P · sfa[col] · sb
            auto fold = [&](const uint32_t (&rr)[32], int c, const float *sfa_row, float sb) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    // four token columns: their A scales (broadcast from shared memory) times sb
                    const float4 sa4 = *reinterpret_cast<const float4 *>(sfa_row + c * 32 + v * 4);
                    const float2 s01 = __fmul2_rn(make_float2(sa4.x, sa4.y), make_float2(sb, sb));
                    const float2 s23 = __fmul2_rn(make_float2(sa4.z, sa4.w), make_float2(sb, sb));
                    const int e = c * 32 + v * 4;
                    const float2 a01 = __ffma2_rn(make_float2(__uint_as_float(rr[v * 4]), __uint_as_float(rr[v * 4 + 1])),
                                                  s01, make_float2(acc[e], acc[e + 1]));
                    const float2 a23 = __ffma2_rn(make_float2(__uint_as_float(rr[v * 4 + 2]), __uint_as_float(rr[v * 4 + 3])),
                                                  s23, make_float2(acc[e + 2], acc[e + 3]));
                    acc[e] = a01.x;
                    acc[e + 1] = a01.y;
                    acc[e + 2] = a23.x;
                    acc[e + 3] = a23.y;
                }
            };
            auto sb_of = [&](int i) {                      // sfb of K block kbs + i (all lanes)
                if ((i & 31) == 0 && i > 0) {
                    sb_win = sb_nxt;
                    sb_nxt = kbs + i + 32 + lane < kbe ? __ldg(sfb_col + kbs + i + 32 + lane) : 0.f;
                }
                return __shfl_sync(0xFFFFFFFFu, sb_win, i & 31);
            };
            auto ready = [&](uint32_t itx) {               // TMEM buffer and A scales of itx (warp-uniform)
                bool r = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[itx % NBUF], (itx / NBUF) & 1, ctx));
                if (r) r = __all_sync(0xFFFFFFFFu, mbar_wait(&sfa_full[itx % L::SFS], (itx / L::SFS) & 1, ctx));
                return r;
            };
            auto taddr_of = [&](uint32_t itx) {
                return tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                       static_cast<uint32_t>((itx % NBUF) * TN + wg * COLS);
            };
            auto release = [&](uint32_t itx) {
                tc_fence_before();
                fence_proxy_async_smem();   // A-scale reads before the slot's next TMA write
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_relaxed(&sfa_empty[itx % L::SFS]);
                    mbar_arrive_relaxed(&tempty[itx % NBUF]);
                }
            };
            if constexpr (COLS == 32) {
                // one 32-column TMEM load per K block, software-pipelined across K blocks: the
                // next block's load is in flight while the current block is folded in
                uint32_t r0[32], r1[32];
                auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32], int i) {
                    const float sb = sb_of(i);
                    if (!ok) return;
                    tmem_ld_wait_regs32(cur);              // block i is in registers
                    const uint32_t itn = it + 1;
                    if (i + 1 < nk) {
                        ok = ready(itn);
                        if (ok) {
                            tc_fence_after();
                            tmem_ld32(taddr_of(itn), nxt);
                        }
                    }
                    fold(cur, 0, sfa_ring + (it % L::SFS) * TN + wg * COLS, sb);
                    release(it);
                };
                if (ok && nk > 0) {
                    ok = ready(it);
                    if (ok) {
                        tc_fence_after();
                        tmem_ld32(taddr_of(it), r0);
                    }
                }
                for (int i = 0; i < nk; i += 2) {
                    step(r0, r1, i);
                    ++it;
                    if (i + 1 < nk) {
                        step(r1, r0, i + 1);
                        ++it;
                    }
                }
                if (ok) tmem_ld_wait_regs32(r0);           // nothing is left in flight
            } else {
                for (int i = 0; i < nk; ++i, ++it) {
                    const float sb = sb_of(i);
                    if (!ok) continue;
                    ok = ready(it);
                    if (!ok) continue;
                    tc_fence_after();
                    const float *sfa_row = sfa_ring + (it % L::SFS) * TN + wg * COLS;
                    const uint32_t taddr = taddr_of(it);
                    uint32_t r[2][32];
                    tmem_ld32(taddr, r[0]);
                    tmem_ld_wait_regs32(r[0]);
#pragma unroll
                    for (int c = 0; c < COLS / 32; ++c) {
                        if (c + 1 < COLS / 32) tmem_ld32(taddr + (c + 1) * 32, r[(c + 1) & 1]);
                        fold(r[c & 1], c, sfa_row, sb);
                        if (c + 1 < COLS / 32) tmem_ld_wait_regs32(r[(c + 1) & 1]);
                    }
                    release(it);
                }
            }
            if (!owner) {
                // a partial (always this CTA's first segment): [TN token rows][128 weight rows] fp32,
                // published to the owner by the CTA's flag once every math thread's stores are
                // ordered before it (gpu-scope fence, then a barrier of the math threads)
                float *ws_self = p.ws + static_cast<size_t>(c_self) * TN * 128;
                if (ok) {
#pragma unroll
                    for (int e = 0; e < COLS; ++e) __stcg(ws_self + (wg * COLS + e) * 128 + n, acc[e]);
                    __threadfence();
                }
                ok = named_barrier_and(2, 128 * L::NWG, ok);
                if (threadIdx.x == 128 && ok && !(p.test_skip_release == 3 && (c_self & 1)))
                    flag_store_release(p.flags + c_self, ticket);
                continue;
            }
            if (kbe < p.Kb) {
                // The tile's later K blocks are partials of CTAs c_self+1 .. j1 (at most
                // MAX_PARTS). Their flags are waited for (each must hold this launch's ticket),
                // the partials copied in bulk into the operand ring, idle now (this is the run's
                // last segment and its MMAs are done), and added in CTA order.
                const int j1 = sk.cta_of(static_cast<long long>(tile) * p.Kb + p.Kb - 1);
                const int nparts = j1 - c_self;
                bool got = ok && nparts <= L::MAX_PARTS;
                if (threadIdx.x == 128 && ok && !got) report_error(ctx->err, ERR_DATA);
                if (threadIdx.x == 128 && got) {
                    const uint64_t t0 = globaltimer_ns();
                    for (int jj = c_self + 1; jj <= j1 && got; ++jj) {
                        while (flag_load_acquire(p.flags + jj) != ticket) {
                            if (*abort_flag) {
                                got = false;
                                break;
                            }
                            if (globaltimer_ns() - t0 > ctx->limit_ns) {
                                report_error(ctx->err, ERR_TIMEOUT);
                                *abort_flag = 1;
                                got = false;
                                break;
                            }
                        }
                    }
                    if (got) mbar_arrive_expect_tx(fix_full, static_cast<uint32_t>(nparts) * L::PART_BYTES);
                }
                ok = named_barrier_and(2, 128 * L::NWG, got);
                float *parts = reinterpret_cast<float *>(smem + L::OFF_W);
                if (ok && warp == 4 && lane < nparts) {   // one bulk copy per lane, all in flight
                    fence_proxy_async_global();
                    bulk_load(parts + static_cast<size_t>(lane) * TN * 128,
                              p.ws + static_cast<size_t>(c_self + 1 + lane) * TN * 128, L::PART_BYTES, fix_full);
                }
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(fix_full, 0, ctx));
                if (ok) {
                    for (int k = 0; k < nparts; ++k) {
#pragma unroll
                        for (int e = 0; e < COLS; ++e) acc[e] += parts[(k * TN + wg * COLS + e) * 128 + n];
                    }
                }
            }
            if (do_c && ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(c_full, ctile & 1, ctx));
            if (do_c) ++ctile;
            if (!ok) continue;
            // tile epilogue: D[g][m0+m][n0+n] for the tile's token rows; a warp stores 32
            // consecutive columns of one token row per instruction; C comes from the tile TMA
            // loaded at the segment's start ([m][n] in shared memory: conflict-free reads)
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

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
    if (threadIdx.x == 0) {
        // the last CTA to finish publishes this launch's ticket as the epoch; the next launch
        // on the stream reads it only after this grid has completed (griddepcontrol.wait)
        __threadfence();
        if (atomicAdd(p.epoch + 1, 1u) == gridDim.x - 1) {
            p.epoch[1] = 0u;
            p.epoch[0] = static_cast<unsigned>(ticket);
            __threadfence();
        }
    }
#endif
}

}  // namespace dg
