// dg_gemm_splitk.cuh — FP8 block-scaled NT GEMM for few rows (decode): swapped operands and a
// split-K over a thread-block cluster whose partials meet in distributed shared memory, sm_100a.
//
// Same result as dg_gemm.cuh, D = C + A·Bᵀ with per-128-K-block promotion (likun.im/craft/
// deepgemm §一; aitangshan.cn/news/1491278 技术原理 §4), for layouts whose row count per group
// is small (the decode shapes and the masked MoE layout, likun.im §二 masked_m). With so few
// rows the GEMM streams the weights B from HBM; the kernel is laid out for that:
//
//   * operands swapped (as in dg_gemm_swap.cuh): the tensor core computes P_kbᵀ = B_tile · A_kbᵀ
//     with the 128 weight rows of a tile on the MMA's M side (TMEM lanes) and TN token rows on
//     its N side (TMEM columns); sfb is one scalar per (tile, K block), sfa a per-column factor;
//   * split-K over a cluster of S CTAs (S in {1, 2, 3, 4, 6, 8, 16}): every CTA of the cluster
//     works on the same tile, CTA r on K blocks [Kb·r/S, Kb·(r+1)/S). The clusters walk the
//     tiles persistently (tile cid, cid + #clusters, ...). At the end of a tile each CTA pushes
//     its fp32 partial, row slice by row slice, into the shared memory of the CTA that reduces
//     that slice (distributed shared memory stores, then each thread's release arrive on the
//     reducer's mbarrier), so CTA j receives its rows [8·floor(16j/S), 8·floor(16(j+1)/S)) of
//     all S partials, sums them in rank order (deterministic), adds C and writes D. No global
//     workspace, no flags: the partials stay on chip;
//   * one tcgen05.commit per K block, from two issuing threads when the stage count is even.
//     A commit holds back the MMAs its thread issues after it until the committed ones are
//     done: four M=128 MMAs and their commit take ~800 cycles whatever N is when one thread
//     issues everything. With the even and the odd K blocks on two threads, each owning its
//     stages and TMEM buffers, the other thread's MMAs keep the tensor pipe busy meanwhile.
//     (An odd stage count keeps one issuer: a stage shared by both could see one issuer wait
//     on a full barrier a phase early.)
//
// CTA layout: warps 0 and 2 TMA producers (weights and activations on two threads each, the A
// scales on four), warps 1 and 3 the tcgen05.mma issuers (kind::f8f6f4, M = 128, N = TN, even
// and odd K blocks; warp 1 also allocates TMEM), warps 4-11 two math warpgroups (thread =
// weight row, registers = its warpgroup's TN/2 token columns), which also push, reduce and
// store.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_gemm_swap.cuh"
#include "dg_ptx.cuh"

namespace dg {

__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// 4-byte store into the shared memory of a CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Arrive (release, cluster scope) on an mbarrier of any CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote_release(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// mbar_wait with cluster-scope acquire: the phase was completed by other CTAs' writes.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, WaitCtx *ctx) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_acq_cluster(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    volatile int *abort = &ctx->abort;
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_acq_cluster(a, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > ctx->limit_ns) {
            report_error(ctx->err, ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

template <int TN, int STAGES>
struct SplitLayout {
    static_assert(TN == 64 || TN == 128, "token tile");
    static constexpr int NWG = 2;
    static constexpr int COLS = TN / NWG;                    // token columns per math warpgroup
    static constexpr int THREADS = 128 + 128 * NWG;
    static constexpr int W_BYTES = 128 * BK;
    static constexpr int X_BYTES = TN * BK;
    static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
    static constexpr int NBUF = 512 / TN;                    // TMEM buffers of TN columns
    static constexpr int KG = 1;                             // K blocks per commit
    static constexpr int SFS = TN == 64 ? 16 : 8;            // A-scale ring (power of two)
    static constexpr int RECV_ROWS = 144;                   // S x ceil(16/S) x 8 for S in {1,2,3,4,6,8,16}
    static constexpr int RECV_BYTES = RECV_ROWS * TN * 4;    // S slices of this CTA's rows x TN fp32
    static constexpr int CHUNKS_MAX = 16 * TN / 256;         // reduce chunks per math thread (S = 1)
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_RECV = OFF_X + STAGES * X_BYTES;
    static constexpr int OFF_SFA = OFF_RECV + RECV_BYTES;
    static constexpr int OFF_BAR = OFF_SFA + SFS * TN * 4;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 2 * SFS + 2;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx));
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(STAGES >= KG, "a commit group needs distinct stages");
    static_assert(OFF_X % 1024 == 0 && OFF_RECV % 1024 == 0 && OFF_SFA % 16 == 0, "aligned tiles");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

template <int TN, int STAGES, int KIND>
__global__ void __launch_bounds__(SplitLayout<TN, STAGES>::THREADS, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_sfa, const SwapParams p) {
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    using L = SplitLayout<TN, STAGES>;
    constexpr int NBUF = L::NBUF;
    constexpr int COLS = L::COLS;
    constexpr int KG = L::KG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *sfa_full = tempty + NBUF;
    uint64_t *sfa_empty = sfa_full + L::SFS;
    uint64_t *recv_full = sfa_empty + L::SFS;    // every math thread of the S CTAs has pushed its row
    uint64_t *send_ok = recv_full + 1;           // every reducer has read this CTA's last push
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    const float *sfa_ring = reinterpret_cast<const float *>(smem + L::OFF_SFA);
    const float *recv = reinterpret_cast<const float *>(smem + L::OFF_RECV);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = static_cast<int>(cluster_nctarank());
    const int rank = static_cast<int>(cluster_ctarank());
    const int cid = static_cast<int>(cluster_id_x());
    const int nclusters = static_cast<int>(cluster_count_x());
    pdl_launch_dependents();
    if (S > 16 || S > p.Kb || S * ((16 + S - 1) / S) * 8 > L::RECV_ROWS) {   // launch contract (host)
        if (threadIdx.x == 0) report_error(p.err, ERR_DATA);
        return;                                            // every CTA of the cluster leaves here
    }
    // the tile's 16 groups of 8 weight rows are dealt out to the S CTAs: CTA j reduces rows
    // [row0(j), row0(j + 1)), row0(j) = 8·floor(16j/S)
    auto row0 = [S](int j) { return 8 * ((16 * j) / S); };
    const int r0 = row0(rank);
    const int R = row0(rank + 1) - r0;                     // weight rows this CTA reduces
    const int kb0 = p.Kb * rank / S, kb1 = p.Kb * (rank + 1) / S;
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
            mbar_init(&sfa_empty[j], 4 * L::NWG);
        }
        mbar_init(recv_full, static_cast<uint32_t>(2 * S * R));   // one arrive per pushing thread
        mbar_init(send_ok, static_cast<uint32_t>(S));
        ctx->abort = 0;
        ctx->err = p.err;
        ctx->limit_ns = p.timeout_ns;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_sfa);
    }
    if (warp == 1) {
        tmem_alloc(&ctx->tmem_base, 512);
        tmem_relinquish();
    }
    pdl_wait();
    const SwapTiles<TN, KIND> tiles(p);
    if (threadIdx.x == 0) {
        if (KIND == KIND_MASKED && blockIdx.x == 0)
            for (int gg = 0; gg < p.G; ++gg)
                if (__ldg(p.masked_m + gg) > p.M) report_error(p.err, ERR_DATA);
    }
    tc_fence_before();
    cluster_sync();                                        // barriers of every CTA initialised
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;
    volatile int *abort_flag = &ctx->abort;

    if (warp < 4) {
        // TMA producers: lanes 0 and 16 of warps 0 (weights) and 2 (activations), even and odd
        // K blocks; lanes 8 and 24 of warps 0 and 2 (A scales), K block mod 4.
        const bool is_producer = (warp == 0 || warp == 2) && (lane & 7) == 0;
        const int stream = !is_producer ? -1 : ((lane & 15) == 0 ? warp >> 1 : 2);
        const uint32_t parity = static_cast<uint32_t>(stream == 2 ? 2 * (warp >> 1) + (lane >> 4) : lane >> 4);
        const uint32_t nlanes = stream == 2 ? 4u : 2u;
        if (stream >= 0) {
            const uint64_t pol = stream == 0 ? l2_policy_evict_first() : l2_policy_evict_last();
            uint32_t it = 0;
            for (int tile = cid; tile < tiles.count && !*abort_flag; tile += nclusters) {
                int tg, tm0, tn0;
                tiles.coords(tile, tg, tm0, tn0);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
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
            static_assert(KG == 1, "one commit per K block");
            const bool two = STAGES % 2 == 0 && NBUF % 2 == 0 && !p.one_issuer;
            const uint32_t mine = warp == 1 ? 0u : 1u;
            constexpr uint32_t IDESC = idesc_f8_e4m3_f32<128, TN>();
            uint32_t it = 0;
            bool ok = true;
            for (int tile = cid; tile < tiles.count && ok; tile += nclusters) {
                int pending = 0;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
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
                    if (++pending == KG || kb + 1 == kb1) {
                        for (uint32_t q = it + 1 - pending; q <= it; ++q) umma_commit(&empty[q % STAGES]);
                        for (uint32_t q = it + 1 - pending; q <= it; ++q) umma_commit(&tfull[q % NBUF]);
                        pending = 0;
                    }
                }
            }
        }
    } else {
        // ---------------- math warpgroups: promotion, push, reduce, store ----------------
        const int wg = (warp - 4) >> 2;                    // token columns [wg·COLS, wg·COLS + COLS)
        const int q = warp & 3;                            // TMEM lane quadrant = weight rows 32q..
        const int n = q * 32 + lane;                       // this thread's weight row in the tile
        const int tid = threadIdx.x - 128;                 // 0..255
        // push target of row n: the CTA j whose rows hold it. A receive buffer is laid out
        // [source][token][row], rows fastest, so that a warp's store of one token column is 32
        // consecutive rows: at most a few contiguous runs over the cluster network
        const int dst = ((n / 8) * S + S - 1) / 16;
        const int dst_r0 = row0(dst), dst_R = row0(dst + 1) - dst_r0;
        const uint32_t push_addr = mapa_shared(smem_u32(smem + L::OFF_RECV) +
                                                   static_cast<uint32_t>(((rank * TN + wg * COLS) * dst_R + n - dst_r0) * 4),
                                               static_cast<uint32_t>(dst));
        const uint32_t push_step = static_cast<uint32_t>(dst_R * 4);          // next token
        const uint32_t push_bar = mapa_shared(smem_u32(recv_full), static_cast<uint32_t>(dst));
        float *push_local = reinterpret_cast<float *>(smem + L::OFF_RECV) + wg * COLS * 128 + n;   // S = 1
        const int nchunks = (R / 8) * TN;                  // reduce outputs: 8 weight rows x 1 token
        uint32_t it = 0;
        bool ok = true;
        float acc[COLS];
        int ti = 0;
        for (int tile = cid; tile < tiles.count; tile += nclusters, ++ti) {
            int g, m0, n0;
            const int rows = tiles.coords(tile, g, m0, n0);
            const int nt = n0 / 128;
            // C for this CTA's reduce outputs, read now so that the load hides behind the K loop
            uint4 cv[L::CHUNKS_MAX];
#pragma unroll
            for (int k = 0; k < L::CHUNKS_MAX; ++k) {
                cv[k] = make_uint4(0, 0, 0, 0);
                const int ch = tid + k * 256;
                if (p.has_c && ch < nchunks) {
                    const int m = ch % TN, col = n0 + r0 + (ch / TN) * 8;
                    if (m < rows && col < p.N)
                        cv[k] = __ldg(reinterpret_cast<const uint4 *>(p.c + (static_cast<size_t>(g) * p.M + m0 + m) * p.N + col));
                }
            }
#pragma unroll
            for (int i = 0; i < COLS; ++i) acc[i] = 0.f;
            const float *sfb_col = p.sfb + (static_cast<size_t>(g) * p.Nb + nt) * p.Kb;
            float sb_win = kb0 + lane < kb1 ? __ldg(sfb_col + kb0 + lane) : 0.f;
            float sb_nxt = kb0 + 32 + lane < kb1 ? __ldg(sfb_col + kb0 + 32 + lane) : 0.f;
            const int nk = kb1 - kb0;
            auto fold = [&](const uint32_t (&rr)[32], int c, const float *sfa_row, float sb) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
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
            auto sb_of = [&](int i) {
                if ((i & 31) == 0 && i > 0) {
                    sb_win = sb_nxt;
                    sb_nxt = kb0 + i + 32 + lane < kb1 ? __ldg(sfb_col + kb0 + i + 32 + lane) : 0.f;
                }
                return __shfl_sync(0xFFFFFFFFu, sb_win, i & 31);
            };
            auto ready = [&](uint32_t itx) {
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
                // next block's load is in flight while the current one is folded in
                uint32_t r0[32], r1[32];
                auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32], int i) {
                    const float sb = sb_of(i);
                    if (!ok) return;
                    tmem_ld_wait_regs32(cur);
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
            if (S == 1) {
                // the whole K range is this CTA's: its rows go to its own receive buffer with
                // plain stores, and a barrier of the math threads orders them before the reads
                if (ok) {
#pragma unroll
                    for (int e = 0; e < COLS; ++e) push_local[e * 128] = acc[e];
                }
                ok = named_barrier_and(3, 128 * L::NWG, ok);
            } else {
                // push: once every reducer has read this CTA's previous slices (send_ok), this
                // thread's row goes to its reducer, one 4-byte store per token, and the thread's
                // release arrive on the reducer's barrier orders them before the reducer's reads
                if (ok && ti > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(send_ok, (ti - 1) & 1, ctx));
                if (ok) {
#pragma unroll
                    for (int e = 0; e < COLS; ++e) st_cluster_f32(push_addr + e * push_step, acc[e]);
                    if (!(p.test_skip_release && blockIdx.x == 0 && warp == 4 && ti == 0))
                        mbar_arrive_remote_release(push_bar);
                }
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(recv_full, ti & 1, ctx));
            }
            // reduce: rows [r0, r0 + R) of the tile, S partials in rank order, + C
            if (ok) {
#pragma unroll
                for (int k = 0; k < L::CHUNKS_MAX; ++k) {
                    const int ch = tid + k * 256;
                    if (ch >= nchunks) break;
                    const int m = ch % TN, lr0 = (ch / TN) * 8;
                    const int col = n0 + r0 + lr0;
                    float sum[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) sum[e] = 0.f;
                    for (int src = 0; src < S; ++src) {
                        const float4 *base = reinterpret_cast<const float4 *>(recv + (src * TN + m) * R + lr0);
                        const float4 lo = base[0], hi = base[1];
                        sum[0] += lo.x; sum[1] += lo.y; sum[2] += lo.z; sum[3] += lo.w;
                        sum[4] += hi.x; sum[5] += hi.y; sum[6] += hi.z; sum[7] += hi.w;
                    }
                    if (m < rows && col < p.N) {
                        const uint32_t cw[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 cf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&cw[e]));
                            const __nv_bfloat162 h = __floats2bfloat162_rn(sum[2 * e] + cf.x, sum[2 * e + 1] + cf.y);
                            o[e] = *reinterpret_cast<const uint32_t *>(&h);
                        }
                        *reinterpret_cast<uint4 *>(p.d + (static_cast<size_t>(g) * p.M + m0 + m) * p.N + col) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            // every math thread's reads of the receive buffer are done: every source may push again
            ok = named_barrier_and(2, 128 * L::NWG, ok);
            if (S > 1 && threadIdx.x == 128 && ok && tile + nclusters < tiles.count)
                for (int j = 0; j < S; ++j) mbar_arrive_remote_release(mapa_shared(smem_u32(send_ok), static_cast<uint32_t>(j)));
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync();                                        // no CTA leaves while a peer may write to it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
#endif
}

}  // namespace dg
