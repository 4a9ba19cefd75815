// dg_gemm.cuh — persistent, warp-specialised FP8 block-scaled NT GEMM for sm_100a.
//
// D = C + A·Bᵀ (likun.im/craft/deepgemm §一) with block-wise scales promoted per 128-wide
// K block (aitangshan.cn/news/1491278 技术原理 §4): for every K block kb the tensor core
// produces the unscaled partial P_kb = A[:, kb]·B[:, kb]ᵀ in TMEM, and the math warps fold it
// into fp32 registers as acc += P_kb · sfa[m,kb] · sfb[n/128,kb].
//
// Two shapes of the same kernel:
//   PAIR = false  one CTA per tile of 128 rows x BN columns (tcgen05 cta_group::1, M = 128);
//   PAIR = true   a cluster of two CTAs per tile of 256 rows x BN columns (cta_group::2,
//                 M = 256): each CTA loads its 128 rows of A and half of the BN rows of B, the
//                 leader CTA issues the MMA for both, and each CTA's TMEM receives its own 128
//                 rows of the partial. Per SM this halves the B bytes that cross L2 -> SMEM.
//
// CTA layout (384 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producers of A (lanes 0 and 16: even and odd K blocks): A tile [128 x
//               128 B] into a STAGES-deep ring guarded by full/empty mbarriers (for a pair, both
//               CTAs' loads count on the leader's full barrier); they arm each stage's bytes.
//               The same thread first loads the K block's A scales into a ring of their own.
//               (A lane of a warp that waits in mbarrier.try_wait holds up the other lanes of
//               the warp: the operand loads are kept away from any lane that waits on another
//               ring's barriers.)
//   warps 1, 3  (leader only) the MMA issuers, one thread each: warp 1 issues the even K
//               blocks, warp 3 the odd ones, each tcgen05.mma kind::f8f6f4, four K=32 steps per
//               K block, into its own TMEM buffer, and commits the buffer (tfull) — to both CTAs
//               of a pair; the math warps hand the operand stage back (empty) once they have
//               seen that commit, which spares the issuer a second commit per K block. A commit
//               holds back the MMAs its thread issues after it until the committed ones are done
//               (~800 cycles per K block with one issuer, measured); MMAs of the other thread
//               keep the tensor pipe busy meanwhile. Two issuers need an
//               even number of stages and buffers: then every stage and buffer belongs to one
//               issuer, which waits on its barriers phase after phase. (With an odd count a
//               stage alternates between the issuers, and one of them could wait for a phase of
//               a full barrier while the previous phase is still open: the parity wait would
//               take the phase before that one, long complete, for it.) Odd stage counts keep
//               one issuer, warp 1, which also allocates TMEM.
//   warp 2      loads B, lanes 0 and 16 as for A (and, for contiguous pair tiles, first lists
//               the pairs once).
//   warps 4-11  two math warpgroups. Warp w reads TMEM lanes 32·(w%4)..+31 (its 32 rows);
//               warpgroup j owns columns [j·BN/2, (j+1)·BN/2). Per K block: wait for the TMEM
//               buffer, load the partial in 32-column batches (the next batch in flight while
//               the previous one is folded in as acc = fma(p, sa·sb, acc)), and release the
//               buffer as soon as the last batch is in registers, before it is folded in.
//               sfa arrives by TMA in a ring of its own (one BM-float column per K block,
//               loaded by the producer ahead of the operands), sfb one 32-K-block window per
//               lane broadcast by shuffle. Epilogue: C (prefetched by TMA at tile start) is added, the
//               result converted to bf16 (round to nearest even) into a 128-byte-swizzled slab
//               and stored by TMA.
//
// Tile order: dense and contiguous tiles are rasterised in bands of 16 128-row blocks so that
// concurrently resident CTAs share B tiles in L2. Contiguous: the expert of a 128-row block is
// grouped_layout[first row] (likun.im §二 grouped_layout; each expert's rows are padded to
// 128); pair tiles are formed inside one expert's run of blocks (a prologue scan builds the
// list in shared memory), and the peer CTA of a pair whose second block belongs to another
// expert computes but does not store. Masked: tiles are enumerated per expert over
// ceil(masked_m[g]/rows per tile) tiles only (likun.im §二 masked_m), and rows >= masked_m[g]
// are never stored.
//
// Last-wave split (dense NT): when the tiles do not fill a whole number of waves of the
// persistent grid, the main launch runs the whole waves and a second launch of the TAIL
// instantiation runs the R tiles of the last wave, each cut along K into S pieces on R·S CTAs
// (pairs) at once. The CTAs of pieces 1..S-1 write their fp32 partials to a global workspace,
// one flag per math warp; the CTA of piece 0 waits for those flags (bounded), adds the partials
// in piece order and writes D. A flag holds the ticket of the launch that wrote it (the epoch
// protocol of the stream-K kernel), so the flags never need clearing. (The split lives in its
// own instantiation because its code, present but idle in the main kernel, measurably slowed
// the main kernel's K loop.)
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

enum GemmKind : int { KIND_DENSE = 0, KIND_CONTIGUOUS = 1, KIND_MASKED = 2, KIND_KGROUPED = 3 };

constexpr int BM = 128;                 // rows per CTA (one TMEM lane per row)
constexpr int BK = 128;                 // K block = scale granularity = one 128-byte swizzle row
constexpr int GEMM_THREADS = 384;
constexpr int RASTER_BLOCKS = 16;       // rasterisation band height, in 128-row blocks
constexpr int MAX_PAIR_BLOCKS = 1024;   // contiguous pair tiles: M_sum <= 1024 x 128 rows
constexpr int MAX_KGROUPS = 511;        // K-grouped: groups whose K-block offsets fit the list area

struct GemmParams {
    int M;            // rows per group of D (dense: M, contiguous: M_sum, masked: M_max)
    int N, K, G;
    int Kb, Nb;       // K/128, ceil(N/128)
    int ld_sfa;       // pad4(M): leading dimension of the MN-major A scales
    int n_blocks;     // ceil(N/BN)
    int num_tiles;    // dense and unpaired contiguous tiles (others: derived on the device)
    int has_c;
    int cd_blocks;    // 1: C and D maps are 3D {64 columns, rows, N/64 column blocks} (one copy per slab)
    int test_skip_release;   // failure test only: warp 4 of CTA 0 skips its first TMEM release
    int one_issuer;          // experiments: warp 1 issues every K block (no second issuer)
    const float *sfa;
    const float *sfb;
    const int32_t *grouped_layout;
    const int32_t *masked_m;
    const int32_t *ks;       // K-grouped: tokens of each group (device), multiples of 128
    // last-wave split (the TAIL kernel): its unit u < tail_units = R·S is piece u % tail_s of
    // tile tail_first + u / tail_s, the tiles before tail_first being the main launch's
    int tail_first, tail_s, tail_units;
    float *ws;               // partials [slot][8 math warps][HALF / 4][32 lanes] float4
    int *flags;              // [slot][8 math warps] tickets
    unsigned *epoch;         // [2]: the last finished launch's ticket, finished-CTA count
    int tail_early;          // TAIL kernel right behind its main kernel: starts without waiting
    int test_skip_tail;      // failure test only: piece CTAs withhold their partial flags
    __nv_bfloat16 *d;
    float *d32;              // K-grouped: fp32 D [G][M][N]
    const float *c32;        // K-grouped: fp32 C [G][M][N] or NULL (may alias d32)
    int *err;
    uint64_t timeout_ns;
};

template <int BN, int STAGES, bool PAIR, bool PAIR_LIST, bool KGRP = false>
struct GemmLayout {
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
    static_assert(BN / 2 / 32 >= 2, "the TMEM release sits after the second-to-last 32-column batch");
    static constexpr int HALF = BN / 2;                      // columns per math warpgroup
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;        // rows of B loaded by one CTA
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = B_ROWS * BK;
    static constexpr uint32_t STAGE_TX = (PAIR ? 2 : 1) * (A_BYTES + B_BYTES);
    static constexpr int SLAB_BYTES = 32 * HALF * 2;         // 32 rows x HALF bf16 per math warp
    static constexpr int NBUF = 512 / BN;                    // TMEM partial buffers
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_D = OFF_B + STAGES * B_BYTES;
    // A-scale ring: one 128-float row per K block, with full/empty barriers of its own (its
    // loads are not on the MMA's path, so the operand ring's barriers cannot pace them). The
    // K-grouped kernel's per-column B scales (BN floats per K block) share its slots.
    static constexpr int SFS = STAGES + NBUF + 2;
    static constexpr int SF_SLOT = BM + (KGRP ? BN : 0);       // floats per scale slot
    static constexpr int OFF_SFA = OFF_D + 8 * SLAB_BYTES;
    static constexpr int OFF_PAIRS = OFF_SFA + SFS * SF_SLOT * 4;
    static constexpr int PAIR_BYTES = PAIR_LIST ? MAX_PAIR_BLOCKS * 2 : (KGRP ? (MAX_KGROUPS + 1) * 4 : 0);
    static constexpr int OFF_BAR = OFF_PAIRS + PAIR_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 8 + 2 * SFS;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + static_cast<int>(sizeof(WaitCtx)) + 16;
    static constexpr int ALLOC = BYTES + 1024;               // slack to align the base to 1024 B
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(OFF_B % 1024 == 0 && OFF_D % 1024 == 0, "1024-byte aligned operand tiles");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

struct TileInfo {
    int row0;     // first row (in the group's row space) of this CTA's 128-row block
    int n_blk;
    int g;
    int kb0;      // first K block (K-grouped: the group's offset; last-wave piece: its start)
    int nkb;      // K blocks of the tile (K-grouped: the group's; last-wave piece: its share)
    int piece;    // last-wave split: piece index (0 writes D); -1 for a whole tile
    bool valid;   // the tile exists (all CTAs of the pair agree)
    bool store;   // this CTA's rows belong to the tile's expert
};

__device__ __forceinline__ int clamp_rows(int v, int M) { return v < 0 ? 0 : (v > M ? M : v); }

// Number of masked tiles: sum over experts of ceil(masked_m[g] / UNIT) · n_blocks.
template <int UNIT>
__device__ __forceinline__ int masked_num_tiles(const GemmParams &p) {
    int total = 0;
    for (int g = 0; g < p.G; ++g)
        total += (clamp_rows(__ldg(p.masked_m + g), p.M) + UNIT - 1) / UNIT * p.n_blocks;
    return total;
}

// Band rasterisation of units x n_blocks: `band` units share each column pass.
__device__ __forceinline__ void raster(int t, int units, int n_blocks, int band, int &unit, int &n) {
    const int per_band = band * n_blocks;
    const int b = t / per_band;
    const int first = b * band;
    const int bu = min(band, units - first);
    const int local = t - b * per_band;
    unit = first + local % bu;
    n = local / bu;
}

template <int KIND, bool PAIR>
__device__ __forceinline__ TileInfo decode_tile(int t, const GemmParams &p, const uint16_t *pair_first,
                                                int num_pairs, uint32_t rank) {
    constexpr int UNIT = PAIR ? 2 * BM : BM;
    TileInfo ti;
    ti.valid = true;
    ti.store = true;
    ti.g = 0;
    ti.kb0 = 0;
    ti.nkb = p.Kb;
    ti.piece = -1;
    if (KIND == KIND_KGROUPED) {
        // group-major: every group's tiles (all of them, also for an empty group, whose D is C)
        // before the next group's, rasterised within the group; the K-block offsets of the
        // groups sit in shared memory where the pair list would be (reinterpreted as int)
        const int m_units = (p.M + UNIT - 1) / UNIT;
        const int per_g = m_units * p.n_blocks;
        const int g = t / per_g;
        int unit, n;
        raster(t - g * per_g, m_units, p.n_blocks, PAIR ? RASTER_BLOCKS / 2 : RASTER_BLOCKS, unit, n);
        const int *kofs = reinterpret_cast<const int *>(pair_first);
        ti.g = g;
        ti.row0 = unit * UNIT + static_cast<int>(rank) * BM;
        ti.n_blk = n;
        ti.kb0 = kofs[g];
        ti.nkb = kofs[g + 1] - kofs[g];
        return ti;
    }
    if (KIND == KIND_MASKED) {
        int rem = t;
        for (int g = 0; g < p.G; ++g) {
            const int mt = (clamp_rows(__ldg(p.masked_m + g), p.M) + UNIT - 1) / UNIT;
            const int cnt = mt * p.n_blocks;
            if (rem < cnt) {
                ti.g = g;
                ti.row0 = (rem % mt) * UNIT + static_cast<int>(rank) * BM;   // row tiles of an expert adjacent
                ti.n_blk = rem / mt;
                return ti;
            }
            rem -= cnt;
        }
        ti.valid = false;
        ti.row0 = ti.n_blk = 0;
        return ti;
    }
    if (KIND == KIND_CONTIGUOUS && PAIR) {
        int pi, n;
        raster(t, num_pairs, p.n_blocks, RASTER_BLOCKS / 2, pi, n);
        const int fb = pair_first[pi];
        const int g = __ldg(p.grouped_layout + fb * BM);
        ti.g = g;
        ti.n_blk = n;
        ti.row0 = (fb + static_cast<int>(rank)) * BM;
        if (rank == 1) {
            const int nblk = p.M / BM;
            ti.store = fb + 1 < nblk && __ldg(p.grouped_layout + (fb + 1) * BM) == g;
        }
        return ti;
    }
    int unit, n;
    raster(t, (p.M + UNIT - 1) / UNIT, p.n_blocks, PAIR ? RASTER_BLOCKS / 2 : RASTER_BLOCKS, unit, n);
    ti.row0 = unit * UNIT + static_cast<int>(rank) * BM;
    ti.n_blk = n;
    if (KIND == KIND_CONTIGUOUS) {
        const int g = __ldg(p.grouped_layout + ti.row0);
        ti.g = g;
        ti.valid = (g >= 0 && g < p.G);
    }
    return ti;
}

// Work unit w of the persistent loop: a whole tile, or (TAIL kernel) a K piece of a tile.
template <int KIND, bool PAIR, bool TAIL>
__device__ __forceinline__ TileInfo decode_unit(int w, const GemmParams &p, const uint16_t *pair_first,
                                                int num_pairs, uint32_t rank) {
    if (!TAIL) return decode_tile<KIND, PAIR>(w, p, pair_first, num_pairs, rank);
    const int r = w / p.tail_s;                  // which last-wave tile
    const int pc = w - r * p.tail_s;             // which piece of it
    TileInfo ti = decode_tile<KIND, PAIR>(p.tail_first + r, p, pair_first, num_pairs, rank);
    ti.kb0 = pc * p.Kb / p.tail_s;
    ti.nkb = (pc + 1) * p.Kb / p.tail_s - ti.kb0;
    ti.piece = pc;
    return ti;
}

// Ticket of a launch that uses the flag workspace: one past the epoch word, never 0 (flags
// start out zero). The last CTA of the grid to finish stores it back into the epoch word.
__device__ __forceinline__ int streamk_ticket(const unsigned *epoch) {
    const unsigned e = *reinterpret_cast<const volatile unsigned *>(epoch);
    return static_cast<int>(e + 1u == 0u ? 1u : e + 1u);
}

// Contiguous layout, pair tiles: one warp lists the first 128-row block of every pair. Pairs
// start at even offsets inside each run of consecutive blocks of one valid expert; blocks whose
// expert id is -1 or >= G belong to no pair (ids >= G raise the device error word). Returns
// the number of pairs (every lane).
__device__ __forceinline__ int build_pair_list(const GemmParams &p, uint16_t *pair_first, int lane) {
    const int nblk = p.M / BM;
    int e[MAX_PAIR_BLOCKS / 32];
#pragma unroll
    for (int k = 0; k < MAX_PAIR_BLOCKS / 32; ++k) {
        const int b = k * 32 + lane;
        e[k] = b < nblk ? __ldg(p.grouped_layout + b * BM) : -1;
    }
    int count = 0;
    int carry_e = -2, carry_start = 0;
#pragma unroll
    for (int k = 0; k < MAX_PAIR_BLOCKS / 32; ++k) {
        if (k * 32 < nblk) {
            const int b = k * 32 + lane;
            int ek = e[k];
            if (ek >= p.G) {
                report_error(p.err, ERR_DATA);
                ek = -1;
            }
            int prev = __shfl_up_sync(0xFFFFFFFFu, ek, 1);
            if (lane == 0) prev = carry_e;
            const bool new_run = ek != prev;
            const uint32_t starts = __ballot_sync(0xFFFFFFFFu, new_run);
            const uint32_t upto = starts & (0xFFFFFFFFu >> (31 - lane));   // run starts at lanes <= this one
            const int run_start = upto ? k * 32 + (31 - __clz(upto)) : carry_start;
            const bool is_pair = ek >= 0 && b < nblk && ((b - run_start) & 1) == 0;
            const uint32_t pm = __ballot_sync(0xFFFFFFFFu, is_pair);
            if (is_pair) pair_first[count + __popc(pm & ((1u << lane) - 1u))] = static_cast<uint16_t>(b);
            count += __popc(pm);
            carry_e = __shfl_sync(0xFFFFFFFFu, ek, 31);
            carry_start = __shfl_sync(0xFFFFFFFFu, run_start, 31);
        }
    }
    return count;
}

// K-grouped layout: one thread turns the device array of group sizes (tokens, multiples of 128)
// into K-block offsets kofs[0..G] in shared memory. A size that is negative, not a multiple of
// 128 or reaches past the K extent the host described sets the device error word and counts
// as empty (its D is C).
__device__ __forceinline__ void build_kgroup_offsets(const GemmParams &p, int *kofs) {
    int acc = 0;
    kofs[0] = 0;
    for (int g = 0; g < p.G; ++g) {
        const int k = __ldg(p.ks + g);
        int kb = k / BK;
        if (k < 0 || k % BK != 0 || acc + kb > p.Kb) {
            report_error(p.err, ERR_DATA);
            kb = 0;
        }
        acc += kb;
        kofs[g + 1] = acc;
    }
}

// tcgen05.wait::ld, then the loaded registers are read. The reads sit in the same asm statement
// as the wait, with separate input and output operands: tied in/out operands would allow the
// compiler to copy a register that the asynchronous load has not written yet in front of the
// wait, and a bare wait would allow it to move uses above the wait.
__device__ __forceinline__ void tmem_ld_wait_regs32(uint32_t (&r)[32]) {
    uint32_t t[32];
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "mov.b32 %0, %32;\n\tmov.b32 %1, %33;\n\tmov.b32 %2, %34;\n\tmov.b32 %3, %35;\n\t"
        "mov.b32 %4, %36;\n\tmov.b32 %5, %37;\n\tmov.b32 %6, %38;\n\tmov.b32 %7, %39;\n\t"
        "mov.b32 %8, %40;\n\tmov.b32 %9, %41;\n\tmov.b32 %10, %42;\n\tmov.b32 %11, %43;\n\t"
        "mov.b32 %12, %44;\n\tmov.b32 %13, %45;\n\tmov.b32 %14, %46;\n\tmov.b32 %15, %47;\n\t"
        "mov.b32 %16, %48;\n\tmov.b32 %17, %49;\n\tmov.b32 %18, %50;\n\tmov.b32 %19, %51;\n\t"
        "mov.b32 %20, %52;\n\tmov.b32 %21, %53;\n\tmov.b32 %22, %54;\n\tmov.b32 %23, %55;\n\t"
        "mov.b32 %24, %56;\n\tmov.b32 %25, %57;\n\tmov.b32 %26, %58;\n\tmov.b32 %27, %59;\n\t"
        "mov.b32 %28, %60;\n\tmov.b32 %29, %61;\n\tmov.b32 %30, %62;\n\tmov.b32 %31, %63;"
        : "=r"(t[0]), "=r"(t[1]), "=r"(t[2]), "=r"(t[3]), "=r"(t[4]), "=r"(t[5]), "=r"(t[6]), "=r"(t[7]),
          "=r"(t[8]), "=r"(t[9]), "=r"(t[10]), "=r"(t[11]), "=r"(t[12]), "=r"(t[13]), "=r"(t[14]), "=r"(t[15]),
          "=r"(t[16]), "=r"(t[17]), "=r"(t[18]), "=r"(t[19]), "=r"(t[20]), "=r"(t[21]), "=r"(t[22]), "=r"(t[23]),
          "=r"(t[24]), "=r"(t[25]), "=r"(t[26]), "=r"(t[27]), "=r"(t[28]), "=r"(t[29]), "=r"(t[30]), "=r"(t[31])
        : "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = t[i];
}

// A_MN / B_MN: A stored [K, M] / B stored [K, N] (M- or N-contiguous, "T" / "N" in the
// layout names of the pages) instead of K-contiguous; tm_a / tm_b then map those arrays and
// the MMA reads them through MN-major descriptors. tm_sfb (K-grouped only) maps the per-column
// B scales [Kb][pad4(N)].
template <int BN, int STAGES, int KIND, bool PAIR, bool A_MN = false, bool B_MN = false, bool TAIL = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_c,
                const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_sfb,
                const GemmParams p) {
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    constexpr bool PAIR_LIST = PAIR && KIND == KIND_CONTIGUOUS;
    constexpr bool KGRP = KIND == KIND_KGROUPED;
    static_assert(!(A_MN || B_MN) || KIND == KIND_DENSE || KGRP, "MN-major operands: dense and K-grouped only");
    static_assert(!TAIL || KIND == KIND_DENSE, "last-wave split: dense only");
    constexpr bool KSUB = KGRP || TAIL;        // units cover a sub-range of the K blocks
    using L = GemmLayout<BN, STAGES, PAIR, PAIR_LIST, KGRP>;
    constexpr int HALF = L::HALF;
    constexpr int NBUF = L::NBUF;
    constexpr int UNIT = PAIR ? 2 * BM : BM;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *cfull = tempty + NBUF;
    uint64_t *sfa_full = cfull + 8;
    uint64_t *sfa_empty = sfa_full + L::SFS;
    const float *sfa_ring = reinterpret_cast<const float *>(smem + L::OFF_SFA);   // slots of SF_SLOT floats
    WaitCtx *ctx = reinterpret_cast<WaitCtx *>(smem + L::OFF_MISC);
    int *num_pairs_smem = reinterpret_cast<int *>(smem + L::OFF_MISC + sizeof(WaitCtx));
    int *ticket_smem = num_pairs_smem + 1;     // last-wave split: this launch's flag ticket
    uint16_t *pair_first = reinterpret_cast<uint16_t *>(smem + L::OFF_PAIRS);
    volatile int *abort_flag = &ctx->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int cid = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int ncid = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    // prologue (overlaps the previous kernel's tail): barriers, descriptors, TMEM
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);   // math warp 4 of this CTA, once the K block's MMAs are done
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], PAIR ? 16 : 8);
        }
        for (int w = 0; w < 8; ++w) mbar_init(&cfull[w], 1);
        for (int j = 0; j < L::SFS; ++j) {
            mbar_init(&sfa_full[j], 1);
            mbar_init(&sfa_empty[j], 8);   // one arrive per math warp
        }
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
        if (KGRP) tma_prefetch_desc(&tm_sfb);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(&ctx->tmem_base, L::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&ctx->tmem_base, L::TMEM_COLS);
            tmem_relinquish();
        }
    }
    // Programmatic dependent launch. A kernel waits for its predecessor here (from here on
    // global memory may be read and written) and only then lets its dependent launch. So a
    // TAIL kernel launched right behind its main kernel (tail_early), whose tiles and workspace
    // the main kernel never touches, may start at once, on SMs the main kernel has left:
    // everything before the main kernel is complete by then. It waits for the main kernel only
    // before it exits, so that it never completes before it (the next kernel's wait covers
    // both). A TAIL kernel with no main kernel before it waits here like any other.
    if (!TAIL || !p.tail_early) pdl_wait();
    pdl_launch_dependents();
    if (PAIR_LIST && warp == 2) {
        const int np = build_pair_list(p, pair_first, lane);
        if (lane == 0) *num_pairs_smem = np;
    }
    if (KGRP && warp == 2 && lane == 0) build_kgroup_offsets(p, reinterpret_cast<int *>(pair_first));
    if (TAIL && threadIdx.x == 0) *ticket_smem = streamk_ticket(p.epoch);
    tc_fence_before();
    if (PAIR)
        cluster_sync();
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctx->tmem_base;
    const int num_pairs = PAIR_LIST ? *num_pairs_smem : 0;

    int num_tiles;
    if (TAIL)
        num_tiles = p.tail_units;
    else if (KIND == KIND_MASKED)
        num_tiles = masked_num_tiles<UNIT>(p);
    else if (PAIR_LIST)
        num_tiles = num_pairs * p.n_blocks;
    else
        num_tiles = p.num_tiles;
    if (KIND == KIND_MASKED && blockIdx.x == 0 && threadIdx.x == 0) {
        for (int g = 0; g < p.G; ++g)
            if (__ldg(p.masked_m + g) > p.M) report_error(p.err, ERR_DATA);
    }

    if (warp < 4) {
        reg_dealloc<56>();
        // TMA producers. One thread's bulk copies are served one after another (a fixed cost
        // per copy, whatever its size), so A and B each get two threads (lanes 0 and 16 of warps
        // 0 and 2: even and odd K blocks); the A thread of a K block also loads its A scales
        // (into a slot of their ring, whose release by the math warps is at most STAGES + NBUF
        // K blocks behind, less than the ring's SFS slots) and arms its stage. All wait on the
        // same "empty" barriers of the operand ring; none can run more than STAGES K blocks
        // ahead of the others, since a stage is only freed once all its loads have landed and
        // the MMA has consumed it.
        const int stream = (warp == 0 || warp == 2) && (lane & 15) == 0 ? warp >> 1 : -1;
        const uint32_t parity = static_cast<uint32_t>(lane >> 4);
        const uint32_t nlanes = 2u;
        if (stream >= 0) {
            uint32_t it = 0;
            for (int t = cid; t < num_tiles && !*abort_flag; t += ncid) {
                const TileInfo ti = decode_unit<KIND, PAIR, TAIL>(t, p, pair_first, num_pairs, rank);
                if (!ti.valid) {
                    if (stream == 0 && parity == 0 && KIND == KIND_CONTIGUOUS && ti.g >= p.G) report_error(p.err, ERR_DATA);
                    continue;
                }
                const int brow = ti.n_blk * BN + static_cast<int>(rank) * L::B_ROWS;
                const int bz = KGRP ? 0 : ti.g;                    // K-grouped B: one [sum_K, N] array
                const int nkb = KSUB ? ti.nkb : p.Kb;
                for (int kbl = 0; kbl < nkb; ++kbl, ++it) {
                    if (it % nlanes != parity) continue;
                    const int kb = KSUB ? ti.kb0 + kbl : kbl;      // K block in the operands' K space
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (stream == 0) {
                        const int j = it % L::SFS;
                        if (!mbar_wait(&sfa_empty[j], ((it / L::SFS) & 1) ^ 1, ctx)) break;
                        float *sf = reinterpret_cast<float *>(smem + L::OFF_SFA) + j * L::SF_SLOT;
                        mbar_arrive_expect_tx(&sfa_full[j], L::SF_SLOT * 4);
                        if (KIND == KIND_MASKED)
                            tma_load_3d(&tm_sfa, &sfa_full[j], sf, ti.row0, kb, ti.g);
                        else
                            tma_load_2d(&tm_sfa, &sfa_full[j], sf, ti.row0, kb);
                        if (KGRP) tma_load_2d(&tm_sfb, &sfa_full[j], sf + BM, ti.n_blk * BN, kb);
                    }
                    if (!mbar_wait(&empty[s], ph ^ 1, ctx)) break;
                    uint8_t *sa = smem + L::OFF_A + s * L::A_BYTES;
                    uint8_t *sb = smem + L::OFF_B + s * L::B_BYTES;
                    if (PAIR) {
                        const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);   // the leader's barrier
                        if (stream == 0) {
                            if (leader) mbar_arrive_expect_tx(&full[s], L::STAGE_TX);
                            if (A_MN)
                                tma_load_2d_pair(&tm_a, fb, sa, ti.row0, kb * BK);
                            else if (KIND == KIND_MASKED)
                                tma_load_3d_pair(&tm_a, fb, sa, kb * BK, ti.row0, ti.g);
                            else
                                tma_load_2d_pair(&tm_a, fb, sa, kb * BK, ti.row0);
                        } else if (B_MN) {
#pragma unroll
                            for (int i = 0; i < L::B_ROWS / 128; ++i)
                                tma_load_3d_pair(&tm_b, fb, sb + i * 128 * BK, brow + 128 * i, kb * BK, bz);
                        } else {
                            tma_load_3d_pair(&tm_b, fb, sb, kb * BK, brow, bz);
                        }
                    } else {
                        if (stream == 0) {
                            mbar_arrive_expect_tx(&full[s], L::STAGE_TX);
                            if (A_MN)
                                tma_load_2d(&tm_a, &full[s], sa, ti.row0, kb * BK);
                            else if (KIND == KIND_MASKED)
                                tma_load_3d(&tm_a, &full[s], sa, kb * BK, ti.row0, ti.g);
                            else
                                tma_load_2d(&tm_a, &full[s], sa, kb * BK, ti.row0);
                        } else if (B_MN) {
#pragma unroll
                            for (int i = 0; i < L::B_ROWS / 128; ++i)
                                tma_load_3d(&tm_b, &full[s], sb + i * 128 * BK, brow + 128 * i, kb * BK, bz);
                        } else {
                            tma_load_3d(&tm_b, &full[s], sb, kb * BK, brow, bz);
                        }
                    }
                }
            }
        } else if ((warp == 1 || (warp == 3 && STAGES % 2 == 0 && NBUF % 2 == 0 && !p.one_issuer)) && lane == 0 &&
                   leader) {
            // ---------------- MMA issuers (the leader CTA of a pair) ----------------
            // warp 1: K blocks with an even running index, warp 3: odd ones; both stage and
            // buffer counts even, so each issuer owns its stages and TMEM buffers
            constexpr bool TWO_OK = STAGES % 2 == 0 && NBUF % 2 == 0;
            const bool two = TWO_OK && !p.one_issuer;
            const uint32_t mine = warp == 1 ? 0u : 1u;
            constexpr uint32_t IDESC = idesc_f8_e4m3_f32<UNIT, BN, A_MN, B_MN>();
            // a K step of 32: 32 bytes along a K-major row (+2 in the 16-byte granular start
            // address), or 32 rows of 128 bytes of an MN-major tile (+256)
            constexpr uint64_t A_STEP = A_MN ? 256 : 2, B_STEP = B_MN ? 256 : 2;
            uint32_t it = 0;
            for (int t = cid; t < num_tiles && !*abort_flag; t += ncid) {
                const TileInfo ti = decode_unit<KIND, PAIR, TAIL>(t, p, pair_first, num_pairs, rank);
                if (!ti.valid) continue;
                const int nkb = KSUB ? ti.nkb : p.Kb;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    if (two && (it & 1u) != mine) continue;
                    const int s = it % STAGES;
                    const int b = it % NBUF;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, ctx)) break;
                    if (!mbar_wait(&tempty[b], ((it / NBUF) & 1) ^ 1, ctx)) break;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::OFF_A + s * L::A_BYTES);
                    const uint32_t b_addr = smem_u32(smem + L::OFF_B + s * L::B_BYTES);
                    // MN-major: 128-element atoms 128 rows x 128 bytes apart (the second B atom
                    // of a 256-column single-CTA tile)
                    const uint64_t ad = A_MN ? sdesc_mn_sw128(a_addr, 128 * BK) : sdesc_k_sw128(a_addr);
                    const uint64_t bd = B_MN ? sdesc_mn_sw128(b_addr, 128 * BK) : sdesc_k_sw128(b_addr);
                    const uint32_t dt = tmem_base + static_cast<uint32_t>(b * BN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        if (PAIR)
                            umma_f8_pair(dt, ad + A_STEP * k, bd + B_STEP * k, IDESC, k > 0 ? 1u : 0u);
                        else
                            umma_f8(dt, ad + A_STEP * k, bd + B_STEP * k, IDESC, k > 0 ? 1u : 0u);
                    }
                    // one commit per K block: the math warps hand the operand stage back once they
                    // have seen the MMAs complete (a commit costs the issuing thread several
                    // times what an MMA does)
                    if (PAIR)
                        umma_commit_pair(&tfull[b], 0x3);
                    else
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
        const uint32_t tempty_leader0 = PAIR ? mapa_shared(smem_u32(&tempty[0]), 0) : smem_u32(&tempty[0]);
        uint32_t it = 0, ctile = 0;
        bool ok = true;
        for (int t = cid; t < num_tiles && ok; t += ncid) {
            const TileInfo ti = decode_unit<KIND, PAIR, TAIL>(t, p, pair_first, num_pairs, rank);
            if (!ti.valid) continue;
            const int col0 = ti.n_blk * BN + wg * HALF;          // first column of this warp
            const int srow0 = ti.row0 + q * 32;                  // first row of this warp's slab
            const int row = srow0 + lane;                        // this thread's row
            const int nblk = min(col0 / 128, p.Nb - 1);
            // (a last-wave piece starts at K block kb0: its window is offset by that)
            const float *sfb_row = p.sfb + (static_cast<size_t>(ti.g) * p.Nb + nblk) * p.Kb + (TAIL ? ti.kb0 : 0);
            const bool do_c = !KGRP && p.has_c && ti.store && (!TAIL || ti.piece == 0);   // piece 0 writes D
            if (do_c && lane == 0) {
                bulk_wait_group_read0();                         // the slab's last store has read it
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&cfull[mw], L::SLAB_BYTES);
                if (KIND != KIND_MASKED && p.cd_blocks) {
                    tma_load_3d(&tm_c, &cfull[mw], slab, 0, srow0, col0 / 64);   // the whole slab
                } else {
#pragma unroll
                    for (int bx = 0; bx < HALF / 64; ++bx) {
                        if (KIND == KIND_MASKED)
                            tma_load_3d(&tm_c, &cfull[mw], slab + bx * 4096, col0 + bx * 64, srow0, ti.g);
                        else
                            tma_load_2d(&tm_c, &cfull[mw], slab + bx * 4096, col0 + bx * 64, srow0);
                    }
                }
            }
            float acc[HALF];
#pragma unroll
            for (int i = 0; i < HALF; ++i) acc[i] = 0.f;
            // sfb of this warp's n-block, 32 K blocks per window (one value per lane, broadcast by
            // shuffle); sfa of this thread's row from the TMA-filled ring. No global load is left
            // in flight across the loop's release-arrives except a window refill every 32 blocks.
            // (K-grouped: one B scale per column, from the same ring slot as sfa)
            const int nkb = KSUB ? ti.nkb : p.Kb;
            float sb_win = !KGRP && lane < nkb ? __ldg(sfb_row + lane) : 0.f;
            float sb_nxt = !KGRP && 32 + lane < nkb ? __ldg(sfb_row + 32 + lane) : 0.f;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int b = it % NBUF;
                const uint32_t phb = (it / NBUF) & 1;
                if (!KGRP && (kb & 31) == 0 && kb > 0) {
                    sb_win = sb_nxt;
                    sb_nxt = kb + 32 + lane < nkb ? __ldg(sfb_row + kb + 32 + lane) : 0.f;
                }
                const float sb = KGRP ? 1.f : __shfl_sync(0xFFFFFFFFu, sb_win, kb & 31);
                const int j = it % L::SFS;
                // every lane waits; the outcome is made warp-uniform before any .sync.aligned op
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], phb, ctx));
                if (!ok) break;
                // the K block's MMAs are complete, so they have read the operand stage: warp 4
                // hands it back to this CTA's producers
                if (warp == 4 && lane == 0) mbar_arrive(&empty[it % STAGES]);
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sfa_full[j], (it / L::SFS) & 1, ctx));
                if (!ok) break;
                const float sa = sfa_ring[j * L::SF_SLOT + q * 32 + lane];
                tc_fence_after();
                const float scale = sa * sb;
                if (!KGRP) {
                    // the slot is read: the generic-proxy read is ordered before the producer's
                    // next TMA write into the slot (async proxy) by a proxy fence, which
                    // release/acquire through the mbarrier alone does not give
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_relaxed(&sfa_empty[j]);
                }
                const float2 scale2 = make_float2(scale, scale);
                const float *sbc = sfa_ring + j * L::SF_SLOT + BM + wg * HALF;   // K-grouped column scales
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
                    for (int i = 0; i < 16; ++i) {   // packed fp32x2 FMA: half the issue slots
                        float2 s2 = scale2;
                        if (KGRP) {                   // sa · sfb[column], sfb broadcast from shared memory
                            const float2 sb2 = *reinterpret_cast<const float2 *>(sbc + c * 32 + 2 * i);
                            s2 = __fmul2_rn(scale2, sb2);
                        }
                        const float2 a2 = __ffma2_rn(
                            make_float2(__uint_as_float(r[c & 1][2 * i]), __uint_as_float(r[c & 1][2 * i + 1])), s2,
                            make_float2(acc[c * 32 + 2 * i], acc[c * 32 + 2 * i + 1]));
                        acc[c * 32 + 2 * i] = a2.x;
                        acc[c * 32 + 2 * i + 1] = a2.y;
                    }
                    if (c + 1 < HALF / 32) tmem_ld_wait_regs32(r[(c + 1) & 1]);
                    if (c + 2 == HALF / 32) {
                        // the last batch is in registers: every TMEM read of the buffer is complete
                        // (wait::ld) and sa was consumed, so the buffer goes back to the MMA before
                        // the last batch is folded in; a relaxed arrive suffices. (A failure test
                        // can withhold one release: the MMA's bounded wait then runs out.)
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0 && !(p.test_skip_release && blockIdx.x == 0 && warp == 4 && it == 0)) {
                            if (PAIR)
                                mbar_arrive_cluster_relaxed(tempty_leader0 + b * 8);
                            else
                                mbar_arrive_relaxed(&tempty[b]);
                        }
                    }
                }
                if (KGRP) {                            // the column scales are read too
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_relaxed(&sfa_empty[j]);
                }
            }
            if (!ok) break;
            if (!ti.store) continue;
            if (TAIL) {
                // last-wave split. This warp's slice of a piece's partial: 32 rows x HALF columns,
                // float4 c4 of lane l at [c4][l] (each store instruction writes 512 contiguous bytes)
                constexpr int SLICE = 32 * HALF;                   // floats per warp slice
                const int ticket = *ticket_smem;
                const int r = t / p.tail_s;
                const int piece = t - r * p.tail_s;
                const int slot0 = r * (p.tail_s - 1) * (PAIR ? 2 : 1) + static_cast<int>(rank);
                if (piece > 0) {
                    const int slot = slot0 + (piece - 1) * (PAIR ? 2 : 1);
                    float4 *dst = reinterpret_cast<float4 *>(p.ws + (static_cast<size_t>(slot) * 8 + mw) * SLICE);
#pragma unroll
                    for (int c4 = 0; c4 < HALF / 4; ++c4)
                        __stcg(dst + c4 * 32 + lane,
                               make_float4(acc[4 * c4], acc[4 * c4 + 1], acc[4 * c4 + 2], acc[4 * c4 + 3]));
                    __threadfence();
                    __syncwarp();
                    if (lane == 0 && !p.test_skip_tail) flag_store_release(p.flags + slot * 8 + mw, ticket);
                    continue;
                }
                // piece 0: wait (bounded) for each later piece's slice, then add them in piece
                // order, so that the sum does not depend on which piece finished first
                bool got = true;
                if (lane == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    for (int pc = 1; pc < p.tail_s && got; ++pc) {
                        const int slot = slot0 + (pc - 1) * (PAIR ? 2 : 1);
                        while (flag_load_acquire(p.flags + slot * 8 + mw) != ticket) {
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
                }
                ok = __shfl_sync(0xFFFFFFFFu, got, 0);
                if (!ok) break;
                for (int pc = 1; pc < p.tail_s; ++pc) {
                    const int slot = slot0 + (pc - 1) * (PAIR ? 2 : 1);
                    const float4 *src = reinterpret_cast<const float4 *>(p.ws + (static_cast<size_t>(slot) * 8 + mw) * SLICE);
#pragma unroll
                    for (int c4 = 0; c4 < HALF / 4; ++c4) {
                        const float4 v = __ldcg(src + c4 * 32 + lane);
                        acc[4 * c4] += v.x;
                        acc[4 * c4 + 1] += v.y;
                        acc[4 * c4 + 2] += v.z;
                        acc[4 * c4 + 3] += v.w;
                    }
                }
            }
            if (KGRP) {
                // fp32 D (a weight gradient): each thread stores its row's HALF columns, 16 bytes
                // at a time, after adding C (read the same way; N % 16 == 0, so a 4-column
                // vector is all in or all out)
                if (row < p.M) {
                    const size_t rbase = (static_cast<size_t>(ti.g) * p.M + row) * p.N;
#pragma unroll
                    for (int c4 = 0; c4 < HALF / 4; ++c4) {
                        const int col = col0 + c4 * 4;
                        if (col < p.N) {
                            float4 v = make_float4(acc[4 * c4], acc[4 * c4 + 1], acc[4 * c4 + 2], acc[4 * c4 + 3]);
                            if (p.c32) {
                                const float4 cv = *reinterpret_cast<const float4 *>(p.c32 + rbase + col);
                                v.x += cv.x;
                                v.y += cv.y;
                                v.z += cv.z;
                                v.w += cv.w;
                            }
                            *reinterpret_cast<float4 *>(p.d32 + rbase + col) = v;
                        }
                    }
                }
                continue;
            }
            if (do_c) {
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&cfull[mw], ctile & 1, ctx));
                if (!ok) break;
                ++ctile;
            } else {
                if (lane == 0) bulk_wait_group_read0();          // the slab's last store has read it
                __syncwarp();
            }
            // bf16 epilogue into the swizzled slab: row `lane`, 16-byte chunk ch of box bx lives
            // at bx*4096 + lane*128 + ((ch ^ (lane & 7)) * 16). A box's 8 C chunks are read before
            // any is overwritten; C is added in packed fp32 pairs (a bf16 widens to fp32 exactly:
            // low half << 16, high half with the low bits cleared).
#pragma unroll
            for (int bx = 0; bx < HALF / 64; ++bx) {
                uint4 cv[8];
                if (do_c) {
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        cv[ch] = *reinterpret_cast<const uint4 *>(slab + bx * 4096 + lane * 128 + ((ch ^ (lane & 7)) * 16));
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t cw[4] = {cv[ch].x, cv[ch].y, cv[ch].z, cv[ch].w};
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 v = make_float2(acc[bx * 64 + ch * 8 + 2 * e], acc[bx * 64 + ch * 8 + 2 * e + 1]);
                        if (do_c)
                            v = __fadd2_rn(v, make_float2(__uint_as_float(cw[e] << 16), __uint_as_float(cw[e] & 0xFFFF0000u)));
                        __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
                        w[e] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    *reinterpret_cast<uint4 *>(slab + bx * 4096 + lane * 128 + ((ch ^ (lane & 7)) * 16)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (KIND == KIND_MASKED) {
                const int mm = clamp_rows(__ldg(p.masked_m + ti.g), p.M);
                const int valid_rows = max(0, min(32, mm - srow0));
                if (valid_rows == 32) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
#pragma unroll
                        for (int bx = 0; bx < HALF / 64; ++bx)
                            tma_store_3d(&tm_d, slab + bx * 4096, col0 + bx * 64, srow0, ti.g);
                        bulk_commit_group();
                    }
                } else if (lane < valid_rows) {
                    // partial slab: only rows below masked_m[g] are written, each by its owner
                    __nv_bfloat16 *drow = p.d + (static_cast<size_t>(ti.g) * p.M + row) * p.N;
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
                    if (p.cd_blocks) {
                        tma_store_3d(&tm_d, slab, 0, srow0, col0 / 64);   // the whole slab
                    } else {
#pragma unroll
                        for (int bx = 0; bx < HALF / 64; ++bx) tma_store_2d(&tm_d, slab + bx * 4096, col0 + bx * 64, srow0);
                    }
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    }

    __syncwarp();                              // reconverge single-lane roles before the barrier
    if (TAIL && p.tail_early) pdl_wait();
    tc_fence_before();
    if (PAIR)
        cluster_sync();
    else
        __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
    if (TAIL && threadIdx.x == 0) {
        // the last CTA to finish publishes this launch's ticket as the epoch; the next launch
        // on the stream reads it only after this grid has completed (griddepcontrol.wait)
        __threadfence();
        if (atomicAdd(p.epoch + 1, 1u) == gridDim.x - 1) {
            p.epoch[1] = 0u;
            p.epoch[0] = static_cast<unsigned>(*ticket_smem);
            __threadfence();
        }
    }
#endif
}

}  // namespace dg
