// dg_api.cu — the C ABI declared in include/dg.h: argument checks, TMA descriptor encoding,
// tile-shape choice and kernel launch. No allocation, no synchronisation on the call path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dg.h"
#include "dg_cast.cuh"
#include "dg_gemm.cuh"
#include "dg_gemm_bs.cuh"
#include "dg_gemm_splitk.cuh"
#include "dg_gemm_swap.cuh"

namespace {

constexpr int kMaxDevices = 64;

__device__ int g_device_error;   // see dg_get_device_error()

// Scratch of dg_fp8_gemm_nt_noalloc: the few-row kernel's stream-K partials and flags for up to
// kStaticSlots CTAs, then the two words of its launch epoch, in the module's own device memory
// (zero-initialised at load).
constexpr int kStaticSlots = 256;
static __device__ __align__(256) float g_static_ws[kStaticSlots * 128 * 128];
static __device__ __align__(256) int g_static_flags[kStaticSlots + 2];

// Device memory this library has allocated (cudaMalloc) so far, all devices; dg_allocated_bytes().
std::atomic<long long> g_allocated{0};

// Name of the GEMM kernel the calling thread's last GEMM call launched; dg_last_kernel().
thread_local const char *t_last_kernel = "";
thread_local char t_kernel_name[96];   // names with a number in them (the last-wave split)
thread_local int t_last_launches = 0;  // kernels the thread's last GEMM call launched

struct DeviceInfo {
    std::atomic<bool> ready{false};
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    int *err = nullptr;          // device address of g_device_error
    float *static_ws = nullptr;  // device addresses of g_static_ws and g_static_flags
    int *static_flags = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

dg_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DG_OK : DG_ERR_CUDA; }

// Per-device facts, queried once per device with that device current.
dg_status device_info(const DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DG_ERR_CUDA;
    DeviceInfo &d = g_dev[dev];
    if (!d.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!d.ready.load(std::memory_order_relaxed)) {
            if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DG_ERR_CUDA;
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
            if (cudaGetSymbolAddress(reinterpret_cast<void **>(&d.err), g_device_error) != cudaSuccess ||
                cudaGetSymbolAddress(reinterpret_cast<void **>(&d.static_ws), g_static_ws) != cudaSuccess ||
                cudaGetSymbolAddress(reinterpret_cast<void **>(&d.static_flags), g_static_flags) != cudaSuccess)
                return DG_ERR_CUDA;
            if (!g_encode) {
                cudaDriverEntryPointQueryResult q;
                void *fn = nullptr;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || !fn)
                    return DG_ERR_CUDA;
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
            d.ready.store(true, std::memory_order_release);
        }
    }
    if (d.cc_major != 10 || d.cc_minor != 0) return DG_ERR_UNSUPPORTED;
    *out = &d;
    return DG_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch configuration of every kernel: programmatic dependent launch (the kernel may start
// while the previous kernel of the stream runs; it waits for it with griddepcontrol.wait before
// touching global memory), plus a cluster shape when `cluster` > 1.
struct Launch {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    Launch(dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster = 1, bool cluster_attr = false) {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        int n = 1;
        if (cluster > 1 || cluster_attr) {
            attr[1].id = cudaLaunchAttributeClusterDimension;
            attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
            attr[1].val.clusterDim.y = 1;
            attr[1].val.clusterDim.z = 1;
            n = 2;
        }
        cfg.attrs = attr;
        cfg.numAttrs = n;
    }
};

int pad4(int x) { return (x + 3) / 4 * 4; }

uint64_t wait_limit_ns() {
    static std::atomic<uint64_t> cached{0};
    uint64_t v = cached.load();
    if (v == 0) {
        v = 4000000000ull;   // 4 s per pipeline wait
        if (const char *s = std::getenv("DG_WAIT_TIMEOUT_MS")) {
            const long long ms = std::atoll(s);
            if (ms > 0) v = static_cast<uint64_t>(ms) * 1000000ull;
        }
        cached.store(v);
    }
    return v;
}

// Tile-width override for experiments (DG_FORCE_BN=128|256); 0 = heuristic.
int forced_bn() {
    static std::atomic<int> cached{-1};
    int v = cached.load();
    if (v < 0) {
        v = 0;
        if (const char *s = std::getenv("DG_FORCE_BN")) v = std::atoi(s);
        if (v != 128 && v != 256) v = 0;
        cached.store(v);
    }
    return v;
}

// CTA-pair override for experiments (DG_FORCE_PAIR=0|1); -1 = heuristic.
int forced_pair() {
    static std::atomic<int> cached{-2};
    int v = cached.load();
    if (v == -2) {
        v = -1;
        if (const char *s = std::getenv("DG_FORCE_PAIR")) v = std::atoi(s) ? 1 : 0;
        cached.store(v);
    }
    return v;
}

// Few-row kernel override for experiments (DG_FORCE_SWAP=0|1); -1 = heuristic.
int forced_swap() {
    static std::atomic<int> cached{-2};
    int v = cached.load();
    if (v == -2) {
        v = -1;
        if (const char *s = std::getenv("DG_FORCE_SWAP")) v = std::atoi(s) ? 1 : 0;
        cached.store(v);
    }
    return v;
}

// Cluster size of the few-row split-K kernel for tests and experiments (DG_SPLITK_S=1|2|3|4|6|8|16);
// 0 = cost model. A forced size that the shape or the device cannot take falls back to the model.
int forced_splitk_s() {
    static std::atomic<int> cached{-1};
    int v = cached.load();
    if (v < 0) {
        v = 0;
        if (const char *s = std::getenv("DG_SPLITK_S")) v = std::atoi(s);
        if (v != 1 && v != 2 && v != 3 && v != 4 && v != 6 && v != 8 && v != 16) v = 0;
        cached.store(v);
    }
    return v;
}

// MMA issue override for experiments (DG_ONE_ISSUER=1: one issuing thread per CTA even where
// the stage count allows two); 0 = the kernels' own choice.
int one_issuer() {
    static std::atomic<int> cached{-1};
    int v = cached.load();
    if (v < 0) {
        const char *s = std::getenv("DG_ONE_ISSUER");
        v = s && std::atoi(s) ? 1 : 0;
        cached.store(v);
    }
    return v;
}

// Few-row kernel by shape: the cluster split-K kernel when every tile fits one round of
// clusters with a moderate K (its partials never leave the chip), stream-K otherwise (it splits
// any tile count evenly over every SM, at the cost of a reduction through global memory).
// DG_FEW_ROW=streamk|cluster overrides.
bool use_streamk(int groups, int m_tiles, int N, int K) {
    static std::atomic<int> cached{-1};
    int v = cached.load();
    if (v < 0) {
        const char *s = std::getenv("DG_FEW_ROW");
        v = s && std::strcmp(s, "streamk") == 0 ? 1 : (s && std::strcmp(s, "cluster") == 0 ? 2 : 0);
        cached.store(v);
    }
    if (v) return v == 1;
    const long long tiles = static_cast<long long>(groups) * m_tiles * ((N + 127) / 128);
    return tiles > 64 || K / 128 > 64;
}

// Last-wave split of the dense tile GEMM for tests and experiments (DG_TAIL_SPLIT=0: off,
// 2..64: pieces per last-wave tile, capped by the grid and by K); -1 = cost model.
int forced_tail_split() {
    static std::atomic<int> cached{-2};
    int v = cached.load();
    if (v == -2) {
        v = -1;
        if (const char *s = std::getenv("DG_TAIL_SPLIT")) {
            v = std::atoi(s);
            if (v != 0 && (v < 2 || v > 64)) v = -1;
        }
        cached.store(v);
    }
    return v;
}

// Failure tests only (DG_TEST_SKIP_RELEASE): 1 = the tile GEMM withholds one TMEM-buffer
// release, 2 = the cluster split-K GEMM withholds one partial-push arrive, 3 = the process's
// first two stream-K launches have their odd-numbered CTAs withhold their partial flags, 4 = the
// process's first tile-GEMM launch with a last-wave split has its piece CTAs withhold their
// partial flags. A bounded wait then runs out of time and reports DG_ERR_TIMEOUT without
// faulting. 0 = off.
int test_skip_release() {
    static std::atomic<int> cached{-1};
    int v = cached.load();
    if (v < 0) {
        const char *s = std::getenv("DG_TEST_SKIP_RELEASE");
        v = s ? std::atoi(s) : 0;
        if (v < 1 || v > 4) v = 0;
        cached.store(v);
    }
    return v;
}

bool test_skip_streamk_flags() {
    static std::atomic<int> launches{0};
    return test_skip_release() == 3 && launches.fetch_add(1) < 2;
}

bool test_skip_tail_flags() {
    static std::atomic<int> launches{0};
    return test_skip_release() == 4 && launches.fetch_add(1) < 1;
}

// Encodes a tiled tensor map. dims/box are innermost first; strides (bytes) for dims 1..rank-1.
bool encode(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw) {
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    cuuint64_t d[5], s[4];
    cuuint32_t b[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        if (i + 1 < rank) s[i] = strides[i];
    }
    const CUresult r = g_encode(m, dt, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, s, b, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct GemmMaps {
    CUtensorMap a, b, sfa, c, d, sfb;
};

// Operand storage of a GEMM call: A [rows][K] or, MN-major, [K][rows]; B [G][N][K] or [G][K][N].
struct OperandMajor {
    bool a_mn = false, b_mn = false;
};

// Operand maps of one GEMM call. rows = rows of A/C/D per group; b_rows = rows of B one CTA
// loads; batched = 3D maps over G groups for A, C and D (masked layout). MN-major operands are
// mapped as {MN, K} boxes of 128 x 128 (one 128-byte swizzled row per K index).
bool build_maps(GemmMaps &mp, const void *a, const float *sfa, const void *b, const void *c, void *d, int rows, int N,
                int K, int G, int b_rows, bool batched, int slab_blocks, OperandMajor om = OperandMajor()) {
    const uint64_t Gg = static_cast<uint64_t>(G);
    mp.sfb = mp.sfa;   // only the K-grouped kernel reads it (build_kgrouped_maps)
    {   // sfa: fp32 [G?][Kb][pad4(rows)], box 128 x 1 (one K block's scales of a 128-row block)
        const uint64_t Kb = static_cast<uint64_t>(K / 128), ld = static_cast<uint64_t>(pad4(rows));
        const uint64_t dims[3] = {ld, Kb, Gg};
        const uint64_t str[2] = {ld * 4, ld * 4 * Kb};
        const uint32_t box[3] = {128, 1, 1};
        if (!encode(&mp.sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, batched ? 3 : 2, sfa, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    }
    if (om.a_mn) {   // A: e4m3 [K][rows], box 128 rows x 128 K, 128-byte swizzle
        const uint64_t dims[2] = {static_cast<uint64_t>(rows), static_cast<uint64_t>(K)};
        const uint64_t str[1] = {static_cast<uint64_t>(rows)};
        const uint32_t box[2] = {128, 128};
        if (!encode(&mp.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    } else {   // A: e4m3 [G?][rows][K], box 128 x 128, 128-byte swizzle
        const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(K) * rows};
        const uint32_t box[3] = {128, 128, 1};
        if (!encode(&mp.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, batched ? 3 : 2, a, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    }
    if (om.b_mn) {   // B: e4m3 [G][K][N], box 128 columns x 128 K x 1 (b_rows / 128 boxes per stage)
        const uint64_t dims[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(K), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(N) * K};
        const uint32_t box[3] = {128, 128, 1};
        if (!encode(&mp.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    } else {   // B: e4m3 [G][N][K], box 128 x b_rows x 1
        const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(K) * N};
        const uint32_t box[3] = {128, static_cast<uint32_t>(b_rows), 1};
        if (!encode(&mp.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    }
    if (slab_blocks > 0) {
        // C, D: bf16 [rows][N] seen as {64 columns, rows, N/64 column blocks}, box 64 x 32 x
        // slab_blocks, 128-byte swizzle: one copy moves a math warp's whole 32-row slab
        const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(N / 64)};
        const uint64_t str[2] = {static_cast<uint64_t>(N) * 2, 128};
        const uint32_t box[3] = {64, 32, static_cast<uint32_t>(slab_blocks)};
        if (!encode(&mp.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, d, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
        if (c) {
            if (!encode(&mp.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, c, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return false;
        } else {
            mp.c = mp.d;   // never read when has_c == 0
        }
        return true;
    }
    {   // C, D: bf16 [G?][rows][N], box 64 x 32, 128-byte swizzle (one box row = 128 bytes)
        const uint64_t dims[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(rows), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(N) * 2, static_cast<uint64_t>(N) * 2 * rows};
        const uint32_t box[3] = {64, 32, 1};
        if (!encode(&mp.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, batched ? 3 : 2, d, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
        if (c) {
            if (!encode(&mp.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, batched ? 3 : 2, c, dims, str, box,
                        CU_TENSOR_MAP_SWIZZLE_128B))
                return false;
        } else {
            mp.c = mp.d;   // never read when has_c == 0
        }
    }
    return true;
}

// Per (kernel, device): dynamic shared memory opt-in and, for CTA pairs, how many two-CTA
// clusters can be resident at once (the persistent grid never exceeds it).
struct KernelInfo {
    std::atomic<int> ready{0};
    int max_clusters = 0;
};

// Flag workspace of a (device, stream): fp32 partials, one flag per slot and the two words of
// the launch epoch (all zero when allocated). Shared by the stream-K few-row kernel (partials
// [CTA][128][128], flags [CTA]) and the tile GEMM's last-wave split (partials [slot][128][256],
// flags [slot][8 math warps]); both follow the same ticket protocol, so their flags never
// need clearing. One per (device, stream), so that launches on different streams never share
// flags; allocated on a stream's first call that wants it, which must not be under graph capture
// (the call then goes without: the tile kernel without the split, the few-row GEMM through the
// tile kernel).
struct StreamWorkspace {
    int dev = -1;
    cudaStream_t stream = nullptr;
    float *ws = nullptr;    // sm_count x 128 KB
    int *flags = nullptr;   // [slots] flags, then the epoch words
    int slots = 0;          // 8 x sm_count
};
std::vector<StreamWorkspace> g_stream_ws;

bool stream_workspace(int dev, int sm_count, cudaStream_t st, StreamWorkspace *out) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const StreamWorkspace &w : g_stream_ws)
        if (w.dev == dev && w.stream == st) {
            *out = w;
            return true;
        }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    StreamWorkspace w;
    w.dev = dev;
    w.stream = st;
    w.slots = 8 * sm_count;
    const size_t ws_bytes = static_cast<size_t>(sm_count) * 128 * 256 * sizeof(float);
    const size_t flag_bytes = static_cast<size_t>(w.slots + 2) * sizeof(int);
    if (cudaMalloc(&w.ws, ws_bytes) != cudaSuccess) return false;
    if (cudaMalloc(&w.flags, flag_bytes) != cudaSuccess) {
        cudaFree(w.ws);
        return false;
    }
    if (cudaMemset(w.flags, 0, flag_bytes) != cudaSuccess) {
        cudaFree(w.ws);
        cudaFree(w.flags);
        return false;
    }
    g_allocated += static_cast<long long>(ws_bytes + flag_bytes);
    g_stream_ws.push_back(w);
    *out = w;
    return true;
}

// Last-wave split plan of a dense NT launch of `tiles` tiles over `units` persistent CTAs
// (pairs): the R = tiles mod units tiles of the last wave are cut along K into S pieces, run
// by a second launch, when that shortens the last wave. Cost model in K-block times (measured
// on B200, 256 x 256 pair tiles): the split saves Kb·(1 - 1/S), costs ~2.7 per extra piece
// (a partial written and read through L2) and a fixed ~20 (the second launch's pipeline fill,
// the exchange, the epilogue; ~26 when whole waves run before it). The best S of at most
// units / R pieces, at least 2 K blocks each, if it saves more than 5. No workspace (a first
// call under graph capture): no split.
void plan_tail(dg::GemmParams &q, int tiles, int units, float *ws, int *flags, unsigned *epoch) {
    q.tail_first = tiles;
    q.tail_s = 1;
    q.tail_units = 0;
    const int forced = forced_tail_split();
    if (!ws || forced == 0 || units <= 0) return;
    const int F = tiles / units, R = tiles - F * units;
    if (R == 0) return;
    const int s_max = std::min(units / R, q.Kb / 2);
    int S = 1;
    if (forced > 0) {
        S = std::min(forced, s_max);
    } else {
        const double fixed = F > 0 ? 26.0 : 20.0;
        double best = 5.0;
        for (int s = 2; s <= s_max; ++s) {
            const double gain = q.Kb * (1.0 - 1.0 / s) - 2.7 * (s - 1) - fixed;
            if (gain > best) {
                best = gain;
                S = s;
            }
        }
    }
    if (S < 2) return;
    q.tail_first = F * units;
    q.tail_s = S;
    q.tail_units = R * S;
    q.ws = ws;
    q.flags = flags;
    q.epoch = epoch;
    q.test_skip_tail = test_skip_tail_flags();
}

template <int BN, int STAGES, int KIND, bool PAIR, bool A_MN = false, bool B_MN = false, bool TAIL = false>
dg_status launch_gemm(const GemmMaps &mp, const dg::GemmParams &p_in, int tiles, const DeviceInfo *di,
                      cudaStream_t st, float *ws = nullptr, int *flags = nullptr, unsigned *epoch = nullptr) {
    constexpr bool PAIR_LIST = PAIR && KIND == dg::KIND_CONTIGUOUS;
    using L = dg::GemmLayout<BN, STAGES, PAIR, PAIR_LIST, KIND == dg::KIND_KGROUPED>;
    auto kern = dg::gemm_kernel<BN, STAGES, KIND, PAIR, A_MN, B_MN, TAIL>;
    static KernelInfo info[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    Launch ln(dim3(1, 1, 1), dim3(dg::GEMM_THREADS, 1, 1), L::ALLOC, st, PAIR ? 2 : 1);
    cudaLaunchConfig_t &cfg = ln.cfg;
    KernelInfo &ki = info[dev];
    if (!ki.ready.load()) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ki.ready.load()) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) != cudaSuccess)
                return DG_ERR_CUDA;
            if (PAIR) {
                cfg.gridDim = dim3(2 * (di->sm_count / 2), 1, 1);
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return DG_ERR_CUDA;
                ki.max_clusters = n;
            }
            ki.ready.store(1);
        }
    }
    const int units = PAIR ? ki.max_clusters : di->sm_count;
    dg::GemmParams p = p_in;
    if constexpr (!TAIL && KIND == dg::KIND_DENSE && !A_MN && !B_MN) {
        plan_tail(p, tiles, units, ws, flags, epoch);
        if (p.tail_s > 1) {
            // the whole waves (if any) in this kernel, then the last wave's pieces in the TAIL
            // instantiation, launched behind it on the stream
            if (p.tail_first > 0) {
                p.tail_early = 1;
                p.num_tiles = p.tail_first;
                cfg.gridDim = dim3(PAIR ? 2 * units : units, 1, 1);
                const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mp.a, mp.b, mp.sfa, mp.c, mp.d, mp.sfb, p);
                if (e != cudaSuccess) return from_cuda(e);
            }
            const dg_status r = launch_gemm<BN, STAGES, KIND, PAIR, A_MN, B_MN, true>(mp, p, p.tail_units, di, st);
            std::snprintf(t_kernel_name, sizeof(t_kernel_name),
                          PAIR ? "gemm_kernel (CTA pairs, last-wave split %d)" : "gemm_kernel (last-wave split %d)",
                          p.tail_s);
            t_last_kernel = t_kernel_name;
            t_last_launches = p.tail_first > 0 ? 2 : 1;
            return r;
        }
    }
    const int n_units = tiles < units ? tiles : units;
    if (n_units <= 0) return DG_OK;
    cfg.gridDim = dim3(PAIR ? 2 * n_units : n_units, 1, 1);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mp.a, mp.b, mp.sfa, mp.c, mp.d, mp.sfb, p);
    t_last_kernel = PAIR ? "gemm_kernel (CTA pairs)" : "gemm_kernel";
    t_last_launches = 1;
    return from_cuda(e);
}

// Tile-shape choice. Pairs of CTAs (256-row tiles, cta_group::2) for every layout with more
// than 128 rows per group; single CTAs (128-row tiles) otherwise. 256 columns per tile unless
// N <= 128. Stages fill the shared-memory budget.
template <int KIND, bool A_MN = false, bool B_MN = false>
dg_status run_gemm(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                   const int32_t *layout, const int32_t *masked_m, int rows, int N, int K, int G, cudaStream_t st,
                   int expected_m = 0) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dg::GemmParams p{};
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.Kb = K / 128;
    p.Nb = (N + 127) / 128;
    p.ld_sfa = pad4(rows);
    p.has_c = c != nullptr;
    p.sfa = sfa;
    p.sfb = sfb;
    p.grouped_layout = layout;
    p.masked_m = masked_m;
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.err = di->err;
    p.timeout_ns = wait_limit_ns();
    p.test_skip_release = test_skip_release() == 1;
    p.one_issuer = one_issuer();
    const bool batched = KIND == dg::KIND_MASKED;
    const int fbn = forced_bn();
    const int bn = fbn ? fbn : (N > 128 ? 256 : 128);
    const int fpair = forced_pair();
    // masked: the expected rows per expert choose the tile height (CTA pairs of 256 rows only
    // when a typical expert fills more than one 128-row tile; measured on G = 16 experts of
    // N x K = 4096 x 7168 and 7168 x 2048: expected_m 32 and 96 run 23 % faster on 128-row
    // tiles, expected_m 192 within 3 % either way)
    const int hint_rows = KIND == dg::KIND_MASKED && expected_m > 0 ? expected_m : rows;
    bool pair = fpair >= 0 ? fpair == 1 : hint_rows > 128;
    if (KIND == dg::KIND_CONTIGUOUS && rows / 128 > dg::MAX_PAIR_BLOCKS) pair = false;
    if (bn != 256) pair = false;                       // pairs are built for 256-column tiles
    GemmMaps mp;
    const int m_units = (rows + (pair ? 255 : 127)) / (pair ? 256 : 128);
    p.n_blocks = (N + bn - 1) / bn;
    int tiles;
    if (KIND == dg::KIND_MASKED) {
        tiles = G * m_units * p.n_blocks;                 // upper bound; the kernel reads masked_m
    } else if (KIND == dg::KIND_CONTIGUOUS && pair) {
        tiles = (rows / 128 / 2 + G) * p.n_blocks;        // upper bound on expert-local pairs
    } else {
        tiles = m_units * p.n_blocks;
    }
    p.num_tiles = (KIND == dg::KIND_MASKED || (KIND == dg::KIND_CONTIGUOUS && pair)) ? 0 : tiles;
    const int b_rows = pair ? bn / 2 : bn;
    // dense and contiguous D rows in whole 64-column blocks: one TMA copy per epilogue slab
    p.cd_blocks = !batched && N % 64 == 0;
    OperandMajor om;
    om.a_mn = A_MN;
    om.b_mn = B_MN;
    if (!build_maps(mp, a, sfa, b, c, d, rows, N, K, G, b_rows, batched, p.cd_blocks ? bn / 128 : 0, om))
        return DG_ERR_INVALID_ARG;
    // dense: the stream's flag workspace for a last-wave split (none: no split)
    float *ws = nullptr;
    int *flags = nullptr;
    unsigned *epoch = nullptr;
    StreamWorkspace w;
    int dev = 0;
    if (KIND == dg::KIND_DENSE && forced_tail_split() != 0 && cudaGetDevice(&dev) == cudaSuccess &&
        stream_workspace(dev, di->sm_count, st, &w)) {
        ws = w.ws;
        flags = w.flags;
        epoch = reinterpret_cast<unsigned *>(w.flags + w.slots);
    }
    if (pair) {
        return launch_gemm<256, 4, KIND, true, A_MN, B_MN>(mp, p, tiles, di, st, ws, flags, epoch);
    }
    if (bn == 256) return launch_gemm<256, 3, KIND, false, A_MN, B_MN>(mp, p, tiles, di, st, ws, flags, epoch);
    return launch_gemm<128, 5, KIND, false, A_MN, B_MN>(mp, p, tiles, di, st, ws, flags, epoch);
}

// K-grouped TN GEMM (the MoE weight gradient): A [sum_K][M] and B [sum_K][N], both MN-major,
// K split into G groups, one fp32 scale per channel per 128 tokens for both operands, fp32 D.
dg_status run_kgrouped(const void *a, const float *sfa, const void *b, const float *sfb, const float *c, float *d,
                       const int32_t *ks_device, int sum_k, int G, int M, int N, cudaStream_t st) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dg::GemmParams p{};
    p.M = M;
    p.N = N;
    p.K = sum_k;
    p.G = G;
    p.Kb = sum_k / 128;
    p.Nb = (N + 127) / 128;
    p.ld_sfa = pad4(M);
    p.has_c = 0;
    p.sfa = sfa;
    p.sfb = sfb;
    p.ks = ks_device;
    p.d32 = d;
    p.c32 = c;
    p.err = di->err;
    p.timeout_ns = wait_limit_ns();
    p.one_issuer = one_issuer();
    const int fbn = forced_bn();
    const int bn = fbn ? fbn : (N > 128 ? 256 : 128);
    const int fpair = forced_pair();
    bool pair = fpair >= 0 ? fpair == 1 : M > 128;
    if (bn != 256) pair = false;
    const int m_units = (M + (pair ? 255 : 127)) / (pair ? 256 : 128);
    p.n_blocks = (N + bn - 1) / bn;
    const long long tiles = static_cast<long long>(G) * m_units * p.n_blocks;
    if (tiles > (1 << 30)) return DG_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tiles);
    const int b_rows = pair ? bn / 2 : bn;
    GemmMaps mp;
    // With no token at all every group is empty and D = C: the kernel then loads nothing (the
    // device offsets are clamped to p.Kb = 0), but a tensor map needs a non-empty extent.
    const int k_ext = sum_k > 0 ? sum_k : 128;
    {   // A [sum_K][M], B [sum_K][N] (one group of B), MN-major
        OperandMajor om;
        om.a_mn = om.b_mn = true;
        if (!build_maps(mp, a, sfa, b, nullptr, d, M, N, k_ext, 1, b_rows, false, 0, om)) return DG_ERR_INVALID_ARG;
    }
    {   // per-column B scales fp32 [sum_K/128][pad4(N)], box bn x 1
        const uint64_t dims[2] = {static_cast<uint64_t>(pad4(N)), static_cast<uint64_t>(k_ext / 128)};
        const uint64_t str[1] = {static_cast<uint64_t>(pad4(N)) * 4};
        const uint32_t box[2] = {static_cast<uint32_t>(bn), 1};
        if (!encode(&mp.sfb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, sfb, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return DG_ERR_INVALID_ARG;
    }
    mp.c = mp.d = mp.sfa;   // C and D are fp32 and written directly, not through TMA
    constexpr int KG = dg::KIND_KGROUPED;
    if (pair) return launch_gemm<256, 4, KG, true, true, true>(mp, p, static_cast<int>(tiles), di, st);
    if (bn == 256) return launch_gemm<256, 3, KG, false, true, true>(mp, p, static_cast<int>(tiles), di, st);
    return launch_gemm<128, 5, KG, false, true, true>(mp, p, static_cast<int>(tiles), di, st);
}

// ---- few-row GEMMs: swapped operands, split-K over a cluster (dg_gemm_swap.cuh) ----
struct SwapMaps {
    CUtensorMap w, x, sfa, c;
};

bool build_swap_maps(SwapMaps &mp, const void *a, const float *sfa, const void *b, const void *c, int rows, int N,
                     int K, int G, int tn, bool batched) {
    const uint64_t Gg = static_cast<uint64_t>(G);
    {   // weights: e4m3 [G][N][K], box 128 x 128 x 1
        const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(K) * N};
        const uint32_t box[3] = {128, 128, 1};
        if (!encode(&mp.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
    }
    {   // activations: e4m3 [G?][rows][K], box 128 x tn
        const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(K) * rows};
        const uint32_t box[3] = {128, static_cast<uint32_t>(tn), 1};
        if (!encode(&mp.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, batched ? 3 : 2, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    }
    {   // sfa: fp32 [G?][Kb][pad4(rows)], box tn x 1
        const uint64_t Kb = static_cast<uint64_t>(K / 128), ld = static_cast<uint64_t>(pad4(rows));
        const uint64_t dims[3] = {ld, Kb, Gg};
        const uint64_t str[2] = {ld * 4, ld * 4 * Kb};
        const uint32_t box[3] = {static_cast<uint32_t>(tn), 1, 1};
        if (!encode(&mp.sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, batched ? 3 : 2, sfa, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    }
    if (c) {   // C: bf16 [G?][rows][N], box 128 columns x tn rows (no swizzle: 256-byte rows)
        const uint64_t dims[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(rows), Gg};
        const uint64_t str[2] = {static_cast<uint64_t>(N) * 2, static_cast<uint64_t>(N) * 2 * rows};
        const uint32_t box[3] = {128, static_cast<uint32_t>(tn), 1};
        if (!encode(&mp.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, batched ? 3 : 2, c, dims, str, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    } else {
        mp.c = mp.sfa;   // never read when has_c == 0
    }
    return true;
}

template <int TN, int STAGES, int KIND>
dg_status launch_swap(const SwapMaps &mp, const dg::SwapParams &p, long long tiles, const DeviceInfo *di,
                      cudaStream_t st) {
    using L = dg::SwapLayout<TN, STAGES>;
    const long long units = tiles * p.Kb;
    auto kern = dg::gemm_swap_kernel<TN, STAGES, KIND>;
    static std::atomic<int> ready[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    if (!ready[dev].load()) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ready[dev].load()) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) != cudaSuccess)
                return DG_ERR_CUDA;
            ready[dev].store(1);
        }
    }
    // one CTA per SM (the shared memory allows one); the kernel cuts the units over as many of
    // them as its per-tile partial limit allows
    const long long grid = units < di->sm_count ? units : di->sm_count;
    if (grid <= 0) return DG_OK;
    Launch ln(dim3(static_cast<unsigned>(grid), 1, 1), dim3(L::THREADS, 1, 1), L::ALLOC, st);
    t_last_kernel = "gemm_swap_kernel (stream-K)";
    t_last_launches = 1;
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, kern, mp.w, mp.x, mp.sfa, mp.c, p));
}

// The few-row GEMM with the given stream-K scratch: partials for `slots` >= sm_count CTAs, then
// `slots` flags followed by the two epoch words.
template <int KIND>
dg_status run_swap_with(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                        const int32_t *masked_m, int expected_m, int rows, int N, int K, int G, cudaStream_t st,
                        const DeviceInfo *di, float *ws, int *flags, int slots) {
    const bool batched = KIND == dg::KIND_MASKED;
    const int hint = batched ? (expected_m > 0 ? expected_m : rows) : rows;
    const int tn = hint <= 64 ? 64 : 128;
    dg::SwapParams p{};
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.Kb = K / 128;
    p.Nb = (N + 127) / 128;
    p.ld_sfa = pad4(rows);
    p.n_tiles = (N + 127) / 128;
    p.m_tiles = (rows + tn - 1) / tn;
    p.has_c = c != nullptr;
    p.sfb = sfb;
    p.masked_m = masked_m;
    p.c = static_cast<const __nv_bfloat16 *>(c);
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.ws = ws;
    p.flags = flags;
    p.epoch = reinterpret_cast<unsigned *>(flags + slots);
    p.err = di->err;
    p.timeout_ns = wait_limit_ns();
    p.test_skip_release = test_skip_streamk_flags() ? 3 : 0;
    p.one_issuer = one_issuer();
    // the largest possible tile set: masked groups may use fewer
    const long long tiles = static_cast<long long>(batched ? G : 1) * p.m_tiles * p.n_tiles;
    SwapMaps mp;
    if (!build_swap_maps(mp, a, sfa, b, c, rows, N, K, G, tn, batched)) return DG_ERR_INVALID_ARG;
    if (tn == 64) return launch_swap<64, 8, KIND>(mp, p, tiles, di, st);
    return launch_swap<128, 5, KIND>(mp, p, tiles, di, st);
}

// The few-row GEMM with the per-stream workspace. Returns DG_ERR_UNSUPPORTED (nothing
// launched) when no workspace is available for `st`.
template <int KIND>
dg_status run_swap(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                   const int32_t *masked_m, int expected_m, int rows, int N, int K, int G, cudaStream_t st) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    StreamWorkspace w;
    if (!stream_workspace(dev, di->sm_count, st, &w)) return DG_ERR_UNSUPPORTED;
    return run_swap_with<KIND>(a, sfa, b, sfb, c, d, masked_m, expected_m, rows, N, K, G, st, di, w.ws, w.flags,
                               w.slots);
}

// ---- few-row GEMMs: cluster split-K (dg_gemm_splitk.cuh) ----
// Per (kernel, device): how many clusters of each size S = 1, 2, 4, 8, 16 can be resident.
constexpr int kSplitSizes[7] = {1, 2, 3, 4, 6, 8, 16};   // cluster sizes the kernel takes
struct SplitInfo {
    std::atomic<int> ready{0};
    int max_clusters[7] = {0, 0, 0, 0, 0, 0, 0};
};

template <int TN, int STAGES, int KIND>
dg_status launch_splitk(const SwapMaps &mp, const dg::SwapParams &p, int tiles, const DeviceInfo *di,
                        cudaStream_t st) {
    using L = dg::SplitLayout<TN, STAGES>;
    auto kern = dg::gemm_splitk_kernel<TN, STAGES, KIND>;
    static SplitInfo info[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    SplitInfo &si = info[dev];
    if (!si.ready.load()) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!si.ready.load()) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) != cudaSuccess)
                return DG_ERR_CUDA;
            const bool big = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
            si.max_clusters[0] = di->sm_count;
            for (int i = 1; i < 7; ++i) {
                const int S = kSplitSizes[i];
                if (S > 8 && !big) break;
                Launch ln(dim3(static_cast<unsigned>(S * (di->sm_count / S)), 1, 1), dim3(L::THREADS, 1, 1), L::ALLOC, st, S);
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, kern, &ln.cfg) != cudaSuccess) {
                    cudaGetLastError();
                    n = 0;
                }
                si.max_clusters[i] = n;
            }
            si.ready.store(1);
        }
    }
    // Cluster size: the modelled time (cycles) of the busiest CTA, rounds x (its K blocks at the
    // rate one SM streams from HBM, ~26 B/clk with this ring depth, which is also every SM's
    // share of the full HBM rate) plus one reduction tail per round.
    const double kb_bytes = 128.0 * 128 + TN * 128;
    int best_s = 0, best_c = 0;
    double best_t = 0;
    for (int i = 0; i < 7; ++i) {
        const int S = kSplitSizes[i];
        if (S > p.Kb || si.max_clusters[i] <= 0) continue;
        const int C = si.max_clusters[i] < tiles ? si.max_clusters[i] : tiles;
        const int rounds = (tiles + C - 1) / C;
        const double per_cta = static_cast<double>(rounds) * ((p.Kb + S - 1) / S);
        const double t = per_cta * kb_bytes / 26.0 + (S > 1 ? 3000.0 : 1500.0) * rounds;
        if (best_s == 0 || t < best_t || S == forced_splitk_s()) {
            best_s = S;
            best_c = C;
            best_t = t;
            if (S == forced_splitk_s()) break;
        }
    }
    if (best_s == 0) return DG_ERR_UNSUPPORTED;
    Launch ln(dim3(static_cast<unsigned>(best_c * best_s), 1, 1), dim3(L::THREADS, 1, 1), L::ALLOC, st, best_s, true);
    t_last_kernel = "gemm_splitk_kernel (cluster split-K)";
    t_last_launches = 1;
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, kern, mp.w, mp.x, mp.sfa, p));
}

template <int KIND>
dg_status run_splitk(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                     const int32_t *masked_m, int expected_m, int rows, int N, int K, int G, cudaStream_t st) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    const bool batched = KIND == dg::KIND_MASKED;
    const int hint = batched ? (expected_m > 0 ? expected_m : rows) : rows;
    const int tn = hint <= 64 ? 64 : 128;
    dg::SwapParams p{};
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.Kb = K / 128;
    p.Nb = (N + 127) / 128;
    p.ld_sfa = pad4(rows);
    p.n_tiles = (N + 127) / 128;
    p.m_tiles = (rows + tn - 1) / tn;
    p.has_c = c != nullptr;
    p.sfb = sfb;
    p.masked_m = masked_m;
    p.c = static_cast<const __nv_bfloat16 *>(c);
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.err = di->err;
    p.timeout_ns = wait_limit_ns();
    p.test_skip_release = test_skip_release() == 2 ? 2 : 0;
    p.one_issuer = one_issuer();
    // tiles the cluster count is sized for: the masked layout's real count depends on masked_m,
    // estimated from expected_m
    const int m_est = batched ? (hint + tn - 1) / tn : p.m_tiles;
    const long long tiles = static_cast<long long>(batched ? G : 1) * (m_est < 1 ? 1 : m_est) * p.n_tiles;
    if (tiles > (1 << 30)) return DG_ERR_INVALID_ARG;
    SwapMaps mp;
    if (!build_swap_maps(mp, a, sfa, b, nullptr, rows, N, K, G, tn, batched)) return DG_ERR_INVALID_ARG;
    if (tn == 64) return launch_splitk<64, 7, KIND>(mp, p, static_cast<int>(tiles), di, st);
    return launch_splitk<128, 4, KIND>(mp, p, static_cast<int>(tiles), di, st);
}

dg_status check_gemm_common(const void *a, const float *sfa, const void *b, const float *sfb, const void *c,
                            const void *d, int N, int K) {
    if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K % 128 != 0 || N % 8 != 0) return DG_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(sfa) || !aligned16(sfb) || !aligned16(d) ||
        (c && !aligned16(c)))
        return DG_ERR_ALIGNMENT;
    return DG_OK;
}

// UE8M0 GEMM: block-scaled MMA with the scales in TMEM (dg_gemm_bs.cuh), one CTA per 128 x 224 tile.
dg_status run_gemm_ue8m0(const void *a, const uint32_t *sfa, const void *b, const uint32_t *sfb, const void *c,
                         void *d, int M, int N, int K, cudaStream_t st) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dg::BsParams p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.Kb = K / 128;
    p.Nb = (N + 127) / 128;
    p.Kq = (p.Kb + 3) / 4;
    p.ld_sfa = pad4(M);
    p.m_blocks = (M + 127) / 128;
    p.n_blocks = (N + dg::BS_BN - 1) / dg::BS_BN;
    const long long tiles = static_cast<long long>(p.m_blocks) * p.n_blocks;
    if (tiles > (1 << 30)) return DG_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tiles);
    p.has_c = c != nullptr;
    p.sfa = sfa;
    p.sfb = sfb;
    p.c = static_cast<const __nv_bfloat16 *>(c);
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.err = di->err;
    p.timeout_ns = wait_limit_ns();
    CUtensorMap tm_a, tm_b;
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
        const uint64_t str[1] = {static_cast<uint64_t>(K)};
        const uint32_t box[2] = {128, 128};
        if (!encode(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return DG_ERR_INVALID_ARG;
    }
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
        const uint64_t str[1] = {static_cast<uint64_t>(K)};
        const uint32_t box[2] = {128, static_cast<uint32_t>(dg::BS_BN)};
        if (!encode(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return DG_ERR_INVALID_ARG;
    }
    static std::atomic<int> ready[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    if (!ready[dev].load()) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ready[dev].load()) {
            if (cudaFuncSetAttribute(dg::gemm_bs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     dg::BsLayout::ALLOC) != cudaSuccess)
                return DG_ERR_CUDA;
            ready[dev].store(1);
        }
    }
    const int grid = p.num_tiles < di->sm_count ? p.num_tiles : di->sm_count;
    if (grid <= 0) return DG_OK;
    Launch ln(dim3(static_cast<unsigned>(grid), 1, 1), dim3(dg::BS_THREADS, 1, 1), dg::BsLayout::ALLOC, st);
    t_last_kernel = "gemm_bs_kernel (UE8M0 block-scaled MMA)";
    t_last_launches = 1;
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::gemm_bs_kernel, tm_a, tm_b, p));
}

// NN / TN / TT: the dense GEMM with MN-major operands, on the tile kernel for every M.
template <bool A_MN, bool B_MN>
dg_status gemm_layout(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d, int M,
                      int N, int K, void *stream) {
    if (M < 0) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, sfa, b, sfb, c, d, N, K);
    if (s != DG_OK) return s;
    if ((A_MN && M % 16 != 0) || (B_MN && N % 16 != 0)) return DG_ERR_INVALID_ARG;   // 16-byte rows
    if (M == 0) return DG_OK;
    return run_gemm<dg::KIND_DENSE, A_MN, B_MN>(a, sfa, b, sfb, c, d, nullptr, nullptr, M, N, K, 1,
                                                static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

dg_status dg_fp8_gemm_nt(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                         int M, int N, int K, void *stream) {
    if (M < 0) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, sfa, b, sfb, c, d, N, K);
    if (s != DG_OK) return s;
    if (M == 0) return DG_OK;
    const int fs = forced_swap();
    if (fs >= 0 ? fs == 1 && M <= 128 : M <= 128) {
        const dg_status r = use_streamk(1, 1, N, K)
                                ? run_swap<dg::KIND_DENSE>(a, sfa, b, sfb, c, d, nullptr, 0, M, N, K, 1,
                                                           static_cast<cudaStream_t>(stream))
                                : run_splitk<dg::KIND_DENSE>(a, sfa, b, sfb, c, d, nullptr, 0, M, N, K, 1,
                                                             static_cast<cudaStream_t>(stream));
        if (r != DG_ERR_UNSUPPORTED) return r;
    }
    return run_gemm<dg::KIND_DENSE>(a, sfa, b, sfb, c, d, nullptr, nullptr, M, N, K, 1,
                                    static_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb, const void *c,
                                 void *d, int M, int N, int K, void *stream) {
    if (M < 0) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, sfa, b, sfb, c, d, N, K);
    if (s != DG_OK) return s;
    if (M > 128) return DG_ERR_UNSUPPORTED;
    if (M == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    s = device_info(&di);
    if (s != DG_OK) return s;
    if (di->sm_count > kStaticSlots) return DG_ERR_UNSUPPORTED;
    return run_swap_with<dg::KIND_DENSE>(a, sfa, b, sfb, c, d, nullptr, 0, M, N, K, 1,
                                         static_cast<cudaStream_t>(stream), di, di->static_ws, di->static_flags,
                                         kStaticSlots);
}

dg_status dg_fp8_gemm_nt_ue8m0(const void *a, const uint32_t *sfa, const void *b, const uint32_t *sfb, const void *c,
                               void *d, int M, int N, int K, void *stream) {
    if (M < 0) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, reinterpret_cast<const float *>(sfa), b, reinterpret_cast<const float *>(sfb), c,
                                    d, N, K);
    if (s != DG_OK) return s;
    if (N % 16 != 0) return DG_ERR_INVALID_ARG;
    if (M == 0) return DG_OK;
    return run_gemm_ue8m0(a, sfa, b, sfb, c, d, M, N, K, static_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_nn(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                         int M, int N, int K, void *stream) {
    return gemm_layout<false, true>(a, sfa, b, sfb, c, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_tn(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                         int M, int N, int K, void *stream) {
    return gemm_layout<true, true>(a, sfa, b, sfb, c, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_tt(const void *a, const float *sfa, const void *b, const float *sfb, const void *c, void *d,
                         int M, int N, int K, void *stream) {
    return gemm_layout<true, false>(a, sfa, b, sfb, c, d, M, N, K, stream);
}

dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                              const float *c, float *d, const int *ks, const int32_t *ks_device,
                                              int G, int M, int N, void *stream) {
    if (!a || !sfa || !b || !sfb || !d || !ks || !ks_device || G <= 0 || G > dg::MAX_KGROUPS || M < 0 || N <= 0)
        return DG_ERR_INVALID_ARG;
    if (M % 16 != 0 || N % 16 != 0) return DG_ERR_INVALID_ARG;            // 16-byte rows of A and B
    if (!aligned16(a) || !aligned16(b) || !aligned16(sfa) || !aligned16(sfb) || !aligned16(d) ||
        (c && !aligned16(c)) || !aligned16(ks_device))
        return DG_ERR_ALIGNMENT;
    long long sum_k = 0;
    for (int g = 0; g < G; ++g) {
        if (ks[g] < 0 || ks[g] % 128 != 0) return DG_ERR_INVALID_ARG;
        sum_k += ks[g];
    }
    if (sum_k > (1LL << 30)) return DG_ERR_INVALID_ARG;
    if (M == 0) return DG_OK;
    return run_kgrouped(a, sfa, b, sfb, c, d, ks_device, static_cast<int>(sum_k), G, M, N,
                        static_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                              const void *c, void *d, const int32_t *grouped_layout, int M_sum,
                                              int N, int K, int G, void *stream) {
    if (M_sum < 0 || M_sum % 128 != 0 || G <= 0 || !grouped_layout) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, sfa, b, sfb, c, d, N, K);
    if (s != DG_OK) return s;
    if (M_sum == 0) return DG_OK;
    return run_gemm<dg::KIND_CONTIGUOUS>(a, sfa, b, sfb, c, d, grouped_layout, nullptr, M_sum, N, K, G,
                                         static_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void *a, const float *sfa, const void *b, const float *sfb,
                                          const void *c, void *d, const int32_t *masked_m, int expected_m, int G,
                                          int M_max, int N, int K, void *stream) {
    if (G <= 0 || M_max < 0 || !masked_m || expected_m < 0) return DG_ERR_INVALID_ARG;
    dg_status s = check_gemm_common(a, sfa, b, sfb, c, d, N, K);
    if (s != DG_OK) return s;
    if (M_max == 0) return DG_OK;
    if (forced_swap() == 1) {   // the tile kernels stream the masked page shapes faster
        const dg_status r = use_streamk(G, 1, N, K)
                                ? run_swap<dg::KIND_MASKED>(a, sfa, b, sfb, c, d, masked_m, expected_m, M_max, N, K,
                                                            G, static_cast<cudaStream_t>(stream))
                                : run_splitk<dg::KIND_MASKED>(a, sfa, b, sfb, c, d, masked_m, expected_m, M_max, N,
                                                              K, G, static_cast<cudaStream_t>(stream));
        if (r != DG_ERR_UNSUPPORTED) return r;
    }
    return run_gemm<dg::KIND_MASKED>(a, sfa, b, sfb, c, d, nullptr, masked_m, M_max, N, K, G,
                                     static_cast<cudaStream_t>(stream), expected_m);
}

dg_status dg_transform_sf(const float *sf_kmajor, float *sf_mnmajor, int batch, int MN, int Kb, void *stream) {
    if (!sf_kmajor || !sf_mnmajor || batch < 0 || MN < 0 || Kb < 0 || batch > 65535) return DG_ERR_INVALID_ARG;
    if (batch == 0 || Kb == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    const int ld = pad4(MN);
    if (ld == 0) return DG_OK;
    dim3 grid((ld + 31) / 32, (Kb + 31) / 32, batch);
    Launch ln(grid, dim3(32, 8, 1), 0, static_cast<cudaStream_t>(stream));
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::transform_sf_kernel, sf_kmajor, sf_mnmajor, MN, Kb, ld));
}

dg_status dg_cast_fp8_per_token(const void *x, void *q, float *sfa, int batch, int M, int K, void *stream) {
    if (!x || !q || !sfa || batch < 0 || M < 0 || K <= 0 || K % 128 != 0 || batch > 65535) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfa)) return DG_ERR_ALIGNMENT;
    if (batch == 0 || M == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    const int Kb = K / 128;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long big_blocks = static_cast<long long>((M + 31) / 32) * ((Kb + 3) / 4) * batch;
    if (big_blocks >= 2LL * di->sm_count) {   // enough 32 x 4 blocks for two per SM
        dim3 grid((M + 31) / 32, (Kb + 3) / 4, batch);
        if (grid.y > 65535) return DG_ERR_INVALID_ARG;
        Launch ln(grid, dim3(256, 1, 1), 0, st);
        return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_token_kernel<32, 4>,
                                            static_cast<const __nv_bfloat16 *>(x), static_cast<uint8_t *>(q), sfa, M,
                                            K, pad4(M), static_cast<const int32_t *>(nullptr), 0,
                                            static_cast<int *>(nullptr)));
    } else {
        dim3 grid((M + 7) / 8, (Kb + 1) / 2, batch);
        if (grid.y > 65535) return DG_ERR_INVALID_ARG;
        Launch ln(grid, dim3(256, 1, 1), 0, st);
        return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_token_kernel<8, 2>,
                                            static_cast<const __nv_bfloat16 *>(x), static_cast<uint8_t *>(q), sfa, M,
                                            K, pad4(M), static_cast<const int32_t *>(nullptr), 0,
                                            static_cast<int *>(nullptr)));
    }
}

dg_status dg_cast_fp8_per_block(const void *x, void *q, float *sfb, int batch, int N, int K, void *stream) {
    if (!x || !q || !sfb || batch < 0 || N < 0 || K <= 0 || K % 128 != 0 || batch > 65535) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfb)) return DG_ERR_ALIGNMENT;
    if (batch == 0 || N == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dim3 grid(K / 128, (N + 127) / 128, batch);
    if (grid.y > 65535) return DG_ERR_INVALID_ARG;
    Launch ln(grid, dim3(256, 1, 1), 0, static_cast<cudaStream_t>(stream));
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_block_kernel<false>, static_cast<const __nv_bfloat16 *>(x),
                                        static_cast<uint8_t *>(q), sfb, N, K));
}

dg_status dg_cast_fp8_per_token_scatter(const void *x, const int32_t *dst_rows, void *q, float *sfa, int T, int M_sum,
                                       int K, void *stream) {
    if (!x || !dst_rows || !q || !sfa || T < 0 || M_sum < 0 || K <= 0 || K % 128 != 0) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfa)) return DG_ERR_ALIGNMENT;
    if (T == 0 || M_sum == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    const int Kb = K / 128;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long big_blocks = static_cast<long long>((T + 31) / 32) * ((Kb + 3) / 4);
    if (big_blocks >= 2LL * di->sm_count) {
        dim3 grid((T + 31) / 32, (Kb + 3) / 4, 1);
        if (grid.y > 65535) return DG_ERR_INVALID_ARG;
        Launch ln(grid, dim3(256, 1, 1), 0, st);
        return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_token_kernel<32, 4, false, true>,
                                            static_cast<const __nv_bfloat16 *>(x), static_cast<uint8_t *>(q), sfa, T, K,
                                            pad4(M_sum), dst_rows, M_sum, di->err));
    }
    dim3 grid((T + 7) / 8, (Kb + 1) / 2, 1);
    if (grid.y > 65535) return DG_ERR_INVALID_ARG;
    Launch ln(grid, dim3(256, 1, 1), 0, st);
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_token_kernel<8, 2, false, true>,
                                        static_cast<const __nv_bfloat16 *>(x), static_cast<uint8_t *>(q), sfa, T, K,
                                        pad4(M_sum), dst_rows, M_sum, di->err));
}

dg_status dg_cast_fp8_per_token_ue8m0(const void *x, void *q, uint32_t *sfa, int batch, int M, int K, void *stream) {
    if (!x || !q || !sfa || batch < 0 || M < 0 || K <= 0 || K % 128 != 0 || batch > 65535) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfa)) return DG_ERR_ALIGNMENT;
    if (batch == 0 || M == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    const int Kq4 = (K / 128 + 3) / 4 * 4;             // the bytes of every packed word are written
    dim3 grid((M + 31) / 32, Kq4 / 4, batch);
    if (grid.y > 65535) return DG_ERR_INVALID_ARG;
    Launch ln(grid, dim3(256, 1, 1), 0, static_cast<cudaStream_t>(stream));
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_token_kernel<32, 4, true>,
                                        static_cast<const __nv_bfloat16 *>(x), static_cast<uint8_t *>(q),
                                        reinterpret_cast<float *>(sfa), M, K, pad4(M),
                                        static_cast<const int32_t *>(nullptr), 0, static_cast<int *>(nullptr)));
}

dg_status dg_cast_fp8_per_block_ue8m0(const void *x, void *q, uint32_t *sfb, int batch, int N, int K, void *stream) {
    if (!x || !q || !sfb || batch < 0 || N < 0 || K <= 0 || K % 128 != 0 || batch > 65535) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sfb)) return DG_ERR_ALIGNMENT;
    if (batch == 0 || N == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dim3 grid(K / 128, (N + 127) / 128, batch);
    if (grid.y > 65535) return DG_ERR_INVALID_ARG;
    Launch ln(grid, dim3(256, 1, 1), 0, static_cast<cudaStream_t>(stream));
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_block_kernel<true>, static_cast<const __nv_bfloat16 *>(x),
                                        static_cast<uint8_t *>(q), reinterpret_cast<float *>(sfb), N, K));
}

dg_status dg_cast_fp8_per_channel(const void *x, void *q, float *sf, int T, int C, void *stream) {
    if (!x || !q || !sf || T < 0 || C < 0 || T % 128 != 0 || C % 8 != 0) return DG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return DG_ERR_ALIGNMENT;
    if (T == 0 || C == 0) return DG_OK;
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    dim3 grid((C + 127) / 128, T / 128, 1);
    if (grid.y > 65535) return DG_ERR_INVALID_ARG;
    Launch ln(grid, dim3(256, 1, 1), 0, static_cast<cudaStream_t>(stream));
    return from_cuda(cudaLaunchKernelEx(&ln.cfg, dg::cast_per_channel_kernel, static_cast<const __nv_bfloat16 *>(x),
                                        static_cast<uint8_t *>(q), sf, T, C, pad4(C)));
}

int dg_sf_ld(int mn) { return mn <= 0 ? 0 : pad4(mn); }

dg_status dg_get_device_error(void *stream) {
    const DeviceInfo *di = nullptr;
    dg_status s = device_info(&di);
    if (s != DG_OK) return s;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DG_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, di->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DG_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(di->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return DG_ERR_CUDA;
    }
    if (v == dg::ERR_TIMEOUT) return DG_ERR_TIMEOUT;
    if (v != 0) return DG_ERR_DEVICE;
    return DG_OK;
}

const char *dg_last_kernel(void) { return t_last_kernel; }

int dg_last_launch_count(void) { return t_last_launches; }

long long dg_allocated_bytes(void) { return g_allocated.load(); }

const char *dg_status_string(dg_status status) {
    switch (status) {
        case DG_OK: return "DG_OK";
        case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
        case DG_ERR_ALIGNMENT: return "DG_ERR_ALIGNMENT";
        case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
        case DG_ERR_CUDA: return "DG_ERR_CUDA";
        case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
        case DG_ERR_DEVICE: return "DG_ERR_DEVICE";
    }
    return "DG_ERR_UNKNOWN";
}

}  // extern "C"
