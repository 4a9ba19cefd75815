// dg_cast.cuh — FP8 cast-and-scale kernels and the scale-layout transform (sm_100a).
//
// Block-wise scaling (aitangshan.cn/news/1491278 技术原理 §4): every 1×128 slice of a token
// row (activations) or every 128×128 block (weights) gets one fp32 scale s = amax/448 (the
// largest finite E4M3 value is 448; s = 1 for an all-zero block), and each value is stored as
// e4m3(x / s), rounded to nearest-even and saturated to ±448. The division is the IEEE fp32
// one (__fdiv_rn) so that the codes are reproducible bit for bit.
//
// Both casts are HBM-bound streams (2 B read, 1 B written per element): 16-byte vector loads
// through the non-coherent path, warp-shuffle reductions, 8-byte stores, and scales staged
// through shared memory so that the MN-major scale rows are written as whole 128-byte lines.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ float amax8(const float (&f)[8]) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

__device__ __forceinline__ float scale_of(float amax) { return amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f); }

// UE8M0 scale (likun.im/craft/deepgemm §五: SM100 scales are UE8M0, a power of two): the
// smallest s = 2^e >= amax/448 (the fp32 quotient of the fp32 scale), e clamped to [-127, 127],
// stored as the byte e + 127; amax == 0 gives s = 1. The exponent is read off the quotient's
// bits: a normal r = 1.m · 2^(E-127) gives e = E - 127, plus one unless m == 0; a subnormal
// r = m · 2^-149 gives e = ceil(log2 m) - 149.
__device__ __forceinline__ uint32_t ue8m0_of_amax(float amax) {
    if (amax == 0.f) return 127u;
    const uint32_t bits = __float_as_uint(__fdiv_rn(amax, 448.f));
    const int E = static_cast<int>((bits >> 23) & 0xFFu);
    const uint32_t m = bits & 0x7FFFFFu;
    int e = E != 0 ? E - 127 + (m != 0 ? 1 : 0) : (32 - __clz(static_cast<int>(m - 1u))) - 149;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    return static_cast<uint32_t>(e + 127);
}

// The fp32 value 2^(byte - 127) of a UE8M0 byte (2^-127 is the one subnormal).
__device__ __forceinline__ float ue8m0_value(uint32_t b) {
    return b >= 1u ? __uint_as_float(b << 23) : __uint_as_float(1u << 22);
}

// 8 values -> 8 e4m3 codes (x / s, nearest-even, saturating), element 0 in the lowest byte.
__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float2 pr = make_float2(__fdiv_rn(f[4 * h + 2 * i], s), __fdiv_rn(f[4 * h + 2 * i + 1], s));
            const uint32_t two = __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
            acc |= (two & 0xFFFFu) << (16 * i);
        }
        w[h] = acc;
    }
    return make_uint2(w[0], w[1]);
}

// Per-token cast. Block: 256 threads covering ROWS rows x KBS K-slices of one batch entry, in
// "slice halves": a half-warp covers one row's 128-value slice (16 lanes x 8 values, 16 bytes
// per lane). Slice s = i·16 + warp·2 + half (i < ROWS·KBS/16) is row s / KBS, slice s % KBS, so
// that one warp-wide load covers two adjacent slices of one row (512 contiguous bytes). All
// loads of a thread are issued before any is used. Two shapes: 32 x 4 (8 slices per thread,
// many bytes in flight per thread) for many rows, 8 x 2 (one slice per thread, 16x the blocks)
// for few rows, where each block's serial chain of divisions would otherwise set the time.
// Grid: (ceil(M/ROWS), ceil(Kb/KBS), batch).
//
// UE = true: the scale is the UE8M0 power of two (ue8m0_of_amax) and `sfa` receives bytes, four
// K blocks per 32-bit word of the MN-major packed layout [batch][ceil(Kb/4)][ld]: the byte of
// (row, kb) at byte offset ((kb/4)·ld + row)·4 + kb%4 (the bytes of K blocks >= Kb are 127).
//
// SCATTER = true (the cast into the M-grouped contiguous layout): input row t is written to row
// dst[t] of q and sfa (dst[t] = -1 drops it; a value >= out_rows sets the error word and drops
// it), with the scale stored by the row's own lane instead of through shared memory.
template <int ROWS, int KBS, bool UE = false, bool SCATTER = false>
__global__ void __launch_bounds__(256) cast_per_token_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             uint8_t *__restrict__ q, float *__restrict__ sfa,
                                                             int M, int K, int ld,
                                                             const int32_t *__restrict__ dst = nullptr,
                                                             int out_rows = 0, int *err = nullptr) {
    constexpr int PER = ROWS * KBS / 16;
    static_assert(PER >= 1 && ROWS * KBS % 16 == 0 && KBS % 2 == 0, "block shape");
    __shared__ float s_sf[KBS][ROWS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, hl = lane & 15;
    const int Kb = K >> 7;
    const size_t bofs = static_cast<size_t>(blockIdx.z) * M;
    const int r0 = blockIdx.x * ROWS, kb0 = blockIdx.y * KBS;
    pdl_launch_dependents();
    pdl_wait();

    uint4 v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int sl = i * 16 + warp * 2 + half;
        const int row = r0 + sl / KBS, kb = kb0 + sl % KBS;
        if (row < M && kb < Kb)
            v[i] = ldg_stream_v4(x + (bofs + row) * K + kb * 128 + hl * 8);
        else
            v[i] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int sl = i * 16 + warp * 2 + half;
        const int rl = sl / KBS, kbl = sl % KBS;
        const int row = r0 + rl, kb = kb0 + kbl;
        float f[8];
        bf16x8_to_f32(v[i], f);
        float m = amax8(f);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        uint32_t ub = 127u;
        float s;
        if constexpr (UE) {
            ub = ue8m0_of_amax(m);
            s = ue8m0_value(ub);
        } else {
            s = scale_of(m);
        }
        if constexpr (SCATTER) {
            if (row < M && kb < Kb) {
                const int orow = __ldg(dst + row);
                if (orow >= out_rows) {
                    if (hl == 0 && kbl == 0) report_error(err, ERR_DATA);
                } else if (orow >= 0) {
                    *reinterpret_cast<uint2 *>(q + static_cast<size_t>(orow) * K + kb * 128 + hl * 8) = quant8(f, s);
                    if (hl == 0) sfa[static_cast<size_t>(kb) * ld + orow] = s;
                }
            }
            continue;
        }
        if (row < M && kb < Kb) {
            *reinterpret_cast<uint2 *>(q + (bofs + row) * K + kb * 128 + hl * 8) = quant8(f, s);
            if (hl == 0) s_sf[kbl][rl] = UE ? __uint_as_float(ub) : s;
        }
    }
    if constexpr (SCATTER) return;
    __syncthreads();
    if constexpr (UE) {
        // packed bytes; the K blocks of the last word past Kb get 127 (scale 1)
        const int Kq = (Kb + 3) / 4;
        uint8_t *sfb8 = reinterpret_cast<uint8_t *>(sfa);
        for (int idx = threadIdx.x; idx < ROWS * KBS; idx += 256) {
            const int kbl = idx / ROWS, rr = idx % ROWS;
            const int row = r0 + rr, kb = kb0 + kbl;
            if (row < M && kb < 4 * Kq) {
                const uint32_t b = kb < Kb ? __float_as_uint(s_sf[kbl][rr]) : 127u;
                sfb8[((static_cast<size_t>(blockIdx.z) * Kq + kb / 4) * ld + row) * 4 + kb % 4] = static_cast<uint8_t>(b);
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < ROWS * KBS; idx += 256) {
            const int kbl = idx / ROWS, rr = idx % ROWS;
            const int row = r0 + rr, kb = kb0 + kbl;
            if (row < M && kb < Kb) sfa[(static_cast<size_t>(blockIdx.z) * Kb + kb) * ld + row] = s_sf[kbl][rr];
        }
    }
}

// Per-block (128 x 128) cast. Block: 256 threads for one (batch, row block, K slice); thread t
// covers rows nb*128 + t/16 + 16*i (i = 0..7), 16-byte chunk t%16 of the slice. Rows >= N do
// not exist and do not enter the amax. Grid: (Kb, Nb, batch). UE = true: a UE8M0 scale, stored
// as the byte kb%4 of the word [batch][nb][kb/4] of the packed layout (the last block of a row
// of words also writes 127 into the bytes of K blocks >= Kb).
template <bool UE = false>
__global__ void __launch_bounds__(256) cast_per_block_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             uint8_t *__restrict__ q, float *__restrict__ sfb,
                                                             int N, int K) {
    __shared__ float s_red[8];
    const int kb = blockIdx.x, nb = blockIdx.y;
    const int Kb = K >> 7, Nb = gridDim.y;
    const size_t bofs = static_cast<size_t>(blockIdx.z) * N;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int chunk = t & 15, rbase = nb * 128 + (t >> 4);
    pdl_launch_dependents();
    pdl_wait();

    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = rbase + 16 * i;
        v[i] = row < N ? ldg_stream_v4(x + (bofs + row) * K + kb * 128 + chunk * 8) : make_uint4(0, 0, 0, 0);
    }
    float m = 0.f;
    float f[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        bf16x8_to_f32(v[i], f[i]);
        m = fmaxf(m, amax8(f[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = s_red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, s_red[w]);
    const uint32_t ub = UE ? ue8m0_of_amax(m) : 127u;
    const float s = UE ? ue8m0_value(ub) : scale_of(m);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = rbase + 16 * i;
        if (row < N) *reinterpret_cast<uint2 *>(q + (bofs + row) * K + kb * 128 + chunk * 8) = quant8(f[i], s);
    }
    if constexpr (UE) {
        const int Kq = (Kb + 3) / 4;
        uint8_t *w8 = reinterpret_cast<uint8_t *>(sfb) + ((static_cast<size_t>(blockIdx.z) * Nb + nb) * Kq) * 4;
        if (t == 0) w8[kb] = static_cast<uint8_t>(ub);
        if (kb == Kb - 1 && t > 0 && kb + t < 4 * Kq) w8[kb + t] = 127;
    } else {
        if (t == 0) sfb[(static_cast<size_t>(blockIdx.z) * Nb + nb) * Kb + kb] = s;
    }
}

// 8 values with one scale each -> 8 e4m3 codes (x / s, nearest-even, saturating).
__device__ __forceinline__ uint2 quant8_each(const float (&f)[8], const float (&s)[8]) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = 4 * h + 2 * i;
            const float2 pr = make_float2(__fdiv_rn(f[e], s[e]), __fdiv_rn(f[e + 1], s[e + 1]));
            const uint32_t two = __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
            acc |= (two & 0xFFFFu) << (16 * i);
        }
        w[h] = acc;
    }
    return make_uint2(w[0], w[1]);
}

// Per-channel cast along the token dimension (the (1,1,128) recipe of the K-grouped GEMM's
// operands, likun.im §二 k_grouped_fp8_gemm_tn_contiguous): x bf16 [T, C] token-major, one
// scale per channel per 128 tokens, sf fp32 [T/128][ld]. Block: 256 threads for 128 tokens x
// 128 channels; thread t covers channels 8·(t%16) .. +7 of tokens t/16 + 16·i (i = 0..7): eight
// 16-byte loads in flight, a per-channel amax over its 8 tokens, then over the 16 token groups
// (a shuffle across the two half-warps, shared memory across the 8 warps). C % 8 == 0.
// Grid: (ceil(C/128), T/128).
__global__ void __launch_bounds__(256) cast_per_channel_kernel(const __nv_bfloat16 *__restrict__ x,
                                                               uint8_t *__restrict__ q, float *__restrict__ sf,
                                                               int T, int C, int ld) {
    __shared__ float s_red[8][128];
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int c8 = t & 15, tg = t >> 4;
    const int col = blockIdx.x * 128 + c8 * 8;
    const int tok0 = blockIdx.y * 128;
    const bool in = col < C;
    pdl_launch_dependents();
    pdl_wait();

    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = in ? ldg_stream_v4(x + static_cast<size_t>(tok0 + tg + 16 * i) * C + col) : make_uint4(0, 0, 0, 0);
    float f[8][8];
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        bf16x8_to_f32(v[i], f[i]);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[i][e]));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], __shfl_xor_sync(0xFFFFFFFFu, m[e], 16));
    if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s_red[warp][c8 * 8 + e] = m[e];
    }
    __syncthreads();
    float sc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float a = s_red[0][c8 * 8 + e];
#pragma unroll
        for (int w = 1; w < 8; ++w) a = fmaxf(a, s_red[w][c8 * 8 + e]);
        sc[e] = scale_of(a);
    }
    if (in) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint2 *>(q + static_cast<size_t>(tok0 + tg + 16 * i) * C + col) = quant8_each(f[i], sc);
        if (tg == 0) {
            float4 *dst = reinterpret_cast<float4 *>(sf + static_cast<size_t>(blockIdx.y) * ld + col);
            dst[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
            dst[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
        }
    }
}

// [batch][MN][Kb] -> [batch][Kb][ld] through a 32x33 shared tile; entries MN..ld-1 get 0.
// Block (32, 8); grid (ceil(ld/32), ceil(Kb/32), batch).
__global__ void __launch_bounds__(256) transform_sf_kernel(const float *__restrict__ in, float *__restrict__ out,
                                                           int MN, int Kb, int ld) {
    __shared__ float tile[32][33];
    const size_t b = blockIdx.z;
    const int m0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int m = m0 + i, k = k0 + threadIdx.x;
        tile[i][threadIdx.x] = (m < MN && k < Kb) ? in[(b * MN + m) * Kb + k] : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int k = k0 + i, m = m0 + threadIdx.x;
        if (k < Kb && m < ld) out[(b * Kb + k) * ld + m] = tile[threadIdx.x][i];
    }
}

}  // namespace dg
