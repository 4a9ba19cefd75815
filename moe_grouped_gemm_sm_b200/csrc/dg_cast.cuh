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
template <int ROWS, int KBS>
__global__ void __launch_bounds__(256) cast_per_token_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             uint8_t *__restrict__ q, float *__restrict__ sfa,
                                                             int M, int K, int ld) {
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
        const float s = scale_of(m);
        if (row < M && kb < Kb) {
            *reinterpret_cast<uint2 *>(q + (bofs + row) * K + kb * 128 + hl * 8) = quant8(f, s);
            if (hl == 0) s_sf[kbl][rl] = s;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < ROWS * KBS; idx += 256) {
        const int kbl = idx / ROWS, rr = idx % ROWS;
        const int row = r0 + rr, kb = kb0 + kbl;
        if (row < M && kb < Kb) sfa[(static_cast<size_t>(blockIdx.z) * Kb + kb) * ld + row] = s_sf[kbl][rr];
    }
}

// Per-block (128 x 128) cast. Block: 256 threads for one (batch, row block, K slice); thread t
// covers rows nb*128 + t/16 + 16*i (i = 0..7), 16-byte chunk t%16 of the slice. Rows >= N do
// not exist and do not enter the amax. Grid: (Kb, Nb, batch).
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
    const float s = scale_of(m);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int row = rbase + 16 * i;
        if (row < N) *reinterpret_cast<uint2 *>(q + (bofs + row) * K + kb * 128 + chunk * 8) = quant8(f[i], s);
    }
    if (t == 0) sfb[(static_cast<size_t>(blockIdx.z) * Nb + nb) * Kb + kb] = s;
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
