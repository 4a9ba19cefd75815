/*
 * dg_oracle.c — plain, slow, exact CPU oracle for the FP8 block-scaled NT GEMM.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library's product path links, loads or calls this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg do. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * Pages cited (the DeepGEMM write-ups this library is built from):
 *   [likun]   likun.im/craft/deepgemm — "DeepGEMM 一句话"; §一 (what it is: D = C + A·Bᵀ in NT
 *             layout, M-grouped contiguous / masked), §二 (the register_apis list), §五 (the
 *             scale-factor layout caveat: the LHS scales need a TMA-aligned transposed layout).
 *   [aitang]  aitangshan.cn/news/1491278 — §5 "平台核心功能" (grouped GEMM: contiguous and masked
 *             layouts) and 技术原理 §4 "FP8 精度优化的核心" (block-wise scaling: one scale per
 *             block, the product restored by the scale after the multiplication).
 *   [zwt]     zwt0204.github.io "DeepGEMM deep dive" — §"它的核心思路" (grouped layout
 *             constraint; masked layout for decoding).
 *   [OCP]     OCP 8-bit Floating Point Specification (OFP8) rev 1.0, format E4M3: bias 7,
 *             no infinities, S.1111.111 is NaN, largest finite 448, subnormal step 2^-9.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - cast scale s = amax / 448 (fp32, correctly rounded); amax == 0 gives s = 1;
 *   - the value is divided by the scale (y = x / s, fp32 correctly rounded), not multiplied
 *     by a reciprocal;
 *   - y is rounded to nearest-even onto the E4M3 grid (subnormals included) and then clamped
 *     to ±448 with its sign kept; a zero keeps its sign (-0 encodes as 0x80);
 *   - a partial 128-row weight block (N not a multiple of 128) takes amax over its valid rows;
 *   - "multiply by the scale after the GEMM" is applied per 128-wide K block:
 *       D[m,n] = C[m,n] + sum_kb sfa[m,kb]·sfb[n/128,kb]·S_kb[m,n],
 *       S_kb[m,n] = sum_{k in kb} e4m3(A[m,k])·e4m3(B[n,k]);
 *     every S_kb is exact in fp64 (each product is a multiple of 2^-18 below 2^17.6 and 128 of
 *     them need at most 43 significant bits), so the only rounding is in the fp64 scale sum;
 *   - sfa layout: fp32 [Kb][pad4(M)] (MN-major, rows padded to a multiple of 4 so each K-block
 *     row starts 16-byte aligned); sfb layout: fp32 [G][ceil(N/128)][Kb];
 *   - masked rows r >= masked_m[g] are never written; contiguous padding rows (-1) have no
 *     defined value.
 *
 * All entry points return 0 on success and a negative value on bad arguments.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define DGO_BLK 128

static int pad4(int x) { return (x + 3) / 4 * 4; }

/* ---------------------------------------------------------------------------------------- */
/* Number formats                                                                            */
/* ---------------------------------------------------------------------------------------- */

/* [OCP] E4M3 decode: exponent field e (4 bits), mantissa m (3 bits), bias 7.
 * e == 0 -> subnormal m * 2^-9; otherwise (1 + m/8) * 2^(e-7); S.1111.111 -> NaN. */
double dgo_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* [OCP] E4M3 encode of a finite fp32 value with round-to-nearest-even, then saturation to
 * the largest finite magnitude 448 (sign kept). Works on the exact value in double. */
uint8_t dgo_e4m3_encode_satrne(float y) {
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;              /* 448 = 1.75 * 2^8: e=15, m=6 */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: grid step 2^-9, codes 0..8 map to n * 2^-9 (8 is the smallest normal) */
        double n = nearbyint(ldexp(a, 9));          /* exact scaling; ties to even */
        return sign | (uint8_t)n;
    }
    int e;
    frexp(a, &e);                                   /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                         /* a in [2^e, 2^(e+1)) */
    /* grid step at this binade is 2^(e-3); n in [8, 16] after rounding */
    double n = nearbyint(ldexp(a, 3 - e));
    int code = ((e + 7) << 3) + ((int)n - 8);       /* n == 16 carries into the next binade */
    return sign | (uint8_t)code;
}

/* bf16 is the upper half of an IEEE binary32 pattern. */
float dgo_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---------------------------------------------------------------------------------------- */
/* Casts (block-wise scaling: [aitang] 技术原理 §4)                                          */
/* ---------------------------------------------------------------------------------------- */

static float scale_from_amax(float amax) {
    if (amax == 0.0f) return 1.0f;
    return amax / 448.0f;                           /* IEEE fp32 division */
}

/* Per-token cast: for every row m and 128-wide K slice kb,
 *   amax = max |x[m, kb*128 .. kb*128+127]|,  s = amax/448,  q = e4m3_satrne(x / s),
 * with sfa written MN-major: sfa[kb * pad4(M) + m] = s. Padding entries are left untouched.
 * x: bf16 bits [M,K]; q: [M,K]; K must be a multiple of 128. */
int dgo_cast_per_token(const uint16_t *x, int M, int K, uint8_t *q, float *sfa) {
    if (M < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, ld = pad4(M);
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; m++) {
        for (int kb = 0; kb < Kb; kb++) {
            const uint16_t *xs = x + (size_t)m * K + (size_t)kb * DGO_BLK;
            float amax = 0.0f;
            for (int i = 0; i < DGO_BLK; i++) {
                float v = fabsf(dgo_bf16_to_f32(xs[i]));
                if (v > amax) amax = v;
            }
            float s = scale_from_amax(amax);
            for (int i = 0; i < DGO_BLK; i++)
                q[(size_t)m * K + (size_t)kb * DGO_BLK + i] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(xs[i]) / s);
            sfa[(size_t)kb * ld + m] = s;
        }
    }
    return 0;
}

/* Per-token cast straight into the M-grouped contiguous layout (the MoE dispatch of
 * [likun] §二 m_grouped_*_contiguous, whose operand rows are the routed tokens grouped by
 * expert): token t of x [T,K] goes to row dst[t] of q [M_sum,K] and of the MN-major sfa
 * [Kb][pad4(M_sum)], with the per-token cast's rule; dst[t] = -1 drops the token. Rows no token
 * maps to are not written. Every dst[t] must be < M_sum and no row may be the target of two
 * tokens (else -2). */
int dgo_cast_per_token_scatter(const uint16_t *x, const int32_t *dst, int T, int K, int M_sum, uint8_t *q,
                               float *sfa) {
    if (T < 0 || M_sum < 0 || K <= 0 || K % DGO_BLK) return -1;
    for (int t = 0; t < T; t++)
        if (dst[t] < -1 || dst[t] >= M_sum) return -2;
    for (int t = 0; t < T; t++)
        for (int u = t + 1; u < T; u++)
            if (dst[t] >= 0 && dst[t] == dst[u]) return -2;
    int Kb = K / DGO_BLK, ld = pad4(M_sum);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        int m = dst[t];
        if (m < 0) continue;
        for (int kb = 0; kb < Kb; kb++) {
            const uint16_t *xs = x + (size_t)t * K + (size_t)kb * DGO_BLK;
            float amax = 0.0f;
            for (int i = 0; i < DGO_BLK; i++) {
                float v = fabsf(dgo_bf16_to_f32(xs[i]));
                if (v > amax) amax = v;
            }
            float s = scale_from_amax(amax);
            for (int i = 0; i < DGO_BLK; i++)
                q[(size_t)m * K + (size_t)kb * DGO_BLK + i] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(xs[i]) / s);
            sfa[(size_t)kb * ld + m] = s;
        }
    }
    return 0;
}

/* Per-block cast of weights: for every batch g, 128-row block nb and K slice kb,
 * amax over rows [nb*128, min(N, nb*128+128)) and the slice's 128 columns; then as above.
 * x: bf16 bits [batch,N,K]; q: [batch,N,K]; sfb: [batch][ceil(N/128)][Kb]. */
int dgo_cast_per_block(const uint16_t *x, int batch, int N, int K, uint8_t *q, float *sfb) {
    if (batch < 0 || N < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, Nb = (N + DGO_BLK - 1) / DGO_BLK;
#pragma omp parallel for collapse(2) schedule(static)
    for (int g = 0; g < batch; g++) {
        for (int nb = 0; nb < Nb; nb++) {
            int n_end = (nb + 1) * DGO_BLK < N ? (nb + 1) * DGO_BLK : N;
            for (int kb = 0; kb < Kb; kb++) {
                float amax = 0.0f;
                for (int n = nb * DGO_BLK; n < n_end; n++)
                    for (int i = 0; i < DGO_BLK; i++) {
                        float v = fabsf(dgo_bf16_to_f32(x[((size_t)g * N + n) * K + (size_t)kb * DGO_BLK + i]));
                        if (v > amax) amax = v;
                    }
                float s = scale_from_amax(amax);
                for (int n = nb * DGO_BLK; n < n_end; n++)
                    for (int i = 0; i < DGO_BLK; i++) {
                        size_t off = ((size_t)g * N + n) * K + (size_t)kb * DGO_BLK + i;
                        q[off] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(x[off]) / s);
                    }
                sfb[((size_t)g * Nb + nb) * Kb + kb] = s;
            }
        }
    }
    return 0;
}

/* Scale-layout transform ([likun] §五: LHS scales in a TMA-aligned transposed layout):
 * in  fp32 [batch][MN][Kb]  (K-major, one row of Kb scales per token)
 * out fp32 [batch][Kb][pad4(MN)] (MN-major); the pad4 tail of each row is set to 0. */
int dgo_transform_sf(const float *in, int batch, int MN, int Kb, float *out) {
    if (batch < 0 || MN < 0 || Kb < 0) return -1;
    int ld = pad4(MN);
    for (int b = 0; b < batch; b++)
        for (int kb = 0; kb < Kb; kb++)
            for (int i = 0; i < ld; i++)
                out[((size_t)b * Kb + kb) * ld + i] = i < MN ? in[((size_t)b * MN + i) * Kb + kb] : 0.0f;
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* GEMM: D = C + A·Bᵀ, NT ([likun] §一), block-scaled ([aitang] 技术原理 §4)                 */
/* ---------------------------------------------------------------------------------------- */

/* One output element: C + sum_kb (sfa·sfb)·S_kb with S_kb summed exactly in fp64.
 * arow, brow: e4m3 codes of length K; sfa_row(kb) = sfa_base[kb * sfa_ld];
 * sfb_row(kb) = sfb_base[kb]. */
static double dot_row(const uint8_t *arow, const float *sfa_base, size_t sfa_ld,
                      const uint8_t *brow, const float *sfb_base, int Kb, const double *lut) {
    double acc = 0.0;
    for (int kb = 0; kb < Kb; kb++) {
        double s = 0.0;
        const uint8_t *ap = arow + (size_t)kb * DGO_BLK, *bp = brow + (size_t)kb * DGO_BLK;
        for (int i = 0; i < DGO_BLK; i++) s += lut[ap[i]] * lut[bp[i]];
        double scale = (double)sfa_base[(size_t)kb * sfa_ld] * (double)sfb_base[kb];
        acc += scale * s;
    }
    return acc;
}

static void fill_lut(double *lut) {
    for (int c = 0; c < 256; c++) lut[c] = dgo_e4m3_decode((uint8_t)c);
}

/* Dense: A e4m3 [M,K], sfa [Kb][pad4(M)], B e4m3 [N,K], sfb [ceil(N/128)][Kb],
 * C bf16 [M,N] or NULL. Computes the rows listed in `rows` (all rows when rows == NULL,
 * nrows is then ignored) into out[nrows or M][N] as fp64. */
int dgo_gemm_nt(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                const uint16_t *c, int M, int N, int K, const int *rows, int nrows, double *out) {
    if (M < 0 || N < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, R = rows ? nrows : M;
    size_t ld = (size_t)pad4(M);
    double lut[256];
    fill_lut(lut);
    for (int r = 0; r < R; r++) if (rows && (rows[r] < 0 || rows[r] >= M)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; r++) {
        int m = rows ? rows[r] : r;
        for (int n = 0; n < N; n++) {
            double v = dot_row(a + (size_t)m * K, sfa + m, ld, b + (size_t)n * K,
                               sfb + (size_t)(n / DGO_BLK) * Kb, Kb, lut);
            if (c) v += (double)dgo_bf16_to_f32(c[(size_t)m * N + n]);
            out[(size_t)r * N + n] = v;
        }
    }
    return 0;
}

/* M-grouped contiguous ([likun] §二 m_grouped_*_contiguous with grouped_layout; [zwt]):
 * row r of A [M_sum,K] belongs to expert g = grouped_layout[r]; -1 marks a padding row.
 * D[r] = C[r] + A[r]·B[g]ᵀ with B [G,N,K], sfb [G][ceil(N/128)][Kb], sfa [Kb][pad4(M_sum)].
 * Padding rows get NaN in `out` (no defined value). rows/nrows as in dgo_gemm_nt. */
int dgo_m_grouped_contiguous(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                             const uint16_t *c, const int32_t *grouped_layout, int M_sum, int N, int K,
                             int G, const int *rows, int nrows, double *out) {
    if (M_sum < 0 || N < 0 || K <= 0 || K % DGO_BLK || G <= 0) return -1;
    int Kb = K / DGO_BLK, Nb = (N + DGO_BLK - 1) / DGO_BLK, R = rows ? nrows : M_sum;
    size_t ld = (size_t)pad4(M_sum);
    double lut[256];
    fill_lut(lut);
    for (int r = 0; r < R; r++) if (rows && (rows[r] < 0 || rows[r] >= M_sum)) return -2;
    for (int m = 0; m < M_sum; m++) if (grouped_layout[m] >= G) return -3;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; r++) {
        int m = rows ? rows[r] : r;
        int g = grouped_layout[m];
        for (int n = 0; n < N; n++) {
            if (g < 0) { out[(size_t)r * N + n] = NAN; continue; }
            const uint8_t *brow = b + ((size_t)g * N + n) * K;
            const float *sfb_row = sfb + ((size_t)g * Nb + n / DGO_BLK) * Kb;
            double v = dot_row(a + (size_t)m * K, sfa + m, ld, brow, sfb_row, Kb, lut);
            if (c) v += (double)dgo_bf16_to_f32(c[(size_t)m * N + n]);
            out[(size_t)r * N + n] = v;
        }
    }
    return 0;
}

/* M-grouped masked ([likun] §二 m_grouped_*_masked with masked_m, expected_m; [zwt] masked
 * layout for decoding): A [G,M_max,K], sfa [G][Kb][pad4(M_max)], B [G,N,K],
 * sfb [G][ceil(N/128)][Kb], C [G,M_max,N] or NULL. For r < masked_m[g]:
 * D[g,r] = C[g,r] + A[g,r]·B[g]ᵀ; rows r >= masked_m[g] are not part of the result and get
 * NaN in `out` [G][M_max][N]. masked_m[g] is clamped to [0, M_max]. */
int dgo_m_grouped_masked(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                         const uint16_t *c, const int32_t *masked_m, int G, int M_max, int N, int K,
                         double *out) {
    if (G <= 0 || M_max < 0 || N < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, Nb = (N + DGO_BLK - 1) / DGO_BLK;
    size_t ld = (size_t)pad4(M_max);
    double lut[256];
    fill_lut(lut);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int g = 0; g < G; g++) {
        for (int m = 0; m < M_max; m++) {
            int mm = masked_m[g] < 0 ? 0 : (masked_m[g] > M_max ? M_max : masked_m[g]);
            double *orow = out + ((size_t)g * M_max + m) * N;
            if (m >= mm) {
                for (int n = 0; n < N; n++) orow[n] = NAN;
                continue;
            }
            const uint8_t *arow = a + ((size_t)g * M_max + m) * K;
            const float *sfa_base = sfa + (size_t)g * Kb * ld + m;
            for (int n = 0; n < N; n++) {
                const uint8_t *brow = b + ((size_t)g * N + n) * K;
                const float *sfb_row = sfb + ((size_t)g * Nb + n / DGO_BLK) * Kb;
                double v = dot_row(arow, sfa_base, ld, brow, sfb_row, Kb, lut);
                if (c) v += (double)dgo_bf16_to_f32(c[((size_t)g * M_max + m) * N + n]);
                orow[n] = v;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* UE8M0 (power-of-two) scales ([likun] §五: on SM100 the scales are packed UE8M0, four per     */
/* 32-bit word; §二: disable_ue8m0_cast in the fp8 GEMM's signature)                          */
/* ---------------------------------------------------------------------------------------- */

/* UE8M0 byte of a block with absolute maximum `amax`: the exponent e of the smallest power of
 * two s = 2^e with s >= r, r = amax/448 computed as an fp32 division (the fp32 scale's own
 * definition), stored as e + 127. amax == 0 gives s = 1 (byte 127). e is clamped to [-127, 127]. */
uint8_t dgo_ue8m0_of_amax(float amax) {
    if (amax == 0.0f) return 127;
    float r = amax / 448.0f;
    int e;
    double f = frexp((double)r, &e);               /* r = f * 2^e, f in [0.5, 1) */
    int ex = (f == 0.5) ? e - 1 : e;               /* r == 2^(e-1) exactly: that power itself */
    if (ex < -127) ex = -127;
    if (ex > 127) ex = 127;
    return (uint8_t)(ex + 127);
}

static float ue8m0_value(uint8_t b) { return (float)ldexp(1.0, (int)b - 127); }

/* Per-token cast with UE8M0 scales: as dgo_cast_per_token, with s = 2^(byte - 127) from
 * dgo_ue8m0_of_amax (x / s is then an exact scaling before the e4m3 rounding). Scales packed
 * four per word: sfa_packed[(kb/4) * pad4(M) + m] holds the byte of K block kb at bits
 * 8·(kb%4); bytes of K blocks >= Kb are 127. */
int dgo_cast_per_token_ue8m0(const uint16_t *x, int M, int K, uint8_t *q, uint32_t *sfa_packed) {
    if (M < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, Kq = (Kb + 3) / 4, ld = pad4(M);
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; m++) {
        for (int kq = 0; kq < Kq; kq++) {
            uint32_t word = 0;
            for (int t = 0; t < 4; t++) {
                int kb = 4 * kq + t;
                uint8_t byte = 127;
                if (kb < Kb) {
                    const uint16_t *xs = x + (size_t)m * K + (size_t)kb * DGO_BLK;
                    float amax = 0.0f;
                    for (int i = 0; i < DGO_BLK; i++) {
                        float v = fabsf(dgo_bf16_to_f32(xs[i]));
                        if (v > amax) amax = v;
                    }
                    byte = dgo_ue8m0_of_amax(amax);
                    float s = ue8m0_value(byte);
                    for (int i = 0; i < DGO_BLK; i++)
                        q[(size_t)m * K + (size_t)kb * DGO_BLK + i] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(xs[i]) / s);
                }
                word |= (uint32_t)byte << (8 * t);
            }
            sfa_packed[(size_t)kq * ld + m] = word;
        }
    }
    return 0;
}

/* Per-block (128x128) cast with UE8M0 scales, as dgo_cast_per_block; scales packed four per
 * word along K: sfb_packed[(g * Nb + nb) * ceil(Kb/4) + kb/4] holds block (nb, kb) at bits
 * 8·(kb%4); bytes of K blocks >= Kb are 127. */
int dgo_cast_per_block_ue8m0(const uint16_t *x, int batch, int N, int K, uint8_t *q, uint32_t *sfb_packed) {
    if (batch < 0 || N < 0 || K <= 0 || K % DGO_BLK) return -1;
    int Kb = K / DGO_BLK, Nb = (N + DGO_BLK - 1) / DGO_BLK, Kq = (Kb + 3) / 4;
#pragma omp parallel for collapse(2) schedule(static)
    for (int g = 0; g < batch; g++) {
        for (int nb = 0; nb < Nb; nb++) {
            int n_end = (nb + 1) * DGO_BLK < N ? (nb + 1) * DGO_BLK : N;
            for (int kq = 0; kq < Kq; kq++) {
                uint32_t word = 0;
                for (int t = 0; t < 4; t++) {
                    int kb = 4 * kq + t;
                    uint8_t byte = 127;
                    if (kb < Kb) {
                        float amax = 0.0f;
                        for (int n = nb * DGO_BLK; n < n_end; n++)
                            for (int i = 0; i < DGO_BLK; i++) {
                                float v = fabsf(dgo_bf16_to_f32(x[((size_t)g * N + n) * K + (size_t)kb * DGO_BLK + i]));
                                if (v > amax) amax = v;
                            }
                        byte = dgo_ue8m0_of_amax(amax);
                        float s = ue8m0_value(byte);
                        for (int n = nb * DGO_BLK; n < n_end; n++)
                            for (int i = 0; i < DGO_BLK; i++) {
                                size_t off = ((size_t)g * N + n) * K + (size_t)kb * DGO_BLK + i;
                                q[off] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(x[off]) / s);
                            }
                    }
                    word |= (uint32_t)byte << (8 * t);
                }
                sfb_packed[((size_t)g * Nb + nb) * Kq + kq] = word;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* K-grouped GEMM for the MoE weight gradient ([likun] §一: k_grouped_fp8_gemm_tn, "MoE 反向";  */
/* §二: k_grouped_fp8_gemm_tn_contiguous with ks_cpu and recipe (1,1,128)).                   */
/* ---------------------------------------------------------------------------------------- */

/* Per-channel cast along the outer dimension, the recipe (1,1,128) quantisation of a
 * token-major tensor: x bf16 [T,C] (T tokens, C channels contiguous), T % 128 == 0. For every
 * 128-token block tb and channel c: amax = max_{t in tb} |x[t,c]|, s = amax/448 (s = 1 when
 * amax = 0), q[t,c] = e4m3_satrne(x[t,c] / s); sf fp32 [T/128][pad4(C)], sf[tb*pad4(C) + c] = s
 * (padding entries untouched). The same readings as the per-token cast, on the transposed
 * tensor. */
int dgo_cast_per_channel(const uint16_t *x, int T, int C, uint8_t *q, float *sf) {
    if (T < 0 || C < 0 || T % DGO_BLK) return -1;
    int Tb = T / DGO_BLK, ld = pad4(C);
#pragma omp parallel for collapse(2) schedule(static)
    for (int tb = 0; tb < Tb; tb++) {
        for (int c = 0; c < C; c++) {
            float amax = 0.0f;
            for (int i = 0; i < DGO_BLK; i++) {
                float v = fabsf(dgo_bf16_to_f32(x[((size_t)tb * DGO_BLK + i) * C + c]));
                if (v > amax) amax = v;
            }
            float s = scale_from_amax(amax);
            for (int i = 0; i < DGO_BLK; i++) {
                size_t off = ((size_t)tb * DGO_BLK + i) * C + c;
                q[off] = dgo_e4m3_encode_satrne(dgo_bf16_to_f32(x[off]) / s);
            }
            sf[(size_t)tb * ld + c] = s;
        }
    }
    return 0;
}

/* K-grouped TN GEMM: the K dimension (tokens) is cut into G consecutive groups of ks[g] rows
 * (each a multiple of 128); group g owns rows [k0_g, k0_g + ks[g]) of both operands.
 *   a  e4m3 [sum_K, M] (M contiguous: "T", the transposed A);  sfa fp32 [sum_K/128][pad4(M)]
 *   b  e4m3 [sum_K, N] (N contiguous: "N");                      sfb fp32 [sum_K/128][pad4(N)]
 *   c  fp32 [G, M, N] or NULL;  out fp64 [G, M, N]
 *   D[g,m,n] = C[g,m,n] + sum_{kb in g} sfa[kb][m]·sfb[kb][n]·S_kb[m,n],
 *   S_kb[m,n] = sum_{k in kb} e4m3(A[k,m])·e4m3(B[k,n])   (exact in fp64, as for the NT GEMM).
 * The recipe (1,1,128) gives one scale per channel (row of D for A, column of D for B) per
 * 128-token block; a group with ks[g] == 0 gives D[g] = C[g]. */
int dgo_k_grouped_tn(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                     const float *c, const int *ks, int G, int M, int N, double *out) {
    if (G <= 0 || M < 0 || N < 0) return -1;
    size_t ldm = (size_t)pad4(M), ldn = (size_t)pad4(N);
    int k0[4097];
    if (G > 4096) return -1;
    k0[0] = 0;
    for (int g = 0; g < G; g++) {
        if (ks[g] < 0 || ks[g] % DGO_BLK) return -2;
        k0[g + 1] = k0[g] + ks[g];
    }
    double lut[256];
    fill_lut(lut);
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int g = 0; g < G; g++) {
        for (int m = 0; m < M; m++) {
            for (int n = 0; n < N; n++) {
                double acc = 0.0;
                for (int kb = k0[g] / DGO_BLK; kb < k0[g + 1] / DGO_BLK; kb++) {
                    double s = 0.0;
                    for (int i = 0; i < DGO_BLK; i++) {
                        size_t k = (size_t)kb * DGO_BLK + i;
                        s += lut[a[k * M + m]] * lut[b[k * N + n]];
                    }
                    acc += (double)sfa[(size_t)kb * ldm + m] * (double)sfb[(size_t)kb * ldn + n] * s;
                }
                if (c) acc += (double)c[((size_t)g * M + m) * N + n];
                out[((size_t)g * M + m) * N + n] = acc;
            }
        }
    }
    return 0;
}

int dgo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
