// gdr_prefill_common.cuh -- pieces shared by the tensor-core prefill kernels:
// sizes, shared-memory operand layouts, the MMA loop, bf16 hi/lo splitting and
// the blocked fp32 inverse of the chunk's unit lower-triangular matrix.
#pragma once

#include "gdr_common.cuh"
#include "gdr_tc.cuh"

namespace gdr {
namespace tcp {

using namespace gdr::tc;

constexpr int D = 128;       // d_k = d_v
constexpr int C = 64;        // chunk
constexpr int LDA = C + 1;   // padded row stride of the fp32 scratch matrices
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: far beyond any chunk's work
constexpr float kGammaFloor = -64.0f;
constexpr int kTimeoutStatus = 6;  // GDR_ERR_TIMEOUT

// Tiles written from registers, K-major: 16-byte chunks along K are R*16 bytes
// apart, 8-row groups 128 bytes apart (LBO = R*16, SBO = 128).
__device__ __forceinline__ uint32_t kmaj(int row, int k, int R) {
    return (uint32_t)((k >> 3) * (R * 16) + (row >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}
// The [K;Q] tile: 8-row groups 2048 bytes apart, 16-byte chunks along d 128
// bytes apart.  K-major over d: LBO = 128, SBO = 2048.  Read as MN-major over
// d with the tokens as K: SBO = 128, LBO = 2048.
__device__ __forceinline__ uint32_t kq_off(int row, int j) {
    return (uint32_t)((row >> 3) * 2048 + (j >> 3) * 128 + (row & 7) * 16 + (j & 7) * 2);
}
// V tile, MN-major over d_v with the tokens as K: SBO = 1024, LBO = 128.
__device__ __forceinline__ uint32_t v_off(int s, int i) {
    return (uint32_t)((i >> 3) * 1024 + (s >> 3) * 128 + (s & 7) * 16 + (i & 7) * 2);
}
// W tile (B operand of S W^T), MN-major over the tokens r with d_k as K:
// SBO = 2048, LBO = 128.
__device__ __forceinline__ uint32_t w_off(int j, int r) {
    return (uint32_t)((r >> 3) * 2048 + (j >> 3) * 128 + (j & 7) * 16 + (r & 7) * 2);
}

// z * sigmoid(z) with the fast exponential (relative error ~1e-7 here).
__device__ __forceinline__ float fast_silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Eight fp32 values as eight bf16 (round to nearest even) in 16 bytes.
__device__ __forceinline__ uint4 pack8(const float *v) {
    uint4 pk;
    __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 b3 = __floats2bfloat162_rn(v[6], v[7]);
    pk.x = *reinterpret_cast<uint32_t *>(&b0);
    pk.y = *reinterpret_cast<uint32_t *>(&b1);
    pk.z = *reinterpret_cast<uint32_t *>(&b2);
    pk.w = *reinterpret_cast<uint32_t *>(&b3);
    return pk;
}
// Split eight fp32 values into bf16 hi = rn(x) and lo = rn(x - hi).
__device__ __forceinline__ void split8(const float *v, uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
        const float2 f = __bfloat1622float2(b);
        // x - hi for both lanes at once (sm_100's two-wide add; exact here).
        const float2 d = __fadd2_rn(make_float2(v[2 * u], v[2 * u + 1]), make_float2(-f.x, -f.y));
        const __nv_bfloat162 r = __floats2bfloat162_rn(d.x, d.y);
        h[u] = *reinterpret_cast<const uint32_t *>(&b);
        l[u] = *reinterpret_cast<const uint32_t *>(&r);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// One distance of the blocked triangular inverse: for every pair of 16-blocks
// (i, j) with i - j = DIST, X = A[i-rows][16j .. 16i) T[16j .. 16i)[j-cols],
// then T_ij = -T_ii X.  One output per thread, fully unrolled so the
// shared-memory loads overlap; for row strides that are not 16-byte aligned.
template <int DIST, int NT, int LD>
__device__ __forceinline__ void offdiag_stage(const float *Ascr, float *Tscr, float *Xscr, int tid) {
    constexpr int NBLK = 4 - DIST, NOUT = NBLK * 256;
#pragma unroll
    for (int e0 = 0; e0 < NOUT; e0 += NT) {
        const int e = e0 + tid;
        if (NOUT % NT == 0 || e < NOUT) {
            const int j = e >> 8, i = j + DIST, rr = (e >> 4) & 15, cc = e & 15;
            const float *arow = Ascr + (16 * i + rr) * LD + 16 * j;
            const float *tcol = Tscr + 16 * j * LD + 16 * j + cc;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16 * DIST; ++k) acc[k & 3] = fmaf(arow[k], tcol[k * LD], acc[k & 3]);
            Xscr[e] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
    }
    __syncthreads();
#pragma unroll
    for (int e0 = 0; e0 < NOUT; e0 += NT) {
        const int e = e0 + tid;
        if (NOUT % NT == 0 || e < NOUT) {
            const int j = e >> 8, i = j + DIST, rr = (e >> 4) & 15, cc = e & 15;
            const float *trow = Tscr + (16 * i + rr) * LD + 16 * i;
            const float *xcol = Xscr + (j << 8) + cc;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 16; ++k) acc[k & 3] = fmaf(trow[k], xcol[k * 16], acc[k & 3]);
            Tscr[(16 * i + rr) * LD + 16 * j + cc] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
        }
    }
    __syncthreads();
}

// The same distance stage with 16-byte aligned rows (LD % 4 == 0): each thread
// computes a strip of four adjacent outputs, so every operand load is a
// 16-byte vector that feeds four (row operand) or sixteen (column operand)
// FMAs instead of one, issued as two-wide FMAs (sm_100; each lane rounds as
// fmaf does).  X is kept as dense 16 x 16 blocks.
template <int DIST, int NT, int LD>
__device__ __forceinline__ void offdiag_stage_strips(const float *Ascr, float *Tscr, float *Xscr,
                                                     int tid) {
    static_assert(LD % 4 == 0, "rows must be 16-byte aligned");
    constexpr int NSTRIP = (4 - DIST) * 64;  // 16 rows x 4 strips per block pair
    for (int e = tid; e < NSTRIP; e += NT) {
        const int j = e >> 6, i = j + DIST, rr = (e >> 2) & 15, c4 = 4 * (e & 3);
        const float *arow = Ascr + (16 * i + rr) * LD + 16 * j;
        const float *tcol = Tscr + 16 * j * LD + 16 * j + c4;
        float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);  // the strip's four sums
#pragma unroll
        for (int k4 = 0; k4 < 4 * DIST; ++k4) {
            const float4 a = *reinterpret_cast<const float4 *>(arow + 4 * k4);
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 t = *reinterpret_cast<const float4 *>(tcol + (4 * k4 + u) * LD);
                const float2 au = make_float2(av[u], av[u]);
                lo = __ffma2_rn(au, make_float2(t.x, t.y), lo);
                hi = __ffma2_rn(au, make_float2(t.z, t.w), hi);
            }
        }
        *reinterpret_cast<float4 *>(Xscr + (j << 8) + rr * 16 + c4) = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    __syncthreads();
    for (int e = tid; e < NSTRIP; e += NT) {
        const int j = e >> 6, i = j + DIST, rr = (e >> 2) & 15, c4 = 4 * (e & 3);
        const float *trow = Tscr + (16 * i + rr) * LD + 16 * i;
        const float *xblk = Xscr + (j << 8) + c4;
        float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const float4 t = *reinterpret_cast<const float4 *>(trow + 4 * k4);
            const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 x = *reinterpret_cast<const float4 *>(xblk + (4 * k4 + u) * 16);
                const float2 tu = make_float2(tv[u], tv[u]);
                lo = __ffma2_rn(tu, make_float2(x.x, x.y), lo);
                hi = __ffma2_rn(tu, make_float2(x.z, x.w), hi);
            }
        }
        *reinterpret_cast<float4 *>(Tscr + (16 * i + rr) * LD + 16 * j + c4) =
            make_float4(-lo.x, -lo.y, -hi.x, -hi.y);
    }
    __syncthreads();
}

// T = (I + A)^{-1} for the strictly lower-triangular 64 x 64 A in Ascr (fp32,
// row stride LD), blocked by 16.  Diagonal blocks first, one column per
// thread, right-looking (each finished x_s is folded into all later rows at
// once, so the dependent chain is 16 steps); then the off-diagonal blocks by
// distance from the diagonal: T_ij = -T_ii sum_{16j <= k < 16i} A[i-rows][k] T[k][j-cols].
// Every thread of the block calls it; it ends with the block synchronised.
template <int NT, int LD = LDA>
__device__ __forceinline__ void invert_unit_lower(const float *Ascr, float *Tscr, float *Xscr, int tid) {
    if (tid < C) {
        const int b = tid >> 4, c = tid & 15, base = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
            // Rows in pairs (two-wide FMA); fmaf(a, -x, y) is fmaf(-a, x, y) exactly.
            const float2 nx = make_float2(-x[s], -x[s]);
#pragma unroll
            for (int r = s + 1; r < 16; r += 2) {
                if (r + 1 < 16) {
                    const float2 y = __ffma2_rn(make_float2(Ascr[(base + r) * LD + base + s],
                                                            Ascr[(base + r + 1) * LD + base + s]),
                                               nx, make_float2(x[r], x[r + 1]));
                    x[r] = y.x;
                    x[r + 1] = y.y;
                } else {
                    x[r] = fmaf(Ascr[(base + r) * LD + base + s], nx.x, x[r]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tscr[(base + r) * LD + base + c] = x[r];
    } else {
        for (int e = tid - C; e < C * C; e += NT - C) {  // zero the blocks above the diagonal
            const int r = e >> 6, s = e & 63;
            if ((s >> 4) > (r >> 4)) Tscr[r * LD + s] = 0.f;
        }
    }
    __syncthreads();
    if constexpr (LD % 4 == 0) {
        offdiag_stage_strips<1, NT, LD>(Ascr, Tscr, Xscr, tid);
        offdiag_stage_strips<2, NT, LD>(Ascr, Tscr, Xscr, tid);
        offdiag_stage_strips<3, NT, LD>(Ascr, Tscr, Xscr, tid);
    } else {
        offdiag_stage<1, NT, LD>(Ascr, Tscr, Xscr, tid);
        offdiag_stage<2, NT, LD>(Ascr, Tscr, Xscr, tid);
        offdiag_stage<3, NT, LD>(Ascr, Tscr, Xscr, tid);
    }
}

}  // namespace tcp
}  // namespace gdr
