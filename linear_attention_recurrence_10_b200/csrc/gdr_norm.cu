// gdr_norm.cu -- RMSNormGated on its own: the output gate of the mixer
// ("gated-delta-rule recurrence and RMSNormGated", Qwen3.5 Chat guide,
// section "Architektur"):
//
//   y = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z)     over each row of d
//
// Memory-bound elementwise work: d/4 lanes per row, one 4-wide vector load of
// o and z per lane, a shuffle reduction of the sum of squares, one vector
// store.  256 threads per CTA cover 256 / (d/4) rows.
#include "gdr_common.cuh"

namespace gdr {

template <int D, typename TO, typename TZ, typename TY>
__global__ void __launch_bounds__(256) rmsnorm_gated_kernel(const NormParams p) {
    constexpr int LPR = D / 4;
    constexpr int ROWS = 256 / LPR;
    const int gl = threadIdx.x % LPR;
    const int64_t row = (int64_t)blockIdx.x * ROWS + threadIdx.x / LPR;
    const bool valid = row < p.rows;
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f), z4 = o4;
    if (valid) {
        o4 = Elem<TO>::load4(static_cast<const TO *>(p.o) + row * p.o_stride + 4 * gl);
        z4 = Elem<TZ>::load4(static_cast<const TZ *>(p.z) + row * p.z_stride + 4 * gl);
    }
    // Every lane takes part in the shuffles; rows past the end carry zeros.
    const float ss = group_sum<LPR>(dot4(o4, o4));
    if (!valid) return;
    const float rstd = rsqrtf(ss * (1.0f / D) + p.eps);
    float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
    if (p.w) w4 = __ldg(reinterpret_cast<const float4 *>(p.w + 4 * gl));
    float4 y;
    y.x = o4.x * rstd * w4.x * silu(z4.x);
    y.y = o4.y * rstd * w4.y * silu(z4.y);
    y.z = o4.z * rstd * w4.z * silu(z4.z);
    y.w = o4.w * rstd * w4.w * silu(z4.w);
    Elem<TY>::store4(static_cast<TY *>(p.out) + row * p.out_stride + 4 * gl, y);
}

template <int D, typename TO, typename TZ, typename TY>
static cudaError_t launch_norm_t(const NormParams &p, cudaStream_t s) {
    constexpr int ROWS = 256 / (D / 4);
    const int64_t blocks = (p.rows + ROWS - 1) / ROWS;
    if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    rmsnorm_gated_kernel<D, TO, TZ, TY><<<(unsigned)blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

template <int D, typename TO, typename TZ>
static cudaError_t launch_norm_y(const NormParams &p, int y_bf16, cudaStream_t s) {
    return y_bf16 ? launch_norm_t<D, TO, TZ, __nv_bfloat16>(p, s)
                  : launch_norm_t<D, TO, TZ, float>(p, s);
}

template <int D, typename TO>
static cudaError_t launch_norm_z(const NormParams &p, int z_bf16, int y_bf16, cudaStream_t s) {
    return z_bf16 ? launch_norm_y<D, TO, __nv_bfloat16>(p, y_bf16, s)
                  : launch_norm_y<D, TO, float>(p, y_bf16, s);
}

template <int D>
static cudaError_t launch_norm_d(const NormParams &p, int o_bf16, int z_bf16, int y_bf16,
                                 cudaStream_t s) {
    return o_bf16 ? launch_norm_z<D, __nv_bfloat16>(p, z_bf16, y_bf16, s)
                  : launch_norm_z<D, float>(p, z_bf16, y_bf16, s);
}

cudaError_t launch_rmsnorm_gated(const NormParams &p, int d, int o_bf16, int z_bf16,
                                 int y_bf16, cudaStream_t s) {
    switch (d) {
        case 16: return launch_norm_d<16>(p, o_bf16, z_bf16, y_bf16, s);
        case 32: return launch_norm_d<32>(p, o_bf16, z_bf16, y_bf16, s);
        case 64: return launch_norm_d<64>(p, o_bf16, z_bf16, y_bf16, s);
        case 128: return launch_norm_d<128>(p, o_bf16, z_bf16, y_bf16, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdr
