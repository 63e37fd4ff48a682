// gdr_common.cuh -- small device helpers shared by the mixer's kernels:
// typed vector loads/stores (fp32 and bf16), warp reductions, and the
// parameter blocks the host side fills in.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

constexpr unsigned kFullMask = 0xffffffffu;

// Workspace of the one-kernel tensor-core prefill: the status word (16 bytes
// reserved) and the longest-first order of n_seq sequences, rounded up to 256.
constexpr size_t prefill_tc_ws_bytes(int64_t n_seq) {
    return (size_t)(16 + 4 * (size_t)n_seq + 255) & ~(size_t)255;
}

// ----------------------------------------------------------------- params

struct DecodeParams {
    int batch, H_k, H_v, hv_per_hk;
    int qk_l2norm;
    int overlap_state_load;  // read the state before waiting on the previous kernel
    float scale, eps_l2, eps_norm;
    int64_t q_stride, k_stride, v_stride, z_stride, gb_stride, out_stride, state_stride;
    const void *q, *k, *v, *z;
    const float *g, *beta;
    const float *state_in;
    float *state_out;
    const float *norm_w;
    void *out;
    // Several tokens per sequence (rows b * n_tokens + t of every token-indexed
    // tensor) and optional state slots; unused by the one-token kernel.
    int n_tokens, n_slots;
    const int *slot;
    int *status;
    // Non-null: g and beta hold the raw projections a, b (see gate_g, gate_beta).
    const float *A_log, *dt_bias;
};

// Gate values from raw projection outputs (gates passed raw): per value head,
//   g = -exp(A_log) softplus(a + dt_bias),   beta = sigmoid(b),
// the parameterisation of the published Gated DeltaNet and Mamba-2 layers;
// softplus(x) as max(x, 0) + log1p(exp(-|x|)), which cannot overflow.
__device__ __forceinline__ float gate_g(float a, float A_log, float dt_bias) {
    const float x = a + dt_bias;
    return -expf(A_log) * (fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
}
__device__ __forceinline__ float gate_beta(float b) { return 1.f / (1.f + expf(-b)); }

struct NormParams {
    int64_t rows;
    float eps;
    int64_t o_stride, z_stride, out_stride;
    const void *o, *z;
    const float *w;
    void *out;
};

struct PrefillParams {
    int n_seq, H_k, H_v, hv_per_hk;
    int qk_l2norm;
    float scale, eps_l2, eps_norm;
    int64_t q_stride, k_stride, v_stride, z_stride, gb_stride, out_stride;
    const void *q, *k, *v, *z;
    const float *g, *beta;
    const int32_t *cu_seqlens;
    const float *initial_state;
    float *final_state;
    const float *norm_w;
    void *out;
    // Non-null: g and beta hold the raw projections a, b (see gate_g, gate_beta).
    const float *A_log, *dt_bias;
    // Diagnostics only, zero in every ordinary call: a limit for the device
    // waits of the tensor-core recurrence (0 = the default), and a flag that
    // withholds every (sequence, head)'s first key tile so that those waits
    // run out and the kernel's unwinding path runs.
    uint64_t wait_ns;
    int withhold_first_k;
};

// ------------------------------------------------------------ typed memory

template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static __forceinline__ float4 load4(const float *p) {
        return __ldg(reinterpret_cast<const float4 *>(p));
    }
    __device__ static __forceinline__ float load1(const float *p) { return __ldg(p); }
    __device__ static __forceinline__ void store1(float *p, float x) { *p = x; }
    __device__ static __forceinline__ void store4(float *p, float4 x) {
        *reinterpret_cast<float4 *>(p) = x;
    }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static __forceinline__ float4 load4(const __nv_bfloat16 *p) {
        uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
        __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
        __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
        float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    __device__ static __forceinline__ float load1(const __nv_bfloat16 *p) {
        return __bfloat162float(p[0]);
    }
    __device__ static __forceinline__ void store1(__nv_bfloat16 *p, float x) {
        *p = __float2bfloat16_rn(x);
    }
    __device__ static __forceinline__ void store4(__nv_bfloat16 *p, float4 x) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(x.x, x.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(x.z, x.w);
        uint2 raw;
        raw.x = *reinterpret_cast<unsigned *>(&lo);
        raw.y = *reinterpret_cast<unsigned *>(&hi);
        *reinterpret_cast<uint2 *>(p) = raw;
    }
};

// State tiles are read once and written once per call; keep them out of L1.
__device__ __forceinline__ float4 ld_state4(const float *p) {
    float4 r;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_state4(float *p, float4 v) {
    asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// ------------------------------------------- programmatic dependent launch

// Wait until the kernel queued before this one has finished and its writes
// are visible (a no-op when this kernel was not launched as a dependent).
__device__ __forceinline__ void wait_for_predecessor() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next kernel on the stream to start launching.  Called only after
// wait_for_predecessor(), so a dependent never starts while anything queued
// before this kernel is still running.
__device__ __forceinline__ void release_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------------------------- math

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
__device__ __forceinline__ float4 scale4(float4 a, float s) {
    return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
// a * s + b * t, componentwise
__device__ __forceinline__ float4 axpby4(float4 a, float s, float4 b, float t) {
    return make_float4(fmaf(a.x, s, b.x * t), fmaf(a.y, s, b.y * t), fmaf(a.z, s, b.z * t),
                       fmaf(a.w, s, b.w * t));
}

// Sum over aligned groups of N lanes (N a power of two <= 32).
template <int N>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = 1; o < N; o <<= 1) x += __shfl_xor_sync(kFullMask, x, o);
    return x;
}

// z * sigmoid(z)
__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

}  // namespace gdr
