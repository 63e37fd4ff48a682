// gdr_decode.cu -- one decode step of the gated delta rule, fused end to end.
//
// The decoder the pages describe advances one token per call against a state
// it keeps across the generation loop (Core ML card for Qwen3.5-0.8B, sections
// "Model" and "Usage"); the state is a fixed-size matrix per head, so nothing
// grows with context (Swiftlet post, "How It Works").  Per (sequence b, value
// head h) this kernel computes, with S the d x d fp32 state (row i = value dim i):
//
//   q_hat, k_hat  L2-normalised (q also scaled)
//   alpha = exp(g),  a = S k_hat,  c = S q_hat            (one pass over S)
//   delta = beta (v - alpha a)
//   S'    = alpha S + delta k_hat^T                        (written once)
//   o     = S' q_hat = alpha c + delta (k_hat . q_hat)
//   y     = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z)
//
// which is S' = exp(g) S (I - beta k k^T) + beta v k^T, o = S' q expanded so
// that S is read exactly once and written exactly once: the kernel is bound by
// HBM bandwidth on the 2 d^2 * 4 bytes of state per head.
//
// Thread layout (one CTA per (b, h), 2d threads): each lane owns one float4 of
// a state row; LPR = d/4 lanes share a row, and every lane holds NS = LPR/2
// rows of its warp's 16.  The partial sums for a and c (2 NS = LPR values per
// lane) are reduced with a reduce-scatter butterfly over the LPR lanes, which
// leaves exactly one finished value per lane (LPR - 1 shuffles instead of
// 2 NS log2(LPR)): lane gl < NS ends with a of its row, lane gl >= NS with c.
#include "gdr_common.cuh"

namespace gdr {

// MULTI: p.n_tokens tokens per sequence in order, the state held in registers
// between them (read once, written once), and optional state slots.  The
// one-token instantiation (MULTI = false) is the plain decode step.
template <int D, typename TIN, typename TOUT, bool MULTI>
__global__ void __launch_bounds__(2 * D) decode_kernel(const DecodeParams p) {
    constexpr int NW = 2 * D / 32;  // warps; each owns 16 state rows
    constexpr int LPR = D / 4;      // lanes per state row (one float4 each)
    constexpr int RPP = 32 / LPR;   // rows one warp-wide pass covers
    constexpr int NS = LPR / 2;     // rows held per lane
    static_assert(NS * RPP == 16, "each warp owns 16 rows");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gl = lane % LPR, rg = lane / LPR;
    const int b = blockIdx.x / p.H_v;
    const int hv = blockIdx.x - b * p.H_v;
    const int hk = hv / p.hv_per_hk;
    const int col = 4 * gl;
    const int row0 = warp * 16 + rg;  // row of slot s is row0 + s * RPP
    const int T = MULTI ? p.n_tokens : 1;

    // The state this sequence owns: its own batch row, or its slot.  A slot
    // table may be written by the preceding kernel, so it is read after it.
    int sb = b;
    if (MULTI && p.slot) {
        wait_for_predecessor();
        sb = p.slot[b];
        if (sb < 0 || sb >= p.n_slots) {
            if (threadIdx.x == 0 && p.status) atomicExch(p.status, 1);  // GDR_ERR_INVALID_ARG
            return;
        }
    }
    const size_t head_off = (size_t)hv * D * D;
    const float *sin = p.state_in + (size_t)sb * p.state_stride + head_off;
    float *sout = p.state_out + (size_t)sb * p.state_stride + head_off;

    // Issue every state load first so the whole tile is in flight at once.  With
    // overlap_state_load the caller guarantees that the kernel before this one
    // does not write the state, so the loads may run while it finishes.
    if (!p.overlap_state_load) wait_for_predecessor();
    float4 S[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) S[s] = ld_state4(sin + (size_t)(row0 + s * RPP) * D + col);
    if (p.overlap_state_load) wait_for_predecessor();
    release_dependents();

    // Row this lane finishes: lanes gl < NS need v of it, lanes gl >= NS need z.
    const bool is_a = gl < NS;
    const int my_row = row0 + (gl % NS) * RPP;
    __shared__ float red[2][NW];

    for (int t = 0; t < T; ++t) {
        const int64_t r = (int64_t)b * T + t;  // token row
        const TIN *qp = static_cast<const TIN *>(p.q) + r * p.q_stride + hk * D;
        const TIN *kp = static_cast<const TIN *>(p.k) + r * p.k_stride + hk * D;
        float4 q4 = Elem<TIN>::load4(qp + col);
        float4 k4 = Elem<TIN>::load4(kp + col);
        float g = __ldg(p.g + r * p.gb_stride + hv);
        float beta = __ldg(p.beta + r * p.gb_stride + hv);
        if (p.A_log) {
            g = gate_g(g, __ldg(p.A_log + hv), __ldg(p.dt_bias + hv));
            beta = gate_beta(beta);
        }
        float vz = 0.f;
        if (is_a) {
            vz = Elem<TIN>::load1(static_cast<const TIN *>(p.v) + r * p.v_stride + hv * D + my_row);
        } else if (p.z) {
            vz = Elem<TIN>::load1(static_cast<const TIN *>(p.z) + r * p.z_stride + hv * D + my_row);
        }

        float qs = p.scale, ks = 1.f;
        if (p.qk_l2norm) {
            const float qq = group_sum<LPR>(dot4(q4, q4));
            const float kk = group_sum<LPR>(dot4(k4, k4));
            qs *= rsqrtf(qq + p.eps_l2);
            ks = rsqrtf(kk + p.eps_l2);
        }
        q4 = scale4(q4, qs);
        k4 = scale4(k4, ks);
        const float kq = group_sum<LPR>(dot4(k4, q4));
        const float alpha = expf(g);

        // Partial S k and S q over this lane's 4 columns, for each held row.
        float x[LPR];
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            x[s] = dot4(S[s], k4);
            x[NS + s] = dot4(S[s], q4);
        }
        // Reduce-scatter: at offset o a lane keeps the half of its 2o values picked
        // by bit o of gl and adds the partner's copy of that half.
#pragma unroll
        for (int o = LPR / 2; o >= 1; o >>= 1) {
            const bool up = (gl & o) != 0;
#pragma unroll
            for (int j = 0; j < o; ++j) {
                const float send = up ? x[j] : x[j + o];
                const float keep = up ? x[j + o] : x[j];
                x[j] = keep + __shfl_xor_sync(kFullMask, send, o);
            }
        }
        // x[0]: a = (S k)_row on lanes gl < NS, c = (S q)_row on lanes gl >= NS.
        const float delta = beta * (vz - alpha * x[0]);                      // valid where is_a
        const float delta_c = __shfl_xor_sync(kFullMask, delta, NS);         // row's delta on c-lanes
        const float o_val = fmaf(alpha, x[0], delta_c * kq);                 // valid where !is_a

#pragma unroll
        for (int s = 0; s < NS; ++s) {
            const float d = __shfl_sync(kFullMask, delta, rg * LPR + s);
            S[s] = axpby4(S[s], alpha, k4, d);
            if (!MULTI) st_state4(sout + (size_t)(row0 + s * RPP) * D + col, S[s]);
        }

        TOUT *op = static_cast<TOUT *>(p.out) + r * p.out_stride + hv * D;
        if (p.z == nullptr) {
            if (!is_a) Elem<TOUT>::store1(op + my_row, o_val);
        } else {
            // Partials double-buffered by token, so one barrier per token suffices.
            float ss = is_a ? 0.f : o_val * o_val;
            ss = group_sum<32>(ss);
            if (lane == 0) red[t & 1][warp] = ss;
            __syncthreads();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) tot += red[t & 1][w];
            if (!is_a) {
                const float rstd = rsqrtf(tot * (1.0f / D) + p.eps_norm);
                const float wv = p.norm_w ? __ldg(p.norm_w + my_row) : 1.0f;
                Elem<TOUT>::store1(op + my_row, o_val * rstd * wv * silu(vz));
            }
        }
    }
    if (MULTI) {
#pragma unroll
        for (int s = 0; s < NS; ++s) st_state4(sout + (size_t)(row0 + s * RPP) * D + col, S[s]);
    }
}

// d = 128, one token: the same arithmetic with 128 threads per (b, h) instead
// of 256.  Each warp owns 32 state rows and takes them in two batches of 16
// (the layout of decode_kernel per batch): the first batch loads into
// registers, the second by cp.async into 8 KB of shared memory per warp, both
// issued before the wait on the preceding kernel.  Half the threads per head
// at the same registers per thread lets four heads share an SM instead of two,
// so a grid of up to 4 x #SMs heads runs as a single wave.
template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(128, 4) decode_rb_kernel(const DecodeParams p) {
    constexpr int D = 128, NW = 4, NS = 16;  // warps; rows per batch
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x / p.H_v;
    const int hv = blockIdx.x - b * p.H_v;
    const int hk = hv / p.hv_per_hk;
    const int col = 4 * lane;
    const size_t head_off = (size_t)hv * D * D;
    const float *sin = p.state_in + (size_t)b * p.state_stride + head_off;
    float *sout = p.state_out + (size_t)b * p.state_stride + head_off;
    __shared__ __align__(16) float4 stage[NW][NS][32];
    __shared__ float red[2 * NW];

    // Rows of batch r: warp * 32 + 16 r + s, s = 0..15.
    if (!p.overlap_state_load) wait_for_predecessor();
    float4 S[NS];
    const float *r0 = sin + (size_t)(warp * 32) * D + col;
#pragma unroll
    for (int s = 0; s < NS; ++s) S[s] = ld_state4(r0 + (size_t)s * D);
#pragma unroll
    for (int s = 0; s < NS; ++s)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         (uint32_t)__cvta_generic_to_shared(&stage[warp][s][lane])),
                     "l"(r0 + (size_t)(NS + s) * D)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (p.overlap_state_load) wait_for_predecessor();
    release_dependents();

    const TIN *qp = static_cast<const TIN *>(p.q) + (int64_t)b * p.q_stride + hk * D;
    const TIN *kp = static_cast<const TIN *>(p.k) + (int64_t)b * p.k_stride + hk * D;
    float4 q4 = Elem<TIN>::load4(qp + col);
    float4 k4 = Elem<TIN>::load4(kp + col);
    float g = __ldg(p.g + (int64_t)b * p.gb_stride + hv);
    float beta = __ldg(p.beta + (int64_t)b * p.gb_stride + hv);
    if (p.A_log) {
        g = gate_g(g, __ldg(p.A_log + hv), __ldg(p.dt_bias + hv));
        beta = gate_beta(beta);
    }
    // Lanes < 16 finish a = (S k)_row of row (lane % 16) of the batch and need
    // v of it; lanes >= 16 finish c = (S q)_row and need z.
    const bool is_a = lane < NS;
    const TIN *vz_base = is_a ? static_cast<const TIN *>(p.v) + (int64_t)b * p.v_stride + hv * D
                              : (p.z ? static_cast<const TIN *>(p.z) + (int64_t)b * p.z_stride + hv * D
                                     : nullptr);
    float vz[2];
#pragma unroll
    for (int r = 0; r < 2; ++r)
        vz[r] = vz_base ? Elem<TIN>::load1(vz_base + warp * 32 + 16 * r + (lane % NS)) : 0.f;

    float qs = p.scale, ks = 1.f;
    if (p.qk_l2norm) {
        const float qq = group_sum<32>(dot4(q4, q4));
        const float kk = group_sum<32>(dot4(k4, k4));
        qs *= rsqrtf(qq + p.eps_l2);
        ks = rsqrtf(kk + p.eps_l2);
    }
    q4 = scale4(q4, qs);
    k4 = scale4(k4, ks);
    const float kq = group_sum<32>(dot4(k4, q4));
    const float alpha = expf(g);

    float o_val[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r == 1) {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncwarp();
#pragma unroll
            for (int s = 0; s < NS; ++s) S[s] = stage[warp][s][lane];
        }
        float x[32];
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            x[s] = dot4(S[s], k4);
            x[NS + s] = dot4(S[s], q4);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int j = 0; j < o; ++j) {
                const float send = up ? x[j] : x[j + o];
                const float keep = up ? x[j + o] : x[j];
                x[j] = keep + __shfl_xor_sync(kFullMask, send, o);
            }
        }
        const float delta = beta * (vz[r] - alpha * x[0]);            // valid where is_a
        const float delta_c = __shfl_xor_sync(kFullMask, delta, NS);  // row's delta on c-lanes
        o_val[r] = fmaf(alpha, x[0], delta_c * kq);                   // valid where !is_a
        float *rowp = sout + (size_t)(warp * 32 + 16 * r) * D + col;
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            const float d = __shfl_sync(kFullMask, delta, s);
            st_state4(rowp + (size_t)s * D, axpby4(S[s], alpha, k4, d));
        }
    }

    TOUT *op = static_cast<TOUT *>(p.out) + (int64_t)b * p.out_stride + hv * D + warp * 32 + (lane % NS);
    if (p.z == nullptr) {
        if (!is_a) {
            Elem<TOUT>::store1(op, o_val[0]);
            Elem<TOUT>::store1(op + 16, o_val[1]);
        }
        return;
    }
    // Sums of squares per 16-row batch, added in row order: the same
    // arithmetic as decode_kernel (whose warps own 16 rows each), so both give
    // bit-identical outputs.
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const float ss = group_sum<32>(is_a ? 0.f : o_val[r] * o_val[r]);
        if (lane == 0) red[2 * warp + r] = ss;
    }
    __syncthreads();
    if (!is_a) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < 2 * NW; ++w) tot += red[w];
        const float rstd = rsqrtf(tot * (1.0f / D) + p.eps_norm);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int row = warp * 32 + 16 * r + (lane % NS);
            const float wv = p.norm_w ? __ldg(p.norm_w + row) : 1.0f;
            Elem<TOUT>::store1(op + 16 * r, o_val[r] * rstd * wv * silu(vz[r]));
        }
    }
}

// Launched as a programmatic dependent of the previous kernel on the stream:
// its blocks may be scheduled while that kernel drains, and wait in
// wait_for_predecessor() before touching anything it may have written.
template <int D, typename TIN, typename TOUT, bool MULTI>
static cudaError_t launch_decode_t(const DecodeParams &p, cudaStream_t stream) {
    constexpr bool RB = D == 128 && !MULTI;  // the 128-thread, two-batch kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)p.batch * p.H_v));
    cfg.blockDim = dim3(RB ? 128 : 2 * D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if constexpr (RB) {
        // Four blocks of 32 KB static shared memory per SM: ask for the
        // carveout that holds them (once per instantiation; thread-safe).
        static const cudaError_t carve = cudaFuncSetAttribute(
            decode_rb_kernel<TIN, TOUT>, cudaFuncAttributePreferredSharedMemoryCarveout,
            (int)cudaSharedmemCarveoutMaxShared);
        if (carve != cudaSuccess) {
            (void)cudaGetLastError();
            return carve;
        }
        e = cudaLaunchKernelEx(&cfg, decode_rb_kernel<TIN, TOUT>, p);
    } else
        e = cudaLaunchKernelEx(&cfg, decode_kernel<D, TIN, TOUT, MULTI>, p);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return e;
    }
    return cudaGetLastError();
}

template <int D, bool MULTI>
static cudaError_t launch_decode_d(const DecodeParams &p, int in_bf16, int out_bf16,
                                   cudaStream_t s) {
    if (in_bf16) {
        return out_bf16 ? launch_decode_t<D, __nv_bfloat16, __nv_bfloat16, MULTI>(p, s)
                        : launch_decode_t<D, __nv_bfloat16, float, MULTI>(p, s);
    }
    return out_bf16 ? launch_decode_t<D, float, __nv_bfloat16, MULTI>(p, s)
                    : launch_decode_t<D, float, float, MULTI>(p, s);
}

template <bool MULTI>
static cudaError_t launch_decode_m(const DecodeParams &p, int d, int in_bf16, int out_bf16,
                                   cudaStream_t s) {
    switch (d) {
        case 16: return launch_decode_d<16, MULTI>(p, in_bf16, out_bf16, s);
        case 32: return launch_decode_d<32, MULTI>(p, in_bf16, out_bf16, s);
        case 64: return launch_decode_d<64, MULTI>(p, in_bf16, out_bf16, s);
        case 128: return launch_decode_d<128, MULTI>(p, in_bf16, out_bf16, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const DecodeParams &p, int d, int in_bf16, int out_bf16,
                          cudaStream_t s) {
    return launch_decode_m<false>(p, d, in_bf16, out_bf16, s);
}

cudaError_t launch_decode_multi(const DecodeParams &p, int d, int in_bf16, int out_bf16,
                                cudaStream_t s) {
    return launch_decode_m<true>(p, d, in_bf16, out_bf16, s);
}

}  // namespace gdr
