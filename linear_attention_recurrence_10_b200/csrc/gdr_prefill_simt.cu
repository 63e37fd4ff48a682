// gdr_prefill_simt.cu -- chunked prefill of the gated delta rule on CUDA
// cores, in fp32.  This is the general path: any supported head size (16, 32,
// 64, 128), chunk 16/32/64, fp32 or bf16 inputs.  bf16 inputs with d = 128
// and chunk 64 go to the tensor-core kernel instead.
//
// One CTA owns one (sequence, value head) and walks its chunks in order,
// keeping the fp32 state in shared memory.  Per chunk of L <= C tokens
// (gamma_r = running sum of g inside the chunk, g clamped at -64):
//   A_rs  = beta_r exp(gamma_r - gamma_s) (k_r . k_s)          s < r
//   [U | W] = (I + A)^{-1} [diag(beta) V | diag(beta e^gamma) K]   (forward substitution)
//   Delta = U - W S^T
//   P_rs  = exp(gamma_r - gamma_s) (q_r . k_s)                 s <= r
//   O     = diag(e^gamma) Q S^T + P Delta   -> RMSNormGated -> out
//   S     = e^{gamma_L} S + Delta^T diag(e^{gamma_L - gamma}) K
// This is the chunkwise (WY / UT transform) form of the recurrence
// S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t
// (the "gated delta rule" of the Qwen3.5 Chat guide, section "Architektur").
//
// Shared-memory tiles use a row stride of d + 1 floats so that the column
// walks below hit 32 different banks.
#include "gdr_common.cuh"

namespace gdr {

constexpr int kSimtThreads = 256;
constexpr float kGammaFloor = -64.0f;  // clamp of g inside a chunk (exp(-64) ~ 1.6e-28)

template <int D, int C>
struct SimtSmem {
    static constexpr int LD = D + 1, LC = C + 1;
    static constexpr size_t floats = (size_t)D * LD + 4 * (size_t)C * LD + (size_t)C * LC + 3 * C;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, int C, typename TIN, typename TOUT>
__global__ void __launch_bounds__(kSimtThreads) prefill_simt_kernel(const PrefillParams p) {
    constexpr int NT = kSimtThreads, NW = NT / 32;
    constexpr int LD = SimtSmem<D, C>::LD, LC = SimtSmem<D, C>::LC;
    extern __shared__ float smem[];
    float *S = smem;            // [D][LD]   state, row i = value dim i
    float *Qs = S + D * LD;     // [C][LD]   q_hat
    float *Ks = Qs + C * LD;    // [C][LD]   k_hat
    float *Vs = Ks + C * LD;    // [C][LD]   v -> beta v -> U -> Delta
    float *Ws = Vs + C * LD;    // [C][LD]   beta e^gamma k -> W -> O
    float *M = Ws + C * LD;     // [C][LC]   A, then P
    float *gam = M + C * LC;    // [C]       running sum of g
    float *bet = gam + C;       // [C]
    float *gin = bet + C;       // [C]       clamped g

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seq = blockIdx.x / p.H_v, hv = blockIdx.x - seq * p.H_v;
    const int hk = hv / p.hv_per_hk;
    const int64_t t0 = p.cu_seqlens[seq], t1 = p.cu_seqlens[seq + 1];
    const size_t state_off = ((size_t)seq * p.H_v + hv) * D * D;

    for (int e = tid; e < D * D; e += NT)
        S[(e / D) * LD + (e % D)] = p.initial_state ? p.initial_state[state_off + e] : 0.f;

    const TIN *qg = static_cast<const TIN *>(p.q);
    const TIN *kg = static_cast<const TIN *>(p.k);
    const TIN *vg = static_cast<const TIN *>(p.v);
    const TIN *zg = static_cast<const TIN *>(p.z);
    TOUT *og = static_cast<TOUT *>(p.out);

    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
        __syncthreads();  // the previous chunk is done with every tile

        // 1. q_hat, k_hat, v rows (one warp per token); rows >= L are zero.
        for (int r = warp; r < C; r += NW) {
            float qv[D / 32 > 0 ? D / 32 : 1], kv[D / 32 > 0 ? D / 32 : 1];
            float qq = 0.f, kk = 0.f;
            const int64_t t = c0 + r;
#pragma unroll
            for (int m = 0; m < (D + 31) / 32; ++m) {
                const int j = lane + 32 * m;
                float a = 0.f, b = 0.f;
                if (r < L && j < D) {
                    a = Elem<TIN>::load1(qg + t * p.q_stride + hk * D + j);
                    b = Elem<TIN>::load1(kg + t * p.k_stride + hk * D + j);
                }
                qv[m] = a; kv[m] = b;
                qq += a * a; kk += b * b;
            }
            qq = group_sum<32>(qq);
            kk = group_sum<32>(kk);
            float qs = p.scale, ks = 1.f;
            if (p.qk_l2norm) {
                qs *= rsqrtf(qq + p.eps_l2);
                ks = rsqrtf(kk + p.eps_l2);
            }
#pragma unroll
            for (int m = 0; m < (D + 31) / 32; ++m) {
                const int j = lane + 32 * m;
                if (j < D) {
                    Qs[r * LD + j] = qv[m] * qs;
                    Ks[r * LD + j] = kv[m] * ks;
                    Vs[r * LD + j] = r < L ? Elem<TIN>::load1(vg + t * p.v_stride + hv * D + j) : 0.f;
                }
            }
        }
        if (tid < C) {
            const int64_t t = c0 + tid;
            float gv = 0.f, bv = 0.f;
            if (tid < L) {
                gv = __ldg(p.g + t * p.gb_stride + hv);
                bv = __ldg(p.beta + t * p.gb_stride + hv);
                if (p.A_log) {  // raw projections
                    gv = gate_g(gv, __ldg(p.A_log + hv), __ldg(p.dt_bias + hv));
                    bv = gate_beta(bv);
                }
            }
            gin[tid] = tid < L ? fmaxf(gv, kGammaFloor) : 0.f;
            bet[tid] = bv;
        }
        __syncthreads();
        if (tid == 0) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += gin[r]; gam[r] = acc; }
        }
        __syncthreads();

        // 2. A (strictly lower), and the right-hand sides beta v and beta e^gamma k.
        for (int e = tid; e < C * C; e += NT) {
            const int r = e / C, s = e % C;
            float val = 0.f;
            if (s < r && r < L) {
                float acc = 0.f;
#pragma unroll 8
                for (int j = 0; j < D; ++j) acc = fmaf(Ks[r * LD + j], Ks[s * LD + j], acc);
                val = bet[r] * expf(gam[r] - gam[s]) * acc;
            }
            M[r * LC + s] = val;
        }
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, i = e % D;
            Vs[r * LD + i] *= bet[r];
            Ws[r * LD + i] = bet[r] * expf(gam[r]) * Ks[r * LD + i];
        }
        __syncthreads();

        // 3. Forward substitution (I + A) X = RHS, one column per thread.
        for (int c = tid; c < 2 * D; c += NT) {
            float *X = c < D ? Vs + c : Ws + (c - D);
            float x[C];
#pragma unroll
            for (int r = 0; r < C; ++r) x[r] = X[r * LD];
#pragma unroll
            for (int r = 1; r < C; ++r) {
                float acc = x[r];
#pragma unroll
                for (int s = 0; s < r; ++s) acc = fmaf(-M[r * LC + s], x[s], acc);
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < C; ++r) X[r * LD] = x[r];
        }
        __syncthreads();

        // 4. Delta = U - W S^T (in place of U);  P (in place of A).
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, i = e % D;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) acc = fmaf(Ws[r * LD + j], S[i * LD + j], acc);
            Vs[r * LD + i] -= acc;
        }
        for (int e = tid; e < C * C; e += NT) {
            const int r = e / C, s = e % C;
            float val = 0.f;
            if (s <= r && r < L) {
                float acc = 0.f;
#pragma unroll 8
                for (int j = 0; j < D; ++j) acc = fmaf(Qs[r * LD + j], Ks[s * LD + j], acc);
                val = expf(gam[r] - gam[s]) * acc;
            }
            M[r * LC + s] = val;
        }
        __syncthreads();

        // 5. O = diag(e^gamma) Q S^T + P Delta (in place of W); the clamped g
        //    is no longer needed, so its slot takes exp(gamma_L - gamma_s).
        if (tid < C) gin[tid] = expf(gam[L - 1] - gam[tid]);
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, i = e % D;
            float inter = 0.f, intra = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) inter = fmaf(Qs[r * LD + j], S[i * LD + j], inter);
            for (int s = 0; s <= r; ++s) intra = fmaf(M[r * LC + s], Vs[s * LD + i], intra);
            Ws[r * LD + i] = expf(gam[r]) * inter + intra;
        }
        __syncthreads();

        // 6. Gate and store the chunk's outputs (one warp per token).
        for (int r = warp; r < L; r += NW) {
            const int64_t t = c0 + r;
            float ov[(D + 31) / 32];
            float ss = 0.f;
#pragma unroll
            for (int m = 0; m < (D + 31) / 32; ++m) {
                const int i = lane + 32 * m;
                ov[m] = i < D ? Ws[r * LD + i] : 0.f;
                ss += ov[m] * ov[m];
            }
            ss = group_sum<32>(ss);
            const float rstd = rsqrtf(ss * (1.0f / D) + p.eps_norm);
#pragma unroll
            for (int m = 0; m < (D + 31) / 32; ++m) {
                const int i = lane + 32 * m;
                if (i >= D) continue;
                float y = ov[m];
                if (zg) {
                    const float zz = Elem<TIN>::load1(zg + t * p.z_stride + hv * D + i);
                    const float wv = p.norm_w ? __ldg(p.norm_w + i) : 1.f;
                    y = y * rstd * wv * silu(zz);
                }
                Elem<TOUT>::store1(og + t * p.out_stride + hv * D + i, y);
            }
        }
        // 7. State to the end of the chunk.
        const float eL = expf(gam[L - 1]);
        for (int e = tid; e < D * D; e += NT) {
            const int i = e / D, j = e % D;
            float acc = eL * S[i * LD + j];
            for (int s = 0; s < L; ++s)
                acc = fmaf(Vs[s * LD + i] * gin[s], Ks[s * LD + j], acc);
            S[i * LD + j] = acc;
        }
    }
    __syncthreads();
    if (p.final_state)
        for (int e = tid; e < D * D; e += NT) p.final_state[state_off + e] = S[(e / D) * LD + (e % D)];
}

template <int D, int C, typename TIN, typename TOUT>
static cudaError_t launch_simt_t(const PrefillParams &p, cudaStream_t s) {
    constexpr size_t smem = SimtSmem<D, C>::bytes;
    auto kern = prefill_simt_kernel<D, C, TIN, TOUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.n_seq * p.H_v;
    kern<<<(unsigned)grid, kSimtThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int D, int C>
static cudaError_t launch_simt_dc(const PrefillParams &p, int in_bf16, int out_bf16,
                                  cudaStream_t s) {
    if (in_bf16)
        return out_bf16 ? launch_simt_t<D, C, __nv_bfloat16, __nv_bfloat16>(p, s)
                        : launch_simt_t<D, C, __nv_bfloat16, float>(p, s);
    return out_bf16 ? launch_simt_t<D, C, float, __nv_bfloat16>(p, s)
                    : launch_simt_t<D, C, float, float>(p, s);
}

template <int D>
static cudaError_t launch_simt_d(const PrefillParams &p, int chunk, int in_bf16, int out_bf16,
                                 cudaStream_t s) {
    switch (chunk) {
        case 16: return launch_simt_dc<D, 16>(p, in_bf16, out_bf16, s);
        case 32: return launch_simt_dc<D, 32>(p, in_bf16, out_bf16, s);
        case 64: return launch_simt_dc<D, 64>(p, in_bf16, out_bf16, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_prefill_simt(const PrefillParams &p, int d, int chunk, int in_bf16,
                                int out_bf16, cudaStream_t s) {
    switch (d) {
        case 16: return launch_simt_d<16>(p, chunk, in_bf16, out_bf16, s);
        case 32: return launch_simt_d<32>(p, chunk, in_bf16, out_bf16, s);
        case 64: return launch_simt_d<64>(p, chunk, in_bf16, out_bf16, s);
        case 128: return launch_simt_d<128>(p, chunk, in_bf16, out_bf16, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdr
