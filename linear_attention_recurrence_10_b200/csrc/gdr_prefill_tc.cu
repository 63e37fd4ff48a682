// gdr_prefill_tc.cu -- chunked prefill of the gated delta rule on the sm_100a
// tensor cores (tcgen05), bf16 inputs, d_k = d_v = 128, chunk 64.
//
// The mixer is the "gated delta rule" recurrence with an RMSNormGated output
// (Qwen3.5 Chat guide, section "Architektur"), with key heads shared by
// groups of value heads (Core AI Qwen3.6-35B-A3B card, first section).  Per
// chunk of C = 64 tokens and value head, with S the state entering the chunk
// (d_v x d_k fp32), raw bf16 rows q_r, k_r, v_r, n_r = 1/|k_r|,
// m_r = scale/|q_r| and gamma_r the running sum of g inside the chunk:
//
//   [KK; QK] = [K; Q] K^T                                bf16 MMA (exact products)
//   A_rs = beta_r e^{gamma_r-gamma_s} n_r n_s KK_rs  (s<r)     on CUDA cores
//   P_rs = e^{gamma_r-gamma_s} m_r n_s QK_rs         (s<=r)
//   T    = (I + A)^{-1}                                 blocked, fp32, CUDA cores
//   U^T  = V^T (T diag(beta))^T                         tf32 MMA
//   W    = T diag(beta e^gamma n) K                     tf32 MMA
//   Delta^T = U^T - S_bf16 W^T                          bf16 MMA into the U^T accumulator
//   O^T  = diag-scaled S_bf16 Q^T + Delta^T P^T         bf16 + tf32 MMA
//   S    = e^{gamma_L} S + (Delta^T diag(e^{gamma_L-gamma} n)) K   tf32 MMA into TMEM
//   y    = RMSNormGated(O) -> out
//
// which is the chunkwise (WY / UT transform) form of
// S_t = e^{g_t} S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
// The state lives in tensor memory in fp32 for the whole sequence; the MMAs
// that read it see a bf16 copy.  Which operands may be bf16 was decided by
// emulating every rounding point against the fp64 recurrence: the inverse T,
// P and Delta must stay tf32 or better; S and W may be bf16.
//
// One CTA (256 threads) owns one (sequence, value head) and walks its chunks
// in order.  Sequences are taken longest first (the order is written to the
// workspace by a small pre-kernel).  Every mbarrier wait is bounded by a
// wall-clock deadline; on expiry the CTA records GDR_ERR_TIMEOUT in the
// workspace status word, frees its tensor memory and returns.
#include "gdr_common.cuh"
#include "gdr_tc.cuh"

namespace gdr {
namespace tcp {

using namespace gdr::tc;

constexpr int D = 128;       // d_k = d_v
constexpr int C = 64;        // chunk
constexpr int NT = 256;      // threads
constexpr int NW = NT / 32;
constexpr int LDA = C + 1;   // padded row stride of the fp32 scratch matrices
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: far beyond any chunk's work
constexpr float kGammaFloor = -64.0f;
constexpr int kTimeoutStatus = 6;  // GDR_ERR_TIMEOUT

// Shared memory map (bytes).
constexpr uint32_t OFF_KQ = 0;          // bf16 [K;Q] K-major, 128 rows x 128 (32 KB)
constexpr uint32_t OFF_VT = 32768;      // fp32 V^T K-major [i][s] (32 KB); later O staging [r][i]
constexpr uint32_t OFF_KT = 65536;      // fp32 K^T K-major [j][s] (32 KB)
constexpr uint32_t OFF_SCR = 98304;     // fp32 A, T [64][65], X [3][16][16]; later W bf16, later Dt~
constexpr uint32_t OFF_TBW = 135168;    // fp32 TB, TW K-major [r][s] (16 KB each); later Delta^T
constexpr uint32_t OFF_P = 167936;      // fp32 P K-major [r][s] (16 KB)
constexpr uint32_t OFF_S = 184320;      // bf16 S K-major [i][j] (32 KB)
constexpr uint32_t OFF_SCAL = 217088;   // per-token scalars and the mbarrier
constexpr uint32_t SMEM_BYTES = OFF_SCAL + 2048;

// Tensor memory columns (512 allocated).
constexpr uint32_t TM_D1 = 0;     // [KK; QK]           M=128, 64 cols
constexpr uint32_t TM_U = 64;     // U^T -> Delta^T     M=128, 64 cols
constexpr uint32_t TM_W = 128;    // W [r][j]           M=64, 128 cols
constexpr uint32_t TM_OI = 256;   // S Q^T              M=128, 64 cols
constexpr uint32_t TM_O2 = 320;   // Delta^T P^T        M=128, 64 cols
constexpr uint32_t TM_S = 384;    // state S [i][j]     M=128, 128 cols

// Byte offset of (row, k) in a K-major tile of R rows (16-byte chunks along K).
__device__ __forceinline__ uint32_t kmaj(int row, int k, int R, int esz) {
    const int E = 16 / esz;
    return (uint32_t)((k / E) * (R * 16) + (row >> 3) * 128 + (row & 7) * 16 + (k % E) * esz);
}

// D (+)= A B^T over `ksteps` instructions; both operands K-major no-swizzle.
template <Kind KD>
__device__ __forceinline__ void gemm(uint32_t d, uint32_t a, uint32_t a_lbo, uint32_t b,
                                     uint32_t b_lbo, int ksteps, uint32_t idesc, bool acc) {
    for (int kk = 0; kk < ksteps; ++kk)
        mma<KD>(d, smem_desc(a + kk * 2 * a_lbo, a_lbo, 128), smem_desc(b + kk * 2 * b_lbo, b_lbo, 128),
                idesc, (acc || kk > 0) ? 1u : 0u);
}

// Eight consecutive fp32 values as eight bf16 (round to nearest even) in 16 bytes.
__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[32], int o) {
    uint4 pk;
    __nv_bfloat162 b0 = __floats2bfloat162_rn(v[o + 0], v[o + 1]);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(v[o + 2], v[o + 3]);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(v[o + 4], v[o + 5]);
    __nv_bfloat162 b3 = __floats2bfloat162_rn(v[o + 6], v[o + 7]);
    pk.x = *reinterpret_cast<uint32_t *>(&b0);
    pk.y = *reinterpret_cast<uint32_t *>(&b1);
    pk.z = *reinterpret_cast<uint32_t *>(&b2);
    pk.w = *reinterpret_cast<uint32_t *>(&b3);
    return pk;
}

struct Scalars {
    float gam[C], eg[C], bet[C], nk[C], nq[C], dec[C];
    uint64_t bar;
    uint32_t tmem;
    int abort;
};

template <typename TOUT>
__global__ void __launch_bounds__(NT, 1) prefill_tc_kernel(const PrefillParams p, const int *order,
                                                           int *status) {
    extern __shared__ __align__(1024) unsigned char sm[];
    Scalars &sc = *reinterpret_cast<Scalars *>(sm + OFF_SCAL);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quad = warp & 3, half = warp >> 2;  // TMEM lane quadrant, column half

    const int unit = blockIdx.x;
    const int seq = order[unit / p.H_v];
    const int hv = unit % p.H_v;
    const int hk = hv / p.hv_per_hk;
    const int64_t t0 = p.cu_seqlens[seq], t1 = p.cu_seqlens[seq + 1];

    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *zg = static_cast<const __nv_bfloat16 *>(p.z);
    TOUT *og = static_cast<TOUT *>(p.out);

    const uint32_t sbase = smem_u32(sm);
    float *Ascr = reinterpret_cast<float *>(sm + OFF_SCR);
    float *Tscr = Ascr + C * LDA;
    float *Xscr = Tscr + C * LDA;

    if (warp == 0) tmem_alloc(&sc.tmem, 512);
    if (tid == 0) {
        mbar_init(&sc.bar, 1);
        mbar_fence_init();
        sc.abort = 0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = sc.tmem;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    uint32_t phase = 0;

    // Wait for the MMAs committed to the barrier; every thread learns together
    // whether the wait gave up.
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait(&sc.bar, phase, kWaitNs);
        phase ^= 1;
        const int bad = __syncthreads_or(!ok);
        fence_after_sync();
        if (bad && tid == 0) atomicExch(status, kTimeoutStatus);
        return !bad;
    };
    auto issue_and_wait = [&](auto issue) -> bool {
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            issue();
            commit(smem_u32(&sc.bar));
        }
        return wait_mma();
    };

    // Initial state into TMEM (fp32) and its bf16 copy into smem.
    {
        const int i = 32 * quad + lane;
        const float *s0 = p.initial_state
                              ? p.initial_state + ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D
                              : nullptr;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int j0 = 64 * half + 32 * cc;
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = s0 ? s0[j0 + j] : 0.f;
            tmem_st32(tm + lane_off + TM_S + j0, v);
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8)
                *reinterpret_cast<uint4 *>(sm + OFF_S + kmaj(i, j0 + 8 * j8, D, 2)) = pack8_bf16(v, 8 * j8);
        }
    }

    const uint32_t ID_BF_64 = instr_desc<Kind::BF16>(128, 64, false, false);
    const uint32_t ID_BF_64_NEG = instr_desc<Kind::BF16>(128, 64, false, false, true);
    const uint32_t ID_TF_64 = instr_desc<Kind::TF32>(128, 64, false, false);
    const uint32_t ID_TF_128 = instr_desc<Kind::TF32>(128, 128, false, false);
    const uint32_t ID_TF_M64_128 = instr_desc<Kind::TF32>(64, 128, false, false);

    bool alive = true;
    for (int64_t c0 = t0; c0 < t1 && alive; c0 += C) {
        const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);

        // ---- P1: inputs.  [K;Q] bf16 tile: lanes take (row % 8, 16-byte chunk) so
        // that each quarter-warp stores one contiguous 128-byte core-matrix column.
        for (int e = tid; e < 128 * 16; e += NT) {
            const int row = (e & 7) + 8 * ((e >> 5) & 15);
            const int jc = ((e >> 3) & 3) + 4 * (e >> 9);
            const int r = row & 63;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (r < L) {
                const __nv_bfloat16 *src = row < 64 ? kg + (c0 + r) * p.k_stride + hk * D
                                                    : qg + (c0 + r) * p.q_stride + hk * D;
                val = __ldg(reinterpret_cast<const uint4 *>(src + 8 * jc));
            }
            *reinterpret_cast<uint4 *>(sm + OFF_KQ + kmaj(row, 8 * jc, 128, 2)) = val;
        }
        // V^T fp32 tile [i][s]: one (i, 4 tokens) chunk per step.
        for (int e = tid; e < D * (C / 4); e += NT) {
            const int i = e & (D - 1), sc4 = e >> 7;
            float4 val;
            float *pv = &val.x;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = 4 * sc4 + u;
                pv[u] = s < L ? __bfloat162float(vg[(c0 + s) * p.v_stride + hv * D + i]) : 0.f;
            }
            *reinterpret_cast<float4 *>(sm + OFF_VT + kmaj(i, 4 * sc4, D, 4)) = val;
        }
        // Per-token scalars: norms (one warp per row), gates.
        for (int row = warp; row < 128; row += NW) {
            const int r = row & 63;
            float ss = 0.f;
            if (r < L) {
                const __nv_bfloat16 *src = row < 64 ? kg + (c0 + r) * p.k_stride + hk * D
                                                    : qg + (c0 + r) * p.q_stride + hk * D;
                const float4 x = Elem<__nv_bfloat16>::load4(src + 4 * lane);
                ss = dot4(x, x);
            }
            ss = group_sum<32>(ss);
            if (lane == 0) {
                const float f = p.qk_l2norm ? rsqrtf(ss + p.eps_l2) : 1.0f;
                if (row < 64) sc.nk[r] = r < L ? f : 0.f;
                else sc.nq[r] = r < L ? f * p.scale : 0.f;
            }
        }
        if (warp == 0) {
            float ga = 0.f, gb = 0.f, ba = 0.f, bb = 0.f;
            if (lane < L) {
                ga = fmaxf(__ldg(p.g + (c0 + lane) * p.gb_stride + hv), kGammaFloor);
                ba = __ldg(p.beta + (c0 + lane) * p.gb_stride + hv);
            }
            if (lane + 32 < L) {
                gb = fmaxf(__ldg(p.g + (c0 + lane + 32) * p.gb_stride + hv), kGammaFloor);
                bb = __ldg(p.beta + (c0 + lane + 32) * p.gb_stride + hv);
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float xa = __shfl_up_sync(kFullMask, ga, o);
                const float xb = __shfl_up_sync(kFullMask, gb, o);
                if (lane >= o) { ga += xa; gb += xb; }
            }
            gb += __shfl_sync(kFullMask, ga, 31);
            sc.gam[lane] = ga;
            sc.gam[lane + 32] = gb;
            sc.bet[lane] = ba;
            sc.bet[lane + 32] = bb;
            sc.eg[lane] = expf(ga);
            sc.eg[lane + 32] = expf(gb);
        }
        __syncthreads();
        if (tid < C) sc.dec[tid] = expf(sc.gam[L - 1] - sc.gam[tid]);
        // K^T fp32 tile [j][s] from the bf16 tile (rows 0..63 hold K).
        for (int e = tid; e < D * (C / 4); e += NT) {
            const int j = e & (D - 1), sc4 = e >> 7;
            float4 val;
            float *pv = &val.x;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                pv[u] = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_KQ + kmaj(4 * sc4 + u, j, 128, 2)));
            *reinterpret_cast<float4 *>(sm + OFF_KT + kmaj(j, 4 * sc4, D, 4)) = val;
        }

        // ---- P2: [KK; QK] = [K;Q] K^T and S Q^T (state entering the chunk).
        alive = issue_and_wait([&] {
            gemm<Kind::BF16>(tm + TM_D1, sbase + OFF_KQ, 2048, sbase + OFF_KQ, 2048, D / 16, ID_BF_64,
                             false);
            gemm<Kind::BF16>(tm + TM_OI, sbase + OFF_S, 2048, sbase + OFF_KQ + 1024, 2048, D / 16,
                             ID_BF_64, false);
        });
        if (!alive) break;

        // ---- P3: A (fp32 scratch) and P (tf32 operand tile).
        {
            const int rr = 32 * (quad & 1) + lane;  // token row
            const int s0 = 32 * half;
            float v[32];
            tmem_ld32(tm + lane_off + TM_D1 + s0, v);
            if (quad < 2) {
                const float f = sc.bet[rr] * sc.nk[rr];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int s = s0 + c;
                    Ascr[rr * LDA + s] = s < rr ? f * expf(sc.gam[rr] - sc.gam[s]) * sc.nk[s] * v[c] : 0.f;
                }
            } else {
                const float f = sc.nq[rr];
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    float4 w;
                    float *pw = &w.x;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s = s0 + 4 * c4 + u;
                        pw[u] = s <= rr ? to_tf32(f * expf(sc.gam[rr] - sc.gam[s]) * sc.nk[s] * v[4 * c4 + u])
                                        : 0.f;
                    }
                    *reinterpret_cast<float4 *>(sm + OFF_P + kmaj(rr, s0 + 4 * c4, C, 4)) = w;
                }
            }
        }
        __syncthreads();

        // ---- P4: T = (I + A)^{-1}, blocked by 16.  Diagonal blocks first, one
        // column per thread; then off-diagonal blocks by distance from the diagonal:
        // T_ij = -T_ii sum_{16j <= k < 16i} A[i-rows][k] T[k][j-cols].
        if (tid < C) {
            const int b = tid >> 4, c = tid & 15, base = 16 * b;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                if (r > c) {
                    float acc = 0.f;
#pragma unroll
                    for (int s = 0; s < r; ++s) acc = fmaf(Ascr[(base + r) * LDA + base + s], x[s], acc);
                    x[r] = -acc;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tscr[(base + r) * LDA + base + c] = x[r];
        }
        for (int e = tid; e < C * C; e += NT) {  // zero the blocks above the diagonal
            const int r = e >> 6, s = e & 63;
            if ((s >> 4) > (r >> 4)) Tscr[r * LDA + s] = 0.f;
        }
        __syncthreads();
        for (int dist = 1; dist < 4; ++dist) {
            const int nblk = 4 - dist;
            for (int e = tid; e < nblk * 256; e += NT) {
                const int j = e >> 8, i = j + dist, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
                for (int k = 16 * j; k < 16 * i; ++k)
                    acc = fmaf(Ascr[(16 * i + rr) * LDA + k], Tscr[k * LDA + 16 * j + cc], acc);
                Xscr[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nblk * 256; e += NT) {
                const int j = e >> 8, i = j + dist, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    acc = fmaf(Tscr[(16 * i + rr) * LDA + 16 * i + k], Xscr[(j << 8) + k * 16 + cc], acc);
                Tscr[(16 * i + rr) * LDA + 16 * j + cc] = -acc;
            }
            __syncthreads();
        }
        // TB = T diag(beta), TW = T diag(beta e^gamma n): tf32 tiles [r][s].
        for (int e = tid; e < C * (C / 4); e += NT) {
            const int r = e & 63, sc4 = e >> 6;
            float4 tb, tw;
            float *pb = &tb.x, *pw = &tw.x;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = 4 * sc4 + u;
                const float t = Tscr[r * LDA + s];
                pb[u] = to_tf32(t * sc.bet[s]);
                pw[u] = to_tf32(t * sc.bet[s] * sc.eg[s] * sc.nk[s]);
            }
            *reinterpret_cast<float4 *>(sm + OFF_TBW + kmaj(r, 4 * sc4, C, 4)) = tb;
            *reinterpret_cast<float4 *>(sm + OFF_TBW + 16384 + kmaj(r, 4 * sc4, C, 4)) = tw;
        }

        // ---- P5: U^T = V^T TB^T (M=128), W = TW K (M=64, tokens in lanes).
        alive = issue_and_wait([&] {
            gemm<Kind::TF32>(tm + TM_U, sbase + OFF_VT, 2048, sbase + OFF_TBW, 1024, C / 8, ID_TF_64,
                             false);
            gemm<Kind::TF32>(tm + TM_W, sbase + OFF_TBW + 16384, 1024, sbase + OFF_KT, 2048, C / 8,
                             ID_TF_M64_128, false);
        });
        if (!alive) break;

        // ---- P6: W -> bf16 operand [r][j]; rescale the TMEM state by e^{gamma_L}.
        {
            // An M=64 accumulator occupies lanes 0..15 of each 32-lane quadrant;
            // the warp-wide tcgen05.ld runs on every lane, lanes 16..31 discard.
            const int r = 16 * quad + (lane & 15);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int j0 = 64 * half + 32 * cc;
                float v[32];
                tmem_ld32(tm + lane_off + TM_W + j0, v);
                if (lane < 16) {
#pragma unroll
                    for (int j8 = 0; j8 < 4; ++j8) {
                        *reinterpret_cast<uint4 *>(sm + OFF_SCR + kmaj(r, j0 + 8 * j8, C, 2)) =
                            pack8_bf16(v, 8 * j8);
                    }
                }
            }
            const float eL = sc.eg[L - 1];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int j0 = 64 * half + 32 * cc;
                float v[32];
                tmem_ld32(tm + lane_off + TM_S + j0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= eL;
                tmem_st32(tm + lane_off + TM_S + j0, v);
            }
        }

        // ---- P7: Delta^T = U^T - S W^T (accumulates into the U^T columns).
        alive = issue_and_wait([&] {
            gemm<Kind::BF16>(tm + TM_U, sbase + OFF_S, 2048, sbase + OFF_SCR, 1024, D / 16, ID_BF_64_NEG,
                             true);
        });
        if (!alive) break;

        // ---- P8: Delta^T (tf32 [i][s]) and its decayed, k-normalised copy.
        {
            const int i = 32 * quad + lane;
            const int s0 = 32 * half;
            float v[32];
            tmem_ld32(tm + lane_off + TM_U + s0, v);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                float4 a, b;
                float *pa = &a.x, *pb = &b.x;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int s = s0 + 4 * c4 + u;
                    const float dlt = v[4 * c4 + u];
                    pa[u] = to_tf32(dlt);
                    pb[u] = to_tf32(dlt * sc.dec[s] * sc.nk[s]);
                }
                *reinterpret_cast<float4 *>(sm + OFF_TBW + kmaj(i, s0 + 4 * c4, D, 4)) = a;
                *reinterpret_cast<float4 *>(sm + OFF_SCR + kmaj(i, s0 + 4 * c4, D, 4)) = b;
            }
        }

        // ---- P9: O_intra^T = Delta^T P^T; S += Dt~ K.
        alive = issue_and_wait([&] {
            gemm<Kind::TF32>(tm + TM_O2, sbase + OFF_TBW, 2048, sbase + OFF_P, 1024, C / 8, ID_TF_64,
                             false);
            gemm<Kind::TF32>(tm + TM_S, sbase + OFF_SCR, 2048, sbase + OFF_KT, 2048, C / 8, ID_TF_128,
                             true);
        });
        if (!alive) break;

        // ---- P10: O = m e^gamma (S Q^T) + Delta P^T staged as [r][i]; the new
        // state's bf16 copy for the next chunk.
        {
            const int i = 32 * quad + lane;
            const int r0 = 32 * half;
            float a[32], b[32];
            tmem_ld32(tm + lane_off + TM_OI + r0, a);
            tmem_ld32(tm + lane_off + TM_O2 + r0, b);
            float *Os = reinterpret_cast<float *>(sm + OFF_VT);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int r = r0 + c;
                Os[r * D + i] = fmaf(sc.nq[r] * sc.eg[r], a[c], b[c]);
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int j0 = 64 * half + 32 * cc;
                float v[32];
                tmem_ld32(tm + lane_off + TM_S + j0, v);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8)
                    *reinterpret_cast<uint4 *>(sm + OFF_S + kmaj(i, j0 + 8 * j8, D, 2)) =
                        pack8_bf16(v, 8 * j8);
            }
        }
        __syncthreads();
        // RMSNormGated per token (one warp per token), store.
        {
            const float *Os = reinterpret_cast<const float *>(sm + OFF_VT);
            for (int r = warp; r < L; r += NW) {
                const int64_t t = c0 + r;
                const float4 o4 = *reinterpret_cast<const float4 *>(Os + r * D + 4 * lane);
                float4 y = o4;
                if (zg) {
                    const float ss = group_sum<32>(dot4(o4, o4));
                    const float rstd = rsqrtf(ss * (1.0f / D) + p.eps_norm);
                    const float4 z4 = Elem<__nv_bfloat16>::load4(zg + t * p.z_stride + hv * D + 4 * lane);
                    float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
                    if (p.norm_w) {
                        w4.x = __ldg(p.norm_w + 4 * lane + 0);
                        w4.y = __ldg(p.norm_w + 4 * lane + 1);
                        w4.z = __ldg(p.norm_w + 4 * lane + 2);
                        w4.w = __ldg(p.norm_w + 4 * lane + 3);
                    }
                    y.x = o4.x * rstd * w4.x * silu(z4.x);
                    y.y = o4.y * rstd * w4.y * silu(z4.y);
                    y.z = o4.z * rstd * w4.z * silu(z4.z);
                    y.w = o4.w * rstd * w4.w * silu(z4.w);
                }
                Elem<TOUT>::store4(og + t * p.out_stride + hv * D + 4 * lane, y);
            }
        }
        __syncthreads();
    }

    // Final state from TMEM.
    if (alive && p.final_state) {
        const int i = 32 * quad + lane;
        float *dst = p.final_state + ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int j0 = 64 * half + 32 * cc;
            float v[32];
            tmem_ld32(tm + lane_off + TM_S + j0, v);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
                *reinterpret_cast<float4 *>(dst + j0 + 4 * j4) =
                    make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_free(tm, 512);
    }
}

// Longest sequences first: order[rank] = sequence.  Also clears the status word.
__global__ void lpt_order_kernel(const int32_t *cu, int n_seq, int *order, int *status) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n_seq; s += gridDim.x * blockDim.x) {
        const int ls = cu[s + 1] - cu[s];
        int rank = 0;
        for (int t = 0; t < n_seq; ++t) {
            const int lt = cu[t + 1] - cu[t];
            rank += (lt > ls) || (lt == ls && t < s);
        }
        order[rank] = s;
    }
}

}  // namespace tcp

size_t prefill_tc_workspace_bytes(int n_seq) {
    return (size_t)(16 + 4 * (size_t)n_seq + 255) & ~(size_t)255;
}

cudaError_t launch_prefill_tc(const PrefillParams &p, void *workspace, int out_bf16,
                              cudaStream_t s) {
    int *status = static_cast<int *>(workspace);
    int *order = status + 4;
    const int blocks = (p.n_seq + 255) / 256;
    tcp::lpt_order_kernel<<<blocks < 64 ? blocks : 64, 256, 0, s>>>(p.cu_seqlens, p.n_seq, order,
                                                                     status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto kern = out_bf16 ? tcp::prefill_tc_kernel<__nv_bfloat16> : tcp::prefill_tc_kernel<float>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcp::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.n_seq * p.H_v;
    kern<<<(unsigned)grid, tcp::NT, tcp::SMEM_BYTES, s>>>(p, order, status);
    return cudaGetLastError();
}

}  // namespace gdr
