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
//   [KK; QK] = [K; Q] K^T                                     (exact bf16 products)
//   A_rs = beta_r e^{gamma_r-gamma_s} n_r n_s KK_rs    (s<r)   on CUDA cores
//   P_rs = e^{gamma_r-gamma_s} m_r n_s QK_rs           (s<=r)
//   T    = (I + A)^{-1}                                       blocked, fp32, CUDA cores
//   U^T  = V^T (T diag(beta))^T
//   W^T  = K^T (T diag(beta e^gamma n))^T
//   Delta^T = U^T - S W^T                                     (into the U^T accumulator)
//   O^T  = diag-scaled S Q^T + Delta^T P^T
//   S    = e^{gamma_L} S + (Delta^T diag(e^{gamma_L-gamma} n)) K     (into the TMEM state)
//   y    = RMSNormGated(O) -> out
//
// which is the chunkwise (WY / UT transform) form of
// S_t = e^{g_t} S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
//
// Every MMA is kind::f16 with bf16 operands and fp32 accumulation in tensor
// memory.  The fp32 state stays in tensor memory for the whole sequence; the
// MMAs that read it see a bf16 copy (harmless: emulating every rounding point
// against the fp64 recurrence showed S and W may be bf16).  The computed
// operands that must keep more precision -- T diag(beta), T diag(beta e^gamma n),
// P, Delta and the decayed Delta -- are split into hi + lo bf16 pairs
// (x = hi + lo to ~16 bits) and multiplied term by term (for P Delta:
// hi*hi + hi*lo + lo*hi).  q, k, v enter the MMAs as the exact bf16 inputs.
//
// One CTA (512 threads) owns one (sequence, value head) and walks its chunks
// in order; each chunk's inputs are fetched by cp.async one chunk ahead.
// Sequences are taken longest first (order written to the workspace by a
// pre-kernel).  Every mbarrier wait is bounded by a wall-clock deadline; on
// expiry the CTA records GDR_ERR_TIMEOUT in the workspace status word, frees
// its tensor memory and returns.
#include "gdr_prefill_common.cuh"

namespace gdr {
namespace tcp {

constexpr int NT = 512;      // threads (16 warps)
constexpr int NW = NT / 32;

// Shared memory map (bytes).
constexpr uint32_t OFF_KQ = 0;          // 2 x bf16 [K;Q], 128 rows x 128, row-group major (32 KB each)
constexpr uint32_t OFF_V = 65536;       // bf16 V, MN-major over d_v (16 KB)
constexpr uint32_t OFF_Z = 81920;       // bf16 z rows [s][i] (16 KB)
constexpr uint32_t OFF_SCR = 98304;     // fp32 A, T [64][65], X; later W^T tile; later Dt~ hi/lo
constexpr uint32_t OFF_TBW = 135168;    // TB hi/lo, TW hi/lo (8 KB each); later Delta hi/lo; later O
constexpr uint32_t OFF_P = 167936;      // P hi/lo (8 KB each)
constexpr uint32_t OFF_S = 184320;      // bf16 S [i][j] (32 KB)
constexpr uint32_t OFF_GB = 217088;     // 2 x (g[64], beta[64]) fp32
constexpr uint32_t OFF_SCAL = 218112;   // per-token scalars, mbarrier
constexpr uint32_t SMEM_BYTES = OFF_SCAL + 2048;
constexpr uint32_t KQ_BYTES = 32768;

// Tensor memory columns (512 allocated).
constexpr uint32_t TM_D1 = 0;     // [KK; QK]         M=128, 64 cols
constexpr uint32_t TM_U = 64;     // U^T -> Delta^T   M=128, 64 cols
constexpr uint32_t TM_W = 128;    // W^T [j][r]       M=128, 64 cols
constexpr uint32_t TM_OI = 192;   // S Q^T            M=128, 64 cols
constexpr uint32_t TM_O2 = 256;   // Delta^T P^T      M=128, 64 cols
constexpr uint32_t TM_S = 384;    // state S [i][j]   M=128, 128 cols

struct Scalars {
    float gam[C], eg[C], bet[C], nk[C], nq[C], dec[C];
    uint64_t bar;
    uint32_t tmem;
};

template <typename TOUT>
__global__ void __launch_bounds__(NT, 1) prefill_tc_kernel(const PrefillParams p, const int *order,
                                                           int *status) {
    extern __shared__ __align__(1024) unsigned char sm[];
    Scalars &sc = *reinterpret_cast<Scalars *>(sm + OFF_SCAL);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quad = warp & 3, part = warp >> 2;  // TMEM lane quadrant, column quarter

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
    float *gbuf = reinterpret_cast<float *>(sm + OFF_GB);  // [2][g 64 | beta 64]

    // ---- asynchronous input fetches (every thread issues its share) ----------
    auto fetch_kq = [&](int64_t c0, int L, int buf) {
        unsigned char *dst = sm + OFF_KQ + buf * KQ_BYTES;
        for (int e = tid; e < 128 * 16; e += NT) {
            // lanes take (row % 8, 16-byte chunk) so each quarter-warp fills one
            // contiguous 128-byte core-matrix column
            const int row = (e & 7) + 8 * ((e >> 5) & 15);
            const int jc = ((e >> 3) & 3) + 4 * (e >> 9);
            const int r = row & 63;
            const bool in = r < L;
            const int64_t t = in ? c0 + r : t0;
            const __nv_bfloat16 *src = row < 64 ? kg + t * p.k_stride + hk * D
                                                : qg + t * p.q_stride + hk * D;
            cp_async16(dst + kq_off(row, 8 * jc), src + 8 * jc, in ? 16u : 0u);
        }
    };
    auto fetch_v = [&](int64_t c0, int L) {
        for (int e = tid; e < C * 16; e += NT) {
            const int s = (e & 7) + 8 * ((e >> 5) & 7);
            const int ic = ((e >> 3) & 3) + 4 * (e >> 8);
            const bool in = s < L;
            const int64_t t = in ? c0 + s : t0;
            cp_async16(sm + OFF_V + v_off(s, 8 * ic), vg + t * p.v_stride + hv * D + 8 * ic,
                       in ? 16u : 0u);
        }
    };
    auto fetch_z = [&](int64_t c0, int L) {
        if (!zg) return;
        for (int e = tid; e < C * 16; e += NT) {
            const int s = e >> 4, ic = e & 15;
            const bool in = s < L;
            const int64_t t = in ? c0 + s : t0;
            cp_async16(sm + OFF_Z + s * 256 + ic * 16, zg + t * p.z_stride + hv * D + 8 * ic,
                       in ? 16u : 0u);
        }
    };
    auto fetch_gb = [&](int64_t c0, int L, int buf) {
        if (tid < 2 * C) {
            const int r = tid & 63;
            const bool in = r < L;
            const int64_t t = in ? c0 + r : t0;
            const float *src = (tid < C ? p.g : p.beta) + t * p.gb_stride + hv;
            cp_async4(gbuf + buf * 2 * C + tid, src, in ? 4u : 0u);
        }
    };

    if (warp == 0) tmem_alloc(&sc.tmem, 512);
    if (tid == 0) {
        mbar_init(&sc.bar, 1);
        mbar_fence_init();
    }
    if (t1 > t0) {
        const int L0 = (int)((t1 - t0) < C ? (t1 - t0) : C);
        fetch_kq(t0, L0, 0);
        fetch_gb(t0, L0, 0);
        fetch_v(t0, L0);
    }
    cp_async_commit();
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
        for (int cc = 0; cc < 1; ++cc) {
            const int j0 = 32 * part;
            float v[32];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                float4 x = s0 ? *reinterpret_cast<const float4 *>(s0 + j0 + 4 * j4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * j4] = x.x; v[4 * j4 + 1] = x.y; v[4 * j4 + 2] = x.z; v[4 * j4 + 3] = x.w;
            }
            tmem_st32(tm + lane_off + TM_S + j0, v);
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8)
                *reinterpret_cast<uint4 *>(sm + OFF_S + kmaj(i, j0 + 8 * j8, D)) = pack8(v + 8 * j8);
        }
    }

    const uint32_t ID_KK = instr_desc<Kind::BF16>(128, 64, false, false);
    const uint32_t ID_U = instr_desc<Kind::BF16>(128, 64, true, false);     // A = V, MN-major
    const uint32_t ID_D = instr_desc<Kind::BF16>(128, 64, false, true, true);  // -S, B = W MN-major
    const uint32_t ID_S = instr_desc<Kind::BF16>(128, 128, false, true);    // B = K, MN-major
    const uint32_t aKQ = sbase + OFF_KQ;

    float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);  // RMSNormGated weight of this lane's 4 columns
    if (p.norm_w)
        w4 = make_float4(__ldg(p.norm_w + 4 * lane), __ldg(p.norm_w + 4 * lane + 1),
                         __ldg(p.norm_w + 4 * lane + 2), __ldg(p.norm_w + 4 * lane + 3));
    bool alive = true;
    int buf = 0;
    for (int64_t c0 = t0; c0 < t1 && alive; c0 += C, buf ^= 1) {
        const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
        const int64_t n0 = c0 + C;
        const int Ln = (int)((t1 - n0) < C ? (t1 - n0) : C);
        const uint32_t kq = aKQ + buf * KQ_BYTES;
        const unsigned char *kqp = sm + OFF_KQ + buf * KQ_BYTES;
        const float *gb = gbuf + buf * 2 * C;

        // ---- P1: this chunk's [K;Q], V, g, beta have landed; fetch the next
        // chunk's [K;Q] and gates and this chunk's z.
        cp_async_wait<0>();
        __syncthreads();
        if (n0 < t1) {
            fetch_kq(n0, Ln, buf ^ 1);
            fetch_gb(n0, Ln, buf ^ 1);
        }
        cp_async_commit();
        fetch_z(c0, L);
        cp_async_commit();

        // Norms: one row of [K;Q] per thread (zero rows past L give zero).
        if (tid < 128) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jc = 0; jc < 16; ++jc) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(kqp + kq_off(tid, 8 * jc));
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 f = __bfloat1622float2(h2[u]);
                    acc[u] = fmaf(f.x, f.x, fmaf(f.y, f.y, acc[u]));
                }
            }
            const float ss = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            const int r = tid & 63;
            const float f = p.qk_l2norm ? rsqrtf(ss + p.eps_l2) : 1.0f;
            if (tid < 64) sc.nk[r] = r < L ? f : 0.f;
            else sc.nq[r] = r < L ? f * p.scale : 0.f;
        } else if (warp == 4) {
            float g0 = gb[lane], g1 = gb[lane + 32], b0 = gb[C + lane], b1 = gb[C + lane + 32];
            if (p.A_log) {  // raw projections; rows past the chunk stay zero
                const float al = __ldg(p.A_log + hv), db = __ldg(p.dt_bias + hv);
                g0 = lane < L ? gate_g(g0, al, db) : 0.f;
                g1 = lane + 32 < L ? gate_g(g1, al, db) : 0.f;
                b0 = lane < L ? gate_beta(b0) : 0.f;
                b1 = lane + 32 < L ? gate_beta(b1) : 0.f;
            }
            float ga = fmaxf(g0, kGammaFloor), gbv = fmaxf(g1, kGammaFloor);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float xa = __shfl_up_sync(kFullMask, ga, o);
                const float xb = __shfl_up_sync(kFullMask, gbv, o);
                if (lane >= o) { ga += xa; gbv += xb; }
            }
            gbv += __shfl_sync(kFullMask, ga, 31);
            sc.gam[lane] = ga;
            sc.gam[lane + 32] = gbv;
            sc.bet[lane] = b0;
            sc.bet[lane + 32] = b1;
            sc.eg[lane] = __expf(ga);
            sc.eg[lane + 32] = __expf(gbv);
        }
        __syncthreads();
        if (tid < C) sc.dec[tid] = __expf(sc.gam[L - 1] - sc.gam[tid]);

        // ---- P2: [KK; QK] = [K;Q] K^T and S Q^T (state entering the chunk).
        alive = issue_and_wait([&] {
            gemm(tm + TM_D1, kq, 128, 2048, 256, kq, 128, 2048, 256, D / 16, ID_KK, false);
            gemm(tm + TM_OI, sbase + OFF_S, 2048, 128, 4096, kq + 16384, 128, 2048, 256, D / 16,
                 ID_KK, false);
        });
        if (!alive) break;

        // ---- P3: A (fp32 scratch) and P (hi/lo bf16, K-major [r][s]).
        {
            const int rr = 32 * (quad & 1) + lane;  // token row
            const int s0 = 16 * part;
            const float gr = sc.gam[rr];
            float v[16];
            tmem_ld16(tm + lane_off + TM_D1 + s0, v);
            if (quad < 2) {
                const float f = sc.bet[rr] * sc.nk[rr];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int s = s0 + c;
                    Ascr[rr * LDA + s] = s < rr ? f * __expf(gr - sc.gam[s]) * sc.nk[s] * v[c] : 0.f;
                }
            } else {
                const float f = sc.nq[rr];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int s = s0 + c;
                    v[c] = s <= rr ? f * __expf(gr - sc.gam[s]) * sc.nk[s] * v[c] : 0.f;
                }
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint4 hi, lo;
                    split8(v + 8 * c8, hi, lo);
                    *reinterpret_cast<uint4 *>(sm + OFF_P + kmaj(rr, s0 + 8 * c8, C)) = hi;
                    *reinterpret_cast<uint4 *>(sm + OFF_P + 8192 + kmaj(rr, s0 + 8 * c8, C)) = lo;
                }
            }
        }
        __syncthreads();

        // ---- P4: T = (I + A)^{-1} (blocked fp32 inverse).
        invert_unit_lower<NT>(Ascr, Tscr, Xscr, tid);
        // TB = T diag(beta), TW = T diag(beta e^gamma n): hi/lo bf16 tiles [r][s].
        for (int e = tid; e < C * (C / 8); e += NT) {
            const int r = e & 63, s8 = 8 * (e >> 6);
            float tb[8], tw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s8 + u;
                const float t = Tscr[r * LDA + s];
                tb[u] = t * sc.bet[s];
                tw[u] = t * sc.bet[s] * sc.eg[s] * sc.nk[s];
            }
            uint4 hi, lo;
            split8(tb, hi, lo);
            *reinterpret_cast<uint4 *>(sm + OFF_TBW + kmaj(r, s8, C)) = hi;
            *reinterpret_cast<uint4 *>(sm + OFF_TBW + 8192 + kmaj(r, s8, C)) = lo;
            split8(tw, hi, lo);
            *reinterpret_cast<uint4 *>(sm + OFF_TBW + 16384 + kmaj(r, s8, C)) = hi;
            *reinterpret_cast<uint4 *>(sm + OFF_TBW + 24576 + kmaj(r, s8, C)) = lo;
        }

        // ---- P5: U^T = V^T TB^T, W^T = K^T TW^T (hi and lo halves).
        alive = issue_and_wait([&] {
            const uint32_t tbw = sbase + OFF_TBW;
            gemm(tm + TM_U, sbase + OFF_V, 128, 1024, 256, tbw, 1024, 128, 2048, C / 16, ID_U, false);
            gemm(tm + TM_U, sbase + OFF_V, 128, 1024, 256, tbw + 8192, 1024, 128, 2048, C / 16, ID_U,
                 true);
            gemm(tm + TM_W, kq, 2048, 128, 4096, tbw + 16384, 1024, 128, 2048, C / 16, ID_U, false);
            gemm(tm + TM_W, kq, 2048, 128, 4096, tbw + 24576, 1024, 128, 2048, C / 16, ID_U, true);
        });
        if (!alive) break;
        // V of this chunk is consumed: fetch the next chunk's.
        if (n0 < t1) fetch_v(n0, Ln);
        cp_async_commit();

        // ---- P6: W^T -> bf16 B tile; rescale the TMEM state by e^{gamma_L}.
        {
            const int j = 32 * quad + lane;
            const int r0 = 16 * part;
            float wv[16];
            tmem_ld16(tm + lane_off + TM_W + r0, wv);
#pragma unroll
            for (int r8 = 0; r8 < 2; ++r8)
                *reinterpret_cast<uint4 *>(sm + OFF_SCR + w_off(j, r0 + 8 * r8)) = pack8(wv + 8 * r8);
            float v[32];
            const float eL = sc.eg[L - 1];
#pragma unroll
            for (int cc = 0; cc < 1; ++cc) {
                const int j0 = 32 * part;
                tmem_ld32(tm + lane_off + TM_S + j0, v);
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] *= eL;
                tmem_st32(tm + lane_off + TM_S + j0, v);
            }
        }

        // ---- P7: Delta^T = U^T - S W^T (accumulates into the U^T columns).
        alive = issue_and_wait([&] {
            gemm(tm + TM_U, sbase + OFF_S, 2048, 128, 4096, sbase + OFF_SCR, 128, 2048, 256, D / 16,
                 ID_D, true);
        });
        if (!alive) break;

        // ---- P8: Delta^T hi/lo and its decayed, k-normalised copy, K-major [i][s].
        {
            const int i = 32 * quad + lane;
            const int s0 = 16 * part;
            float v[16], w[16];
            tmem_ld16(tm + lane_off + TM_U + s0, v);
#pragma unroll
            for (int c = 0; c < 16; ++c) w[c] = v[c] * sc.dec[s0 + c] * sc.nk[s0 + c];
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8) {
                uint4 hi, lo;
                const uint32_t o = kmaj(i, s0 + 8 * c8, D);
                split8(v + 8 * c8, hi, lo);
                *reinterpret_cast<uint4 *>(sm + OFF_TBW + o) = hi;
                *reinterpret_cast<uint4 *>(sm + OFF_TBW + 16384 + o) = lo;
                split8(w + 8 * c8, hi, lo);
                *reinterpret_cast<uint4 *>(sm + OFF_SCR + o) = hi;
                *reinterpret_cast<uint4 *>(sm + OFF_SCR + 16384 + o) = lo;
            }
        }

        // ---- P9: O_intra^T = Delta^T P^T (hi*hi + hi*lo + lo*hi); S += Dt~ K.
        alive = issue_and_wait([&] {
            const uint32_t dh = sbase + OFF_TBW, dl = dh + 16384;
            const uint32_t ph = sbase + OFF_P, pl = ph + 8192;
            gemm(tm + TM_O2, dh, 2048, 128, 4096, ph, 1024, 128, 2048, C / 16, ID_KK, false);
            gemm(tm + TM_O2, dh, 2048, 128, 4096, pl, 1024, 128, 2048, C / 16, ID_KK, true);
            gemm(tm + TM_O2, dl, 2048, 128, 4096, ph, 1024, 128, 2048, C / 16, ID_KK, true);
            const uint32_t eh = sbase + OFF_SCR, el = eh + 16384;
            gemm(tm + TM_S, eh, 2048, 128, 4096, kq, 2048, 128, 4096, C / 16, ID_S, true);
            gemm(tm + TM_S, el, 2048, 128, 4096, kq, 2048, 128, 4096, C / 16, ID_S, true);
        });
        if (!alive) break;

        // ---- P10: O = m e^gamma (S Q^T) + Delta P^T staged as [r][i]; the new
        // state's bf16 copy for the next chunk.
        {
            const int i = 32 * quad + lane;
            const int r0 = 16 * part;
            float a[16], b[16];
            tmem_ld16(tm + lane_off + TM_OI + r0, a);
            tmem_ld16(tm + lane_off + TM_O2 + r0, b);
            float *Os = reinterpret_cast<float *>(sm + OFF_TBW);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int r = r0 + c;
                Os[r * D + i] = fmaf(sc.nq[r] * sc.eg[r], a[c], b[c]);
            }
#pragma unroll
            for (int cc = 0; cc < 1; ++cc) {
                const int j0 = 32 * part;
                float v[32];
                tmem_ld32(tm + lane_off + TM_S + j0, v);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8)
                    *reinterpret_cast<uint4 *>(sm + OFF_S + kmaj(i, j0 + 8 * j8, D)) = pack8(v + 8 * j8);
            }
        }
        cp_async_wait<1>();  // z of this chunk (the next chunk's V may still be in flight)
        __syncthreads();
        // RMSNormGated per token (one warp per token, C / NW tokens per warp,
        // unrolled so the tokens' reductions overlap), store.
        {
            const float *Os = reinterpret_cast<const float *>(sm + OFF_TBW);
#pragma unroll
            for (int u = 0; u < C / NW; ++u) {
                const int r = warp + NW * u;
                const float4 o4 = *reinterpret_cast<const float4 *>(Os + r * D + 4 * lane);
                float4 y = o4;
                if (zg) {
                    const float ss = group_sum<32>(dot4(o4, o4));
                    const float rstd = rsqrtf(ss * (1.0f / D) + p.eps_norm);
                    const uint2 zr = *reinterpret_cast<const uint2 *>(sm + OFF_Z + r * 256 + 8 * lane);
                    const float2 za = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zr.x));
                    const float2 zb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zr.y));
                    y.x = o4.x * rstd * w4.x * fast_silu(za.x);
                    y.y = o4.y * rstd * w4.y * fast_silu(za.y);
                    y.z = o4.z * rstd * w4.z * fast_silu(zb.x);
                    y.w = o4.w * rstd * w4.w * fast_silu(zb.y);
                }
                if (r < L) Elem<TOUT>::store4(og + (c0 + r) * p.out_stride + hv * D + 4 * lane, y);
            }
        }
    }
    cp_async_wait<0>();  // nothing may land in shared memory after the CTA ends

    // Final state from TMEM.
    if (alive && p.final_state) {
        const int i = 32 * quad + lane;
        float *dst = p.final_state + ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D;
#pragma unroll
        for (int cc = 0; cc < 1; ++cc) {
            const int j0 = 32 * part;
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

size_t prefill_tc_workspace_bytes(int n_seq) { return prefill_tc_ws_bytes(n_seq); }

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
