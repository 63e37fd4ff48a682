// gdr_prefill_2p.cu -- the tensor-core chunked prefill (bf16, d = 128, chunk 64)
// as two kernels, for calls whose workspace has room for per-chunk results.
//
// Most of a chunk's work does not depend on the state entering it: the gates,
// the q/k norms, A and P, the inverse T = (I + A)^{-1}, T diag(beta) (U is
// T diag(beta) V) and W = T diag(beta e^gamma n) K (the chunkwise WY / UT form
// of the gated delta rule named in the Qwen3.5 Chat guide, section
// "Architektur").  So:
//
//   prep kernel:  one CTA per (chunk, value head), every chunk at once, over
//                 the whole GPU (three CTAs per SM; K and Q by tensor copies).
//                 Writes, per unit, a 49 KB record to the workspace: W (bf16,
//                 already in the MMA operand layout), P and T diag(beta) (hi +
//                 lo bf16) and the per-token scalars.
//   recur kernel: one CTA per (sequence, value head), chunks in order, only
//                 the state-dependent part:
//                   U^T     = V^T (T diag(beta))^T      (off the chain)
//                   Delta^T = U^T - S W^T
//                   O^T     = diag-scaled S Q^T + Delta^T P^T
//                   S       = e^{gamma_L} S + (Delta^T diag(e^{gamma_L-gamma} n)) K
//                   y       = RMSNormGated(O)
//
// Operand precisions (bf16 MMAs, hi + lo pairs for T, P, Delta) are those of
// the one-kernel version in gdr_prefill_tc.cu; the output gate here takes its
// sigmoid from tanh.approx (tanh_approx below) where that version divides.
#include "gdr_prefill_common.cuh"
#include "gdr_tmap.cuh"

namespace gdr {
namespace tcp2 {

using namespace gdr::tcp;


// Per-(chunk, value head) record in the workspace, staged in shared memory by
// the recurrence by bulk copies.
constexpr uint32_t REC_W = 0;        // bf16 W, MN-major B tile (w_off), 16 KB
constexpr uint32_t REC_P = 16384;    // P hi, then lo, K-major [r][s] (kmaj R=64), 8 KB each
constexpr uint32_t REC_SCAL = 32768; // fp32 eg[64] | nqe[64] | dn[64] | eL | pad
constexpr uint32_t REC_TB = 33792;   // T diag(beta) hi, then lo, K-major [s][r] (kmaj R=64), 8 KB each
constexpr uint32_t REC_BYTES = 50176;

// The prefill may run as up to MAX_SEG segments of chunk indices [lo_k, lo_k+1)
// of every sequence, so that the prep of segment k+1 overlaps the recurrence
// of segment k on the SMs the recurrence leaves idle.
constexpr int MAX_SEG = 3;
struct SegPlan {
    int n;                  // segments (1 = one prep and one recurrence pass)
    int lo[MAX_SEG + 1];    // chunk-index boundaries, lo[n] >= every sequence's chunk count
};

// Workspace: status word, longest-first order, chunk offsets, per-segment unit
// offsets, the state carried between segments, then records.
struct WsLayout {
    size_t order, chunk_off, seg_off, carry, rec, total;
};
__host__ __device__ inline WsLayout ws_layout(int n_seq, int64_t n_chunks, int H_v, int n_seg = 1) {
    WsLayout w;
    w.order = 16;
    w.chunk_off = (w.order + 4 * (size_t)n_seq + 15) & ~(size_t)15;
    w.seg_off = (w.chunk_off + 4 * ((size_t)n_seq + 1) + 15) & ~(size_t)15;
    w.carry = (w.seg_off + 4 * (size_t)n_seg * ((size_t)n_seq + 1) + 255) & ~(size_t)255;
    const size_t carry_bytes = n_seg > 1 ? (size_t)n_seq * H_v * D * D * 4 : 0;
    w.rec = (w.carry + carry_bytes + 255) & ~(size_t)255;
    w.total = w.rec + (size_t)n_chunks * H_v * REC_BYTES;
    return w;
}

// ------------------------------------------------------------- pre-kernel
// Longest-first order (as the one-kernel path), the status word, and the
// running count of chunks before each sequence.  One block of 1024 threads.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *cu, int n_seq, int *status,
                                                    int *order, int *chunk_off, SegPlan sp,
                                                    int *seg_off) {
    __shared__ int part[1024];
    const int tid = threadIdx.x;
    // The first prep grid may be scheduled now; it waits for this grid before
    // it reads what this grid writes.
    release_dependents();
    if (tid == 0) *status = 0;
    for (int s = tid; s < n_seq; s += 1024) {
        const int ls = cu[s + 1] - cu[s];
        int rank = 0;
        for (int t = 0; t < n_seq; ++t) {
            const int lt = cu[t + 1] - cu[t];
            rank += (lt > ls) || (lt == ls && t < s);
        }
        order[rank] = s;
    }
    // Exclusive scan of ceil(len / C) over sequences: each thread a contiguous range.
    const int per = (n_seq + 1023) / 1024;
    const int lo = tid * per, hi = min(n_seq, lo + per);
    int sum = 0;
    for (int s = lo; s < hi; ++s) sum += (cu[s + 1] - cu[s] + C - 1) / C;
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int add = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += add;
        __syncthreads();
    }
    int run = tid ? part[tid - 1] : 0;
    for (int s = lo; s < hi; ++s) {
        chunk_off[s] = run;
        run += (cu[s + 1] - cu[s] + C - 1) / C;
    }
    if (tid == 1023) chunk_off[n_seq] = part[1023];
    // Per segment k, the exclusive scan of each sequence's chunk count inside
    // [lo_k, lo_k+1): the prep grid of segment k is laid out by it.
    for (int k = 0; k < sp.n; ++k) {
        auto n_in = [&](int s) {
            const int n = (cu[s + 1] - cu[s] + C - 1) / C;
            return max(0, min(n, sp.lo[k + 1]) - sp.lo[k]);
        };
        __syncthreads();
        sum = 0;
        for (int s = lo; s < hi; ++s) sum += n_in(s);
        part[tid] = sum;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {
            const int add = tid >= o ? part[tid - o] : 0;
            __syncthreads();
            part[tid] += add;
            __syncthreads();
        }
        int *off = seg_off + (size_t)k * (n_seq + 1);
        run = tid ? part[tid - 1] : 0;
        for (int s = lo; s < hi; ++s) {
            off[s] = run;
            run += n_in(s);
        }
        if (tid == 1023) off[n_seq] = part[1023];
    }
}

// ------------------------------------------------------------ prep kernel

// 256 threads, ~73 KB of shared memory and 128 TMEM columns, so three prep
// CTAs share an SM and hide each other's latencies. TW is staged over A once
// T is built (TB goes straight into the record).
constexpr int PNT = 256;
constexpr int PSL = 512 / PNT;      // 16-column slices of a 64-column accumulator per thread
constexpr uint32_t A_KQ = 0;        // bf16 [K;Q] tiles (32 KB, kq_sw)
constexpr int PLD = 68;             // row stride of the fp32 scratch (16-byte aligned rows)
constexpr uint32_t A_T = 32768;     // fp32 T [64][PLD]
constexpr uint32_t A_AX = 50176;    // fp32 A [64][PLD] and X; once T is built, TW (16 KB) over A
constexpr uint32_t A_TBW = A_AX;
constexpr uint32_t A_GB = 70656;    // g[64], beta[64]
constexpr uint32_t A_SCAL = 71168;  // scalars, mbarriers
constexpr uint32_t A_SMEM = A_SCAL + 3072;
constexpr uint32_t A_SMEM_LAUNCH = A_SMEM + 1024;  // with the alignment slack
static_assert(3 * (A_SMEM_LAUNCH + 1024) <= 228 * 1024, "three prep blocks must share an SM");

constexpr int DTL = C + 4;  // row stride of dtab
struct PrepScalars {
    float gam[C], eg[C], bet[C], nk[C], nq[C], dec[C];
    float tw[C];  // beta e^gamma n_k: the column factor of TW
    // dtab[R][s] = e^{gamma_{16R} - gamma_s} for s < 16R: with the per-row
    // e^{gamma_r - gamma_{16R}} it gives e^{gamma_r - gamma_s} below the
    // diagonal 16-block as a product of two factors that are at most one.
    float dtab[4 * DTL];  // rows DTL apart: a warp's two rows sit in different banks
    uint64_t bar;
    uint64_t tbar;  // the K and Q tiles landed
    uint32_t tmem;
};
static_assert(sizeof(PrepScalars) <= A_SMEM - A_SCAL, "prep scalars overflow");
static_assert(A_T + C * PLD * 4 <= A_AX && A_AX + C * PLD * 4 + 3 * 1024 <= A_GB &&
                  16384 <= C * PLD * 4,
              "prep scratch overlap");

// Tensor maps of the packed q, k and v (rows = tokens; boxes of 64 elements x
// 64 tokens, 128-byte swizzle) for the prep kernel's tensor copies.
struct PrepMaps {
    CUtensorMap k, q, v;
};
// The [K;Q] tile as the tensor copies leave it: per half of d (64 values),
// 64 rows of K then 64 of Q, 128 bytes a row, 16-byte chunks swizzled by the
// row's index mod 8.
__device__ __forceinline__ uint32_t kq_sw(int row, int jc) {
    return (uint32_t)((jc >> 3) * 16384 + row * 128 + (((jc & 7) ^ (row & 7)) << 4));
}

// The block's unit within a segment: the sequence (the last s with
// seg_off[s] <= unit) and its chunk index (from the segment's first chunk).
struct PrepUnit {
    int seq, chunk;
};
__device__ __forceinline__ PrepUnit prep_unit(const int *seg_off, int seg_lo, int n_seq, int unit) {
    int lo = 0, hi = n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg_off[mid] <= unit) lo = mid; else hi = mid - 1;
    }
    return {lo, seg_lo + unit - seg_off[lo]};
}

// One block per (chunk of the segment, value head).  seg_off: the segment's
// unit offsets per sequence, seg_lo its first chunk index.
// wait_prev_at_exit: launched as a programmatic dependent of the previous
// segment's recurrence; the block of the highest index waits for it before
// exiting, so that this grid completes only after it (the next recurrence
// segment, queued after this grid, reads the state it carries).
// wait_prev_at_start: launched as a programmatic dependent of the plan
// kernel (the first segment); every block waits for it before reading the
// order and offsets it writes.
// K, Q and V come by tensor copies (maps) into 128-byte-swizzled tiles.
__global__ void __launch_bounds__(PNT, 3) prep_kernel(const PrefillParams p,
                                                     const __grid_constant__ PrepMaps maps,
                                                     const int *chunk_off,
                                                     const int *seg_off, int seg_lo,
                                                     unsigned char *records, int *status,
                                                     int wait_prev_at_exit, int wait_prev_at_start) {
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    // The swizzled tiles must start on a 1024-byte boundary (A_SMEM_LAUNCH
    // leaves room to round up).
    unsigned char *sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
    PrepScalars &sc = *reinterpret_cast<PrepScalars *>(sm + A_SCAL);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quad = warp & 3, part = warp >> 2;
    const int hv = blockIdx.x % p.H_v;
    const int hk = hv / p.hv_per_hk;
    if (wait_prev_at_start) wait_for_predecessor();
    const PrepUnit pu = prep_unit(seg_off, seg_lo, p.n_seq, blockIdx.x / p.H_v);
    const int seq = pu.seq;
    const int gchunk = chunk_off[seq] + pu.chunk;
    const int64_t t0 = p.cu_seqlens[seq], t1 = p.cu_seqlens[seq + 1];
    const int64_t c0 = t0 + (int64_t)pu.chunk * C;
    const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
    unsigned char *rec = records + ((size_t)gchunk * p.H_v + hv) * REC_BYTES;

    const uint32_t sbase = smem_u32(sm);
    float *Ascr = reinterpret_cast<float *>(sm + A_AX);
    float *Xscr = Ascr + C * PLD;
    float *Tscr = reinterpret_cast<float *>(sm + A_T);
    float *gbuf = reinterpret_cast<float *>(sm + A_GB);

    // Thread 0 starts the tile copies first; warp 7 (idle until the first
    // product) takes the TMEM columns.  (Warming L2 for the unit that next
    // takes this block's slot measured slower: the copy engine is shared.)
    if (warp == 7) tmem_alloc(&sc.tmem, 128);
    if (tid == 0) {
        mbar_init(&sc.bar, 1);
        mbar_init(&sc.tbar, 1);
        mbar_fence_init();
        // Four boxes of 64 tokens x 64 values: K and Q, each d half. Tokens
        // past the sequence belong to the next one (zeroed below) or lie past
        // the tensor (read as zero).
        bulk_expect(&sc.tbar, 4 * 8192);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tma_load_2d(sbase + A_KQ + h * 16384, &maps.k, hk * D + 64 * h, (int)c0, &sc.tbar);
            tma_load_2d(sbase + A_KQ + h * 16384 + 8192, &maps.q, hk * D + 64 * h, (int)c0, &sc.tbar);
        }
    }
    if (tid < 2 * C) {
        const int r = tid & 63;
        const bool in = r < L;
        const int64_t t = in ? c0 + r : c0;
        cp_async4(gbuf + tid, (tid < C ? p.g : p.beta) + t * p.gb_stride + hv, in ? 4u : 0u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    // g and beta landed, the barriers' initialisation seen by every thread.
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const bool loads_ok = mbar_wait(&sc.tbar, 0u, kWaitNs);
    // Rows past a ragged chunk's end are zero (the products scale them by zero
    // factors too, but the next sequence's values must not reach them).
    // nboxes boxes of 8 KB from `at0`, `stride` apart: rows L..63 to zero.
    auto zero_tail = [&](uint32_t at0, uint32_t stride, int nboxes) {
        const int nz = (C - L) * 8;
        for (int e = tid; e < nboxes * nz; e += PNT) {
            const int box = e / nz, r = L + ((e - box * nz) >> 3), ch = e & 7;
            *reinterpret_cast<uint4 *>(sm + at0 + box * stride + r * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
    };
    if (loads_ok && L < C) zero_tail(A_KQ, 8192, 4);
    fence_before_sync();
    const bool loads_bad = __syncthreads_or(!loads_ok) != 0;
    fence_after_sync();
    if (loads_bad && tid == 0) atomicExch(status, kTimeoutStatus);
    const uint32_t tm = sc.tmem;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    // [KK;QK] in columns 0..63, W^T beside it.
    constexpr uint32_t TM_D1 = 0, TM_W = 64;

    // Norms (one row of [K;Q] per thread) and the running sums of g.
    if (tid < 128) {
        // Sums of squares in pairs (two-wide FMA), four pair accumulators.
        float2 acc[4] = {};
#pragma unroll
        for (int jc = 0; jc < 16; ++jc) {
            const uint4 raw =
                *reinterpret_cast<const uint4 *>(sm + A_KQ + kq_sw(tid, jc));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(h2[u]);
                acc[u] = __ffma2_rn(f, f, acc[u]);
            }
        }
        const float ss = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                         ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        const int r = tid & 63;
        const float f = p.qk_l2norm ? rsqrtf(ss + p.eps_l2) : 1.0f;
        if (tid < 64) sc.nk[r] = r < L ? f : 0.f;
        else sc.nq[r] = r < L ? f * p.scale : 0.f;
    } else if (warp == 4) {
        float g0 = gbuf[lane], g1 = gbuf[lane + 32], b0 = gbuf[C + lane], b1 = gbuf[C + lane + 32];
        if (p.A_log) {  // raw projections; rows past the chunk stay zero
            const float al = __ldg(p.A_log + hv), db = __ldg(p.dt_bias + hv);
            g0 = lane < L ? gate_g(g0, al, db) : 0.f;
            g1 = lane + 32 < L ? gate_g(g1, al, db) : 0.f;
            b0 = lane < L ? gate_beta(b0) : 0.f;
            b1 = lane + 32 < L ? gate_beta(b1) : 0.f;
        }
        float ga = fmaxf(g0, kGammaFloor), gb = fmaxf(g1, kGammaFloor);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float xa = __shfl_up_sync(kFullMask, ga, o);
            const float xb = __shfl_up_sync(kFullMask, gb, o);
            if (lane >= o) { ga += xa; gb += xb; }
        }
        gb += __shfl_sync(kFullMask, ga, 31);
        sc.gam[lane] = ga;
        sc.gam[lane + 32] = gb;
        sc.bet[lane] = b0;
        sc.bet[lane + 32] = b1;
        sc.eg[lane] = __expf(ga);
        sc.eg[lane + 32] = __expf(gb);
    }
    __syncthreads();
    if (tid < C) {
        sc.dec[tid] = __expf(sc.gam[L - 1] - sc.gam[tid]);
        sc.tw[tid] = sc.bet[tid] * sc.eg[tid] * sc.nk[tid];
    }
    {
        const int R = tid >> 6, s = tid & 63;  // PNT == 4 * C entries
        sc.dtab[R * DTL + s] = s < 16 * R ? __expf(sc.gam[16 * R] - sc.gam[s]) : 0.f;
    }

    uint32_t phase = 0;
    // `ready`: this thread's operands are in place (all must be, or nothing
    // is issued).
    auto issue_and_wait = [&](bool ready, auto issue) -> bool {
        fence_smem_to_async();
        fence_before_sync();
        if (__syncthreads_or(!ready)) {
            if (tid == 0) atomicExch(status, kTimeoutStatus);
            return false;
        }
        if (tid == 0) {
            fence_after_sync();
            issue();
            commit(smem_u32(&sc.bar));
        }
        const bool ok = mbar_wait(&sc.bar, phase, kWaitNs);
        phase ^= 1;
        const int bad = __syncthreads_or(!ok);
        fence_after_sync();
        if (bad && tid == 0) atomicExch(status, kTimeoutStatus);
        return !bad;
    };
    const uint32_t ID_KK = instr_desc<Kind::BF16>(128, 64, false, false);
    const uint32_t ID_U = instr_desc<Kind::BF16>(128, 64, true, false);
    const uint32_t kq = sbase + A_KQ;

    bool alive = !loads_bad && issue_and_wait(true, [&] {
        // K-major, 128-byte swizzle: a K step is 32 bytes inside a row, the
        // second half of d 16 KB on.
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t dk = smem_desc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            mma<Kind::BF16>(tm + TM_D1, dk, dk, ID_KK, kk > 0 ? 1u : 0u);
        }
    });
    if (alive) {
        // A (fp32 scratch) and P (hi/lo bf16 straight into the record).  The
        // decay e^{gamma_r - gamma_s}: zero above the diagonal 16-block, a
        // row factor times a table entry below it, exact on it.
        const int rr = 32 * (quad & 1) + lane, R = rr >> 4;
        const float gr = sc.gam[rr];
        // v[c] <- f e[c] n_k[s0+c] v[c] on or below the diagonal (strictly
        // below for A), else 0; pairs by two-wide multiplies, n_k by 16 bytes.
        auto scale_row = [&](float (&v)[16], const float (&e)[16], float f, int s0, int rr,
                             bool diag) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 nk = *reinterpret_cast<const float4 *>(sc.nk + s0 + 4 * c4);
                const float2 ff = make_float2(f, f);
                const float2 a = __fmul2_rn(__fmul2_rn(ff, make_float2(e[4 * c4], e[4 * c4 + 1])),
                                            __fmul2_rn(make_float2(nk.x, nk.y),
                                                       make_float2(v[4 * c4], v[4 * c4 + 1])));
                const float2 b = __fmul2_rn(__fmul2_rn(ff, make_float2(e[4 * c4 + 2], e[4 * c4 + 3])),
                                            __fmul2_rn(make_float2(nk.z, nk.w),
                                                       make_float2(v[4 * c4 + 2], v[4 * c4 + 3])));
                const float r4[4] = {a.x, a.y, b.x, b.y};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int s = s0 + 4 * c4 + u;
                    v[4 * c4 + u] = (diag ? s <= rr : s < rr) ? r4[u] : 0.f;
                }
            }
        };
        const float rowf = R > 0 ? __expf(gr - sc.gam[16 * R]) : 1.f;
#pragma unroll
        for (int sl = 0; sl < PSL; ++sl) {
        const int s0 = 16 * (part * PSL + sl), Sb = s0 >> 4;
        float v[16], e[16];
        tmem_ld16(tm + lane_off + TM_D1 + s0, v);
        if (Sb < R) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 t = *reinterpret_cast<const float4 *>(sc.dtab + R * DTL + s0 + 4 * c4);
                const float2 a = __fmul2_rn(make_float2(rowf, rowf), make_float2(t.x, t.y));
                const float2 b = __fmul2_rn(make_float2(rowf, rowf), make_float2(t.z, t.w));
                e[4 * c4] = a.x; e[4 * c4 + 1] = a.y; e[4 * c4 + 2] = b.x; e[4 * c4 + 3] = b.y;
            }
        } else if (Sb == R) {
#pragma unroll
            for (int c = 0; c < 16; ++c) e[c] = __expf(gr - sc.gam[s0 + c]);
        } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) e[c] = 0.f;
        }
        if (quad < 2) {
            // 16-byte stores: with rows PLD floats apart, a quarter-warp's eight
            // rows cover all 32 banks once.
            const float f = sc.bet[rr] * sc.nk[rr];
            scale_row(v, e, f, s0, rr, false);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                *reinterpret_cast<float4 *>(Ascr + rr * PLD + s0 + 4 * c4) =
                    make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
        } else {
            scale_row(v, e, sc.nq[rr], s0, rr, true);
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8) {
                uint4 h, l;
                split8(v + 8 * c8, h, l);
                *reinterpret_cast<uint4 *>(rec + REC_P + kmaj(rr, s0 + 8 * c8, C)) = h;
                *reinterpret_cast<uint4 *>(rec + REC_P + 8192 + kmaj(rr, s0 + 8 * c8, C)) = l;
            }
        }
        }
        __syncthreads();
        invert_unit_lower<PNT, PLD>(Ascr, Tscr, Xscr, tid);
        // T diag(f) as bf16 hi/lo tiles at dst: TB (f = beta) into the record,
        // the B operand of the recurrence's U product; TW (f = beta e^gamma
        // n_k) over A, the B operand of W's.
        auto stage_t = [&](bool w_side, unsigned char *dst) {
            for (int e = tid; e < C * (C / 8); e += PNT) {
                const int r = e & 63, s8 = 8 * (e >> 6);
                float t[8];
                *reinterpret_cast<float4 *>(t) = *reinterpret_cast<const float4 *>(Tscr + r * PLD + s8);
                *reinterpret_cast<float4 *>(t + 4) =
                    *reinterpret_cast<const float4 *>(Tscr + r * PLD + s8 + 4);
                const float *fs = (w_side ? sc.tw : sc.bet) + s8;
#pragma unroll
                for (int u4 = 0; u4 < 2; ++u4) {
                    const float4 f = *reinterpret_cast<const float4 *>(fs + 4 * u4);
                    const float2 a = __fmul2_rn(make_float2(t[4 * u4], t[4 * u4 + 1]), make_float2(f.x, f.y));
                    const float2 b = __fmul2_rn(make_float2(t[4 * u4 + 2], t[4 * u4 + 3]), make_float2(f.z, f.w));
                    t[4 * u4] = a.x; t[4 * u4 + 1] = a.y; t[4 * u4 + 2] = b.x; t[4 * u4 + 3] = b.y;
                }
                uint4 h, l;
                split8(t, h, l);
                *reinterpret_cast<uint4 *>(dst + kmaj(r, s8, C)) = h;
                *reinterpret_cast<uint4 *>(dst + 8192 + kmaj(r, s8, C)) = l;
            }
        };
        stage_t(false, rec + REC_TB);
        stage_t(true, sm + A_TBW);
        // W^T = K^T TW^T: K as MN-major A (d across the two 64-value atoms 16 KB
        // apart, the tokens as K, 16 of them = 2 KB a step); B = TW hi, lo.
        alive = issue_and_wait(true, [&] {
            const uint32_t tbw = sbase + A_TBW;
            for (int kk = 0; kk < C / 16; ++kk) {
                const uint64_t a = smem_desc_sw128(kq + kk * 2048, 16384, 1024);
                mma<Kind::BF16>(tm + TM_W, a, smem_desc(tbw + kk * 2048, 1024, 128), ID_U,
                                kk > 0 ? 1u : 0u);
                mma<Kind::BF16>(tm + TM_W, a, smem_desc(tbw + 8192 + kk * 2048, 1024, 128), ID_U, 1u);
            }
        });
    }
    if (alive) {
        // W^T [j][r] -> bf16 MN-major B tile; scalars.
        const int x = 32 * quad + lane;  // j
#pragma unroll
        for (int sl = 0; sl < PSL; ++sl) {
        const int c0l = 16 * (part * PSL + sl);
        float w[16];
        tmem_ld16(tm + lane_off + TM_W + c0l, w);
#pragma unroll
        for (int r8 = 0; r8 < 2; ++r8)
            *reinterpret_cast<uint4 *>(rec + REC_W + w_off(x, c0l + 8 * r8)) = pack8(w + 8 * r8);
        }
        float *scal = reinterpret_cast<float *>(rec + REC_SCAL);
        if (tid < C) {
            scal[tid] = sc.eg[tid];
            scal[C + tid] = sc.nq[tid] * sc.eg[tid];
            scal[2 * C + tid] = sc.dec[tid] * sc.nk[tid];
        } else if (tid == C) {
            scal[3 * C] = sc.eg[L - 1];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 7) {
        fence_after_sync();
        tmem_free(tm, 128);
    }
    // A tensor copy that did not land in time must not land after the block ends.
    if (loads_bad && tid == 0) mbar_wait(&sc.tbar, 0u, 1000000ull);
    if (wait_prev_at_exit && blockIdx.x == gridDim.x - 1) wait_for_predecessor();
}

// ----------------------------------------------------------- recur kernel
//
// One CTA per (sequence, value head) walks the chunks in order.  Only the
// state path is serial: Delta = U - W S^T needs the state entering the chunk,
// and the next state needs Delta.  The output of a chunk (O = (m e^gamma) Q S^T
// + P Delta, then RMSNormGated) feeds nothing later, so the CTA is split into
// five roles that run concurrently and hand work over on mbarriers:
//   warps 0-7   state group: the Delta epilogue -- first the decayed,
//               k-normalised copy of Delta^T as hi/lo tiles in TMEM, all the
//               state update waits for, then Delta's hi/lo tiles for P Delta --
//               and, once the update is done, from one read of the state, the
//               bf16 copy of S that the next chunk's first products wait for
//               and the state pre-scaled by the next chunk's e^{gamma_L};
//   warps 8-15  output group, one chunk behind: S Q^T and P Delta out of
//               double-buffered TMEM, staged through shared memory so that
//               one warp normalises, gates and stores whole tokens;
//   warp 16     producer for the state path: K and Q tiles by tensor copies
//               (a sequence's ragged last chunk by 16-byte copies that read
//               zero past its end), V the same way, and by bulk copy each
//               chunk's W and T diag(beta), every one into its stage as soon
//               as the previous chunk is done with it (no L2 prefetch: it
//               shared the copy engine with these loads and measured slower);
//   warp 18     producer for the output side: P and the per-token scalars,
//               whose stages the output group frees;
//   warp 17     MMA issue, state path first (-S W^T before S Q^T, the state
//               update, then the next chunk's U product, before P Delta), each
//               group committed on its own barrier so the state group never
//               waits for output products.

// tanh.approx (relative error below 2^-10.9): with sigma(z) = (1 + tanh(z/2))
// / 2 the gate z sigma(z) costs one special-function op where e^{-z} and a
// reciprocal take two; the output warps run 32 per lane a chunk.
__device__ __forceinline__ float tanh_approx(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
    return t;
}
// The output warps' element-wise fp32 work runs in pairs (sm_100's two-wide
// FMA and multiply; each lane rounds as the scalar op does).
__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }

constexpr int RNT = 608;                       // 19 warps
constexpr int OG_BAR = 1, OG_N = 256;
constexpr uint32_t B_KQ = 0;                   // bf16 [K;Q] (32 KB, as kq_sw lays it out)
constexpr uint32_t B_W = 32768;                // bf16 W of the current chunk (16 KB)
constexpr uint32_t B_P = 49152;                // bf16 P hi/lo of the current chunk (16 KB)
constexpr uint32_t B_SC = 65536;               // 2 x scalars (eg, nqe, dn, eL: 1 KB each)
constexpr uint32_t B_DL = 67584;               // Delta hi/lo (32 KB)
constexpr uint32_t B_V = 133120;               // bf16 V of the current chunk (16 KB, two 128-byte-swizzled boxes)
constexpr uint32_t B_TB = 149504;              // T diag(beta) hi/lo of the current chunk (16 KB, record layout)
constexpr uint32_t B_OS = 165888;              // fp32 O [r][i] of the chunk being output (32 KB)
constexpr uint32_t B_BAR = 198656;             // 18 mbarriers, then the TMEM address
constexpr uint32_t B_SMEM = B_BAR + 160;
constexpr uint32_t B_SMEM_LAUNCH = B_SMEM + 1024;  // with the alignment slack
constexpr uint32_t SC_BYTES = REC_TB - REC_SCAL;
// The stages in order and apart; 18 mbarriers and the TMEM address after them.
static_assert(B_KQ + 32768 <= B_W && B_W + 16384 <= B_P && B_P + 16384 <= B_SC &&
                  B_SC + 2 * SC_BYTES <= B_DL && B_DL + 32768 <= B_V && B_V + 16384 <= B_TB &&
                  B_TB + 16384 <= B_OS && B_OS + C * D * 4 <= B_BAR &&
                  B_BAR + 18 * 8 + 4 <= B_SMEM && B_SMEM_LAUNCH <= 227 * 1024,
              "recurrence shared-memory layout");
static_assert(B_KQ % 1024 == 0 && B_V % 1024 == 0, "128-byte-swizzled tiles start on 1024 bytes");
// TMEM columns: the fp32 state, Delta^T = U^T - S W^T (the U product first,
// then -S W^T onto it), two buffers of S Q^T, one of P Delta, and the bf16 copy
// of S (two values per column) that -S W^T and S Q^T read as their A operand.
constexpr uint32_t TM_S = 0, TM_D = 128, TM_OI = 192, TM_O2 = 320, TM_SB = 384;
// ... and the decayed Delta^T tiles (hi, lo; two values per column), the A
// operand of the state update.
constexpr uint32_t TM_DTH = 448, TM_DTL = 480;
// A recurrence block holds all 512 TMEM columns, so a prep block (which the
// next segment may start beside it) must never fit on the same SM: their
// shared memory together exceeds an SM's (228 KB, 1 KB reserved per block).
static_assert(B_SMEM_LAUNCH + A_SMEM_LAUNCH + 2 * 1024 > 228 * 1024,
              "a prep block could share an SM with a recurrence block");

// Chunks [seg_lo, seg_hi) of every sequence.  The state enters from the
// caller's initial state in the first segment (seg_lo == 0), else from
// `carry`; it leaves to the caller's final state in the segment where the
// sequence ends, else to `carry` (both [n_seq, H_v, d_v, d_k]).
// maps: the tensor maps of k and q (those of prep).
template <typename TOUT>
__global__ void __launch_bounds__(RNT, 1) recur_kernel(const PrefillParams p,
                                                       const __grid_constant__ PrepMaps maps,
                                                       const int *order, const int *chunk_off,
                                                       const unsigned char *records, int *status,
                                                       int seg_lo, int seg_hi, float *carry) {
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    // The swizzled [K;Q] tile must start on a 1024-byte boundary.
    unsigned char *sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
    // The next kernel on the stream (the following segment's prep) may start
    // on the SMs this grid leaves free; it reads nothing this grid writes.
    release_dependents();
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + B_BAR);
    uint64_t *bar_q = bars, *bar_k = bars + 1;   // tiles landed
    uint64_t *bar_w = bars + 2;                  // W landed
    uint64_t *bar_p = bars + 3;                  // P landed
    uint64_t *bar_sc = bars + 4;                 // [2] scalars landed
    uint64_t *bar_u = bars + 6;                  // V and T diag(beta) landed
    uint64_t *bar_gd = bars + 7;                 // -S W^T done (W may be refilled)
    uint64_t *bar_qfree = bars + 8;              // S Q^T done (Q may be refilled)
    uint64_t *bar_gs = bars + 9;                 // state update done (K may be refilled)
    uint64_t *bar_oready = bars + 10;            // [2] P Delta (and S Q^T) of a chunk done
    uint64_t *bar_ofree = bars + 12;             // [2] output group done with a chunk's buffers
    uint64_t *bar_sready = bars + 14;            // state group: bf16 S staged (8 warps)
    uint64_t *bar_dready = bars + 15;            // state group: Delta tiles for P Delta staged (8 warps)
    uint64_t *bar_dtready = bars + 16;           // state group: decayed Delta^T in TMEM (8 warps)
    uint64_t *bar_scaled = bars + 17;            // state group: fp32 S pre-scaled for the update (8 warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + B_BAR + 144);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seq = order[blockIdx.x / p.H_v];
    const int hv = blockIdx.x % p.H_v;
    const int hk = hv / p.hv_per_hk;
    const int64_t t1 = p.cu_seqlens[seq + 1];
    const int total_chunks = (int)((t1 - p.cu_seqlens[seq] + C - 1) / C);
    // A sequence that ended in an earlier segment has nothing left to do (an
    // empty sequence belongs to the first segment, which passes its state on).
    if (seg_lo > 0 && seg_lo >= total_chunks) return;
    const int seg_end = total_chunks < seg_hi ? total_chunks : seg_hi;
    const int n_chunks = seg_end - seg_lo;
    const int64_t t0 = p.cu_seqlens[seq] + (int64_t)seg_lo * C;  // first token of the segment
    const float *state_in = seg_lo == 0 ? p.initial_state : carry;
    float *state_out = seg_end == total_chunks ? p.final_state : carry;
    const unsigned char *rec0 =
        records + ((size_t)(chunk_off[seq] + seg_lo) * p.H_v + hv) * REC_BYTES;
    const size_t rec_step = (size_t)p.H_v * REC_BYTES;
    const uint32_t sbase = smem_u32(sm);
    auto chunk_len = [&](int c) {
        const int64_t left = t1 - t0 - (int64_t)c * C;
        return (int)(left < C ? left : C);
    };
    auto fail = [&]() { atomicExch(status, kTimeoutStatus); };
    // Every wait below gives up after wait_ns (2 s unless a diagnostic call
    // shortens it) and the CTA then unwinds: status word, copies, TMEM.
    const uint64_t wait_ns = p.wait_ns ? p.wait_ns : kWaitNs;
    auto scal = [&](int c) { return reinterpret_cast<const float *>(sm + B_SC + (c & 1) * SC_BYTES); };
    // Bytes [src_off, src_off + bytes) of chunk c's record into shared memory at
    // dst, landing on bar (issued by lane 0 of a producer warp).
    auto bulk = [&](uint32_t dst, uint32_t src_off, uint32_t bytes, uint64_t *bar, int c) {
        if (lane == 0) {
            bulk_expect(bar, bytes);
            bulk_copy(sm + dst, rec0 + (size_t)c * rec_step + src_off, bytes, bar);
        }
    };

    if (warp == 0) tmem_alloc(tmem_slot, 512);
    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_k, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_sc + b, 1);
            mbar_init(bar_oready + b, 1);
            mbar_init(bar_ofree + b, 8);
        }
        mbar_init(bar_w, 1);
        mbar_init(bar_p, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_gd, 1);
        mbar_init(bar_qfree, 1);
        mbar_init(bar_gs, 1);
        mbar_init(bar_sready, 8);
        mbar_init(bar_dready, 8);
        mbar_init(bar_dtready, 8);
        mbar_init(bar_scaled, 8);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tmem_slot;
    bool state_ok = false;

    if (warp == 17) {
        // ------------------------------------------------------ MMA issue
        if (lane == 0 && n_chunks > 0) {
            const uint32_t ID_KK = instr_desc<Kind::BF16>(128, 64, false, false);
            const uint32_t ID_D = instr_desc<Kind::BF16>(128, 64, false, true, true);  // -S, B = W MN-major
            const uint32_t ID_S = instr_desc<Kind::BF16>(128, 128, false, true);       // B = K, MN-major
            const uint32_t kq = sbase + B_KQ;
            // U^T = V^T (T diag(beta))^T into the Delta accumulator: A = V,
            // MN-major (d_v across the two 64-value boxes 8 KB apart, 16 tokens
            // = 2 KB a step); B = T diag(beta) hi, lo.  The -S W^T that follows
            // accumulates onto it (same accumulator and shape: issued in order).
            const uint32_t ID_U = instr_desc<Kind::BF16>(128, 64, true, false);
            auto issue_u = [&]() {
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t av = smem_desc_sw128(sbase + B_V + kk * 2048, 8192, 1024);
                    mma<Kind::BF16>(tm + TM_D, av, smem_desc(sbase + B_TB + kk * 2048, 1024, 128), ID_U,
                                    kk > 0 ? 1u : 0u);
                    mma<Kind::BF16>(tm + TM_D, av, smem_desc(sbase + B_TB + 8192 + kk * 2048, 1024, 128),
                                    ID_U, 1u);
                }
            };
            bool ok = mbar_wait(bar_u, 0u, wait_ns);
            if (ok) {
                fence_after_sync();
                issue_u();
            }
            for (int c = 0; c < n_chunks && ok; ++c) {
                const int b = c & 1;
                const uint32_t ph = (uint32_t)c & 1u;
                ok = mbar_wait(bar_sready, ph, wait_ns) && mbar_wait(bar_w, ph, wait_ns) &&
                     mbar_wait(bar_q, ph, wait_ns) &&
                     (c < 2 || mbar_wait(bar_ofree + b, (uint32_t)((c >> 1) - 1) & 1u, wait_ns));
                if (!ok) break;
                fence_after_sync();
                fence_smem_to_async();
                gemm_ta(tm + TM_D, tm + TM_SB, sbase + B_W, 128, 2048, 256, D / 16, ID_D, true);
                commit(smem_u32(bar_gd));
                // B = Q, K-major with the 128-byte swizzle (kq_sw).
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ta(tm + TM_OI + 64 * b, tm + TM_SB + 8 * kk,
                           smem_desc_sw128(kq + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), ID_KK,
                           kk > 0 ? 1u : 0u);
                commit(smem_u32(bar_qfree));
                // The update needs only the decayed Delta^T tiles (TMEM) and the
                // pre-scaled state; the Delta tiles of P Delta may still be coming.
                ok = mbar_wait(bar_dtready, ph, wait_ns) && mbar_wait(bar_k, ph, wait_ns) &&
                     mbar_wait(bar_scaled, ph, wait_ns);
                if (!ok) break;
                fence_after_sync();
                fence_smem_to_async();
                // S <- e^{gamma_L} S + Dt~^T K (hi + lo, Dt~^T from TMEM); then
                // O_intra^T = Delta^T P^T (hi*hi + hi*lo + lo*hi) into its buffer.
                // B = K, MN-major (d_k across the two 64-value atoms 16 KB
                // apart, 16 tokens = 2 KB a step).
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t bk = smem_desc_sw128(kq + kk * 2048, 16384, 1024);
                    mma_ta(tm + TM_S, tm + TM_DTH + 8 * kk, bk, ID_S, 1u);
                    mma_ta(tm + TM_S, tm + TM_DTL + 8 * kk, bk, ID_S, 1u);
                }
                commit(smem_u32(bar_gs));
                // The next chunk's U product, now that this chunk's Delta has
                // been read out of its accumulator (dtready, waited above).
                if (c + 1 < n_chunks) {
                    ok = mbar_wait(bar_u, (uint32_t)(c + 1) & 1u, wait_ns);
                    if (!ok) break;
                    fence_after_sync();
                    issue_u();
                }
                // P Delta has one accumulator: chunk c-1's output must have left it.
                ok = mbar_wait(bar_p, ph, wait_ns) && mbar_wait(bar_dready, ph, wait_ns) &&
                     (c < 1 || mbar_wait(bar_ofree + ((c - 1) & 1), (uint32_t)((c - 1) >> 1) & 1u, wait_ns));
                if (!ok) break;
                fence_after_sync();
                fence_smem_to_async();
                const uint32_t dh = sbase + B_DL, dl = dh + 16384, pb = sbase + B_P, pl = pb + 8192;
                const uint32_t o2 = tm + TM_O2;
                gemm(o2, dh, 2048, 128, 4096, pb, 1024, 128, 2048, C / 16, ID_KK, false);
                gemm(o2, dh, 2048, 128, 4096, pl, 1024, 128, 2048, C / 16, ID_KK, true);
                gemm(o2, dl, 2048, 128, 4096, pb, 1024, 128, 2048, C / 16, ID_KK, true);
                commit(smem_u32(bar_oready + b));
            }
            if (!ok) fail();
        }
        __syncwarp();
    } else if (warp == 16) {
        // ------------------------------------------------------ producer
        const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q) + hk * D;
        const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(p.k) + hk * D;
        // Copies counted so that an early exit can wait for them.
        int n_w = 0, n_u = 0, n_tile[2] = {0, 0};
        // The K or Q tile of a chunk (kq_sw layout): a full chunk by two tensor
        // copies; a sequence's ragged last chunk by 16-byte copies that read
        // zero past its end (this lane waits for its own, then one arrival).
        auto fetch = [&](int64_t c0, int L, bool q_half) {
            uint64_t *bar = q_half ? bar_q : bar_k;
            const uint32_t dst = B_KQ + (q_half ? 8192u : 0u);
            ++n_tile[q_half ? 1 : 0];
            if (L == C) {
                if (lane == 0) {
                    const CUtensorMap *map = q_half ? &maps.q : &maps.k;
                    bulk_expect(bar, 16384);
                    tma_load_2d(sbase + dst, map, hk * D, (int)c0, bar);
                    tma_load_2d(sbase + dst + 16384, map, hk * D + 64, (int)c0, bar);
                }
                return;
            }
            const __nv_bfloat16 *base = q_half ? qg : kg;
            const int64_t stride = q_half ? p.q_stride : p.k_stride;
#pragma unroll 8
            for (int e = lane; e < 64 * 16; e += 32) {
                const int r = e >> 4, jc = e & 15;
                const bool in = r < L;
                const int64_t t = in ? c0 + r : t0;
                cp_async16(sm + dst + (jc >> 3) * 16384 + r * 128 + (((jc & 7) ^ (r & 7)) << 4),
                           base + t * stride + 8 * jc, in ? 16u : 0u);
            }
            cp_async_wait_all();
            fence_smem_to_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // V of chunk c (two 128-byte-swizzled boxes: tensor copies, or for a
        // ragged last chunk 16-byte copies that read zero past its end, waited
        // for here) and its T diag(beta) tiles from the record, on bar_u.
        auto fetch_vt = [&](int64_t c0, int L, int c) {
            if (L < C) {
                const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(p.v) + hv * D;
#pragma unroll 8
                for (int e = lane; e < 64 * 16; e += 32) {
                    const int r = e >> 4, jc = e & 15;
                    const bool in = r < L;
                    const int64_t t = in ? c0 + r : t0;
                    cp_async16(sm + B_V + (jc >> 3) * 8192 + r * 128 + (((jc & 7) ^ (r & 7)) << 4),
                               vb + t * p.v_stride + 8 * jc, in ? 16u : 0u);
                }
                cp_async_wait_all();
                fence_smem_to_async();
                __syncwarp();
            }
            if (lane == 0) {
                bulk_expect(bar_u, L == C ? 32768u : 16384u);
                if (L == C) {
                    tma_load_2d(sbase + B_V, &maps.v, hv * D, (int)c0, bar_u);
                    tma_load_2d(sbase + B_V + 8192, &maps.v, hv * D + 64, (int)c0, bar_u);
                }
                bulk_copy(sm + B_TB, rec0 + (size_t)c * rec_step + REC_TB, 16384, bar_u);
            }
        };
        bool ok = true;
        for (int c = 0; c < n_chunks && ok; ++c) {
            const int64_t c0 = t0 + (int64_t)c * C;
            const int L = chunk_len(c);
            const uint32_t pp = (uint32_t)(c - 1) & 1u;  // phase of chunk c-1's events
            // V and T diag(beta) of chunk c once chunk c-1's U product (under
            // the same commit as its -S W^T) is done with the stage.
            if (c > 0) ok = mbar_wait(bar_gd, pp, wait_ns);
            if (!ok) break;
            fetch_vt(c0, L, c);
            ++n_u;
            // Q and W of chunk c once chunk c-1's S Q^T (issued after -S W^T) is done.
            if (c > 0) ok = mbar_wait(bar_qfree, pp, wait_ns);
            if (!ok) break;
            fetch(c0, L, true);
            bulk(B_W, REC_W, REC_P - REC_W, bar_w, c);
            ++n_w;
            // K once chunk c-1's state update is done.  A diagnostic call may
            // withhold chunk 0's K tile, so that the waits on it run out.
            if (c > 0) ok = mbar_wait(bar_gs, pp, wait_ns);
            if (!ok) break;
            if (!(p.withhold_first_k && c == 0)) fetch(c0, L, false);
        }
        // The last chunk's S Q^T commit is the one tcgen05 arrival nobody else
        // waits for; it must land before the CTA ends (after an expired wait,
        // only if its product was issued: it comes within microseconds then).
        if (lane == 0 && n_chunks > 0)
            mbar_wait(bar_qfree, (uint32_t)(n_chunks - 1) & 1u, ok ? wait_ns : 1000000ull);
        if (!ok) {
            if (lane == 0) fail();
            // No bulk copy may land after the CTA ends.
            if (n_w) mbar_wait(bar_w, (uint32_t)(n_w - 1) & 1u, wait_ns);
            if (n_tile[0]) mbar_wait(bar_k, (uint32_t)(n_tile[0] - 1) & 1u, wait_ns);
            if (n_tile[1]) mbar_wait(bar_q, (uint32_t)(n_tile[1] - 1) & 1u, wait_ns);
            if (n_u) mbar_wait(bar_u, (uint32_t)(n_u - 1) & 1u, wait_ns);
        }
        __syncwarp();
    } else if (warp == 18) {
        // --------------------------------------------- output-side producer
        // P and the per-token scalars.  Their stages are freed by the output
        // group, a chunk behind; on a warp of their own these waits no longer
        // hold up the copies the state path waits for.
        int n_p = 0, n_sc[2] = {0, 0};
        bool ok = true;
        for (int c = 0; c < n_chunks && c < 2; ++c) {
            bulk(B_SC + (c & 1) * SC_BYTES, REC_SCAL, SC_BYTES, bar_sc + (c & 1), c);
            ++n_sc[c & 1];
        }
        for (int c = 0; c < n_chunks && ok; ++c) {
            // P once chunk c-1's P Delta is done.
            if (c > 0) ok = mbar_wait(bar_oready + ((c - 1) & 1), (uint32_t)((c - 1) >> 1) & 1u, wait_ns);
            if (!ok) break;
            bulk(B_P, REC_P, REC_SCAL - REC_P, bar_p, c);
            ++n_p;
            // Scalars of chunk c+1 replace chunk c-1's once the output group is
            // done with them.
            if (c >= 1 && c + 1 < n_chunks) {
                ok = mbar_wait(bar_ofree + ((c + 1) & 1), (uint32_t)((c - 1) >> 1) & 1u, wait_ns);
                if (!ok) break;
                bulk(B_SC + ((c + 1) & 1) * SC_BYTES, REC_SCAL, SC_BYTES, bar_sc + ((c + 1) & 1), c + 1);
                ++n_sc[(c + 1) & 1];
            }
        }
        if (!ok) {
            if (lane == 0) fail();
            // No bulk copy may land after the CTA ends.
            if (n_p) mbar_wait(bar_p, (uint32_t)(n_p - 1) & 1u, wait_ns);
            for (int b = 0; b < 2; ++b)
                if (n_sc[b]) mbar_wait(bar_sc + b, (uint32_t)(n_sc[b] - 1) & 1u, wait_ns);
        }
        __syncwarp();
    } else if (warp < 8) {
        // --------------------------------------------------- state group
        const int quad = warp & 3, half = warp >> 2;
        const int i = 32 * quad + lane;
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        // Every wait's outcome is made warp-uniform, so a warp stops as a whole.
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wait_ns)) != 0;
        };
        // Hand the staged tiles and TMEM to the MMA warp: one arrival per warp.
        auto publish = [&](uint64_t *bar) {
            fence_smem_to_async();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // Row i of S (32 columns from j0): the bf16 copy, the A operand of the
        // next chunk's first MMAs ...
        auto stage_bf16 = [&](const float (&v)[32], int j0) {
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
                pk[u] = *reinterpret_cast<const uint32_t *>(&b2);
            }
            tmem_st16(tm + lane_off + TM_SB + j0 / 2, pk);
        };
        // ... and, scaled by e^{gamma_L} of the coming chunk, the fp32 state for
        // its update.
        auto stage_scaled = [&](float (&v)[32], int j0, float eL) {
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] *= eL;
            tmem_st32(tm + lane_off + TM_S + j0, v);
        };

        if (n_chunks == 0) {
            // An empty sequence leaves its state as it came in.
            if (state_out) {
                const size_t off = ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D + 64 * half;
#pragma unroll 4
                for (int j4 = 0; j4 < 16; ++j4)
                    *reinterpret_cast<float4 *>(state_out + off + 4 * j4) =
                        state_in ? __ldg(reinterpret_cast<const float4 *>(state_in + off + 4 * j4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        bool ok = n_chunks > 0 && wait_all(bar_sc, 0);
        if (ok) {
            const float eL = scal(0)[3 * C];
            const float *s0 = state_in
                                  ? state_in + ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D
                                  : nullptr;
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                const int j0 = 64 * half + 32 * jj;
                float v[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 x = s0 ? __ldg(reinterpret_cast<const float4 *>(s0 + j0 + 4 * j4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * j4] = x.x; v[4 * j4 + 1] = x.y; v[4 * j4 + 2] = x.z; v[4 * j4 + 3] = x.w;
                }
                stage_bf16(v, j0);
                stage_scaled(v, j0, eL);
            }
            publish(bar_sready);
            publish(bar_scaled);
        }
        int c = 0;
        for (; c < n_chunks && ok; ++c) {
            const float *sc = scal(c);  // landed: it gave this chunk's e^{gamma_L}
            // Delta^T = U^T - S W^T as hi/lo tiles, and its decayed, k-normalised copy.
            ok = wait_all(bar_gd, (uint32_t)c & 1u);
            if (!ok) break;
            fence_after_sync();
            // Decayed Delta^T first: it is all the state update waits for.
            float dv[2][16];
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                const int s0 = 32 * half + 16 * h16;
                float *v = dv[h16];
                float w[16];
                tmem_ld16(tm + lane_off + TM_D + s0, dv[h16]);
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    // (Delta^T itself: the U product with -S W^T accumulated onto it)
                    const float4 dn = *reinterpret_cast<const float4 *>(sc + 2 * C + s0 + 4 * s4);
                    w[4 * s4] = v[4 * s4] * dn.x; w[4 * s4 + 1] = v[4 * s4 + 1] * dn.y;
                    w[4 * s4 + 2] = v[4 * s4 + 2] * dn.z; w[4 * s4 + 3] = v[4 * s4 + 3] * dn.w;
                }
                uint32_t th[8], tl[8];
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint4 hi, lo;
                    split8(w + 8 * c8, hi, lo);
                    th[4 * c8] = hi.x; th[4 * c8 + 1] = hi.y; th[4 * c8 + 2] = hi.z; th[4 * c8 + 3] = hi.w;
                    tl[4 * c8] = lo.x; tl[4 * c8 + 1] = lo.y; tl[4 * c8 + 2] = lo.z; tl[4 * c8 + 3] = lo.w;
                }
                // Tokens s0 .. s0+15 of row i: columns s0/2 .. s0/2+7 of each tile.
                tmem_st8(tm + lane_off + TM_DTH + s0 / 2, th);
                tmem_st8(tm + lane_off + TM_DTL + s0 / 2, tl);
            }
            publish(bar_dtready);
            // Then Delta itself as hi/lo tiles in shared memory, the B operand of P Delta.
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                const int s0 = 32 * half + 16 * h16;
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint4 hi, lo;
                    split8(dv[h16] + 8 * c8, hi, lo);
                    const uint32_t o = kmaj(i, s0 + 8 * c8, D);
                    *reinterpret_cast<uint4 *>(sm + B_DL + o) = hi;
                    *reinterpret_cast<uint4 *>(sm + B_DL + 16384 + o) = lo;
                }
            }
            publish(bar_dready);

            // Once the state update is done: the next chunk's bf16 S (what its
            // first products wait for) and the state scaled for its update.
            ok = wait_all(bar_gs, (uint32_t)c & 1u);
            if (!ok || c + 1 == n_chunks) continue;
            ok = wait_all(bar_sc + ((c + 1) & 1), (uint32_t)((c + 1) >> 1) & 1u);
            if (!ok) continue;
            fence_after_sync();
            const float eL = scal(c + 1)[3 * C];
            // One read of each half row: its bf16 copy, then the pre-scaled
            // state in place (published together; reading the row twice, to
            // publish the copy first, measured slower).
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                const int j0 = 64 * half + 32 * jj;
                float v[32];
                tmem_ld32(tm + lane_off + TM_S + j0, v);
                stage_bf16(v, j0);
                stage_scaled(v, j0, eL);
            }
            publish(bar_sready);
            publish(bar_scaled);
        }
        state_ok = ok && n_chunks > 0 && c == n_chunks;
        if (n_chunks > 0 && !state_ok && lane == 0) fail();
    } else {
        // -------------------------------------------------- output group
        const int quad = warp & 3, half = (warp >> 2) & 1;
        const int og = warp - 8;                // 0..7: tokens 8*og .. 8*og+7 in the norm
        const int i = 32 * quad + lane;
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        const __nv_bfloat16 *zg = static_cast<const __nv_bfloat16 *>(p.z);
        TOUT *out = static_cast<TOUT *>(p.out);
        float *Os = reinterpret_cast<float *>(sm + B_OS);
        float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
        if (zg && p.norm_w)
            w4 = make_float4(__ldg(p.norm_w + 4 * lane), __ldg(p.norm_w + 4 * lane + 1),
                             __ldg(p.norm_w + 4 * lane + 2), __ldg(p.norm_w + 4 * lane + 3));
        // z of this warp's 8 tokens of chunk c (4 values per lane), loaded a
        // whole chunk before it is used.
        auto load_z = [&](int c, uint2 (&zr)[8]) {
            const int64_t c0 = t0 + (int64_t)c * C;
            const int L = c < n_chunks ? chunk_len(c) : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = 8 * og + u;
                zr[u] = r < L ? __ldg(reinterpret_cast<const uint2 *>(zg + (c0 + r) * p.z_stride + hv * D + 4 * lane))
                              : make_uint2(0u, 0u);
            }
        };
        uint2 zr[8];
        if (zg) load_z(0, zr);
        bool dead = false;
        for (int c = 0; c < n_chunks && !dead; ++c) {
            const int b = c & 1;
            const int64_t c0 = t0 + (int64_t)c * C;
            const int L = chunk_len(c);
            uint2 zn[8];
            if (zg) load_z(c + 1, zn);
            bool ok = mbar_wait(bar_oready + b, (uint32_t)(c >> 1) & 1u, wait_ns) &&
                      mbar_wait(bar_sc + b, (uint32_t)(c >> 1) & 1u, wait_ns);  // (long landed)
            if (ok) {
                // O^T [i][r] = (m e^gamma)_r (S Q^T) + (P Delta)^T, staged as O [r][i].
                fence_after_sync();
                const float *sc = scal(c);
                const int r0 = 32 * half;
#pragma unroll
                for (int h16 = 0; h16 < 2; ++h16) {
                    float a[16], d[16];
                    tmem_ld16(tm + lane_off + TM_OI + 64 * b + r0 + 16 * h16, a);
                    tmem_ld16(tm + lane_off + TM_O2 + r0 + 16 * h16, d);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int r = r0 + 16 * h16 + 4 * k4;
                        const float4 m = *reinterpret_cast<const float4 *>(sc + C + r);
                        const float2 o01 = __ffma2_rn(f2(m.x, m.y), f2(a[4 * k4], a[4 * k4 + 1]),
                                                      f2(d[4 * k4], d[4 * k4 + 1]));
                        const float2 o23 = __ffma2_rn(f2(m.z, m.w), f2(a[4 * k4 + 2], a[4 * k4 + 3]),
                                                      f2(d[4 * k4 + 2], d[4 * k4 + 3]));
                        Os[r * D + i] = o01.x;
                        Os[(r + 1) * D + i] = o01.y;
                        Os[(r + 2) * D + i] = o23.x;
                        Os[(r + 3) * D + i] = o23.y;
                    }
                }
            }
            // TMEM buffers and the chunk's scalars go back to the MMA warp and producer.
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_ofree + b);
            dead = group_sync_or(OG_BAR, OG_N, !ok);
            if (dead) break;
            // RMSNormGated: a warp holds 8 whole tokens, 4 values per lane.
            float4 o4[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) o4[u] = *reinterpret_cast<const float4 *>(Os + (8 * og + u) * D + 4 * lane);
            float rstd_l = 0.f;
            if (zg) {
                // Sums of squares of the 8 tokens by a transposing butterfly: after
                // the xor-4/2/1 stages lane l holds token (l & 7) summed over 8
                // lanes; xor 8 and 16 finish the sum (9 shuffles for 8 tokens).
                float ps[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float2 xy = f2(o4[u].x, o4[u].y), zw = f2(o4[u].z, o4[u].w);
                    const float2 q = __ffma2_rn(zw, zw, __fmul2_rn(xy, xy));
                    ps[u] = q.x + q.y;
                }
#pragma unroll
                for (int st = 4; st >= 1; st >>= 1) {
                    const bool upper = (lane & st) != 0;
#pragma unroll
                    for (int j = 0; j < st; ++j) {
                        const float send = upper ? ps[j] : ps[j + st];
                        const float keep = upper ? ps[j + st] : ps[j];
                        ps[j] = keep + __shfl_xor_sync(0xffffffffu, send, st);
                    }
                }
                float t = ps[0];
                t += __shfl_xor_sync(0xffffffffu, t, 8);
                t += __shfl_xor_sync(0xffffffffu, t, 16);
                rstd_l = rsqrtf(t * (1.0f / D) + p.eps_norm);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = 8 * og + u;
                float4 y = o4[u];
                if (zg) {
                    // y = (o rstd) (w z / 2) (1 + tanh(z / 2)), two values at a time.
                    const float rstd = __shfl_sync(0xffffffffu, rstd_l, u);
                    const float2 za = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zr[u].x));
                    const float2 zb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zr[u].y));
                    const float2 ha = __fmul2_rn(za, f2(0.5f, 0.5f)), hb = __fmul2_rn(zb, f2(0.5f, 0.5f));
                    const float2 ta = f2(tanh_approx(ha.x), tanh_approx(ha.y));
                    const float2 tb = f2(tanh_approx(hb.x), tanh_approx(hb.y));
                    const float2 ua = __fmul2_rn(f2(w4.x, w4.y), ha), ub = __fmul2_rn(f2(w4.z, w4.w), hb);
                    const float2 ga = __ffma2_rn(ua, ta, ua), gb = __ffma2_rn(ub, tb, ub);
                    const float2 ya = __fmul2_rn(__fmul2_rn(f2(y.x, y.y), f2(rstd, rstd)), ga);
                    const float2 yb = __fmul2_rn(__fmul2_rn(f2(y.z, y.w), f2(rstd, rstd)), gb);
                    y = make_float4(ya.x, ya.y, yb.x, yb.y);
                }
                if (r < L) Elem<TOUT>::store4(out + (c0 + r) * p.out_stride + hv * D + 4 * lane, y);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) zr[u] = zn[u];
            // The stage is rewritten by the next chunk.
            group_sync_or(OG_BAR, OG_N, false);
        }
        if (dead && tid == 256) fail();
    }

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp < 8 && state_ok && state_out) {
        const int quad = warp & 3, half = warp >> 2;
        const int i = 32 * quad + lane;
        const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
        float *dst = state_out + ((size_t)seq * p.H_v + hv) * D * D + (size_t)i * D;
#pragma unroll 1
        for (int jj = 0; jj < 2; ++jj) {
            const int j0 = 64 * half + 32 * jj;
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

}  // namespace tcp2

// How many segments: several only when the recurrence leaves at least half of
// the SMs idle (so the next segment's prep has room beside it) and the longest
// sequence is long enough to split.
int prefill_tc2p_segments(int n_seq, int H_v, int max_chunks, int n_sm) {
    return (2 * (int64_t)n_seq * H_v <= n_sm && max_chunks >= 12) ? tcp2::MAX_SEG : 1;
}

size_t prefill_tc2p_workspace_bytes(int n_seq, int64_t n_chunks, int H_v, int n_seg) {
    return tcp2::ws_layout(n_seq, n_chunks, H_v, n_seg).total;
}

// cu_host: the sequence offsets on the host (segment sizes are planned here).
// Segment boundaries: 34% and 66% of the longest sequence's chunks, so that
// each later segment's prep (on the SMs the recurrence leaves free) takes
// about as long as the recurrence of the segment before it.
cudaError_t launch_prefill_tc2p(const PrefillParams &p, const int32_t *cu_host, int n_seg,
                                void *workspace, int out_bf16, cudaStream_t s) {
    int64_t n_chunks = 0;
    int max_chunks = 0;
    for (int q = 0; q < p.n_seq; ++q) {
        const int n = (cu_host[q + 1] - cu_host[q] + tcp2::C - 1) / tcp2::C;
        n_chunks += n;
        max_chunks = n > max_chunks ? n : max_chunks;
    }
    tcp2::SegPlan sp = {};
    sp.n = n_seg < 1 ? 1 : (n_seg > tcp2::MAX_SEG ? tcp2::MAX_SEG : n_seg);
    if (sp.n == 3) {
        sp.lo[1] = (int)((max_chunks * 34 + 99) / 100);
        sp.lo[2] = (int)((max_chunks * 66 + 99) / 100);
    } else if (sp.n == 2) {
        sp.lo[1] = (int)((max_chunks * 60 + 99) / 100);
    }
    sp.lo[0] = 0;
    sp.lo[sp.n] = max_chunks;
    for (int k = 1; k <= sp.n; ++k)
        if (sp.lo[k] <= sp.lo[k - 1]) sp.n = k - 1 > 0 ? k - 1 : 1, sp.lo[sp.n] = max_chunks;
    const tcp2::WsLayout w = tcp2::ws_layout(p.n_seq, n_chunks, p.H_v, n_seg);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    int *order = reinterpret_cast<int *>(ws + w.order);
    int *chunk_off = reinterpret_cast<int *>(ws + w.chunk_off);
    int *seg_off = reinterpret_cast<int *>(ws + w.seg_off);
    float *carry = n_seg > 1 ? reinterpret_cast<float *>(ws + w.carry) : nullptr;
    unsigned char *records = ws + w.rec;
    tcp2::plan_kernel<<<1, 1024, 0, s>>>(p.cu_seqlens, p.n_seq, status, order, chunk_off, sp,
                                          seg_off);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // Tensor maps for prep's K, Q and V (the caller's bases and row strides
    // are 16-byte aligned; token offsets fit in int32).
    tcp2::PrepMaps maps;
    memset(&maps, 0, sizeof maps);
    const uint64_t n_tok = (uint64_t)cu_host[p.n_seq];
    const bool tma = n_tok > 0 && n_tok < 0x7fffffffull &&
                     encode_bf16_2d(&maps.k, p.k, (uint64_t)p.H_k * tcp2::D, n_tok,
                                    (uint64_t)p.k_stride * 2, 64, 64) &&
                     encode_bf16_2d(&maps.q, p.q, (uint64_t)p.H_k * tcp2::D, n_tok,
                                    (uint64_t)p.q_stride * 2, 64, 64) &&
                     encode_bf16_2d(&maps.v, p.v, (uint64_t)p.H_v * tcp2::D, n_tok,
                                    (uint64_t)p.v_stride * 2, 64, 64);
    if (!tma && n_tok > 0) return cudaErrorInvalidValue;  // no encoder in the driver
    e = cudaFuncSetAttribute(tcp2::prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcp2::A_SMEM_LAUNCH);
    if (e != cudaSuccess) return e;
    auto kern = out_bf16 ? tcp2::recur_kernel<__nv_bfloat16> : tcp2::recur_kernel<float>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcp2::B_SMEM_LAUNCH);
    if (e != cudaSuccess) return e;
    for (int k = 0; k < sp.n; ++k) {
        int64_t units = 0;
        for (int q = 0; q < p.n_seq; ++q) {
            const int n = (cu_host[q + 1] - cu_host[q] + tcp2::C - 1) / tcp2::C;
            const int m = (n < sp.lo[k + 1] ? n : sp.lo[k + 1]) - sp.lo[k];
            units += m > 0 ? m : 0;
        }
        const int *seg_off_k = seg_off + (size_t)k * (p.n_seq + 1);
        if (units > 0) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(units * p.H_v));
            cfg.blockDim = dim3(tcp2::PNT);
            cfg.dynamicSmemBytes = tcp2::A_SMEM_LAUNCH;
            cfg.stream = s;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            // Programmatic dependents: the first segment's prep of the plan
            // kernel, the later ones of the recurrence before them (which they
            // overlap).
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, tcp2::prep_kernel, p, maps, (const int *)chunk_off, seg_off_k,
                                   sp.lo[k], records, status, k > 0 ? 1 : 0, k == 0 ? 1 : 0);
            if (e != cudaSuccess) {
                (void)cudaGetLastError();
                return e;
            }
        } else if (k > 0) {
            continue;  // no sequence reaches this segment
        }
        kern<<<(unsigned)((int64_t)p.n_seq * p.H_v), tcp2::RNT, tcp2::B_SMEM_LAUNCH, s>>>(
            p, maps, order, chunk_off, records, status, sp.lo[k], k + 1 == sp.n ? 0x7fffffff : sp.lo[k + 1],
            carry);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr
