// gdr_moe.cu -- the routed-expert MoE feed-forward block at decode time, reading
// only the experts the router picks.
//
// The Core AI card for the Qwen3.6-35B-A3B text decoder (first section) makes
// every FFN a 256-expert top-8 mixture with a shared expert: a router
// Linear(hidden, 256), a softmax over all experts in fp32, the top 8
// renormalised by their sum, SwitchGLU experts gathered by index, and an
// always-on shared SwitchGLU scaled by sigmoid(shared_expert_gate(x)); its
// "Speed" section puts the cost of a decode step in reading only the routed
// experts' weights instead of all of them.  Per token x:
//
//   p     = softmax(W_router x)                 (fp32)
//   top-k by p (ties to the lower index), w_e = p_e / sum_{top-k} p
//   y     = sum_e w_e W_down,e (silu(W_gate,e x) * (W_up,e x))
//         + sigmoid(w_sgate . x) W_down,s (silu(W_gate,s x) * (W_up,s x))
//
// Five kernels on the caller's stream, each a programmatic dependent of the
// one before (each waits for it before reading what it wrote):
//   router:  one warp per router row (and one for the shared gate row): the
//            row's dot products with every token, fp32.
//   route:   one block: per token the softmax, the top-k and the weights; then
//            the (token, slot) pairs grouped by expert, the shared expert last
//            with every token, so that each expert's weights are read once
//            for all the tokens that chose it.
//   gate_up: per (active expert, 16 intermediate rows): the gate and up rows
//            against each of the expert's tokens, h = silu(g) * u (fp32).
//   down:    per (active expert, 32 output rows): w * (W_down h) per pair.
//   combine: per (token, 256 outputs), the sum of its pairs' partial outputs.
// Weights are bf16; all arithmetic is fp32.  Bound by HBM on the weights read.
#include "gdr.h"
#include "gdr_common.cuh"

namespace gdr {

struct MoeParams {
    int n_tok, hidden, n_exp, top_k, inter, s_inter;
    int64_t x_stride, out_stride;
    const __nv_bfloat16 *x, *w_router, *w_gate_up, *w_down, *ws_gate_up, *ws_down, *w_sgate;
    void *out;
    int32_t *topk_idx;
    float *topk_w;
    // workspace
    float *logits;      // [n_tok][n_exp + 1]  (the last column: the shared gate's dot product)
    int *n_active;      // active experts (shared expert included)
    int *act_expert;    // [n_exp + 1] expert of active slot a (n_exp = the shared expert)
    int *act_off;       // [n_exp + 2] first pair of slot a
    int *pair_tok;      // [n_pairs] token of pair i (pairs grouped by expert)
    float *pair_w;      // [n_pairs] the pair's weight
    int *tok_pair;      // [n_tok][top_k + 1] pair index of (token, slot); the shared one last
    int router_tg;      // tokens the router stages in shared memory per pass (1..8)
    float *h;           // [n_pairs][max(inter, s_inter)]
    float *part;        // [n_pairs][hidden]
};

namespace moe {

constexpr int GU_ROWS = 16;   // intermediate rows per gate_up block (x 2: gate and up)
constexpr int ROUTE_THREADS = 1024;  // also the most experts (one thread each in the scans)

// Dot products of ROWS bf16 rows with one bf16 vector x of n values (n a
// multiple of 8), by one warp: lane l takes 16-byte chunks l, l + 32, ...; the
// rows' chunks for a batch of 8 chunk steps are all loaded before any is used,
// so each lane keeps 8 * ROWS 16-byte loads in flight.  Returns the warp sums.
template <int ROWS>
__device__ __forceinline__ void warp_dots_bf16(const __nv_bfloat16 *const (&w)[ROWS],
                                               const __nv_bfloat16 *x, int n, int lane,
                                               float (&out)[ROWS]) {
    float acc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) acc[r] = 0.f;
    const int nc = n / 8;
    for (int c0 = 0; c0 < nc; c0 += 32 * 8) {
        uint4 a[ROWS][8], b[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = c0 + lane + 32 * u;
            b[u] = c < nc ? __ldg(reinterpret_cast<const uint4 *>(x) + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < ROWS; ++r)
                a[r][u] = c < nc ? __ldg(reinterpret_cast<const uint4 *>(w[r]) + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&b[u]);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const __nv_bfloat162 *a2 = reinterpret_cast<const __nv_bfloat162 *>(&a[r][u]);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float2 fa = __bfloat1622float2(a2[v]), fb = __bfloat1622float2(b2[v]);
                    acc[r] = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc[r]));
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) out[r] = group_sum<32>(acc[r]);
}

// The dot product of 8 bf16 weights with 8 bf16 inputs, added to acc (fp32),
// in the order warp_dots_bf16 uses.
__device__ __forceinline__ float dot8_bf16(const uint4 &a, const uint4 &b, float acc) {
    const __nv_bfloat162 *a2 = reinterpret_cast<const __nv_bfloat162 *>(&a);
    const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&b);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const float2 fa = __bfloat1622float2(a2[v]), fb = __bfloat1622float2(b2[v]);
        acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
    }
    return acc;
}

constexpr int TG = 8;  // tokens that share one pass over a weight row

// ------------------------------------------------------------------ router
// One warp per router row e (e == n_exp: the shared-expert gate), every token.
// The block stages up to router_tg token rows in shared memory at a time, and
// each warp streams its row past them once per group: one load per 16-byte
// chunk of the row, the token values read from shared memory.
__global__ void __launch_bounds__(256) router_kernel(const MoeParams p) {
    extern __shared__ uint4 xs[];  // [router_tg][hidden / 8]
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
    const bool shared_row = e == p.n_exp;
    const bool active = e < p.n_exp || (shared_row && p.s_inter > 0);
    const uint4 *w = reinterpret_cast<const uint4 *>(
        shared_row ? p.w_sgate : p.w_router + (size_t)min(e, p.n_exp - 1) * p.hidden);
    const int nc = p.hidden / 8;
    // The row's first RPRE chunks per lane come in before the wait on the
    // previous kernel (which may write x, never the weights).
    constexpr int RPRE = 8;
    uint4 wpre[RPRE];
#pragma unroll
    for (int u = 0; u < RPRE; ++u) {
        const int c = lane + 32 * u;
        wpre[u] = active && c < nc ? __ldg(w + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    wait_for_predecessor();
    release_dependents();
    for (int t0 = 0; t0 < p.n_tok; t0 += p.router_tg) {
        const int ng = min(p.router_tg, p.n_tok - t0);
        __syncthreads();  // the previous group is done with xs
        for (int i = threadIdx.x; i < ng * nc; i += blockDim.x) {
            const int t = i / nc, c = i - t * nc;
            xs[i] = __ldg(reinterpret_cast<const uint4 *>(p.x + (int64_t)(t0 + t) * p.x_stride) + c);
        }
        __syncthreads();
        if (!active) continue;
        float acc[TG];
#pragma unroll
        for (int t = 0; t < TG; ++t) acc[t] = 0.f;
#pragma unroll
        for (int u = 0; u < RPRE; ++u) {
            const int c = lane + 32 * u;
            if (c < nc) {
#pragma unroll
                for (int t = 0; t < TG; ++t)
                    if (t < ng) acc[t] = dot8_bf16(wpre[u], xs[t * nc + c], acc[t]);
            }
        }
#pragma unroll 8
        for (int c = lane + 32 * RPRE; c < nc; c += 32) {
            const uint4 wv = __ldg(w + c);
#pragma unroll
            for (int t = 0; t < TG; ++t)
                if (t < ng) acc[t] = dot8_bf16(wv, xs[t * nc + c], acc[t]);
        }
#pragma unroll
        for (int t = 0; t < TG; ++t) {
            if (t >= ng) break;
            const float d = group_sum<32>(acc[t]);
            if (lane == 0) p.logits[(size_t)(t0 + t) * (p.n_exp + 1) + e] = d;
        }
    }
}

// Exclusive prefix sums of a and c over the block's threads (in thread order)
// and their totals; every thread of the block calls it.
__device__ __forceinline__ void block_scan2(int a, int c, int &ea, int &ec, int &ta, int &tc,
                                            int *scratch /* 2 * 32 ints */) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int ia = a, ic = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int xa = __shfl_up_sync(kFullMask, ia, o), xc = __shfl_up_sync(kFullMask, ic, o);
        if (lane >= o) {
            ia += xa;
            ic += xc;
        }
    }
    if (lane == 31) {
        scratch[warp] = ia;
        scratch[32 + warp] = ic;
    }
    __syncthreads();
    if (warp == 0) {
        int wa = lane < nw ? scratch[lane] : 0, wc = lane < nw ? scratch[32 + lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int xa = __shfl_up_sync(kFullMask, wa, o), xc = __shfl_up_sync(kFullMask, wc, o);
            if (lane >= o) {
                wa += xa;
                wc += xc;
            }
        }
        if (lane < nw) {
            scratch[lane] = wa;  // inclusive over warps 0..lane
            scratch[32 + lane] = wc;
        }
    }
    __syncthreads();
    const int pa = warp > 0 ? scratch[warp - 1] : 0, pc = warp > 0 ? scratch[32 + warp - 1] : 0;
    ea = pa + ia - a;
    ec = pc + ic - c;
    ta = scratch[nw - 1];
    tc = scratch[32 + nw - 1];
    __syncthreads();
}

// ------------------------------------------------------------------- route
// One block: softmax, top-k and weights per token (one warp per token), then
// the pairs grouped by expert.  MAXE: experts per lane in the softmax
// (n_exp <= 32 * MAXE), held in registers.
template <int MAXE>
__global__ void __launch_bounds__(ROUTE_THREADS) route_kernel(const MoeParams p) {
    wait_for_predecessor();
    release_dependents();
    extern __shared__ int rsm[];
    int *cnt = rsm;                      // [n_exp + 1] tokens per expert
    int *fill = cnt + (p.n_exp + 1);     // [n_exp + 1] running fill per expert
    int *slot_of = fill + (p.n_exp + 1); // [n_exp + 1] active slot of expert e (or -1)
    int *scan = slot_of + (p.n_exp + 1); // [64] block-scan scratch
    int *sel = scan + 64;                // [n_tok][top_k] selected experts
    float *selw = reinterpret_cast<float *>(sel + p.n_tok * p.top_k);  // [n_tok][top_k]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = p.n_exp, K = p.top_k;
    const bool has_shared = p.s_inter > 0;
    for (int e = tid; e <= E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int t = warp; t < p.n_tok; t += blockDim.x / 32) {
        // Lane l holds the probabilities of experts l, l + 32, ... in registers.
        const float *lg = p.logits + (size_t)t * (E + 1);
        float pr[MAXE];
        float m = -INFINITY;
#pragma unroll
        for (int u = 0; u < MAXE; ++u) {
            const int e = lane + 32 * u;
            pr[u] = e < E ? lg[e] : -INFINITY;
            m = fmaxf(m, pr[u]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        float z = 0.f;
#pragma unroll
        for (int u = 0; u < MAXE; ++u) {
            pr[u] = lane + 32 * u < E ? expf(pr[u] - m) : 0.f;
            z += pr[u];
        }
        z = group_sum<32>(z);
        const float rz = 1.f / z;
#pragma unroll
        for (int u = 0; u < MAXE; ++u) pr[u] = lane + 32 * u < E ? pr[u] * rz : -1.f;
        // Top-k, ties to the lower index: k rounds of a warp arg-max over each
        // lane's best untaken expert; the winner's lane marks it taken.
        uint32_t taken = 0;
        float wsum = 0.f;
        for (int k = 0; k < K; ++k) {
            float bv = -1.f;
            int bi = 0x7fffffff;
#pragma unroll
            for (int u = 0; u < MAXE; ++u) {
                if (!((taken >> u) & 1u) && pr[u] > bv) {  // u ascending: ties keep the lower index
                    bv = pr[u];
                    bi = lane + 32 * u;
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(kFullMask, bv, o);
                const int oi = __shfl_xor_sync(kFullMask, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            if (lane == 0) {
                sel[t * K + k] = bi;
                selw[t * K + k] = bv;
                atomicAdd(&cnt[bi], 1);
            }
            wsum += bv;
        }
        __syncwarp();
        if (lane < K) {
            const float wk = selw[t * K + lane] / wsum;
            selw[t * K + lane] = wk;
            if (p.topk_idx) p.topk_idx[(size_t)t * K + lane] = sel[t * K + lane];
            if (p.topk_w) p.topk_w[(size_t)t * K + lane] = wk;
        }
    }
    __syncthreads();
    // Active slots in expert order (thread e = expert e), the shared expert
    // last; pair offsets.  Exclusive scans of "chosen at all" and of the counts.
    {
        const int e = tid;
        const int ce = e < E ? cnt[e] : 0;
        int slot, off, n_routed, n_pairs;
        block_scan2(ce > 0 ? 1 : 0, ce, slot, off, n_routed, n_pairs, scan);
        if (e < E) {
            slot_of[e] = ce > 0 ? slot : -1;
            if (ce > 0) {
                p.act_expert[slot] = e;
                p.act_off[slot] = off;
                fill[e] = off;
            }
        }
        if (tid == 0) {
            int a = n_routed, end_off = n_pairs;
            if (has_shared) {
                slot_of[E] = a;
                p.act_expert[a] = E;
                p.act_off[a] = end_off;
                fill[E] = end_off;
                end_off += p.n_tok;
                ++a;
            }
            p.act_off[a] = end_off;
            *p.n_active = a;
        }
    }
    __syncthreads();
    // Pairs: (token, slot k) under its expert, in token order (one thread per token).
    for (int t = tid; t < p.n_tok; t += blockDim.x) {
        for (int k = 0; k < K; ++k) {
            const int e = sel[t * K + k];
            const int i = atomicAdd(&fill[e], 1);
            p.pair_tok[i] = t;
            p.pair_w[i] = selw[t * K + k];
            p.tok_pair[(size_t)t * (K + 1) + k] = i;
        }
        if (has_shared) {
            const int i = p.act_off[slot_of[E]] + t;
            const float s = p.logits[(size_t)t * (E + 1) + E];
            p.pair_tok[i] = t;
            p.pair_w[i] = 1.f / (1.f + expf(-s));
            p.tok_pair[(size_t)t * (K + 1) + K] = i;
        }
    }
}

// ---------------------------------------------------------------- gate_up
// Block (a, j0): rows j0 .. j0+15 of the gate and up matrices of active
// expert a; warp w takes rows j0 + 2w, j0 + 2w + 1.  h = silu(g) * u per pair.
__global__ void __launch_bounds__(256, 2) gate_up_kernel(const MoeParams p) {
    wait_for_predecessor();
    release_dependents();
    const int a = blockIdx.y;
    if (a >= *p.n_active) return;
    const int e = p.act_expert[a];
    const bool sh = e == p.n_exp;
    const int I = sh ? p.s_inter : p.inter;
    const int j0 = blockIdx.x * GU_ROWS;
    if (j0 >= I) return;
    const __nv_bfloat16 *W = sh ? p.ws_gate_up : p.w_gate_up + (size_t)e * 2 * p.inter * p.hidden;
    const int p0 = p.act_off[a], p1 = p.act_off[a + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hmax = p.inter > p.s_inter ? p.inter : p.s_inter;
    // The warp's two rows of the gate matrix and the same two of the up matrix,
    // all four streamed together for each of the expert's tokens.
    const int j = j0 + 2 * warp;
    if (j >= I) return;
    const int j1 = j + 1 < I ? j + 1 : j;
    const __nv_bfloat16 *w[4] = {W + (size_t)j * p.hidden, W + (size_t)j1 * p.hidden,
                                 W + (size_t)(I + j) * p.hidden, W + (size_t)(I + j1) * p.hidden};
    if (p1 - p0 == 1) {
        // One token (every routed expert at small batch): all of the four rows'
        // loads in flight at once.
        float d[4];
        warp_dots_bf16<4>(w, p.x + (int64_t)p.pair_tok[p0] * p.x_stride, p.hidden, lane, d);
        if (lane == 0) {
            p.h[(size_t)p0 * hmax + j] = d[0] / (1.f + expf(-d[0])) * d[2];
            if (j1 != j) p.h[(size_t)p0 * hmax + j1] = d[1] / (1.f + expf(-d[1])) * d[3];
        }
        return;
    }
    // Several tokens (the shared expert, or a popular one): each chunk of the
    // four rows is loaded once per group of up to GU_TG tokens.
    constexpr int GU_TG = 4;
    const int nc = p.hidden / 8;
    for (int g0 = p0; g0 < p1; g0 += GU_TG) {
        const int ng = min(GU_TG, p1 - g0);
        const uint4 *xr[GU_TG];
#pragma unroll
        for (int t = 0; t < GU_TG; ++t)
            xr[t] = reinterpret_cast<const uint4 *>(p.x + (int64_t)p.pair_tok[g0 + min(t, ng - 1)] * p.x_stride);
        float acc[GU_TG][4];
#pragma unroll
        for (int t = 0; t < GU_TG; ++t)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[t][r] = 0.f;
#pragma unroll 2
        for (int c = lane; c < nc; c += 32) {
            uint4 wv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) wv[r] = __ldg(reinterpret_cast<const uint4 *>(w[r]) + c);
#pragma unroll
            for (int t = 0; t < GU_TG; ++t) {  // rows past ng repeat the last token (unused)
                const uint4 xv = __ldg(xr[t] + c);
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[t][r] = dot8_bf16(wv[r], xv, acc[t][r]);
            }
        }
#pragma unroll
        for (int t = 0; t < GU_TG; ++t) {
            if (t >= ng) break;
            float d[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) d[r] = group_sum<32>(acc[t][r]);
            if (lane == 0) {
                const size_t i = (size_t)(g0 + t);
                p.h[i * hmax + j] = d[0] / (1.f + expf(-d[0])) * d[2];
                if (j1 != j) p.h[i * hmax + j1] = d[1] / (1.f + expf(-d[1])) * d[3];
            }
        }
    }
}

// ------------------------------------------------------------------- down
// Block (a, i0): output rows i0 .. i0 + 8 RPW - 1 of active expert a's down
// matrix; warp w takes RPW rows from i0 + RPW w.  part[pair] = w_pair * W_down h.
// MAXC: 16-byte chunks of a row per lane (I <= 256 MAXC).  The routing (expert
// list, offsets, pair weights) was complete before the gate/up kernel started,
// and this grid starts after that: a block reads it, and streams in its
// expert's weight rows, before it waits for h.
template <int RPW, int MAXC>
__global__ void __launch_bounds__(256, 2) down_kernel(const MoeParams p) {
    static_assert(RPW % 4 == 0, "rows per warp in groups of four");
    const int a = blockIdx.y;
    // Read at L2 (the buffers are rewritten by every layer's routing).
    if (a >= __ldcg(p.n_active)) return;
    const int e = __ldcg(p.act_expert + a);
    const bool sh = e == p.n_exp;
    const int I = sh ? p.s_inter : p.inter;
    const __nv_bfloat16 *W = sh ? p.ws_down : p.w_down + (size_t)e * p.hidden * p.inter;
    const int p0 = __ldcg(p.act_off + a), p1 = __ldcg(p.act_off + a + 1);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hmax = p.inter > p.s_inter ? p.inter : p.s_inter;
    const int row0 = blockIdx.x * (8 * RPW) + RPW * warp;
    const bool wactive = row0 < p.hidden;
    const int nc = I / 8;
    auto wrow = [&](int r) {
        return reinterpret_cast<const uint4 *>(W + (size_t)min(row0 + r, p.hidden - 1) * I);
    };
    // 8 weights (one 16-byte chunk) against 8 fp32 values of h.
    auto dot8_h = [](const uint4 &w, const float4 &h0, const float4 &h1, float acc) {
        const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
        const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float2 f = __bfloat1622float2(w2[v]);
            acc = fmaf(f.x, hv[2 * v], fmaf(f.y, hv[2 * v + 1], acc));
        }
        return acc;
    };
    // Rows row0 + rb .. row0 + rb + N - 1 of pair i.
    auto store = [&](int i, const float *acc, int rb, int N) {
        for (int r = 0; r < N; ++r) {
            const float v = group_sum<32>(acc[r]);
            if (lane == 0 && row0 + rb + r < p.hidden)
                p.part[(size_t)i * p.hidden + row0 + rb + r] = p.pair_w[i] * v;
        }
    };
    if (p1 - p0 == 1) {
        // One pair (every routed expert at small batch): the warp's rows stream
        // past once, all of a lane's chunks in flight together, issued before
        // the wait for h.
        uint4 wv[RPW][MAXC];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const uint4 *wr = wrow(r);
#pragma unroll
            for (int u = 0; u < MAXC; ++u) {
                const int c = lane + 32 * u;
                wv[r][u] = wactive && c < nc ? __ldg(wr + c) : make_uint4(0, 0, 0, 0);
            }
        }
        wait_for_predecessor();
        release_dependents();
        if (!wactive) return;
        const float *hp = p.h + (size_t)p0 * hmax;
        float4 h0[MAXC], h1[MAXC];
#pragma unroll
        for (int u = 0; u < MAXC; ++u) {
            const int c = lane + 32 * u;
            const bool in = c < nc;
            h0[u] = in ? *reinterpret_cast<const float4 *>(hp + 8 * c) : make_float4(0.f, 0.f, 0.f, 0.f);
            h1[u] = in ? *reinterpret_cast<const float4 *>(hp + 8 * c + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float acc[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) acc[r] = 0.f;
#pragma unroll
        for (int u = 0; u < MAXC; ++u)
#pragma unroll
            for (int r = 0; r < RPW; ++r) acc[r] = dot8_h(wv[r][u], h0[u], h1[u], acc[r]);
        store(p0, acc, 0, RPW);
        return;
    }
    // Several pairs (the shared expert, or a popular one): up to DN_G pairs' h
    // staged in shared memory, and each chunk of four rows applied to all of
    // them once it is loaded (the warp's rows four at a time).
    wait_for_predecessor();
    release_dependents();
    constexpr int DN_G = 8;
    __shared__ __align__(16) float hs[DN_G][1024];
    for (int g0 = p0; g0 < p1; g0 += DN_G) {
        const int ng = min(DN_G, p1 - g0);
        __syncthreads();  // the previous group is done with hs
        for (int e = threadIdx.x; e < ng * (I / 4); e += blockDim.x) {
            const int t = e / (I / 4), c4 = e - t * (I / 4);
            *reinterpret_cast<float4 *>(&hs[t][4 * c4]) =
                *reinterpret_cast<const float4 *>(p.h + (size_t)(g0 + t) * hmax + 4 * c4);
        }
        __syncthreads();
        if (!wactive) continue;
        for (int rb = 0; rb < RPW && row0 + rb < p.hidden; rb += 4) {
            const uint4 *wr[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) wr[r] = wrow(rb + r);
            float acc[DN_G][4];
#pragma unroll
            for (int t = 0; t < DN_G; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[t][r] = 0.f;
            for (int c = lane; c < nc; c += 32) {
                uint4 wv[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) wv[r] = __ldg(wr[r] + c);
#pragma unroll
                for (int t = 0; t < DN_G; ++t) {  // rows past ng repeat the last pair (unused)
                    const float *hp = hs[min(t, ng - 1)];
                    const float4 a = *reinterpret_cast<const float4 *>(hp + 8 * c);
                    const float4 b = *reinterpret_cast<const float4 *>(hp + 8 * c + 4);
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[t][r] = dot8_h(wv[r], a, b, acc[t][r]);
                }
            }
#pragma unroll
            for (int t = 0; t < DN_G; ++t)
                if (t < ng) store(g0 + t, acc[t], rb, 4);
        }
    }
}

// ---------------------------------------------------------------- combine
// Block (t, c): outputs 256c .. 256c+255 of token t, one per thread, each the
// sum of the token's pairs' partials (their loads all in flight together).
template <typename TOUT>
__global__ void __launch_bounds__(256) combine_kernel(const MoeParams p) {
    wait_for_predecessor();
    release_dependents();
    __shared__ int tp[33];  // top_k <= 32, and the shared pair
    const int t = blockIdx.x, i = blockIdx.y * 256 + threadIdx.x;
    const int np = p.top_k + (p.s_inter > 0 ? 1 : 0);
    if (threadIdx.x < np) tp[threadIdx.x] = p.tok_pair[(size_t)t * (p.top_k + 1) + threadIdx.x];
    __syncthreads();
    if (i >= p.hidden) return;
    float y = 0.f;
    for (int k = 0; k < np; ++k) y += p.part[(size_t)tp[k] * p.hidden + i];
    Elem<TOUT>::store1(static_cast<TOUT *>(p.out) + (int64_t)t * p.out_stride + i, y);
}

}  // namespace moe

// Workspace layout (256-byte aligned pieces).
struct MoeWs {
    size_t logits, n_active, act_expert, act_off, pair_tok, pair_w, tok_pair, h, part, total;
};
static MoeWs moe_ws(int n_tok, int n_exp, int top_k, int inter, int s_inter, int hidden) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t pairs = (size_t)n_tok * (top_k + (s_inter > 0 ? 1 : 0));
    const int hmax = inter > s_inter ? inter : s_inter;
    MoeWs w;
    size_t o = 0;
    w.logits = o; o = al(o + (size_t)n_tok * (n_exp + 1) * 4);
    w.n_active = o; o = al(o + 4);
    w.act_expert = o; o = al(o + (size_t)(n_exp + 1) * 4);
    w.act_off = o; o = al(o + (size_t)(n_exp + 2) * 4);
    w.pair_tok = o; o = al(o + pairs * 4);
    w.pair_w = o; o = al(o + pairs * 4);
    w.tok_pair = o; o = al(o + (size_t)n_tok * (top_k + 1) * 4);
    w.h = o; o = al(o + pairs * hmax * 4);
    w.part = o; o = al(o + pairs * hidden * 4);
    w.total = o;
    return w;
}

size_t moe_workspace_bytes(int n_tok, int n_exp, int top_k, int inter, int s_inter, int hidden) {
    return moe_ws(n_tok, n_exp, top_k, inter, s_inter, hidden).total;
}

size_t moe_route_smem_bytes(int n_tok, int n_exp, int top_k) {
    return (size_t)3 * (n_exp + 1) * 4 + 64 * 4 + (size_t)n_tok * top_k * 8;
}

cudaError_t launch_moe_args(const gdr_moe_args *a, void *workspace, cudaStream_t s) {
    MoeParams p = {};
    p.n_tok = a->n_tok;
    p.hidden = a->hidden;
    p.n_exp = a->n_exp;
    p.top_k = a->top_k;
    p.inter = a->inter;
    p.s_inter = a->ws_gate_up ? a->s_inter : 0;
    p.x_stride = a->x_stride;
    p.out_stride = a->out_stride;
    p.x = static_cast<const __nv_bfloat16 *>(a->x);
    p.w_router = static_cast<const __nv_bfloat16 *>(a->w_router);
    p.w_gate_up = static_cast<const __nv_bfloat16 *>(a->w_gate_up);
    p.w_down = static_cast<const __nv_bfloat16 *>(a->w_down);
    p.ws_gate_up = static_cast<const __nv_bfloat16 *>(a->ws_gate_up);
    p.ws_down = static_cast<const __nv_bfloat16 *>(a->ws_down);
    p.w_sgate = static_cast<const __nv_bfloat16 *>(a->w_sgate);
    p.out = a->out;
    p.topk_idx = a->topk_idx;
    p.topk_w = a->topk_w;
    const MoeWs w = moe_ws(p.n_tok, p.n_exp, p.top_k, p.inter, p.s_inter, p.hidden);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    p.logits = reinterpret_cast<float *>(ws + w.logits);
    p.n_active = reinterpret_cast<int *>(ws + w.n_active);
    p.act_expert = reinterpret_cast<int *>(ws + w.act_expert);
    p.act_off = reinterpret_cast<int *>(ws + w.act_off);
    p.pair_tok = reinterpret_cast<int *>(ws + w.pair_tok);
    p.pair_w = reinterpret_cast<float *>(ws + w.pair_w);
    p.tok_pair = reinterpret_cast<int *>(ws + w.tok_pair);
    p.h = reinterpret_cast<float *>(ws + w.h);
    p.part = reinterpret_cast<float *>(ws + w.part);

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    auto launch = [&](auto kern, dim3 grid, unsigned block, size_t smem) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(block);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t r = cudaLaunchKernelEx(&cfg, kern, p);
        if (r != cudaSuccess) (void)cudaGetLastError();
        return r;
    };
    cudaError_t e;
    const int rows = p.n_exp + 1;
    // Token rows staged per router pass: up to TG, within 96 KB of shared memory.
    const size_t row_bytes = (size_t)p.hidden * 2;
    size_t tg = (96 * 1024) / row_bytes;
    tg = tg < 1 ? 1 : (tg > (size_t)moe::TG ? (size_t)moe::TG : tg);
    p.router_tg = (int)tg;
    const size_t xsm = tg * row_bytes;
    if (xsm > 48 * 1024) {
        e = cudaFuncSetAttribute(moe::router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)xsm);
        if (e != cudaSuccess) return e;
    }
    if ((e = launch(moe::router_kernel, dim3((rows + 7) / 8), 256, xsm)) != cudaSuccess) return e;
    const size_t rsm = moe_route_smem_bytes(p.n_tok, p.n_exp, p.top_k);
    // Fewer experts per lane in registers when they fit.
    auto route = p.n_exp <= 256 ? moe::route_kernel<8> : moe::route_kernel<32>;
    if (rsm > 48 * 1024) {
        e = cudaFuncSetAttribute(route, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsm);
        if (e != cudaSuccess) return e;
    }
    if ((e = launch(route, dim3(1), moe::ROUTE_THREADS, rsm)) != cudaSuccess) return e;
    // Active slots: at most min(n_tok * top_k, n_exp) routed experts and the shared one.
    const long routed = (long)p.n_tok * p.top_k < p.n_exp ? (long)p.n_tok * p.top_k : p.n_exp;
    const unsigned max_active = (unsigned)(routed + (p.s_inter > 0 ? 1 : 0));
    const int imax = p.inter > p.s_inter ? p.inter : p.s_inter;
    if ((e = launch(moe::gate_up_kernel, dim3((imax + moe::GU_ROWS - 1) / moe::GU_ROWS, max_active),
                    256, 0)) != cudaSuccess)
        return e;
    // Eight rows per warp while a row fits in two chunks per lane (I <= 512):
    // twice the bytes in flight per block, half the blocks.
    if (imax <= 512)
        e = launch(moe::down_kernel<8, 2>, dim3((p.hidden + 63) / 64, max_active), 256, 0);
    else
        e = launch(moe::down_kernel<4, 4>, dim3((p.hidden + 31) / 32, max_active), 256, 0);
    if (e != cudaSuccess) return e;
    const dim3 cgrid(p.n_tok, (p.hidden + 255) / 256);
    if (a->out_dtype == GDR_BF16)
        e = launch(moe::combine_kernel<__nv_bfloat16>, cgrid, 256, 0);
    else
        e = launch(moe::combine_kernel<float>, cgrid, 256, 0);
    return e;
}

}  // namespace gdr
