// gdr_attn.cu -- one decode step of the gated full-attention layer, the other
// mixer of the hybrid decoder (GatedAttention in the Qwen3.5 Chat guide,
// section "Architektur": standard scaled-dot-product attention over a KV
// cache; on the Core AI Qwen3.6-35B-A3B card, first section: head_dim 256,
// 16 query heads over 2 key/value heads, partial rotary embedding with
// theta = 1e7).  Per sequence b with L = cache_len[b] tokens already cached:
//
//   q_rot, k_rot = RoPE(q), RoPE(k) at position L on the first rot_dim dims
//                  (dim i paired with i + rot_dim/2, angle L theta^(-2i/rot_dim))
//   cache[L]     = (k_rot, v)                               (appended)
//   o_h          = sum_{t <= L} softmax_t(scale q_rot_h . k_t) v_t
//   y_h          = o_h * sigmoid(gate_h)
//
// Three kernels on the caller's stream, each a programmatic dependent of the
// one before:
//   rope_append: per (b, kv head): rotates q (the group's query heads) and k in
//     fp32 with angles taken in double, appends the key and value at row L,
//     and stages the rotated queries as the bf16 MMA operand tile of the group.
//   attend: persistent; each work item is one (b, kv head, split of the
//     tokens).  One thread streams the K and V rows through two three-slot
//     rings of 32 KB shared-memory slots (one d-half of a 128-token tile each) with
//     TMA tensor copies into 128-byte-swizzled tiles, so that the memory
//     instruction pipe stays free for the softmax warps; MMA warps issue
//     S^T = K Q^T (M = 128 tokens, N = 16 query-head columns, K = 256) and
//     O^T += V^T P^T (M = 128 dims per half, N = 16, K = 128 tokens) on
//     tcgen05 with the accumulators in TMEM; four softmax warps (thread = TMEM
//     lane) keep the running maxima and sums, write P as bf16 and rescale O^T
//     when a maximum moves.  The item's (m, l, O) go to the workspace.
//   combine: per (b, kv head): merges the splits' partials and applies the
//     output gate.  When every (b, kv head) is one work item there is nothing
//     to merge: the attend kernel's softmax warps apply the gate and store
//     the output themselves, and combine is not launched.
//
// The contraction per token and key/value head is 2 x 256 MACs per query head:
// at decode the layer is bound by HBM, reading the cache once.  Every wait is
// bounded (2 s); on expiry the kernel records GDR_ERR_TIMEOUT in the workspace
// status word, waits (bounded) for its copies in flight, frees its tensor
// memory and returns.
#include "gdr_tmap.cuh"
#include <math.h>

#include "gdr.h"
#include "gdr_common.cuh"
#include "gdr_tc.cuh"

namespace gdr {

struct AttnParams {
    // 2-D TMA maps of the caches: [batch * H_kv * max_len rows][256] bf16,
    // boxes of 64 dims x 128 rows, 128-byte swizzle.
    CUtensorMap tm_k, tm_v;
    int batch, H_q, H_kv, n_rep, rot_dim, max_len, kv_bound;
    int n_split, split_tok, n_items;
    int out_bf16;
    float scale;
    double log2_theta;
    int64_t q_stride, gate_stride, k_stride, v_stride, out_stride;
    const __nv_bfloat16 *q, *gate, *k, *v;
    __nv_bfloat16 *k_cache, *v_cache;
    const int32_t *cache_len;
    void *out;
    // workspace
    int *status;             // the call's status: rope_append's length check, GDR_ERR_TIMEOUT on expiry
    __nv_bfloat16 *q_tiles;  // [batch * H_kv][16 x 256] bf16, operand layout
    float *part_o;           // [n_items][16][256]
    float *part_ml;          // [n_items][16][2]
};

namespace attn {

using namespace gdr::tc;

constexpr int D = 256;
constexpr int TILE = 128;                 // tokens per tile
constexpr int NH = 16;                    // query-head columns per key/value head
constexpr int NSLOT = 6;
// Two rings of three slots: K quarters only in slots 0-2, V quarters only in
// 3-5.  Each slot's uses then all belong to one consumer, in order, so a
// consumer never waits for a use whose slot still holds an earlier,
// unfinished use of the other kind (a parity wait would take that older
// phase for this one).
constexpr int NRING = 3;
constexpr uint32_t SLOT = 32768;          // one d-half of a K or V tile, bf16
constexpr uint32_t BOX = 16384;           // one TMA box: 128 tokens x 64 dims
constexpr uint32_t QTILE = NH * D * 2;    // 8 KB
constexpr uint32_t PTILE = NH * TILE * 2; // 4 KB
constexpr uint32_t S_RING = 0;
constexpr uint32_t S_Q = S_RING + NSLOT * SLOT;   // 2 x Q tile
constexpr uint32_t S_P = S_Q + 2 * QTILE;         // 2 x P tile
constexpr uint32_t S_RED = S_P + 2 * PTILE;       // 4 warps x 16 floats
constexpr uint32_t S_BAR = S_RED + 256;
constexpr uint32_t S_BYTES = S_BAR + 256;
constexpr uint32_t S_ALLOC = S_BYTES + 1024;  // room to align the ring to 1024 bytes
constexpr int NTHR = 224;  // warps 0-3 softmax, 4 producer, 5 S^T issue, 6 O^T issue
constexpr uint64_t kWaitNs = 2000000000ull;
// Unwinding after an expired wait: arrivals still owed to this CTA come
// within microseconds if their operations were issued, never if not.
constexpr uint64_t kDrainNs = 1000000ull;
constexpr int kTimeout = 6;  // GDR_ERR_TIMEOUT
constexpr int kBadLen = 1;   // GDR_ERR_INVALID_ARG
// TMEM columns: S^T double buffer, O^T two d-halves.
constexpr uint32_t TM_S = 0, TM_O = 32, TM_COLS = 64;

// K / V slot: two TMA boxes (dims 0-63 and 64-127 of the half), each 128
// token rows of 128 bytes with 128-byte swizzle: the 16-byte chunk j (8 dims)
// of row r sits at box + r * 128 + (j ^ (r % 8)) * 16.  Read as K-major A for
// S^T (M = tokens: SBO 1024 between 8-row groups; a K step of 16 dims moves
// the start 32 bytes inside the row, a box every 4 steps) and as MN-major A
// for O^T (M = dims: LBO = BOX between the two 64-dim boxes, SBO 1024 between
// 8-token groups; a K step of 16 tokens moves the start 2048 bytes).
// Q tile: query-head column h of 16, dim chunk c of 32 (K-major B for S^T):
//   byte = c * 256 + h * 16   (LBO 256 between chunks, SBO 128 between 8-head groups)
__host__ __device__ constexpr uint32_t q_off(int h, int c) { return (uint32_t)(c * 256 + h * 16); }
// P tile: token t, query-head column h (MN-major B for O^T, the heads
// contiguous): byte = (h / 8) * 2048 + t * 16 + (h % 8) * 2, so a thread's
// token row is two 16-byte stores (LBO 128 between 8-token groups, SBO 2048
// between the two 8-head chunks).
__host__ __device__ constexpr uint32_t p_off(int h, int t) {
    return (uint32_t)((h >> 3) * 2048 + t * 16 + (h & 7) * 2);
}

// Maximum over the warp's 32 lanes of each of 16 values, by a transposing
// butterfly: each stage sends half of what a lane still holds, so 16 shuffles
// in all; lane l ends with the maximum of value l / 2.
__device__ __forceinline__ float warp_max16_scatter(const float (&v)[16], int lane) {
    float u[8], w[4], x[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        u[i] = fmaxf(b4 ? v[i + 8] : v[i], __shfl_xor_sync(0xffffffffu, b4 ? v[i] : v[i + 8], 16));
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = fmaxf(b3 ? u[i + 4] : u[i], __shfl_xor_sync(0xffffffffu, b3 ? u[i] : u[i + 4], 8));
#pragma unroll
    for (int i = 0; i < 2; ++i)
        x[i] = fmaxf(b2 ? w[i + 2] : w[i], __shfl_xor_sync(0xffffffffu, b2 ? w[i] : w[i + 2], 4));
    float y = fmaxf(b1 ? x[1] : x[0], __shfl_xor_sync(0xffffffffu, b1 ? x[0] : x[1], 2));
    return fmaxf(y, __shfl_xor_sync(0xffffffffu, y, 1));
}

struct Item {
    int b, g, t0, t1;  // tokens [t0, t1) of the cache rows of (b, g)
    int L;             // cache_len[b]: the row this call appends
};
__device__ __forceinline__ Item item_of(const AttnParams &p, int it) {
    Item w;
    const int bg = it / p.n_split, s = it - bg * p.n_split;
    w.b = bg / p.H_kv;
    w.g = bg - w.b * p.H_kv;
    const int L = p.cache_len[w.b];
    w.L = L;
    // Attended rows: 0 .. L (the new token was appended at row L).  A length
    // outside the checked range reads nothing past the bound.
    int end = min(L, min(p.kv_bound, p.max_len - 1)) + 1;
    if (L < 0) end = 0;
    w.t0 = s * p.split_tok;
    w.t1 = min(end, w.t0 + p.split_tok);
    if (w.t1 < w.t0) w.t1 = w.t0;
    return w;
}

// ------------------------------------------------------------ rope_append
// One block of 256 threads (thread = dim) per (b, kv head).
__global__ void __launch_bounds__(256) rope_append_kernel(const AttnParams p) {
    wait_for_predecessor();
    release_dependents();
    const int bg = blockIdx.x, b = bg / p.H_kv, g = bg - b * p.H_kv, d = threadIdx.x;
    const int L = p.cache_len[b];
    const bool ok = L >= 0 && L < p.max_len && L <= p.kv_bound;
    if (bg == 0) {
        // The call's status: a cache length out of range (the attend kernel,
        // which runs after this grid, overwrites it if one of its waits expires).
        __shared__ int bad;
        if (d == 0) bad = 0;
        __syncthreads();
        for (int i = d; i < p.batch; i += blockDim.x) {
            const int Li = p.cache_len[i];
            if (Li < 0 || Li >= p.max_len || Li > p.kv_bound) bad = 1;
        }
        __syncthreads();
        if (d == 0) p.status[0] = bad ? kBadLen : 0;
    }
    const int half = p.rot_dim >> 1;
    float c = 1.f, s = 0.f;
    int partner = d;
    float sign = 0.f;
    if (d < p.rot_dim && ok) {
        const int i = d < half ? d : d - half;
        // angle = L * theta^(-2i/rot_dim), in double so that large positions keep
        // their precision.
        const double ang = (double)L * exp2(-(2.0 * i / p.rot_dim) * p.log2_theta);
        double sd, cd;
        sincos(ang, &sd, &cd);
        c = (float)cd;
        s = (float)sd;
        partner = d < half ? d + half : d - half;
        sign = d < half ? -1.f : 1.f;  // x_i c - x_{i+h} s ;  x_{i+h} c + x_i s
    }
    auto rot = [&](const __nv_bfloat16 *row) {
        const float x = __bfloat162float(row[d]);
        if (d >= p.rot_dim) return x;
        return x * c + sign * __bfloat162float(row[partner]) * s;
    };
    if (ok) {
        const __nv_bfloat16 *kr = p.k + (int64_t)b * p.k_stride + g * D;
        const __nv_bfloat16 *vr = p.v + (int64_t)b * p.v_stride + g * D;
        const size_t crow = (((size_t)b * p.H_kv + g) * p.max_len + L) * D;
        p.k_cache[crow + d] = __float2bfloat16_rn(rot(kr));
        p.v_cache[crow + d] = vr[d];
    }
    unsigned char *qt = reinterpret_cast<unsigned char *>(p.q_tiles) + (size_t)bg * QTILE;
    for (int h = 0; h < NH; ++h) {
        float x = 0.f;
        if (h < p.n_rep && ok) x = rot(p.q + (int64_t)b * p.q_stride + (g * p.n_rep + h) * D);
        *reinterpret_cast<__nv_bfloat16 *>(qt + q_off(h, d >> 3) + (d & 7) * 2) =
            __float2bfloat16_rn(x);
    }
}

// ---------------------------------------------------------------- attend
__global__ void __launch_bounds__(NTHR, 1) attend_kernel(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    // The swizzled ring must start on a 1024-byte boundary.
    unsigned char *sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S_BAR);
    uint64_t *full = bars;           // [6] slot landed (TMA bytes, or the producer's arrival)
    uint64_t *empty = bars + 6;      // [6] slot consumed (MMA commit)
    uint64_t *bar_s = bars + 12;     // [2] S^T of a tile in TMEM
    uint64_t *bar_p = bars + 14;     // [2] P of a tile staged, O^T rescaled (4 warps)
    uint64_t *bar_o = bars + 16;     // [2] O^T += V^T P^T of a tile done (by P buffer)
    uint64_t *bar_q = bars + 18;     // [2] Q tile of an item landed
    uint64_t *bar_qfree = bars + 20; // [2] an item's S^T products done with its Q tile
    uint64_t *bar_aux = bars + 22;   // a partial V quarter landed (before its zero fill)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S_BAR + 192);
    float *red = reinterpret_cast<float *>(sm + S_RED);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t ring = sbase + S_RING;

    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    if (tid == 0) {
        for (int i = 0; i < NSLOT; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        mbar_init(bar_aux, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_s + i, 1);
            mbar_init(bar_p + i, 4);
            mbar_init(bar_q + i, 1);
            mbar_init(bar_qfree + i, 1);
            mbar_init(bar_o + i, 1);
        }
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tmem_slot;
    // The set-up above overlaps the kernel before (rope_append).  Everything
    // that reads what it wrote (the query tiles, the appended cache row, the
    // status word) comes after this grid's wait on it; the producer waits
    // only once it needs to (below), so that cache tiles wholly below the
    // appended row stream in meanwhile.  Dependents start when this grid
    // completes.
    if (warp != 4) wait_for_predecessor();
    auto fail = [&]() { atomicExch(p.status, kTimeout); };
    auto n_tiles_of = [&](const Item &w) { return (w.t1 - w.t0 + TILE - 1) / TILE; };

    if (warp == 4) {
        // ------------------------------------------------------ producer
        // Lane 0 streams each quarter of a tile (K0, K1, V0, V1: one d-half)
        // as two TMA box copies.  Slot uses are counted in one sequence (c)
        // over this CTA's non-empty items (nq), tiles and quarters; the MMA
        // warps walk the same sequence.  Past the end of a split's last,
        // partial tile the rows hold other tokens (or zeros past the tensor):
        // the softmax gives them zero weight, and in V the warp overwrites
        // them with zeros before it releases the slot, so that no value stored
        // there (a NaN in an unwritten cache row) can reach O.
        // Uses of each ring are counted per tile (tt: this CTA's tiles in
        // order), two per tile: use u = 2 tt + half sits in slot u % 3 of the
        // K ring (kind 0) or the V ring (kind 1), round u / 3.  n_iss: uses
        // issued per ring.
        int tt = 0, nq = 0, n_qcopy[2] = {0, 0}, n_aux = 0, n_iss[2] = {0, 0};
        bool ok = true, aux_pending = false, waited = false;
        if (lane == 0) {
            tma_prefetch_map(&p.tm_k);
            tma_prefetch_map(&p.tm_v);
        }
        auto ensure_waited = [&]() {
            if (waited) return;
            wait_for_predecessor();
            if (lane == 0) fence_proxy_async_global();  // the rows appended by the kernel before
            waited = true;
        };
        for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
            const Item w = item_of(p, it);
            const int nt = n_tiles_of(w);
            if (nt == 0) continue;
            const int qb = nq & 1;
            // The item's Q tile, once the item two back is done with the buffer.
            if (nq >= 2) {
                ensure_waited();
                if (lane == 0) ok = mbar_wait(bar_qfree + qb, (uint32_t)((nq - 2) >> 1) & 1u, kWaitNs);
            }
            ok = __shfl_sync(kFullMask, ok, 0);
            if (!ok) break;
            ++nq;
            bool q_issued = false;
            // The query tile comes from the kernel before: it is copied once the
            // producer has waited for that kernel, before the first quarter that
            // needs the wait or waits on a slot itself (whose release needs Q).
            auto issue_q = [&]() {
                ensure_waited();
                if (lane == 0) {
                    bulk_expect(bar_q + qb, QTILE);
                    bulk_copy(sm + S_Q + qb * QTILE,
                              reinterpret_cast<const unsigned char *>(p.q_tiles) +
                                  (size_t)(w.b * p.H_kv + w.g) * QTILE,
                              QTILE, bar_q + qb);
                }
                ++n_qcopy[qb];
                q_issued = true;
            };
            // Cache row of (b, g, token 0); below 2^31 (checked on the host).
            const int head_row = (w.b * p.H_kv + w.g) * p.max_len;
            for (int j = 0; j < nt && ok; ++j) {
                const int r0 = w.t0 + j * TILE;
                const int nvalid = min(TILE, w.t1 - r0);
                // A tile wholly below the appended row may stream in before the
                // wait on the kernel that appends it.
                const bool early = !waited && r0 + TILE <= w.L;
#pragma unroll 1
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int kind = q4 >> 1, use = 2 * tt + (q4 & 1);
                    const int slot = NRING * kind + use % NRING, round = use / NRING;
                    if (!q_issued && (round > 0 || !early)) issue_q();
                    if (round > 0 && lane == 0) ok = mbar_wait(empty + slot, (uint32_t)(round - 1) & 1u, kWaitNs);
                    ok = __shfl_sync(kFullMask, ok, 0);
                    if (!ok) break;
                    const uint32_t dst = ring + slot * SLOT;
                    const void *map = q4 < 2 ? static_cast<const void *>(&p.tm_k)
                                             : static_cast<const void *>(&p.tm_v);
                    const bool zero_tail = q4 >= 2 && nvalid < TILE;
                    uint64_t *bar = zero_tail ? bar_aux : full + slot;
                    if (lane == 0) {
                        bulk_expect(bar, SLOT);
                        tma_load_2d(dst, map, (q4 & 1) * 128, head_row + r0, bar);
                        tma_load_2d(dst + BOX, map, (q4 & 1) * 128 + 64, head_row + r0, bar);
                    }
                    if (!zero_tail) {
                        n_iss[kind] = use + 1;
                        continue;
                    }
                    aux_pending = true;
                    ok = __all_sync(kFullMask, mbar_wait(bar_aux, (uint32_t)n_aux & 1u, kWaitNs)) != 0;
                    if (!ok) break;
                    aux_pending = false;
                    ++n_aux;
                    // Rows nvalid .. 127 of both boxes: a row keeps its 128 bytes
                    // under the swizzle, which only permutes chunks inside it.
                    for (int i = nvalid * 8 + lane; i < TILE * 8; i += 32) {
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + i * 16), "r"(0u)
                                     : "memory");
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + BOX + i * 16),
                                     "r"(0u)
                                     : "memory");
                    }
                    fence_smem_to_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full + slot);
                    n_iss[kind] = use + 1;
                }
                if (ok) ++tt;
            }
            if (ok && !q_issued) issue_q();
        }
        if (!ok) ensure_waited();  // the status word is the previous kernel's before this
        if (!ok && lane == 0) {
            fail();
            // No copy may land after the CTA ends: the Q tiles, the last use
            // of every slot, a partial V quarter.
            for (int b = 0; b < 2; ++b)
                if (n_qcopy[b]) mbar_wait(bar_q + b, (uint32_t)(n_qcopy[b] - 1) & 1u, kWaitNs);
            for (int k = 0; k < 2; ++k)
                for (int u = n_iss[k] > NRING ? n_iss[k] - NRING : 0; u < n_iss[k]; ++u)
                    mbar_wait(full + NRING * k + u % NRING, (uint32_t)(u / NRING) & 1u, kWaitNs);
            if (aux_pending) mbar_wait(bar_aux, (uint32_t)n_aux & 1u, kWaitNs);
        }
        // Every arrival a tcgen05.commit owes this CTA's barriers must land
        // before the CTA ends, or it lands in shared memory that is another
        // CTA's by then: the MMA warps' releases of the last use of every slot
        // and of each query buffer's last item.  The phases waited for are the
        // last ones, so none can be lapped.
        if (lane == 0) {
            const uint64_t lim = ok ? kWaitNs : kDrainNs;
            for (int k = 0; k < 2; ++k)
                for (int u = n_iss[k] > NRING ? n_iss[k] - NRING : 0; u < n_iss[k]; ++u)
                    mbar_wait(empty + NRING * k + u % NRING, (uint32_t)(u / NRING) & 1u, lim);
            for (int b = 0; b < 2; ++b)
                if (n_qcopy[b]) mbar_wait(bar_qfree + b, (uint32_t)(n_qcopy[b] - 1) & 1u, lim);
        }
        __syncwarp();
    } else if (warp == 5 || warp == 6) {
        // ------------------------------------------- MMA issue, two threads
        // Warp 5 issues S^T = K Q^T of each tile as soon as its K has landed
        // (and the softmax is done with the S^T buffer it reuses); warp 6
        // issues O^T += V^T P^T of each tile as soon as its P and V are ready.
        // Neither waits behind the other's operands.
        if (lane == 0) {
            const bool s_role = warp == 5;
            const uint32_t ID_S = instr_desc<Kind::BF16>(128, NH, false, false);
            const uint32_t ID_O = instr_desc<Kind::BF16>(128, NH, true, true);
            bool ok = true;
            int jt = 0, nq = 0;
            for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
                const Item w = item_of(p, it);
                const int nt = n_tiles_of(w);
                if (nt == 0) continue;
                const int qb = nq & 1;
                if (s_role) ok = mbar_wait(bar_q + qb, (uint32_t)(nq >> 1) & 1u, kWaitNs);
                ++nq;
                for (int j = 0; j < nt && ok; ++j, ++jt) {
                    const int u0 = 2 * jt, u1 = u0 + 1;  // this tile's uses of each ring
                    if (s_role) {
                        // K halves in uses c, c + 1 of the ring; S^T buffer jt & 1
                        // was read by the softmax of tile jt - 2.
                        const int s0 = u0 % NRING, s1 = u1 % NRING;  // K ring
                        ok = mbar_wait(full + s0, (uint32_t)(u0 / NRING) & 1u, kWaitNs) &&
                             mbar_wait(full + s1, (uint32_t)(u1 / NRING) & 1u, kWaitNs) &&
                             (jt < 2 || mbar_wait(bar_p + (jt & 1), (uint32_t)((jt - 2) >> 1) & 1u, kWaitNs));
                        if (!ok) break;
                        fence_after_sync();
                        const uint32_t d = tm + TM_S + 16 * (jt & 1);
                        const uint32_t qa = sbase + S_Q + qb * QTILE;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t a0 = ring + (hh ? s1 : s0) * SLOT;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma<Kind::BF16>(
                                    d, smem_desc_sw128(a0 + (kk >> 2) * BOX + (kk & 3) * 32, 16, 1024),
                                    smem_desc(qa + hh * 4096 + kk * 512, 256, 128), ID_S, (hh | kk) ? 1u : 0u);
                        }
                        commit(smem_u32(bar_s + (jt & 1)));
                        commit(smem_u32(empty + s0));
                        commit(smem_u32(empty + s1));
                        if (j == nt - 1) commit(smem_u32(bar_qfree + qb));
                    } else {
                        const int v0 = NRING + u0 % NRING, v1 = NRING + u1 % NRING;  // V ring
                        ok = mbar_wait(bar_p + (jt & 1), (uint32_t)(jt >> 1) & 1u, kWaitNs) &&
                             mbar_wait(full + v0, (uint32_t)(u0 / NRING) & 1u, kWaitNs) &&
                             mbar_wait(full + v1, (uint32_t)(u1 / NRING) & 1u, kWaitNs);
                        if (!ok) break;
                        fence_after_sync();
                        const uint32_t pb = sbase + S_P + (jt & 1) * PTILE;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t a0 = ring + (hh ? v1 : v0) * SLOT;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma<Kind::BF16>(tm + TM_O + 16 * hh, smem_desc_sw128(a0 + kk * 2048, BOX, 1024),
                                                smem_desc(pb + kk * 256, 128, 2048), ID_O,
                                                (j > 0 || kk > 0) ? 1u : 0u);
                        }
                        commit(smem_u32(bar_o + (jt & 1)));
                        commit(smem_u32(empty + v0));
                        commit(smem_u32(empty + v1));
                    }
                }
            }
            if (!ok) fail();
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax warps
        // Every decision that leads to a named barrier is made by all four
        // warps together (an OR over the barrier), so none waits for a warp
        // that has stopped.
        //
        // The weights are taken against a reference maximum m_ref that only
        // moves when a tile's maximum passes it by more than kLazy (so P stays
        // below e^kLazy): then O^T and l are rescaled, which needs the previous
        // tile's O^T product finished.  Otherwise a tile waits only for the
        // product two tiles back, whose P buffer it reuses.
        constexpr float kLazy = 8.0f;
        const int t = tid;  // TMEM lane: token of the tile for S^T, dim for O^T
        const bool fused = p.n_split == 1;  // each item is a whole (b, kv head): no combine
        // Output element (query head h of the item's group, dim) as out's type.
        auto store_out = [&](const Item &w, int h, int dim, float y) {
            const int64_t i = (int64_t)w.b * p.out_stride + (w.g * p.n_rep + h) * D + dim;
            if (p.out_bf16)
                static_cast<__nv_bfloat16 *>(p.out)[i] = __float2bfloat16_rn(y);
            else
                static_cast<float *>(p.out)[i] = y;
        };
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        bool dead = false;
        int jt = 0;
        auto wait_o_lim = [&](int tile, uint64_t lim) {  // O^T product of `tile` done
            return mbar_wait(bar_o + (tile & 1), (uint32_t)(tile >> 1) & 1u, lim);
        };
        auto wait_o = [&](int tile) { return wait_o_lim(tile, kWaitNs); };
        for (int it = blockIdx.x; it < p.n_items && !dead; it += gridDim.x) {
            const Item w = item_of(p, it);
            const int nt = n_tiles_of(w);
            float *po = p.part_o + (size_t)it * NH * D;
            float *pml = p.part_ml + (size_t)it * NH * 2;
            if (nt == 0) {
                if (fused) {
                    for (int h = 0; h < p.n_rep; ++h)
                        for (int hd = 0; hd < 2; ++hd) store_out(w, h, 128 * hd + t, 0.f);
                } else if (t < NH) {
                    pml[2 * t] = -INFINITY;
                    pml[2 * t + 1] = 0.f;
                }
                continue;
            }
            float m_ref[NH], l_run[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                m_ref[h] = -INFINITY;
                l_run[h] = 0.f;
            }
            const int jt0 = jt;
            for (int j = 0; j < nt; ++j, ++jt) {
                const int nvalid = min(TILE, w.t1 - (w.t0 + j * TILE));
                bool ok = mbar_wait(bar_s + (jt & 1), (uint32_t)(jt >> 1) & 1u, kWaitNs);
                // P's buffer was last read by the product two tiles back.
                if (ok && jt >= 2) ok = wait_o(jt - 2);
                dead = group_sync_or(1, 128, !ok);
                if (dead) break;
                fence_after_sync();
                float s[NH];
                tmem_ld16(tm + lane_off + TM_S + 16 * (jt & 1), s);
                const bool valid = t < nvalid;
                // Columns past the group's query heads are padding: their
                // scores are -inf and their weights zero.
#pragma unroll
                for (int h = 0; h < NH; ++h) s[h] = valid && h < p.n_rep ? s[h] * p.scale : -INFINITY;
                {
                    const float mx = warp_max16_scatter(s, lane);
                    if (!(lane & 1)) red[warp * NH + (lane >> 1)] = mx;
                }
                group_sync_or(1, 128, false);
                // The tile's maxima over the four warps, then the weights
                // against the reference maxima (every thread takes the same
                // decisions, from the same red[]).
                float alpha[NH];
                bool moved = false;
#pragma unroll
                for (int k4 = 0; k4 < NH / 4; ++k4) {
                    const float4 r0 = *reinterpret_cast<const float4 *>(red + 4 * k4);
                    const float4 r1 = *reinterpret_cast<const float4 *>(red + NH + 4 * k4);
                    const float4 r2 = *reinterpret_cast<const float4 *>(red + 2 * NH + 4 * k4);
                    const float4 r3 = *reinterpret_cast<const float4 *>(red + 3 * NH + 4 * k4);
                    const float m4v[4] = {fmaxf(fmaxf(r0.x, r1.x), fmaxf(r2.x, r3.x)),
                                          fmaxf(fmaxf(r0.y, r1.y), fmaxf(r2.y, r3.y)),
                                          fmaxf(fmaxf(r0.z, r1.z), fmaxf(r2.z, r3.z)),
                                          fmaxf(fmaxf(r0.w, r1.w), fmaxf(r2.w, r3.w))};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int h = 4 * k4 + u;
                        const float m4 = m4v[u];
                        // The first tile of the item sets the reference (O^T
                        // starts from zero); later it moves only past kLazy.
                        const bool first = m_ref[h] == -INFINITY;
                        const bool mv = !first && m4 > m_ref[h] + kLazy;
                        const float a = __expf(m_ref[h] - m4);
                        alpha[h] = mv ? a : 1.f;
                        m_ref[h] = (first || mv) ? m4 : m_ref[h];
                        moved |= mv;
                        const float pv = (valid && m_ref[h] > -INFINITY) ? __expf(s[h] - m_ref[h]) : 0.f;
                        l_run[h] = l_run[h] * alpha[h] + pv;
                        s[h] = pv;
                    }
                }
                // P as bf16: this thread's token row, 16 heads in two 16-byte stores.
                {
                    unsigned char *pt = sm + S_P + (jt & 1) * PTILE;
                    uint32_t pk[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(s[2 * u], s[2 * u + 1]);
                        pk[u] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    *reinterpret_cast<uint4 *>(pt + p_off(0, t)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(pt + p_off(8, t)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
                // Rescale O^T (lane = dim) when a reference maximum moved: the
                // previous tile's product must have finished adding into it.
                // (`moved` is the same in every thread: it comes from red[].)
                if (moved) {
                    const bool ok2 = jt == jt0 || wait_o(jt - 1);
                    dead = group_sync_or(1, 128, !ok2);
                    if (dead) break;
                    fence_after_sync();
#pragma unroll
                    for (int hd = 0; hd < 2; ++hd) {
                        float o[16];
                        tmem_ld16(tm + lane_off + TM_O + 16 * hd, o);
                        uint32_t ou[16];
#pragma unroll
                        for (int h = 0; h < NH; ++h) ou[h] = __float_as_uint(o[h] * alpha[h]);
                        tmem_st16(tm + lane_off + TM_O + 16 * hd, ou);
                    }
                }
                fence_smem_to_async();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p + (jt & 1));
                group_sync_or(1, 128, false);  // red[] is rewritten next
            }
            if (dead) break;
            // Item done: the partial (m, l, O) of every query head of the group,
            // or, when the item is the whole (b, kv head), the gated output.
            const bool ok = wait_o(jt - 1);
            dead = group_sync_or(1, 128, !ok);
            if (dead) break;
            fence_after_sync();
            float o[2][16];
            tmem_ld16(tm + lane_off + TM_O, o[0]);
            tmem_ld16(tm + lane_off + TM_O + 16, o[1]);
            if (!fused) {
#pragma unroll
                for (int hd = 0; hd < 2; ++hd)
#pragma unroll
                    for (int h = 0; h < NH; ++h)
                        if (h < p.n_rep) po[(size_t)h * D + 128 * hd + t] = o[hd][h];
            }
            // l: sum over the 128 token lanes.
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float x = l_run[h];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(kFullMask, x, o);
                l_run[h] = x;
            }
            if (lane < NH) {
                float mine = l_run[0];
#pragma unroll
                for (int h = 1; h < NH; ++h) mine = lane == h ? l_run[h] : mine;
                red[warp * NH + lane] = mine;
            }
            group_sync_or(1, 128, false);
            if (fused) {
                // y = (O / l) * sigmoid(gate); thread t holds dims t and 128 + t.
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    if (h >= p.n_rep) break;
                    const float l = (red[h] + red[NH + h]) + (red[2 * NH + h] + red[3 * NH + h]);
#pragma unroll
                    for (int hd = 0; hd < 2; ++hd) {
                        const int dim = 128 * hd + t;
                        const float gt = __bfloat162float(
                            p.gate[(int64_t)w.b * p.gate_stride + (w.g * p.n_rep + h) * D + dim]);
                        store_out(w, h, dim, (l > 0.f ? o[hd][h] / l : 0.f) / (1.f + __expf(-gt)));
                    }
                }
            } else if (t < NH) {
                float m = m_ref[0];
#pragma unroll
                for (int h = 1; h < NH; ++h) m = t == h ? m_ref[h] : m;
                pml[2 * t] = m;
                pml[2 * t + 1] = (red[t] + red[NH + t]) + (red[2 * NH + t] + red[3 * NH + t]);
            }
            group_sync_or(1, 128, false);
        }
        if (dead && tid == 0) fail();
        // The O^T product two tiles before the last one is never waited for
        // on the way (its buffer is not reused): its commit must land too.
        if (jt >= 2) wait_o_lim(jt - 2, dead ? kDrainNs : kWaitNs);
    }

    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_free(tm, TM_COLS);
    }
}

// --------------------------------------------------------------- combine
// One block of 256 threads (thread = dim) per (b, kv head): every query head of
// the group merges its splits, y = (sum_s e^{m_s - m} O_s) / (sum_s e^{m_s - m} l_s)
// * sigmoid(gate).
template <typename TOUT>
__global__ void __launch_bounds__(256) combine_kernel(const AttnParams p) {
    wait_for_predecessor();
    release_dependents();
    const int bg = blockIdx.x, b = bg / p.H_kv, g = bg - b * p.H_kv, d = threadIdx.x;
    const size_t it0 = (size_t)bg * p.n_split;
    for (int h = 0; h < p.n_rep; ++h) {
        float m = -INFINITY;
        for (int s = 0; s < p.n_split; ++s) m = fmaxf(m, p.part_ml[((it0 + s) * NH + h) * 2]);
        float o = 0.f, l = 0.f;
        if (m > -INFINITY) {
            for (int s = 0; s < p.n_split; ++s) {
                const float ms = p.part_ml[((it0 + s) * NH + h) * 2];
                if (ms == -INFINITY) continue;
                const float f = __expf(ms - m);
                l += f * p.part_ml[((it0 + s) * NH + h) * 2 + 1];
                o += f * p.part_o[((it0 + s) * NH + h) * D + d];
            }
        }
        const int hq = g * p.n_rep + h;
        const float gt = __bfloat162float(p.gate[(int64_t)b * p.gate_stride + hq * D + d]);
        const float y = (l > 0.f ? o / l : 0.f) / (1.f + __expf(-gt));
        Elem<TOUT>::store1(static_cast<TOUT *>(p.out) + (int64_t)b * p.out_stride + hq * D + d, y);
    }
}

}  // namespace attn

size_t attn_workspace_bytes(int batch, int H_kv, int n_items) {
    size_t off = 256;  // status word
    off += (size_t)batch * H_kv * attn::QTILE;
    off = (off + 255) & ~(size_t)255;
    off += (size_t)n_items * attn::NH * attn::D * 4;
    off += (size_t)n_items * attn::NH * 2 * 4;
    return (off + 255) & ~(size_t)255;
}

// Cost of starting and finishing one work item (waiting for its last
// product, writing its partials), in tiles of 128 tokens.
#ifndef GDR_ATTN_ITEM_COST
#define GDR_ATTN_ITEM_COST 1.0
#endif

// Splits of the attended tokens per (b, kv head): the count that minimises the
// busiest CTA's work (tiles plus per-item cost) over the persistent grid.
void attn_plan(int batch, int H_kv, int kv_bound, int n_sm, int *n_split, int *split_tok) {
    const int tiles = (kv_bound + 1 + attn::TILE - 1) / attn::TILE;
    const int bg = batch * H_kv;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= tiles && s <= 64; ++s) {
        const int per = (tiles + s - 1) / s;  // tiles per split
        const long items = (long)bg * s;
        const long rounds = (items + n_sm - 1) / n_sm;
        const double cost = (double)rounds * (per + GDR_ATTN_ITEM_COST);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = s;
        }
    }
    *n_split = best;
    *split_tok = ((tiles + best - 1) / best) * attn::TILE;
}

namespace {

// A cache as `rows` rows of 256 bf16 (512-byte stride); boxes of 64 dims x
// 128 rows, 128-byte swizzle, rows past the end read as zero.
bool encode_cache_map(CUtensorMap *m, void *base, uint64_t rows) {
    return encode_bf16_2d(m, base, attn::D, rows, (uint64_t)attn::D * 2, 64, attn::TILE);
}

}  // namespace

cudaError_t launch_attn_decode(AttnParams p, void *workspace, int out_bf16, cudaStream_t s) {
    p.out_bf16 = out_bf16;
    const uint64_t rows = (uint64_t)p.batch * p.H_kv * p.max_len;
    if (!encode_cache_map(&p.tm_k, p.k_cache, rows) || !encode_cache_map(&p.tm_v, p.v_cache, rows))
        return cudaErrorInvalidValue;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    p.status = reinterpret_cast<int *>(ws);
    size_t off = 256;
    p.q_tiles = reinterpret_cast<__nv_bfloat16 *>(ws + off);
    off += (size_t)p.batch * p.H_kv * attn::QTILE;
    off = (off + 255) & ~(size_t)255;
    p.part_o = reinterpret_cast<float *>(ws + off);
    off += (size_t)p.n_items * attn::NH * attn::D * 4;
    p.part_ml = reinterpret_cast<float *>(ws + off);
    cudaError_t e;
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaGetLastError();
    e = cudaFuncSetAttribute(attn::attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)attn::S_ALLOC);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    auto launch = [&](auto kern, unsigned grid, unsigned block, size_t smem) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(block);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t r = cudaLaunchKernelEx(&cfg, kern, p);
        if (r != cudaSuccess) (void)cudaGetLastError();
        return r;
    };
    const unsigned bg = (unsigned)(p.batch * p.H_kv);
    if ((e = launch(attn::rope_append_kernel, bg, 256, 0)) != cudaSuccess) return e;
    const unsigned grid = (unsigned)(p.n_items < n_sm ? p.n_items : n_sm);
    if ((e = launch(attn::attend_kernel, grid, attn::NTHR, attn::S_ALLOC)) != cudaSuccess) return e;
    if (p.n_split == 1) return cudaSuccess;  // the attend kernel stored the output
    if (out_bf16)
        e = launch(attn::combine_kernel<__nv_bfloat16>, bg, 256, 0);
    else
        e = launch(attn::combine_kernel<float>, bg, 256, 0);
    return e;
}

// Fills the kernels' parameters from checked ABI arguments (strides resolved).
cudaError_t launch_attn_decode_args(const gdr_attn_decode_args *a, int n_split, int split_tok,
                                    void *workspace, cudaStream_t s) {
    AttnParams p = {};
    p.batch = a->batch;
    p.H_q = a->H_q;
    p.H_kv = a->H_kv;
    p.n_rep = a->H_q / a->H_kv;
    p.rot_dim = a->rot_dim;
    p.max_len = a->max_len;
    p.kv_bound = a->kv_bound;
    p.n_split = n_split;
    p.split_tok = split_tok;
    p.n_items = a->batch * a->H_kv * n_split;
    p.scale = a->scale;
    p.log2_theta = log2((double)a->rope_theta);
    p.q_stride = a->q_stride;
    p.gate_stride = a->gate_stride;
    p.k_stride = a->k_stride;
    p.v_stride = a->v_stride;
    p.out_stride = a->out_stride;
    p.q = static_cast<const __nv_bfloat16 *>(a->q);
    p.gate = static_cast<const __nv_bfloat16 *>(a->gate);
    p.k = static_cast<const __nv_bfloat16 *>(a->k);
    p.v = static_cast<const __nv_bfloat16 *>(a->v);
    p.k_cache = static_cast<__nv_bfloat16 *>(a->k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(a->v_cache);
    p.cache_len = a->cache_len;
    p.out = a->out;
    return launch_attn_decode(p, workspace, a->out_dtype == GDR_BF16, s);
}

}  // namespace gdr
