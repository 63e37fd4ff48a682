// gdr_api.cu -- the C ABI declared in include/gdr.h: argument checks on the
// host, then one kernel launch per call on the caller's stream.  Nothing here
// allocates, synchronises or keeps state between calls.
#include <stdint.h>
#include <string.h>

#include "gdr.h"
#include "gdr_common.cuh"

namespace gdr {
cudaError_t launch_decode(const DecodeParams &p, int d, int in_bf16, int out_bf16, cudaStream_t s);
cudaError_t launch_decode_multi(const DecodeParams &p, int d, int in_bf16, int out_bf16,
                                cudaStream_t s);
cudaError_t launch_rmsnorm_gated(const NormParams &p, int d, int o_bf16, int z_bf16, int y_bf16,
                                 cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillParams &p, int d, int chunk, int in_bf16,
                                int out_bf16, cudaStream_t s);
size_t prefill_tc_workspace_bytes(int n_seq);
cudaError_t launch_prefill_tc(const PrefillParams &p, void *workspace, int out_bf16,
                              cudaStream_t s);
size_t prefill_tc2p_workspace_bytes(int n_seq, int64_t n_chunks, int H_v, int n_seg);
int prefill_tc2p_segments(int n_seq, int H_v, int max_chunks, int n_sm);
cudaError_t launch_prefill_tc2p(const PrefillParams &p, const int32_t *cu_host, int n_seg,
                                void *workspace, int out_bf16, cudaStream_t s);
struct AttnParams;
size_t attn_workspace_bytes(int batch, int H_kv, int n_items);
void attn_plan(int batch, int H_kv, int kv_bound, int n_sm, int *n_split, int *split_tok);
cudaError_t launch_attn_decode_args(const gdr_attn_decode_args *a, int n_split, int split_tok,
                                    void *workspace, cudaStream_t s);
size_t moe_workspace_bytes(int n_tok, int n_exp, int top_k, int inter, int s_inter, int hidden);
size_t moe_route_smem_bytes(int n_tok, int n_exp, int top_k);
cudaError_t launch_moe_args(const gdr_moe_args *a, void *workspace, cudaStream_t s);
}  // namespace gdr

namespace {

using gdr::DecodeParams;
using gdr::NormParams;
using gdr::PrefillParams;

bool dtype_ok(int32_t t) { return t == GDR_F32 || t == GDR_BF16; }
size_t dtype_bytes(int32_t t) { return t == GDR_BF16 ? 2 : 4; }
bool head_dim_ok(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool aligned4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

// Row stride: 0 selects the packed default; otherwise it must not let rows
// overlap.  The byte stride must keep every row 16-byte aligned.
gdr_status resolve_stride(int64_t given, int64_t packed, size_t elem, int64_t *out) {
    if (given < 0) return GDR_ERR_INVALID_ARG;
    const int64_t s = given == 0 ? packed : given;
    if (s < packed) return GDR_ERR_INVALID_ARG;
    if (((uint64_t)s * elem) % 16 != 0) return GDR_ERR_MISALIGNED;
    *out = s;
    return GDR_OK;
}

gdr_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA; }

#define GDR_TRY(expr)                         \
    do {                                      \
        gdr_status _st = (expr);              \
        if (_st != GDR_OK) return _st;        \
    } while (0)

// Common shape checks of the mixer (decode and prefill).
gdr_status check_heads(int32_t H_k, int32_t H_v, int32_t d_k, int32_t d_v) {
    if (H_k <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0) return GDR_ERR_INVALID_ARG;
    if (H_v % H_k != 0) return GDR_ERR_INVALID_ARG;
    if (d_k != d_v || !head_dim_ok(d_k)) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

bool ranges_overlap(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + bn && b0 < a0 + an;
}

}  // namespace

extern "C" {

const char *gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG: invalid argument";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: shape, dtype or chunk not supported";
        case GDR_ERR_MISALIGNED: return "GDR_ERR_MISALIGNED: pointer or stride not 16-byte aligned";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE: workspace missing or too small";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: the CUDA runtime refused the launch";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a bounded device wait gave up";
        default: return "GDR_ERR_UNKNOWN: not a gdr_status value";
    }
}

int gdr_version(void) { return 100; }

// With GDR_GATE_FROM_RAW both per-head gate parameter arrays must be given.
static gdr_status check_raw_gate(int32_t flags, const float *A_log, const float *dt_bias) {
    if (!(flags & GDR_GATE_FROM_RAW)) return GDR_OK;
    if (!A_log || !dt_bias) return GDR_ERR_INVALID_ARG;
    if (!aligned4(A_log) || !aligned4(dt_bias)) return GDR_ERR_MISALIGNED;
    return GDR_OK;
}

// Shared validation of the decode arguments.  `slots` is the number of state
// rows the state buffers hold (batch for the one-token step).
static gdr_status decode_params(const gdr_decode_args *a, int64_t slots, DecodeParams *out) {
    if (a->batch < 0 || (a->flags & ~(GDR_DECODE_OVERLAP_STATE_LOAD | GDR_GATE_FROM_RAW)) != 0)
        return GDR_ERR_INVALID_ARG;
    GDR_TRY(check_raw_gate(a->flags, a->A_log, a->dt_bias));
    if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return GDR_ERR_INVALID_ARG;
    GDR_TRY(check_heads(a->H_k, a->H_v, a->d_k, a->d_v));
    if (a->batch == 0) return GDR_OK;
    if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->state_in || !a->state_out || !a->out)
        return GDR_ERR_INVALID_ARG;
    const int d = a->d_k;
    const size_t ein = dtype_bytes(a->in_dtype), eout = dtype_bytes(a->out_dtype);
    DecodeParams &p = *out;
    memset(&p, 0, sizeof(p));
    GDR_TRY(resolve_stride(a->q_stride, (int64_t)a->H_k * d, ein, &p.q_stride));
    GDR_TRY(resolve_stride(a->k_stride, (int64_t)a->H_k * d, ein, &p.k_stride));
    GDR_TRY(resolve_stride(a->v_stride, (int64_t)a->H_v * d, ein, &p.v_stride));
    GDR_TRY(resolve_stride(a->z_stride, (int64_t)a->H_v * d, ein, &p.z_stride));
    GDR_TRY(resolve_stride(a->out_stride, (int64_t)a->H_v * d, eout, &p.out_stride));
    GDR_TRY(resolve_stride(a->state_stride, (int64_t)a->H_v * d * d, 4, &p.state_stride));
    if (a->gb_stride < 0 || (a->gb_stride != 0 && a->gb_stride < a->H_v)) return GDR_ERR_INVALID_ARG;
    p.gb_stride = a->gb_stride == 0 ? a->H_v : a->gb_stride;
    const void *p16[] = {a->q, a->k, a->v, a->z, a->state_in, a->state_out, a->out};
    for (const void *ptr : p16)
        if (ptr && !aligned16(ptr)) return GDR_ERR_MISALIGNED;
    if (!aligned4(a->g) || !aligned4(a->beta) || (a->norm_w && !aligned4(a->norm_w)))
        return GDR_ERR_MISALIGNED;
    if ((int64_t)a->batch * a->H_v > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    if (a->state_in != a->state_out) {
        const size_t span = ((size_t)(slots - 1) * p.state_stride + (size_t)a->H_v * d * d) * 4;
        if (ranges_overlap(a->state_in, span, a->state_out, span)) return GDR_ERR_INVALID_ARG;
    }
    p.batch = a->batch;
    p.H_k = a->H_k;
    p.H_v = a->H_v;
    p.hv_per_hk = a->H_v / a->H_k;
    p.qk_l2norm = a->qk_l2norm ? 1 : 0;
    p.overlap_state_load = (a->flags & GDR_DECODE_OVERLAP_STATE_LOAD) ? 1 : 0;
    p.scale = a->scale;
    p.eps_l2 = a->eps_l2;
    p.eps_norm = a->eps_norm;
    p.q = a->q; p.k = a->k; p.v = a->v; p.z = a->z;
    p.g = a->g; p.beta = a->beta;
    p.state_in = a->state_in; p.state_out = a->state_out;
    p.norm_w = a->norm_w; p.out = a->out;
    p.n_tokens = 1;
    if (a->flags & GDR_GATE_FROM_RAW) {
        p.A_log = a->A_log;
        p.dt_bias = a->dt_bias;
    }
    return GDR_OK;
}

gdr_status gdr_decode_step(const gdr_decode_args *a, gdr_stream_t stream) {
    if (!a) return GDR_ERR_INVALID_ARG;
    DecodeParams p;
    GDR_TRY(decode_params(a, a->batch, &p));
    if (a->batch == 0) return GDR_OK;
    return from_cuda(gdr::launch_decode(p, a->d_k, a->in_dtype == GDR_BF16,
                                        a->out_dtype == GDR_BF16, (cudaStream_t)stream));
}

gdr_status gdr_decode_multi(const gdr_decode_multi_args *m, gdr_stream_t stream) {
    if (!m) return GDR_ERR_INVALID_ARG;
    const gdr_decode_args *a = &m->base;
    if (m->n_tokens < 1 || m->n_tokens > GDR_DECODE_MAX_TOKENS) return GDR_ERR_INVALID_ARG;
    if (m->state_slot && m->n_slots < 1) return GDR_ERR_INVALID_ARG;
    if ((m->state_slot && !aligned4(m->state_slot)) || (m->status && !aligned4(m->status)))
        return GDR_ERR_MISALIGNED;
    if ((int64_t)a->batch * m->n_tokens > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    DecodeParams p;
    GDR_TRY(decode_params(a, m->state_slot ? m->n_slots : a->batch, &p));
    if (a->batch == 0) return GDR_OK;
    p.n_tokens = m->n_tokens;
    p.n_slots = m->state_slot ? m->n_slots : a->batch;
    p.slot = m->state_slot;
    p.status = m->status;
    return from_cuda(gdr::launch_decode_multi(p, a->d_k, a->in_dtype == GDR_BF16,
                                              a->out_dtype == GDR_BF16, (cudaStream_t)stream));
}

gdr_status gdr_rmsnorm_gated(const gdr_norm_args *a, gdr_stream_t stream) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->rows < 0 || a->reserved != 0) return GDR_ERR_INVALID_ARG;
    if (!dtype_ok(a->o_dtype) || !dtype_ok(a->z_dtype) || !dtype_ok(a->out_dtype))
        return GDR_ERR_INVALID_ARG;
    if (a->d <= 0) return GDR_ERR_INVALID_ARG;
    if (!head_dim_ok(a->d)) return GDR_ERR_UNSUPPORTED;
    if (a->rows == 0) return GDR_OK;
    if (!a->o || !a->z || !a->out) return GDR_ERR_INVALID_ARG;
    NormParams p;
    memset(&p, 0, sizeof(p));
    GDR_TRY(resolve_stride(a->o_stride, a->d, dtype_bytes(a->o_dtype), &p.o_stride));
    GDR_TRY(resolve_stride(a->z_stride, a->d, dtype_bytes(a->z_dtype), &p.z_stride));
    GDR_TRY(resolve_stride(a->out_stride, a->d, dtype_bytes(a->out_dtype), &p.out_stride));
    if (!aligned16(a->o) || !aligned16(a->z) || !aligned16(a->out) ||
        (a->w && !aligned16(a->w)))
        return GDR_ERR_MISALIGNED;
    if (a->out == a->o && (a->out_dtype != a->o_dtype || p.out_stride != p.o_stride))
        return GDR_ERR_INVALID_ARG;
    p.rows = a->rows;
    p.eps = a->eps;
    p.o = a->o; p.z = a->z; p.w = a->w; p.out = a->out;
    return from_cuda(gdr::launch_rmsnorm_gated(p, a->d, a->o_dtype == GDR_BF16,
                                               a->z_dtype == GDR_BF16,
                                               a->out_dtype == GDR_BF16, (cudaStream_t)stream));
}

// Shape checks shared by the workspace query and the prefill call.  Fills
// *chunk_out with the chunk the launch will use.
static gdr_status check_prefill(const gdr_prefill_args *a, int *chunk_out) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->n_seq < 0 || a->n_tok < 0) return GDR_ERR_INVALID_ARG;
    if ((a->flags & ~GDR_GATE_FROM_RAW) != 0 || a->reserved != 0) return GDR_ERR_INVALID_ARG;
    GDR_TRY(check_raw_gate(a->flags, a->A_log, a->dt_bias));
    if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return GDR_ERR_INVALID_ARG;
    GDR_TRY(check_heads(a->H_k, a->H_v, a->d_k, a->d_v));
    int chunk = a->chunk;
    if (chunk == 0) chunk = 64;
    if (chunk != 16 && chunk != 32 && chunk != 64) return GDR_ERR_UNSUPPORTED;
    if (a->n_tok > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    if ((int64_t)a->n_seq * a->H_v > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    *chunk_out = chunk;
    return GDR_OK;
}

// bf16 inputs with d = 128 and chunk 64 run on the tensor cores.
static bool tensor_core_path(const gdr_prefill_args *a, int chunk) {
    return a->in_dtype == GDR_BF16 && a->d_k == 128 && chunk == 64;
}

// Chunks of 64 tokens over all sequences: exact from the host offsets when
// given, otherwise an upper bound.
static int64_t count_chunks(const gdr_prefill_args *a) {
    if (!a->cu_seqlens_host) return a->n_tok / 64 + a->n_seq;
    int64_t n = 0;
    for (int s = 0; s < a->n_seq; ++s) {
        const int64_t len = (int64_t)a->cu_seqlens_host[s + 1] - a->cu_seqlens_host[s];
        if (len > 0) n += (len + 63) / 64;
    }
    return n;
}

// The longest sequence's chunk count (an upper bound without host offsets).
static int max_chunks(const gdr_prefill_args *a) {
    if (!a->cu_seqlens_host) return (int)(a->n_tok / 64 + 1);
    int m = 0;
    for (int s = 0; s < a->n_seq; ++s) {
        const int n = (int)(((int64_t)a->cu_seqlens_host[s + 1] - a->cu_seqlens_host[s] + 63) / 64);
        m = n > m ? n : m;
    }
    return m;
}

static int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    return n;
}

static int prefill_segments(const gdr_prefill_args *a) {
    return gdr::prefill_tc2p_segments(a->n_seq, a->H_v, max_chunks(a), device_sm_count());
}

// The tensor-core path runs as two kernels (prep and recurrence, in segments
// that overlap when the recurrence leaves SMs idle) when the workspace holds
// the per-chunk records, else as one kernel that needs only the sequence order.
static size_t workspace_bytes(const gdr_prefill_args *a, int chunk) {
    if (!tensor_core_path(a, chunk)) return 0;
    return gdr::prefill_tc2p_workspace_bytes(a->n_seq, count_chunks(a), a->H_v,
                                             prefill_segments(a));
}

gdr_status gdr_prefill_workspace_size(const gdr_prefill_args *a, size_t *bytes) {
    if (!bytes) return GDR_ERR_INVALID_ARG;
    int chunk = 0;
    GDR_TRY(check_prefill(a, &chunk));
    *bytes = workspace_bytes(a, chunk);
    return GDR_OK;
}

}  // extern "C"

// The prefill behind gdr_prefill_chunked.  diag_wait_ns / diag_withhold: zero
// for every ordinary call; the wait-expiry self-test sets them (and then needs
// the two-kernel tensor-core path).
static gdr_status prefill_impl(const gdr_prefill_args *a, void *workspace, size_t ws_bytes,
                               gdr_stream_t stream, uint64_t diag_wait_ns, int diag_withhold) {
    int chunk = 0;
    GDR_TRY(check_prefill(a, &chunk));
    if (a->n_seq == 0) return GDR_OK;
    if (!a->cu_seqlens || !a->cu_seqlens_host) return GDR_ERR_INVALID_ARG;
    // The host copy of the offsets must start at 0, never fall, and end at n_tok.
    if (a->cu_seqlens_host[0] != 0 || a->cu_seqlens_host[a->n_seq] != a->n_tok)
        return GDR_ERR_INVALID_ARG;
    for (int s = 0; s < a->n_seq; ++s)
        if (a->cu_seqlens_host[s + 1] < a->cu_seqlens_host[s]) return GDR_ERR_INVALID_ARG;
    if (a->n_tok > 0 && (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->out))
        return GDR_ERR_INVALID_ARG;
    const int d = a->d_k;
    const size_t ein = dtype_bytes(a->in_dtype), eout = dtype_bytes(a->out_dtype);
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    GDR_TRY(resolve_stride(a->q_stride, (int64_t)a->H_k * d, ein, &p.q_stride));
    GDR_TRY(resolve_stride(a->k_stride, (int64_t)a->H_k * d, ein, &p.k_stride));
    GDR_TRY(resolve_stride(a->v_stride, (int64_t)a->H_v * d, ein, &p.v_stride));
    GDR_TRY(resolve_stride(a->z_stride, (int64_t)a->H_v * d, ein, &p.z_stride));
    GDR_TRY(resolve_stride(a->out_stride, (int64_t)a->H_v * d, eout, &p.out_stride));
    if (a->gb_stride < 0 || (a->gb_stride != 0 && a->gb_stride < a->H_v)) return GDR_ERR_INVALID_ARG;
    p.gb_stride = a->gb_stride == 0 ? a->H_v : a->gb_stride;
    const void *p16[] = {a->q, a->k, a->v, a->z, a->initial_state, a->final_state, a->out};
    for (const void *ptr : p16)
        if (ptr && !aligned16(ptr)) return GDR_ERR_MISALIGNED;
    if ((a->g && !aligned4(a->g)) || (a->beta && !aligned4(a->beta)) ||
        (a->norm_w && !aligned4(a->norm_w)) || !aligned4(a->cu_seqlens))
        return GDR_ERR_MISALIGNED;
    if (a->initial_state && a->final_state && a->initial_state != a->final_state) {
        const size_t span = (size_t)a->n_seq * a->H_v * d * d * 4;
        if (ranges_overlap(a->initial_state, span, a->final_state, span)) return GDR_ERR_INVALID_ARG;
    }
    const bool tc = tensor_core_path(a, chunk);
    const int64_t n_chunks = tc ? count_chunks(a) : 0;
    const size_t need_one = tc ? gdr::prefill_tc_workspace_bytes(a->n_seq) : 0;
    const int n_seg = tc ? prefill_segments(a) : 1;
    const size_t need_two = tc ? gdr::prefill_tc2p_workspace_bytes(a->n_seq, n_chunks, a->H_v, 1) : 0;
    const size_t need_seg =
        tc ? gdr::prefill_tc2p_workspace_bytes(a->n_seq, n_chunks, a->H_v, n_seg) : 0;
    if (tc) {
        if (!workspace || ws_bytes < need_one) return GDR_ERR_WORKSPACE;
        if (!aligned16(workspace)) return GDR_ERR_MISALIGNED;
    }
    p.n_seq = a->n_seq;
    p.H_k = a->H_k;
    p.H_v = a->H_v;
    p.hv_per_hk = a->H_v / a->H_k;
    p.qk_l2norm = a->qk_l2norm ? 1 : 0;
    p.scale = a->scale;
    p.eps_l2 = a->eps_l2;
    p.eps_norm = a->eps_norm;
    p.q = a->q; p.k = a->k; p.v = a->v; p.z = a->z;
    if (a->flags & GDR_GATE_FROM_RAW) {
        p.A_log = a->A_log;
        p.dt_bias = a->dt_bias;
    }
    p.g = a->g; p.beta = a->beta;
    p.cu_seqlens = a->cu_seqlens;
    p.initial_state = a->initial_state;
    p.final_state = a->final_state;
    p.norm_w = a->norm_w;
    p.out = a->out;
    if (diag_withhold) {
        if (!tc) return GDR_ERR_UNSUPPORTED;
        if (ws_bytes < need_two) return GDR_ERR_WORKSPACE;
        p.wait_ns = diag_wait_ns;
        p.withhold_first_k = 1;
    }
    if (tc && ws_bytes >= need_two)
        return from_cuda(gdr::launch_prefill_tc2p(p, a->cu_seqlens_host,
                                                  ws_bytes >= need_seg ? n_seg : 1, workspace,
                                                  a->out_dtype == GDR_BF16, (cudaStream_t)stream));
    if (tc)
        return from_cuda(gdr::launch_prefill_tc(p, workspace, a->out_dtype == GDR_BF16,
                                                (cudaStream_t)stream));
    return from_cuda(gdr::launch_prefill_simt(p, d, chunk, a->in_dtype == GDR_BF16,
                                              a->out_dtype == GDR_BF16, (cudaStream_t)stream));
}

extern "C" {

gdr_status gdr_prefill_chunked(const gdr_prefill_args *a, void *workspace, size_t ws_bytes,
                               gdr_stream_t stream) {
    return prefill_impl(a, workspace, ws_bytes, stream, 0, 0);
}

gdr_status gdr_prefill_selftest_wait_expiry(const gdr_prefill_args *a, void *workspace,
                                            size_t ws_bytes, uint64_t wait_ns,
                                            gdr_stream_t stream) {
    if (wait_ns < GDR_SELFTEST_MIN_WAIT_NS || wait_ns > GDR_SELFTEST_MAX_WAIT_NS)
        return GDR_ERR_INVALID_ARG;
    if (!a || a->n_seq == 0) return GDR_ERR_INVALID_ARG;
    return prefill_impl(a, workspace, ws_bytes, stream, wait_ns, 1);
}

}  // extern "C"

// ------------------------------------------------------ gated attention

// Shape and pointer checks of the attention step; fills the work split.
static gdr_status attn_check(const gdr_attn_decode_args *a, int *n_split, int *split_tok,
                             size_t *ws_bytes) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->batch < 0 || a->H_q <= 0 || a->H_kv <= 0 || a->d <= 0) return GDR_ERR_INVALID_ARG;
    if (a->H_q % a->H_kv != 0) return GDR_ERR_INVALID_ARG;
    if (a->H_q / a->H_kv > 16 || a->d != 256) return GDR_ERR_UNSUPPORTED;
    if (a->rot_dim < 0 || a->rot_dim > a->d || (a->rot_dim & 1)) return GDR_ERR_INVALID_ARG;
    if (a->max_len < 1 || a->kv_bound < 0 || a->kv_bound >= a->max_len) return GDR_ERR_INVALID_ARG;
    if (!dtype_ok(a->out_dtype)) return GDR_ERR_INVALID_ARG;
    if (!(a->rope_theta > 0.f)) return GDR_ERR_INVALID_ARG;
    // Cache rows are addressed with 32-bit signed coordinates.
    if ((int64_t)a->batch * a->H_kv * a->max_len > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    gdr::attn_plan(a->batch, a->H_kv, a->kv_bound, device_sm_count(), n_split, split_tok);
    if ((int64_t)a->batch * a->H_kv * *n_split > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
    *ws_bytes = gdr::attn_workspace_bytes(a->batch, a->H_kv, a->batch * a->H_kv * *n_split);
    return GDR_OK;
}

extern "C" {

gdr_status gdr_attn_decode_workspace_size(const gdr_attn_decode_args *a, size_t *bytes) {
    if (!bytes) return GDR_ERR_INVALID_ARG;
    int n_split = 0, split_tok = 0;
    size_t need = 0;
    GDR_TRY(attn_check(a, &n_split, &split_tok, &need));
    *bytes = a->batch == 0 ? 0 : need;
    return GDR_OK;
}

gdr_status gdr_attn_decode_step(const gdr_attn_decode_args *a, void *workspace,
                                size_t ws_bytes, gdr_stream_t stream) {
    int n_split = 0, split_tok = 0;
    size_t need = 0;
    GDR_TRY(attn_check(a, &n_split, &split_tok, &need));
    if (a->batch == 0) return GDR_OK;
    if (!a->q || !a->gate || !a->k || !a->v || !a->k_cache || !a->v_cache || !a->cache_len ||
        !a->out)
        return GDR_ERR_INVALID_ARG;
    const int64_t d = a->d;
    int64_t qs, gs, ks, vs, os;
    GDR_TRY(resolve_stride(a->q_stride, a->H_q * d, 2, &qs));
    GDR_TRY(resolve_stride(a->gate_stride, a->H_q * d, 2, &gs));
    GDR_TRY(resolve_stride(a->k_stride, a->H_kv * d, 2, &ks));
    GDR_TRY(resolve_stride(a->v_stride, a->H_kv * d, 2, &vs));
    GDR_TRY(resolve_stride(a->out_stride, a->H_q * d, dtype_bytes(a->out_dtype), &os));
    const void *p16[] = {a->q, a->gate, a->k, a->v, a->k_cache, a->v_cache, a->out};
    for (const void *ptr : p16)
        if (!aligned16(ptr)) return GDR_ERR_MISALIGNED;
    if (!aligned4(a->cache_len)) return GDR_ERR_MISALIGNED;
    if (!workspace || ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDR_ERR_MISALIGNED;
    gdr_attn_decode_args r = *a;
    r.q_stride = qs;
    r.gate_stride = gs;
    r.k_stride = ks;
    r.v_stride = vs;
    r.out_stride = os;
    return from_cuda(gdr::launch_attn_decode_args(&r, n_split, split_tok, workspace,
                                                  (cudaStream_t)stream));
}

}  // extern "C"

// ------------------------------------------------------------------ MoE

static gdr_status moe_check(const gdr_moe_args *a) {
    if (!a) return GDR_ERR_INVALID_ARG;
    if (a->n_tok < 0 || a->hidden <= 0 || a->n_exp <= 0 || a->inter <= 0 || a->reserved != 0)
        return GDR_ERR_INVALID_ARG;
    if (a->top_k < 1 || a->top_k > a->n_exp) return GDR_ERR_INVALID_ARG;
    if (a->top_k > 32 || a->n_tok > 4096 || a->n_exp > 1024) return GDR_ERR_UNSUPPORTED;
    if (a->ws_gate_up && a->s_inter <= 0) return GDR_ERR_INVALID_ARG;
    if (a->hidden % 8 || a->inter % 8 || (a->ws_gate_up && a->s_inter % 8)) return GDR_ERR_UNSUPPORTED;
    if (a->inter > 1024 || (a->ws_gate_up && a->s_inter > 1024)) return GDR_ERR_UNSUPPORTED;
    if (!dtype_ok(a->out_dtype)) return GDR_ERR_INVALID_ARG;
    if (gdr::moe_route_smem_bytes(a->n_tok, a->n_exp, a->top_k) > 200 * 1024) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

extern "C" {

gdr_status gdr_moe_workspace_size(const gdr_moe_args *a, size_t *bytes) {
    if (!bytes) return GDR_ERR_INVALID_ARG;
    GDR_TRY(moe_check(a));
    *bytes = a->n_tok == 0 ? 0
                           : gdr::moe_workspace_bytes(a->n_tok, a->n_exp, a->top_k, a->inter,
                                                      a->ws_gate_up ? a->s_inter : 0, a->hidden);
    return GDR_OK;
}

gdr_status gdr_moe_decode(const gdr_moe_args *a, void *workspace, size_t ws_bytes,
                          gdr_stream_t stream) {
    GDR_TRY(moe_check(a));
    if (a->n_tok == 0) return GDR_OK;
    if (!a->x || !a->w_router || !a->w_gate_up || !a->w_down || !a->out) return GDR_ERR_INVALID_ARG;
    if (a->ws_gate_up && (!a->ws_down || !a->w_sgate)) return GDR_ERR_INVALID_ARG;
    int64_t xs, os;
    GDR_TRY(resolve_stride(a->x_stride, a->hidden, 2, &xs));
    GDR_TRY(resolve_stride(a->out_stride, a->hidden, dtype_bytes(a->out_dtype), &os));
    const void *p16[] = {a->x, a->w_router, a->w_gate_up, a->w_down, a->ws_gate_up, a->ws_down,
                         a->w_sgate, a->out};
    for (const void *ptr : p16)
        if (ptr && !aligned16(ptr)) return GDR_ERR_MISALIGNED;
    if ((a->topk_idx && !aligned4(a->topk_idx)) || (a->topk_w && !aligned4(a->topk_w)))
        return GDR_ERR_MISALIGNED;
    const size_t need = gdr::moe_workspace_bytes(a->n_tok, a->n_exp, a->top_k, a->inter,
                                                 a->ws_gate_up ? a->s_inter : 0, a->hidden);
    if (!workspace || ws_bytes < need) return GDR_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDR_ERR_MISALIGNED;
    gdr_moe_args r = *a;
    r.x_stride = xs;
    r.out_stride = os;
    return from_cuda(gdr::launch_moe_args(&r, workspace, (cudaStream_t)stream));
}

}  // extern "C"
