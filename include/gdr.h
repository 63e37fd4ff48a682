/*
 * gdr.h -- C ABI of the Gated DeltaNet (gated delta rule) token mixer for
 * NVIDIA B200 (sm_100a).
 *
 * The mixer: the pages name it as the "gated delta rule" recurrence with an
 * RMSNormGated output (Qwen3.5 Chat guide, soniqo.audio/de/guides/chat,
 * section "Architektur"), 18 of the 24 layers of Qwen3.5-0.8B; on the Core AI
 * Qwen3.6-35B-A3B card (first section) it has 16 key heads, each serving two
 * of its 32 value heads (GVA).  Its state is a
 * fixed-size matrix per head, so memory does not grow with context (Swiftlet
 * post, "How It Works").  The equations follow the published gated delta rule
 * (Gated Delta Networks, Yang, Kautz, Hatamizadeh, ICLR 2025).  Per sequence,
 * per value head h_v with key head h_k = floor(h_v * H_k / H_v):
 *
 *     q_hat = scale * q / sqrt(|q|^2 + eps_l2),   k_hat = k / sqrt(|k|^2 + eps_l2)
 *     S_t   = exp(g_t) S_{t-1} (I - beta_t k_hat k_hat^T) + beta_t v_t k_hat^T
 *     o_t   = S_t q_hat
 *     y_t   = o_t / sqrt(mean(o_t^2) + eps_norm) * w * z_t * sigmoid(z_t)
 *
 * S is d_v x d_k fp32, row-major ([d_v][d_k]: row i is value dimension i).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Memory.  Every pointer is device memory owned by the caller unless its
 *    comment says host.  The library allocates nothing and keeps no state
 *    between calls; it only reads and writes the buffers it is given.
 *  - Streams.  Work is queued on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and the call returns without waiting for it.
 *  - Errors.  Arguments are checked on the host before anything is queued; a
 *    failed check returns its status and queues nothing.  A launch the CUDA
 *    runtime refuses returns GDR_ERR_CUDA (the runtime's own error is cleared
 *    and not reported further).  Faults inside a running kernel surface on the
 *    stream like any CUDA error.  No C++ exception crosses this ABI.
 *  - Layout.  Activations are token-major and head-contiguous: element
 *    (row, head, i) of a [rows, H, d] tensor is at row*row_stride + head*d + i,
 *    where row_stride (in elements) defaults to H*d when passed as 0.
 *  - Alignment.  Pointers to rows of d values (q, k, v, z, out, o, states,
 *    and the RMSNormGated weight w) must be 16-byte aligned and their row
 *    strides multiples of 16 bytes; g, beta, cu_seqlens and the mixer's
 *    norm_w need 4-byte alignment (GDR_ERR_MISALIGNED otherwise).
 *  - Threads.  Calls are independent and may be made from several host
 *    threads at once.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdr_status {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size */
    GDR_ERR_UNSUPPORTED = 2, /* valid, but no kernel for this shape / dtype / chunk */
    GDR_ERR_MISALIGNED = 3,  /* pointer or stride breaks the 16-byte rule */
    GDR_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
    GDR_ERR_CUDA = 5,        /* the CUDA runtime refused a launch or query */
    GDR_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up */
} gdr_status;

typedef enum gdr_dtype { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/* Opaque CUDA stream (binary-compatible with cudaStream_t). */
typedef struct CUstream_st *gdr_stream_t;

/* ------------------------------------------------------------------------
 * One decode step: every sequence in the batch advances by one token.
 *
 * The pages' decoder keeps the layer state between calls and moves forward by
 * a single token each time it is invoked (Core ML card for Qwen3.5-0.8B,
 * section "Model"); the state lives across the generation loop (same card,
 * "Usage").  Here the caller owns the state buffer and this call updates it.
 *
 *   q, k       [batch, H_k, d_k]   in_dtype    row strides q_stride, k_stride
 *   v, z       [batch, H_v, d_v]   in_dtype    row strides v_stride, z_stride
 *   g, beta    [batch, H_v]        fp32        row stride  gb_stride (both)
 *   state_in   [batch, H_v, d_v, d_k] fp32    batch stride state_stride
 *   state_out  same layout; may be the same buffer as state_in (in place).
 *              Any other overlap between them is undefined.
 *   norm_w     [d_v] fp32, shared by all heads; NULL means all ones
 *   out        [batch, H_v, d_v]   out_dtype   row stride out_stride
 *
 *   z == NULL skips the output gate: out receives o_t itself.
 *   qk_l2norm == 0 uses q and k as given (the caller has normalised them);
 *   `scale` still multiplies q.  g = -inf is allowed (state reset).
 *   Supported: d_k == d_v in {16, 32, 64, 128}, H_v a multiple of H_k.
 *   batch == 0 is a no-op.  state_stride must be >= H_v*d_v*d_k (0 = that).
 *   flags: GDR_DECODE_OVERLAP_STATE_LOAD, GDR_GATE_FROM_RAW (below) or 0;
 *   other bits are rejected with GDR_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
/* gdr_decode_args.flags
 *
 * GDR_DECODE_OVERLAP_STATE_LOAD: the decode kernel is launched as a
 * programmatic dependent of the kernel queued just before it on the stream and
 * may start reading the state while that kernel is still finishing (q, k, v,
 * z, g, beta are always read after it has finished).  Set it only when that
 * preceding kernel does not write this call's state -- e.g. consecutive
 * decode calls of different layers.  Kernels of this library let their own
 * dependents start only after everything queued before them has finished, so
 * a chain of such calls is safe as long as each call's immediate predecessor
 * leaves its state alone.  Without the flag the state is read only after
 * the preceding kernel has finished. */
#define GDR_DECODE_OVERLAP_STATE_LOAD 1

/* gdr_decode_args.flags and gdr_prefill_args.flags
 *
 * GDR_GATE_FROM_RAW: g and beta hold the raw per-token gate projections a and
 * b instead of the gate values; the kernel forms, per value head h,
 *     g    = -exp(A_log[h]) * softplus(a + dt_bias[h])
 *     beta = sigmoid(b)
 * from the [H_v] fp32 arrays A_log and dt_bias, which must then be given.
 * The pages do not spell this parameterisation out; it is the one of the
 * published Gated DeltaNet and Mamba-2 layers, and saves the caller a
 * separate elementwise pass over g and beta. */
#define GDR_GATE_FROM_RAW 2

typedef struct gdr_decode_args {
    int32_t batch, H_k, H_v, d_k, d_v;
    int32_t in_dtype;  /* gdr_dtype of q, k, v, z */
    int32_t out_dtype; /* gdr_dtype of out */
    int32_t qk_l2norm; /* 1: normalise q, k in the kernel */
    float scale;       /* multiplies q_hat; 1.0 for the plain o_t = S_t q_t */
    float eps_l2;      /* under the square root of the q/k norms */
    float eps_norm;    /* added to mean(o^2) in RMSNormGated */
    int32_t flags;     /* 0, or GDR_DECODE_OVERLAP_STATE_LOAD | GDR_GATE_FROM_RAW */
    int64_t q_stride, k_stride, v_stride, z_stride, gb_stride, out_stride;
    int64_t state_stride;
    const void *q, *k, *v, *z;
    const float *g, *beta;
    const float *state_in;
    float *state_out;
    const float *norm_w;
    void *out;
    const float *A_log, *dt_bias; /* [H_v] fp32, with GDR_GATE_FROM_RAW only */
} gdr_decode_args;

gdr_status gdr_decode_step(const gdr_decode_args *args, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * Several decode tokens per sequence in one call, with optional state slots.
 *
 * The same recurrence as gdr_decode_step, applied to n_tokens consecutive
 * tokens of every sequence; the Swiftlet post checks that advancing token by
 * token matches processing the tokens together ("Correctness & Validation").
 * The state is read once and written once per call, whatever n_tokens, which
 * is the whole point: per token it costs 1/n_tokens of a single step's state
 * traffic.  State slots let a server keep sequences' states in a pool and
 * advance any subset of them (the caller owns the state across the generation
 * loop: Core ML card for Qwen3.5-0.8B, "Usage").
 *
 *   base       as for gdr_decode_step, except that every token-indexed tensor
 *              (q, k, v, z, g, beta, out) holds base.batch * n_tokens rows:
 *              row b * n_tokens + t is token t of sequence b (same row strides).
 *              base.batch is the number of sequences.
 *   n_tokens   1 .. GDR_DECODE_MAX_TOKENS tokens per sequence, applied in order.
 *   state_slot NULL: sequence b uses state row b, as in gdr_decode_step.
 *              Otherwise a device array of base.batch int32: sequence b reads
 *              and writes state row state_slot[b] of state_in / state_out (row
 *              stride base.state_stride).  Slots must be distinct within a call.
 *   n_slots    with state_slot: the number of state rows the buffers hold
 *              (>= 1).  A slot outside [0, n_slots) leaves that sequence's state
 *              and outputs untouched and, if `status` is given, sets *status to
 *              GDR_ERR_INVALID_ARG on the device; other sequences proceed.
 *   status     optional device int32, written only on such an error.
 * With state_slot the slot table is read after the preceding kernel on the
 * stream has finished, so it may be produced by that kernel.
 * ------------------------------------------------------------------------ */
#define GDR_DECODE_MAX_TOKENS 8

typedef struct gdr_decode_multi_args {
    gdr_decode_args base;
    int32_t n_tokens;
    int32_t n_slots;
    const int32_t *state_slot;
    int32_t *status;
} gdr_decode_multi_args;

gdr_status gdr_decode_multi(const gdr_decode_multi_args *args, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * Chunked prefill over packed variable-length sequences.
 *
 * The pages' Core ML build pairs a prefill model with the decode model
 * (Qwen3.5 Chat guide, "Architektur"), and the Swiftlet post checks that
 * incremental decoding matches whole-sequence processing ("Correctness &
 * Validation").  This call processes whole prompts with the chunkwise
 * (WY / UT transform) form of the same recurrence: within a chunk of C tokens,
 *   A_rs  = beta_r exp(gamma_r - gamma_s) (k_r . k_s)            s < r
 *   Delta = (I + A)^{-1} (diag(beta) V - diag(beta e^gamma) K S_0^T)
 *   O     = diag(e^gamma) Q S_0^T + (exp(gamma_r - gamma_s) q_r . k_s)_{s<=r} Delta
 *   S_C   = e^{gamma_C} S_0 + Delta^T diag(e^{gamma_C - gamma}) K
 * with gamma the running sum of g inside the chunk.  The result equals the
 * token-by-token recurrence up to rounding.
 *
 *   q, k        [n_tok, H_k, d_k]  in_dtype   row strides q_stride, k_stride
 *   v, z        [n_tok, H_v, d_v]  in_dtype   row strides v_stride, z_stride
 *   g, beta     [n_tok, H_v]       fp32       row stride gb_stride
 *   cu_seqlens       device int32 [n_seq + 1]: sequence s is tokens
 *                    [cu_seqlens[s], cu_seqlens[s+1]); chunks never cross it.
 *   cu_seqlens_host  HOST int32 [n_seq + 1], the same values; read during the
 *                    call (validation, work ordering), not kept.
 *   initial_state    [n_seq, H_v, d_v, d_k] fp32, or NULL for zeros
 *   final_state      same layout, or NULL; may equal initial_state (in place)
 *   norm_w, out, z, qk_l2norm, scale, eps_*: as for gdr_decode_step;
 *   out is [n_tok, H_v, d_v] with row stride out_stride.
 *
 *   g is clamped below at -64 inside chunks (exp(-64) ~ 1.6e-28): the chunk
 *   form takes differences of running sums of g, which a g of -inf would turn
 *   into NaN.  Empty sequences are allowed (their final state = initial state).
 *   chunk: 16, 32 or 64, or 0 for the library's choice.
 *   Supported: d_k == d_v in {16, 32, 64, 128}; bf16 inputs with d = 128 and
 *   chunk 64 (or 0) run on the tensor cores, everything else on CUDA cores
 *   (chunk 64 with d = 128 needs the tensor-core path).
 *   workspace: device memory, 16-byte aligned, owned by the caller, free for
 *   reuse once the queued work has finished.  gdr_prefill_workspace_size()
 *   bytes select the fastest variant: on the tensor-core path that is two
 *   kernels, the first computing every chunk's state-independent part at
 *   once into the workspace (about 65 KB per chunk of 64 tokens and value
 *   head).  A tensor-core call given less, but at least
 *   (16 + 4 * n_seq) rounded up to 256 bytes, runs as one kernel instead
 *   (same results up to rounding, less parallel).  Below that:
 *   GDR_ERR_WORKSPACE.  When the size is non-zero its first 4 bytes (int32) hold,
 *   once the work has finished, 0 or GDR_ERR_TIMEOUT if a bounded device-side
 *   wait gave up (the outputs of that call are then incomplete).
 * ------------------------------------------------------------------------ */
typedef struct gdr_prefill_args {
    int32_t n_seq, H_k, H_v, d_k, d_v;
    int32_t chunk;
    int32_t in_dtype, out_dtype;
    int32_t qk_l2norm;
    float scale, eps_l2, eps_norm;
    int64_t n_tok;
    int64_t q_stride, k_stride, v_stride, z_stride, gb_stride, out_stride;
    const void *q, *k, *v, *z;
    const float *g, *beta;
    const int32_t *cu_seqlens;
    const int32_t *cu_seqlens_host;
    const float *initial_state;
    float *final_state;
    const float *norm_w;
    void *out;
    int32_t flags;                /* 0 or GDR_GATE_FROM_RAW; other bits are rejected */
    int32_t reserved;             /* 0 */
    const float *A_log, *dt_bias; /* [H_v] fp32, with GDR_GATE_FROM_RAW only */
} gdr_prefill_args;

/* Bytes of workspace gdr_prefill_chunked needs for these arguments (the same
 * struct that will be passed to it; only sizes, dtypes and chunk are read).
 * Returns 0 and sets *bytes on success; an invalid or unsupported shape
 * returns the status gdr_prefill_chunked would. */
gdr_status gdr_prefill_workspace_size(const gdr_prefill_args *args, size_t *bytes);

gdr_status gdr_prefill_chunked(const gdr_prefill_args *args, void *workspace,
                               size_t workspace_bytes, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * gdr_prefill_chunked without a caller-provided workspace.
 *
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory where they run the prefill -- a runtime
 * that hands all free device memory to its own pools at start-up, or a plain
 * C caller embedding the library with no memory manager.  It allocates
 * nothing: the workspace is a fixed array inside the library's own device
 * memory (about 16 KB, held by every GPU that loads the library until the
 * process exits), and calls no cudaMalloc or cudaFree.
 *
 *   Arguments, results and errors are those of gdr_prefill_chunked, plus:
 *   n_seq > GDR_PREFILL_NOALLOC_MAX_SEQS returns GDR_ERR_WORKSPACE (nothing
 *   is queued); GDR_ERR_CUDA if the array's device address cannot be found.
 *   The first call on a device looks the array's address up for that device
 *   (the device must be current); make that first call before any stream
 *   capture.
 *   Every call shares the one array per device: calls that may run at the
 *   same time on the GPU (different streams, or host threads, without
 *   ordering between them) race on it and must not be made.  Each call
 *   rewrites everything it reads from the array before reading it, so
 *   results never depend on an earlier call.
 *   The looked-up address belongs to the device's primary context and is kept
 *   for the life of the process: after cudaDeviceReset, or from a context the
 *   caller created itself, this entry point must not be used.
 *   The array's first 4 bytes are the status word gdr_prefill_chunked writes
 *   to its workspace; gdr_prefill_noalloc_status reads it back.
 * ------------------------------------------------------------------------ */
#define GDR_PREFILL_NOALLOC_MAX_SEQS 4096

gdr_status gdr_prefill_chunked_noalloc(const gdr_prefill_args *args, gdr_stream_t stream);

/* Queue on `stream` a copy of the current device's status word of
 * gdr_prefill_chunked_noalloc (an int32: 0, or GDR_ERR_TIMEOUT if a bounded
 * device-side wait of the last call on this device gave up, its outputs then
 * being incomplete) into `status`, which may be device memory or host memory
 * (with pageable host memory the copy completes before the call returns).
 * Read it once the prefill's work on the stream has finished.  Like the
 * prefill, it has no counterpart in the pages and allocates nothing.
 * Returns GDR_ERR_INVALID_ARG for a NULL `status`, GDR_ERR_CUDA if the copy
 * cannot be queued. */
gdr_status gdr_prefill_noalloc_status(int32_t *status, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics: the expiry path of the prefill's bounded device waits.
 *
 * The pages have no counterpart; this exists so that a test can watch the
 * failure handling of the tensor-core prefill without faulting or hanging a
 * GPU.  Every device-side wait of that prefill gives up after a deadline,
 * records GDR_ERR_TIMEOUT in the workspace status word, waits (again bounded)
 * for its own copies in flight, frees its tensor memory and returns.  This
 * call runs gdr_prefill_chunked's two-kernel tensor-core path with the
 * recurrence's waits limited to `wait_ns` nanoseconds and each (sequence,
 * value head)'s first key tile never delivered, so those waits run out:
 * once the work has finished, the status word reads GDR_ERR_TIMEOUT, the
 * outputs and final states are incomplete (unspecified), and the device is
 * left usable for the calls that follow.
 *
 *   args, workspace, workspace_bytes: as for gdr_prefill_chunked; the shape
 *   must take the tensor-core path (else GDR_ERR_UNSUPPORTED) with a
 *   workspace of at least gdr_prefill_workspace_size() bytes (else
 *   GDR_ERR_WORKSPACE), and n_seq >= 1.
 *   wait_ns in [GDR_SELFTEST_MIN_WAIT_NS, GDR_SELFTEST_MAX_WAIT_NS], else
 *   GDR_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
#define GDR_SELFTEST_MIN_WAIT_NS 100000ull      /* 0.1 ms */
#define GDR_SELFTEST_MAX_WAIT_NS 2000000000ull  /* 2 s, the ordinary limit */

gdr_status gdr_prefill_selftest_wait_expiry(const gdr_prefill_args *args, void *workspace,
                                            size_t workspace_bytes, uint64_t wait_ns,
                                            gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * RMSNormGated on its own (the output gate of the mixer; Qwen3.5 Chat guide,
 * "Architektur"):  y = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z), one
 * row of d values at a time.
 *
 *   o    [rows, d] o_dtype, row stride o_stride
 *   z    [rows, d] z_dtype, row stride z_stride
 *   w    [d] fp32 or NULL (ones)
 *   out  [rows, d] out_dtype, row stride out_stride; may equal o when the
 *        dtypes and strides match (in place).
 *   d in {16, 32, 64, 128}; rows == 0 is a no-op.
 * ------------------------------------------------------------------------ */
typedef struct gdr_norm_args {
    int64_t rows;
    int32_t d;
    int32_t o_dtype, z_dtype, out_dtype;
    float eps;
    int32_t reserved; /* must be 0 */
    int64_t o_stride, z_stride, out_stride;
    const void *o, *z;
    const float *w;
    void *out;
} gdr_norm_args;

gdr_status gdr_rmsnorm_gated(const gdr_norm_args *args, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * One decode step of the gated full-attention layer: the other mixer of the
 * hybrid decoder, one layer in four (Qwen3.5 Chat guide, "Architektur":
 * GatedAttention layers, standard scaled-dot-product attention over a KV
 * cache; Core AI card for Qwen3.6-35B-A3B, first section: head_dim 256,
 * 16 query heads over 2 key/value heads, partial rotary embedding with
 * theta = 1e7).  For every sequence b, with L = cache_len[b] tokens cached
 * before this step and kv head g = floor(h * H_kv / H_q) of query head h:
 *
 *     q_rot, k_rot = RoPE(q, L), RoPE(k, L): the first rot_dim dims turned in
 *                    pairs (i, i + rot_dim/2) by L * theta^(-2i/rot_dim)
 *     cache[b, g, L] = (k_rot, v)                              (appended)
 *     o_h = sum_{t <= L} softmax_t(scale * q_rot_h . k_cache[t]) v_cache[t]
 *     y_h = o_h * sigmoid(gate_h)                              (elementwise)
 *
 * For text tokens the three position components of mRoPE coincide, which
 * makes it this one-dimensional rotation.  The new key is stored and
 * attended as bf16, like every cached key.
 *
 *   q, gate    [batch, H_q, d]  bf16   row strides q_stride, gate_stride
 *   k, v       [batch, H_kv, d] bf16   row strides k_stride, v_stride
 *   k_cache, v_cache  [batch, H_kv, max_len, d] bf16, packed; row L of each
 *              (b, g) is written by this call, rows < L are read.
 *   cache_len  device int32 [batch]; read, not updated (the caller advances it)
 *   kv_bound   host: an upper bound of cache_len over the batch, < max_len;
 *              it sizes the split of the work.  A cache_len outside
 *              [0, kv_bound] is not attended past kv_bound, is not appended
 *              and sets the status word to GDR_ERR_INVALID_ARG.
 *   out        [batch, H_q, d] out_dtype, row stride out_stride
 *   rot_dim    even, 0 .. d (64 in the Qwen3.5 / 3.6 layers); rope_theta;
 *   scale      multiplies q.k (d^-1/2 for standard attention)
 *   Supported: d = 256, H_q a multiple of H_kv with H_q / H_kv <= 16,
 *   batch * H_kv * max_len < 2^31 (GDR_ERR_UNSUPPORTED otherwise).
 *   batch == 0 is a no-op.  k_cache and v_cache are read with TMA tensor
 *   copies: they need 16-byte alignment, like every pointer here.
 *   workspace: device memory, 16-byte aligned, of gdr_attn_decode_workspace_size
 *   bytes (per-split partial results); its first 4 bytes (int32) hold, once
 *   the work has finished, 0, GDR_ERR_INVALID_ARG (a cache_len out of range)
 *   or GDR_ERR_TIMEOUT (a bounded device-side wait gave up; outputs incomplete).
 * ------------------------------------------------------------------------ */
typedef struct gdr_attn_decode_args {
    int32_t batch, H_q, H_kv, d;
    int32_t rot_dim, max_len, kv_bound;
    int32_t out_dtype;                /* gdr_dtype of out */
    float rope_theta, scale;
    int64_t q_stride, gate_stride, k_stride, v_stride, out_stride;
    const void *q, *gate, *k, *v;
    void *k_cache, *v_cache;
    const int32_t *cache_len;
    void *out;
} gdr_attn_decode_args;

/* Workspace bytes gdr_attn_decode_step needs for these arguments (only sizes
 * are read).  Returns the status gdr_attn_decode_step's checks would. */
gdr_status gdr_attn_decode_workspace_size(const gdr_attn_decode_args *args, size_t *bytes);

gdr_status gdr_attn_decode_step(const gdr_attn_decode_args *args, void *workspace,
                                size_t workspace_bytes, gdr_stream_t stream);

/* ------------------------------------------------------------------------
 * The routed-expert MoE feed-forward block at decode time (the FFN of the
 * hybrid decoder's MoE models: Core AI card for Qwen3.6-35B-A3B, first
 * section -- a router over the experts, an fp32 softmax, the top k
 * renormalised by their sum, SwitchGLU experts gathered by index, and an
 * always-on shared SwitchGLU scaled by sigmoid(shared_expert_gate(x)); its
 * "Speed" section puts a decode step's cost in reading only the routed
 * experts' weights).  Per token x:
 *
 *     p = softmax(W_router x);  top_k experts by p (ties to the lower index)
 *     w_e = p_e / sum_{top_k} p
 *     y = sum_e w_e W_down,e (silu(W_gate,e x) * (W_up,e x))
 *       + sigmoid(w_sgate . x) W_down,s (silu(W_gate,s x) * (W_up,s x))
 *
 * Only the experts some token chose are read, each once for all the tokens
 * that chose it.  bf16 weights and activations, fp32 arithmetic.
 *
 *   x          [n_tok, hidden] bf16, row stride x_stride
 *   w_router   [n_exp, hidden] bf16
 *   w_gate_up  [n_exp, 2 * inter, hidden] bf16: rows 0 .. inter-1 of an
 *              expert are its gate matrix, rows inter .. 2 inter - 1 its up
 *   w_down     [n_exp, hidden, inter] bf16
 *   ws_gate_up [2 * s_inter, hidden], ws_down [hidden, s_inter], w_sgate
 *              [hidden] bf16: the shared expert and its gate row; ws_gate_up
 *              NULL (and s_inter 0) for a block without a shared expert
 *   out        [n_tok, hidden] out_dtype, row stride out_stride
 *   topk_idx, topk_w   optional device outputs [n_tok, top_k]: the chosen
 *              experts (int32, in decreasing probability) and their weights
 *   Supported: hidden and inter (s_inter) multiples of 8, inter and s_inter
 *   <= 1024; 1 <= top_k <= 32, top_k <= n_exp <= 1024; n_tok <= 4096.
 *   n_tok == 0 is a no-op.
 *   workspace: gdr_moe_workspace_size bytes, 16-byte aligned.
 * ------------------------------------------------------------------------ */
typedef struct gdr_moe_args {
    int32_t n_tok, hidden, n_exp, top_k, inter, s_inter;
    int32_t out_dtype;                /* gdr_dtype of out */
    int32_t reserved;                 /* 0 */
    int64_t x_stride, out_stride;
    const void *x, *w_router, *w_gate_up, *w_down;
    const void *ws_gate_up, *ws_down, *w_sgate;
    void *out;
    int32_t *topk_idx;
    float *topk_w;
} gdr_moe_args;

gdr_status gdr_moe_workspace_size(const gdr_moe_args *args, size_t *bytes);

gdr_status gdr_moe_decode(const gdr_moe_args *args, void *workspace, size_t workspace_bytes,
                          gdr_stream_t stream);

/* Static, human-readable name of a status (never NULL). */
const char *gdr_status_string(gdr_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDR_H_ */
