/*
 * gdn.h -- C ABI of the gated delta rule for NVIDIA B200 (sm_100a).
 *
 * The operation.  Per sequence and head, a d_v x d_k state S evolves token by
 * token as
 *
 *     S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t (scale q_t)
 *
 * with D_t = alpha_t I (one gate per head: Gated DeltaNet) or
 * D_t = Diag(alpha_t), alpha_t in (0,1]^{d_k} (one gate per key channel: the
 * KDA variant).  Decay comes first, the delta correction is applied to the
 * decayed state, and the output reads the state after the write.
 *   - "Hybrid models: what Gated DeltaNet replaces in the KV cache", section
 *     "Gated DeltaNet: add decay" (the update and the d_v x d_k state);
 *   - "From Traditional Attention to hybrid ones", section 5 (decay, then the
 *     delta update on the decayed state, then o_t = S_t q_t) and section 7
 *     (the per-channel form S_{t-1} Diag(alpha_t)(I - beta_t k_t k_t^T) + ...);
 *   - "Attention, Part 4: Linear Attention, Gated DeltaNet and Hybrid Models",
 *     "Where alpha and beta come from" (the gate arrives as g = log alpha).
 *
 * Conventions shared by every entry point.
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates device memory; scratch memory comes only from
 *     the caller's workspace.
 *   - Layouts are dense row-major (C order), no strides:
 *       q, k      (B, T, H, d_k)      dtype per gdn_desc.dtype
 *       v, out    (B, T, H, d_v)      dtype per gdn_desc.dtype
 *       log_gate  (B, T, H) fp32      one gate per head, or
 *                 (B, T, H, d_k) fp32 one gate per key channel
 *       beta      (B, T, H) fp32
 *       states    (N, H, d_v, d_k) fp32, N = number of sequences
 *     log_gate holds g = log(alpha): finite and <= 0 (alpha = 1 is allowed).
 *     beta is used as given (the pages keep it in (0,1); 0 and 1 work).
 *   - q, k, v, out and states must be 16-byte aligned, the workspace 256-byte;
 *     log_gate, beta and cu_seqlens 4-byte aligned, except that the chunked
 *     calls take a per-channel log_gate 16-byte aligned (its rows are d_k
 *     floats, so any row of an aligned tensor qualifies).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are detected on the host before
 *     anything is launched and leave all outputs untouched.  A failed launch
 *     returns GDN_ERR_CUDA.  gdn_last_error() gives a one-line reason for the
 *     most recent failure on the calling thread.
 *   - Supported sizes: d_k, d_v in {64, 128}.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gdn_stream_t; /* same type as cudaStream_t */

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* a size, pointer, alignment or flag is wrong      */
    GDN_ERR_UNSUPPORTED = 2, /* valid request the library does not implement     */
    GDN_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required       */
    GDN_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed             */
    GDN_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (gdn_chunk_status) */
    GDN_ERR_INTERNAL = 6     /* a device-side consistency check failed           */
} gdn_status;

/* Device status codes of the chunked prefill: the int32 at byte 0 of the
 * workspace (or of the built-in scratch of gdn_chunk_fwd_static).  Every
 * gdn_chunk_fwd call zeroes it on its stream before its kernels run; a kernel
 * that gives up a bounded wait (on a tile copy or a tensor-core commit) writes
 * its code there, waits (again bounded) for its copies and products in
 * flight, frees its tensor memory and returns without trapping.  The first
 * code written wins.  Read it with gdn_chunk_status. */
typedef enum gdn_device_code {
    GDN_DEV_OK = 0,
    GDN_DEV_TIMEOUT_PREP = 1, /* the chunk-local kernel gave up a wait          */
    GDN_DEV_TIMEOUT_SCAN = 2, /* the sequential scan gave up a wait             */
    GDN_DEV_BOUNDS = 16       /* bounds-checked builds only: an index left the
                                 range the descriptor gives (the access was
                                 skipped)                                       */
} gdn_device_code;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

typedef enum gdn_gate_kind {
    GDN_GATE_HEAD = 0,   /* alpha_t is one scalar per head and token (Gated DeltaNet) */
    GDN_GATE_CHANNEL = 1 /* alpha_t is a d_k vector per head and token (KDA)          */
} gdn_gate_kind;

/* Problem description.  For packed sequences B = 1 and T is the total number
 * of packed tokens.  For gdn_decode_step T = 1 and B is the number of live
 * sequences. */
typedef struct gdn_desc {
    int64_t B, T, H, dk, dv;
    int32_t dtype; /* gdn_dtype of q, k, v and out (gates, beta, states: fp32)  */
    int32_t gate;  /* gdn_gate_kind                                              */
    float scale;   /* multiplies q before the read; 1.0 gives o_t = S_t q_t      */
    int32_t hk;    /* query/key heads: 0 (= H) or a divisor of H; value head h
                      reads query/key head h / (H / hk)                         */
} gdn_desc;

/* ---------------------------------------------------------------------------
 * gdn_chunk_workspace_size -- bytes of device workspace gdn_chunk_fwd needs.
 *
 * num_seqs: number of sequences (B when cu_seqlens is NULL).  The bound
 * covers any packing of d->T tokens into num_seqs sequences.
 * Returns GDN_ERR_INVALID_ARG for a bad descriptor or a NULL `bytes`.
 * ------------------------------------------------------------------------- */
gdn_status gdn_chunk_workspace_size(const gdn_desc *d, int32_t num_seqs, size_t *bytes);

/* ---------------------------------------------------------------------------
 * gdn_chunk_fwd -- chunkwise-parallel prefill.
 *
 * Computes the outputs o_t of every token and the state after each sequence,
 * exactly as the token-by-token recurrence above (up to rounding), by the
 * chunkwise form: within a chunk of 64 tokens the writes are coupled only
 * through a small lower-triangular system, solved with matrix products; only
 * the d_v x d_k state passes from one chunk to the next.
 *   - "Hybrid attention: why new LLMs keep full attention in only a few
 *     layers", section "Training a recurrence in parallel";
 *   - "Hybrid Linear Attention Architecture Design Explained", section 4
 *     (state update S[t+1] and output O[t] per chunk, cumulative decay in the
 *     log domain);
 *   - "Hybrid models ...", section "What a recurrent state changes for
 *     serving", item 1 (snapshots of the state at chosen positions).
 *
 * Arguments
 *   d              problem description (d->T >= 0; T = 0 is a no-op apart from
 *                  copying initial states to final states)
 *   q, k, v        inputs, layouts above
 *   log_gate, beta gates, layouts above (log_gate per channel iff
 *                  d->gate == GDN_GATE_CHANNEL)
 *   initial_state  (N, H, d_v, d_k) fp32, or NULL for zero states
 *   cu_seqlens     NULL: N = B sequences of T tokens each.  Otherwise a device
 *                  array of num_seqs+1 non-decreasing int32 offsets into the
 *                  B*T token rows with cu_seqlens[0] = 0 and
 *                  cu_seqlens[num_seqs] = T (B must be 1).  Chunks restart at
 *                  every sequence start.  The offsets are read on the device
 *                  and are not validated there: wrong offsets give wrong
 *                  results, but every access stays inside the B*T rows.
 *   num_seqs       number of sequences when cu_seqlens != NULL (else ignored)
 *   snapshot_stride 0 for none, else a positive multiple of 64: the state
 *                  after the first n*stride tokens of each sequence,
 *                  n = 1 .. floor(T/stride), is written to `snapshots`.
 *                  Only without cu_seqlens (GDN_ERR_UNSUPPORTED otherwise).
 *   out            (B, T, H, d_v), must not overlap any input
 *   final_state    (N, H, d_v, d_k) fp32 or NULL; may be the same pointer as
 *                  initial_state (read fully before it is written)
 *   snapshots      (B, floor(T/stride), H, d_v, d_k) fp32, required iff
 *                  snapshot_stride > 0
 *   workspace      device scratch of at least gdn_chunk_workspace_size bytes,
 *                  256-byte aligned; contents on entry do not matter and are
 *                  clobbered.  Its first 4 bytes hold the call's device status
 *                  (gdn_chunk_status).  Two calls in flight at once need two
 *                  workspaces.
 *   stream         CUDA stream
 * ------------------------------------------------------------------------- */
gdn_status gdn_chunk_fwd(const gdn_desc *d,
                         const void *q, const void *k, const void *v,
                         const float *log_gate, const float *beta,
                         const float *initial_state,
                         const int32_t *cu_seqlens, int32_t num_seqs,
                         int64_t snapshot_stride,
                         void *out, float *final_state, float *snapshots,
                         void *workspace, size_t workspace_bytes,
                         gdn_stream_t stream);

/* ---------------------------------------------------------------------------
 * gdn_chunk_status -- the device status of the last gdn_chunk_fwd call that
 * used `workspace` on `stream`.
 *
 * Waits for `stream` (cudaStreamSynchronize), then reads the int32 status
 * word at byte 0 of the workspace (one 4-byte device-to-host copy) into
 * *device_code (a gdn_device_code).  Returns GDN_OK when it is zero,
 * GDN_ERR_TIMEOUT for a timeout code, GDN_ERR_INTERNAL for a bounds code, and
 * GDN_ERR_CUDA when the wait or the copy fails.  Not for use during stream
 * capture (it synchronises).  The outputs of a call whose status is not
 * GDN_OK are incomplete.
 * ------------------------------------------------------------------------- */
gdn_status gdn_chunk_status(const void *workspace, gdn_stream_t stream, int32_t *device_code);

/* ---------------------------------------------------------------------------
 * gdn_chunk_fwd_static -- gdn_chunk_fwd without a caller-provided workspace.
 *
 * The source pages have no counterpart to this entry point; it exists for
 * callers that cannot allocate device memory (a serving loop whose allocator
 * owns a fixed, pre-partitioned budget, a real-time path that must not take
 * the device synchronisation an allocation may cause, a plugin that is handed
 * pointers but no allocator).  It computes exactly what gdn_chunk_fwd
 * computes, with the same arguments minus `workspace`/`workspace_bytes`; its
 * scratch is a 64 MiB array built into the library, which every GPU that
 * loads the library holds until the process exits.
 *
 *   - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call.
 *   - Requests whose scratch need (gdn_chunk_workspace_size) exceeds 64 MiB
 *     return GDN_ERR_WORKSPACE before touching the device.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the array and it keeps the previous call's contents;
 *     nothing needs to start at zero, but two calls that overlap on the GPU
 *     (e.g. on unordered streams) race on it: serialise them.
 * ------------------------------------------------------------------------- */
gdn_status gdn_chunk_fwd_static(const gdn_desc *d,
                                const void *q, const void *k, const void *v,
                                const float *log_gate, const float *beta,
                                const float *initial_state,
                                const int32_t *cu_seqlens, int32_t num_seqs,
                                int64_t snapshot_stride,
                                void *out, float *final_state, float *snapshots,
                                gdn_stream_t stream);

/* gdn_chunk_status for gdn_chunk_fwd_static: the status word in the built-in
 * scratch of the current device (same waits and return values). */
gdn_status gdn_chunk_status_static(gdn_stream_t stream, int32_t *device_code);

/* ---------------------------------------------------------------------------
 * gdn_decode_step -- one token of every live sequence, state updated in place.
 *
 * For each of the d->B sequences and d->H heads (d->T must be 1):
 *     y = S D k,  z = S D (scale q)           (one read of S)
 *     delta = beta (v - y)
 *     S'  = S D + delta k^T                   (written over S)
 *     o   = z + delta (k . scale q)  ( = S' scale q )
 * with D = alpha I or Diag(alpha), alpha = exp(log_gate).
 *   - "From Traditional Attention to hybrid ones", section 5 (the update on the
 *     decayed state and the read o_t = S_t q_t) and "vLLM Storage" (the
 *     recurrent state is fixed per live sequence and updated in place);
 *   - "Attention, Part 4 ...", section 8 (one decode step updates the
 *     32 x 128 x 128 memory once per token).
 *
 *   q, k (B, 1, H, d_k); v, out (B, 1, H, d_v); log_gate (B, 1, H) or
 *   (B, 1, H, d_k); beta (B, 1, H); state (B, H, d_v, d_k) fp32, read and
 *   overwritten.  `out` must not overlap the state or the inputs.
 * ------------------------------------------------------------------------- */
gdn_status gdn_decode_step(const gdn_desc *d,
                           const void *q, const void *k, const void *v,
                           const float *log_gate, const float *beta,
                           float *state, void *out, gdn_stream_t stream);

/* ---------------------------------------------------------------------------
 * gdn_decode_multi -- up to d->T tokens of every live sequence in one pass over
 * its state: the verify step of speculative decoding and multi-token decode.
 *
 * A recurrent state has absorbed every token it saw, so rejecting draft tokens
 * needs the state from before them ("Hybrid models: what Gated DeltaNet
 * replaces in the KV cache", section "What a recurrent state changes for
 * serving", item 2; "Hybrid attention: why new LLMs keep full attention in
 * only a few layers", closing section: rolling back a rejected speculative
 * token needs the state from a step earlier).
 *
 * For sequence b (d->B of them) and head h, with n_b = n_tokens[b] clamped to
 * [0, d->T] (d->T when n_tokens is NULL), tokens t = 0 .. n_b - 1 are applied in
 * order exactly as gdn_decode_step would apply them, starting from state[b, h]:
 *   out[b, t, h]          = the token's output (rows t >= n_b are not written);
 *   step_states[b, t, h]  = the state after token t, if step_states != NULL
 *                           (entries t >= n_b are not written);
 *   state[b, h]           = the state after n_b tokens if commit == 1; left
 *                           unchanged (the pre-draft state) if commit == 0.
 * The state is read from HBM once for all tokens.
 *
 *   d        B = live sequences, T = token slots per sequence (1 .. 64), H, d_k, d_v,
 *            dtype, gate, scale as for gdn_decode_step
 *   q, k     (B, T, H, d_k); v, out (B, T, H, d_v); log_gate (B, T, H) or
 *            (B, T, H, d_k); beta (B, T, H)  -- token t of sequence b at [b, t]
 *   n_tokens device int32 (B), or NULL for all T tokens
 *   state    (B, H, d_v, d_k) fp32
 *   commit   0 or 1
 *   step_states (B, T, H, d_v, d_k) fp32 or NULL
 * Alignment as for gdn_decode_step (step_states 16-byte, n_tokens 4-byte);
 * out, state and step_states must not overlap each other or the inputs.
 * Returns GDN_ERR_INVALID_ARG for T outside 1 .. 64, a bad commit value, NULL
 * required pointers, misalignment or overlap (nothing launched).
 * ------------------------------------------------------------------------- */
gdn_status gdn_decode_multi(const gdn_desc *d,
                            const void *q, const void *k, const void *v,
                            const float *log_gate, const float *beta,
                            const int32_t *n_tokens, float *state, int32_t commit,
                            void *out, float *step_states, gdn_stream_t stream);

/* ---------------------------------------------------------------------------
 * gdn_state_select -- adopt the state after an accepted prefix of the drafts.
 *
 * For every sequence b with m = accept[b] > 0 (clamped to d->T) and every head
 * h: state[b, h] = step_states[b, m - 1, h], the state gdn_decode_multi wrote
 * after token m - 1; sequences with accept[b] <= 0 keep their state (the
 * pre-draft state when the verify call did not commit).
 *   d            B, T (token slots of step_states), H, d_k, d_v as in the
 *                gdn_decode_multi call that wrote step_states
 *   step_states  (B, T, H, d_v, d_k) fp32, 16-byte aligned
 *   accept       device int32 (B), 4-byte aligned
 *   state        (B, H, d_v, d_k) fp32, 16-byte aligned, not overlapping the others
 * ------------------------------------------------------------------------- */
gdn_status gdn_state_select(const gdn_desc *d, const float *step_states, const int32_t *accept,
                            float *state, gdn_stream_t stream);

/* ---------------------------------------------------------------------------
 * gdn_prerule -- the layer's work before the recurrence, from its raw
 * projections, producing the inputs of gdn_chunk_fwd / gdn_decode_step /
 * gdn_decode_multi ("Attention, Part 4: Linear Attention, Gated DeltaNet and
 * Hybrid Models", section 6, "Where alpha and beta come from" and the paragraph
 * after it: short convolution, SiLU and length-1 queries and keys, beta =
 * sigmoid(b), g = -exp(A_log) softplus(a + dt_bias); "From Traditional
 * Attention to hybrid ones", "vLLM Storage": the convolution history kept per
 * live sequence).
 *
 * For every token of every sequence and every channel c of the mixed projection
 * x = [q heads (hk x d_k) | k heads (hk x d_k) | v heads (H x d_v)]:
 *     y_c = SiLU( sum_{j<K} conv_w[c, j] * x_c(t - (K-1) + j) )
 * (tap K-1 on the current token; inputs before the sequence's first token from
 * conv_state_in, the sequence's last K-1 raw inputs oldest first, zeros if NULL);
 * q, k = y / sqrt(|y|^2 + 1e-6) per head, v = y (written in d->dtype);
 * beta = sigmoid(b), log_gate = -exp(A_log[h]) softplus(a + dt_bias[h]) (fp32).
 * If conv_state_out != NULL it receives each sequence's last K-1 raw inputs
 * (older history where the sequence is shorter); it may be conv_state_in.
 *
 *   d          B, T, H (value heads), hk, d_k, d_v, dtype; gate must be
 *              GDN_GATE_HEAD (the formula is the per-head one)
 *   x          (B, T, 2 hk d_k + H d_v) in d->dtype, 16-byte aligned
 *   a, b       (B, T, H) in d->dtype
 *   conv_w     (2 hk d_k + H d_v, K) fp32;  K in 1 .. 4
 *   A_log, dt_bias (H) fp32
 *   cu_seqlens / num_seqs  packed sequences as for gdn_chunk_fwd (B == 1), or
 *              NULL: B sequences of T tokens (a decode step is T = 1)
 *   conv_state_in, conv_state_out  (N, 2 hk d_k + H d_v, K-1) fp32, or NULL
 *   q, k       (B, T, hk, d_k); v (B, T, H, d_v) -- 16-byte aligned
 *   log_gate, beta (B, T, H) fp32
 * Rows of a packed batch outside every sequence are not written.  Outputs must
 * not overlap the inputs or each other.  GDN_ERR_UNSUPPORTED for more than
 * 2^31 - 1 token rows.  SiLU is evaluated through the hardware tanh for bf16
 * (relative error about 2^-11, below the rounding of the bf16 result).
 * ------------------------------------------------------------------------- */
gdn_status gdn_prerule(const gdn_desc *d, const void *x, const void *a, const void *b,
                       const float *conv_w, int32_t K, const float *A_log, const float *dt_bias,
                       const int32_t *cu_seqlens, int32_t num_seqs,
                       const float *conv_state_in, float *conv_state_out,
                       void *q, void *k, void *v, float *log_gate, float *beta,
                       gdn_stream_t stream);

/* Static description of a status code. */
/* -------------------------------------------------------------------------
 * gdn_decode_step_prerule -- one decode step from the layer's raw projections:
 * for every sequence's new token, the work of gdn_prerule (short causal
 * convolution with the sequence's history, SiLU, length-1 q and k, beta =
 * sigmoid(b), g = -exp(A_log) softplus(a + dt_bias); "Attention, Part 4: Linear
 * Attention, Gated DeltaNet and Hybrid Models", section 6) and then the step of
 * gdn_decode_step ("From Traditional Attention to hybrid ones", section 5), in
 * one kernel: q, k, v, g and beta stay in registers (fp32).  The convolution
 * history is then shifted by a second small kernel (so it is updated in place).
 *
 *   d          B sequences, T == 1, H (value heads), hk, d_k, d_v, dtype, scale;
 *              gate must be GDN_GATE_HEAD
 *   x          (B, 2 hk d_k + H d_v) raw mixed projection in d->dtype
 *   a, b       (B, H) in d->dtype;  conv_w (2 hk d_k + H d_v, K) fp32, K in 1 .. 4
 *   A_log, dt_bias (H) fp32
 *   conv_state (B, 2 hk d_k + H d_v, K-1) fp32, the last K-1 raw inputs (oldest
 *              first), updated in place; NULL: zero history, none kept
 *   state      (B, H, d_v, d_k) fp32, updated in place; out (B, H, d_v) in d->dtype
 * state and out 16-byte aligned; outputs must not overlap the inputs or each
 * other.  Errors as gdn_decode_step.
 * ------------------------------------------------------------------------- */
gdn_status gdn_decode_step_prerule(const gdn_desc *d, const void *x, const void *a, const void *b,
                                   const float *conv_w, int32_t K, const float *A_log, const float *dt_bias,
                                   float *conv_state, float *state, void *out, gdn_stream_t stream);

const char *gdn_status_string(gdn_status s);

/* One-line reason for the most recent failed call on this thread ("" if none). */
const char *gdn_last_error(void);

/* ---------------------------------------------------------------------------
 * Kernel timing.  While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the launch stream; gdn_profile_read
 * waits for them and returns per kernel name the number of launches and the
 * summed device time.  Events are created lazily (host resources only; no
 * device memory is allocated).  Reading resets the counters.
 * ------------------------------------------------------------------------- */
typedef struct gdn_kernel_time {
    const char *name;   /* static string, valid for the life of the library */
    int64_t launches;
    double total_ms;
} gdn_kernel_time;

gdn_status gdn_profile_enable(int on);
/* Writes up to `cap` entries and stores the number of distinct kernels seen in
 * *count (which may exceed cap). */
gdn_status gdn_profile_read(gdn_kernel_time *entries, int32_t cap, int32_t *count);

/* Launch log.  With the environment variable GDN_LOG=1 (read once, at the first
 * launch), every kernel launch of the chunked prefill prints one line to
 * stderr: the kernel, its grid, block and dynamic shared memory. */

#ifdef __cplusplus
}
#endif
#endif /* GDN_H_ */
