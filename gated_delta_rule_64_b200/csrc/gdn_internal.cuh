// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kChunk = 64;  // tokens per chunk of the chunkwise form

// Where a kernel launch came from, for the optional event timer.
struct LaunchScope {
    LaunchScope(const char *name, cudaStream_t s);
    ~LaunchScope();
    const char *name_;
    cudaStream_t stream_;
    int slot_;
};

// Query/key heads of a description (hk = 0 means H).
inline int64_t qk_heads(const gdn_desc &d) { return d.hk > 0 ? d.hk : d.H; }

// Records a failure reason for gdn_last_error() and returns `st`.
gdn_status fail(gdn_status st, const char *fmt, ...);

// Map the result of a launch to a status.
gdn_status check_launch(const char *what);

// One line per launch on stderr when GDN_LOG=1 (the grid, block and shared memory).
void log_launch(const char *name, dim3 grid, dim3 block, size_t smem);

// ---------------------------------------------------------------------------
// Workspace of the chunked forward pass.
// ---------------------------------------------------------------------------
struct ChunkPlan {
    int64_t N;           // sequences
    int64_t rows;        // B*T packed token rows
    int64_t H, dk, dv;
    int64_t max_chunks;  // upper bound on sum_n ceil(len_n / 64)
    bool packed;
    bool per_channel;
    bool tc;             // tensor-core path (bf16, d_k = d_v = 128)
    size_t tc_block;     // bytes per chunk-head of the tensor-core workspace
    int32_t split_G;     // tensor-core path, fixed-length sequences: segments per sequence (1: none)
    int32_t split_seg;   // chunks per segment
    // byte offsets into the workspace
    size_t off_status;         // int32 device status word (kStatusBytes reserved), zeroed by every call
    size_t off_chunk_offsets;  // int32 (N+1): first global chunk index of each sequence, then
                               // int32 (N): the sequences by decreasing chunk count (packed batches)
    size_t off_W, off_U, off_P, off_b;
    size_t off_split;    // [N][G][3][H][d_v][d_k] fp32 segment maps and start states, then the
                         // int32 [N][G][H] segment records (see ScanSplit)
    size_t total;
};
constexpr size_t kStatusBytes = 256;  // the status word's slot at the start of the workspace

// Segments per sequence for the split scan of N fixed-length sequences of
// `nch` chunks on `sms` multiprocessors (G = 1: no split).
struct SplitChoice {
    int32_t G, seg;
};
SplitChoice choose_split(int64_t N, int64_t H, int64_t nch, int sms);

ChunkPlan make_plan(const gdn_desc &d, int64_t num_seqs, bool packed);


struct ChunkArgs {
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    const int32_t *cu_seqlens;  // nullptr: fixed-length sequences of length T
    int64_t T;                  // per-sequence length when not packed
    int64_t N, H;
    int64_t Hk;                 // query/key heads (divides H)
    float scale;
    int64_t snapshot_stride;
    int64_t n_snap;             // snapshots per sequence (fixed-length only)
    void *out;
    float *final_state, *snapshots;
    char *ws;
    int *status;                // device status word (workspace offset off_status)
};

gdn_status launch_chunk_table(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s);
gdn_status launch_chunk_simt(const ChunkPlan &p, const ChunkArgs &a, int dtype, cudaStream_t s);
gdn_status launch_chunk_tc(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s);
bool tc_eligible(const gdn_desc &d);

// Per chunk-head workspace block of the tensor-core path (bytes), both gate kinds:
//   [W^T rows 16K][Qs (channels 0-63) 8K][Qs (64-127) 8K]
//   [K~ 16K][P rows 8K][-T'' rows 8K][gate factors 1K]
// Every operand is 128-byte swizzled rows of 128 bytes (64 bf16), in 8-row groups
// 1 KB apart.  W^T (row = key channel, 64 tokens) is the MN-major B operand of
// S0 W^T; Qs = scale Q * Gam (per-channel gate only; row = token, the layout of a
// Q tile) the K-major one of S0 Qs^T.  K~ = K * exp(b_L - b) (per-channel gate only;
// the layout of a K tile: rows = tokens, two 64-channel halves) is the MN-major B
// operand of U'^T K~; P (row = query token i, 64 key tokens j) the K-major one of
// U'^T P^T; -T'' = -T diag(beta) (row = token i, 64 tokens j) the K-major one of
// V^T (-T'')^T, which the scan accumulates onto S0 W^T to get -U'^T.  The scan
// copies a block with two or three bulk copies.
constexpr size_t kTcWQ = 32768, kTcKt = 64 * 128 * 2, kTcPImg = 64 * 128, kTcTn = 64 * 128, kTcFac = 1024;
constexpr size_t kTcRest = kTcKt + kTcPImg + kTcTn + kTcFac;  // 33792
constexpr size_t kTcBlock = kTcWQ + kTcRest;                  // 66560
gdn_status launch_decode(const gdn_desc &d, const void *q, const void *k, const void *v,
                         const float *g, const float *beta, float *state, void *out,
                         cudaStream_t s);
constexpr int64_t kMaxMultiTokens = 64;  // tokens per sequence of one gdn_decode_multi call
gdn_status launch_decode_multi(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const int32_t *n_tokens, float *state, int commit, void *out,
                               float *step_states, cudaStream_t s);
gdn_status launch_state_select(const gdn_desc &d, const float *step_states, const int32_t *accept, float *state,
                               cudaStream_t s);

// The work before the recurrence (short convolution, SiLU, q/k length, gates).
struct PreruleArgs {
    int dtype, K;
    int64_t T, N, rows, H, Hk, dk, dv;
    const void *x, *a, *b;
    const float *conv_w, *A_log, *dt_bias;
    const int32_t *cu_seqlens;  // nullptr: N sequences of T tokens
    const float *hist_in;
    float *hist_out;
    void *q, *k, *v;
    float *g, *beta;
};
gdn_status launch_prerule(const PreruleArgs &a, cudaStream_t s);
// Only the convolution history update of launch_prerule (hist_in -> hist_out, in place
// allowed), for the leading `channels` channels of every row (< 0: all).
gdn_status launch_prerule_history(const PreruleArgs &a, int64_t channels, cudaStream_t s);
// A decode step from the raw projections (one token per sequence, T = 1): the pre-rule
// work for the token in registers, then the recurrence; the history is updated after.
gdn_status launch_decode_prerule(const gdn_desc &d, const PreruleArgs &a, float *state, void *out, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace gdn
