// Several tokens of every live sequence in one pass over the state, for
// speculative decoding: verify k draft tokens, keep the pre-draft state or the
// state after any accepted prefix, and select an accepted step's state later.
//
// Rolling back rejected drafts needs the state from before them, because the
// recurrent state has already absorbed every token it saw ("Hybrid models: what
// Gated DeltaNet replaces in the KV cache", section "What a recurrent state
// changes for serving", item 2; "Hybrid attention: why new LLMs keep full
// attention in only a few layers", closing section on the costs of hybrids).
//
// The recurrence per token is the one of the single-token step
// ("From Traditional Attention to hybrid ones", section 5): decay, the delta
// correction on the decayed state, then the read of the updated state.  Rows of
// the d_v x d_k state evolve independently, so the block's threads keep the state
// in registers (a warp per eight rows, a lane per d_k/32 columns) and apply the tokens in order:
// the state is read from HBM once for all tokens and written back at most once
// (plus one copy per token when the caller asks for every step's state).
#include "decode_rows.cuh"

namespace gdn {
namespace {

using dec::kRowsPerWarp;
using dec::kWarps;

// See decode_rows: a warp per eight state rows, a lane per d_k / 32 columns.
template <int DK, int DV, typename Tin, bool PER_CHANNEL>
__global__ void __launch_bounds__(kWarps * 32)
gdn_decode_multi_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                        const float *__restrict__ g, const float *__restrict__ beta,
                        const int32_t *__restrict__ n_tokens, float *__restrict__ state, int commit,
                        Tin *__restrict__ out, float *__restrict__ step_states, int T, int64_t H, int64_t Hk,
                        float scale) {
    int n = T;
    if (n_tokens) {
        n = n_tokens[blockIdx.x / H];
        n = n < 0 ? 0 : (n > T ? T : n);
    }
    if (n == 0) return;
    const dec::ArraySrc<DK, DV, Tin, PER_CHANNEL> src{q, k, v, g, beta, Hk, scale};
    dec::decode_rows<DK, DV, Tin>(src, state, commit != 0, out, step_states, n, T, H);
}

// state[b, h] = step_states[b, accept[b] - 1, h] where accept[b] > 0.
__global__ void __launch_bounds__(256)
gdn_state_select_kernel(const float *__restrict__ step_states, const int32_t *__restrict__ accept,
                        float *__restrict__ state, int T, int64_t H, int64_t per_state4) {
    const int64_t unit = blockIdx.x, b = unit / H, h = unit % H;
    int m = accept[b];
    if (m <= 0) return;
    m = m > T ? T : m;
    const float4 *src = reinterpret_cast<const float4 *>(step_states) + ((b * T + (m - 1)) * H + h) * per_state4;
    float4 *dst = reinterpret_cast<float4 *>(state) + unit * per_state4;
    for (int64_t e = threadIdx.x; e < per_state4; e += blockDim.x) dst[e] = src[e];
}

template <int DK, int DV, typename Tin>
gdn_status launch_multi(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const int32_t *n_tokens, float *state, int commit, void *out,
                        float *step_states, cudaStream_t s) {
    const int64_t units = d.B * d.H;
    if (units > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many (sequence, head) pairs");
    auto kern = d.gate == GDN_GATE_CHANNEL ? gdn_decode_multi_kernel<DK, DV, Tin, true>
                                           : gdn_decode_multi_kernel<DK, DV, Tin, false>;
    {
        LaunchScope ls("gdn_decode_multi_kernel", s);
        kern<<<dim3((unsigned)units, (unsigned)(DV / (kWarps * kRowsPerWarp))), kWarps * 32, 0, s>>>(
            (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, n_tokens, state, commit, (Tin *)out, step_states,
            (int)d.T, d.H, qk_heads(d), d.scale);
    }
    return check_launch("gdn_decode_multi_kernel");
}

template <typename Tin>
gdn_status launch_multi_t(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const int32_t *n_tokens, float *state, int commit, void *out,
                          float *step_states, cudaStream_t s) {
    if (d.dk == 128)
        return d.dv == 128 ? launch_multi<128, 128, Tin>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s)
                           : launch_multi<128, 64, Tin>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s);
    return d.dv == 128 ? launch_multi<64, 128, Tin>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s)
                       : launch_multi<64, 64, Tin>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s);
}

}  // namespace

gdn_status launch_decode_multi(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const int32_t *n_tokens, float *state, int commit, void *out,
                               float *step_states, cudaStream_t s) {
    return d.dtype == GDN_BF16
               ? launch_multi_t<__nv_bfloat16>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s)
               : launch_multi_t<float>(d, q, k, v, g, beta, n_tokens, state, commit, out, step_states, s);
}

gdn_status launch_state_select(const gdn_desc &d, const float *step_states, const int32_t *accept, float *state,
                               cudaStream_t s) {
    const int64_t units = d.B * d.H;
    if (units > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many (sequence, head) pairs");
    {
        LaunchScope ls("gdn_state_select_kernel", s);
        gdn_state_select_kernel<<<(unsigned)units, 256, 0, s>>>(step_states, accept, state, (int)d.T, d.H,
                                                                d.dv * d.dk / 4);
    }
    return check_launch("gdn_state_select_kernel");
}

}  // namespace gdn
