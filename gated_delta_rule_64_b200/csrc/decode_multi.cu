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
// in registers (two or four threads per row) and apply the tokens to it in order:
// the state is read from HBM once for all tokens and written back at most once
// (plus one copy per token when the caller asks for every step's state).
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Shared memory per token t of the block's (sequence, head): a_t k_t, a_t q_t,
// a_t, k_t (d_k each; q already scaled) and v_t (d_v); then beta_t and k_t . q_t.
// The 256 threads split the state into TPR = 256 / d_v threads per row; thread
// part p of a row holds the 16-byte column chunks p, p + TPR, p + 2 TPR, ... in
// registers, so one warp instruction moves whole 32-byte sectors of 8 or 16 rows.
// A token's two dot products are per-thread sums (four independent partial sums)
// finished by log2(TPR) shuffles.
template <int DK, int DV, typename Tin, bool PER_CHANNEL>
__global__ void __launch_bounds__(kWarps * 32, 2)
gdn_decode_multi_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                        const float *__restrict__ g, const float *__restrict__ beta,
                        const int32_t *__restrict__ n_tokens, float *__restrict__ state, int commit,
                        Tin *__restrict__ out, float *__restrict__ step_states, int T, int64_t H, int64_t Hk,
                        float scale) {
    constexpr int TPR = kWarps * 32 / DV, NCH = DK / 4 / TPR, VEC = DK / 32;  // NCH chunks per thread
    extern __shared__ float4 dm_raw[];
    float *sm = reinterpret_cast<float *>(dm_raw);
    constexpr int per_tok = 4 * DK + DV;
    float *s_beta = sm + (size_t)T * per_tok, *s_kq = s_beta + T;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t unit = blockIdx.x, b = unit / H, h = unit % H;
    int n = T;
    if (n_tokens) {
        n = n_tokens[b];
        n = n < 0 ? 0 : (n > T ? T : n);
    }
    if (n == 0) return;

    // stage the tokens' vectors (warp w takes tokens w, w + 8, ...)
    for (int t = warp; t < n; t += kWarps) {
        const int64_t tk = (b * T + t) * H + h;             // (b, t, h)
        const int64_t tq = (b * T + t) * Hk + h / (H / Hk);  // its query/key head
        float *st = sm + (size_t)t * per_tok;
        float kq = 0.f;
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            const int col = lane * VEC + c;
            const float kc = to_f32<Tin>(k[tq * DK + col]);
            const float qc = scale * to_f32<Tin>(q[tq * DK + col]);
            const float a = expf(PER_CHANNEL ? g[tk * DK + col] : g[tk]);
            st[col] = a * kc;
            st[DK + col] = a * qc;
            st[2 * DK + col] = a;
            st[3 * DK + col] = kc;
            kq += kc * qc;
        }
        for (int r = lane; r < DV; r += 32) st[4 * DK + r] = to_f32<Tin>(v[tk * DV + r]);
        kq = warp_sum(kq);
        if (lane == 0) {
            s_beta[t] = beta[tk];
            s_kq[t] = kq;
        }
    }

    const int row = tid / TPR, part = tid % TPR;
    float4 s[NCH];  // chunk j holds columns 4 (j TPR + part) .. + 3
    float *S = state + (unit * DV + row) * (int64_t)DK + 4 * part;
#pragma unroll
    for (int j = 0; j < NCH; ++j) s[j] = *reinterpret_cast<const float4 *>(S + 4 * j * TPR);
    __syncthreads();

    for (int t = 0; t < n; ++t) {
        const float *st = sm + (size_t)t * per_tok + 4 * part;
        float y[4] = {0.f, 0.f, 0.f, 0.f}, z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
            const float4 ak = *reinterpret_cast<const float4 *>(st + 4 * j * TPR);
            const float4 aq = *reinterpret_cast<const float4 *>(st + DK + 4 * j * TPR);
            y[0] = fmaf(s[j].x, ak.x, y[0]); y[1] = fmaf(s[j].y, ak.y, y[1]);
            y[2] = fmaf(s[j].z, ak.z, y[2]); y[3] = fmaf(s[j].w, ak.w, y[3]);
            z[0] = fmaf(s[j].x, aq.x, z[0]); z[1] = fmaf(s[j].y, aq.y, z[1]);
            z[2] = fmaf(s[j].z, aq.z, z[2]); z[3] = fmaf(s[j].w, aq.w, z[3]);
        }
        float yy = (y[0] + y[1]) + (y[2] + y[3]), zz = (z[0] + z[1]) + (z[2] + z[3]);
#pragma unroll
        for (int o = 1; o < TPR; o <<= 1) {
            yy += __shfl_xor_sync(0xffffffffu, yy, o);
            zz += __shfl_xor_sync(0xffffffffu, zz, o);
        }
        const float d = s_beta[t] * (st[4 * DK - 4 * part + row] - yy);
        const int64_t tk = (b * T + t) * H + h;
        if (part == 0) out[tk * DV + row] = from_f32<Tin>(zz + d * s_kq[t]);
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(st + 2 * DK + 4 * j * TPR);
            const float4 kk = *reinterpret_cast<const float4 *>(st + 3 * DK + 4 * j * TPR);
            s[j].x = fmaf(a.x, s[j].x, d * kk.x);
            s[j].y = fmaf(a.y, s[j].y, d * kk.y);
            s[j].z = fmaf(a.z, s[j].z, d * kk.z);
            s[j].w = fmaf(a.w, s[j].w, d * kk.w);
        }
        if (step_states) {
            float *p = step_states + (tk * DV + row) * (int64_t)DK + 4 * part;
#pragma unroll
            for (int j = 0; j < NCH; ++j) *reinterpret_cast<float4 *>(p + 4 * j * TPR) = s[j];
        }
    }
    if (commit) {
#pragma unroll
        for (int j = 0; j < NCH; ++j) *reinterpret_cast<float4 *>(S + 4 * j * TPR) = s[j];
    }
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
    const size_t smem = ((size_t)d.T * (4 * DK + DV) + 2 * (size_t)d.T) * sizeof(float);
    auto kern = d.gate == GDN_GATE_CHANNEL ? gdn_decode_multi_kernel<DK, DV, Tin, true>
                                           : gdn_decode_multi_kernel<DK, DV, Tin, false>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return check_launch("gdn_decode_multi attributes");
    {
        LaunchScope ls("gdn_decode_multi_kernel", s);
        kern<<<(unsigned)units, kWarps * 32, smem, s>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta,
                                                        n_tokens, state, commit, (Tin *)out, step_states,
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
