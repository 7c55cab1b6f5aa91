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
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kWarps = 4;        // warps per block
constexpr int kRowsPerWarp = 8;  // state rows of one warp (a block: 32 rows)

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Sums over the 32 lanes of eight per-lane values x[0..7] (one per row), left
// reduce-scattered: lane l returns the total of row (l >> 2) & 7.  Nine shuffles
// instead of 40 for eight separate reductions.
__device__ __forceinline__ float reduce8(const float (&x)[8], int lane) {
    float a[4], b2[2];
    const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = (u16 ? x[i + 4] : x[i]) + __shfl_xor_sync(0xffffffffu, u16 ? x[i] : x[i + 4], 16);
#pragma unroll
    for (int i = 0; i < 2; ++i) b2[i] = (u8 ? a[i + 2] : a[i]) + __shfl_xor_sync(0xffffffffu, u8 ? a[i] : a[i + 2], 8);
    float c = (u4 ? b2[1] : b2[0]) + __shfl_xor_sync(0xffffffffu, u4 ? b2[0] : b2[1], 4);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    return c;
}

template <int VEC> struct Vec4;
template <> struct Vec4<4> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
        const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <> struct Vec4<2> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[2]) {
        const float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = t.x; x[1] = t.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[2]) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};

// Warp w of block (unit, y) owns rows 32 y + 8 w .. + 7 of the unit's state; lane l
// holds columns l VEC .. l VEC + VEC - 1 of those rows in registers (one
// coalesced row per load / store instruction).  Per token the lane reads its
// columns of k, q and the gate straight into registers (the same for all eight
// rows), the eight rows' dot products are reduce-scattered over the warp, and each
// row's correction d is broadcast back for the update.
template <int DK, int DV, typename Tin, bool PER_CHANNEL>
__global__ void __launch_bounds__(kWarps * 32)
gdn_decode_multi_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                        const float *__restrict__ g, const float *__restrict__ beta,
                        const int32_t *__restrict__ n_tokens, float *__restrict__ state, int commit,
                        Tin *__restrict__ out, float *__restrict__ step_states, int T, int64_t H, int64_t Hk,
                        float scale) {
    constexpr int VEC = DK / 32;
    static_assert(DV % (kWarps * kRowsPerWarp) == 0, "layout");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t unit = blockIdx.x, b = unit / H, h = unit % H;
    int n = T;
    if (n_tokens) {
        n = n_tokens[b];
        n = n < 0 ? 0 : (n > T ? T : n);
    }
    if (n == 0) return;
    const int row0 = (int)blockIdx.y * (kWarps * kRowsPerWarp) + warp * kRowsPerWarp;
    float *S = state + (unit * DV + row0) * (int64_t)DK + lane * VEC;
    float s[kRowsPerWarp][VEC];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) Vec4<VEC>::ld(S + (int64_t)r * DK, s[r]);
    const int R = (lane >> 2) & 7;  // the row whose reduced sums this lane receives

    for (int t = 0; t < n; ++t) {
        const int64_t tk = (b * T + t) * H + h;             // (b, t, h)
        const int64_t tq = (b * T + t) * Hk + h / (H / Hk);  // its query/key head
        float kr[VEC], qr[VEC], a[VEC];
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            kr[c] = to_f32<Tin>(k[tq * DK + lane * VEC + c]);
            qr[c] = scale * to_f32<Tin>(q[tq * DK + lane * VEC + c]);
        }
        if (PER_CHANNEL) {
#pragma unroll
            for (int c = 0; c < VEC; ++c) a[c] = expf(g[tk * DK + lane * VEC + c]);
        } else {
            const float al = expf(g[tk]);
#pragma unroll
            for (int c = 0; c < VEC; ++c) a[c] = al;
        }
        const float vb = lane < kRowsPerWarp ? to_f32<Tin>(v[tk * DV + row0 + lane]) : 0.f;
        const float bt = beta[tk];
        float kq = 0.f;
#pragma unroll
        for (int c = 0; c < VEC; ++c) kq = fmaf(kr[c], qr[c], kq);
        kq = warp_sum(kq);
        // what the decayed state predicts for k, and its read by q, for the eight rows
        float yp[kRowsPerWarp], zp[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            float y = 0.f, z = 0.f;
#pragma unroll
            for (int c = 0; c < VEC; ++c) {
                const float sa = s[r][c] * a[c];
                y = fmaf(sa, kr[c], y);
                z = fmaf(sa, qr[c], z);
            }
            yp[r] = y;
            zp[r] = z;
        }
        const float y = reduce8(yp, lane), z = reduce8(zp, lane);
        const float d = bt * (__shfl_sync(0xffffffffu, vb, R) - y);
        if ((lane & 3) == 0) out[tk * DV + row0 + R] = from_f32<Tin>(z + d * kq);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const float dr = __shfl_sync(0xffffffffu, d, 4 * r);
#pragma unroll
            for (int c = 0; c < VEC; ++c) s[r][c] = fmaf(a[c], s[r][c], dr * kr[c]);
        }
        if (step_states) {
            float *p = step_states + (tk * DV + row0) * (int64_t)DK + lane * VEC;
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) Vec4<VEC>::st(p + (int64_t)r * DK, s[r]);
        }
    }
    if (commit) {
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) Vec4<VEC>::st(S + (int64_t)r * DK, s[r]);
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
