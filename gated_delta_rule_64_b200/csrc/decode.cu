// Fused single-token decode step of the gated delta rule, state updated in place.
//
// Per (sequence, head) the d_v x d_k fp32 state is streamed from HBM once and
// written back once; everything else (q, k, v, gates, the output) is a few
// hundred bytes.  The kernel is bound by HBM bandwidth.
//
// The recurrence ("From Traditional Attention to hybrid ones", section 5):
// decay, then the delta correction on the decayed state, then the read of the
// updated state.  With a_c = alpha (head gate) or alpha_c (per-channel gate,
// section 7 of the same page), row i of the state evolves independently:
//     y_i  = sum_c S_ic a_c k_c          (what the decayed state predicts for k)
//     z_i  = sum_c S_ic a_c q_c          (the decayed state read by the query)
//     d_i  = beta (v_i - y_i)
//     S'_ic = a_c S_ic + d_i k_c
//     o_i  = z_i + d_i (k . q)           (= (S' q)_i)
// so one warp owns one row at a time: each lane holds d_k/32 consecutive
// columns as a 16-byte (or 8-byte) vector, the two dot products are warp
// reductions, and the row is written back from the same registers.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecodeWarps = 8;
constexpr int kRowsInFlight = 8;  // rows loaded before the first reduction

template <int N> struct FVec;
template <> struct FVec<4> {
    using T = float4;
    static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
        float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <> struct FVec<2> {
    static __device__ __forceinline__ void ld(const float *p, float (&x)[2]) {
        float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = t.x; x[1] = t.y;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[2]) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};

// Load N consecutive input elements (fp32 or bf16) as floats.
template <int N, typename Tin>
__device__ __forceinline__ void load_in(const Tin *p, float (&x)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] = to_f32<Tin>(p[i]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <int DK, typename Tin, bool PER_CHANNEL>
__global__ void __launch_bounds__(kDecodeWarps * 32)
gdn_decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta, float *__restrict__ state,
                  Tin *__restrict__ out, int dv, int64_t H, int64_t Hk, float scale) {
    constexpr int VEC = DK / 32;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t unit = blockIdx.x;  // b * H + h
    const int64_t qu = (unit / H) * Hk + (unit % H) / (H / Hk);  // its query/key head

    float kr[VEC], qr[VEC], a[VEC];
    load_in<VEC>(k + qu * DK + lane * VEC, kr);
    load_in<VEC>(q + qu * DK + lane * VEC, qr);
    if (PER_CHANNEL) {
#pragma unroll
        for (int c = 0; c < VEC; ++c) a[c] = expf(g[unit * DK + lane * VEC + c]);
    } else {
        const float al = expf(g[unit]);
#pragma unroll
        for (int c = 0; c < VEC; ++c) a[c] = al;
    }
    float kq = 0.f;
    float ak[VEC], aq[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
        qr[c] *= scale;
        kq += kr[c] * qr[c];
        ak[c] = a[c] * kr[c];
        aq[c] = a[c] * qr[c];
    }
    kq = warp_sum(kq);
    const float b = beta[unit];

    const int rows_per_warp = dv / kDecodeWarps;  // 16 or 8
    const int row0 = warp * rows_per_warp;
    const float v_mine = lane < rows_per_warp ? to_f32<Tin>(v[unit * dv + row0 + lane]) : 0.f;
    float o_mine = 0.f;
    float *S = state + unit * (int64_t)dv * DK;

    for (int rb = 0; rb < rows_per_warp; rb += kRowsInFlight) {
        float s[kRowsInFlight][VEC];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r)
            if (rb + r < rows_per_warp) FVec<VEC>::ld(S + (int64_t)(row0 + rb + r) * DK + lane * VEC, s[r]);
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            if (rb + r >= rows_per_warp) break;
            float y = 0.f, z = 0.f;
#pragma unroll
            for (int c = 0; c < VEC; ++c) {
                y += s[r][c] * ak[c];
                z += s[r][c] * aq[c];
            }
            y = warp_sum(y);
            z = warp_sum(z);
            const float vi = __shfl_sync(0xffffffffu, v_mine, rb + r);
            const float d = b * (vi - y);
            if (lane == rb + r) o_mine = z + d * kq;
#pragma unroll
            for (int c = 0; c < VEC; ++c) s[r][c] = a[c] * s[r][c] + d * kr[c];
            FVec<VEC>::st(S + (int64_t)(row0 + rb + r) * DK + lane * VEC, s[r]);
        }
    }
    if (lane < rows_per_warp) out[unit * dv + row0 + lane] = from_f32<Tin>(o_mine);
}

template <int DK, typename Tin>
gdn_status launch_dk(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                     const float *beta, float *state, void *out, cudaStream_t s) {
    const int64_t units = d.B * d.H;
    if (units > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many (sequence, head) pairs");
    dim3 grid((unsigned)units), block(kDecodeWarps * 32);
    if (d.gate == GDN_GATE_CHANNEL) {
        LaunchScope ls("gdn_decode_kernel", s);
        gdn_decode_kernel<DK, Tin, true><<<grid, block, 0, s>>>(
            (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, state, (Tin *)out, (int)d.dv, d.H, qk_heads(d),
            d.scale);
    } else {
        LaunchScope ls("gdn_decode_kernel", s);
        gdn_decode_kernel<DK, Tin, false><<<grid, block, 0, s>>>(
            (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, state, (Tin *)out, (int)d.dv, d.H, qk_heads(d),
            d.scale);
    }
    return check_launch("gdn_decode_kernel");
}

}  // namespace

gdn_status launch_decode(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                         const float *beta, float *state, void *out, cudaStream_t s) {
    if (d.dtype == GDN_BF16)
        return d.dk == 128 ? launch_dk<128, __nv_bfloat16>(d, q, k, v, g, beta, state, out, s)
                           : launch_dk<64, __nv_bfloat16>(d, q, k, v, g, beta, state, out, s);
    return d.dk == 128 ? launch_dk<128, float>(d, q, k, v, g, beta, state, out, s)
                       : launch_dk<64, float>(d, q, k, v, g, beta, state, out, s);
}

}  // namespace gdn
