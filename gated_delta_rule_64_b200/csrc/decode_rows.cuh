// Decode of a few tokens per (sequence, head) with the fp32 state in
// registers: the device code shared by the single-token step and the
// multi-token call.
//
// The recurrence per token ("From Traditional Attention to hybrid ones", section
// 5): decay, the delta correction on the decayed state, then the read of the
// updated state.  With a_c = alpha (head gate) or alpha_c (per-channel gate,
// section 7 of the same page), row i of the d_v x d_k state evolves on its own:
//     y_i  = sum_c S_ic a_c k_c          (what the decayed state predicts for k)
//     z_i  = sum_c S_ic a_c q_c          (the decayed state read by the query)
//     d_i  = beta (v_i - y_i)
//     S'_ic = a_c S_ic + d_i k_c
//     o_i  = z_i + d_i (k . q)           (= (S' q)_i)
#pragma once

#include "gdn_internal.cuh"

namespace gdn {
namespace dec {

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

// Where a token's vectors come from: the q, k, v, gate and beta arrays.
// token() gives lane l's columns l VEC .. l VEC + VEC - 1 of k and of scale * q and
// the decay a = exp(g) on them, v of row row0 + l (lanes 0 .. 7) and beta.
template <int DK, int DV, typename Tin, bool PER_CHANNEL>
struct ArraySrc {
    const Tin *q, *k, *v;
    const float *g, *beta;
    int64_t Hk;
    float scale;
    template <int VEC>
    __device__ __forceinline__ void token(int64_t b, int t, int T, int64_t H, int64_t h, int row0, int lane,
                                          float (&kr)[VEC], float (&qr)[VEC], float (&a)[VEC], float &vb,
                                          float &bt) const {
        const int64_t tk = (b * T + t) * H + h;             // (b, t, h)
        const int64_t tq = (b * T + t) * Hk + h / (H / Hk);  // its query/key head
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
        vb = lane < 8 ? to_f32<Tin>(v[tk * DV + row0 + lane]) : 0.f;
        bt = beta[tk];
    }
};

// Warp w of block (unit, y) owns rows 8 (y W + w) .. + 7 of the unit's state (W warps
// per block; the decode kernels use 4, i.e. 32 rows per block); lane l
// holds columns l VEC .. l VEC + VEC - 1 of those rows in registers (one
// coalesced row per load / store instruction).  Per token the lane takes its
// columns of k, q and the decay from `src` straight into registers (the same for
// all eight rows), the eight rows' dot products are reduce-scattered over the
// warp, and each row's correction d is broadcast back for the update.
//   tokens n (<= T) of unit = b H + h, outputs laid out (B, T, H, d_v);
//   commit: write the state back; step_states: (B, T, H, d_v, d_k) or nullptr.
template <int DK, int DV, typename Tin, typename Src>
__device__ __forceinline__ void decode_rows(const Src &src, float *__restrict__ state, bool commit,
                                            Tin *__restrict__ out, float *__restrict__ step_states, int n, int T,
                                            int64_t H) {
    constexpr int VEC = DK / 32;
    static_assert(DV % (kWarps * kRowsPerWarp) == 0, "layout");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t unit = blockIdx.x, b = unit / H, h = unit % H;
    const int row0 = ((int)blockIdx.y * (int)(blockDim.x >> 5) + warp) * kRowsPerWarp;  // eight rows per warp
    float *S = state + (unit * DV + row0) * (int64_t)DK + lane * VEC;
    float s[kRowsPerWarp][VEC];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) Vec4<VEC>::ld(S + (int64_t)r * DK, s[r]);
    const int R = (lane >> 2) & 7;  // the row whose reduced sums this lane receives

    for (int t = 0; t < n; ++t) {
        const int64_t tk = (b * T + t) * H + h;  // (b, t, h)
        float kr[VEC], qr[VEC], a[VEC], vb, bt;
        src.template token<VEC>(b, t, T, H, h, row0, lane, kr, qr, a, vb, bt);
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

}  // namespace dec
}  // namespace gdn
