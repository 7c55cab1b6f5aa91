// A decode step straight from the layer's raw projections: for the one new token
// of every sequence, the work before the recurrence ("Attention, Part 4: Linear
// Attention, Gated DeltaNet and Hybrid Models", section 6, "Where alpha and beta
// come from" and the paragraph after it: short causal convolution with the
// sequence's history, SiLU, length-1 queries and keys, beta = sigmoid(b),
// g = -exp(A_log) softplus(a + dt_bias)) is done once per (sequence, value head)
// into shared memory, and the recurrence follows in the same kernel ("From
// Traditional Attention to hybrid ones", section 5).  q, k, v, g and beta never reach HBM; a
// second small kernel shifts each sequence's convolution history afterwards, so
// the history can be updated in place.
#include "decode_rows.cuh"

namespace gdn {
namespace {

__device__ __forceinline__ float silu_exact(float y) { return y / (1.f + expf(-y)); }
__device__ __forceinline__ float softplus(float x) { return x > 20.f ? x : log1pf(expf(x)); }

// Channel ch of sequence b after the short convolution and SiLU: tap j < K-1 on
// the history (oldest first), tap K-1 on the token itself.
template <typename Tin, int K>
__device__ __forceinline__ float conv_silu(const Tin *__restrict__ x, const float *__restrict__ w,
                                           const float *__restrict__ hist, int64_t C, int64_t b, int64_t ch) {
    float acc = w[ch * K + (K - 1)] * to_f32<Tin>(x[b * C + ch]);
    if (hist) {
#pragma unroll
        for (int j = 0; j < K - 1; ++j) acc = fmaf(w[ch * K + j], hist[(b * C + ch) * (K - 1) + j], acc);
    }
    return silu_exact(acc);
}

// The token source of decode_rows: the pre-rule results of the block's token in
// shared memory (q and k after SiLU, not yet at length 1; v; alpha, beta).
template <int DK, int DV>
struct SmemSrc {
    const float *qk;  // [2 DK]: q channels, then k channels
    const float *vv;  // [DV]
    float alpha, beta, scale;
    template <int VEC>
    __device__ __forceinline__ void token(int64_t, int, int, int64_t, int64_t, int row0, int lane,
                                          float (&kr)[VEC], float (&qr)[VEC], float (&al)[VEC], float &vb,
                                          float &bt) const {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            qr[c] = qk[lane * VEC + c];
            kr[c] = qk[DK + lane * VEC + c];
            sq = fmaf(qr[c], qr[c], sq);
            sk = fmaf(kr[c], kr[c], sk);
        }
        const float nq = scale * rsqrtf(dec::warp_sum(sq) + 1e-6f), nk = rsqrtf(dec::warp_sum(sk) + 1e-6f);
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            qr[c] *= nq;
            kr[c] *= nk;
            al[c] = alpha;
        }
        vb = lane < 8 ? vv[row0 + lane] : 0.f;
        bt = beta;
    }
};

// One block per (sequence, value head) with a warp per eight state rows: the
// block's threads first do the pre-rule work for the token's q and k channels (of
// the value head's query/key head) and its v channels, one channel per thread,
// into shared memory; then each warp runs the step on its rows.
template <int DK, int DV, typename Tin, int K>
__global__ void __launch_bounds__(DV / 8 * 32)
gdn_decode_prerule_kernel(const Tin *__restrict__ x, const Tin *__restrict__ a, const Tin *__restrict__ b,
                          const float *__restrict__ w, const float *__restrict__ A_log,
                          const float *__restrict__ dt_bias, const float *__restrict__ hist, int64_t C, int64_t H,
                          int64_t Hk, float scale, float *__restrict__ state, Tin *__restrict__ out) {
    __shared__ float qk[2 * DK], vv[DV], gates[2];
    const int64_t unit = blockIdx.x, bs = unit / H, h = unit % H, hq = h / (H / Hk);
    for (int e = threadIdx.x; e < 2 * DK + DV; e += blockDim.x) {
        if (e < DK) qk[e] = conv_silu<Tin, K>(x, w, hist, C, bs, hq * DK + e);
        else if (e < 2 * DK) qk[e] = conv_silu<Tin, K>(x, w, hist, C, bs, (Hk + hq) * DK + e - DK);
        else vv[e - 2 * DK] = conv_silu<Tin, K>(x, w, hist, C, bs, 2 * Hk * DK + h * DV + e - 2 * DK);
    }
    if (threadIdx.x == 0) {
        gates[0] = expf(-expf(A_log[h]) * softplus(to_f32<Tin>(a[unit]) + dt_bias[h]));  // alpha
        gates[1] = 1.f / (1.f + expf(-to_f32<Tin>(b[unit])));                             // beta
    }
    __syncthreads();
    const SmemSrc<DK, DV> src{qk, vv, gates[0], gates[1], scale};
    dec::decode_rows<DK, DV, Tin>(src, state, true, out, nullptr, 1, 1, H);
}

template <int DK, int DV, typename Tin, int K>
gdn_status launch_k(const gdn_desc &d, const PreruleArgs &p, float *state, void *out, cudaStream_t s) {
    const int64_t units = d.B * d.H;
    if (units > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many (sequence, head) pairs");
    const int64_t C = 2 * p.Hk * DK + p.H * DV;
    {
        LaunchScope ls("gdn_decode_prerule_kernel", s);
        gdn_decode_prerule_kernel<DK, DV, Tin, K><<<(unsigned)units, DV / dec::kRowsPerWarp * 32, 0, s>>>(
                (const Tin *)p.x, (const Tin *)p.a, (const Tin *)p.b, p.conv_w, p.A_log, p.dt_bias, p.hist_in, C, d.H,
                p.Hk, d.scale, state, (Tin *)out);
    }
    gdn_status st = check_launch("gdn_decode_prerule_kernel");
    if (st != GDN_OK) return st;
    // the history moves after every block has read it (q/k channels are read by every
    // value head sharing them); shifting it inside the kernel was measured slower
    return launch_prerule_history(p, -1, s);
}

template <int DK, int DV, typename Tin>
gdn_status launch_dkv(const gdn_desc &d, const PreruleArgs &p, float *state, void *out, cudaStream_t s) {
    switch (p.K) {
        case 1: return launch_k<DK, DV, Tin, 1>(d, p, state, out, s);
        case 2: return launch_k<DK, DV, Tin, 2>(d, p, state, out, s);
        case 3: return launch_k<DK, DV, Tin, 3>(d, p, state, out, s);
        case 4: return launch_k<DK, DV, Tin, 4>(d, p, state, out, s);
        default: return fail(GDN_ERR_UNSUPPORTED, "convolution width %d (1 .. 4 supported)", p.K);
    }
}

template <typename Tin>
gdn_status launch_t(const gdn_desc &d, const PreruleArgs &p, float *state, void *out, cudaStream_t s) {
    if (d.dk == 128)
        return d.dv == 128 ? launch_dkv<128, 128, Tin>(d, p, state, out, s) : launch_dkv<128, 64, Tin>(d, p, state, out, s);
    return d.dv == 128 ? launch_dkv<64, 128, Tin>(d, p, state, out, s) : launch_dkv<64, 64, Tin>(d, p, state, out, s);
}

}  // namespace

gdn_status launch_decode_prerule(const gdn_desc &d, const PreruleArgs &p, float *state, void *out, cudaStream_t s) {
    return d.dtype == GDN_BF16 ? launch_t<__nv_bfloat16>(d, p, state, out, s) : launch_t<float>(d, p, state, out, s);
}

}  // namespace gdn
