// Fused single-token decode step of the gated delta rule, state updated in place.
//
// Per (sequence, head) the d_v x d_k fp32 state is streamed from HBM once and
// written back once; everything else (q, k, v, gates, the output) is a few
// hundred bytes.  The kernel is bound by HBM bandwidth.  The recurrence and the
// row-parallel layout (a warp per eight state rows, a lane per d_k / 32 columns,
// the eight rows' dot products reduce-scattered over the warp) are those of
// decode_rows.cuh, here with one token.
#include "decode_rows.cuh"

namespace gdn {
namespace {

// One token per (sequence, head): the row-parallel decode of decode_rows with a
// single token, the state written back in place.
template <int DK, int DV, typename Tin, bool PER_CHANNEL>
__global__ void __launch_bounds__(dec::kWarps * 32)
gdn_decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta, float *__restrict__ state,
                  Tin *__restrict__ out, int64_t H, int64_t Hk, float scale) {
    const dec::ArraySrc<DK, DV, Tin, PER_CHANNEL> src{q, k, v, g, beta, Hk, scale};
    dec::decode_rows<DK, DV, Tin>(src, state, true, out, nullptr, 1, 1, H);
}

template <int DK, int DV, typename Tin>
gdn_status launch_dkv(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state, void *out, cudaStream_t s) {
    const int64_t units = d.B * d.H;
    if (units > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many (sequence, head) pairs");
    const dim3 grid((unsigned)units, (unsigned)(DV / (dec::kWarps * dec::kRowsPerWarp))), block(dec::kWarps * 32);
    auto kern = d.gate == GDN_GATE_CHANNEL ? gdn_decode_kernel<DK, DV, Tin, true> : gdn_decode_kernel<DK, DV, Tin, false>;
    {
        LaunchScope ls("gdn_decode_kernel", s);
        kern<<<grid, block, 0, s>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, state, (Tin *)out, d.H,
                                    qk_heads(d), d.scale);
    }
    return check_launch("gdn_decode_kernel");
}

template <typename Tin>
gdn_status launch_t(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                    const float *beta, float *state, void *out, cudaStream_t s) {
    if (d.dk == 128)
        return d.dv == 128 ? launch_dkv<128, 128, Tin>(d, q, k, v, g, beta, state, out, s)
                           : launch_dkv<128, 64, Tin>(d, q, k, v, g, beta, state, out, s);
    return d.dv == 128 ? launch_dkv<64, 128, Tin>(d, q, k, v, g, beta, state, out, s)
                       : launch_dkv<64, 64, Tin>(d, q, k, v, g, beta, state, out, s);
}

}  // namespace

gdn_status launch_decode(const gdn_desc &d, const void *q, const void *k, const void *v, const float *g,
                         const float *beta, float *state, void *out, cudaStream_t s) {
    return d.dtype == GDN_BF16 ? launch_t<__nv_bfloat16>(d, q, k, v, g, beta, state, out, s)
                               : launch_t<float>(d, q, k, v, g, beta, state, out, s);
}

}  // namespace gdn
