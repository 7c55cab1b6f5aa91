// The work before the recurrence, from the layer's raw projections ("Attention,
// Part 4: Linear Attention, Gated DeltaNet and Hybrid Models", section 6, "Where
// alpha and beta come from" and the paragraph after it; "From Traditional
// Attention to hybrid ones", "vLLM Storage", for the convolution history a live
// sequence keeps):
//   y = SiLU(causal depthwise convolution of the last K tokens), per channel of
//       the mixed [q heads | k heads | v heads] projection;
//   q, k = y / sqrt(|y|^2 + 1e-6) per head;  v = y;
//   beta = sigmoid(b);  g = -exp(A_log) softplus(a + dt_bias)  (per value head).
// Tap j of a channel's K weights multiplies the input K-1-j tokens back; inputs
// before a sequence's first token come from its convolution history (the last
// K-1 raw inputs, oldest first; zeros when none is given).
//
// One block per (64-token tile, head): the block copies the head's channels of
// the tile's rows and of the K-1 rows before them into shared memory with 16-byte
// loads; then a thread takes (token, 8 channels), reads its K input rows from
// shared memory (from the sequence's history where a row lies before the
// sequence's start), and writes 8 outputs with one 16-byte store.  A query/key
// head's length is a reduction over the 16 (or 8) threads of its token.  The
// value-head blocks also compute beta and g for their tokens.  A second kernel
// writes each sequence's new history.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kTok = 64;       // tokens per block
constexpr int kThreads = 256;
constexpr int kMaxK = 4;

// SiLU with the hardware exponential and reciprocal (relative error ~1e-6).
__device__ __forceinline__ float silu(float y) { return __fdividef(y, 1.f + __expf(-y)); }
__device__ __forceinline__ float softplus(float x) { return x > 20.f ? x : log1pf(expf(x)); }

// Sequence of packed row r: n with cu[n] <= r < cu[n+1] (false if r is in none).
__device__ __forceinline__ bool find_seq(const int32_t *cu, int64_t N, int64_t T, int64_t r, int64_t &n,
                                         int64_t &start, int64_t &len) {
    if (!cu) {
        n = r / T;
        start = n * T;
        len = T;
        return n < N;
    }
    if (N <= 0 || r < cu[0] || r >= cu[N]) return false;
    int64_t lo = 0, hi = N;  // largest n with cu[n] <= r (skips empty sequences)
    while (hi - lo > 1) {
        const int64_t mid = (lo + hi) / 2;
        if (cu[mid] <= r) lo = mid; else hi = mid;
    }
    n = lo;
    start = cu[n];
    len = cu[n + 1] - start;
    return true;
}

// 8 consecutive elements as floats / from floats (16 bytes of bf16, 32 of fp32).
template <typename Tin> __device__ __forceinline__ void load8(const Tin *p, float *f);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float *f) {
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
template <> __device__ __forceinline__ void load8<float>(const float *p, float *f) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
template <typename Tin> __device__ __forceinline__ void store8(Tin *p, const float *f);
template <> __device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *p, const float *f) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        u[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(u[0], u[1], u[2], u[3]);
}
template <> __device__ __forceinline__ void store8<float>(float *p, const float *f) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

template <typename Tin, int K>
__global__ void __launch_bounds__(kThreads)
gdn_prerule_kernel(const Tin *__restrict__ x, const Tin *__restrict__ a, const Tin *__restrict__ b,
                   const float *__restrict__ w, const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                   const int32_t *__restrict__ cu, int64_t N, int64_t T, int64_t rows, int64_t Hk, int64_t H,
                   int dk, int dv, const float *__restrict__ hist, Tin *__restrict__ q, Tin *__restrict__ k,
                   Tin *__restrict__ v, float *__restrict__ g, float *__restrict__ beta) {
    // rows r0 - (K-1) .. r1 - 1 of the head's channels (up to 128), as floats; a row
    // holds the first 4 channels of every 8-channel chunk, then the last 4, and 4
    // floats of padding, so the 16-byte reads of a warp (two rows, 16 chunks) hit
    // distinct banks
    constexpr int kRow = 132;
    __shared__ __align__(16) float tile[(kTok + kMaxK - 1) * kRow];
    __shared__ __align__(16) float ws[128 * kMaxK];  // the head's taps, [channel][tap]
    const int64_t C = 2 * Hk * dk + H * dv;
    const int64_t hh = blockIdx.x;  // heads vary fastest: blocks in flight share their token rows
    const int kind = hh < Hk ? 0 : (hh < 2 * Hk ? 1 : 2);  // q, k or v head
    const int64_t head = kind == 0 ? hh : (kind == 1 ? hh - Hk : hh - 2 * Hk);
    const int d = kind < 2 ? dk : dv;
    const int64_t ch0 = kind == 0 ? head * dk : (kind == 1 ? (Hk + head) * dk : 2 * Hk * dk + head * dv);
    const int64_t r0 = (int64_t)blockIdx.y * kTok, r1 = r0 + kTok < rows ? r0 + kTok : rows;
    const int tid = threadIdx.x;
    const int lc = d == 128 ? 4 : 3, cpr = 1 << lc;  // 8-channel chunks per row: 16 or 8
    const int64_t base = r0 - (K - 1);
    const int nrow = (int)(r1 - base);

    for (int e = tid; e < d * K; e += kThreads) ws[e] = w[ch0 * K + e];
    // stage the rows (16-byte loads, coalesced along the channels)
    {
        const Tin *xs = x + base * C + ch0;
        for (int e = tid; e < nrow * cpr; e += kThreads) {
            const int i = e >> lc, cc = e & (cpr - 1);
            float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (base + i >= 0) load8<Tin>(xs + (int64_t)i * C + 8 * cc, f);
            *reinterpret_cast<float4 *>(&tile[i * kRow + 4 * cc]) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4 *>(&tile[i * kRow + 64 + 4 * cc]) = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
    __syncthreads();

    Tin *dst = kind == 0 ? q : (kind == 1 ? k : v);
    const int64_t hstride = kind < 2 ? Hk : H;
    // a thread keeps one chunk (8 channels) for all its tokens: their K taps, loaded once
    const int cc = tid & (cpr - 1);
    float wt[8][K];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int j = 0; j < K; ++j) wt[u][j] = ws[(8 * cc + u) * K + j];
    // the sequence of the tile's first row; later rows look it up again only past its end
    int64_t n = 0, start = 0, len = 0;
    bool have = find_seq(cu, N, T, r0, n, start, len);
    // tokens ti of this thread (the cpr threads of a token are an aligned lane group;
    // every lane runs the same number of iterations)
    for (int ti = tid >> lc; ti < kTok; ti += kThreads >> lc) {
        const int64_t r = r0 + ti;
        bool in_seq = false;
        if (r < r1) {
            if (!(have && r >= start && r < start + len)) have = find_seq(cu, N, T, r, n, start, len);
            in_seq = have;
        }
        float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (in_seq) {
            const int p = (int)(r - start < K ? r - start : K);  // only p < K - 1 reads the history
            if (p >= K - 1) {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const float4 lo = *reinterpret_cast<const float4 *>(&tile[(ti + j) * kRow + 4 * cc]);
                    const float4 hi = *reinterpret_cast<const float4 *>(&tile[(ti + j) * kRow + 64 + 4 * cc]);
                    const float in[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int u = 0; u < 8; ++u) y[u] = fmaf(wt[u][j], in[u], y[u]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int pj = p - (K - 1) + j;  // position of the input this tap reads
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float in = pj >= 0 ? tile[(ti + j) * kRow + (u < 4 ? 4 * cc + u : 64 + 4 * cc + u - 4)]
                                                 : (hist ? hist[(n * C + ch0 + 8 * cc + u) * (K - 1) + (K - 1) + pj] : 0.f);
                        y[u] = fmaf(wt[u][j], in, y[u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] = silu(y[u]);
        }
        if (kind < 2) {  // length 1 per query/key head: the token's cpr threads (aligned lane groups)
            float ss = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) ss = fmaf(y[u], y[u], ss);
            for (int o = 1; o < cpr; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float sc = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] *= sc;
        }
        if (in_seq) store8<Tin>(dst + (r * hstride + head) * d + 8 * cc, y);
    }

    // gates of this value head for the tile's tokens
    if (kind == 2) {
        for (int64_t r = r0 + tid; r < r1; r += kThreads) {
            int64_t sn, ss, sl;
            if (find_seq(cu, N, T, r, sn, ss, sl)) {
                const int64_t e = r * H + head;
                beta[e] = 1.f / (1.f + expf(-to_f32<Tin>(b[e])));
                g[e] = -expf(A_log[head]) * softplus(to_f32<Tin>(a[e]) + dt_bias[head]);
            }
        }
    }
}

// New history of sequence n: its last K-1 raw inputs (older history where the
// sequence is shorter).  Each thread reads all it needs before writing, so
// hist_out may be hist_in.
template <typename Tin, int K>
__global__ void gdn_prerule_history(const Tin *__restrict__ x, const int32_t *__restrict__ cu, int64_t N, int64_t T,
                                    int64_t C, const float *hist_in, float *hist_out) {
    const int64_t n = blockIdx.x, ch = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
    if (ch >= C || K < 2) return;
    int64_t start, len;
    if (cu) {
        start = cu[n];
        len = cu[n + 1] - start;
    } else {
        start = n * T;
        len = T;
    }
    float nv[K > 1 ? K - 1 : 1];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t p = len - (K - 1) + j;
        nv[j] = p >= 0 ? to_f32<Tin>(x[(start + p) * C + ch])
                       : (hist_in ? hist_in[(n * C + ch) * (K - 1) + (K - 1) + p] : 0.f);
    }
#pragma unroll
    for (int j = 0; j < K - 1; ++j) hist_out[(n * C + ch) * (K - 1) + j] = nv[j];
}

template <typename Tin, int K>
gdn_status launch_k(const PreruleArgs &a, cudaStream_t s) {
    const int64_t C = 2 * a.Hk * a.dk + a.H * a.dv;
    if (a.rows > 0) {
        const int64_t tiles = (a.rows + kTok - 1) / kTok;
        if (tiles > 65535 || 2 * a.Hk + a.H > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
        LaunchScope ls("gdn_prerule_kernel", s);
        gdn_prerule_kernel<Tin, K><<<dim3((unsigned)(2 * a.Hk + a.H), (unsigned)tiles), kThreads, 0, s>>>(
            (const Tin *)a.x, (const Tin *)a.a, (const Tin *)a.b, a.conv_w, a.A_log, a.dt_bias, a.cu_seqlens, a.N,
            a.T, a.rows, a.Hk, a.H, (int)a.dk, (int)a.dv, a.hist_in, (Tin *)a.q, (Tin *)a.k, (Tin *)a.v, a.g,
            a.beta);
    }
    gdn_status st = check_launch("gdn_prerule_kernel");
    if (st != GDN_OK || !a.hist_out || K < 2 || a.N == 0) return st;
    {
        LaunchScope ls("gdn_prerule_history", s);
        gdn_prerule_history<Tin, K><<<dim3((unsigned)a.N, (unsigned)((C + 255) / 256)), 256, 0, s>>>(
            (const Tin *)a.x, a.cu_seqlens, a.N, a.T, C, a.hist_in, a.hist_out);
    }
    return check_launch("gdn_prerule_history");
}

template <typename Tin>
gdn_status launch_t(const PreruleArgs &a, cudaStream_t s) {
    switch (a.K) {
        case 1: return launch_k<Tin, 1>(a, s);
        case 2: return launch_k<Tin, 2>(a, s);
        case 3: return launch_k<Tin, 3>(a, s);
        case 4: return launch_k<Tin, 4>(a, s);
        default: return fail(GDN_ERR_UNSUPPORTED, "convolution width %d (1 .. 4 supported)", a.K);
    }
}

}  // namespace

gdn_status launch_prerule(const PreruleArgs &a, cudaStream_t s) {
    return a.dtype == GDN_BF16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdn
