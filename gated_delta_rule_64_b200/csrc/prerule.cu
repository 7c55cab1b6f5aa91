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
// One block per (head, span of kTiles x 64 rows).  The block stages a tile's rows
// (the head's channels, with the K-1 rows before the tile) in shared memory with
// asynchronous 16-byte copies, the next tile's copies in flight while the current
// one is worked on.  Thread (chunk c, token lane l) takes channels 8c .. 8c+7 and
// the consecutive tokens l*m .. l*m+m-1 of the tile: it keeps its K taps and the
// last K-1 inputs in registers and reads one new row per token.  A query/key
// head's length is a reduction over the d/8 lanes of a token (an aligned lane
// group).  The first K-1 tokens of a sequence read the taps before it from its
// history (fp32).  Value-head blocks also compute beta and g for their rows.  A
// second kernel writes each sequence's new history.
#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;

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

// 8 consecutive elements from floats (16 bytes of bf16, 32 of fp32).
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

constexpr int kTile = 64;   // rows per tile
constexpr int kTiles = 8;   // tiles per block
constexpr int kStages = 4;  // staged tiles (up to kStages - 1 in flight ahead of the current one)
constexpr int kMaxK = 4;

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    // (an invalid source is not read: the 16 bytes are zero-filled)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 8 consecutive elements of a staged row, kept as loaded (bf16 pairs or floats).
template <typename Tin> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint32_t u[4];
    __device__ __forceinline__ void lds(const __nv_bfloat16 *p) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        u[0] = w.x; u[1] = w.y; u[2] = w.z; u[3] = w.w;
    }
    __device__ __forceinline__ float at(int e) const {
        return __uint_as_float((e & 1) ? (u[e >> 1] & 0xffff0000u) : (u[e >> 1] << 16));
    }
};
template <> struct Raw8<float> {
    float f[8];
    __device__ __forceinline__ void lds(const float *p) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    __device__ __forceinline__ float at(int e) const { return f[e]; }
};

// SiLU for the bf16 path: y sigma(y) = y/2 (1 + tanh(y/2)) with the hardware
// tanh (relative error about 2^-11, below the bf16 rounding of the result).
__device__ __forceinline__ float silu_tanh(float y) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * y));
    const float h = 0.5f * y;
    return fmaf(h, t, h);
}

// The tiles of one block for a head of CPR 8-channel chunks (d = 8 CPR).
template <typename Tin, int K, int CPR>
__device__ __forceinline__ void prerule_tiles(const Tin *__restrict__ x, const float *__restrict__ w,
                                              const int32_t *__restrict__ cu, int64_t N, int64_t T, int64_t rows,
                                              int64_t C, int64_t ch0, const float *__restrict__ hist, Tin *__restrict__ out,
                                              int64_t ostride, bool normalise, Tin *stage, int64_t span0) {
    constexpr int d = 8 * CPR, kEpc = 16 / (int)sizeof(Tin), kCpy = d / kEpc;  // 16-byte copies per row
    constexpr int kRows = kTile + K - 1;                                        // staged rows per tile
    constexpr int M = kTile * CPR / kThreads;                                   // consecutive tokens per thread
    static_assert((kCpy & (kCpy - 1)) == 0 && M >= 1, "layout");
    const int tid = threadIdx.x, lane = tid & 31;
    const int cc = tid & (CPR - 1), tl = tid / CPR;
    const unsigned gmask = ((1u << CPR) - 1u) << (lane & ~(CPR - 1));

    auto issue = [&](int t) {  // stage tile t of the span (one commit group, empty past the span)
        const int64_t base = span0 + (int64_t)t * kTile - (K - 1);
        Tin *sb = stage + (size_t)(t % kStages) * kRows * d;
        if (t < kTiles && span0 + (int64_t)t * kTile < rows) {
            const Tin *src = x + base * C + ch0;
            for (int e = tid; e < kRows * kCpy; e += kThreads) {
                const int i = e / kCpy, c = e % kCpy;
                const bool ok = base + i >= 0 && base + i < rows;
                cp_async16(sb + i * d + c * kEpc, ok ? (const void *)(src + i * C + c * kEpc) : (const void *)x, ok);
            }
        }
        cp_async_commit();
    };

    float wt[8][K];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int j = 0; j < K; ++j) wt[u][j] = w[(ch0 + 8 * cc + u) * K + j];
    const float *hrow = hist ? hist + (ch0 + 8 * cc) * (K - 1) : nullptr;  // + n C (K-1): this lane's channels
    Tin *obase = out + 8 * cc;

    int32_t n = 0, start = 0, len = 0;  // the current row's sequence (rows < 2^31)
    bool have = false;
#pragma unroll 1
    for (int t = 0; t < kStages - 1; ++t) issue(t);
#pragma unroll 1
    for (int t = 0; t < kTiles; ++t) {
        const int64_t t0 = span0 + (int64_t)t * kTile;
        if (t0 >= rows) break;  // (uniform over the block)
        cp_async_wait<kStages - 2>();  // tile t has landed (later tiles may still be in flight)
        __syncthreads();
        const Tin *sb = stage + (size_t)(t % kStages) * kRows * d + 8 * cc + tl * M * d;
        Raw8<Tin> win[kMaxK - 1];  // inputs of the K-1 rows before the current token
#pragma unroll
        for (int j = 0; j < K - 1; ++j) win[j].lds(sb + j * d);
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const int32_t r = (int32_t)t0 + tl * M + i;
            Raw8<Tin> cur;
            cur.lds(sb + (i + K - 1) * d);
            bool in_seq = false;
            if (r < rows) {
                if (!(have && r >= start && r - start < len)) {
                    int64_t n64, s64, l64;
                    have = find_seq(cu, N, T, r, n64, s64, l64);
                    n = (int32_t)n64;
                    start = (int32_t)s64;
                    len = (int32_t)l64;
                }
                in_seq = have;
            }
            float y[8];
            const int32_t p = r - start;
            if (in_seq && p >= K - 1) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float acc = wt[u][K - 1] * cur.at(u);
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) acc = fmaf(wt[u][j], win[j].at(u), acc);
                    y[u] = acc;
                }
            } else {  // the sequence's first K-1 tokens: taps before it read its history
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float acc = wt[u][K - 1] * cur.at(u);
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) {
                        const int32_t pos = p - (K - 1) + j;
                        const float in = pos >= 0 ? win[j].at(u)
                                                  : (hrow ? hrow[(int64_t)n * C * (K - 1) + u * (K - 1) + (K - 1) + pos] : 0.f);
                        acc = fmaf(wt[u][j], in, acc);
                    }
                    y[u] = in_seq ? acc : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] = sizeof(Tin) == 2 ? silu_tanh(y[u]) : silu(y[u]);
#pragma unroll
            for (int j = 0; j + 1 < K - 1; ++j) win[j] = win[j + 1];
            if (K > 1) win[K > 1 ? K - 2 : 0] = cur;
            if (normalise) {  // length 1 per query/key head
                float ss = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) ss = fmaf(y[u], y[u], ss);
#pragma unroll
                for (int o = 1; o < CPR; o <<= 1) ss += __shfl_xor_sync(gmask, ss, o);
                const float sc = rsqrtf(ss + 1e-6f);
#pragma unroll
                for (int u = 0; u < 8; ++u) y[u] *= sc;
            }
            if (in_seq) store8<Tin>(obase + (int64_t)r * ostride, y);
        }
        __syncthreads();         // every thread is done with buffer t % kStages ...
        issue(t + kStages - 1);  // ... which now takes tile t + kStages - 1
    }
    cp_async_wait<0>();
}

// (bf16: 3 blocks per multiprocessor; fp32 stages take 137 KB of shared memory: 1)
template <typename Tin, int K>
__global__ void __launch_bounds__(kThreads, sizeof(Tin) == 2 ? 3 : 1)
gdn_prerule_kernel(const Tin *__restrict__ x, const Tin *__restrict__ a, const Tin *__restrict__ b,
                   const float *__restrict__ w, const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                   const int32_t *__restrict__ cu, int64_t N, int64_t T, int64_t rows, int64_t Hk, int64_t H,
                   int dk, int dv, const float *__restrict__ hist, Tin *__restrict__ q, Tin *__restrict__ k,
                   Tin *__restrict__ v, float *__restrict__ g, float *__restrict__ beta) {
    extern __shared__ float4 pr_raw[];
    Tin *stage = reinterpret_cast<Tin *>(pr_raw);  // [kStages][kTile + K - 1][d]
    const int64_t C = 2 * Hk * dk + H * dv;
    const int64_t hh = blockIdx.x;  // heads vary fastest: blocks in flight share their rows
    const int kind = hh < Hk ? 0 : (hh < 2 * Hk ? 1 : 2);  // q, k or v head
    const int64_t head = kind == 0 ? hh : (kind == 1 ? hh - Hk : hh - 2 * Hk);
    const int d = kind < 2 ? dk : dv;
    const int64_t ch0 = kind == 0 ? head * dk : (kind == 1 ? (Hk + head) * dk : 2 * Hk * dk + head * dv);
    Tin *dst = (kind == 0 ? q : (kind == 1 ? k : v)) + head * d;
    const int64_t ostride = (kind < 2 ? Hk : H) * d;  // elements from one row to the next
    const int64_t span0 = (int64_t)blockIdx.y * kTile * kTiles;
    if (d == 128)
        prerule_tiles<Tin, K, 16>(x, w, cu, N, T, rows, C, ch0, hist, dst, ostride, kind < 2, stage, span0);
    else
        prerule_tiles<Tin, K, 8>(x, w, cu, N, T, rows, C, ch0, hist, dst, ostride, kind < 2, stage, span0);

    // a value head: beta and g of the span's rows
    if (kind == 2) {
        const int64_t r1 = span0 + kTile * kTiles < rows ? span0 + kTile * kTiles : rows;
        const float A = expf(A_log[head]), dtb = dt_bias[head];
        for (int64_t r = span0 + threadIdx.x; r < r1; r += kThreads) {
            int64_t sn, ss, sl;
            if (find_seq(cu, N, T, r, sn, ss, sl)) {
                const int64_t e = r * H + head;
                beta[e] = 1.f / (1.f + expf(-to_f32<Tin>(b[e])));
                g[e] = -A * softplus(to_f32<Tin>(a[e]) + dtb);
            }
        }
    }
}

// New history of sequence n: its last K-1 raw inputs (older history where the
// sequence is shorter).  Each thread reads all it needs before writing, so
// hist_out may be hist_in.
template <typename Tin, int K>
__global__ void gdn_prerule_history(const Tin *__restrict__ x, const int32_t *__restrict__ cu, int64_t N, int64_t T,
                                    int64_t C, int64_t Cn, const float *hist_in, float *hist_out) {
    // channels [0, Cn) of rows of C channels
    const int64_t n = blockIdx.x, ch = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
    if (ch >= Cn || K < 2) return;
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
        const int dmax = a.dk > a.dv ? (int)a.dk : (int)a.dv;
        const size_t smem = kStages * (size_t)(kTile + K - 1) * dmax * sizeof(Tin);
        auto kern = gdn_prerule_kernel<Tin, K>;
        static std::once_flag once;
        static cudaError_t attr = cudaSuccess;
        std::call_once(once, [&] {
            attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(kStages * (kTile + K - 1) * 128 * sizeof(Tin)));
            if (attr == cudaSuccess)
                attr = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                            (int)cudaSharedmemCarveoutMaxShared);
        });
        if (attr != cudaSuccess) return fail(GDN_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(attr));
        const int64_t spans = (a.rows + kTile * kTiles - 1) / (kTile * kTiles);
        if (spans > 65535 || 2 * a.Hk + a.H > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
        LaunchScope ls("gdn_prerule_kernel", s);
        kern<<<dim3((unsigned)(2 * a.Hk + a.H), (unsigned)spans), kThreads, smem, s>>>(
            (const Tin *)a.x, (const Tin *)a.a, (const Tin *)a.b, a.conv_w, a.A_log, a.dt_bias, a.cu_seqlens, a.N,
            a.T, a.rows, a.Hk, a.H, (int)a.dk, (int)a.dv, a.hist_in, (Tin *)a.q, (Tin *)a.k, (Tin *)a.v, a.g,
            a.beta);
    }
    gdn_status st = check_launch("gdn_prerule_kernel");
    if (st != GDN_OK || !a.hist_out || K < 2 || a.N == 0) return st;
    {
        LaunchScope ls("gdn_prerule_history", s);
        gdn_prerule_history<Tin, K><<<dim3((unsigned)a.N, (unsigned)((C + 255) / 256)), 256, 0, s>>>(
            (const Tin *)a.x, a.cu_seqlens, a.N, a.T, C, C, a.hist_in, a.hist_out);
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

namespace {
template <typename Tin, int K>
gdn_status launch_history_k(const PreruleArgs &a, int64_t channels, cudaStream_t s) {
    const int64_t C = 2 * a.Hk * a.dk + a.H * a.dv, Cn = channels < 0 || channels > C ? C : channels;
    if (!a.hist_out || K < 2 || a.N == 0 || Cn == 0) return GDN_OK;
    {
        LaunchScope ls("gdn_prerule_history", s);
        gdn_prerule_history<Tin, K><<<dim3((unsigned)a.N, (unsigned)((Cn + 255) / 256)), 256, 0, s>>>(
            (const Tin *)a.x, a.cu_seqlens, a.N, a.T, C, Cn, a.hist_in, a.hist_out);
    }
    return check_launch("gdn_prerule_history");
}
template <typename Tin>
gdn_status launch_history_t(const PreruleArgs &a, int64_t channels, cudaStream_t s) {
    switch (a.K) {
        case 2: return launch_history_k<Tin, 2>(a, channels, s);
        case 3: return launch_history_k<Tin, 3>(a, channels, s);
        case 4: return launch_history_k<Tin, 4>(a, channels, s);
        default: return GDN_OK;  // K = 1 keeps no history
    }
}
}  // namespace

gdn_status launch_prerule_history(const PreruleArgs &a, int64_t channels, cudaStream_t s) {
    return a.dtype == GDN_BF16 ? launch_history_t<__nv_bfloat16>(a, channels, s)
                               : launch_history_t<float>(a, channels, s);
}

}  // namespace gdn
