// Chunkwise prefill on CUDA cores in fp32 (the exact-precision path: fp32
// inputs, and any input type when no tensor-core path applies).
//
// The chunkwise form ("Hybrid attention: why new LLMs keep full attention in
// only a few layers", section "Training a recurrence in parallel"; "Hybrid
// Linear Attention Architecture Design Explained", section 4), written in the
// d_v x d_k state convention.  For a chunk of L <= 64 tokens with start state
// S0 and in-chunk cumulative log gate b_i = sum_{j<=i} g_j (a d_k vector for
// the per-channel gate; Gam_i = exp(b_i)):
//
//   A_ij = beta_i sum_c k_ic k_jc exp(b_ic - b_jc)      (j < i)
//   P_ij = sum_c q_ic k_jc exp(b_ic - b_jc)             (j <= i)
//   T    = (I + A)^-1                                   (unit lower triangular)
//   W    = T diag(beta) (K * Gam)        U = T diag(beta) V
//   U'   = U - W S0^T                                   (delta-corrected writes)
//   O    = (Q * Gam) S0^T + P U'
//   S    = S0 Diag(Gam_L) + U'^T (K * Gam_L / Gam)
//
// Every exponent above is <= 0 (the gate is a log <= 0 and j <= i), so no term
// can overflow; the pairwise decay is formed per term instead of as
// (K * Gam)(K / Gam)^T, which would overflow for strong decays.
//
// Two kernels: `gdn_prep_simt` computes the state-independent part (b, P, W,
// U) of every chunk in parallel and writes it to the workspace;
// `gdn_scan_simt` walks the chunks of each sequence in order, carrying a
// 32-row slice of the state in shared memory.
#include "chunk_common.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int kPrepThreads = 256;
constexpr int kScanThreads = 128;
constexpr int kScanRows = 32;  // rows of the state per scan block

// Exclusive prefix sum of ceil(len_n / 64) over the packed sequences.
__global__ void gdn_chunk_table(const int32_t *__restrict__ cu, int64_t N, int64_t rows, int32_t *__restrict__ off) {
    __shared__ int32_t warp_tot[32];
    __shared__ int64_t running;
    if (threadIdx.x == 0) running = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t base = 0; base < N; base += blockDim.x) {
        const int64_t i = base + threadIdx.x;
        int32_t cnt = 0;
        if (i < N) {
            int64_t s, l;
            seq_bounds(cu, i, 0, rows, s, l);
            cnt = (int32_t)((l + C - 1) / C);
        }
        int32_t x = cnt;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_tot[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int32_t before = (warp > 0 ? warp_tot[warp - 1] : 0) + x - cnt;
        if (i < N) off[i] = (int32_t)(running + before);
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) running += before + cnt;
        __syncthreads();
    }
    if (threadIdx.x == 0) off[N] = (int32_t)running;

    // The sequences by decreasing chunk count (ties by index), after the offsets: the
    // scan's blocks start longest first, so the long sequences do not end up in a
    // last wave.  Bitonic sort of (count, ~index) keys in shared memory, for up to
    // 2 x blockDim.x sequences; larger batches keep their own order.
    __shared__ uint64_t key[2048];
    int32_t *order = off + N + 1;
    const int64_t P2 = N <= 1 ? 1 : (int64_t)1 << (64 - __clzll((unsigned long long)(N - 1)));
    if (N > 2 * (int64_t)blockDim.x || P2 > 2048) {
        for (int64_t i = threadIdx.x; i < N; i += blockDim.x) order[i] = (int32_t)i;
        return;
    }
    __syncthreads();  // off[] complete
    for (int64_t i = threadIdx.x; i < P2; i += blockDim.x)
        key[i] = i < N ? ((uint64_t)(uint32_t)(off[i + 1] - off[i]) << 32) | (uint32_t)~(uint32_t)i : 0ull;
    __syncthreads();
    for (int64_t k = 2; k <= P2; k <<= 1) {
        for (int64_t j = k >> 1; j > 0; j >>= 1) {
            for (int64_t i = threadIdx.x; i < P2; i += blockDim.x) {
                const int64_t ij = i ^ j;
                if (ij > i) {
                    const uint64_t a = key[i], b = key[ij];
                    const bool down = (i & k) == 0;  // this run sorts in decreasing order
                    if (down ? a < b : a > b) {
                        key[i] = b;
                        key[ij] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int64_t i = threadIdx.x; i < N; i += blockDim.x) order[i] = (int32_t)~(uint32_t)(key[i] & 0xffffffffu);
}

template <typename Tin, int DK, int DV, bool PC>
struct PrepSmem {
    float K[C][DK + 1];
    float Q[C][DK + 1];
    float V[C][DV + 1];
    float b[C][PC ? DK + 1 : 1];
    float A[C][C + 1];
    float Tm[C][C + 1];
    float beta[C];
};

template <typename Tin, int DK, int DV, bool PC>
__global__ void __launch_bounds__(kPrepThreads)
gdn_prep_simt(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ g, const float *__restrict__ beta, const int32_t *__restrict__ cu,
              const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows, int64_t H, int64_t Hk,
              float scale, float *__restrict__ Wg, float *__restrict__ Ug, float *__restrict__ Pg,
              float *__restrict__ bg, int *err) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<PrepSmem<Tin, DK, DV, PC> *>(smem_raw);
    const int64_t chunk = blockIdx.x, h = blockIdx.y;
    ChunkLoc loc;
    if (!locate_chunk(chunk, cu, off, N, T, rows, loc)) return;
    if (!in_bounds(loc.start >= 0 && loc.start + loc.len <= rows && h < H && H % Hk == 0, err)) return;
    const int L = (int)loc.len;
    const int tid = threadIdx.x;
    const int64_t ch = chunk * H + h;  // chunk-head index into the workspace
    const int64_t hk = h / (H / Hk);   // query/key head of value head h

    // 1. inputs of the chunk (rows >= L are zero)
    for (int idx = tid; idx < C * DK; idx += kPrepThreads) {
        const int i = idx / DK, c = idx % DK;
        float kv = 0.f, qv = 0.f;
        if (i < L) {
            const int64_t e = ((loc.start + i) * Hk + hk) * DK + c;
            kv = to_f32<Tin>(k[e]);
            qv = to_f32<Tin>(q[e]) * scale;
        }
        sm.K[i][c] = kv;
        sm.Q[i][c] = qv;
        if (PC) sm.b[i][c] = i < L ? g[((loc.start + i) * H + h) * DK + c] : 0.f;
    }
    for (int idx = tid; idx < C * DV; idx += kPrepThreads) {
        const int i = idx / DV, c = idx % DV;
        sm.V[i][c] = i < L ? to_f32<Tin>(v[((loc.start + i) * H + h) * DV + c]) : 0.f;
    }
    if (tid < C) {
        sm.beta[tid] = tid < L ? beta[(loc.start + tid) * H + h] : 0.f;
        if (!PC) sm.b[tid][0] = tid < L ? g[(loc.start + tid) * H + h] : 0.f;
    }
    __syncthreads();

    // 2. in-chunk cumulative log gate
    if (PC) {
        if (tid < DK) {
            float acc = 0.f;
            for (int i = 0; i < C; ++i) { acc += sm.b[i][tid]; sm.b[i][tid] = acc; }
        }
    } else if (tid == 0) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) { acc += sm.b[i][0]; sm.b[i][0] = acc; }
    }
    __syncthreads();

    // 3. A (strictly lower) and P (lower incl. diagonal)
    for (int idx = tid; idx < C * C; idx += kPrepThreads) {
        const int i = idx / C, j = idx % C;
        float a = 0.f, p = 0.f;
        if (i < L && j <= i) {
            float kk = 0.f, qk = 0.f;
            if (PC) {
#pragma unroll 8
                for (int c = 0; c < DK; ++c) {
                    const float dcy = expf(sm.b[i][c] - sm.b[j][c]);
                    kk += sm.K[i][c] * sm.K[j][c] * dcy;
                    qk += sm.Q[i][c] * sm.K[j][c] * dcy;
                }
            } else {
#pragma unroll 8
                for (int c = 0; c < DK; ++c) {
                    kk += sm.K[i][c] * sm.K[j][c];
                    qk += sm.Q[i][c] * sm.K[j][c];
                }
                const float dcy = expf(sm.b[i][0] - sm.b[j][0]);
                kk *= dcy;
                qk *= dcy;
            }
            p = qk;
            if (j < i) a = sm.beta[i] * kk;
        }
        sm.A[i][j] = a;
        Pg[ch * C * C + idx] = p;
    }
    __syncthreads();

    // 4. T = (I + A)^-1, one column per thread by forward substitution
    if (tid < C) {
        const int col = tid;
        for (int i = 0; i < C; ++i) {
            float acc = 0.f;
            for (int j = 0; j < i; ++j) acc += sm.A[i][j] * sm.Tm[j][col];
            sm.Tm[i][col] = i < col ? 0.f : (i == col ? 1.f : -acc);
        }
    }
    __syncthreads();

    // 5. scale K and V rows: beta_j Gam_j K_j and beta_j V_j
    for (int idx = tid; idx < C * DK; idx += kPrepThreads) {
        const int j = idx / DK, c = idx % DK;
        const float gam = expf(PC ? sm.b[j][c] : sm.b[j][0]);
        sm.K[j][c] *= sm.beta[j] * gam;
    }
    for (int idx = tid; idx < C * DV; idx += kPrepThreads) {
        const int j = idx / DV, c = idx % DV;
        sm.V[j][c] *= sm.beta[j];
    }
    __syncthreads();

    // 6. W = T (beta Gam K), U = T (beta V); b to the workspace
    for (int idx = tid; idx < C * DK; idx += kPrepThreads) {
        const int i = idx / DK, c = idx % DK;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc += sm.Tm[i][j] * sm.K[j][c];
        Wg[ch * C * DK + idx] = acc;
    }
    for (int idx = tid; idx < C * DV; idx += kPrepThreads) {
        const int i = idx / DV, c = idx % DV;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc += sm.Tm[i][j] * sm.V[j][c];
        Ug[ch * C * DV + idx] = acc;
    }
    if (PC) {
        for (int idx = tid; idx < C * DK; idx += kPrepThreads) bg[ch * C * DK + idx] = sm.b[idx / DK][idx % DK];
    } else if (tid < C) {
        bg[ch * C + tid] = sm.b[tid][0];
    }
}

template <int DK, bool PC>
struct ScanSmem {
    float S[kScanRows][DK + 1];
    float W[C][DK + 1];
    float Qg[C][DK + 1];
    float Kg[C][DK + 1];
    float Up[C][kScanRows + 1];
    float P[C][C + 1];
    float gl[DK];  // Gam at the chunk's last token
};

template <typename Tin, int DK, int DV, bool PC>
__global__ void __launch_bounds__(kScanThreads)
gdn_scan_simt(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ h0,
              const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int64_t N, int64_t T,
              int64_t rows, int64_t H, int64_t Hk, int64_t max_chunks, float scale, int64_t snap_stride,
              int64_t n_snap,
              const float *__restrict__ Wg, const float *__restrict__ Ug, const float *__restrict__ Pg,
              const float *__restrict__ bg, Tin *__restrict__ out, float *final_state, float *__restrict__ snaps,
              int *err) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto &sm = *reinterpret_cast<ScanSmem<DK, PC> *>(smem_raw);
    // packed batches: blocks in launch order take the sequences longest first (the
    // order the chunk table wrote after the chunk offsets)
    int64_t n = blockIdx.x, h = blockIdx.y, zb = blockIdx.z;
    if (cu) {
        const int64_t per = (int64_t)gridDim.y * gridDim.z;
        const int64_t id = blockIdx.x + (int64_t)gridDim.x * (blockIdx.y + (int64_t)gridDim.y * blockIdx.z);
        n = off[N + 1 + id / per];
        h = (id % per) % gridDim.y;
        zb = (id % per) / gridDim.y;
    }
    const int r0 = (int)zb * kScanRows;
    const int tid = threadIdx.x;
    if (!in_bounds(n >= 0 && n < N && h >= 0 && h < H && r0 + kScanRows <= DV, err)) return;
    const int64_t state_off = ((n * H + h) * DV + r0) * (int64_t)DK;

    for (int idx = tid; idx < kScanRows * DK; idx += kScanThreads)
        sm.S[idx / DK][idx % DK] = h0 ? h0[state_off + idx] : 0.f;

    int64_t start, len;
    seq_bounds(cu, n, T, rows, start, len);
    if (!in_bounds(start >= 0 && start + len <= rows, err)) return;
    const int64_t nchunks = (len + C - 1) / C;
    const int64_t chunk0 = cu ? (int64_t)off[n] : n * ((T + C - 1) / C);

    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t chunk = chunk0 + c;
        if (chunk >= max_chunks) break;  // inconsistent offsets: stay inside the workspace
        const int L = (int)(len - c * C < C ? len - c * C : C);
        const int64_t tok0 = start + c * C;
        const int64_t ch = chunk * H + h;
        const float *bch = bg + ch * C * (PC ? DK : 1);
        __syncthreads();  // previous chunk done with the buffers

        // gated operands of this chunk
        for (int idx = tid; idx < C * DK; idx += kScanThreads) {
            const int i = idx / DK, cc = idx % DK;
            float wq = 0.f, kq = 0.f, kg = 0.f;
            if (i < L) {
                const int64_t e = ((tok0 + i) * Hk + h / (H / Hk)) * DK + cc;
                const float bi = PC ? bch[i * DK + cc] : bch[i];
                const float bl = PC ? bch[(L - 1) * DK + cc] : bch[L - 1];
                wq = Wg[ch * C * DK + idx];
                kq = to_f32<Tin>(q[e]) * scale * expf(bi);
                kg = to_f32<Tin>(k[e]) * expf(bl - bi);
            }
            sm.W[i][cc] = wq;
            sm.Qg[i][cc] = kq;
            sm.Kg[i][cc] = kg;
        }
        for (int idx = tid; idx < C * kScanRows; idx += kScanThreads) {
            const int i = idx / kScanRows, r = idx % kScanRows;
            sm.Up[i][r] = i < L ? Ug[ch * C * DV + i * DV + r0 + r] : 0.f;
        }
        for (int idx = tid; idx < C * C; idx += kScanThreads) sm.P[idx / C][idx % C] = Pg[ch * C * C + idx];
        for (int cc = tid; cc < DK; cc += kScanThreads) sm.gl[cc] = expf(PC ? bch[(L - 1) * DK + cc] : bch[L - 1]);
        __syncthreads();

        // U' = U - W S0^T
        for (int idx = tid; idx < C * kScanRows; idx += kScanThreads) {
            const int i = idx / kScanRows, r = idx % kScanRows;
            float acc = 0.f;
#pragma unroll 8
            for (int cc = 0; cc < DK; ++cc) acc += sm.W[i][cc] * sm.S[r][cc];
            sm.Up[i][r] -= acc;
        }
        __syncthreads();

        // O = (Q Gam) S0^T + P U'
        for (int idx = tid; idx < C * kScanRows; idx += kScanThreads) {
            const int i = idx / kScanRows, r = idx % kScanRows;
            if (i >= L) continue;
            float acc = 0.f;
#pragma unroll 8
            for (int cc = 0; cc < DK; ++cc) acc += sm.Qg[i][cc] * sm.S[r][cc];
            for (int j = 0; j <= i; ++j) acc += sm.P[i][j] * sm.Up[j][r];
            out[((tok0 + i) * H + h) * DV + r0 + r] = from_f32<Tin>(acc);
        }
        __syncthreads();

        // S = S0 Diag(Gam_L) + U'^T (K Gam_L / Gam)
        for (int idx = tid; idx < kScanRows * DK; idx += kScanThreads) {
            const int r = idx / DK, cc = idx % DK;
            float acc = sm.S[r][cc] * sm.gl[cc];
            for (int j = 0; j < L; ++j) acc += sm.Up[j][r] * sm.Kg[j][cc];
            sm.S[r][cc] = acc;
        }

        // snapshot after n*stride tokens of the sequence
        if (snaps && snap_stride > 0 && ((c + 1) * C) % snap_stride == 0 && (c + 1) * C <= len) {
            const int64_t s = (c + 1) * C / snap_stride - 1;
            if (s < n_snap) {
                __syncthreads();
                float *dst = snaps + (((n * n_snap + s) * H + h) * DV + r0) * (int64_t)DK;
                for (int idx = tid; idx < kScanRows * DK; idx += kScanThreads) dst[idx] = sm.S[idx / DK][idx % DK];
            }
        }
    }
    __syncthreads();
    if (final_state)
        for (int idx = tid; idx < kScanRows * DK; idx += kScanThreads)
            final_state[state_off + idx] = sm.S[idx / DK][idx % DK];
}

template <typename Tin, int DK, int DV, bool PC>
gdn_status launch_typed(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s) {
    const int32_t *off = a.cu_seqlens ? reinterpret_cast<const int32_t *>(a.ws + p.off_chunk_offsets) : nullptr;
    float *W = reinterpret_cast<float *>(a.ws + p.off_W);
    float *U = reinterpret_cast<float *>(a.ws + p.off_U);
    float *P = reinterpret_cast<float *>(a.ws + p.off_P);
    float *b = reinterpret_cast<float *>(a.ws + p.off_b);
    gdn_status st = launch_chunk_table(p, a, s);
    if (st != GDN_OK) return st;
    if (p.max_chunks > 0 && p.rows > 0) {
        const size_t smem = sizeof(PrepSmem<Tin, DK, DV, PC>);
        auto kern = gdn_prep_simt<Tin, DK, DV, PC>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return check_launch("gdn_prep_simt attributes");
        if (p.max_chunks > 0x7fffffffLL || p.H > 65535) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
        log_launch("gdn_prep_simt", dim3((unsigned)p.max_chunks, (unsigned)p.H), dim3(kPrepThreads), smem);
        LaunchScope ls("gdn_prep_simt", s);
        kern<<<dim3((unsigned)p.max_chunks, (unsigned)p.H), kPrepThreads, smem, s>>>(
            (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v, a.g, a.beta, a.cu_seqlens, off, a.N, a.T, p.rows,
            p.H, a.Hk, a.scale, W, U, P, b, a.status);
    }
    st = check_launch("gdn_prep_simt");
    if (st != GDN_OK) return st;
    {
        const size_t smem = sizeof(ScanSmem<DK, PC>);
        auto kern = gdn_scan_simt<Tin, DK, DV, PC>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return check_launch("gdn_scan_simt attributes");
        if (a.N > 0x7fffffffLL || p.H > 65535) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
        log_launch("gdn_scan_simt", dim3((unsigned)a.N, (unsigned)p.H, DV / kScanRows), dim3(kScanThreads), smem);
        LaunchScope ls("gdn_scan_simt", s);
        kern<<<dim3((unsigned)a.N, (unsigned)p.H, DV / kScanRows), kScanThreads, smem, s>>>(
            (const Tin *)a.q, (const Tin *)a.k, a.h0, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, a.Hk, p.max_chunks,
            a.scale, a.snapshot_stride, a.n_snap, W, U, P, b, (Tin *)a.out, a.final_state, a.snapshots, a.status);
    }
    return check_launch("gdn_scan_simt");
}

template <typename Tin>
gdn_status launch_dtype(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s) {
    const bool pc = p.per_channel;
#define GDN_CASE(DK_, DV_)                                                                  \
    if (p.dk == DK_ && p.dv == DV_)                                                         \
        return pc ? launch_typed<Tin, DK_, DV_, true>(p, a, s) : launch_typed<Tin, DK_, DV_, false>(p, a, s);
    GDN_CASE(128, 128)
    GDN_CASE(64, 64)
    GDN_CASE(128, 64)
    GDN_CASE(64, 128)
#undef GDN_CASE
    return fail(GDN_ERR_UNSUPPORTED, "head sizes");
}

}  // namespace

gdn_status launch_chunk_table(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s) {
    if (!a.cu_seqlens) return GDN_OK;
    {
        LaunchScope ls("gdn_chunk_table", s);
        gdn_chunk_table<<<1, 1024, 0, s>>>(a.cu_seqlens, a.N, p.rows,
                                           reinterpret_cast<int32_t *>(a.ws + p.off_chunk_offsets));
    }
    return check_launch("gdn_chunk_table");
}

gdn_status launch_chunk_simt(const ChunkPlan &p, const ChunkArgs &a, int dtype, cudaStream_t s) {
    return dtype == GDN_BF16 ? launch_dtype<__nv_bfloat16>(p, a, s) : launch_dtype<float>(p, a, s);
}

}  // namespace gdn
