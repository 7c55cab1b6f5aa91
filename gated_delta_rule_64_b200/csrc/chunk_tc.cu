// Chunkwise prefill on the 5th-generation tensor cores (tcgen05, TMEM, TMA):
// bf16 q/k/v, one gate per head, d_k = d_v = 128, fp32 state.
//
// The algebra is the chunkwise form of the gated delta rule ("Hybrid attention:
// why new LLMs keep full attention in only a few layers", section "Training a
// recurrence in parallel"; "Hybrid Linear Attention Architecture Design
// Explained", section 4), in the d_v x d_k state convention.  For a chunk of
// L <= 64 tokens, start state S0, b_i = sum_{j<=i} g_j and gam_i = exp(b_i):
//
//   A  = strictly-lower( diag(beta) (K K^T) * exp(b_i - b_j) )
//   P  = lower-incl( scale (Q K^T) * exp(b_i - b_j) )
//   T  = (I + A)^-1
//   W  = T diag(beta gam) K,   U = T diag(beta) V                (chunk-local)
//   U' = U - W S0^T                                               (per chunk, in order)
//   O  = scale gam_i (S0 q_i) + P U'
//   S  = gam_L S0 + U'^T (K * exp(b_L - b_j))
//
// Every exponent is <= 0 (gates are logs <= 0 and j <= i), so nothing
// overflows.
//
// Two kernels:
//   gdn_prep_tc  one CTA per (chunk, head), all chunks in parallel.  TMA loads
//                K and Q; one M = 128 MMA gives [K;Q] K^T (the K rows give the
//                Gram matrix, the Q rows Q K^T); the unit-lower-triangular
//                system is solved blockwise (16 x 16 diagonal blocks by forward
//                substitution in fp32, off-diagonal blocks by tf32 warp MMAs);
//                one MMA gives W^T.  W^T, P, -T'' = -T diag(beta) and the gate
//                factors are written as ready-made operand images (16-byte
//                stores of 128-byte swizzled rows) into one contiguous block per
//                chunk-head; U itself is never formed.
//   gdn_scan_tc  one CTA per (sequence, head).  The fp32 state lives in
//                registers (two threads per state row, 64 columns each); per
//                chunk it is rounded to a bf16 A operand in TMEM and two MMA
//                groups with fp32 accumulators in TMEM produce
//                [S0 W^T + V^T (-T'')^T | S0 Q^T] (the first part is -U'^T:
//                U' = U - W S0^T with U = T diag(beta) V) and then
//                [(diag(w) U')^T K | U'^T P^T] with w_j = exp(b_L - b_j) (the
//                state increment and the intra-chunk output).  The next chunk's
//                block is prefetched (bulk copies; Q, K and V tiles by TMA) into
//                the second of two stages, and the previous chunk's output is
//                stored while the MMA groups run.
//
// All tcgen05 MMAs are M = 128 (the 128 rows of the state, or the 64 K rows
// stacked on the 64 Q rows), so accumulator rows map 1:1 onto TMEM lanes and
// every thread reads its own row.
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>

#include "tc_common.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace tc;

// ===========================================================================
// Prep
// ===========================================================================
// Shared memory (1024-aligned):
//   [0, 32K)    K and Q tiles stacked as the M = 128 operand of the first MMA:
//               [c-block 0: K rows | Q rows][c-block 1: K rows | Q rows].
//               After that MMA the Q rows hold A (fp32; rows 0-31 | 32-63),
//               then T diag(beta gam) at [8K,16K) (the bf16 operand image of W)
//   [32K, 48K)  T (fp32)
//   [48K, 52K)  per-warp 16 x 16 scratch of the blocked solve
// The results (W^T rows, P rows, -T'' rows, gate factors) are written straight to
// the workspace block of the chunk-head; U = T'' V is not formed here (the scan
// accumulates V^T (-T'')^T onto S0 W^T).  About 54 KB of shared memory and 64
// registers a thread let four blocks share an SM.
constexpr uint32_t kPrepTf = 32768, kPrepY = 49152;
constexpr uint32_t kPrepSmem = kPrepY + 4096 + 1024;

__device__ __forceinline__ uint32_t a_offset(int i, int j) {
    // A (fp32) in the Q rows of the first operand: rows 0..31 at 8K, 32..63 at 24K
    return (i < 32 ? 8192u : 24576u) + f32_offset(i & 31, j);
}

__global__ void __launch_bounds__(kThreads, 4)
gdn_prep_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
            const float *__restrict__ g, const float *__restrict__ beta,
            const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows,
            int64_t H, int64_t Hk, float scale, uint8_t *__restrict__ blocks, int want_bound, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    // (one barrier per commit: a waiter two phases behind could not tell them apart)
    __shared__ uint64_t bar_ld, bar_mma, bar_w, bar_drain;
    __shared__ uint32_t tmem_base;
    __shared__ float s_b[C], s_sg[C];
    __shared__ __align__(16) float s_beta[C], s_bg[C];
    __shared__ __align__(16) float s_b2[C];  // b in log2 units
    __shared__ __align__(16) float s_f[C];   // 2^(m - b2_j), m = b2 at row 31 (the factored decay)

    const int64_t chunk = blockIdx.x, h = blockIdx.y;
    ChunkLoc loc;
    if (!locate_chunk(chunk, cu, off, N, T, rows, loc)) return;
    if (!in_bounds(loc.start >= 0 && loc.start + loc.len <= rows && h < H && H % Hk == 0, err)) return;
    const int L = (int)loc.len;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;
    const int64_t ch = chunk * H + h;
    const int32_t tok0 = (int32_t)loc.start;
    uint8_t *blk = blocks + (size_t)ch * kTcBlock;
    uint8_t *rest = blk + kBlkRest;

    // gate loads first: their latency overlaps the set-up and the TMA loads
    float g_in = 0.f, beta_in = 0.f;
    if (tid < L) {
        g_in = g[(int64_t)(tok0 + tid) * H + h];
        beta_in = beta[(int64_t)(tok0 + tid) * H + h];
    }
    if (tid == 0) {  // the tile loads first: their latency overlaps the rest of the set-up
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_w, 1);
        mbar_init(&bar_drain, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar_ld, 4 * 8192);
        const int32_t hq = (int32_t)(h / (H / Hk));  // query/key head of value head h
        tma_load_3d(sm + 0, &mk, 0, hq, tok0, &bar_ld);
        tma_load_3d(sm + 16384, &mk, 64, hq, tok0, &bar_ld);
        tma_load_3d(sm + 8192, &mq, 0, hq, tok0, &bar_ld);
        tma_load_3d(sm + 24576, &mq, 64, hq, tok0, &bar_ld);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    // Gates (rows >= L: beta = 0, g = 0): in-chunk inclusive cumsum of the log gate.
    if (tid < C) {
        s_beta[tid] = beta_in;
        float x = g_in;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        s_b[tid] = x;
    }
    __syncthreads();
    if (tid >= 32 && tid < C) s_b[tid] += s_b[31];
    // (a gate above 0, outside the documented range, makes b non-monotone)
    const bool monotone = !__syncthreads_or(tid < L && !(g_in <= 0.f));
    if (tid < C) {
        const bool in = tid < L;
        const float bl = s_b[L - 1], bi = s_b[tid];
        s_b2[tid] = bi * 1.4426950408889634f;
        s_f[tid] = ex2((s_b[31] - bi) * 1.4426950408889634f);
        s_bg[tid] = s_beta[tid] * __expf(bi);
        s_sg[tid] = in ? scale * __expf(bi) : 0.f;
        float *fac = reinterpret_cast<float *>(rest + kRestFac);
        fac[kFacQs + tid] = s_sg[tid];  // the scan scales its output by these (it reads Q itself)
        fac[kFacW + tid] = in ? __expf(bl - bi) : 0.f;  // and its U' rows by these (it reads K itself)
        if (tid == 0) fac[kFacGL] = __expf(bl);
    }
    __syncthreads();

    bool ok = mbar_wait(&bar_ld, 0);
    if (warp == 0 && __all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const uint64_t dkq = sdesc_sw128(smem_u32(sm), 16, 1024);
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t o = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_bf16_ss(tm, dkq + o, dkq + o, id, kk > 0);
        }
        mma_commit_warp(&bar_mma);
    }
    ok = ok && mbar_wait(&bar_mma, 0);
    tc_fence_after();

    // Epilogue 1: accumulator row r = qd*32 + lane, columns [32 hf, 32 hf + 32).
    // Rows 0..63 (K K^T) -> A in fp32; rows 64..127 (Q K^T) -> P rows (bf16).  A's
    // diagonal, which the solve never reads, holds beta_i |k_i|^2 for the decay bound.
    if (ok) {
        const int r = qd * 32 + lane;
        const uint32_t taddr = tm + ((uint32_t)(qd * 32) << 16) + 32 * hf;
        const bool is_a = r < C;
        const int i = is_a ? r : r - C;
        const float pre = is_a ? s_beta[i] : scale;
        float v0[16], v1[16];
        tmem_ld16(taddr, v0);
        tmem_ld16(taddr + 16, v1);
        tmem_wait_ld();
        // in-chunk decay exp(b_i - b_j) = 2^(b2_i - b2_j) (used only for j <= i, where it is <= 1).
        // When the chunk's whole decay is at most 120 log2 units it is the product
        // 2^(b2_i - m) 2^(m - b2_j) around m = b2 at row 31, both factors inside the fp32
        // range (one exponential per row instead of one per entry); else entry by entry.
        const float bi2 = s_b2[i];
        const bool fact = monotone && s_b2[0] - s_b2[C - 1] <= 120.f;  // uniform over the block
        const float ei = fact ? ex2(bi2 - s_b2[31]) : 0.f;
        // (in pairs: fp32 x2 multiplies)
        const float2 pe = make_float2(pre * ei, pre * ei);
        float rr[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float2 d01, d23;  // pre exp(b_i - b_j) for the 4 columns j
            if (fact) {
                const float4 f4 = *reinterpret_cast<const float4 *>(s_f + 32 * hf + 4 * q);
                d01 = __fmul2_rn(pe, make_float2(f4.x, f4.y));
                d23 = __fmul2_rn(pe, make_float2(f4.z, f4.w));
            } else {
                const float4 b4 = *reinterpret_cast<const float4 *>(s_b2 + 32 * hf + 4 * q);
                d01 = make_float2(pre * ex2(bi2 - b4.x), pre * ex2(bi2 - b4.y));
                d23 = make_float2(pre * ex2(bi2 - b4.z), pre * ex2(bi2 - b4.w));
            }
            const float *vv = q < 4 ? &v0[4 * q] : &v1[4 * (q - 4)];
            const float2 r01 = __fmul2_rn(d01, make_float2(vv[0], vv[1])), r23 = __fmul2_rn(d23, make_float2(vv[2], vv[3]));
            const float r4[4] = {r01.x, r01.y, r23.x, r23.y};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = 4 * q + e, j = 32 * hf + t;
                rr[t] = i < L && j <= i ? r4[e] : 0.f;
            }
        }
        if (is_a) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(sm + a_offset(i, 32 * hf + 4 * q)) =
                    make_float4(rr[4 * q], rr[4 * q + 1], rr[4 * q + 2], rr[4 * q + 3]);
        } else {
            // P row i (key tokens j = 32 hf ..) straight to the block: four 16-byte chunks
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4 *>(rest + kRestP + sw128_offset(i, 4 * hf + q)) =
                    make_uint4(pack_bf16(rr[8 * q], rr[8 * q + 1]), pack_bf16(rr[8 * q + 2], rr[8 * q + 3]),
                               pack_bf16(rr[8 * q + 4], rr[8 * q + 5]), pack_bf16(rr[8 * q + 6], rr[8 * q + 7]));
        }
    }
    tc_fence_before();
    __syncthreads();
    // a token outside the decay bound's range: beta_i < 0 or beta_i |k_i|^2 > kBetaK2Max
    bool bad = false;
    if (want_bound && ok && (tid & 3) == 0) {
        const int i = tid >> 2;
        bad = i < L && !(s_beta[i] >= 0.f && *reinterpret_cast<const float *>(sm + a_offset(i, i)) <= kBetaK2Max);
    }

    // Blocked solve of T = (I + A)^-1 with 16 x 16 blocks.
    uint8_t *Tf = sm + kPrepTf;
    blocked_solve<kPrepTf, kPrepY>(sm, [](int i, int j) { return a_offset(i, j); },
                                   [](int i) { return (i < 32 ? 8192u : 24576u) + (uint32_t)(i & 31) * 256u; }, ok);

    // T' = T diag(beta gam) as the bf16 operand image of W (K-major rows i, shared
    // memory) and -T'' = -T diag(beta) as rows of the block (the scan's operand); the
    // blocks of T above its block diagonal are zero (the solve leaves them unwritten).
    if (ok) {
        const int i = tid >> 2, j0 = (tid & 3) * 16;
        const bool upper = (tid & 3) > (i >> 4);
        float tv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!upper) f = *reinterpret_cast<const float4 *>(Tf + f32_offset(i, j0 + 4 * q));
            tv[4 * q] = f.x; tv[4 * q + 1] = f.y; tv[4 * q + 2] = f.z; tv[4 * q + 3] = f.w;
        }
        const uint32_t tp = smem_u32(sm + 8192);
        const float4 *bg4 = reinterpret_cast<const float4 *>(s_bg + j0), *be4 = reinterpret_cast<const float4 *>(s_beta + j0);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            uint32_t a[4], b[4];  // packed bf16 pairs (fp32 x2 multiplies)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const float4 g4 = bg4[2 * q + h2], e4 = be4[2 * q + h2];
                const float *t4 = &tv[8 * q + 4 * h2];
                const float2 a01 = __fmul2_rn(make_float2(t4[0], t4[1]), make_float2(g4.x, g4.y));
                const float2 a23 = __fmul2_rn(make_float2(t4[2], t4[3]), make_float2(g4.z, g4.w));
                const float2 b01 = __fmul2_rn(make_float2(t4[0], t4[1]), make_float2(-e4.x, -e4.y));
                const float2 b23 = __fmul2_rn(make_float2(t4[2], t4[3]), make_float2(-e4.z, -e4.w));
                a[2 * h2] = pack_bf16(a01.x, a01.y); a[2 * h2 + 1] = pack_bf16(a23.x, a23.y);
                b[2 * h2] = pack_bf16(b01.x, b01.y); b[2 * h2 + 1] = pack_bf16(b23.x, b23.y);
            }
            const uint32_t o = sw128_offset(i, (j0 >> 3) + q);
            st_shared_v4(tp + o, a[0], a[1], a[2], a[3]);
            *reinterpret_cast<uint4 *>(rest + kRestTn + o) = make_uint4(b[0], b[1], b[2], b[3]);
        }
    }
    fence_async_smem();  // (T' is read by the tensor core)
    tc_fence_before();
    const bool any_bad = __syncthreads_or(bad);
    tc_fence_after();
    // (a gate above 0, outside the documented range, also leaves the chunk without a bound)
    if (tid == 0)
        reinterpret_cast<float *>(rest + kRestFac)[kFacLam] = (!want_bound || !monotone || any_bad) ? kLamNone : s_b2[L - 1];

    // W^T = K^T T'^T (M = d_k, K = 64 tokens)
    if (warp == 0 && __all_sync(0xffffffffu, ok)) {
        const uint32_t id_w = idesc_bf16(128, 64, 1, 0);
        const uint64_t dk = sdesc_sw128(smem_u32(sm), 16384, 1024), dtp = sdesc_sw128(smem_u32(sm + 8192), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tm, dk + ((kk * 2048) >> 4), dtp + ((kk * 32) >> 4), id_w, kk > 0);
        mma_commit_warp(&bar_w);
    }

    // Epilogue 2: thread row r is channel r of W^T, tokens [32 hf, 32 hf + 32), out as
    // 128-byte swizzled rows (row = channel).
    ok = ok && mbar_wait(&bar_w, 0);
    tc_fence_after();
    if (ok) store_w(tm, blk, qd, hf, lane);
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
        // A wait gave up: record it, then wait (bounded) for the tile copies and for
        // every MMA issued before the TMEM columns are freed.
        if (tid == 0) {
            flag_error(err, GDN_DEV_TIMEOUT_PREP);
            mbar_wait(&bar_ld, 0);
        }
        if (warp == 0) {
            mma_commit_warp(&bar_drain);
            mbar_wait(&bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == 0) tmem_dealloc(tm, 64);
}

// ===========================================================================
// Scan
// ===========================================================================
// Shared memory (1024-aligned), two stages of per-chunk operands, each the
// chunk-head's workspace block as it is (bulk copies; with one gate per head the Q
// and K tiles come from q and k themselves, by TMA, where the block holds Qs and K~)
// followed by the V tile (TMA):
//   [0, 16K)      W^T rows: the MN-major B operand of S0 W^T (N = 64)
//   [16K, 32K)    Q or Qs, two 64-channel halves: the K-major B operand of S0 Q^T
//   [32K, 48K)    K (one gate per head) or K~: the MN-major B operand of the state
//                 increment (N = 128)
//   [48K, 56K)    P rows: the K-major B operand of U'^T P^T (N = 64)
//   [56K, 64K)    -T'' rows: the K-major B operand of V^T (-T'')^T
//   [64K, 65K)    gate factors
//   [65K, 81K)    the V tile: the MN-major A operand of V^T (-T'')^T
// The operands the threads produce (S0 and U' in bf16) are written to TMEM and
// used as A operands straight from there.
// TMEM columns: [0,128) D1 = [S0 W^T - U^T | S0 Q^T], [128,320) D2 = [increment |
// U'^T P^T], [320,384) S0, [384,416) U', [416,448) diag(w) U' (one gate per head).
// A tcgen05.ld waits for the MMAs in flight, so every accumulator is read once
// the chunk's MMAs are done (the output with the state increment), and the
// output leaves from registers while the next chunk's first MMA group runs.
constexpr uint32_t kStW = kBlkW, kStQ = kBlkQs, kStRest = kBlkRest, kStV = (uint32_t)kTcBlock;
constexpr uint32_t kStage = kStV + 16384;
static_assert(kStV % 1024 == 0 && kStage % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled operands");
constexpr int kStages = 2;
constexpr uint32_t kScanSmem = kStages * kStage + 1024;
constexpr uint32_t kTmD1 = 0, kTmD2 = 128, kTmAS = 320, kTmAU = 384, kTmAUw = 416;

struct ScanBars {
    uint64_t full[kStages];
    uint64_t mma[3];  // per chunk: -U'^T done; the increment done; every product of the chunk done
    uint64_t drain;   // after a failed wait: every MMA issued has completed
};

// KDA: per-channel gate (the carried state is then scaled per key channel by
// exp(b_L) instead of one factor).
// Sequence split of long fixed-length sequences (G >= 2 segments of `seg` chunks).
// A segment's end state is an affine function of its start state,
// S_end = S_start M_g + B_g, and the weight of S_start in whatever the segment
// computes after its first m chunks is at most 2^(lam_0 + .. + lam_{m-1}) times
// |S_start| (the chunks' decay bounds, kFacLam).  Pass 1 runs all segments at
// once: segment 0 from the true initial state, every other one from a zero
// start.  A zero-start segment writes the outputs and snapshots of the chunks
// where that sum is below kLamDrop (there they equal the true ones to fp32
// precision), its end state B_g, and m_g: the chunks before that point, or all
// of them when the sum never gets there.  Only in that last case does the start
// state reach the segment's end, and only then is the transition M_g formed,
// from the identity with the writes dropped (the state then has d_k rows, which
// needs d_v = d_k); those blocks come after all others in the grid and leave at
// once when M_g is not needed.  gdn_seg_combine chains the start states,
// S_{g+1} = S_g M_g + B_g (B_g where M_g was not needed), and pass 2 reruns the
// first m_g chunks of every segment g >= 1 from its true start state.  With gates
// that forget within a few chunks (every workload here) pass 2 is a few chunks
// long; with gates that keep the state alive it reruns whole segments.
struct ScanSplit {
    int32_t G;       // segments per sequence; 1: no split
    int32_t seg;     // chunks per segment
    int32_t pass;    // 1 or 2 (with G >= 2)
    float *states;   // [N][G][3][H][D][D] fp32: B_g, M_g and the true start state S_g of segment g
    int32_t *rec;    // [2][N][G][H] int32: m_g, and 1 where M_g was formed
};
__device__ __forceinline__ float *split_state(const ScanSplit &sp, int64_t n, int64_t g, int slot, int64_t H,
                                              int64_t h) {
    return sp.states + ((((n * sp.G + g) * 3 + slot) * H + h) * (int64_t)D) * D;
}
__device__ __forceinline__ int32_t *split_rec(const ScanSplit &sp, int which, int64_t N, int64_t n, int64_t g,
                                              int64_t H, int64_t h) {
    return sp.rec + ((which * N + n) * sp.G + g) * H + h;
}

// SPLIT: launched as a pass of the split scan (1-D grid; the block's work comes from `sp`).
// Eight warps hold the state (two threads per row, 64 columns each); warp 0 also
// issues the MMAs and warp 4 the copies.
#define GDN_SCAN_PARAMS                                                                                              \
    const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,                                  \
        const __grid_constant__ CUtensorMap mv, const float *h0,                                                     \
        const int32_t *__restrict__ cu,                                                                              \
        const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows, int64_t H, int64_t Hk,                  \
        int64_t max_chunks, int64_t snap_stride, int64_t n_snap, const uint8_t *__restrict__ blocks,                  \
        __nv_bfloat16 *__restrict__ out, float *final_state, float *__restrict__ snaps, const ScanSplit sp, int *err
#define GDN_SCAN_ARGS \
    mq, mk, mv, h0, cu, off, N, T, rows, H, Hk, max_chunks, snap_stride, n_snap, blocks, out, final_state, snaps, sp, err

template <bool KDA, bool SPLIT>
__device__ __forceinline__ void scan_body(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                          const float *h0,
                                          const int32_t *__restrict__ cu,
                                          const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows,
                                          int64_t H, int64_t Hk, int64_t max_chunks, int64_t snap_stride,
                                          int64_t n_snap, const uint8_t *__restrict__ blocks,
                                          __nv_bfloat16 *__restrict__ out, float *final_state,
                                          float *__restrict__ snaps, const ScanSplit sp, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    __shared__ ScanBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ float s_red[kThreads / 32];
    // Packed batches: blocks in launch order take the sequences longest first (the
    // order the chunk table wrote after the chunk offsets), all heads of one
    // sequence after another, so the long sequences start in the first wave.
    int64_t n = blockIdx.x;
    int h = (int)blockIdx.y;
    if (!SPLIT && cu) {
        const int id = (int)(blockIdx.y * gridDim.x + blockIdx.x);  // < N H, checked at launch
        n = off[N + 1 + id / (int)H];
        h = id % (int)H;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;
    const int v = qd * 32 + lane;  // state row; this thread holds columns [64 hf, 64 hf + 64)
    constexpr int kIssuer = 0, kLoader = 128;  // warp 0 issues the MMAs, warp 4 lane 0 the copies

    // This block's work: sequence n, chunks [cb, cb + nchunks) of it (a segment of the
    // split scan), its start state and where its end state goes.
    enum { kStartGiven, kStartZero, kStartIdentity };
    int64_t g = 0;
    int start_kind = kStartGiven;
    bool spec = false;      // zero start: outputs only where the start state no longer matters
    bool emit_any = true;   // false: a transition map (no outputs)
    if (SPLIT) {
        const int64_t id = blockIdx.x, nh_all = N * H;
        int64_t nh;
        if (sp.pass == 1) {
            if (id < nh_all * sp.G) {
                nh = id / sp.G;
                g = id % sp.G;
                if (g > 0) {
                    start_kind = kStartZero;
                    spec = true;
                }
            } else {
                const int64_t j = id - nh_all * sp.G;
                nh = j / (sp.G - 2);
                g = 1 + j % (sp.G - 2);
                start_kind = kStartIdentity;
                emit_any = false;
            }
        } else {
            nh = id / (sp.G - 1);
            g = 1 + id % (sp.G - 1);
        }
        n = nh / H;
        h = (int)(nh % H);
    }
    const int64_t sh = (n * H + h) * (int64_t)D * D;  // this (sequence, head)'s state in h0 / final_state
    const float *s_init = h0 ? h0 + sh : nullptr;     // kStartGiven: this state (nullptr: zero)
    float *s_end = final_state ? final_state + sh : nullptr;
    if (SPLIT) {
        if (sp.pass == 1)
            s_end = g == 0 ? split_state(sp, n, 1, 2, H, h) : split_state(sp, n, g, spec ? 0 : 1, H, h);
        else  // S_g, or B_{g-1} itself where M_{g-1} was not formed (gdn_seg_combine wrote nothing)
            s_init = (g >= 2 && *split_rec(sp, 1, N, n, g - 1, H, h) == 0) ? split_state(sp, n, g - 1, 0, H, h)
                                                                           : split_state(sp, n, g, 2, H, h);
    }

    int64_t start, len;
    seq_bounds(cu, n, T, rows, start, len);
    int64_t ntot = (len + C - 1) / C;
    const int64_t chunk0 = cu ? (int64_t)off[n] : n * ((T + C - 1) / C);
    if (!in_bounds(n >= 0 && n < N && h >= 0 && h < H && start >= 0 && start + len <= rows && chunk0 >= 0 &&
                       (!SPLIT || (g >= 0 && g < sp.G)),
                   err))
        return;
    if (chunk0 + ntot > max_chunks) ntot = max_chunks > chunk0 ? max_chunks - chunk0 : 0;
    const int64_t cb = SPLIT ? g * sp.seg : 0;
    const int64_t ce = SPLIT && g < sp.G - 1 ? (cb + sp.seg < ntot ? cb + sp.seg : ntot) : ntot;
    const int64_t nchunks = ce > cb ? ce - cb : 0;  // chunks of the segment; chunk i is cb + i of the sequence
    int64_t nrun = nchunks;                         // chunks this block runs
    const bool ident = SPLIT && start_kind == kStartIdentity;
    const auto block_of = [&](int64_t c) { return blocks + (size_t)((chunk0 + cb + c) * H + h) * kTcBlock; };

    if (ident) {
        // The transition of the segment is needed only where the decay bound of the
        // whole segment does not reach kLamDrop (a margin of 1 covers the order of
        // the sum, which the zero-start block forms chunk by chunk).
        float part = 0.f;
        for (int64_t c = tid; c < nchunks; c += blockDim.x)
            part += reinterpret_cast<const float *>(block_of(c) + kBlkRest + kRestFac)[kFacLam];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) s_red[warp] = part;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < (int)(blockDim.x / 32); ++w) tot += s_red[w];
        const bool need = !(tot < kLamDrop - 1.f);  // (NaN: needed)
        if (tid == 0) *split_rec(sp, 1, N, n, g, H, h) = need ? 1 : 0;
        if (!need) return;
    }
    if (SPLIT && sp.pass == 2) {
        const int32_t m = *split_rec(sp, 0, N, n, g, H, h);
        nrun = m < 0 ? 0 : (m < nchunks ? m : nchunks);
        // the final state comes from here only when the whole last segment is rerun
        s_end = (g == sp.G - 1 && nrun == nchunks && final_state) ? final_state + sh : nullptr;
    }

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&bars.full[i], 1);
        for (int i = 0; i < 3; ++i) mbar_init(&bars.mma[i], 1);
        mbar_init(&bars.drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;

    int64_t issued = 0;  // (loader) chunks whose copies are issued
    // the V tile (and, one gate per head, the Q and K tiles) of chunk c: token rows
    // q_row0 + 64 c; query/key head hq
    int32_t q_row0 = 0, hq = 0;
    if (tid == kLoader) {
        q_row0 = (int32_t)(start + cb * C);
        hq = (int32_t)(h / (H / Hk));
    }
    auto issue_loads = [&](int64_t c) {
        const int stage = (int)(c % kStages);
        uint8_t *st = sm + stage * kStage;
        const uint8_t *blk = block_of(c);
        uint64_t *bar = &bars.full[stage];
        const int32_t row0 = q_row0 + (int32_t)c * C;
        if (ident) {  // a transition map reads W^T, K~ (or K) and the factors only
            mbar_arrive_expect_tx(bar, (uint32_t)(16384 + kTcKt + kTcFac));
            bulk_load(st + kStW, blk + kBlkW, 16384u, bar);
            if (KDA) {
                bulk_load(st + kStRest + kRestKt, blk + kBlkRest + kRestKt, (uint32_t)kTcKt, bar);
            } else {
                tma_load_3d(st + kStRest + kRestKt, &mk, 0, hq, row0, bar);
                tma_load_3d(st + kStRest + kRestKt + 8192, &mk, 64, hq, row0, bar);
            }
            bulk_load(st + kStRest + kRestFac, blk + kBlkRest + kRestFac, (uint32_t)kTcFac, bar);
        } else if (KDA) {
            mbar_arrive_expect_tx(bar, kStage);
            bulk_load(st, blk, (uint32_t)kTcWQ, bar);
            bulk_load(st + kStRest, blk + kBlkRest, (uint32_t)kTcRest, bar);
            tma_load_3d(st + kStV, &mv, 0, h, row0, bar);
            tma_load_3d(st + kStV + 8192, &mv, 64, h, row0, bar);
        } else {  // one gate per head: the Q and K tiles themselves (the output and U' are scaled)
            mbar_arrive_expect_tx(bar, kStage);
            bulk_load(st + kStW, blk + kBlkW, 16384u, bar);
            tma_load_3d(st + kStQ, &mq, 0, hq, row0, bar);
            tma_load_3d(st + kStQ + 8192, &mq, 64, hq, row0, bar);
            tma_load_3d(st + kStRest + kRestKt, &mk, 0, hq, row0, bar);
            tma_load_3d(st + kStRest + kRestKt + 8192, &mk, 64, hq, row0, bar);
            bulk_load(st + kStRest + kRestP, blk + kBlkRest + kRestP, (uint32_t)(kTcRest - kTcKt), bar);
            tma_load_3d(st + kStV, &mv, 0, h, row0, bar);
            tma_load_3d(st + kStV + 8192, &mv, 64, h, row0, bar);
        }
        issued = c + 1;
    };
    if (tid == kLoader)
        for (int64_t c = 0; c < kStages && c < nrun; ++c) issue_loads(c);

    float S[64];
    const int64_t srow = (int64_t)v * D + 64 * hf;  // this thread's part of a state
    if (start_kind == kStartGiven && s_init) {
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
            const float4 t = *reinterpret_cast<const float4 *>(s_init + srow + c);
            S[c] = t.x; S[c + 1] = t.y; S[c + 2] = t.z; S[c + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = (ident && 64 * hf + c == v) ? 1.f : 0.f;
    }

    // Output of chunk c held in registers: o[t / 16][t % 16] = token 32 hf + t, channel v;
    // stored in two halves (tokens 32 hf + 16 half ..), one during each MMA group.
    float o[2][16];
    auto store_output = [&](int64_t c, int half) {
        const int64_t ca = cb + c;
        const int L = (int)(len - ca * C < C ? len - ca * C : C);
        // 4 x 4 transposes (bf16) among the quads of lanes (4 adjacent channels):
        // afterwards lane j of a quad holds those 4 channels of token 4 b + j -> one
        // 8-byte store.
        const int j4 = lane & 3;
        const int64_t tstride = H * D;
        __nv_bfloat16 *op = out + ((start + ca * C + 32 * hf + j4) * H + h) * D + (v - j4);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
            const int b = 4 * half + bb;
            const float *x = &o[b >> 2][4 * (b & 3)];
            uint32_t p01 = pack_bf16(x[0], x[1]), p23 = pack_bf16(x[2], x[3]);
            quad_transpose_bf16(p01, p23, lane);
            if (32 * hf + 4 * b + j4 < L) *reinterpret_cast<uint2 *>(op + (int64_t)(4 * b) * tstride) = make_uint2(p01, p23);
        }
    };

    // Decay bound summed over the chunks run so far (zero-start segments) and the
    // first chunk from which the start state no longer matters.
    float lam = 0.f;
    int64_t m_first = nchunks;
    bool emit_prev = false;  // chunk c - 1 has an output to store
    // chunks until the next snapshot, and its index (snapshot strides are multiples of C)
    const int32_t kc = snap_stride > 0 ? (int32_t)(snap_stride / C) : 0;
    int32_t snap_left = kc > 0 ? kc - (int32_t)(cb % kc) : 0;
    int64_t snap_idx = kc > 0 ? cb / kc : 0;
    bool ok = true;
    int64_t c = 0;
    for (; c < nrun; ++c) {
        const int stage = (int)(c % kStages);
        uint8_t *st = sm + stage * kStage;
        const uint32_t st_u = smem_u32(st);
        const uint32_t par = (uint32_t)(c & 1);
        const uint8_t *rest = st + kStRest;
        const float *fac = reinterpret_cast<const float *>(rest + kRestFac);

        // (a) S0 -> bf16 pairs -> TMEM A operand (this thread: 32 columns of its row)
        {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = pack_bf16(S[32 * q + 2 * e], S[32 * q + 2 * e + 1]);
                tmem_st16u(tm + lane_off + kTmAS + 32 * hf + 16 * q, w);
            }
            tmem_wait_st();
        }
        ok = mbar_wait(&bars.full[stage], (uint32_t)((c / kStages) & 1)) && ok;
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // does this chunk write outputs, and its snapshot?
        const float lam_next = lam + fac[kFacLam];
        const bool emit = spec ? lam < kLamDrop : emit_any;
        const bool emit_state = spec ? lam_next < kLamDrop : emit_any;
        if (spec && emit && m_first == nchunks) m_first = c;

        // (b) D1 = [S0 W^T + V^T (-T'')^T | S0 Q^T]   (N = 64 + 64): [-U'^T, with U = T'' V |
        //     inter-chunk output]; a transition map drops the writes (D1 = S0 W^T, so
        //     again -U'^T) and has no output.  -U'^T is committed on its own: U' is formed
        //     from it while S0 Q^T runs.
        if (warp == kIssuer) {
            const uint64_t bw = sdesc_sw128(st_u + kStW, 8192, 1024), bq = sdesc_sw128(st_u + kStQ, 16, 1024);
            const uint32_t id_w = idesc_bf16(128, 64, 0, 1), id_q = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ts(tm + kTmD1, tm + kTmAS + kk * 8, bw + (uint64_t)((kk * 2048) >> 4), id_w, kk > 0);
            if (!ident) {
                const uint64_t av = sdesc_sw128(st_u + kStV, 8192, 1024), bt = sdesc_sw128(st_u + kStRest + kRestTn, 16, 1024);
                const uint32_t id_v = idesc_bf16(128, 64, 1, 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tm + kTmD1, av + (uint64_t)((kk * 2048) >> 4), bt + (uint64_t)((kk * 32) >> 4), id_v, 1);
            }
            mma_commit_warp(&bars.mma[0]);
            if (emit)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tm + kTmD1 + 64, tm + kTmAS + kk * 8,
                                bq + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id_q, kk > 0);
        }
        // every MMA of chunk c-1 has completed (step (e) waited for them), so its
        // stage can take chunk c+2
        if (tid == kLoader && c >= 1 && c + kStages - 1 < nrun) issue_loads(c + kStages - 1);
        // (d) D2 = [increment | U'^T P^T]   (N = 128 + 64, K = 64 tokens): [state increment |
        //     intra-chunk output] (the increment only, for a chunk without outputs); the
        //     increment is U'^T K~ (per-channel gate) or (diag(w) U')^T K (one gate per
        //     head).  It is committed on its own (the state is updated while U'^T P^T
        //     runs), then every product of the chunk.
        auto issue_d2 = [&] {
            const uint64_t bk = sdesc_sw128(st_u + kStRest + kRestKt, 8192, 1024),
                           bp = sdesc_sw128(st_u + kStRest + kRestP, 16, 1024);
            const uint32_t id_k = idesc_bf16(128, 128, 0, 1), id_p = idesc_bf16(128, 64, 0, 0);
            const uint32_t a_inc = tm + (KDA ? kTmAU : kTmAUw);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(tm + kTmD2, a_inc + kk * 8, bk + (uint64_t)((kk * 2048) >> 4), id_k, kk > 0);
            mma_commit_warp(&bars.mma[1]);
            if (emit)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tm + kTmD2 + 128, tm + kTmAU + kk * 8, bp + (uint64_t)((kk * 32) >> 4), id_p, kk > 0);
            mma_commit_warp(&bars.mma[2]);
        };
        // the first half of the previous chunk's output, while these MMAs run
        if (c >= 1 && emit_prev) store_output(c - 1, 0);

        // (c) U' = -D1 over tokens [32 hf, 32 hf + 32) -> TMEM A operand (and diag(w) U')
        ok = mbar_wait(&bars.mma[0], par) && ok;
        tc_fence_after();
        {
            float a0[16], a1[16];
            tmem_ld16(tm + lane_off + kTmD1 + 32 * hf, a0);
            tmem_ld16(tm + lane_off + kTmD1 + 32 * hf + 16, a1);
            tmem_wait_ld();
            const float4 *w4 = reinterpret_cast<const float4 *>(fac + kFacW + 32 * hf);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // tokens 32 hf + 16 hh .. + 15: 8 columns of each operand
                uint32_t wu[8], ww[8];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = 2 * hh + qq;  // tokens 32 hf + 8 q .. + 7
                    float wt[8] = {};
                    if (!KDA) {
                        const float4 wa = w4[2 * q], wb = w4[2 * q + 1];
                        wt[0] = wa.x; wt[1] = wa.y; wt[2] = wa.z; wt[3] = wa.w;
                        wt[4] = wb.x; wt[5] = wb.y; wt[6] = wb.z; wt[7] = wb.w;
                    }
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const float *acc = hh == 0 ? &a0[8 * qq + e] : &a1[8 * qq + e];
                        const float2 d = make_float2(-acc[0], -acc[1]);  // U'
                        wu[4 * qq + e / 2] = pack_bf16(d.x, d.y);
                        if (!KDA) {
                            const float2 dw = __fmul2_rn(make_float2(wt[e], wt[e + 1]), d);
                            ww[4 * qq + e / 2] = pack_bf16(dw.x, dw.y);
                        }
                    }
                }
                tmem_st8u(tm + lane_off + kTmAU + 16 * hf + 8 * hh, wu);
                if (!KDA) tmem_st8u(tm + lane_off + kTmAUw + 16 * hf + 8 * hh, ww);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // (d)
        if (warp == kIssuer) issue_d2();

        // the second half of the previous chunk's output, while these MMAs run
        if (c >= 1 && emit_prev) store_output(c - 1, 1);

        // (e) S = gam_L S0 + increment (columns [64 hf, 64 hf + 64); per key channel
        // for KDA) and the output o = S0 Qs^T + U'^T P^T (one gate per head: Qs^T = Q^T
        // scaled per token)
        const float gl = fac[kFacGL];
        ok = mbar_wait(&bars.mma[1], par) && ok;
        tc_fence_after();
        {
            float a[4][16];
#pragma unroll
            for (int c0 = 0; c0 < 4; ++c0) tmem_ld16(tm + lane_off + kTmD2 + 64 * hf + 16 * c0, a[c0]);
            tmem_wait_ld();
            if (KDA) {
                const float4 *gl4 = reinterpret_cast<const float4 *>(fac + kFacGL + 64 * hf);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 f = gl4[c4];
                    const float *ai = &a[c4 >> 2][(4 * c4) & 15];
                    const float2 s01 = __ffma2_rn(make_float2(f.x, f.y), make_float2(S[4 * c4], S[4 * c4 + 1]),
                                                  make_float2(ai[0], ai[1]));
                    const float2 s23 = __ffma2_rn(make_float2(f.z, f.w), make_float2(S[4 * c4 + 2], S[4 * c4 + 3]),
                                                  make_float2(ai[2], ai[3]));
                    S[4 * c4] = s01.x; S[4 * c4 + 1] = s01.y; S[4 * c4 + 2] = s23.x; S[4 * c4 + 3] = s23.y;
                }
            } else {
                const float2 gl2 = make_float2(gl, gl);
#pragma unroll
                for (int c0 = 0; c0 < 4; ++c0)
#pragma unroll
                    for (int t = 0; t < 16; t += 2) {
                        const float2 r = __ffma2_rn(gl2, make_float2(S[16 * c0 + t], S[16 * c0 + t + 1]),
                                                    make_float2(a[c0][t], a[c0][t + 1]));
                        S[16 * c0 + t] = r.x;
                        S[16 * c0 + t + 1] = r.y;
                    }
            }
        }
        ok = mbar_wait(&bars.mma[2], par) && ok;
        tc_fence_after();
        {
            // (the output columns are read whether or not this chunk writes them: a
            // value that is sometimes kept would stay live across the whole chunk)
            float o2[2][16];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tmem_ld16(tm + lane_off + kTmD1 + 64 + 32 * hf + 16 * q, o[q]);
                tmem_ld16(tm + lane_off + kTmD2 + 128 + 32 * hf + 16 * q, o2[q]);
            }
            tmem_wait_ld();
            if (KDA) {
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                    for (int t = 0; t < 16; t += 2) {
                        const float2 r = __fadd2_rn(make_float2(o[q][t], o[q][t + 1]), make_float2(o2[q][t], o2[q][t + 1]));
                        o[q][t] = r.x;
                        o[q][t + 1] = r.y;
                    }
            } else {  // S0 Q^T scaled per token by scale exp(b_i)
                const float4 *sg4 = reinterpret_cast<const float4 *>(fac + kFacQs + 32 * hf);
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                    for (int t4 = 0; t4 < 4; ++t4) {
                        const float4 f = sg4[4 * q + t4];
                        float *ot = &o[q][4 * t4];
                        const float *o2t = &o2[q][4 * t4];
                        const float2 r01 = __ffma2_rn(make_float2(ot[0], ot[1]), make_float2(f.x, f.y), make_float2(o2t[0], o2t[1]));
                        const float2 r23 = __ffma2_rn(make_float2(ot[2], ot[3]), make_float2(f.z, f.w), make_float2(o2t[2], o2t[3]));
                        ot[0] = r01.x; ot[1] = r01.y; ot[2] = r23.x; ot[3] = r23.y;
                    }
            }
        }

        // snapshot after every snap_stride tokens of the sequence (a multiple of the
        // chunk): snapshot snap_idx follows chunk (snap_idx + 1) kc - 1 of the sequence
        if (kc > 0 && --snap_left == 0) {
            snap_left = kc;
            if (emit_state && snaps && snap_idx < n_snap) {
                float *dst = snaps + (((n * n_snap + snap_idx) * H + h) * D + v) * (int64_t)D + 64 * hf;
#pragma unroll
                for (int cc = 0; cc < 64; cc += 4)
                    *reinterpret_cast<float4 *>(dst + cc) = make_float4(S[cc], S[cc + 1], S[cc + 2], S[cc + 3]);
            }
            ++snap_idx;
        }
        lam = lam_next;
        emit_prev = emit;
        if (__syncthreads_or(!ok)) {  // a wait gave up: every thread leaves as failed
            ok = false;
            break;
        }
    }
    if (ok && nrun > 0 && emit_prev) {
        store_output(nrun - 1, 0);
        store_output(nrun - 1, 1);
    }
    if (!ok) {
        // A wait gave up: record it, then wait (bounded) for the copies still in
        // flight and for every MMA issued, before the shared memory and the TMEM
        // columns are given back.
        if (tid == 0) flag_error(err, GDN_DEV_TIMEOUT_SCAN);
        if (tid == kLoader)
            for (int64_t j = c; j < issued; ++j) mbar_wait(&bars.full[j % kStages], (uint32_t)((j / kStages) & 1));
        if (warp == kIssuer) {
            mma_commit_warp(&bars.drain);
            mbar_wait(&bars.drain, 0);
        }
    }
    float *s_end2 = nullptr;  // a zero-start last segment whose end no longer depends on its start
    if (SPLIT && spec) {
        const bool exact_end = lam < kLamDrop;
        if (ok && tid == 0) *split_rec(sp, 0, N, n, g, H, h) = (int32_t)(exact_end ? m_first : nchunks);
        if (exact_end && g == sp.G - 1 && final_state) s_end2 = final_state + sh;
    }
    if (ok) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            float *dst = k ? s_end2 : s_end;
            if (!dst) continue;
#pragma unroll
            for (int cc = 0; cc < 64; cc += 4)
                *reinterpret_cast<float4 *>(dst + srow + cc) = make_float4(S[cc], S[cc + 1], S[cc + 2], S[cc + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

__global__ void __launch_bounds__(kThreads, 1) gdn_scan_tc(GDN_SCAN_PARAMS) { scan_body<false, false>(GDN_SCAN_ARGS); }
__global__ void __launch_bounds__(kThreads, 1) gdn_scan_split_tc(GDN_SCAN_PARAMS) { scan_body<false, true>(GDN_SCAN_ARGS); }
template <bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1) gdn_scan_kda_tc(GDN_SCAN_PARAMS) { scan_body<true, SPLIT>(GDN_SCAN_ARGS); }

// Start states of the segments: S_{g+1} = S_g M_g + B_g for g = 1 .. G-2 where M_g
// was formed (S_1 comes from pass 1; where M_g was not formed the start of segment
// g+1 is B_g itself, which pass 2 reads from where pass 1 left it), one block per
// (sequence, head), fp32 on the CUDA cores.  S_g is S_1, the result of the previous
// step, or B_{g-1}.
// Thread t computes a 4-row x 16-column tile (rows 4 (t % 32) .., columns
// 16 (t / 32) ..), so every value loaded from shared memory feeds 4 or 16 FMAs.
// S_g is kept transposed (column k = row of St) so the 4 row values of a k are
// one 16-byte load.
constexpr uint32_t kCombSmem = (uint32_t)(2 * D * D) * 4;

__global__ void __launch_bounds__(kThreads, 1) gdn_seg_combine(const ScanSplit sp, int64_t N, int64_t H) {
    extern __shared__ float4 comb_raw[];
    float *St = reinterpret_cast<float *>(comb_raw);  // S_g transposed: St[k][v]
    float *Ms = St + D * D;                             // M_g: Ms[k][c]
    const int64_t n = blockIdx.x, h = blockIdx.y;
    const int tid = threadIdx.x, r0 = 4 * (tid & 31), c0 = 16 * (tid >> 5);
    auto load_st = [&](const float *src) {  // St = src^T
        for (int e = tid; e < D * D / 4; e += kThreads) {  // lanes take consecutive rows v
            const int v = e & 127, c4 = e >> 7;
            const float4 x = *reinterpret_cast<const float4 *>(src + v * D + 4 * c4);
            St[(4 * c4) * D + v] = x.x;
            St[(4 * c4 + 1) * D + v] = x.y;
            St[(4 * c4 + 2) * D + v] = x.z;
            St[(4 * c4 + 3) * D + v] = x.w;
        }
    };
    bool have = false;  // St holds S_g
    for (int g = 1; g <= sp.G - 2; ++g) {
        if (*split_rec(sp, 1, N, n, g, H, h) == 0) {  // uniform over the block
            have = false;
            continue;
        }
        if (!have) {
            __syncthreads();
            load_st(g == 1 ? split_state(sp, n, 1, 2, H, h) : split_state(sp, n, g - 1, 0, H, h));
        }
        const float *M = split_state(sp, n, g, 1, H, h), *B = split_state(sp, n, g, 0, H, h);
        for (int e = tid; e < D * D / 4; e += kThreads)
            reinterpret_cast<float4 *>(Ms)[e] = reinterpret_cast<const float4 *>(M)[e];
        float acc[4][16];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 16; c += 4) {
                const float4 b4 = *reinterpret_cast<const float4 *>(B + (r0 + i) * D + c0 + c);
                acc[i][c] = b4.x; acc[i][c + 1] = b4.y; acc[i][c + 2] = b4.z; acc[i][c + 3] = b4.w;
            }
        __syncthreads();
#pragma unroll 2
        for (int k = 0; k < D; ++k) {
            const float4 s4 = *reinterpret_cast<const float4 *>(St + k * D + r0);
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
            float mv[16];
#pragma unroll
            for (int c = 0; c < 16; c += 4) *reinterpret_cast<float4 *>(mv + c) = *reinterpret_cast<const float4 *>(Ms + k * D + c0 + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[i][c] = fmaf(sv[i], mv[c], acc[i][c]);
        }
        __syncthreads();  // every read of S_g and M_g is done
        float *dst = split_state(sp, n, g + 1, 2, H, h);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int c = 0; c < 16; c += 4)
                *reinterpret_cast<float4 *>(dst + (r0 + i) * D + c0 + c) =
                    make_float4(acc[i][c], acc[i][c + 1], acc[i][c + 2], acc[i][c + 3]);
#pragma unroll
            for (int c = 0; c < 16; ++c) St[(c0 + c) * D + r0 + i] = acc[i][c];
        }
        have = true;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// (rows, H, 128) tensor of bf16 (tiles of 64 tokens x 64 channels of one head) or
// fp32 (tiles of 64 tokens x 32 channels), 128-byte swizzle.
gdn_status make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t H, bool f32 = false) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(GDN_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t es_bytes = f32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * es_bytes, (cuuint64_t)H * D * es_bytes};
    cuuint32_t box[3] = {f32 ? 32u : 64u, 1, 64}, es[3] = {1, 1, 1};
    CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GDN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return GDN_OK;
}

}  // namespace

bool tc_eligible(const gdn_desc &d) {
    return d.dtype == GDN_BF16 && d.dk == 128 && d.dv == 128 && (d.gate == GDN_GATE_HEAD || d.gate == GDN_GATE_CHANNEL);
}

gdn_status launch_chunk_tc(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s) {
    gdn_status st = launch_chunk_table(p, a, s);
    if (st != GDN_OK) return st;
    const int32_t *off = a.cu_seqlens ? reinterpret_cast<const int32_t *>(a.ws + p.off_chunk_offsets) : nullptr;
    uint8_t *blocks = reinterpret_cast<uint8_t *>(a.ws + p.off_W);
    if (p.H > 65535 || p.max_chunks > 0x7fffffffLL || a.N > 0x7fffffffLL)
        return fail(GDN_ERR_UNSUPPORTED, "grid too large");
    CUtensorMap mq, mk, mv, mg;
    memset(&mq, 0, sizeof mq);
    memset(&mk, 0, sizeof mk);
    memset(&mv, 0, sizeof mv);
    memset(&mg, 0, sizeof mg);
    if (p.rows > 0) {
        if ((st = make_map(&mq, a.q, p.rows, a.Hk)) != GDN_OK) return st;
        if ((st = make_map(&mk, a.k, p.rows, a.Hk)) != GDN_OK) return st;
        if ((st = make_map(&mv, a.v, p.rows, p.H)) != GDN_OK) return st;
        if (p.per_channel && (st = make_map(&mg, a.g, p.rows, p.H, true)) != GDN_OK) return st;
    }
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(gdn_prep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem);
        // four blocks per SM need the whole shared-memory carveout
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gdn_prep_tc, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        const void *scans[4] = {(const void *)gdn_scan_tc, (const void *)gdn_scan_split_tc,
                                (const void *)gdn_scan_kda_tc<false>, (const void *)gdn_scan_kda_tc<true>};
        for (const void *k : scans)
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScanSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gdn_seg_combine, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)kCombSmem);
    });
    if (attr_err != cudaSuccess) return fail(GDN_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(attr_err));
    if (p.max_chunks > 0 && p.rows > 0) {
        if (p.per_channel) {
            if ((st = tc::launch_prep_kda(mq, mk, mg, p, a, off, blocks, s)) != GDN_OK) return st;
        } else {
            const dim3 grid((unsigned)p.max_chunks, (unsigned)p.H);
            log_launch("gdn_prep_tc", grid, dim3(kThreads), kPrepSmem);
            LaunchScope ls("gdn_prep_tc", s);
            gdn_prep_tc<<<grid, kThreads, kPrepSmem, s>>>(mq, mk, a.g, a.beta, a.cu_seqlens, off, a.N, a.T, p.rows,
                                                          p.H, a.Hk, a.scale, blocks, p.split_G >= 2 ? 1 : 0,
                                                          a.status);
            if ((st = check_launch("gdn_prep_tc")) != GDN_OK) return st;
        }
    }
    ScanSplit sp{1, 0, 0, nullptr, nullptr};
    const int scan_block = kThreads;
    if (p.split_G < 2) {
        if (a.N * p.H > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
        auto kern = p.per_channel ? gdn_scan_kda_tc<false> : gdn_scan_tc;
        const dim3 grid((unsigned)a.N, (unsigned)p.H);
        log_launch(p.per_channel ? "gdn_scan_kda_tc" : "gdn_scan_tc", grid, dim3(scan_block), kScanSmem);
        LaunchScope ls(p.per_channel ? "gdn_scan_kda_tc" : "gdn_scan_tc", s);
        kern<<<grid, scan_block, kScanSmem, s>>>(mq, mk, mv, a.h0, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, a.Hk,
                                                 p.max_chunks, a.snapshot_stride, a.n_snap, blocks,
                                                 (__nv_bfloat16 *)a.out, a.final_state, a.snapshots, sp, a.status);
        return check_launch("gdn_scan_tc");
    }
    // sequence split: pass 1 (every segment, then the transition maps), the chained
    // start states (G >= 3), pass 2 (the leading chunks of segments 1 .. G-1)
    const int split_block = kThreads;
    auto kern = p.per_channel ? gdn_scan_kda_tc<true> : gdn_scan_split_tc;
    float *states = reinterpret_cast<float *>(a.ws + p.off_split);
    sp = ScanSplit{p.split_G, p.split_seg, 1, states,
                   reinterpret_cast<int32_t *>(states + (size_t)a.N * p.split_G * 3 * p.H * p.dv * p.dk)};
    const int64_t nh = a.N * p.H, grid1 = nh * (2 * (int64_t)p.split_G - 2), grid2 = nh * (p.split_G - 1);
    if (grid1 > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "grid too large");
    {
        log_launch("gdn_scan (pass 1)", dim3((unsigned)grid1), dim3(split_block), kScanSmem);
        LaunchScope ls(p.per_channel ? "gdn_scan_kda_tc (pass 1)" : "gdn_scan_split_tc (pass 1)", s);
        kern<<<(unsigned)grid1, split_block, kScanSmem, s>>>(mq, mk, mv, a.h0, nullptr, nullptr, a.N, a.T, p.rows,
                                                             p.H, a.Hk, p.max_chunks, a.snapshot_stride, a.n_snap,
                                                             blocks,
                                                             (__nv_bfloat16 *)a.out, a.final_state, a.snapshots, sp,
                                                             a.status);
    }
    if ((st = check_launch("gdn_scan_tc")) != GDN_OK) return st;
    if (p.split_G >= 3) {
        const dim3 grid((unsigned)a.N, (unsigned)p.H);
        log_launch("gdn_seg_combine", grid, dim3(kThreads), kCombSmem);
        LaunchScope ls("gdn_seg_combine", s);
        gdn_seg_combine<<<grid, kThreads, kCombSmem, s>>>(sp, a.N, p.H);
        if ((st = check_launch("gdn_seg_combine")) != GDN_OK) return st;
    }
    sp.pass = 2;
    {
        log_launch("gdn_scan (pass 2)", dim3((unsigned)grid2), dim3(split_block), kScanSmem);
        LaunchScope ls(p.per_channel ? "gdn_scan_kda_tc (pass 2)" : "gdn_scan_split_tc (pass 2)", s);
        kern<<<(unsigned)grid2, split_block, kScanSmem, s>>>(mq, mk, mv, a.h0, nullptr, nullptr, a.N, a.T, p.rows,
                                                             p.H, a.Hk, p.max_chunks, a.snapshot_stride, a.n_snap,
                                                             blocks,
                                                             (__nv_bfloat16 *)a.out, a.final_state, a.snapshots, sp,
                                                             a.status);
    }
    return check_launch("gdn_scan_tc");
}

SplitChoice choose_split(int64_t N, int64_t H, int64_t nch, int sms) {
    SplitChoice best{1, (int32_t)nch};
    if (sms <= 0 || nch < 64) return best;
    auto waves = [sms](int64_t ctas) { return (double)((ctas + sms - 1) / sms); };
    // Costs in chunk steps of one block.  An extra launch costs about 4, a combine
    // step about 4 with a transition map and 0.5 without.  With gates that forget
    // within a few chunks pass 1 is the whole cost apart from a short pass 2
    // (kRerun chunks, a guess); with gates that keep the state alive pass 1 also
    // forms the transition maps and pass 2 reruns whole segments.  The split is
    // chosen for the first case, as long as the second stays within 1.3 times the
    // unsplit scan.
    constexpr double kRerun = 16.0;
    const double unsplit = waves(N * H) * (double)nch;
    double best_cost = 0.95 * unsplit;
    for (int64_t G = 2; G <= 128; ++G) {
        const int64_t seg = (nch + G - 1) / G;
        if (seg < 32) break;
        const int64_t Gr = (nch + seg - 1) / seg;  // no empty segments
        if (Gr < 2) continue;
        const double comb = Gr >= 3 ? 4.0 : 0.0;
        const double fast = waves(N * H * Gr) * seg + (seg < kRerun ? seg : kRerun) + 4.0 + comb + 0.5 * (Gr - 2);
        const double slow = waves(N * H * (2 * Gr - 2)) * seg + waves(N * H * (Gr - 1)) * seg + 4.0 + comb +
                            4.0 * (Gr - 2);
        if (fast < best_cost && slow <= 1.3 * unsplit) {
            best_cost = fast;
            best = SplitChoice{(int32_t)Gr, (int32_t)seg};
        }
    }
    return best;
}

}  // namespace gdn
