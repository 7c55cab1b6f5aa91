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
//                K, Q, V; one MMA gives [K;Q] K^T (M = 128: the K rows give the
//                Gram matrix, the Q rows give Q K^T); the unit-lower-triangular
//                system is solved on CUDA cores in fp32; two MMAs give W^T and
//                U^T.  W^T and P are written to the workspace as ready-made
//                128-byte-swizzled shared-memory operand images, so the scan
//                copies them with plain bulk copies.
//   gdn_scan_tc  one CTA per (sequence, head).  The fp32 state lives in
//                registers (thread v owns row v); per chunk it is rounded to a
//                bf16 operand in shared memory and four MMAs (S0 W^T, S0 Q^T,
//                U' P^T, U'_w K) with fp32 accumulators in TMEM produce U', O and
//                the state increment.  The next chunk's operands are prefetched
//                by TMA / bulk copies into a second stage while this one runs.
//
// All MMAs are M = 128 (the 128 rows of the state, or the 64 K rows stacked
// on the 64 Q rows), so the accumulator rows map 1:1 onto TMEM lanes and
// every thread reads exactly its own row.
#include <cudaTypedefs.h>

#include <string.h>

#include <mutex>

#include "chunk_common.cuh"
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = kChunk;  // 64
constexpr int D = 128;     // d_k = d_v
constexpr int kThreads = 128;

// ---------------------------------------------------------------------------
// Device error flag: set by a kernel whose bounded wait ran out.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void flag_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint8_t *align1024(unsigned char *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// ===========================================================================
// Prep: chunk-local quantities
// ===========================================================================
// Shared memory (1024-aligned):
//   KQ   [0, 32K)     K and Q tiles stacked as the M = 128 operand:
//                     [c-block 0: K rows | Q rows][c-block 1: K rows | Q rows]
//   V    [32K, 48K)   V tile [c-block 0][c-block 1]
//   Tp   [48K, 56K)   T diag(beta gam)  (bf16, K-major rows i)
//   Tpp  [56K, 64K)   T diag(beta)
//   A (fp32 64 x 64) reuses the Q rows once the first MMA has consumed them:
//     rows 0..31 in [8K, 16K), rows 32..63 in [24K, 32K).
constexpr uint32_t kPrepSmem = 65536 + 1024;

__device__ __forceinline__ uint32_t a_offset(int i, int q4) {
    // row i of A, 16-byte chunk q4 (floats 4*q4 .. 4*q4+3), chunks rotated per row
    const uint32_t base = i < 32 ? 8192u : 24576u;
    return base + (uint32_t)(i & 31) * 256u + (uint32_t)((q4 ^ (i & 15)) << 4);
}

__global__ void __launch_bounds__(kThreads)
gdn_prep_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
            const __grid_constant__ CUtensorMap mv, const float *__restrict__ g, const float *__restrict__ beta,
            const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows,
            int64_t H, float scale, uint8_t *__restrict__ Wimg, uint8_t *__restrict__ Pimg,
            __nv_bfloat16 *__restrict__ Ut, float *__restrict__ bcum, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *KQ = sm, *Vt = sm + 32768, *Tp = sm + 49152, *Tpp = sm + 57344;
    __shared__ uint64_t bar_ld, bar_mma;
    __shared__ uint32_t tmem_base;
    __shared__ float s_b[C], s_beta[C];

    const int64_t chunk = blockIdx.x, h = blockIdx.y;
    ChunkLoc loc;
    if (!locate_chunk(chunk, cu, off, N, T, rows, loc)) return;
    const int L = (int)loc.len;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ch = chunk * H + h;
    const int32_t tok0 = (int32_t)loc.start;

    if (tid == 0) {
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_ld, 6 * 8192);
        tma_load_3d(KQ + 0, &mk, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(KQ + 16384, &mk, 64, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(KQ + 8192, &mq, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(KQ + 24576, &mq, 64, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(Vt + 0, &mv, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(Vt + 8192, &mv, 64, (int32_t)h, tok0, &bar_ld);
    }
    // gates: beta and the in-chunk cumulative log gate (rows >= L: beta = 0, g = 0)
    if (tid < C) {
        const bool in = tid < L;
        s_beta[tid] = in ? beta[(int64_t)(tok0 + tid) * H + h] : 0.f;
        float x = in ? g[(int64_t)(tok0 + tid) * H + h] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        s_b[tid] = x;
    }
    __syncthreads();
    if (tid >= 32 && tid < C) s_b[tid] += s_b[31];
    __syncthreads();

    bool ok = mbar_wait(&bar_ld, 0);
    if (tid == 0 && ok) {
        tc_fence_after();
        const uint32_t kq = smem_u32(KQ);
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16(tm, sdesc_sw128(kq + o, 16, 1024), sdesc_sw128(kq + o, 16, 1024), id, kk > 0);
        }
        mma_commit(&bar_mma);
    }
    ok = ok && mbar_wait(&bar_mma, 0);
    tc_fence_after();

    // Epilogue 1: rows 0..63 of the accumulator are K K^T -> A (fp32, smem);
    // rows 64..127 are Q K^T -> P (bf16 operand image, workspace).
    if (ok) {
        const uint32_t taddr = tm + ((uint32_t)(warp * 32) << 16);
        const bool is_a = tid < C;
        const int i = is_a ? tid : tid - C;
        const float bi = s_b[i];
        const float pre = is_a ? s_beta[i] : scale;
        uint8_t *prow = Pimg + (size_t)ch * kTcPImg + (size_t)i * 128;
#pragma unroll
        for (int c0 = 0; c0 < C; c0 += 16) {
            float v[16];
            tmem_ld16(taddr + c0, v);
            tmem_wait_ld();
            float r[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int j = c0 + t;
                const bool keep = i < L && (is_a ? j < i : j <= i);
                r[t] = keep ? pre * __expf(bi - s_b[j]) * v[t] : 0.f;
            }
            if (is_a) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(KQ + a_offset(i, c0 / 4 + q)) =
                        make_float4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            } else {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int chunk16 = c0 / 8 + q;  // 8 bf16 per 16-byte chunk
                    st_global_v4(prow + ((chunk16 ^ (i & 7)) << 4), pack_bf16(r[8 * q], r[8 * q + 1]),
                                 pack_bf16(r[8 * q + 2], r[8 * q + 3]), pack_bf16(r[8 * q + 4], r[8 * q + 5]),
                                 pack_bf16(r[8 * q + 6], r[8 * q + 7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // Solve T = (I + A)^-1, one column per thread (forward substitution in
    // fp32); then T' = T diag(beta gam), T'' = T diag(beta) as bf16 operands.
    if (ok && tid < C) {
        const int col = tid;
        float x[C];
#pragma unroll
        for (int i = 0; i < C; ++i) {
            float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
            for (int q = 0; q < (i + 3) / 4; ++q) {
                const float4 a4 = *reinterpret_cast<const float4 *>(KQ + a_offset(i, q));
                if (4 * q + 0 < i) acc0 += a4.x * x[4 * q + 0];
                if (4 * q + 1 < i) acc1 += a4.y * x[4 * q + 1];
                if (4 * q + 2 < i) acc2 += a4.z * x[4 * q + 2];
                if (4 * q + 3 < i) acc3 += a4.w * x[4 * q + 3];
            }
            x[i] = (i == col) ? 1.f : -((acc0 + acc1) + (acc2 + acc3));
        }
        const float bc = s_beta[col];
        const float bgc = bc * __expf(s_b[col]);
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const uint32_t o = sw128_offset(i, col >> 3) + (col & 7) * 2;
            *reinterpret_cast<__nv_bfloat16 *>(Tp + o) = __float2bfloat16_rn(x[i] * bgc);
            *reinterpret_cast<__nv_bfloat16 *>(Tpp + o) = __float2bfloat16_rn(x[i] * bc);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // W^T = K^T T'^T (M = d_k rows), U^T = V^T T''^T (M = d_v rows); K = 64 tokens.
    if (tid == 0 && ok) {
        const uint32_t kq = smem_u32(KQ), vt = smem_u32(Vt), tp = smem_u32(Tp), tpp = smem_u32(Tpp);
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tm, sdesc_sw128(kq + kk * 2048, 16384, 1024), sdesc_sw128(tp + kk * 32, 16, 1024), id, kk > 0);
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tm + 64, sdesc_sw128(vt + kk * 2048, 8192, 1024), sdesc_sw128(tpp + kk * 32, 16, 1024), id,
                     kk > 0);
        mma_commit(&bar_mma);
    }
    ok = ok && mbar_wait(&bar_mma, 1);
    tc_fence_after();

    // Epilogue 2: thread r owns row r (channel r) of W^T and U^T.
    if (ok) {
        const uint32_t taddr = tm + ((uint32_t)(warp * 32) << 16);
        const int r = tid;
        uint8_t *wrow = Wimg + (size_t)ch * kTcWImg + (size_t)r * 128;
        uint8_t *urow = reinterpret_cast<uint8_t *>(Ut) + (size_t)ch * kTcUt + (size_t)r * 128;
#pragma unroll
        for (int c0 = 0; c0 < C; c0 += 16) {
            float w[16], u[16];
            tmem_ld16(taddr + c0, w);
            tmem_ld16(taddr + 64 + c0, u);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int chunk16 = c0 / 8 + q;
                st_global_v4(wrow + ((chunk16 ^ (r & 7)) << 4), pack_bf16(w[8 * q], w[8 * q + 1]),
                             pack_bf16(w[8 * q + 2], w[8 * q + 3]), pack_bf16(w[8 * q + 4], w[8 * q + 5]),
                             pack_bf16(w[8 * q + 6], w[8 * q + 7]));
                st_global_v4(urow + chunk16 * 16, pack_bf16(u[8 * q], u[8 * q + 1]), pack_bf16(u[8 * q + 2], u[8 * q + 3]),
                             pack_bf16(u[8 * q + 4], u[8 * q + 5]), pack_bf16(u[8 * q + 6], u[8 * q + 7]));
            }
        }
        if (tid < C) bcum[ch * C + tid] = s_b[tid];
    } else if (tid == 0) {
        flag_error(err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 128);
}

// ===========================================================================
// Scan: the chunks of each sequence in order
// ===========================================================================
// Shared memory (1024-aligned): two stages of per-chunk operands, then the
// per-chunk A operands written by the threads.
constexpr uint32_t kStQ = 0, kStK = 16384, kStW = 32768, kStP = 49152, kStB = 57344, kStage = 58368;
constexpr uint32_t kSImg = 2 * kStage;          // state, bf16, K-major rows v, 2 x 16K
constexpr uint32_t kUpImg = kSImg + 32768;      // U' (rows v, K = tokens)
constexpr uint32_t kUwImg = kUpImg + 16384;     // U' scaled by exp(b_L - b_i)
constexpr uint32_t kScanSmem = kUwImg + 16384 + 1024;
constexpr uint32_t kStageBytes = 2 * 16384 + 16384 + 8192 + 256;

struct ScanBars {
    uint64_t full[2];
    uint64_t mma[4];
};

__global__ void __launch_bounds__(kThreads, 1)
gdn_scan_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
            const float *h0, const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int64_t N, int64_t T,
            int64_t rows, int64_t H, int64_t max_chunks, float scale, int64_t snap_stride, int64_t n_snap,
            const uint8_t *__restrict__ Wimg, const uint8_t *__restrict__ Pimg, const __nv_bfloat16 *__restrict__ Ut,
            const float *__restrict__ bcum, __nv_bfloat16 *__restrict__ out, float *final_state,
            float *__restrict__ snaps, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    __shared__ ScanBars bars;
    __shared__ uint32_t tmem_base;
    const int64_t n = blockIdx.x, h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int v = tid;  // state row owned by this thread

    int64_t start, len;
    seq_bounds(cu, n, T, rows, start, len);
    int64_t nchunks = (len + C - 1) / C;
    const int64_t chunk0 = cu ? (int64_t)off[n] : n * ((T + C - 1) / C);
    if (chunk0 + nchunks > max_chunks) nchunks = max_chunks > chunk0 ? max_chunks - chunk0 : 0;

    if (tid == 0) {
        mbar_init(&bars.full[0], 1);
        mbar_init(&bars.full[1], 1);
        for (int i = 0; i < 4; ++i) mbar_init(&bars.mma[i], 1);
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
    const uint32_t acc1 = tm, acc2 = tm + 64, acc3 = tm + 128, acc4 = tm + 256;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    auto issue_loads = [&](int64_t c) {
        const int stage = (int)(c & 1);
        uint8_t *st = sm + stage * kStage;
        const int64_t chh = (chunk0 + c) * H + h;
        const int32_t tok = (int32_t)(start + c * C);
        uint64_t *bar = &bars.full[stage];
        mbar_arrive_expect_tx(bar, kStageBytes);
        tma_load_3d(st + kStQ, &mq, 0, (int32_t)h, tok, bar);
        tma_load_3d(st + kStQ + 8192, &mq, 64, (int32_t)h, tok, bar);
        tma_load_3d(st + kStK, &mk, 0, (int32_t)h, tok, bar);
        tma_load_3d(st + kStK + 8192, &mk, 64, (int32_t)h, tok, bar);
        bulk_load(st + kStW, Wimg + (size_t)chh * kTcWImg, (uint32_t)kTcWImg, bar);
        bulk_load(st + kStP, Pimg + (size_t)chh * kTcPImg, (uint32_t)kTcPImg, bar);
        bulk_load(st + kStB, bcum + (size_t)chh * C, (uint32_t)kTcB, bar);
    };
    if (tid == 0) {
        if (nchunks > 0) issue_loads(0);
        if (nchunks > 1) issue_loads(1);
    }

    // state row v in registers
    float S[D];
    const int64_t srow = ((n * H + h) * D + v) * (int64_t)D;
    if (h0) {
#pragma unroll
        for (int c = 0; c < D; c += 4) {
            const float4 t = *reinterpret_cast<const float4 *>(h0 + srow + c);
            S[c] = t.x; S[c + 1] = t.y; S[c + 2] = t.z; S[c + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < D; ++c) S[c] = 0.f;
    }

    const uint32_t s_img = smem_u32(sm + kSImg), up_img = smem_u32(sm + kUpImg), uw_img = smem_u32(sm + kUwImg);
    bool ok = true;
    for (int64_t c = 0; c < nchunks && ok; ++c) {
        const int stage = (int)(c & 1);
        uint8_t *st = sm + stage * kStage;
        const uint32_t st_u = smem_u32(st);
        const int64_t chh = (chunk0 + c) * H + h;
        const int L = (int)(len - c * C < C ? len - c * C : C);
        const int64_t tok0 = start + c * C;
        const uint32_t par = (uint32_t)(c & 1);

        // this chunk's U row (U[i, v], i = 0..63), bf16
        uint4 ur[8];
        const uint4 *usrc = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(Ut) +
                                                            (size_t)chh * kTcUt + (size_t)v * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) ur[q] = usrc[q];

        // (a) S0 -> bf16 operand (K-major rows v, two 64-column blocks)
#pragma unroll
        for (int blk = 0; blk < 2; ++blk)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float *s8 = S + blk * 64 + q * 8;
                st_shared_v4(s_img + blk * 16384 + sw128_offset(v, q), pack_bf16(s8[0], s8[1]), pack_bf16(s8[2], s8[3]),
                             pack_bf16(s8[4], s8[5]), pack_bf16(s8[6], s8[7]));
            }
        fence_async_smem();
        ok = mbar_wait(&bars.full[stage], (uint32_t)((c >> 1) & 1));
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (!ok) break;

        // (b) acc1 = S0 W^T, acc2 = S0 Q^T
        if (tid == 0) {
            const uint32_t id_w = idesc_bf16(128, 64, 0, 1), id_q = idesc_bf16(128, 64, 0, 0);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(acc1, sdesc_sw128(s_img + o, 16, 1024), sdesc_sw128(st_u + kStW + kk * 2048, 16384, 1024),
                         id_w, kk > 0);
            }
            mma_commit(&bars.mma[0]);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16(acc2, sdesc_sw128(s_img + o, 16, 1024),
                         sdesc_sw128(st_u + kStQ + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_q, kk > 0);
            }
            mma_commit(&bars.mma[1]);
        }

        // (c) U' = U - S0 W^T; write U' and U' * exp(b_L - b_i) as bf16 operands
        const float *bs = reinterpret_cast<const float *>(st + kStB);
        const float bl = bs[L - 1];
        ok = mbar_wait(&bars.mma[0], par);
        tc_fence_after();
        if (ok) {
#pragma unroll
            for (int c0 = 0; c0 < C; c0 += 16) {
                float a[16];
                tmem_ld16(acc1 + lane_off + c0, a);
                tmem_wait_ld();
                float up[16], uw[16];
#pragma unroll
                for (int t = 0; t < 16; t += 2) {
                    const uint32_t pr = (&ur[0].x)[(c0 + t) / 2];
                    const __nv_bfloat162 u2 = *reinterpret_cast<const __nv_bfloat162 *>(&pr);
                    const int i = c0 + t;
                    up[t] = i < L ? __low2float(u2) - a[t] : 0.f;
                    up[t + 1] = i + 1 < L ? __high2float(u2) - a[t + 1] : 0.f;
                    uw[t] = up[t] * __expf(bl - bs[i]);
                    uw[t + 1] = up[t + 1] * __expf(bl - bs[i + 1]);
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int chunk16 = c0 / 8 + q;
                    st_shared_v4(up_img + sw128_offset(v, chunk16), pack_bf16(up[8 * q], up[8 * q + 1]),
                                 pack_bf16(up[8 * q + 2], up[8 * q + 3]), pack_bf16(up[8 * q + 4], up[8 * q + 5]),
                                 pack_bf16(up[8 * q + 6], up[8 * q + 7]));
                    st_shared_v4(uw_img + sw128_offset(v, chunk16), pack_bf16(uw[8 * q], uw[8 * q + 1]),
                                 pack_bf16(uw[8 * q + 2], uw[8 * q + 3]), pack_bf16(uw[8 * q + 4], uw[8 * q + 5]),
                                 pack_bf16(uw[8 * q + 6], uw[8 * q + 7]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (!ok) break;

        // (d) acc4 = U'_w K (state increment), acc3 = U' P^T (intra-chunk output)
        if (tid == 0) {
            const uint32_t id_k = idesc_bf16(128, 128, 0, 1), id_p = idesc_bf16(128, 64, 0, 0);
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(acc4, sdesc_sw128(uw_img + kk * 32, 16, 1024), sdesc_sw128(st_u + kStK + kk * 2048, 8192, 1024),
                         id_k, kk > 0);
            mma_commit(&bars.mma[2]);
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(acc3, sdesc_sw128(up_img + kk * 32, 16, 1024), sdesc_sw128(st_u + kStP + kk * 32, 16, 1024),
                         id_p, kk > 0);
            mma_commit(&bars.mma[3]);
        }

        // (e) S = gam_L S0 + acc4
        const float gl = __expf(bl);
        ok = mbar_wait(&bars.mma[2], par);
        tc_fence_after();
        if (ok) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                float a[16];
                tmem_ld16(acc4 + lane_off + c0, a);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) S[c0 + t] = gl * S[c0 + t] + a[t];
            }
        }

        // (f) O = scale gam_i (S0 q_i) + (P U')_i
        ok = ok && mbar_wait(&bars.mma[1], par) && mbar_wait(&bars.mma[3], par);
        tc_fence_after();
        if (ok) {
            __nv_bfloat16 *op = out + (tok0 * H + h) * D + v;
#pragma unroll
            for (int c0 = 0; c0 < C; c0 += 16) {
                float a2[16], a3[16];
                tmem_ld16(acc2 + lane_off + c0, a2);
                tmem_ld16(acc3 + lane_off + c0, a3);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int i = c0 + t;
                    if (i < L) op[(int64_t)i * H * D] = __float2bfloat16_rn(scale * __expf(bs[i]) * a2[t] + a3[t]);
                }
            }
        }

        // snapshot after n * stride tokens of the sequence
        if (ok && snaps && snap_stride > 0 && ((c + 1) * C) % snap_stride == 0 && (c + 1) * C <= len) {
            const int64_t s = (c + 1) * C / snap_stride - 1;
            if (s < n_snap) {
                float *dst = snaps + (((n * n_snap + s) * H + h) * D + v) * (int64_t)D;
#pragma unroll
                for (int cc = 0; cc < D; cc += 4)
                    *reinterpret_cast<float4 *>(dst + cc) = make_float4(S[cc], S[cc + 1], S[cc + 2], S[cc + 3]);
            }
        }

        // release this stage: every MMA that read it has completed; refill with chunk c+2
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok && c + 2 < nchunks) issue_loads(c + 2);
    }
    if (!ok && tid == 0) flag_error(err, 2);
    if (ok && final_state) {
#pragma unroll
        for (int cc = 0; cc < D; cc += 4)
            *reinterpret_cast<float4 *>(final_state + srow + cc) = make_float4(S[cc], S[cc + 1], S[cc + 2], S[cc + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
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

// (rows, H, 128) bf16 tensor, tiles of 64 tokens x 64 channels of one head, 128-byte swizzle.
gdn_status make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t H) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(GDN_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64}, es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GDN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return GDN_OK;
}

}  // namespace

bool tc_eligible(const gdn_desc &d) {
    return d.dtype == GDN_BF16 && d.dk == 128 && d.dv == 128 && d.gate == GDN_GATE_HEAD;
}

gdn_status launch_chunk_tc(const ChunkPlan &p, const ChunkArgs &a, cudaStream_t s) {
    gdn_status st = launch_chunk_table(p, a, s);
    if (st != GDN_OK) return st;
    const int32_t *off = a.cu_seqlens ? reinterpret_cast<const int32_t *>(a.ws + p.off_chunk_offsets) : nullptr;
    uint8_t *Wimg = reinterpret_cast<uint8_t *>(a.ws + p.off_W);
    uint8_t *Pimg = reinterpret_cast<uint8_t *>(a.ws + p.off_P);
    __nv_bfloat16 *Ut = reinterpret_cast<__nv_bfloat16 *>(a.ws + p.off_U);
    float *bcum = reinterpret_cast<float *>(a.ws + p.off_b);
    if (p.H > 65535 || p.max_chunks > 0x7fffffffLL || a.N > 0x7fffffffLL)
        return fail(GDN_ERR_UNSUPPORTED, "grid too large");
    CUtensorMap mq, mk, mv;
    const int64_t map_rows = p.rows > 0 ? p.rows : 1;
    if (p.rows > 0) {
        if ((st = make_map(&mq, a.q, map_rows, p.H)) != GDN_OK) return st;
        if ((st = make_map(&mk, a.k, map_rows, p.H)) != GDN_OK) return st;
        if ((st = make_map(&mv, a.v, map_rows, p.H)) != GDN_OK) return st;
    } else {
        memset(&mq, 0, sizeof mq);
        memset(&mk, 0, sizeof mk);
    }
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(gdn_prep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gdn_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScanSmem);
    });
    if (attr_err != cudaSuccess) return fail(GDN_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(attr_err));
    if (p.max_chunks > 0 && p.rows > 0) {
        LaunchScope ls("gdn_prep_tc", s);
        gdn_prep_tc<<<dim3((unsigned)p.max_chunks, (unsigned)p.H), kThreads, kPrepSmem, s>>>(
            mq, mk, mv, a.g, a.beta, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, a.scale, Wimg, Pimg, Ut, bcum, nullptr);
    }
    if ((st = check_launch("gdn_prep_tc")) != GDN_OK) return st;
    {
        LaunchScope ls("gdn_scan_tc", s);
        gdn_scan_tc<<<dim3((unsigned)a.N, (unsigned)p.H), kThreads, kScanSmem, s>>>(
            mq, mk, a.h0, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, p.max_chunks, a.scale, a.snapshot_stride, a.n_snap,
            Wimg, Pimg, Ut, bcum, (__nv_bfloat16 *)a.out, a.final_state, a.snapshots, nullptr);
    }
    return check_launch("gdn_scan_tc");
}

}  // namespace gdn
