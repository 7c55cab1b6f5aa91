// Pieces shared by the tensor-core prefill kernels (one gate per head, and the
// per-channel gate): workspace block layout, the blocked solve of the
// unit-lower-triangular chunk system and the W/U epilogue.
#pragma once

#include <cudaTypedefs.h>

#include <type_traits>

#include "chunk_common.cuh"
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int C = kChunk;  // 64 tokens per chunk
constexpr int D = 128;     // d_k = d_v
constexpr int kThreads = 256;

// Offsets inside one workspace block: W^T rows at 0, the Qs halves (per-channel
// gate) at kBlkQs and kBlkQs + 8K, then the rest at kBlkRest: K~, P rows, -T'' rows,
// gate factors.
constexpr uint32_t kBlkW = 0, kBlkQs = 16384, kBlkRest = (uint32_t)kTcWQ;
constexpr uint32_t kRestKt = 0, kRestP = 16384, kRestTn = 24576, kRestFac = 32768;
static_assert(kBlkQs + 16384 == kTcWQ && kRestP == kTcKt && kRestTn == kRestP + kTcPImg &&
                  kRestFac == kRestTn + kTcTn && kRestFac + kTcFac == kTcRest,
              "block layout");
// Gate factors (floats): exp(b_L), at [0] for the per-head gate and per key
// channel at [0, 128) for the per-channel gate; at [kFacLam] a bound on how much
// the chunk can shrink a state, in log2 units (below).
constexpr int kFacGL = 0, kFacLam = 128;
// One gate per head: scale exp(b_i) per token at [kFacQs, kFacQs + 64) (the scan
// scales its S0 Q^T output columns by them) and w_j = exp(b_L - b_j) per token at
// [kFacW, kFacW + 64) (zero past the chunk's end): the state increment
// U'^T (K * w) is taken as (diag(w) U')^T K, so the block holds no K~ for this gate.
constexpr int kFacW = 64, kFacQs = 192;

// Decay bound of a chunk.  One token maps a state S to S D_t (I - beta_t k_t k_t^T)
// (+ a write that does not depend on S).  When 0 <= beta_t |k_t|^2 <= 2 the
// factor (I - beta_t k_t k_t^T) has spectral norm <= 1, so the chunk shrinks the
// part of the state that came from before it by at least prod_t max_c alpha_{t,c}:
// lam = sum_t max_c g_{t,c} log2(e) (for one gate per head, b_L log2(e)).  A chunk
// with a token outside that range gets kLamNone (no bound).  Summed over chunks,
// lam bounds the weight of a start state in everything computed after them; below
// kLamDrop (2^-126, the end of the fp32 normal range, where an fp32 product of
// the transitions flushes to zero as well) the start state no longer matters.
// Only the split scan reads it: the prep kernels form it only when the scan splits
// (`want_bound`; packed batches never split).
constexpr float kLamNone = 1e30f;
constexpr float kLamDrop = -126.f;
constexpr float kBetaK2Max = 1.999f;  // beta |k|^2 bound, with room for rounding of |k|^2

__device__ __forceinline__ void flag_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint8_t *align1024(unsigned char *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// fp32 64 x 64 matrix, rows of 256 bytes, 16-byte chunks rotated per row (conflict-free row/column access).
__device__ __forceinline__ uint32_t f32_offset(int i, int j) {
    return (uint32_t)i * 256u + (uint32_t)((((j >> 2) ^ (i & 15)) << 4) + (j & 3) * 4);
}

// C (16x16) = sum over `nk` 16-wide K blocks of X_k (16x16) * Y_k (16x16); X and Y
// are fp32 blocks in shared memory given by their (row, col) origins and an
// offset function.  Warp-level m16n8k8 tf32 MMAs, fp32 accumulate; the fp32
// bit patterns are passed as they are (the tensor core reads them as tf32,
// dropping the low mantissa bits).  The result is returned in the MMA
// accumulator layout: c[nt][0..3] for the 8-column tiles nt = 0, 1.
template <typename OffX, typename OffY>
__device__ __forceinline__ void warp_gemm16(const uint8_t *base, int nk, const int *xr, const int *xc, const int *yr,
                                            const int *yc, OffX offx, OffY offy, float (&c)[2][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
    for (int kb = 0; kb < nk; ++kb) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int k0 = ks * 8;
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t *>(base + offx(xr[kb] + g, xc[kb] + k0 + t));
            a[1] = *reinterpret_cast<const uint32_t *>(base + offx(xr[kb] + g + 8, xc[kb] + k0 + t));
            a[2] = *reinterpret_cast<const uint32_t *>(base + offx(xr[kb] + g, xc[kb] + k0 + t + 4));
            a[3] = *reinterpret_cast<const uint32_t *>(base + offx(xr[kb] + g + 8, xc[kb] + k0 + t + 4));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t b[2];
                b[0] = *reinterpret_cast<const uint32_t *>(base + offy(yr[kb] + k0 + t, yc[kb] + nt * 8 + g));
                b[1] = *reinterpret_cast<const uint32_t *>(base + offy(yr[kb] + k0 + t + 4, yc[kb] + nt * 8 + g));
                mma_tf32_16x8x8(c[nt], a, b);
            }
        }
    }
}

// Store a 16x16 accumulator (times `sign`) at (r0, c0) through the offset function.
template <typename Off>
__device__ __forceinline__ void warp_store16(uint8_t *base, int r0, int c0, const float (&c)[2][4], float sign, Off off) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int col = c0 + nt * 8 + 2 * t;
        *reinterpret_cast<float *>(base + off(r0 + g, col)) = sign * c[nt][0];
        *reinterpret_cast<float *>(base + off(r0 + g, col + 1)) = sign * c[nt][1];
        *reinterpret_cast<float *>(base + off(r0 + g + 8, col)) = sign * c[nt][2];
        *reinterpret_cast<float *>(base + off(r0 + g + 8, col + 1)) = sign * c[nt][3];
    }
}

// 4 x 4 transpose of bf16 values among the 4 lanes of a quad: lane j holds row j as
// two packed pairs, p01 = (x_j0, x_j1) and p23 = (x_j2, x_j3) (low half first);
// afterwards p01 = (x_0j, x_1j), p23 = (x_2j, x_3j).  Two exchanges: 32-bit words
// across lanes j ^ 2, then 16-bit halves across lanes j ^ 1 (byte permutes).
__device__ __forceinline__ void quad_transpose_bf16(uint32_t &p01, uint32_t &p23, int lane) {
    const bool b1 = lane & 2, b0 = lane & 1;
    // lanes 0, 1 keep their columns 0-1 and take those of row j + 2; lanes 2, 3 the reverse
    const uint32_t r = __shfl_xor_sync(0xffffffffu, b1 ? p01 : p23, 2);
    const uint32_t A = b1 ? r : p01, B = b1 ? p23 : r;  // rows {j&1, (j&1) + 2}, columns 2 b1 + {0, 1}
    // even lanes keep column 2 b1 and send the other; odd lanes the reverse
    const uint32_t R = __shfl_xor_sync(0xffffffffu, __byte_perm(A, B, b0 ? 0x5410u : 0x7632u), 1);
    p01 = __byte_perm(A, R, b0 ? 0x3254u : 0x5410u);
    p23 = __byte_perm(B, R, b0 ? 0x3276u : 0x7610u);
}

// Eight bf16 values (one 16-byte chunk) times f, rounded back to bf16.
__device__ __forceinline__ uint4 scale8(const uint4 &src, float f) {
    const uint32_t in[4] = {src.x, src.y, src.z, src.w};
    uint32_t o[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&in[w]);
        o[w] = pack_bf16(f * __low2float(b2), f * __high2float(b2));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Sum of the squares of eight bf16 values (one 16-byte chunk), in fp32.
__device__ __forceinline__ float sum_sq8(const uint4 &src) {
    const uint32_t in[4] = {src.x, src.y, src.z, src.w};
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&in[w]);
        s = fmaf(__low2float(b2), __low2float(b2), s);
        s = fmaf(__high2float(b2), __high2float(b2), s);
    }
    return s;
}

// Byte offset of the bf16 element (row, col) of a 64-column operand image with
// 128-byte rows and the 128-byte swizzle.
__device__ __forceinline__ uint32_t img_offset(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2);
}

// T = (I + A)^-1 for the 64 x 64 strictly lower A of a chunk, in 16 x 16 blocks.
// A is read through `offA` (only its strictly lower part: the diagonal blocks
// below their diagonal and the blocks below the block diagonal); T is written
// in fp32 at byte offset TF of `sm` (f32_offset layout), its blocks on and below
// the block diagonal only: the blocks above it are zero and never written (the
// readers of T skip them).  TY is 4 KB of scratch.  Diagonal blocks: forward
// substitution in fp32 (one column per lane, two blocks per warp); off-diagonal
// blocks by the block recurrence T_pq = -T_pp sum_{q <= r < p} A_pr T_rq with
// tf32 warp MMAs (the first level by the warps that formed its diagonal
// blocks).  Every thread of the block calls it (it synchronises internally).
// rowA(i) is the byte offset of row i of A, whose element (i, j) sits at
// rowA(i) + f32_offset(0, j) with row i's swizzle (the f32_offset layout per row).
template <uint32_t TF, uint32_t TY, typename OffA, typename RowA>
__device__ __forceinline__ void blocked_solve(uint8_t *sm, OffA offA, RowA rowA, bool ok) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto offT = [](int i, int j) { return TF + f32_offset(i, j); };
    auto offY = [](int i, int j) { return TY + (uint32_t)i * 64u + (uint32_t)j * 4u; };  // 4 blocks, rows of 16
    if (warp < 2) {
        // diagonal blocks 2 warp and 2 warp + 1 (lanes 0-15 and 16-31): column `col` of
        // (I + A_pp)^-1 by forward substitution (fp32) ...
        const int p = 2 * warp + (lane >> 4), col = lane & 15;
        // Element (16p + i, 16p + j) of the f32_offset layout, i, j < 16: row 16p + i,
        // then the 16-byte chunk ((4p + j / 4) ^ i) = (4p ^ (i & 12)) + ((j / 4) ^ (i & 3))
        // (disjoint bits): one run-time term per row, the rest a constant.
        uint32_t xv[4], cv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            xv[k] = ((uint32_t)(4 * p) ^ (uint32_t)(4 * k)) << 4;
            cv[k] = ((uint32_t)(col >> 2) ^ (uint32_t)k) << 4;
        }
        if (ok) {
            // x_i = [i == col] - sum_{j < i} A_ij x_j.  The sums are built up four
            // columns j at a time, in increasing j as a row-by-row sum would add them:
            // once x of a 4-column panel is known, every row below takes the panel's
            // terms, so the chain from one x to the next is one multiply-add.
            const uint8_t *a0 = sm + rowA(16 * p);
            uint8_t *t0 = sm + TF + (uint32_t)(16 * p) * 256u + (uint32_t)(col & 3) * 4u;
            auto panel = [&](int i, int J) {  // A_{i, 4J .. 4J + 3}: one 16-byte chunk of row i
                return *reinterpret_cast<const float4 *>(a0 + i * 256 + xv[i >> 2] + ((J ^ (i & 3)) << 4));
            };
            float acc[16], x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int i = 4 * J + r;
                    if (r > 0) {
                        const float4 a = panel(i, J);
                        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int k = 0; k < r; ++k) acc[i] += av[k] * x[4 * J + k];
                    }
                    x[i] = (i == col) ? 1.f : -acc[i];
                    *reinterpret_cast<float *>(t0 + i * 256 + xv[i >> 2] + cv[i & 3]) = x[i];
                }
#pragma unroll
                for (int i = 4 * J + 4; i < 16; ++i) {
                    const float4 a = panel(i, J);
                    acc[i] += a.x * x[4 * J];
                    acc[i] += a.y * x[4 * J + 1];
                    acc[i] += a.z * x[4 * J + 2];
                    acc[i] += a.w * x[4 * J + 3];
                }
            }
        }
        __syncwarp();
        // ... then level 1: T_pq = -D_p (A_pq D_q) for (p, q) = (2 warp + 1, 2 warp)
        if (ok) {
            const int pp = 2 * warp + 1, q = 2 * warp;
            float c[2][4];
            const int xr[1] = {16 * pp}, xc[1] = {16 * q}, yr[1] = {16 * q}, yc[1] = {16 * q};
            warp_gemm16(sm, 1, xr, xc, yr, yc, offA, offT, c);
            warp_store16(sm, 16 * warp, 0, c, 1.f, offY);
            __syncwarp();
            const int xr2[1] = {16 * pp}, xc2[1] = {16 * pp}, yr2[1] = {16 * warp}, yc2[1] = {0};
            warp_gemm16(sm, 1, xr2, xc2, yr2, yc2, offT, offY, c);
            warp_store16(sm, 16 * pp, 16 * q, c, -1.f, offT);
        }
    }
    __syncthreads();
    // level 2, step 1: Y_pq = sum_{r in {0,1}} A_pr T_rq for p in {2,3}, q in {0,1}
    if (ok && warp < 4) {
        const int p = 2 + (warp >> 1), q = warp & 1;
        float c[2][4];
        if (q == 0) {
            const int xr[2] = {16 * p, 16 * p}, xc[2] = {0, 16}, yr[2] = {0, 16}, yc[2] = {0, 0};
            warp_gemm16(sm, 2, xr, xc, yr, yc, offA, offT, c);
        } else {
            const int xr[1] = {16 * p}, xc[1] = {16}, yr[1] = {16}, yc[1] = {16};
            warp_gemm16(sm, 1, xr, xc, yr, yc, offA, offT, c);
        }
        warp_store16(sm, 16 * warp, 0, c, 1.f, offY);
    }
    __syncthreads();
    // level 2, step 2: T_pq = -sum_{r in {2,3}, r <= p} T_pr Y_rq
    if (ok && warp < 4) {
        const int p = 2 + (warp >> 1), q = warp & 1;
        float c[2][4];
        // Y_rq lives in scratch block (r - 2) * 2 + q
        if (p == 2) {
            const int xr[1] = {32}, xc[1] = {32}, yr[1] = {16 * (0 * 2 + q)}, yc[1] = {0};
            warp_gemm16(sm, 1, xr, xc, yr, yc, offT, offY, c);
        } else {
            const int xr[2] = {48, 48}, xc[2] = {32, 48}, yr[2] = {16 * (0 * 2 + q), 16 * (1 * 2 + q)}, yc[2] = {0, 0};
            warp_gemm16(sm, 2, xr, xc, yr, yc, offT, offY, c);
        }
        warp_store16(sm, 16 * p, 16 * q, c, -1.f, offT);
    }
    __syncthreads();
}

// Epilogue of the W MMA: TMEM columns [0, 64) hold W^T (lane = channel, column =
// token).  Thread row r = qd*32 + lane writes tokens [32 hf, 32 hf + 32) of its
// channel row of W^T (128-byte swizzled rows).
// (Kept out of line: inlined, it pushes the per-head prep kernel past its register budget.)
static __device__ __noinline__ void store_rows(uint32_t taddr, uint8_t *dst, int r, int hf) {
    float u0[16], u1[16];
    tmem_ld16(taddr, u0);
    tmem_ld16(taddr + 16, u1);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float *u = q < 2 ? u0 + 8 * q : u1 + 8 * (q - 2);
        *reinterpret_cast<uint4 *>(dst + sw128_offset(r, 4 * hf + q)) =
            make_uint4(pack_bf16(u[0], u[1]), pack_bf16(u[2], u[3]), pack_bf16(u[4], u[5]), pack_bf16(u[6], u[7]));
    }
}
__device__ __forceinline__ void store_w(uint32_t tm, uint8_t *blk, int qd, int hf, int lane) {
    store_rows(tm + ((uint32_t)(qd * 32) << 16) + 32 * hf, blk + kBlkW, qd * 32 + lane, hf);
}

// Prep kernel of the per-channel gate (its own translation unit).
// (mg: the per-channel log gate as a (rows, H, 128) fp32 tensor, 32 x 1 x 64 boxes, 128-byte swizzle.)
gdn_status launch_prep_kda(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mg,
                           const ChunkPlan &p, const ChunkArgs &a, const int32_t *off, uint8_t *blocks,
                           cudaStream_t s);

}  // namespace tc
}  // namespace gdn
