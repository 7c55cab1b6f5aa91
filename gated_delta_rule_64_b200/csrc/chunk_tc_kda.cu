// Chunk preparation for the per-key-channel gate (the KDA variant) on the
// tensor cores: bf16 q/k/v, d_k = d_v = 128.
//
// With a gate per key channel the decay between tokens j <= i is a vector,
// exp(b_i - b_j) with b_i = sum_{t<=i} g_t over the chunk ("Hybrid Linear
// Attention Architecture Design Explained", section 4, fine-grained decay;
// "Hybrid attention", "Training a recurrence in parallel"), so the in-chunk
// matrices are
//
//   A_ij = beta_i sum_c k_ic k_jc exp(b_ic - b_jc)       (j < i)
//   P_ij = scale  sum_c q_ic k_jc exp(b_ic - b_jc)       (j <= i)
//   W    = T diag(beta) (K * Gam),   U = T diag(beta) V,   T = (I + A)^-1
//   (U itself is not formed here: the block holds -T diag(beta) and the scan
//   accumulates V^T (-T diag(beta))^T onto S0 W^T)
//   Qs   = scale Q * Gam,            K~ = K * exp(b_L - b)
//
// (Gam_i = exp(b_i)); the scan then carries S0 Diag(Gam_L) + U'^T K~.
// Writing the decay as one product (K * Gam)(K / Gam)^T overflows for strong
// gates, so A and P are formed in 16 x 16 blocks.  With r_p = b at the row
// before block p (r_0 = 0) and e_p = b at its last row, every row i of block p
// gets the two factors L_i = exp(b_i - r_p) <= 1 and R_i = exp(e_p - b_i) <= 1,
// and for i in block p, j in block q:
//   * q < p:  exp(b_i - b_j) = L_i * exp(r_p - e_q) * R_j, all three <= 1, so the
//             block is the tensor-core product of K * L (or Q * L) with K * R
//             scaled per channel by exp(r_p - e_q) (= 1 for q = p - 1);
//   * q = p:  exp(b_i - b_j) = L_i * exp(r_p - e_p) * R_j where the middle
//             factor is >= 1: fine as long as the block's decay is moderate
//             (2^64 at most); otherwise the block is formed term by term from
//             exp(b_i - b_j) on the CUDA cores.
// Most chunks decay moderately: with m = b at row 31 and every channel's
// b_0 - m and m - b_63 at most 2^kSpanFast, the factors E+_i = exp(b_i - m) and
// E-_j = exp(m - b_j) stay far inside the bf16 range, exp(b_i - b_j) = E+_i E-_j,
// and the whole of A and P is one tensor-core product [K * E+ ; Q * E+] (K * E-)^T
// (tcgen05, M = 128, N = 64, K = 128), as in the per-head kernel; the entries above
// the diagonal, which may overflow, are never used.  Other chunks take the blocks.
// The triangular solve and the W / U tensor-core products are those of the
// per-head kernel.
#include <string.h>

#include <mutex>

#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

// Shared memory (1024-aligned):
//   [0, 32K)    K and Q tiles: [K ch 0-63 | Q ch 0-63 | K ch 64-127 | Q ch 64-127],
//               64 token rows of 128 bytes each, 128-byte swizzle (TMA).  They become
//               K * L and Q * L, and then K * L becomes K * Gam (the A operand of W).
//   [32K, 64K)  gate tile (TMA: four [64 tokens][32 channels] fp32 quarters, 128-byte
//               swizzle), turned in place into b in log2 units; once the factors are
//               formed: A (fp32, f32_offset layout) at 32K
//   [64K, 80K)  K * R (layout of a K tile, channel halves 8K apart); after the blocks:
//               T (fp32)
//   [80K, 96K)  after the blocks: the solve's scratch (4K) and T diag(beta) (8K at 88K)
//   [96K, 104K) P rows (bf16, row = query token i, 64 key tokens j, 128-byte swizzle)
constexpr uint32_t kSmKQ = 0, kSmB = 32768, kSmA = 32768, kSmZ = 65536, kSmP = 98304;
constexpr uint32_t kSmT = 65536, kSmY = 81920, kSmTp = 90112;
constexpr uint32_t kSmem = kSmP + 8192 + 1024;
constexpr float kLog2e = 1.4426950408889634f;
// Largest decay inside a diagonal block (log2 units) for which the block is a
// product of scaled operands: its middle factor reaches 2^kSpanMax (far inside
// the bf16 / fp32 range).
constexpr float kSpanMax = 64.f;
// Largest decay on either side of row 31 (log2 units) for the one-product form.
constexpr float kSpanFast = 60.f;

// Element (token i, channel c) of the gate / b tile.
__device__ __forceinline__ uint32_t b_off(int i, int c) {
    return (uint32_t)((c >> 5) * 8192 + i * 128 + ((((c & 31) >> 2) ^ (i & 7)) << 4) + (c & 3) * 4);
}
// 8-channel chunk `cc` (0..15) of row i of the K (qk = 0) or Q (qk = 1) tile.
__device__ __forceinline__ uint32_t kq_chunk(int qk, int i, int cc) {
    return (uint32_t)((cc >> 3) * 16384 + qk * 8192 + i * 128 + (((cc & 7) ^ (i & 7)) << 4));
}
// 8-channel chunk `cc` of row i of the K * R image.
__device__ __forceinline__ uint32_t z_chunk(int i, int cc) {
    return (uint32_t)(kSmZ + (cc >> 3) * 8192 + i * 128 + (((cc & 7) ^ (i & 7)) << 4));
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t scale_pair(uint32_t w, float2 f) { return pack_bf16(bf_lo(w) * f.x, bf_hi(w) * f.y); }

__device__ __forceinline__ void unpack8(const uint4 &w, float *f) {
    f[0] = bf_lo(w.x); f[1] = bf_hi(w.x); f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
    f[4] = bf_lo(w.z); f[5] = bf_hi(w.z); f[6] = bf_lo(w.w); f[7] = bf_hi(w.w);
}
__device__ __forceinline__ void ld_f8(const uint8_t *sm, int i, int c8, float *f) {
    *reinterpret_cast<float4 *>(f) = *reinterpret_cast<const float4 *>(sm + kSmB + b_off(i, c8));
    *reinterpret_cast<float4 *>(f + 4) = *reinterpret_cast<const float4 *>(sm + kSmB + b_off(i, c8 + 4));
}

// Per-channel factors of one chunk (fp32): exp(r_p) per block, exp(r_p - e_p) per
// diagonal block, exp(r_p - e_q) for the blocks (2,0), (3,0), (3,1).
struct Factors {
    float rp[4][D];
    float sp[4][D];
    float d[3][D];
};

// One warp's share of A and P by bf16 m16n8k16 MMAs: row block p against
// column blocks q0 .. q0 + nq - 1 (q <= p).  Operands from the K * L, Q * L and
// K * R images; the right operand is scaled per channel by exp(r_p - e_q).
__device__ __forceinline__ void ap_blocks(uint8_t *sm, const Factors &f, int p, int q0, int nq, int L, float scale,
                                          const float *s_beta) {
    const int lane = threadIdx.x & 31, g8 = lane >> 2, t = lane & 3;
    const int i0 = 16 * p + g8, i1 = i0 + 8;
    const uint32_t sb = smem_u32(sm);
    // ldmatrix row of this lane: left operand (matrix m = lane / 8: rows +8 (m & 1), columns +8 (m >> 1));
    // right operand (rows +8 (m >> 1) = second n-tile, columns +8 (m & 1))
    const int m = lane >> 3, lr = lane & 7;
    const int arow = 16 * p + lr + 8 * (m & 1), acol = m >> 1;
    float cA[2][2][4], cP[2][2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) cA[b][nt][e] = cP[b][nt][e] = 0.f;
#pragma unroll 2
    for (int kk = 0; kk < 8; ++kk) {
        uint32_t ak[4], aq[4];
        ldsm_x4(sb + kq_chunk(0, arow, 2 * kk + acol), ak);
        ldsm_x4(sb + kq_chunk(1, arow, 2 * kk + acol), aq);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            if (b >= nq) continue;
            const int q = q0 + b;
            uint32_t bz[4];
            ldsm_x4(sb + z_chunk(16 * q + lr + 8 * (m >> 1), 2 * kk + (m & 1)), bz);
            const float *sc = q == p ? f.sp[p] : (q == p - 1 ? nullptr : f.d[p == 2 ? 0 : (q == 0 ? 1 : 2)]);
            if (sc) {
                const int c = 16 * kk + 2 * t;
                const float2 lo = *reinterpret_cast<const float2 *>(sc + c), hi = *reinterpret_cast<const float2 *>(sc + c + 8);
                bz[0] = scale_pair(bz[0], lo);
                bz[1] = scale_pair(bz[1], hi);
                bz[2] = scale_pair(bz[2], lo);
                bz[3] = scale_pair(bz[3], hi);
            }
            const uint32_t b0[2] = {bz[0], bz[1]}, b1[2] = {bz[2], bz[3]};
            mma_bf16_16x8x16(cA[b][0], ak, b0);
            mma_bf16_16x8x16(cP[b][0], aq, b0);
            mma_bf16_16x8x16(cA[b][1], ak, b1);
            mma_bf16_16x8x16(cP[b][1], aq, b1);
        }
    }
    const float be0 = s_beta[i0], be1 = s_beta[i1];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        if (b >= nq) continue;
        const bool diag = q0 + b == p;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * (q0 + b) + 8 * nt + 2 * t;
            // A: the solve reads only below the diagonal, so the whole block is stored
            *reinterpret_cast<float2 *>(sm + kSmA + f32_offset(i0, col)) =
                make_float2(be0 * cA[b][nt][0], be0 * cA[b][nt][1]);
            *reinterpret_cast<float2 *>(sm + kSmA + f32_offset(i1, col)) =
                make_float2(be1 * cA[b][nt][2], be1 * cA[b][nt][3]);
            // P: causal (j <= i) and rows of the chunk only
            const bool k00 = i0 < L && (!diag || col <= i0), k01 = i0 < L && (!diag || col + 1 <= i0);
            const bool k10 = i1 < L && (!diag || col <= i1), k11 = i1 < L && (!diag || col + 1 <= i1);
            // P rows: the pair of columns (col, col + 1) of rows i0 and i1, one 4-byte store each
            *reinterpret_cast<uint32_t *>(sm + kSmP + img_offset(i0, col)) =
                pack_bf16(k00 ? scale * cP[b][nt][0] : 0.f, k01 ? scale * cP[b][nt][1] : 0.f);
            *reinterpret_cast<uint32_t *>(sm + kSmP + img_offset(i1, col)) =
                pack_bf16(k10 ? scale * cP[b][nt][2] : 0.f, k11 ? scale * cP[b][nt][3] : 0.f);
        }
    }
}

// Diagonal blocks term by term, for chunks whose gates decay too fast for the
// factored form: warp pair (2p, 2p+1) takes block p; lane = (row pair, 16-channel
// group); rows r and 15 - r of a block together need 17 (i, j) steps.  It reads
// the raw K and Q tiles and b; the butterfly leaves every sum in all 8 lanes of a
// group, and lane s keeps the steps it = s (mod 8) for diag_exact_store.
struct DiagKeep {
    float a[3], p[3];
};
__device__ __forceinline__ void diag_exact(const uint8_t *sm, DiagKeep &keep) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = warp >> 1, rl = lane >> 3, s = lane & 7;
    const int r = 4 * (warp & 1) + rl, base = 16 * p;
    float ki[16], qi[16], bi[16];
    auto load_b = [&](int R, float *f) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4 *>(f + 4 * m) = *reinterpret_cast<const float4 *>(sm + kSmB + b_off(R, 16 * s + 4 * m));
    };
    auto load_row = [&](int R) {
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, R, 2 * s)), ki);
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, R, 2 * s + 1)), ki + 8);
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(1, R, 2 * s)), qi);
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(1, R, 2 * s + 1)), qi + 8);
        load_b(R, bi);
    };
    load_row(base + r);
#pragma unroll 1
    for (int it = 0; it < 17; ++it) {
        const bool first = it <= r;
        const int il = first ? r : 15 - r, jl = first ? r - it : 16 - it;
        if (it == r + 1) load_row(base + il);
        float kj[16], bj[16];
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, base + jl, 2 * s)), kj);
        unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, base + jl, 2 * s + 1)), kj + 8);
        load_b(base + jl, bj);
        float a0 = 0.f, a1 = 0.f, p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
            const float t0 = kj[c] * ex2(bi[c] - bj[c]), t1 = kj[c + 1] * ex2(bi[c + 1] - bj[c + 1]);
            a0 = fmaf(ki[c], t0, a0);
            a1 = fmaf(ki[c + 1], t1, a1);
            p0 = fmaf(qi[c], t0, p0);
            p1 = fmaf(qi[c + 1], t1, p1);
        }
        float a = a0 + a1, pp = p0 + p1;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, o);
            pp += __shfl_xor_sync(0xffffffffu, pp, o);
        }
        if ((it & 7) == s) {
            const int k = it >> 3;
            if (k == 0) { keep.a[0] = a; keep.p[0] = pp; }
            else if (k == 1) { keep.a[1] = a; keep.p[1] = pp; }
            else { keep.a[2] = a; keep.p[2] = pp; }
        }
    }
}
__device__ __forceinline__ void diag_exact_store(uint8_t *sm, const DiagKeep &keep, int L, float scale,
                                                 const float *s_beta) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = warp >> 1, rl = lane >> 3, s = lane & 7;
    const int r = 4 * (warp & 1) + rl, base = 16 * p;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int it = 8 * k + s;
        if (it >= 17) continue;
        const bool first = it <= r;
        const int i = base + (first ? r : 15 - r), j = base + (first ? r - it : 16 - it);
        *reinterpret_cast<float *>(sm + kSmA + f32_offset(i, j)) = s_beta[i] * keep.a[k];
        *reinterpret_cast<__nv_bfloat16 *>(sm + kSmP + img_offset(i, j)) = __float2bfloat16_rn(i < L ? scale * keep.p[k] : 0.f);
    }
}

__global__ void __launch_bounds__(kThreads, 2)
gdn_prep_kda_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mg,
                const float *__restrict__ beta, const int32_t *__restrict__ cu, const int32_t *__restrict__ off,
                int64_t N, int64_t T, int64_t rows, int64_t H, int64_t Hk, float scale, uint8_t *__restrict__ blocks,
                int want_bound, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    __shared__ uint64_t bar_g, bar_ld, bar_mma, bar_drain;
    __shared__ uint32_t tmem_base;
    __shared__ float s_beta[C], s_tot[D], s_lam[kThreads / 32];
    __shared__ __align__(16) Factors fct;

    const int64_t chunk = blockIdx.x, h = blockIdx.y;
    ChunkLoc loc;
    if (!locate_chunk(chunk, cu, off, N, T, rows, loc)) return;
    if (!in_bounds(loc.start >= 0 && loc.start + loc.len <= rows && h < H && H % Hk == 0, err)) return;
    const int L = (int)loc.len;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;
    const int32_t tok0 = (int32_t)loc.start;
    uint8_t *blk = blocks + (size_t)(chunk * H + h) * kTcBlock;
    uint8_t *rest = blk + kBlkRest;

    const float beta_in = tid < L ? beta[(int64_t)(tok0 + tid) * H + h] : 0.f;
    if (tid == 0) {
        mbar_init(&bar_g, 1);
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_drain, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar_g, 4 * 8192);
#pragma unroll
        for (int qt = 0; qt < 4; ++qt) tma_load_3d(sm + kSmB + qt * 8192, &mg, 32 * qt, (int32_t)h, tok0, &bar_g);
        mbar_arrive_expect_tx(&bar_ld, 4 * 8192);
        const int32_t hq = (int32_t)(h / (H / Hk));  // query/key head of value head h
        tma_load_3d(sm + kSmKQ, &mk, 0, hq, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 16384, &mk, 64, hq, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 8192, &mq, 0, hq, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 24576, &mq, 64, hq, tok0, &bar_ld);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 128);
        tmem_relinquish();
    }
    for (int e = tid; e < 512; e += kThreads) *reinterpret_cast<uint4 *>(sm + kSmP + e * 16) = make_uint4(0, 0, 0, 0);
    if (tid < C) s_beta[tid] = beta_in;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;

    // In-chunk inclusive cumsum of the log gate per key channel (rows >= L count
    // as g = 0), stored in log2 units; thread (c, half) scans 32 rows.  The
    // largest decay inside any 16-token block decides how the diagonal blocks
    // are formed.
    bool ok = mbar_wait(&bar_g, 0);
    bool fast = false;  // A and P as one product
    const int c_own = tid & 127, half = tid >> 7;
    bool gate_bad = false;  // a gate above 0 (outside the documented range): no decay bound
    {
        // decay bound of the chunk: the sum over its tokens of the largest gate over the
        // channels (thread: token tid / 4, channels 32 (tid % 4) ..); before the tile
        // becomes b in place
        // (the 16-byte chunks of a row are visited from a row-dependent start, so the
        // lanes of a warp, eight rows, read eight different bank groups)
        float gmax = -INFINITY;
        if (want_bound && ok && (tid >> 2) < L) {
            const uint8_t *row = sm + kSmB + (tid & 3) * 8192 + (tid >> 2) * 128;
            const int rot = (tid >> 2) & 7;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const float4 f = *reinterpret_cast<const float4 *>(row + ((ch ^ rot) << 4));
                gmax = fmaxf(gmax, fmaxf(fmaxf(f.x, f.y), fmaxf(f.z, f.w)));
            }
        }
        gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 1));
        gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 2));
        gate_bad = (tid >> 2) < L && !(gmax <= 0.f);
        float lsum = ((tid & 3) == 0 && (tid >> 2) < L) ? gmax : 0.f;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
        if (lane == 0) s_lam[warp] = lsum;
    }
    {
        float vals[32];
        if (ok) {
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const int i = 32 * half + r;
                vals[r] = i < L ? *reinterpret_cast<const float *>(sm + kSmB + b_off(i, c_own)) : 0.f;
            }
#pragma unroll
            for (int r = 1; r < 32; ++r) vals[r] += vals[r - 1];
            if (half == 0) s_tot[c_own] = vals[31];
        }
        __syncthreads();
        bool wide = false, narrow = true;
        if (ok) {
            const float base = half ? s_tot[c_own] : 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                vals[r] = (vals[r] + base) * kLog2e;
                *reinterpret_cast<float *>(sm + kSmB + b_off(32 * half + r, c_own)) = vals[r];
            }
            // block p = 2 half (+1): r_p = b before it, e_p = b at its last row
            const float r0 = base * kLog2e, e0 = vals[15], e1 = vals[31];
            fct.rp[2 * half][c_own] = ex2(r0);
            fct.rp[2 * half + 1][c_own] = ex2(e0);
            fct.sp[2 * half][c_own] = ex2(r0 - e0);
            fct.sp[2 * half + 1][c_own] = ex2(e0 - e1);
            wide = (r0 - e0 > kSpanMax) || (e0 - e1 > kSpanMax);
            // half 1: r0 = b at row 31 (= m), e1 = b at row 63
            if (half) narrow = -r0 <= kSpanFast && r0 - e1 <= kSpanFast;
        }
        const bool any_wide = __syncthreads_or(wide);  // uniform over the block
        fast = !__syncthreads_or(!narrow);
        // one product: K * Gam = (K * E+) exp(m), for the pass after A and P
        if (ok && fast && tid < D) {
            const float em = ex2(*reinterpret_cast<const float *>(sm + kSmB + b_off(31, tid)));
#pragma unroll
            for (int q = 0; q < 4; ++q) fct.rp[q][tid] = em;
        }
        // exp(r_p - e_q) for (p, q) = (2, 0), (3, 0), (3, 1)
        if (ok && tid < D) {
            const float e0 = *reinterpret_cast<const float *>(sm + kSmB + b_off(15, tid));
            const float e1 = *reinterpret_cast<const float *>(sm + kSmB + b_off(31, tid));
            const float r3 = *reinterpret_cast<const float *>(sm + kSmB + b_off(47, tid));
            fct.d[0][tid] = ex2(e1 - e0);
            fct.d[1][tid] = ex2(r3 - e0);
            fct.d[2][tid] = ex2(r3 - e1);
        }
        ok = mbar_wait(&bar_ld, 0) && ok;
        bool bad = gate_bad;  // a token outside the decay bound's range (|k_i|^2 below)
        // exact diagonal blocks need the raw tiles and b: before the factor pass
        DiagKeep keep = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
        if (any_wide) {
            if (ok) diag_exact(sm, keep);
            __syncthreads();
        }

        // Factor pass over (token, 8-channel) chunks: K * L and Q * L in place,
        // K * R to its image; Qs = scale Q * Gam and K~ = K * exp(b_L - b) to the block.
        // The same pass sums |k_i|^2 for the decay bound: thread (row tid / 8, 16-byte
        // chunk tid % 8) sees rows tid / 8 and 32 + tid / 8 in both channel halves.
        if (ok) {
            const int Lm1 = L - 1;
            float k2a = 0.f, k2b = 0.f;  // rows tid / 8 and 32 + tid / 8
#pragma unroll 1
            for (int k = 0; k < 4; ++k) {
                const int e = tid + kThreads * k;
                const int hc = e >> 9, i = (e & 511) >> 3, pc = e & 7, p = i >> 4;
                const int c8 = hc * 64 + ((pc ^ (i & 7)) << 3);
                const uint32_t so = (uint32_t)(hc * 16384 + i * 128 + pc * 16);
                float kf[8], qf[8], bi[8], rr[8], ee[8], bl[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + so), kf);
                unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + so + 8192), qf);
                ld_f8(sm, i, c8, bi);
                ld_f8(sm, Lm1, c8, bl);
                float er[8];  // exp(r_p): Gam_i = L_i exp(r_p), both factors <= 1
                if (fast) {
                    // one product: L -> E+ = exp(b - m), R -> E- = exp(m - b), Gam = E+ exp(m)
                    ld_f8(sm, 31, c8, ee);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        rr[u] = ee[u];
                        er[u] = ex2(ee[u]);
                    }
                } else {
                    ld_f8(sm, 16 * p + 15, c8, ee);
                    if (p > 0) ld_f8(sm, 16 * p - 1, c8, rr);
                    else
#pragma unroll
                        for (int u = 0; u < 8; ++u) rr[u] = 0.f;
                    *reinterpret_cast<float4 *>(er) = *reinterpret_cast<const float4 *>(fct.rp[p] + c8);
                    *reinterpret_cast<float4 *>(er + 4) = *reinterpret_cast<const float4 *>(fct.rp[p] + c8 + 4);
                }
                if (want_bound) {
                    float ss = 0.f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) ss = fmaf(kf[u], kf[u], ss);
                    if (k & 1) k2b += ss; else k2a += ss;
                }
                uint32_t xk[4], xq[4], zr[4], kt[4], qs[4];
                const bool in = i < L;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int a = 2 * u, b = 2 * u + 1;
                    const float la = ex2(bi[a] - rr[a]), lb = ex2(bi[b] - rr[b]);
                    const float ra = ex2(ee[a] - bi[a]), rb = ex2(ee[b] - bi[b]);
                    const float ga = la * er[a], gb = lb * er[b];
                    const float ta = ex2(bl[a] - bi[a]), tb = ex2(bl[b] - bi[b]);
                    xk[u] = pack_bf16(kf[a] * la, kf[b] * lb);
                    xq[u] = pack_bf16(qf[a] * la, qf[b] * lb);
                    zr[u] = pack_bf16(kf[a] * ra, kf[b] * rb);
                    kt[u] = in ? pack_bf16(kf[a] * ta, kf[b] * tb) : 0u;
                    qs[u] = in ? pack_bf16(scale * qf[a] * ga, scale * qf[b] * gb) : 0u;
                }
                *reinterpret_cast<uint4 *>(rest + kRestKt + hc * 8192 + i * 128 + pc * 16) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
                *reinterpret_cast<uint4 *>(blk + kBlkQs + hc * 8192 + i * 128 + pc * 16) =
                    make_uint4(qs[0], qs[1], qs[2], qs[3]);
                // (no other thread reads this chunk of the tiles)
                *reinterpret_cast<uint4 *>(sm + kSmKQ + so) = make_uint4(xk[0], xk[1], xk[2], xk[3]);
                *reinterpret_cast<uint4 *>(sm + kSmKQ + so + 8192) = make_uint4(xq[0], xq[1], xq[2], xq[3]);
                *reinterpret_cast<uint4 *>(sm + kSmZ + hc * 8192 + i * 128 + pc * 16) = make_uint4(zr[0], zr[1], zr[2], zr[3]);
            }
            if (want_bound) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float x = r ? k2b : k2a;
                    x += __shfl_xor_sync(0xffffffffu, x, 1);
                    x += __shfl_xor_sync(0xffffffffu, x, 2);
                    x += __shfl_xor_sync(0xffffffffu, x, 4);
                    const int i = 32 * r + (tid >> 3);
                    bad = bad || (i < L && !(s_beta[i] >= 0.f && s_beta[i] * x <= kBetaK2Max));
                }
            }
            float *fac = reinterpret_cast<float *>(rest + kRestFac);
            if (tid < D) fac[kFacGL + tid] = ex2(*reinterpret_cast<const float *>(sm + kSmB + b_off(Lm1, tid)));
        }
        const bool any_bad = __syncthreads_or(bad);
        if (tid == 0) {
            float lam = 0.f;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) lam += s_lam[w];
            reinterpret_cast<float *>(rest + kRestFac)[kFacLam] = (!want_bound || any_bad) ? kLamNone : lam * kLog2e;
        }

        // A and P.  Warp w takes row block p against column blocks [q0, q0 + nq);
        // (p, q0, nq) per warp, one hex digit each, with the diagonal blocks (10
        // blocks) or without them (6), spread so that warps w and w + 4 (which
        // share a scheduler) hold at most 3 blocks between them.
        if (fast) {
            // [K * E+ ; Q * E+] (K * E-)^T: rows 0..63 give beta_i A_ij, rows 64..127 P_ij
            if (warp == 0 && __all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                const uint64_t da = sdesc_sw128(smem_u32(sm + kSmKQ), 16, 1024), dz = sdesc_sw128(smem_u32(sm + kSmZ), 16, 1024);
                const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tm, da + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                dz + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id, kk > 0);
                mma_commit_warp(&bar_mma);
            }
            ok = ok && mbar_wait(&bar_mma, 0);
            tc_fence_after();
            if (ok) {
                // accumulator row r = qd*32 + lane, columns [32 hf, 32 hf + 32); only the
                // entries below (A) or on and below (P) the diagonal are kept
                const int r = qd * 32 + lane;
                const bool is_a = r < C;
                const int i = is_a ? r : r - C;
                float v0[16], v1[16];
                const uint32_t taddr = tm + ((uint32_t)(qd * 32) << 16) + 32 * hf;
                tmem_ld16(taddr, v0);
                tmem_ld16(taddr + 16, v1);
                tmem_wait_ld();
                const float pre = is_a ? s_beta[i] : scale;
                float rr[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int j = 32 * hf + t;
                    const bool keep = i < L && (is_a ? j < i : j <= i);
                    rr[t] = keep ? pre * (t < 16 ? v0[t] : v1[t - 16]) : 0.f;
                }
                if (is_a) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(sm + kSmA + f32_offset(i, 32 * hf + 4 * q)) =
                            make_float4(rr[4 * q], rr[4 * q + 1], rr[4 * q + 2], rr[4 * q + 3]);
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_shared_v4(smem_u32(sm + kSmP) + sw128_offset(i, 4 * hf + q), pack_bf16(rr[8 * q], rr[8 * q + 1]),
                                     pack_bf16(rr[8 * q + 2], rr[8 * q + 3]), pack_bf16(rr[8 * q + 4], rr[8 * q + 5]),
                                     pack_bf16(rr[8 * q + 6], rr[8 * q + 7]));
                }
            }
            tc_fence_before();  // the W / U products later reuse these TMEM columns
        } else if (ok) {
            if (any_wide) diag_exact_store(sm, keep, L, scale, s_beta);
            const uint32_t P = any_wide ? 0x00100233u : 0x01102233u, Q0 = any_wide ? 0x00000020u : 0x01002020u,
                           NQ = any_wide ? 0x00100212u : 0x01111222u;
            const int p = (P >> (4 * warp)) & 15, q0 = (Q0 >> (4 * warp)) & 15, nq = (NQ >> (4 * warp)) & 15;
            if (nq > 0) ap_blocks(sm, fct, p, q0, nq, L, scale, s_beta);
        }
    }
    __syncthreads();

    // P rows to the block; K * L -> K * Gam = K * L * exp(r_p) in place.
    if (ok) {
        for (int e = tid; e < 512; e += kThreads)
            *reinterpret_cast<uint4 *>(rest + kRestP + e * 16) = *reinterpret_cast<const uint4 *>(sm + kSmP + e * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int e = tid + kThreads * k;
            const int hc = e >> 9, i = (e & 511) >> 3, pc = e & 7;
            const int c8 = hc * 64 + ((pc ^ (i & 7)) << 3);
            const uint32_t so = (uint32_t)(hc * 16384 + i * 128 + pc * 16);
            const uint4 w = *reinterpret_cast<const uint4 *>(sm + kSmKQ + so);
            const float *rp = fct.rp[i >> 4] + c8;
            const float4 f0 = *reinterpret_cast<const float4 *>(rp), f1 = *reinterpret_cast<const float4 *>(rp + 4);
            *reinterpret_cast<uint4 *>(sm + kSmKQ + so) =
                make_uint4(scale_pair(w.x, make_float2(f0.x, f0.y)), scale_pair(w.y, make_float2(f0.z, f0.w)),
                           scale_pair(w.z, make_float2(f1.x, f1.y)), scale_pair(w.w, make_float2(f1.z, f1.w)));
        }
    }
    fence_async_smem();  // K * Gam is read by the tensor core
    __syncthreads();

    // T = (I + A)^-1 into the (now free) K * R region.
    blocked_solve<kSmT, kSmY>(sm, [](int i, int j) { return kSmA + f32_offset(i, j); },
                              [](int i) { return kSmA + (uint32_t)i * 256u; }, ok);

    // T'' = T diag(beta) as a bf16 operand image (K-major rows i), and -T'' as rows of
    // the block (the scan's operand); the blocks of T above its block diagonal are zero
    // (the solve leaves them unwritten).
    if (ok) {
        const int i = tid >> 2, j0 = (tid & 3) * 16;
        const bool upper = (tid & 3) > (i >> 4);
        float tv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!upper) f = *reinterpret_cast<const float4 *>(sm + kSmT + f32_offset(i, j0 + 4 * q));
            tv[4 * q] = f.x; tv[4 * q + 1] = f.y; tv[4 * q + 2] = f.z; tv[4 * q + 3] = f.w;
        }
        const uint32_t tp = smem_u32(sm + kSmTp);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) b[e] = tv[8 * q + e] * s_beta[j0 + 8 * q + e];
            const uint32_t o = sw128_offset(i, (j0 >> 3) + q);
            st_shared_v4(tp + o, pack_bf16(b[0], b[1]), pack_bf16(b[2], b[3]), pack_bf16(b[4], b[5]), pack_bf16(b[6], b[7]));
            *reinterpret_cast<uint4 *>(rest + kRestTn + o) = make_uint4(pack_bf16(-b[0], -b[1]), pack_bf16(-b[2], -b[3]),
                                                                        pack_bf16(-b[4], -b[5]), pack_bf16(-b[6], -b[7]));
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // W^T = (K * Gam)^T T''^T (M = d_k, K = 64 tokens)
    if (warp == 0 && __all_sync(0xffffffffu, ok)) {
        const uint64_t dk = sdesc_sw128(smem_u32(sm + kSmKQ), 16384, 1024), dt = sdesc_sw128(smem_u32(sm + kSmTp), 16, 1024);
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tm, dk + ((kk * 2048) >> 4), dt + ((kk * 32) >> 4), id, kk > 0);
        mma_commit_warp(&bar_mma);
    }
    ok = ok && mbar_wait(&bar_mma, fast ? 1 : 0);
    tc_fence_after();
    if (ok) store_w(tm, blk, qd, hf, lane);
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
        // A wait gave up: record it, then wait (bounded) for the tile copies and for
        // every MMA issued before the TMEM columns are freed.
        if (tid == 0) {
            flag_error(err, GDN_DEV_TIMEOUT_PREP);
            mbar_wait(&bar_g, 0);
            mbar_wait(&bar_ld, 0);
        }
        if (warp == 0) {
            mma_commit_warp(&bar_drain);
            mbar_wait(&bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == 0) tmem_dealloc(tm, 128);
}

}  // namespace

gdn_status launch_prep_kda(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mg,
                           const ChunkPlan &p, const ChunkArgs &a, const int32_t *off, uint8_t *blocks,
                           cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = cudaFuncSetAttribute(gdn_prep_kda_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    });
    if (attr != cudaSuccess) return fail(GDN_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(attr));
    log_launch("gdn_prep_kda_tc", dim3((unsigned)p.max_chunks, (unsigned)p.H), dim3(kThreads), kSmem);
    LaunchScope ls("gdn_prep_kda_tc", s);
    gdn_prep_kda_tc<<<dim3((unsigned)p.max_chunks, (unsigned)p.H), kThreads, kSmem, s>>>(
        mq, mk, mg, a.beta, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, a.Hk, a.scale, blocks, p.split_G >= 2 ? 1 : 0,
        a.status);
    return check_launch("gdn_prep_kda_tc");
}

}  // namespace tc
}  // namespace gdn
