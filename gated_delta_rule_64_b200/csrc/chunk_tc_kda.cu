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
//   Qs   = scale Q * Gam,            K~ = K * exp(b_L - b)
//
// (Gam_i = exp(b_i)); the scan then carries S0 Diag(Gam_L) + U'^T K~.
// Writing the decay as a product of per-token factors (K * Gam)(K / Gam)^T
// overflows for strong gates, so A and P are formed in 16 x 16 blocks:
//   * a block (p, q) below the diagonal (rows 16p.., columns 16q.., q < p) is
//     a tensor-core product of K_p * exp(b - r) and K_q * exp(r - b) with the
//     reference r = b at row 16p - 1; both factors are <= 1 because the
//     cumulative log gate does not increase;
//   * a diagonal block is formed on the CUDA cores from running products of
//     alpha = exp(g): walking j down from i, exp(b_i - b_j) gains one factor
//     alpha_{j+1} per step, so no exponential of a large argument appears.
// The triangular solve and the W / U tensor-core products are those of the
// per-head kernel.
#include <string.h>

#include <mutex>

#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

// Shared memory (1024-aligned):
//   [0, 32K)     K and Q tiles: [K ch 0-63 | Q ch 0-63 | K ch 64-127 | Q ch 64-127],
//                64 token rows of 128 bytes each, 128-byte swizzle (TMA).  K is
//                replaced by K * Gam (the A operand of the W product) before the solve.
//   [32K, 48K)   V tile
//   [48K, 80K)   b in log2 units, fp32 [64][128]; after the gate passes: T (16K) + solve scratch (4K)
//   [80K, 112K)  alpha = exp(g), fp32 [64][128]; after the blocks: the T diag(beta) operand image
//   [112K, 128K) A (fp32, f32_offset layout)
//   [128K, 136K) P image (bf16, K-major rows of 64 tokens)
constexpr uint32_t kSmKQ = 0, kSmV = 32768, kSmB = 49152, kSmAl = 81920, kSmA = 114688, kSmP = 131072;
constexpr uint32_t kSmem = kSmP + 8192 + 1024;
constexpr float kLog2e = 1.4426950408889634f;

// fp32 [64][128] table, rows of 512 bytes, 16-byte chunks XOR-rotated by row & 7.
__device__ __forceinline__ uint32_t gb_offset(int i, int c) {
    return (uint32_t)i * 512u + (uint32_t)((((c >> 2) ^ (i & 7)) << 4) + (c & 3) * 4);
}
// 8-channel chunk `cc` (0..15) of row i of the K (qk = 0) or Q (qk = 1) tile.
__device__ __forceinline__ uint32_t kq_chunk(int qk, int i, int cc) {
    return (uint32_t)((cc >> 3) * 16384 + qk * 8192 + i * 128 + (((cc & 7) ^ (i & 7)) << 4));
}
// bf16 pair (c, c+1), c even, of row i of the K / Q tile.
__device__ __forceinline__ uint32_t kq_pair(int qk, int i, int c) { return kq_chunk(qk, i, c >> 3) + (c & 7) * 2; }

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &w, float *f) {
    f[0] = bf_lo(w.x); f[1] = bf_hi(w.x); f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
    f[4] = bf_lo(w.z); f[5] = bf_hi(w.z); f[6] = bf_lo(w.w); f[7] = bf_hi(w.w);
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_prep_kda_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const float *__restrict__ g, const float *__restrict__ beta,
                const int32_t *__restrict__ cu, const int32_t *__restrict__ off, int64_t N, int64_t T, int64_t rows,
                int64_t H, float scale, uint8_t *__restrict__ blocks, int *err) {
    extern __shared__ unsigned char smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    __shared__ uint64_t bar_ld, bar_mma;
    __shared__ uint32_t tmem_base;
    __shared__ float s_beta[C];

    const int64_t chunk = blockIdx.x, h = blockIdx.y;
    ChunkLoc loc;
    if (!locate_chunk(chunk, cu, off, N, T, rows, loc)) return;
    const int L = (int)loc.len;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;
    const int32_t tok0 = (int32_t)loc.start;
    uint8_t *blk = blocks + (size_t)(chunk * H + h) * kTcBlockKda;

    if (tid < C) s_beta[tid] = tid < L ? beta[(int64_t)(tok0 + tid) * H + h] : 0.f;
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
        tma_load_3d(sm + kSmKQ, &mk, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 16384, &mk, 64, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 8192, &mq, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(sm + kSmKQ + 24576, &mq, 64, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(sm + kSmV, &mv, 0, (int32_t)h, tok0, &bar_ld);
        tma_load_3d(sm + kSmV + 8192, &mv, 64, (int32_t)h, tok0, &bar_ld);
    }

    // Gates of the chunk (rows >= L: g = 0): g into the b table, alpha = exp(g) into its own table.
    {
        const float *gsrc = g + ((int64_t)tok0 * H + h) * D;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int e = tid + kThreads * k, i = e >> 5, c = (e & 31) * 4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < L) x = *reinterpret_cast<const float4 *>(gsrc + (int64_t)i * H * D + c);
            *reinterpret_cast<float4 *>(sm + kSmB + gb_offset(i, c)) = x;
            *reinterpret_cast<float4 *>(sm + kSmAl + gb_offset(i, c)) =
                make_float4(ex2(x.x * kLog2e), ex2(x.y * kLog2e), ex2(x.z * kLog2e), ex2(x.w * kLog2e));
        }
        for (int e = tid; e < 512; e += kThreads) *reinterpret_cast<uint4 *>(sm + kSmP + e * 16) = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    // In-chunk inclusive cumsum per key channel, stored in log2 units.
    if (tid < D) {
        float x = 0.f;
#pragma unroll 16
        for (int i = 0; i < C; ++i) {
            float *pb = reinterpret_cast<float *>(sm + kSmB + gb_offset(i, tid));
            x += *pb;
            *pb = x * kLog2e;
        }
    }
    __syncthreads();
    bool ok = mbar_wait(&bar_ld, 0);

    auto bval = [&](int i, int c) { return *reinterpret_cast<const float *>(sm + kSmB + gb_offset(i, c)); };
    auto bpair = [&](int i, int c) { return *reinterpret_cast<const float2 *>(sm + kSmB + gb_offset(i, c)); };

    // Diagonal blocks: warp pair (2p, 2p+1) takes block p; lane = (row pair, 16-channel group).
    // Rows r and 15 - r of a block together need 17 (i, j) steps.
    if (ok) {
        const int p = warp >> 1, rl = lane >> 3, s = lane & 7;
        const int r = 4 * (warp & 1) + rl, base = 16 * p;
        float ki[16], qi[16], d[16];
        auto load_row = [&](int R) {
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, R, 2 * s)), ki);
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, R, 2 * s + 1)), ki + 8);
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(1, R, 2 * s)), qi);
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(1, R, 2 * s + 1)), qi + 8);
#pragma unroll
            for (int c = 0; c < 16; ++c) d[c] = 1.f;
        };
        load_row(base + r);
        for (int it = 0; it < 17; ++it) {
            const bool first = it <= r;
            const int il = first ? r : 15 - r, jl = first ? r - it : 16 - it;
            if (it == r + 1) {
                load_row(base + il);
            } else if (it > 0) {
                // exp(b_i - b_j) = exp(b_i - b_{j+1}) * alpha_{j+1}
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(sm + kSmAl + gb_offset(base + jl + 1, 16 * s + 4 * m));
                    d[4 * m] *= a4.x; d[4 * m + 1] *= a4.y; d[4 * m + 2] *= a4.z; d[4 * m + 3] *= a4.w;
                }
            }
            float kj[16];
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, base + jl, 2 * s)), kj);
            unpack8(*reinterpret_cast<const uint4 *>(sm + kSmKQ + kq_chunk(0, base + jl, 2 * s + 1)), kj + 8);
            float a = 0.f, pp = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float t = kj[c] * d[c];
                a = fmaf(ki[c], t, a);
                pp = fmaf(qi[c], t, pp);
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, o);
                pp += __shfl_xor_sync(0xffffffffu, pp, o);
            }
            if (s == 0) {
                const int i = base + il, j = base + jl;
                if (jl < il) *reinterpret_cast<float *>(sm + kSmA + f32_offset(i, j)) = s_beta[i] * a;
                *reinterpret_cast<__nv_bfloat16 *>(sm + kSmP + i * 128 + (((j >> 3) ^ (i & 7)) << 4) + (j & 7) * 2) =
                    __float2bfloat16_rn(i < L ? scale * pp : 0.f);
            }
        }
    }
    // Blocks below the diagonal: warp w < 6 takes block (p, q) with bf16 m16n8k16 MMAs.
    if (ok && warp < 6) {
        const int p = warp < 1 ? 1 : (warp < 3 ? 2 : 3);
        const int q = warp < 1 ? 0 : (warp < 3 ? warp - 1 : warp - 3);
        const int g8 = lane >> 2, t = lane & 3;
        const int R = 16 * p - 1, i0 = 16 * p + g8, i1 = i0 + 8;
        float cA[2][4], cP[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) cA[nt][e] = cP[nt][e] = 0.f;
        // rows scaled by exp(b - r) (left) or exp(r - b) (right), as bf16 pairs
        auto scaled = [&](int qk, int i, int c, float2 r2, bool left) {
            const float2 bi = bpair(i, c);
            const float e0 = left ? ex2(bi.x - r2.x) : ex2(r2.x - bi.x);
            const float e1 = left ? ex2(bi.y - r2.y) : ex2(r2.y - bi.y);
            const uint32_t w = *reinterpret_cast<const uint32_t *>(sm + kSmKQ + kq_pair(qk, i, c));
            return pack_bf16(bf_lo(w) * e0, bf_hi(w) * e1);
        };
#pragma unroll 2
        for (int kk = 0; kk < 8; ++kk) {
            const int ca = 16 * kk + 2 * t, cb = ca + 8;
            const float2 ra = bpair(R, ca), rb = bpair(R, cb);
            const uint32_t ak[4] = {scaled(0, i0, ca, ra, true), scaled(0, i1, ca, ra, true),
                                    scaled(0, i0, cb, rb, true), scaled(0, i1, cb, rb, true)};
            const uint32_t aq[4] = {scaled(1, i0, ca, ra, true), scaled(1, i1, ca, ra, true),
                                    scaled(1, i0, cb, rb, true), scaled(1, i1, cb, rb, true)};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int j = 16 * q + 8 * nt + g8;
                const uint32_t bz[2] = {scaled(0, j, ca, ra, false), scaled(0, j, cb, rb, false)};
                mma_bf16_16x8x16(cA[nt], ak, bz);
                mma_bf16_16x8x16(cP[nt], aq, bz);
            }
        }
        const float be0 = s_beta[i0], be1 = s_beta[i1];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * q + 8 * nt + 2 * t;
            *reinterpret_cast<float2 *>(sm + kSmA + f32_offset(i0, col)) = make_float2(be0 * cA[nt][0], be0 * cA[nt][1]);
            *reinterpret_cast<float2 *>(sm + kSmA + f32_offset(i1, col)) = make_float2(be1 * cA[nt][2], be1 * cA[nt][3]);
            const uint32_t p0 = i0 < L ? pack_bf16(scale * cP[nt][0], scale * cP[nt][1]) : 0u;
            const uint32_t p1 = i1 < L ? pack_bf16(scale * cP[nt][2], scale * cP[nt][3]) : 0u;
            *reinterpret_cast<uint32_t *>(sm + kSmP + i0 * 128 + (((col >> 3) ^ (i0 & 7)) << 4) + (col & 7) * 2) = p0;
            *reinterpret_cast<uint32_t *>(sm + kSmP + i1 * 128 + (((col >> 3) ^ (i1 & 7)) << 4) + (col & 7) * 2) = p1;
        }
    }
    __syncthreads();

    // Gate passes over the K and Q tiles (16-byte chunks, 8 channels each):
    // K * Gam in place, K~ = K * exp(b_L - b) and Qs = scale Q * Gam to the block.
    if (ok) {
        const int Lm1 = L - 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int e = tid + kThreads * k;
            const int half = e >> 9, i = (e & 511) >> 3, pc = e & 7;
            const int c8 = half * 64 + ((pc ^ (i & 7)) << 3);
            const uint32_t so = (uint32_t)(half * 16384 + i * 128 + pc * 16);
            const uint4 kw = *reinterpret_cast<const uint4 *>(sm + kSmKQ + so);
            const uint4 qw = *reinterpret_cast<const uint4 *>(sm + kSmKQ + so + 8192);
            float kf[8], qf[8], bi[8], bl[8];
            unpack8(kw, kf);
            unpack8(qw, qf);
            *reinterpret_cast<float4 *>(bi) = *reinterpret_cast<const float4 *>(sm + kSmB + gb_offset(i, c8));
            *reinterpret_cast<float4 *>(bi + 4) = *reinterpret_cast<const float4 *>(sm + kSmB + gb_offset(i, c8 + 4));
            *reinterpret_cast<float4 *>(bl) = *reinterpret_cast<const float4 *>(sm + kSmB + gb_offset(Lm1, c8));
            *reinterpret_cast<float4 *>(bl + 4) = *reinterpret_cast<const float4 *>(sm + kSmB + gb_offset(Lm1, c8 + 4));
            uint32_t kg[4], kt[4], qs[4];
            const bool in = i < L;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float g0 = ex2(bi[2 * m]), g1 = ex2(bi[2 * m + 1]);
                const float t0 = ex2(bl[2 * m] - bi[2 * m]), t1 = ex2(bl[2 * m + 1] - bi[2 * m + 1]);
                kg[m] = in ? pack_bf16(kf[2 * m] * g0, kf[2 * m + 1] * g1) : 0u;
                kt[m] = in ? pack_bf16(kf[2 * m] * t0, kf[2 * m + 1] * t1) : 0u;
                qs[m] = in ? pack_bf16(scale * qf[2 * m] * g0, scale * qf[2 * m + 1] * g1) : 0u;
            }
            *reinterpret_cast<uint4 *>(sm + kSmKQ + so) = make_uint4(kg[0], kg[1], kg[2], kg[3]);
            *reinterpret_cast<uint4 *>(blk + kBlkKt + half * 8192 + i * 128 + pc * 16) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
            *reinterpret_cast<uint4 *>(blk + kBlkWQ + 8192 + half * 16384 + i * 128 + pc * 16) =
                make_uint4(qs[0], qs[1], qs[2], qs[3]);
        }
        // the P image, and the gate factors
        for (int e = tid; e < 512; e += kThreads)
            *reinterpret_cast<uint4 *>(blk + kBlkP + e * 16) = *reinterpret_cast<const uint4 *>(sm + kSmP + e * 16);
        float *fac = reinterpret_cast<float *>(blk + kBlkFac);
        if (tid < D) fac[kFacGL + tid] = ex2(bval(Lm1, tid));
        else if (tid < D + C) fac[kFacW + tid - D] = tid - D < L ? 1.f : 0.f;
        else if (tid < D + 2 * C) fac[kFacSG + tid - D - C] = 0.f;
    }
    fence_async_smem();  // K * Gam is read by the tensor core
    __syncthreads();

    // T = (I + A)^-1 into the (now free) b table region.
    blocked_solve<kSmB, kSmB + 16384>(sm, [](int i, int j) { return kSmA + f32_offset(i, j); }, ok);

    // T'' = T diag(beta) as a bf16 operand image (K-major rows i) in the alpha table region.
    if (ok) {
        const int i = tid >> 2, j0 = (tid & 3) * 16;
        float tv[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = *reinterpret_cast<const float4 *>(sm + kSmB + f32_offset(i, j0 + 4 * q));
            tv[4 * q] = f.x; tv[4 * q + 1] = f.y; tv[4 * q + 2] = f.z; tv[4 * q + 3] = f.w;
        }
        const uint32_t tp = smem_u32(sm + kSmAl);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) b[e] = tv[8 * q + e] * s_beta[j0 + 8 * q + e];
            st_shared_v4(tp + sw128_offset(i, (j0 >> 3) + q), pack_bf16(b[0], b[1]), pack_bf16(b[2], b[3]),
                         pack_bf16(b[4], b[5]), pack_bf16(b[6], b[7]));
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // W^T = (K * Gam)^T T''^T (M = d_k), U^T = V^T T''^T (M = d_v); K = 64 tokens.
    if (warp == 0 && __all_sync(0xffffffffu, ok)) {
        const uint64_t dk = sdesc_sw128(smem_u32(sm + kSmKQ), 16384, 1024), dv = sdesc_sw128(smem_u32(sm + kSmV), 8192, 1024),
                       dt = sdesc_sw128(smem_u32(sm + kSmAl), 16, 1024);
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tm, dk + ((kk * 2048) >> 4), dt + ((kk * 32) >> 4), id, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(tm + 64, dv + ((kk * 2048) >> 4), dt + ((kk * 32) >> 4), id, kk > 0);
        mma_commit_warp(&bar_mma);
    }
    ok = ok && mbar_wait(&bar_mma, 0);
    tc_fence_after();
    if (ok) {
        store_wu(tm, blk, qd, hf, lane);
    } else if (tid == 0) {
        flag_error(err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 128);
}

}  // namespace

gdn_status launch_prep_kda(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const ChunkPlan &p,
                           const ChunkArgs &a, const int32_t *off, uint8_t *blocks, cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = cudaFuncSetAttribute(gdn_prep_kda_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    });
    if (attr != cudaSuccess) return fail(GDN_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(attr));
    LaunchScope ls("gdn_prep_kda_tc", s);
    gdn_prep_kda_tc<<<dim3((unsigned)p.max_chunks, (unsigned)p.H), kThreads, kSmem, s>>>(
        mq, mk, mv, a.g, a.beta, a.cu_seqlens, off, a.N, a.T, p.rows, p.H, a.scale, blocks, nullptr);
    return check_launch("gdn_prep_kda_tc");
}

}  // namespace tc
}  // namespace gdn
