// Chunk bookkeeping shared by the chunked-prefill kernels: where each chunk
// of each (packed or fixed-length) sequence starts and how long it is.
#pragma once

#include <stdint.h>

#include "gdn_internal.cuh"

namespace gdn {

// Bounds-checked builds (compiled with -DGDN_CHECKED): the chunked-prefill kernels
// check the sequence, head and token range each block derives from the sizes the
// host passed against those sizes before touching memory; a failed check records
// GDN_DEV_BOUNDS in the call's status word and the block does nothing.  In the
// ordinary build the checks compile away.
#ifdef GDN_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
__device__ __forceinline__ bool in_bounds(bool cond, int *err) {
    if (!kChecked) return true;
    if (!cond && err) atomicCAS(err, 0, (int)GDN_DEV_BOUNDS);
    return cond;
}

// Token range of the chunk `chunk` (global index), or false when the index is
// past the last chunk.  Offsets from cu_seqlens are clamped into [0, rows].
struct ChunkLoc {
    int64_t n, c, start, len;  // sequence, chunk within it, first token row, tokens (<= 64)
};

__device__ __forceinline__ void seq_bounds(const int32_t *cu, int64_t n, int64_t T, int64_t rows,
                                           int64_t &start, int64_t &len) {
    if (cu) {
        int64_t a = cu[n], b = cu[n + 1];
        a = a < 0 ? 0 : (a > rows ? rows : a);
        b = b < a ? a : (b > rows ? rows : b);
        start = a;
        len = b - a;
    } else {
        start = n * T;
        len = T;
    }
}

__device__ __forceinline__ bool locate_chunk(int64_t chunk, const int32_t *cu, const int32_t *off, int64_t N, int64_t T,
                             int64_t rows, ChunkLoc &loc) {
    int64_t n, c;
    if (cu) {
        if (chunk >= off[N]) return false;
        int64_t lo = 0, hi = N;  // find n with off[n] <= chunk < off[n+1]
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) / 2;
            if (off[mid] <= chunk) lo = mid; else hi = mid;
        }
        n = lo;
        c = chunk - off[n];
    } else {
        const int64_t cps = (T + kChunk - 1) / kChunk;
        if (cps == 0) return false;
        n = chunk / cps;
        c = chunk % cps;
        if (n >= N) return false;
    }
    int64_t start, len;
    seq_bounds(cu, n, T, rows, start, len);
    if (c * kChunk >= len) return false;
    loc.n = n;
    loc.c = c;
    loc.start = start + c * kChunk;
    loc.len = len - c * kChunk < kChunk ? len - c * kChunk : kChunk;
    return true;
}

}  // namespace gdn
