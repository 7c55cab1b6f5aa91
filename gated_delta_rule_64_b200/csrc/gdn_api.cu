// C-ABI entry points: argument validation, workspace planning, launches and
// the optional per-kernel event timer.  No device memory is allocated here.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "gdn_internal.cuh"

namespace gdn {

// ---------------------------------------------------------------------------
// Error reporting
// ---------------------------------------------------------------------------
static thread_local char g_last_error[512] = "";

gdn_status fail(gdn_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

gdn_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return GDN_OK;
}

void log_launch(const char *name, dim3 grid, dim3 block, size_t smem) {
    static const bool on = [] {
        const char *e = getenv("GDN_LOG");
        return e && e[0] && strcmp(e, "0") != 0;
    }();
    if (on)
        fprintf(stderr, "gdn: launch %s grid (%u, %u, %u) block (%u, %u, %u) smem %zu\n", name, grid.x, grid.y, grid.z,
                block.x, block.y, block.z, smem);
}

// ---------------------------------------------------------------------------
// Event timer
// ---------------------------------------------------------------------------
namespace {
struct ProfRecord {
    const char *name;
    cudaEvent_t start, stop;
};
struct ProfState {
    std::mutex mu;
    bool on = false;
    std::vector<ProfRecord> open;     // recorded, not yet read
    std::vector<cudaEvent_t> pool;    // free events
    cudaEvent_t get() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        return e;
    }
};
ProfState &prof() {
    static ProfState *p = new ProfState();  // never destroyed: events may outlive static teardown
    return *p;
}
}  // namespace

LaunchScope::LaunchScope(const char *name, cudaStream_t s) : name_(name), stream_(s), slot_(-1) {
    ProfState &P = prof();
    std::lock_guard<std::mutex> lk(P.mu);
    if (!P.on) return;
    cudaEvent_t a = P.get(), b = P.get();
    if (!a || !b) return;
    cudaEventRecord(a, s);
    P.open.push_back({name, a, b});
    slot_ = (int)P.open.size() - 1;
}

LaunchScope::~LaunchScope() {
    if (slot_ < 0) return;
    ProfState &P = prof();
    std::lock_guard<std::mutex> lk(P.mu);
    if (slot_ < (int)P.open.size()) cudaEventRecord(P.open[slot_].stop, stream_);
}

// ---------------------------------------------------------------------------
// Workspace plan of the chunked forward pass
// ---------------------------------------------------------------------------
static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

ChunkPlan make_plan(const gdn_desc &d, int64_t num_seqs, bool packed) {
    ChunkPlan p{};
    p.N = num_seqs;
    p.rows = d.B * d.T;
    p.H = d.H;
    p.dk = d.dk;
    p.dv = d.dv;
    p.packed = packed;
    p.per_channel = d.gate == GDN_GATE_CHANNEL;
    // Every sequence of length L has ceil(L/64) chunks; over any packing of
    // `rows` tokens into N sequences that is at most rows/64 + N.
    p.max_chunks = packed ? (p.rows / kChunk + p.N) : (d.B * ((d.T + kChunk - 1) / kChunk));
    p.tc = tc_eligible(d) && p.rows < (1LL << 31);
    const int64_t ch = p.max_chunks * p.H;
    size_t off = 0;
    p.off_status = off;
    off += kStatusBytes;
    p.off_chunk_offsets = off;
    off = align_up(off + sizeof(int32_t) * (size_t)(2 * p.N + 1), 256);
    p.split_G = 1;
    p.split_seg = 0;
    p.off_split = 0;
    if (p.tc) {
        p.tc_block = kTcBlock;
        p.off_W = p.off_U = p.off_P = p.off_b = off;  // one block of tc_block bytes per chunk-head
        off = align_up(off + p.tc_block * (size_t)ch, 256);
        if (!packed && d.T > 0) {
            int dev = 0, sms = 0;
            if (cudaGetDevice(&dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
                cudaGetLastError();
                sms = 148;
            }
            const SplitChoice sc = choose_split(p.N, p.H, (d.T + kChunk - 1) / kChunk, sms);
            if (sc.G >= 2) {
                p.split_G = sc.G;
                p.split_seg = sc.seg;
                p.off_split = off;
                off = align_up(off + sizeof(float) * (size_t)p.N * sc.G * 3 * p.H * p.dv * p.dk +
                                   sizeof(int32_t) * 2 * (size_t)p.N * sc.G * p.H,
                               256);
            }
        }
    } else {
        p.off_W = off;
        off = align_up(off + sizeof(float) * (size_t)ch * kChunk * p.dk, 256);
        p.off_U = off;
        off = align_up(off + sizeof(float) * (size_t)ch * kChunk * p.dv, 256);
        p.off_P = off;
        off = align_up(off + sizeof(float) * (size_t)ch * kChunk * kChunk, 256);
        p.off_b = off;
        off = align_up(off + sizeof(float) * (size_t)ch * kChunk * (p.per_channel ? p.dk : 1), 256);
    }
    p.total = off;
    return p;
}

// ---------------------------------------------------------------------------
// Validation helpers
// ---------------------------------------------------------------------------
static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
static bool aligned4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

static gdn_status check_desc(const gdn_desc *d) {
    if (!d) return fail(GDN_ERR_INVALID_ARG, "descriptor is NULL");
    if (d->B < 0 || d->T < 0 || d->H <= 0)
        return fail(GDN_ERR_INVALID_ARG, "need B >= 0, T >= 0, H > 0 (got B=%lld T=%lld H=%lld)",
                    (long long)d->B, (long long)d->T, (long long)d->H);
    if (d->dk <= 0 || d->dv <= 0)
        return fail(GDN_ERR_INVALID_ARG, "head sizes must be positive");
    if (!((d->dk == 64 || d->dk == 128) && (d->dv == 64 || d->dv == 128)))
        return fail(GDN_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %lld, %lld)",
                    (long long)d->dk, (long long)d->dv);
    if (d->dtype != GDN_F32 && d->dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "unknown dtype %d", d->dtype);
    if (d->gate != GDN_GATE_HEAD && d->gate != GDN_GATE_CHANNEL)
        return fail(GDN_ERR_INVALID_ARG, "unknown gate kind %d", d->gate);
    if (d->hk < 0 || d->hk > d->H || (d->hk > 0 && d->H % d->hk != 0))
        return fail(GDN_ERR_INVALID_ARG, "hk must be 0 or a divisor of H (got %d for H = %lld)", d->hk,
                    (long long)d->H);
    if (!isfinite(d->scale)) return fail(GDN_ERR_INVALID_ARG, "scale must be finite");
    // Keep every element index of every tensor well inside int64.
    const double elems = (double)d->B * (double)d->T * (double)d->H * (double)(d->dk > d->dv ? d->dk : d->dv);
    if (elems > 4.0e15) return fail(GDN_ERR_INVALID_ARG, "problem too large");
    return GDN_OK;
}

struct Range {
    uintptr_t lo, hi;
};
static bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }
static Range range_of(const void *p, size_t bytes) { return {(uintptr_t)p, (uintptr_t)p + bytes}; }

}  // namespace gdn

using namespace gdn;

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device wait timed out";
        case GDN_ERR_INTERNAL: return "internal error";
    }
    return "unknown status";
}

const char *gdn_last_error(void) { return g_last_error; }

gdn_status gdn_profile_enable(int on) {
    ProfState &P = prof();
    std::lock_guard<std::mutex> lk(P.mu);
    P.on = on != 0;
    return GDN_OK;
}

gdn_status gdn_profile_read(gdn_kernel_time *entries, int32_t cap, int32_t *count) {
    if (!count || cap < 0 || (cap > 0 && !entries)) return fail(GDN_ERR_INVALID_ARG, "bad profile_read args");
    ProfState &P = prof();
    std::lock_guard<std::mutex> lk(P.mu);
    std::vector<gdn_kernel_time> acc;
    gdn_status st = GDN_OK;
    for (auto &r : P.open) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            st = fail(GDN_ERR_CUDA, "profile: event query failed");
        size_t i = 0;
        for (; i < acc.size(); ++i)
            if (strcmp(acc[i].name, r.name) == 0) break;
        if (i == acc.size()) acc.push_back({r.name, 0, 0.0});
        acc[i].launches += 1;
        acc[i].total_ms += ms;
        P.pool.push_back(r.start);
        P.pool.push_back(r.stop);
    }
    P.open.clear();
    *count = (int32_t)acc.size();
    for (int32_t i = 0; i < cap && i < (int32_t)acc.size(); ++i) entries[i] = acc[i];
    return st;
}

gdn_status gdn_chunk_workspace_size(const gdn_desc *d, int32_t num_seqs, size_t *bytes) {
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (!bytes) return fail(GDN_ERR_INVALID_ARG, "bytes is NULL");
    if (num_seqs < 0) return fail(GDN_ERR_INVALID_ARG, "num_seqs < 0");
    // The packed-sequence bound covers B fixed-length sequences too
    // (B * ceil(T/64) <= B*T/64 + B); fixed-length sequences may add the state
    // maps of the split scan.
    size_t total = make_plan(*d, num_seqs, true).total;
    if (num_seqs == d->B) {
        const size_t fixed = make_plan(*d, num_seqs, false).total;
        total = fixed > total ? fixed : total;
    }
    *bytes = total;
    return GDN_OK;
}

gdn_status gdn_chunk_fwd(const gdn_desc *d, const void *q, const void *k, const void *v,
                         const float *log_gate, const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens, int32_t num_seqs, int64_t snapshot_stride,
                         void *out, float *final_state, float *snapshots, void *workspace,
                         size_t workspace_bytes, gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    const bool packed = cu_seqlens != nullptr;
    if (packed) {
        if (d->B != 1) return fail(GDN_ERR_INVALID_ARG, "packed sequences need B == 1");
        if (num_seqs < 0) return fail(GDN_ERR_INVALID_ARG, "num_seqs < 0");
        if (((uintptr_t)cu_seqlens & 3u) != 0) return fail(GDN_ERR_INVALID_ARG, "cu_seqlens misaligned");
        if (snapshot_stride != 0)
            return fail(GDN_ERR_UNSUPPORTED, "snapshots are only supported without cu_seqlens");
    }
    const int64_t N = packed ? num_seqs : d->B;
    if (snapshot_stride < 0 || snapshot_stride % kChunk != 0)
        return fail(GDN_ERR_INVALID_ARG, "snapshot_stride must be 0 or a positive multiple of 64");
    const int64_t n_snap = (snapshot_stride > 0 && !packed) ? d->T / snapshot_stride : 0;
    const int64_t rows = d->B * d->T;
    const size_t in_el = d->dtype == GDN_F32 ? 4 : 2;
    const size_t qk_bytes = (size_t)rows * qk_heads(*d) * d->dk * in_el;
    const size_t v_bytes = (size_t)rows * d->H * d->dv * in_el;
    const size_t g_bytes = (size_t)rows * d->H * (d->gate == GDN_GATE_CHANNEL ? d->dk : 1) * 4;
    const size_t b_bytes = (size_t)rows * d->H * 4;
    const size_t st_bytes = (size_t)N * d->H * d->dv * d->dk * 4;
    const size_t snap_bytes = (size_t)N * n_snap * d->H * d->dv * d->dk * 4;
    if (rows > 0) {
        if (!q || !k || !v || !log_gate || !beta || !out)
            return fail(GDN_ERR_INVALID_ARG, "q, k, v, log_gate, beta and out are required");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
            return fail(GDN_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
        if (!aligned4(log_gate) || !aligned4(beta))
            return fail(GDN_ERR_INVALID_ARG, "log_gate and beta must be 4-byte aligned");
        if (d->gate == GDN_GATE_CHANNEL && !aligned16(log_gate))
            return fail(GDN_ERR_INVALID_ARG, "a per-channel log_gate must be 16-byte aligned");
        const Range ro = range_of(out, v_bytes);
        const Range ins[] = {range_of(q, qk_bytes), range_of(k, qk_bytes), range_of(v, v_bytes),
                             range_of(log_gate, g_bytes), range_of(beta, b_bytes)};
        for (const Range &r : ins)
            if (overlaps(ro, r)) return fail(GDN_ERR_INVALID_ARG, "out overlaps an input");
        if (initial_state && overlaps(ro, range_of(initial_state, st_bytes)))
            return fail(GDN_ERR_INVALID_ARG, "out overlaps initial_state");
        if (final_state && overlaps(ro, range_of(final_state, st_bytes)))
            return fail(GDN_ERR_INVALID_ARG, "out overlaps final_state");
    }
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)) ||
        (snapshots && !aligned16(snapshots)))
        return fail(GDN_ERR_INVALID_ARG, "state pointers must be 16-byte aligned");
    if (final_state && initial_state && final_state != initial_state &&
        overlaps(range_of(final_state, st_bytes), range_of(initial_state, st_bytes)))
        return fail(GDN_ERR_INVALID_ARG, "final_state partially overlaps initial_state");
    if (n_snap > 0 && !snapshots) return fail(GDN_ERR_INVALID_ARG, "snapshots buffer is required");
    if (n_snap > 0 && final_state && overlaps(range_of(snapshots, snap_bytes), range_of(final_state, st_bytes)))
        return fail(GDN_ERR_INVALID_ARG, "snapshots overlap final_state");

    ChunkPlan p = make_plan(*d, N, packed);
    if (N == 0) return GDN_OK;
    if (!workspace) return fail(GDN_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", p.total);
    if (((uintptr_t)workspace & 255u) != 0) return fail(GDN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (workspace_bytes < p.total)
        return fail(GDN_ERR_WORKSPACE, "workspace has %zu bytes, need %zu", workspace_bytes, p.total);

    ChunkArgs a{};
    a.status = reinterpret_cast<int *>(reinterpret_cast<char *>(workspace) + p.off_status);
    {
        const cudaError_t e = cudaMemsetAsync(a.status, 0, sizeof(int32_t), (cudaStream_t)stream);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
    }
    a.q = q; a.k = k; a.v = v; a.g = log_gate; a.beta = beta; a.h0 = initial_state;
    a.cu_seqlens = cu_seqlens;
    a.T = d->T;
    a.N = N;
    a.H = d->H;
    a.Hk = qk_heads(*d);
    a.scale = d->scale;
    a.snapshot_stride = snapshot_stride;
    a.n_snap = n_snap;
    a.out = out;
    a.final_state = final_state;
    a.snapshots = snapshots;
    a.ws = (char *)workspace;
    return p.tc ? launch_chunk_tc(p, a, (cudaStream_t)stream) : launch_chunk_simt(p, a, d->dtype, (cudaStream_t)stream);
}

gdn_status gdn_chunk_status(const void *workspace, gdn_stream_t stream, int32_t *device_code) {
    g_last_error[0] = 0;
    if (!workspace || !device_code) return fail(GDN_ERR_INVALID_ARG, "workspace and device_code are required");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    int32_t code = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&code, workspace, sizeof code, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    *device_code = code;
    if (code == GDN_DEV_OK) return GDN_OK;
    if (code == GDN_DEV_TIMEOUT_PREP || code == GDN_DEV_TIMEOUT_SCAN)
        return fail(GDN_ERR_TIMEOUT, "a device-side wait gave up (%s)",
                    code == GDN_DEV_TIMEOUT_PREP ? "chunk-local kernel" : "scan");
    return fail(GDN_ERR_INTERNAL, "device status %d", (int)code);
}

gdn_status gdn_decode_step(const gdn_desc *d, const void *q, const void *k, const void *v,
                           const float *log_gate, const float *beta, float *state, void *out,
                           gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (d->T != 1) return fail(GDN_ERR_INVALID_ARG, "decode needs T == 1 (got %lld)", (long long)d->T);
    if (d->B == 0) return GDN_OK;
    if (!q || !k || !v || !log_gate || !beta || !state || !out)
        return fail(GDN_ERR_INVALID_ARG, "all decode pointers are required");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, state and out must be 16-byte aligned");
    if (!aligned4(log_gate) || !aligned4(beta))
        return fail(GDN_ERR_INVALID_ARG, "log_gate and beta must be 4-byte aligned");
    const size_t in_el = d->dtype == GDN_F32 ? 4 : 2;
    const Range ro = range_of(out, (size_t)d->B * d->H * d->dv * in_el);
    const Range rs = range_of(state, (size_t)d->B * d->H * d->dv * d->dk * 4);
    const Range ins[] = {range_of(q, (size_t)d->B * qk_heads(*d) * d->dk * in_el),
                         range_of(k, (size_t)d->B * qk_heads(*d) * d->dk * in_el),
                         range_of(v, (size_t)d->B * d->H * d->dv * in_el),
                         range_of(log_gate, (size_t)d->B * d->H * (d->gate == GDN_GATE_CHANNEL ? d->dk : 1) * 4),
                         range_of(beta, (size_t)d->B * d->H * 4)};
    if (overlaps(ro, rs)) return fail(GDN_ERR_INVALID_ARG, "out overlaps state");
    for (const Range &r : ins)
        if (overlaps(ro, r) || overlaps(rs, r)) return fail(GDN_ERR_INVALID_ARG, "out or state overlaps an input");
    return launch_decode(*d, q, k, v, log_gate, beta, state, out, (cudaStream_t)stream);
}

gdn_status gdn_decode_step_prerule(const gdn_desc *d, const void *x, const void *a, const void *b,
                                   const float *conv_w, int32_t K, const float *A_log, const float *dt_bias,
                                   float *conv_state, float *state, void *out, gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (d->T != 1) return fail(GDN_ERR_INVALID_ARG, "decode needs T == 1 (got %lld)", (long long)d->T);
    if (d->gate != GDN_GATE_HEAD)
        return fail(GDN_ERR_UNSUPPORTED, "the pre-rule gate formula is the per-head one");
    if (K < 1 || K > 4) return fail(GDN_ERR_UNSUPPORTED, "convolution width %d (1 .. 4 supported)", K);
    if (d->B == 0) return GDN_OK;
    if (!x || !a || !b || !conv_w || !A_log || !dt_bias || !state || !out)
        return fail(GDN_ERR_INVALID_ARG, "x, a, b, conv_w, A_log, dt_bias, state and out are required");
    const size_t el = d->dtype == GDN_F32 ? 4 : 2;
    if (!aligned16(state) || !aligned16(out)) return fail(GDN_ERR_INVALID_ARG, "state and out must be 16-byte aligned");
    if (((uintptr_t)x % el) || ((uintptr_t)a % el) || ((uintptr_t)b % el) || !aligned4(conv_w) || !aligned4(A_log) ||
        !aligned4(dt_bias) || (conv_state && !aligned4(conv_state)))
        return fail(GDN_ERR_INVALID_ARG, "x, a, b: element-aligned; conv_w, A_log, dt_bias, conv_state: 4-byte aligned");
    const int64_t Hk = qk_heads(*d), C = 2 * Hk * d->dk + d->H * d->dv;
    const Range outs[] = {range_of(out, (size_t)d->B * d->H * d->dv * el),
                          range_of(state, (size_t)d->B * d->H * d->dv * d->dk * 4),
                          range_of(conv_state, conv_state ? (size_t)d->B * C * (K - 1) * 4 : 0)};
    const Range ins[] = {range_of(x, (size_t)d->B * C * el), range_of(a, (size_t)d->B * d->H * el),
                         range_of(b, (size_t)d->B * d->H * el), range_of(conv_w, (size_t)C * K * 4),
                         range_of(A_log, (size_t)d->H * 4), range_of(dt_bias, (size_t)d->H * 4)};
    for (int i = 0; i < 3; ++i) {
        for (const Range &r : ins)
            if (overlaps(outs[i], r)) return fail(GDN_ERR_INVALID_ARG, "an output overlaps an input");
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], outs[j])) return fail(GDN_ERR_INVALID_ARG, "outputs overlap");
    }
    PreruleArgs p{};
    p.dtype = d->dtype;
    p.K = K;
    p.T = 1;
    p.N = d->B;
    p.rows = d->B;
    p.H = d->H;
    p.Hk = Hk;
    p.dk = d->dk;
    p.dv = d->dv;
    p.x = x;
    p.a = a;
    p.b = b;
    p.conv_w = conv_w;
    p.A_log = A_log;
    p.dt_bias = dt_bias;
    p.cu_seqlens = nullptr;
    p.hist_in = conv_state;
    p.hist_out = conv_state;
    return launch_decode_prerule(*d, p, state, out, (cudaStream_t)stream);
}

gdn_status gdn_decode_multi(const gdn_desc *d, const void *q, const void *k, const void *v,
                            const float *log_gate, const float *beta, const int32_t *n_tokens, float *state,
                            int32_t commit, void *out, float *step_states, gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (d->T < 1 || d->T > kMaxMultiTokens)
        return fail(GDN_ERR_INVALID_ARG, "multi-token decode needs 1 <= T <= %lld (got %lld)",
                    (long long)kMaxMultiTokens, (long long)d->T);
    if (commit != 0 && commit != 1) return fail(GDN_ERR_INVALID_ARG, "commit must be 0 or 1");
    if (d->B == 0) return GDN_OK;
    if (!q || !k || !v || !log_gate || !beta || !state || !out)
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, log_gate, beta, state and out are required");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out) ||
        (step_states && !aligned16(step_states)))
        return fail(GDN_ERR_INVALID_ARG, "q, k, v, state, out and step_states must be 16-byte aligned");
    if (!aligned4(log_gate) || !aligned4(beta) || (n_tokens && !aligned4(n_tokens)))
        return fail(GDN_ERR_INVALID_ARG, "log_gate, beta and n_tokens must be 4-byte aligned");
    const size_t in_el = d->dtype == GDN_F32 ? 4 : 2;
    const size_t bth = (size_t)d->B * d->T * d->H;
    const size_t sbytes = (size_t)d->dv * d->dk * 4;
    const Range ro = range_of(out, bth * d->dv * in_el);
    const Range rs = range_of(state, (size_t)d->B * d->H * sbytes);
    const Range rss = range_of(step_states, step_states ? bth * sbytes : 0);
    const size_t btk = (size_t)d->B * d->T * qk_heads(*d);
    const Range ins[] = {range_of(q, btk * d->dk * in_el), range_of(k, btk * d->dk * in_el),
                         range_of(v, bth * d->dv * in_el),
                         range_of(log_gate, bth * (d->gate == GDN_GATE_CHANNEL ? d->dk : 1) * 4),
                         range_of(beta, bth * 4), range_of(n_tokens, n_tokens ? (size_t)d->B * 4 : 0)};
    if (overlaps(ro, rs) || overlaps(ro, rss) || overlaps(rs, rss))
        return fail(GDN_ERR_INVALID_ARG, "out, state and step_states must not overlap");
    for (const Range &r : ins)
        if (overlaps(ro, r) || overlaps(rs, r) || overlaps(rss, r))
            return fail(GDN_ERR_INVALID_ARG, "out, state or step_states overlaps an input");
    return launch_decode_multi(*d, q, k, v, log_gate, beta, n_tokens, state, commit, out, step_states,
                               (cudaStream_t)stream);
}

gdn_status gdn_prerule(const gdn_desc *d, const void *x, const void *a, const void *b, const float *conv_w,
                       int32_t K, const float *A_log, const float *dt_bias, const int32_t *cu_seqlens,
                       int32_t num_seqs, const float *conv_state_in, float *conv_state_out, void *q, void *k,
                       void *v, float *log_gate, float *beta, gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (d->gate != GDN_GATE_HEAD)
        return fail(GDN_ERR_UNSUPPORTED, "the pre-rule gate formula is the per-head one");
    if (K < 1 || K > 4) return fail(GDN_ERR_UNSUPPORTED, "convolution width %d (1 .. 4 supported)", K);
    const bool packed = cu_seqlens != nullptr;
    if (packed && d->B != 1) return fail(GDN_ERR_INVALID_ARG, "packed sequences need B == 1");
    if (packed && num_seqs < 0) return fail(GDN_ERR_INVALID_ARG, "num_seqs < 0");
    const int64_t N = packed ? num_seqs : d->B;
    const int64_t rows = d->B * d->T, Hk = qk_heads(*d);
    const int64_t C = 2 * Hk * d->dk + d->H * d->dv;
    if (rows == 0 && N == 0) return GDN_OK;
    if (rows > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "more than 2^31 - 1 token rows");
    if (!x || !a || !b || !conv_w || !A_log || !dt_bias || !q || !k || !v || !log_gate || !beta)
        return fail(GDN_ERR_INVALID_ARG, "x, a, b, conv_w, A_log, dt_bias and the five outputs are required");
    const size_t el = d->dtype == GDN_F32 ? 4 : 2;
    if (!aligned16(x) || !aligned16(q) || !aligned16(k) || !aligned16(v))
        return fail(GDN_ERR_INVALID_ARG, "x, q, k and v must be 16-byte aligned");
    if (((uintptr_t)a % el) || ((uintptr_t)b % el) || !aligned4(conv_w) || !aligned4(A_log) || !aligned4(dt_bias) ||
        !aligned4(log_gate) || !aligned4(beta) || (conv_state_in && !aligned4(conv_state_in)) ||
        (conv_state_out && !aligned4(conv_state_out)) || (cu_seqlens && !aligned4(cu_seqlens)))
        return fail(GDN_ERR_INVALID_ARG, "a, b: element-aligned; conv_w, A_log, dt_bias, gates, states, "
                                         "cu_seqlens: 4-byte aligned");
    const size_t hist_bytes = (size_t)N * C * (K - 1) * 4;
    const Range outs[] = {range_of(q, (size_t)rows * Hk * d->dk * el), range_of(k, (size_t)rows * Hk * d->dk * el),
                          range_of(v, (size_t)rows * d->H * d->dv * el), range_of(log_gate, (size_t)rows * d->H * 4),
                          range_of(beta, (size_t)rows * d->H * 4),
                          range_of(conv_state_out, conv_state_out ? hist_bytes : 0)};
    const Range ins[] = {range_of(x, (size_t)rows * C * el), range_of(a, (size_t)rows * d->H * el),
                         range_of(b, (size_t)rows * d->H * el), range_of(conv_w, (size_t)C * K * 4),
                         range_of(A_log, (size_t)d->H * 4), range_of(dt_bias, (size_t)d->H * 4),
                         range_of(cu_seqlens, cu_seqlens ? (size_t)(N + 1) * 4 : 0)};
    for (int i = 0; i < 6; ++i) {
        for (const Range &r : ins)
            if (overlaps(outs[i], r)) return fail(GDN_ERR_INVALID_ARG, "an output overlaps an input");
        for (int j = i + 1; j < 6; ++j)
            if (overlaps(outs[i], outs[j])) return fail(GDN_ERR_INVALID_ARG, "outputs overlap");
    }
    // the new history may replace the old one in place, but not overlap it partly
    if (conv_state_in && conv_state_out && conv_state_in != conv_state_out &&
        overlaps(range_of(conv_state_in, hist_bytes), range_of(conv_state_out, hist_bytes)))
        return fail(GDN_ERR_INVALID_ARG, "conv_state_out partially overlaps conv_state_in");
    PreruleArgs pa{};
    pa.dtype = d->dtype;
    pa.K = K;
    pa.T = d->T;
    pa.N = N;
    pa.rows = rows;
    pa.H = d->H;
    pa.Hk = Hk;
    pa.dk = d->dk;
    pa.dv = d->dv;
    pa.x = x; pa.a = a; pa.b = b;
    pa.conv_w = conv_w; pa.A_log = A_log; pa.dt_bias = dt_bias;
    pa.cu_seqlens = cu_seqlens;
    pa.hist_in = conv_state_in; pa.hist_out = conv_state_out;
    pa.q = q; pa.k = k; pa.v = v; pa.g = log_gate; pa.beta = beta;
    return launch_prerule(pa, (cudaStream_t)stream);
}

gdn_status gdn_state_select(const gdn_desc *d, const float *step_states, const int32_t *accept, float *state,
                            gdn_stream_t stream) {
    g_last_error[0] = 0;
    gdn_status st = check_desc(d);
    if (st != GDN_OK) return st;
    if (d->T < 1 || d->T > kMaxMultiTokens)
        return fail(GDN_ERR_INVALID_ARG, "state select needs 1 <= T <= %lld (got %lld)",
                    (long long)kMaxMultiTokens, (long long)d->T);
    if (d->B == 0) return GDN_OK;
    if (!step_states || !accept || !state)
        return fail(GDN_ERR_INVALID_ARG, "step_states, accept and state are required");
    if (!aligned16(step_states) || !aligned16(state) || !aligned4(accept))
        return fail(GDN_ERR_INVALID_ARG, "step_states and state must be 16-byte aligned, accept 4-byte");
    const size_t sbytes = (size_t)d->dv * d->dk * 4;
    const Range rs = range_of(state, (size_t)d->B * d->H * sbytes);
    if (overlaps(rs, range_of(step_states, (size_t)d->B * d->T * d->H * sbytes)) ||
        overlaps(rs, range_of(accept, (size_t)d->B * 4)))
        return fail(GDN_ERR_INVALID_ARG, "state overlaps step_states or accept");
    return launch_state_select(*d, step_states, accept, state, (cudaStream_t)stream);
}

}  // extern "C"
