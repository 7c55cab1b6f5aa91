// gdn_chunk_fwd_static: the chunked prefill with its scratch memory in a
// fixed-size array that is part of the library image, for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not
// affordable -- a serving loop on a fixed, pre-partitioned memory budget whose
// allocator owns every byte of the device, a real-time path that must not
// take the implicit device synchronisation an allocation can cause, or a
// plugin called through a C interface that gives it pointers but no allocator.
// Such a caller still passes its own inputs and outputs; only the scratch the
// kernels need between the chunk-local pass and the sequential pass comes from
// here.
//
// The array (`g_gdn_static_scratch`, kStaticScratchBytes) is a file-scope
// __device__ variable: every GPU that loads the library holds it until the
// process exits.  Host code may not pass the symbol itself to a kernel (on the
// host it names a host-side stand-in, not device memory), so the first call on
// each device looks up its device address with cudaGetSymbolAddress while that
// device is current and remembers it, together with the identity of the CUDA
// context it belongs to; a later call in another context (after a device reset,
// say) looks the address up again.  The first call on a device should therefore
// be made before any stream capture begins.
//
// Every call shares the one array.  Its contents carry over from the previous
// call, which is harmless: every byte the kernels read is written earlier in
// the same call (the device status word at its start is zeroed by each call), so
// nothing has to start at zero.  Two calls whose work overlaps on the GPU
// (different streams, no ordering between them) race on the array and give
// wrong results; serialise them.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_gdn_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mu;
struct Cached {
    unsigned long long ctx;  // unique id of the context the address belongs to (0: none)
    void *ptr;
};
Cached g_scratch[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context, or 0 when there is
// none or the driver does not report one (the address is then looked up on
// every call).
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrent)(CUcontext *);
    typedef CUresult (*GetId)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
        cudaGetLastError();
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

gdn_status static_scratch(void **ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDN_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_setup_mu);
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || g_scratch[dev].ctx != ctx || !g_scratch[dev].ptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gdn_static_scratch);
        if (e != cudaSuccess || !p)
            return fail(GDN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_scratch[dev] = Cached{current_context_id(), p};  // (the lookup may have created the context)
    }
    *ptr = g_scratch[dev].ptr;
    return GDN_OK;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" gdn_status gdn_chunk_fwd_static(const gdn_desc *d, const void *q, const void *k, const void *v,
                                           const float *log_gate, const float *beta, const float *initial_state,
                                           const int32_t *cu_seqlens, int32_t num_seqs, int64_t snapshot_stride,
                                           void *out, float *final_state, float *snapshots, gdn_stream_t stream) {
    // Size check first, on the host: a request whose scratch would not fit is
    // rejected before anything touches the device.
    size_t need = 0;
    const int32_t n = cu_seqlens ? num_seqs : (d ? (int32_t)d->B : 0);
    gdn_status st = gdn_chunk_workspace_size(d, n, &need);
    if (st != GDN_OK) return st;
    if (need > kStaticScratchBytes)
        return fail(GDN_ERR_WORKSPACE,
                    "problem needs %zu bytes of scratch; the built-in scratch holds %zu (use gdn_chunk_fwd "
                    "with a caller-provided workspace)",
                    need, kStaticScratchBytes);
    void *ws = nullptr;
    if ((st = static_scratch(&ws)) != GDN_OK) return st;
    return gdn_chunk_fwd(d, q, k, v, log_gate, beta, initial_state, cu_seqlens, num_seqs, snapshot_stride, out,
                         final_state, snapshots, ws, kStaticScratchBytes, stream);
}

extern "C" gdn_status gdn_chunk_status_static(gdn_stream_t stream, int32_t *device_code) {
    void *ws = nullptr;
    const gdn_status st = static_scratch(&ws);
    if (st != GDN_OK) return st;
    return gdn_chunk_status(ws, stream, device_code);
}
