// noalloc.cu -- tensor-core prefill for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point where
// they run a prefill: for example a plugin whose host framework owns every device
// allocation and hands it only fixed input and output buffers, or code that must not
// block on an allocation on its hot path.  gdn_chunk_prefill needs a caller-provided
// workspace; gdn_chunk_prefill_noalloc instead uses a scratch buffer that lives in this
// library's own device memory: a file-scope static __device__ array of
// GDN_NOALLOC_SCRATCH_BYTES bytes.  Every GPU that loads the library holds that array
// until the process exits.
//
// The array's name is only a host-side stand-in in host code, not a device address, so
// the first call on each device (with that device current) looks up its real address
// with cudaGetSymbolAddress and caches it together with the identity of the device's
// current context; later calls in the same context reuse it.  When the context changes
// (cudaDeviceReset, or the primary context released and created again, reloads the
// library's device code, so the array may sit elsewhere) the next call looks the address
// up again.  The first call in a context therefore does a little one-time set-up work and
// should come before any stream capture.
//
// All calls on a device share the one array and it keeps the previous call's contents.
// The prefill clears what must start at zero (the header with the device error word)
// on every call, and everything else is written before it is read.  Calls whose
// executions overlap on the GPU (different streams, no ordering between them) race on
// the array; order them on one stream or with events.
#include <cuda.h>

#include <mutex>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

struct CachedAddress {
    unsigned long long ctx_id;  // unique id of the context the address was taken in
    void* ptr;
};

std::mutex g_mutex;
CachedAddress g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (CUDA 12 context ids are never reused
// within a process), or 0 if the driver cannot tell; 0 makes every call look the address up.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_prefill_scratch on the current device, in its current context.
gdn_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    CachedAddress& c = g_cache[dev];
    unsigned long long id = current_context_id();
    if (!c.ptr || id == 0 || id != c.ctx_id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
        if (id == 0) id = current_context_id();  // the lookup may have created the context
        c.ptr = p;
        c.ctx_id = id;
    }
    *out = c.ptr;
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_chunk_prefill_noalloc(const void* q, const void* k, const void* v,
                                                const float* g, const float* beta,
                                                const float* initial_state,
                                                const int32_t* cu_seqlens, void* out,
                                                float* final_state, const gdn_shape* shape,
                                                void* stream) {
    if (!shape) return GDN_ERR_NULL;
    if (shape->io_dtype != GDN_BF16 || shape->algo == GDN_ALGO_SIMT) return GDN_ERR_UNSUPPORTED;
    const size_t need = gdn_prefill_workspace_bytes(shape);
    if (need == 0) return GDN_ERR_SHAPE;
    if (need > kScratchBytes) return GDN_ERR_WORKSPACE;  // beyond the static maximum
    void* scratch = nullptr;
    const gdn_status st = scratch_address(&scratch);
    if (st != GDN_OK) return st;
    return gdn_chunk_prefill(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, shape,
                             scratch, kScratchBytes, stream);
}

// The device error word of the static scratch: the caller of gdn_chunk_prefill_noalloc
// never sees the array's address, so it cannot pass it to gdn_get_device_error.
extern "C" gdn_status gdn_get_noalloc_device_error(void* stream) {
    void* scratch = nullptr;
    const gdn_status st = scratch_address(&scratch);
    if (st != GDN_OK) return st;
    return gdn_get_device_error(scratch, stream);
}
