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
// with cudaGetSymbolAddress and caches it; later calls on that device reuse it.  That
// first call therefore does a little one-time set-up work and should come before any
// stream capture.
//
// All calls on a device share the one array and it keeps the previous call's contents.
// The prefill clears what must start at zero (the header with the device error word)
// on every call, and everything else is written before it is read.  Calls whose
// executions overlap on the GPU (different streams, no ordering between them) race on
// the array; order them on one stream or with events.
#include <mutex>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_prefill_scratch on the current device (set up once per device).
gdn_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
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
