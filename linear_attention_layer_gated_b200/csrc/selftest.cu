// selftest.cu -- exercises the device-side failure path without faulting the GPU.
//
// The kernel runs, with a caller-chosen limit, each kind of bounded wait the prefill and
// decode kernels use, on something that nothing will ever complete: a flag in global memory
// (the one-launch prefill's per-chunk "records complete" flag), a pair of marks (its ring
// slots' "consumed" marks), and an mbarrier phase.  When a wait gives up it records
// GDN_ERR_DEVICE_TIMEOUT's device word in the workspace header, exactly as a stuck kernel
// would, and returns normally, so the CUDA context stays usable.  Nothing here traps, spins
// without a limit or touches invalid memory.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

__global__ void wait_timeout_kernel(int32_t* header, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // header[8], header[10..11]: zero (the caller cleared the header) and written by nothing,
        // so both waits must expire; they run before any error is recorded, which would stop them
        const bool flag_ok = sm100::wait_flag_set(header + 8, nullptr, limit_ns);
        const bool marks_ok = sm100::wait_marks_reach(header + 10, 1, nullptr, limit_ns);
        if (!flag_ok || !marks_ok) atomicOr(header, 1);
    }
    // No thread arrives: phase 0 never completes, so the bounded wait must expire.
    const bool ok = sm100::mbar_wait(&bar, 0, limit_ns);
    if (!ok && threadIdx.x == 0) atomicOr(header, 1);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(void* workspace, uint64_t limit_ns, cudaStream_t stream) {
    wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<int32_t*>(workspace), limit_ns);
    return cudaGetLastError();
}

}  // namespace gdn
