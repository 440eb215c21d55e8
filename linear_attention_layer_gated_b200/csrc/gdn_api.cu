// gdn_api.cu -- C ABI of libgdn.so: argument validation, workspace sizing and kernel
// dispatch on the caller's stream.  Declarations and contracts are in include/gdn.h.
//
// Nothing here allocates, synchronises or reads device memory inside the prefill and
// decode entry points, so both are stream-ordered and graph-capturable.  On the
// tensor-core prefill path every piece of device work is a kernel (its first kernel
// clears the workspace header); the fp32 path clears the 256-byte header with a memset.
#include <cstdint>
#include <cstring>

#include "gdn_internal.cuh"

namespace {

constexpr size_t kHeaderBytes = 256;  // workspace header: device error word + reserved

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn_status check_common(const gdn_shape* s) {
    if (!s) return GDN_ERR_NULL;
    if (s->io_dtype != GDN_BF16 && s->io_dtype != GDN_F32) return GDN_ERR_DTYPE;
    if (s->head_dim != gdn::kD) return GDN_ERR_SHAPE;
    if (s->num_seqs < 0 || s->num_qk_heads < 1 || s->num_v_heads < 1) return GDN_ERR_SHAPE;
    if (s->num_v_heads % s->num_qk_heads != 0) return GDN_ERR_SHAPE;
    if (s->num_v_heads > 4096) return GDN_ERR_SHAPE;
    return GDN_OK;
}

gdn_status check_prefill_shape(const gdn_shape* s) {
    gdn_status st = check_common(s);
    if (st != GDN_OK) return st;
    if (s->total_tokens < 0 || s->max_seqlen < 0 || s->max_seqlen > s->total_tokens) return GDN_ERR_SHAPE;
    if (s->algo != GDN_ALGO_AUTO && s->algo != GDN_ALGO_SIMT && s->algo != GDN_ALGO_TENSOR) return GDN_ERR_SHAPE;
    if ((int64_t)s->num_seqs * s->num_v_heads * 4 > INT32_MAX) return GDN_ERR_SHAPE;
    return GDN_OK;
}

}  // namespace

extern "C" {

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

const char* gdn_status_string(gdn_status status) {
    switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_NULL: return "GDN_ERR_NULL: a required pointer is NULL";
    case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE: unsupported or inconsistent sizes";
    case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN: device pointer not 16-byte aligned";
    case GDN_ERR_DTYPE: return "GDN_ERR_DTYPE: io_dtype must be GDN_BF16 or GDN_F32";
    case GDN_ERR_NUM_TOKENS: return "GDN_ERR_NUM_TOKENS: decode num_tokens must be in [1, 4]";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA runtime error";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: algorithm not available for these inputs";
    }
    return "unknown gdn_status";
}

// Which kernel family serves a (validated) shape: true = tensor cores.  The tensor-core
// kernels take the V heads in pairs that read one QK head, so they need an even number of V
// heads per QK head; GDN_ALGO_AUTO takes the fp32 kernels otherwise.
static bool tensor_shape_ok(const gdn_shape* s) {
    return s->io_dtype == GDN_BF16 && (s->num_v_heads / s->num_qk_heads) % 2 == 0;
}
static bool use_tensor_path(const gdn_shape* s) {
    if (s->algo == GDN_ALGO_TENSOR) return true;
    if (s->algo == GDN_ALGO_SIMT) return false;
    return tensor_shape_ok(s);
}

size_t gdn_prefill_workspace_bytes(const gdn_shape* shape) {
    if (check_prefill_shape(shape) != GDN_OK) return 0;
    if (use_tensor_path(shape) && tensor_shape_ok(shape)) {
        if (gdn::fused_prefill_applies(shape->num_seqs, shape->total_tokens, shape->num_v_heads))
            return gdn::tc_fused_workspace_bytes(shape->num_seqs, shape->total_tokens, shape->num_qk_heads,
                                                 shape->num_v_heads);
        return gdn::tc_workspace_bytes(shape->num_seqs, shape->total_tokens, shape->num_qk_heads,
                                       shape->num_v_heads);
    }
    return kHeaderBytes;
}

size_t gdn_prefill_phase_workspace_bytes(const gdn_shape* shape) {
    if (check_prefill_shape(shape) != GDN_OK) return 0;
    if (!use_tensor_path(shape) || !tensor_shape_ok(shape)) return 0;
    return gdn::tc_workspace_bytes(shape->num_seqs, shape->total_tokens, shape->num_qk_heads, shape->num_v_heads);
}

}  // extern "C"

namespace {

gdn_status prefill_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                        const float* initial_state, const int32_t* cu_seqlens, void* out, float* final_state,
                        gdn::StateSlots map, float* chunk_states, const gdn_shape* shape, void* workspace,
                        size_t workspace_bytes, gdn::GateAct act, void* stream) {
    gdn_status st = check_prefill_shape(shape);
    if (st != GDN_OK) return st;
    const size_t need = gdn_prefill_workspace_bytes(shape);
    if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGN;
    if (shape->num_seqs == 0) return GDN_OK;
    if (!cu_seqlens) return GDN_ERR_NULL;
    if (shape->total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_NULL;
    const void* ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, chunk_states};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;

    gdn_dtype io = (gdn_dtype)shape->io_dtype;
    const bool tensor = use_tensor_path(shape);
    if (tensor && !tensor_shape_ok(shape)) return GDN_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The tensor-core path's first kernel (the chunk table) clears the device error word
    // itself; the fp32 path's header is cleared here.
    if (!tensor && cudaMemsetAsync(workspace, 0, kHeaderBytes, s) != cudaSuccess) return GDN_ERR_CUDA;
    cudaError_t e;
    if (tensor && gdn::fused_prefill_applies(shape->num_seqs, shape->total_tokens, shape->num_v_heads)) {
        e = gdn::launch_prefill_tc_fused(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, map,
                                         chunk_states, shape->num_seqs, shape->total_tokens, shape->num_qk_heads,
                                         shape->num_v_heads, workspace, act, s);
    } else if (tensor) {
        e = gdn::launch_prefill_tc_prep(q, k, g, beta, cu_seqlens, shape->num_seqs, shape->total_tokens,
                                        shape->num_qk_heads, shape->num_v_heads, workspace, act, s);
        if (e == cudaSuccess)
            e = gdn::launch_prefill_tc_state(k, v, initial_state, cu_seqlens, out, final_state, map, chunk_states,
                                             shape->num_seqs, shape->total_tokens,
                                             shape->num_qk_heads, shape->num_v_heads, workspace, s);
    } else
        e = gdn::launch_prefill_simt(q, k, v, g, beta, initial_state, cu_seqlens, out,
                                     final_state, map, chunk_states, shape->num_seqs, shape->num_qk_heads,
                                     shape->num_v_heads, io, act, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status decode_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       float* state, gdn::StateSlots map, void* out, float* snapshots, int32_t num_tokens,
                       const gdn_shape* shape, gdn::GateAct act, void* stream) {
    gdn_status st = check_common(shape);
    if (st != GDN_OK) return st;
    if (num_tokens < 1 || num_tokens > 4) return GDN_ERR_NUM_TOKENS;
    if ((int64_t)shape->num_seqs * shape->num_v_heads * num_tokens > INT32_MAX) return GDN_ERR_SHAPE;
    if (shape->num_seqs == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !out) return GDN_ERR_NULL;
    const void* ptrs[] = {q, k, v, g, beta, state, out, snapshots, map.slots};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    cudaError_t e = gdn::launch_decode(q, k, v, g, beta, state, map, out, snapshots, num_tokens,
                                       shape->num_seqs, shape->num_qk_heads, shape->num_v_heads,
                                       (gdn_dtype)shape->io_dtype, act, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status commit_impl(float* state, gdn::StateSlots map, const float* snapshots, const int32_t* accepted,
                       int32_t num_tokens, const gdn_shape* shape, void* stream) {
    gdn_status st = check_common(shape);
    if (st != GDN_OK) return st;
    if (num_tokens < 1 || num_tokens > 4) return GDN_ERR_NUM_TOKENS;
    if ((int64_t)shape->num_seqs * shape->num_v_heads > INT32_MAX) return GDN_ERR_SHAPE;
    if (shape->num_seqs == 0) return GDN_OK;
    if (!state || !snapshots || !accepted) return GDN_ERR_NULL;
    const void* ptrs[] = {state, snapshots, accepted, map.slots};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    cudaError_t e = gdn::launch_decode_commit(state, map, snapshots, accepted, num_tokens, shape->num_seqs,
                                              shape->num_v_heads, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

constexpr gdn::StateSlots kDense{nullptr, 0};
constexpr gdn::GateAct kActivated{nullptr, nullptr};  // g and beta are the activated gates

// The raw-gate parameters: both present and aligned like every other device pointer.
gdn_status check_gate_params(const float* a, const float* b) {
    if (!a || !b) return GDN_ERR_NULL;
    if (!aligned16(a) || !aligned16(b)) return GDN_ERR_ALIGN;
    return GDN_OK;
}

gdn_status check_slots(const float* pool, const int32_t* slots, int32_t num_slots) {
    if (!pool || !slots) return GDN_ERR_NULL;
    if (num_slots < 0) return GDN_ERR_SHAPE;
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* initial_state,
                             const int32_t* cu_seqlens, void* out, float* final_state,
                             const gdn_shape* shape, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return prefill_impl(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, kDense, nullptr, shape,
                        workspace, workspace_bytes, kActivated, stream);
}

gdn_status gdn_chunk_prefill_chunk_states(const void* q, const void* k, const void* v, const float* g,
                                          const float* beta, const float* initial_state,
                                          const int32_t* cu_seqlens, void* out, float* final_state,
                                          float* chunk_states, const gdn_shape* shape, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (shape && shape->num_seqs > 0 && shape->total_tokens > 0 && !chunk_states) return GDN_ERR_NULL;
    return prefill_impl(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, kDense, chunk_states,
                        shape, workspace, workspace_bytes, kActivated, stream);
}

gdn_status gdn_chunk_prefill_slots(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, float* state_pool, const int32_t* state_slots,
                                   int32_t num_slots, const int32_t* cu_seqlens, void* out,
                                   const gdn_shape* shape, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    if (shape && shape->num_seqs == 0) return check_prefill_shape(shape);
    gdn_status st = check_slots(state_pool, state_slots, num_slots);
    if (st != GDN_OK) return st;
    return prefill_impl(q, k, v, g, beta, state_pool, cu_seqlens, out, state_pool,
                        gdn::StateSlots{state_slots, num_slots}, nullptr, shape, workspace, workspace_bytes, kActivated,
                        stream);
}

// Shared validation of the two tensor-core prefill phases.
static gdn_status check_phase(const gdn_shape* shape, const int32_t* cu_seqlens, void* workspace,
                              size_t workspace_bytes) {
    gdn_status st = check_prefill_shape(shape);
    if (st != GDN_OK) return st;
    if (!use_tensor_path(shape) || !tensor_shape_ok(shape)) return GDN_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < gdn_prefill_phase_workspace_bytes(shape)) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGN;
    if (shape->num_seqs > 0 && !cu_seqlens) return GDN_ERR_NULL;
    if (cu_seqlens && !aligned16(cu_seqlens)) return GDN_ERR_ALIGN;
    return GDN_OK;
}

gdn_status gdn_chunk_prefill_prep(const void* q, const void* k, const float* g, const float* beta,
                                  const int32_t* cu_seqlens, const gdn_shape* shape, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    gdn_status st = check_phase(shape, cu_seqlens, workspace, workspace_bytes);
    if (st != GDN_OK) return st;
    if (shape->num_seqs == 0) return GDN_OK;
    if (shape->total_tokens > 0 && (!q || !k || !g || !beta)) return GDN_ERR_NULL;
    const void* ptrs[] = {q, k, g, beta};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = gdn::launch_prefill_tc_prep(q, k, g, beta, cu_seqlens, shape->num_seqs, shape->total_tokens,
                                                shape->num_qk_heads, shape->num_v_heads, workspace, kActivated, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_chunk_prefill_state(const void* k, const void* v, const float* initial_state,
                                   const int32_t* cu_seqlens, void* out, float* final_state,
                                   const gdn_shape* shape, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    gdn_status st = check_phase(shape, cu_seqlens, workspace, workspace_bytes);
    if (st != GDN_OK) return st;
    if (shape->num_seqs == 0) return GDN_OK;
    if (shape->total_tokens > 0 && (!k || !v || !out)) return GDN_ERR_NULL;
    const void* ptrs[] = {k, v, initial_state, out, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_ALIGN;
    cudaError_t e = gdn::launch_prefill_tc_state(k, v, initial_state, cu_seqlens, out, final_state, kDense, nullptr,
                                                 shape->num_seqs, shape->total_tokens,
                                                 shape->num_qk_heads, shape->num_v_heads,
                                                 workspace, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, float* state_inout, void* out, int32_t num_tokens,
                           const gdn_shape* shape, void* stream) {
    return decode_impl(q, k, v, g, beta, state_inout, kDense, out, nullptr, num_tokens, shape, kActivated, stream);
}

gdn_status gdn_decode_verify(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* state, void* out, float* snapshots,
                             int32_t num_tokens, const gdn_shape* shape, void* stream) {
    if (shape && shape->num_seqs > 0 && !snapshots) return GDN_ERR_NULL;
    return decode_impl(q, k, v, g, beta, const_cast<float*>(state), kDense, out, snapshots, num_tokens,
                       shape, kActivated, stream);
}

gdn_status gdn_chunk_prefill_raw_gates(const void* q, const void* k, const void* v, const float* x,
                                       const float* y, const float* a, const float* b,
                                       const float* initial_state, const int32_t* cu_seqlens, void* out,
                                       float* final_state, const gdn_shape* shape, void* workspace,
                                       size_t workspace_bytes, void* stream) {
    if (shape && shape->num_seqs > 0 && shape->total_tokens > 0) {
        gdn_status st = check_gate_params(a, b);
        if (st != GDN_OK) return st;
    }
    return prefill_impl(q, k, v, x, y, initial_state, cu_seqlens, out, final_state, kDense, nullptr, shape,
                        workspace, workspace_bytes, gdn::GateAct{a, b}, stream);
}

gdn_status gdn_decode_step_raw_gates(const void* q, const void* k, const void* v, const float* x,
                                     const float* y, const float* a, const float* b, float* state_inout,
                                     void* out, int32_t num_tokens, const gdn_shape* shape, void* stream) {
    if (shape && shape->num_seqs > 0) {
        gdn_status st = check_gate_params(a, b);
        if (st != GDN_OK) return st;
    }
    return decode_impl(q, k, v, x, y, state_inout, kDense, out, nullptr, num_tokens, shape, gdn::GateAct{a, b},
                       stream);
}

gdn_status gdn_decode_verify_raw_gates(const void* q, const void* k, const void* v, const float* x,
                                       const float* y, const float* a, const float* b, const float* state,
                                       void* out, float* snapshots, int32_t num_tokens, const gdn_shape* shape,
                                       void* stream) {
    if (shape && shape->num_seqs > 0) {
        gdn_status st = check_gate_params(a, b);
        if (st != GDN_OK) return st;
        if (!snapshots) return GDN_ERR_NULL;
    }
    return decode_impl(q, k, v, x, y, const_cast<float*>(state), kDense, out, snapshots, num_tokens, shape,
                       gdn::GateAct{a, b}, stream);
}

gdn_status gdn_decode_commit(float* state, const float* snapshots, const int32_t* accepted,
                             int32_t num_tokens, const gdn_shape* shape, void* stream) {
    return commit_impl(state, kDense, snapshots, accepted, num_tokens, shape, stream);
}

gdn_status gdn_decode_step_slots(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float* state_pool, const int32_t* state_slots,
                                 int32_t num_slots, void* out, int32_t num_tokens, const gdn_shape* shape,
                                 void* stream) {
    if (shape && shape->num_seqs > 0) {
        gdn_status st = check_slots(state_pool, state_slots, num_slots);
        if (st != GDN_OK) return st;
    }
    return decode_impl(q, k, v, g, beta, state_pool, gdn::StateSlots{state_slots, num_slots}, out, nullptr,
                       num_tokens, shape, kActivated, stream);
}

gdn_status gdn_decode_verify_slots(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* state_pool, const int32_t* state_slots,
                                   int32_t num_slots, void* out, float* snapshots, int32_t num_tokens,
                                   const gdn_shape* shape, void* stream) {
    if (shape && shape->num_seqs > 0) {
        gdn_status st = check_slots(state_pool, state_slots, num_slots);
        if (st != GDN_OK) return st;
        if (!snapshots) return GDN_ERR_NULL;
    }
    return decode_impl(q, k, v, g, beta, const_cast<float*>(state_pool), gdn::StateSlots{state_slots, num_slots},
                       out, snapshots, num_tokens, shape, kActivated, stream);
}

gdn_status gdn_decode_commit_slots(float* state_pool, const int32_t* state_slots, int32_t num_slots,
                                   const float* snapshots, const int32_t* accepted, int32_t num_tokens,
                                   const gdn_shape* shape, void* stream) {
    if (shape && shape->num_seqs > 0) {
        gdn_status st = check_slots(state_pool, state_slots, num_slots);
        if (st != GDN_OK) return st;
    }
    return commit_impl(state_pool, gdn::StateSlots{state_slots, num_slots}, snapshots, accepted, num_tokens,
                       shape, stream);
}

gdn_status gdn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                      void* stream) {
    if (!workspace) return GDN_ERR_NULL;
    if (workspace_bytes < kHeaderBytes) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_ALIGN;
    if (limit_us < 1 || limit_us > 2000000) return GDN_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, s) != cudaSuccess) return GDN_ERR_CUDA;
    cudaError_t e = gdn::launch_wait_timeout_selftest(workspace, (uint64_t)limit_us * 1000u, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_get_device_error(void* workspace, void* stream) {
    if (!workspace) return GDN_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    int32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    return word != 0 ? GDN_ERR_DEVICE_TIMEOUT : GDN_OK;
}

}  // extern "C"
