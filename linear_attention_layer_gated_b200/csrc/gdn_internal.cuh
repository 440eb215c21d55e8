// gdn_internal.cuh -- shared device helpers and internal launcher declarations of
// libgdn.so.  Not part of the public ABI (that is include/gdn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

constexpr int kD = 128;       // head dimension (d_k = d_v), Qwen3-Next model card "Model Overview"
constexpr int kChunk = 64;    // tokens per chunk of the chunked form
constexpr float kNormEps = 1e-6f;  // x / sqrt(sum(x^2) + eps)

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Loads 4 consecutive elements (16-byte aligned for fp32, 8-byte for bf16) as fp32.
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// ---------------------------------------------------------------- state addressing
// States are either dense ([N][HV][D][D], state of sequence n at index n) or held in a
// pool indexed through a slot table: sequence n's state is pool[slots[n]].  A slot outside
// [0, num_slots) marks a sequence without a state (decode skips it; prefill starts it from
// zeros and writes no final state).
struct StateSlots {
    const int32_t* slots;  // nullptr: dense
    int num_slots;
};
__device__ __forceinline__ int state_index(const StateSlots& m, int n, bool& valid) {
    if (!m.slots) { valid = true; return n; }
    const int s = m.slots[n];
    valid = s >= 0 && s < m.num_slots;
    return valid ? s : 0;
}

// ---------------------------------------------------------------- gates
// Gates given as raw projections (the *_raw_gates entry points): when `a` is non-null the g
// and beta arrays hold the raw projections x and y, and every kernel applies, per V head h,
// g = -a[h] * softplus(x + b[h]) and beta = sigmoid(y) where it loads them.  With `a` null
// they are the activated gates and are used as they are.
struct GateAct {
    const float* a;  // [HV] decay rates (> 0), or nullptr
    const float* b;  // [HV] biases of the decay projection
};
__device__ __forceinline__ float softplus_f32(float z) {  // log(1 + e^z) without overflow
    return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z)));
}
__device__ __forceinline__ float act_g(float x, float a, float b) { return -a * softplus_f32(x + b); }
__device__ __forceinline__ float act_beta(float y) { return 1.f / (1.f + expf(-y)); }
__device__ __forceinline__ float load_g(const float* g, size_t idx, const GateAct& act, int h) {
    const float x = g[idx];
    return act.a ? act_g(x, act.a[h], act.b[h]) : x;
}
__device__ __forceinline__ float load_beta(const float* beta, size_t idx, const GateAct& act) {
    const float y = beta[idx];
    return act.a ? act_beta(y) : y;
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments were validated by the caller.
// snap == nullptr: decode step in place; otherwise verify (state read only, per-token
// states to snap).
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, StateSlots map, void* out, float* snap,
                          int num_tokens, int num_seqs, int hk, int hv, gdn_dtype io, GateAct act,
                          cudaStream_t stream);
cudaError_t launch_decode_commit(float* state, StateSlots map, const float* snap, const int32_t* accepted,
                                 int num_tokens, int num_seqs, int hv, cudaStream_t stream);

cudaError_t launch_prefill_simt(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* s0, const int32_t* cu,
                                void* out, float* sT, StateSlots map, float* cstates, int num_seqs, int hk,
                                int hv, gdn_dtype io, GateAct act, cudaStream_t stream);

// Tensor-core prefill (bf16 I/O, num_v_heads / num_qk_heads even): total workspace bytes
// (header included) and launch.
size_t tc_workspace_bytes(int num_seqs, int total_tokens, int hk, int hv);
// The one-launch pass's smaller workspace: its records live in a ring of a few chunks.
size_t tc_fused_workspace_bytes(int num_seqs, int total_tokens, int hk, int hv);
// Phase 1 (chunk table + per-chunk coefficient images, from q, k and the gates) and phase 2
// (state pass, from k, v and the images).
cudaError_t launch_prefill_tc_prep(const void* q, const void* k, const float* g, const float* beta,
                                   const int32_t* cu, int num_seqs, int total_tokens, int hk, int hv,
                                   void* workspace, GateAct act, cudaStream_t stream);
// cstates (nullable): the state after every chunk, [total chunks][HV][D][D], chunks in
// sequence order.
cudaError_t launch_prefill_tc_state(const void* k, const void* v, const float* s0, const int32_t* cu, void* out,
                                    float* sT, StateSlots map, float* cstates, int num_seqs, int total_tokens, int hk,
                                    int hv, void* workspace, cudaStream_t stream);

// Both phases in one cooperative launch (the state passes wait per chunk for the prep
// workers of the same launch); applies when the (sequence, V head) chains fill at most half of
// the SMs and the device supports cooperative launches.
bool fused_prefill_applies(int num_seqs, int total_tokens, int hv);
cudaError_t launch_prefill_tc_fused(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                   const float* s0, const int32_t* cu, void* out, float* sT, StateSlots map,
                                   float* cstates, int num_seqs, int total_tokens, int hk, int hv, void* workspace,
                                   GateAct act, cudaStream_t stream);

// Diagnostic: a bounded wait that is guaranteed to expire (failure-path self-test).
cudaError_t launch_wait_timeout_selftest(void* workspace, uint64_t limit_ns, cudaStream_t stream);

}  // namespace gdn
