// decode.cu -- memory-bound decode / multi-token-verify step of the Gated DeltaNet
// layer (gated delta rule; Qwen3-Next-80B-A3B model card, "Model Overview": 16 QK /
// 32 V heads, head dim 128; multi-token prediction serving verifies up to 4 draft
// tokens per step, Qwen3-Next model card "Deployment" and the vLLM blog post,
// "Multi-Token Prediction").
//
// One CTA per (sequence n, V head h) streams that head's 128x128 fp32 state (64 KiB)
// once from HBM and once back, whatever the number of tokens m = 1..4.  The m tokens
// are folded into one pass over the state with the closed form of m consecutive
// updates.  For state row s0 (one d_v index i) with cumulative gate sums
// G_t = g_1 + ... + g_t and Gam_t = exp(G_t):
//
//   x_t = s0 . k_t,  y_t = s0 . q_t                         (2m dot products per row)
//   delta_t = beta_t (v_t[i] - Gam_t x_t - sum_{j<t} exp(G_t - G_j) (k_j . k_t) delta_j)
//   o_t[i]  = Gam_t y_t + sum_{j<=t} exp(G_t - G_j) (k_j . q_t) delta_j
//   s_m     = Gam_m s0 + sum_j exp(G_m - G_j) delta_j k_j
//
// which is the token recurrence unrolled (delta_t is beta_t (v_t - alpha_t S_{t-1} k_t)).
// The k.k and k.q scalars and the gate factors are per (n, h) and computed once per
// CTA.  Each half-warp owns one state row per step: lane l holds columns 4l..4l+3 and
// 64+4l..64+4l+3, so a row is two coalesced 256-byte loads and stores, and the dot
// products reduce over 16 lanes with shuffles.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecodeThreads = 128;  // 4 warps; warp w owns state rows [32w, 32w + 32)
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

__device__ __forceinline__ float dot8(const float* a, const float* b) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) s = fmaf(a[c], b[c], s);
    return s;
}

template <typename IO>
__device__ __forceinline__ void load_cols(const IO* row, int l, float* dst) {
    float4 a = load4(row + 4 * l), b = load4(row + 64 + 4 * l);
    dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
    dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}

template <typename IO, int NTOK, int UNR>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
              const float* __restrict__ g, const float* __restrict__ beta,
              float* __restrict__ state, IO* __restrict__ out, int hk, int hv)
{
    const int n = blockIdx.x / hv;
    const int h = blockIdx.x % hv;
    const int qh = h / (hv / hk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int half = lane >> 4;
    const int l = lane & 15;

    __shared__ float v_s[NTOK][kD];
    __shared__ float o_s[NTOK][kD];

    for (int idx = threadIdx.x; idx < NTOK * kD; idx += kDecodeThreads) {
        const int t = idx / kD, i = idx % kD;
        v_s[t][i] = to_f32(v[(((size_t)n * NTOK + t) * hv + h) * kD + i]);
    }

    // Normalised key / query columns owned by this lane (both half-warps hold the same).
    float kr[NTOK][8], qr[NTOK][8];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) {
        const size_t base = (((size_t)n * NTOK + t) * hk + qh) * kD;
        load_cols(k + base, l, kr[t]);
        load_cols(q + base, l, qr[t]);
        const float rk = rsqrtf(sum16(dot8(kr[t], kr[t])) + kNormEps);
        const float rq = rsqrtf(sum16(dot8(qr[t], qr[t])) + kNormEps) * kInvSqrtD;
#pragma unroll
        for (int c = 0; c < 8; ++c) { kr[t][c] *= rk; qr[t][c] *= rq; }
    }

    // Per-(n, h) scalars: gate sums, decay-weighted k.k and k.q, final weights.
    float G[NTOK], bt[NTOK];
    {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const size_t gi = ((size_t)n * NTOK + t) * hv + h;
            acc += g[gi];
            G[t] = acc;
            bt[t] = beta[gi];
        }
    }
    float Dm[NTOK][NTOK], Em[NTOK][NTOK], Gam[NTOK], F[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) {
        Gam[t] = expf(G[t]);
        F[t] = expf(G[NTOK - 1] - G[t]);
#pragma unroll
        for (int j = 0; j < NTOK; ++j) {
            Dm[t][j] = 0.f;
            Em[t][j] = 0.f;
            if (j < t) Dm[t][j] = expf(G[t] - G[j]) * sum16(dot8(kr[j], kr[t]));
            if (j <= t) Em[t][j] = expf(G[t] - G[j]) * sum16(dot8(kr[j], qr[t]));
        }
    }
    __syncthreads();

    float* S = state + ((size_t)n * hv + h) * kD * kD;
#pragma unroll 1
    for (int p0 = 0; p0 < 16; p0 += UNR) {
        float4 sa[UNR], sb[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = warp * 32 + 2 * (p0 + u) + half;
            sa[u] = __ldcs(reinterpret_cast<const float4*>(S + row * kD + 4 * l));
            sb[u] = __ldcs(reinterpret_cast<const float4*>(S + row * kD + 64 + 4 * l));
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = warp * 32 + 2 * (p0 + u) + half;
            float s[8] = {sa[u].x, sa[u].y, sa[u].z, sa[u].w, sb[u].x, sb[u].y, sb[u].z, sb[u].w};
            float x[NTOK], y[NTOK];
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                x[t] = sum16(dot8(s, kr[t]));
                y[t] = sum16(dot8(s, qr[t]));
            }
            float delta[NTOK];
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                float a = Gam[t] * x[t];
#pragma unroll
                for (int j = 0; j < t; ++j) a = fmaf(Dm[t][j], delta[j], a);
                delta[t] = bt[t] * (v_s[t][row] - a);
                float o = Gam[t] * y[t];
#pragma unroll
                for (int j = 0; j <= t; ++j) o = fmaf(Em[t][j], delta[j], o);
                if (l == 0) o_s[t][row] = o;
            }
            float w[NTOK];
#pragma unroll
            for (int j = 0; j < NTOK; ++j) w[j] = F[j] * delta[j];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float r = Gam[NTOK - 1] * s[c];
#pragma unroll
                for (int j = 0; j < NTOK; ++j) r = fmaf(w[j], kr[j][c], r);
                s[c] = r;
            }
            __stcs(reinterpret_cast<float4*>(S + row * kD + 4 * l), make_float4(s[0], s[1], s[2], s[3]));
            __stcs(reinterpret_cast<float4*>(S + row * kD + 64 + 4 * l), make_float4(s[4], s[5], s[6], s[7]));
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < NTOK * kD; idx += kDecodeThreads) {
        const int t = idx / kD, i = idx % kD;
        out[(((size_t)n * NTOK + t) * hv + h) * kD + i] = from_f32<IO>(o_s[t][i]);
    }
}

template <typename IO>
cudaError_t launch_typed(const IO* q, const IO* k, const IO* v, const float* g,
                         const float* beta, float* state, IO* out, int ntok, int num_seqs,
                         int hk, int hv, cudaStream_t stream)
{
    const dim3 grid((unsigned)num_seqs * (unsigned)hv);
    const dim3 block(kDecodeThreads);
    switch (ntok) {
    case 1: decode_kernel<IO, 1, 4><<<grid, block, 0, stream>>>(q, k, v, g, beta, state, out, hk, hv); break;
    case 2: decode_kernel<IO, 2, 4><<<grid, block, 0, stream>>>(q, k, v, g, beta, state, out, hk, hv); break;
    case 3: decode_kernel<IO, 3, 2><<<grid, block, 0, stream>>>(q, k, v, g, beta, state, out, hk, hv); break;
    default: decode_kernel<IO, 4, 2><<<grid, block, 0, stream>>>(q, k, v, g, beta, state, out, hk, hv); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, void* out, int num_tokens,
                          int num_seqs, int hk, int hv, gdn_dtype io, cudaStream_t stream)
{
    if (num_seqs == 0) return cudaSuccess;
    if (io == GDN_BF16) {
        using T = __nv_bfloat16;
        return launch_typed<T>((const T*)q, (const T*)k, (const T*)v, g, beta, state, (T*)out,
                               num_tokens, num_seqs, hk, hv, stream);
    }
    return launch_typed<float>((const float*)q, (const float*)k, (const float*)v, g, beta, state,
                               (float*)out, num_tokens, num_seqs, hk, hv, stream);
}

}  // namespace gdn
