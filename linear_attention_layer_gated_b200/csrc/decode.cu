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
// CTA.
//
// Memory: at entry every warp issues asynchronous 16-byte copies (cp.async, no waits
// that could spin) of its 32 state rows into shared memory, so a CTA has its whole
// 64 KiB head in flight before it does anything else; three CTAs fit on an SM.
// Compute: a half-warp takes R rows at a time; lane l holds columns 4l..4l+3 and
// 64+4l..64+4l+3 of each.  The 2m dot products of R rows (16 partial sums per lane)
// are reduced over the 16 lanes with a transposing butterfly -- each exchange step
// sends half of the remaining sums and keeps the other half -- so 15 shuffles leave
// lane l with the complete sum number l, instead of 4 shuffles per sum.  The 16 sums
// go through shared memory to every lane of the half-warp, each lane evaluates the
// scalar recurrence for the R rows, and the new rows are streamed to HBM.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecodeThreads = 128;  // 4 warps; warp w owns state rows [32w, 32w + 32)
constexpr int kRowsPerWarp = kD / 4;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)
constexpr size_t kStateSmemBytes = (size_t)kD * kD * sizeof(float);  // 64 KiB

__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

// A lane's 8 columns are kept as 4 float2 pairs so that the products run on the packed
// two-wide fp32 FMA of sm_100 (__ffma2_rn): half the instructions of scalar FMAs.
__device__ __forceinline__ float dot8(const float2* a, const float2* b) {
    float2 acc = __fmul2_rn(a[0], b[0]);
    acc = __ffma2_rn(a[1], b[1], acc);
    acc = __ffma2_rn(a[2], b[2], acc);
    acc = __ffma2_rn(a[3], b[3], acc);
    return acc.x + acc.y;
}

template <typename IO>
__device__ __forceinline__ void load_cols(const IO* row, int l, float2* dst) {
    float4 a = load4(row + 4 * l), b = load4(row + 64 + 4 * l);
    dst[0] = make_float2(a.x, a.y); dst[1] = make_float2(a.z, a.w);
    dst[2] = make_float2(b.x, b.y); dst[3] = make_float2(b.z, b.w);
}

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Transposing butterfly over the 16 lanes of a half-warp.  On entry a[0..CUR) are this
// lane's partial sums of CUR quantities; each level with CUR >= 2 swaps half of them
// with the partner lane (l ^ M) and keeps the other half, adding the partner's copy.
// On exit (16 quantities) lane l holds in a[0] the full sum of quantity number l.
template <int CUR, int M>
__device__ __forceinline__ void xpose_reduce(float* a, int l) {
    if constexpr (M > 0) {
        static_assert(CUR >= 2, "needs at least as many quantities as lanes");
        const bool up = (l & M) != 0;
#pragma unroll
        for (int i = 0; i < CUR / 2; ++i) {
            const float send = up ? a[i] : a[i + CUR / 2];
            const float keep = up ? a[i + CUR / 2] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
        }
        xpose_reduce<CUR / 2, M / 2>(a, l);
    }
}

// NTOK tokens of one step; R rows per half-warp per iteration, with 2 * NT * R == 16
// partial sums per lane (NT = NTOK rounded up to a power of two; a padding slot is 0).
// SNAP = false: the state after the last token overwrites `state` in place.
// SNAP = true (speculative verify): `state` is only read; the state after each token t,
//   s_t = Gam_t s0 + sum_{j<=t} exp(G_t - G_j) delta_j k_j (the same closed form), goes to
//   snap[n][t][h] ([N][NTOK][HV][D][D] fp32).
template <typename IO, int NTOK, int R, bool SNAP>
__global__ void __launch_bounds__(kDecodeThreads, 3)
decode_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
              const float* __restrict__ g, const float* __restrict__ beta,
              float* __restrict__ state, StateSlots map, IO* __restrict__ out, float* __restrict__ snap,
              int hk, int hv)
{
    constexpr int NT = NTOK == 3 ? 4 : NTOK;
    constexpr int VR = 2 * NT;           // sums per row: x_0..x_{NT-1}, y_0..y_{NT-1}
    static_assert(VR * R == 16, "one sum per lane after the butterfly");
    constexpr int kRowsPerIter = 2 * R;  // both half-warps
    constexpr int kIters = kRowsPerWarp / kRowsPerIter;
    constexpr int kGroups = kIters < 4 ? kIters : 4;  // cp.async groups per warp
    constexpr int kItersPerGroup = kIters / kGroups;
    constexpr int kRowsPerGroup = kRowsPerWarp / kGroups;

    const int n = blockIdx.x / hv;
    const int h = blockIdx.x % hv;
    const int qh = h / (hv / hk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int half = lane >> 4;
    const int l = lane & 15;

    extern __shared__ __align__(16) float s_state[];  // [kD][kD], row-major like HBM
    __shared__ float v_s[NTOK][kD];
    __shared__ float o_s[NTOK][kD];
    __shared__ __align__(16) float red_s[2][4][2][16];  // [parity][warp][half][sum]

    bool has_state;
    const int sidx = state_index(map, n, has_state);
    if (!has_state) return;  // a sequence without a state slot is skipped (whole CTA)
    float* S = state + ((size_t)sidx * hv + h) * kD * kD;

    // 1. This warp's 32 rows start moving HBM -> shared memory immediately.
#pragma unroll
    for (int grp = 0; grp < kGroups; ++grp) {
#pragma unroll
        for (int j = 0; j < kRowsPerGroup; ++j) {
            const int row = warp * kRowsPerWarp + grp * kRowsPerGroup + j;
            cp_async16(s_state + row * kD + 4 * lane, S + row * kD + 4 * lane);
        }
        cp_async_commit();
    }

    // 2. Per-(n, h) inputs while the state is in flight.
    for (int idx = threadIdx.x; idx < NTOK * kD; idx += kDecodeThreads) {
        const int t = idx / kD, i = idx % kD;
        v_s[t][i] = to_f32(v[(((size_t)n * NTOK + t) * hv + h) * kD + i]);
    }
    float2 kr[NTOK][4], qr[NTOK][4];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) {
        const size_t base = (((size_t)n * NTOK + t) * hk + qh) * kD;
        load_cols(k + base, l, kr[t]);
        load_cols(q + base, l, qr[t]);
        const float rk = rsqrtf(sum16(dot8(kr[t], kr[t])) + kNormEps);
        const float rq = rsqrtf(sum16(dot8(qr[t], qr[t])) + kNormEps) * kInvSqrtD;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            kr[t][c] = __fmul2_rn(kr[t][c], make_float2(rk, rk));
            qr[t][c] = __fmul2_rn(qr[t][c], make_float2(rq, rq));
        }
    }
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
    float Dm[NTOK][NTOK], Em[NTOK][NTOK], Et[NTOK][NTOK], Gam[NTOK];
#pragma unroll
    for (int t = 0; t < NTOK; ++t) {
        Gam[t] = expf(G[t]);
#pragma unroll
        for (int j = 0; j < NTOK; ++j) {
            Dm[t][j] = 0.f;
            Em[t][j] = 0.f;
            Et[t][j] = (j <= t) ? expf(G[t] - G[j]) : 0.f;  // decay from token j to token t
            if (j < t) Dm[t][j] = Et[t][j] * sum16(dot8(kr[j], kr[t]));
            if (j <= t) Em[t][j] = Et[t][j] * sum16(dot8(kr[j], qr[t]));
        }
    }
    __syncthreads();  // v_s

    // 3. Rows, group by group as their copies land.
#pragma unroll
    for (int grp = 0; grp < kGroups; ++grp) {
        if (grp == 0) cp_async_wait<kGroups - 1>();
        else if (grp == 1) cp_async_wait<(kGroups > 1 ? kGroups - 2 : 0)>();
        else if (grp == 2) cp_async_wait<(kGroups > 2 ? kGroups - 3 : 0)>();
        else cp_async_wait<0>();
        __syncwarp();  // every lane's copies of this group are visible to the warp
#pragma unroll 1
        for (int it = grp * kItersPerGroup; it < (grp + 1) * kItersPerGroup; ++it) {
            const int row0 = warp * kRowsPerWarp + it * kRowsPerIter + half * R;
            float2 s[R][4];
            float a[16];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                load_cols(s_state + (row0 + r) * kD, l, s[r]);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    a[r * VR + t] = t < NTOK ? dot8(s[r], kr[t < NTOK ? t : 0]) : 0.f;
                    a[r * VR + NT + t] = t < NTOK ? dot8(s[r], qr[t < NTOK ? t : 0]) : 0.f;
                }
            }
            xpose_reduce<16, 8>(a, l);
            float* red = red_s[it & 1][warp][half];
            red[l] = a[0];
            __syncwarp();
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float xy[VR];
#pragma unroll
                for (int c4 = 0; c4 < VR; c4 += 4) {
                    const float4 u = *reinterpret_cast<const float4*>(red + r * VR + c4);
                    xy[c4] = u.x; xy[c4 + 1] = u.y; xy[c4 + 2] = u.z; xy[c4 + 3] = u.w;
                }
                const int row = row0 + r;
                float delta[NTOK];
#pragma unroll
                for (int t = 0; t < NTOK; ++t) {
                    float x = Gam[t] * xy[t];
#pragma unroll
                    for (int j = 0; j < t; ++j) x = fmaf(Dm[t][j], delta[j], x);
                    delta[t] = bt[t] * (v_s[t][row] - x);
                    float o = Gam[t] * xy[NT + t];
#pragma unroll
                    for (int j = 0; j <= t; ++j) o = fmaf(Em[t][j], delta[j], o);
                    if (l == 0) o_s[t][row] = o;
                }
                if constexpr (SNAP) {
#pragma unroll
                    for (int t = 0; t < NTOK; ++t) {
                        float2 w[NTOK];
#pragma unroll
                        for (int j = 0; j <= t; ++j) w[j] = make_float2(Et[t][j] * delta[j], Et[t][j] * delta[j]);
                        const float2 gt = make_float2(Gam[t], Gam[t]);
                        float2 y[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            y[c] = __fmul2_rn(gt, s[r][c]);
#pragma unroll
                            for (int j = 0; j <= t; ++j) y[c] = __ffma2_rn(w[j], kr[j][c], y[c]);
                        }
                        float* St = snap + (((size_t)n * NTOK + t) * hv + h) * kD * kD + row * kD;
                        __stcs(reinterpret_cast<float4*>(St + 4 * l), make_float4(y[0].x, y[0].y, y[1].x, y[1].y));
                        __stcs(reinterpret_cast<float4*>(St + 64 + 4 * l), make_float4(y[2].x, y[2].y, y[3].x, y[3].y));
                    }
                } else {
                    float2 w[NTOK];
#pragma unroll
                    for (int j = 0; j < NTOK; ++j)
                        w[j] = make_float2(Et[NTOK - 1][j] * delta[j], Et[NTOK - 1][j] * delta[j]);
                    const float2 gl = make_float2(Gam[NTOK - 1], Gam[NTOK - 1]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float2 y = __fmul2_rn(gl, s[r][c]);
#pragma unroll
                        for (int j = 0; j < NTOK; ++j) y = __ffma2_rn(w[j], kr[j][c], y);
                        s[r][c] = y;
                    }
                    __stcs(reinterpret_cast<float4*>(S + row * kD + 4 * l),
                           make_float4(s[r][0].x, s[r][0].y, s[r][1].x, s[r][1].y));
                    __stcs(reinterpret_cast<float4*>(S + row * kD + 64 + 4 * l),
                           make_float4(s[r][2].x, s[r][2].y, s[r][3].x, s[r][3].y));
                }
            }
        }
    }
    __syncthreads();  // o_s
    for (int idx = threadIdx.x; idx < NTOK * kD; idx += kDecodeThreads) {
        const int t = idx / kD, i = idx % kD;
        out[(((size_t)n * NTOK + t) * hv + h) * kD + i] = from_f32<IO>(o_s[t][i]);
    }
}

template <typename IO, int NTOK, int R, bool SNAP>
cudaError_t launch_one(const IO* q, const IO* k, const IO* v, const float* g, const float* beta,
                       float* state, StateSlots map, IO* out, float* snap, int num_seqs, int hk, int hv,
                       cudaStream_t stream)
{
    auto kernel = decode_kernel<IO, NTOK, R, SNAP>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<dim3((unsigned)num_seqs * (unsigned)hv), dim3(kDecodeThreads), kStateSmemBytes,
             stream>>>(q, k, v, g, beta, state, map, out, snap, hk, hv);
    return cudaGetLastError();
}

template <typename IO, bool SNAP>
cudaError_t launch_typed(const IO* q, const IO* k, const IO* v, const float* g,
                         const float* beta, float* state, StateSlots map, IO* out, float* snap, int ntok,
                         int num_seqs, int hk, int hv, cudaStream_t stream)
{
    switch (ntok) {
    case 1: return launch_one<IO, 1, 8, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, stream);
    case 2: return launch_one<IO, 2, 4, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, stream);
    case 3: return launch_one<IO, 3, 2, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, stream);
    default: return launch_one<IO, 4, 2, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, stream);
    }
}

// Commit of a verify step: state[n][h] <- snap[n][accepted[n] - 1][h] for accepted[n] in
// 1..ntok; any other count leaves the state as it was.  One CTA per (n, h), 64 KiB each.
__global__ void __launch_bounds__(kDecodeThreads)
commit_kernel(float* __restrict__ state, StateSlots map, const float* __restrict__ snap,
              const int32_t* __restrict__ accepted, int ntok, int hv)
{
    const int n = blockIdx.x / hv, h = blockIdx.x % hv;
    const int acc = accepted[n];
    bool has_state;
    const int sidx = state_index(map, n, has_state);
    if (acc < 1 || acc > ntok || !has_state) return;
    const float4* src = reinterpret_cast<const float4*>(snap + (((size_t)n * ntok + acc - 1) * hv + h) * kD * kD);
    float4* dst = reinterpret_cast<float4*>(state + ((size_t)sidx * hv + h) * kD * kD);
#pragma unroll 4
    for (int i = threadIdx.x; i < kD * kD / 4; i += kDecodeThreads) __stcs(dst + i, __ldcs(src + i));
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, StateSlots map, void* out, float* snap,
                          int num_tokens, int num_seqs, int hk, int hv, gdn_dtype io, cudaStream_t stream)
{
    if (num_seqs == 0) return cudaSuccess;
    if (io == GDN_BF16) {
        using T = __nv_bfloat16;
        if (snap)
            return launch_typed<T, true>((const T*)q, (const T*)k, (const T*)v, g, beta, state, map, (T*)out, snap,
                                         num_tokens, num_seqs, hk, hv, stream);
        return launch_typed<T, false>((const T*)q, (const T*)k, (const T*)v, g, beta, state, map, (T*)out, nullptr,
                                      num_tokens, num_seqs, hk, hv, stream);
    }
    if (snap)
        return launch_typed<float, true>((const float*)q, (const float*)k, (const float*)v, g, beta, state,
                                         map, (float*)out, snap, num_tokens, num_seqs, hk, hv, stream);
    return launch_typed<float, false>((const float*)q, (const float*)k, (const float*)v, g, beta, state,
                                      map, (float*)out, nullptr, num_tokens, num_seqs, hk, hv, stream);
}

cudaError_t launch_decode_commit(float* state, StateSlots map, const float* snap, const int32_t* accepted,
                                 int num_tokens, int num_seqs, int hv, cudaStream_t stream)
{
    if (num_seqs == 0) return cudaSuccess;
    commit_kernel<<<dim3((unsigned)num_seqs * (unsigned)hv), dim3(kDecodeThreads), 0, stream>>>(
        state, map, snap, accepted, num_tokens, hv);
    return cudaGetLastError();
}

}  // namespace gdn
