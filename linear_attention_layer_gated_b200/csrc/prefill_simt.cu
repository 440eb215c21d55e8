// prefill_simt.cu -- chunked prefill of the Gated DeltaNet layer on CUDA cores, fp32.
//
// This is the fp32-accurate path (fp32 I/O) and the correctness baseline for bf16 I/O.
// It evaluates the chunked form of the gated delta rule (chunks of 64 tokens) entirely
// in fp32 FFMA; the tensor-core path (prefill_tc.cu) evaluates the same algebra with
// bf16 operands.
//
// Chunked form, one chunk of L <= 64 tokens entering with state S (d_v x d_k), rows
// of Q, K, V are the chunk's normalised queries, keys and values, and
// G_r = g_1 + ... + g_r is the in-chunk inclusive gate sum:
//   A[r][j] = b_r exp(G_r - G_j) (k_r . k_j)   for j < r          (strictly lower)
//   P[r][j] =     exp(G_r - G_j) (q_r . k_j)   for j <= r
//   T = (I + A)^-1                       (unit lower triangular, forward substitution)
//   W = T diag(b gam) K,  U = T diag(b) V,  gam_r = exp(G_r)
//   Delta = U - W S^T                    (the chunk's delta-rule corrections)
//   O = diag(gam) Q S^T + P Delta        (outputs; read the post-update state)
//   S <- gam_L S + Delta^T diag(c) K,    c_j = exp(G_L - G_j)
// Decays are formed as exp(G_r - G_j) with r >= j only, never as ratios.
//
// One CTA per (sequence, V head, 32-wide d_v slice): the rows of S evolve
// independently, so four CTAs share a head and each carries a 32 x 128 slice of the
// state across all chunks of its sequence.  Each CTA recomputes the slice-independent
// chunk quantities (normalisation, A, P, T, W) for its head.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSlice = 32;            // d_v rows of S per CTA
constexpr int kSlices = kD / kSlice;  // 4
constexpr int kLdK = kD + 1;          // padded fp32 row strides (bank-conflict free)
constexpr int kLdC = kChunk + 1;
constexpr int kLdS = kSlice + 1;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

struct SimtSmem {
    float Kn[kChunk][kLdK];   // normalised keys
    float Qn[kChunk][kLdK];   // normalised, scaled queries
    float W[kChunk][kLdK];
    float St[kSlice][kLdK];   // state slice: rows = d_v index, cols = d_k index
    float A[kChunk][kLdC];    // A, then T = (I + A)^-1 in place
    float P[kChunk][kLdC];
    float V[kChunk][kLdS];    // V slice, then U, then Delta
    float G[kChunk], b[kChunk], gam[kChunk], c[kChunk];
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_inclusive_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

template <typename IO>
__global__ void __launch_bounds__(kSimtThreads, 1)
prefill_simt_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                    const float* __restrict__ g, const float* __restrict__ beta,
                    const float* s0, const int32_t* __restrict__ cu, IO* __restrict__ out,
                    float* sT, StateSlots map, float* cstates, int hk, int hv, GateAct act)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);

    const int slice = blockIdx.x % kSlices;
    const int h = (blockIdx.x / kSlices) % hv;
    const int n = blockIdx.x / (kSlices * hv);
    const int qh = h / (hv / hk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ty = tid / 16, tx = tid % 16;
    const int cv0 = slice * kSlice;
    const int seq_begin = cu[n], seq_end = cu[n + 1];
    bool has_state;
    const int sidx = state_index(map, n, has_state);
    if (!has_state) { s0 = nullptr; sT = nullptr; }  // no slot: start from zeros, keep no state
    const size_t state_base = ((size_t)sidx * hv + h) * kD * kD + (size_t)cv0 * kD;

    for (int idx = tid; idx < kSlice * kD; idx += kSimtThreads) {
        const int i = idx / kD, j = idx % kD;
        sm.St[i][j] = s0 ? s0[state_base + (size_t)i * kD + j] : 0.f;
    }

    // Chunk-end states (optional): chunk c of sequence n goes to row chunk0 + c of
    // cstates, chunk0 = sum over earlier sequences of their chunk counts.
    __shared__ int s_chunk0;
    if (cstates) {
        int part = 0;
        for (int m = tid; m < n; m += kSimtThreads) part += (cu[m + 1] - cu[m] + kChunk - 1) / kChunk;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (tid == 0) s_chunk0 = 0;
        __syncthreads();
        if (lane == 0) atomicAdd(&s_chunk0, part);
    }
    int chunk_no = 0;

    for (int t0 = seq_begin; t0 < seq_end; t0 += kChunk, ++chunk_no) {
        const int L = min(kChunk, seq_end - t0);
        __syncthreads();

        // ---- 1. load, normalise (rows >= L are zero)
        for (int r = warp; r < kChunk; r += kSimtThreads / 32) {
            float kv[4] = {0.f, 0.f, 0.f, 0.f}, qv[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < L) {
                const size_t base = ((size_t)(t0 + r) * hk + qh) * kD + 4 * lane;
                const float4 a = load4(k + base), bq = load4(q + base);
                kv[0] = a.x; kv[1] = a.y; kv[2] = a.z; kv[3] = a.w;
                qv[0] = bq.x; qv[1] = bq.y; qv[2] = bq.z; qv[3] = bq.w;
            }
            const float rk = rsqrtf(warp_sum(kv[0] * kv[0] + kv[1] * kv[1] + kv[2] * kv[2] + kv[3] * kv[3]) + kNormEps);
            const float rq = rsqrtf(warp_sum(qv[0] * qv[0] + qv[1] * qv[1] + qv[2] * qv[2] + qv[3] * qv[3]) + kNormEps) * kInvSqrtD;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sm.Kn[r][4 * lane + e] = kv[e] * rk;
                sm.Qn[r][4 * lane + e] = qv[e] * rq;
            }
        }
        for (int idx = tid; idx < kChunk * kSlice; idx += kSimtThreads) {
            const int r = idx / kSlice, cc = idx % kSlice;
            sm.V[r][cc] = (r < L) ? to_f32(v[((size_t)(t0 + r) * hv + h) * kD + cv0 + cc]) : 0.f;
        }
        if (warp == 0) {
            const float g0 = (lane < L) ? load_g(g, (size_t)(t0 + lane) * hv + h, act, h) : 0.f;
            const float g1 = (lane + 32 < L) ? load_g(g, (size_t)(t0 + lane + 32) * hv + h, act, h) : 0.f;
            const float G0 = warp_inclusive_scan(g0, lane);
            const float G1 = warp_inclusive_scan(g1, lane) + __shfl_sync(0xffffffffu, G0, 31);
            sm.G[lane] = G0;
            sm.G[lane + 32] = G1;   // rows >= L repeat the last sum (their g is 0)
            sm.b[lane] = (lane < L) ? load_beta(beta, (size_t)(t0 + lane) * hv + h, act) : 0.f;
            sm.b[lane + 32] = (lane + 32 < L) ? load_beta(beta, (size_t)(t0 + lane + 32) * hv + h, act) : 0.f;
        }
        __syncthreads();
        if (tid < kChunk) {
            const float Gl = sm.G[L - 1];
            sm.gam[tid] = expf(sm.G[tid]);
            sm.c[tid] = (tid < L) ? expf(Gl - sm.G[tid]) : 0.f;
        }

        // ---- 2. Gram matrices and decay masks: A (strictly lower), P (lower)
        {
            float kk[4][4], qk[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) { kk[i][jj] = 0.f; qk[i][jj] = 0.f; }
#pragma unroll 4
            for (int cc = 0; cc < kD; ++cc) {
                float kr[4], qr[4], kj[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) { kr[i] = sm.Kn[ty + 16 * i][cc]; qr[i] = sm.Qn[ty + 16 * i][cc]; }
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) kj[jj] = sm.Kn[tx + 16 * jj][cc];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        kk[i][jj] = fmaf(kr[i], kj[jj], kk[i][jj]);
                        qk[i][jj] = fmaf(qr[i], kj[jj], qk[i][jj]);
                    }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = ty + 16 * i;
                const float Gr = sm.G[r], br = sm.b[r];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = tx + 16 * jj;
                    const float dec = (j <= r) ? expf(Gr - sm.G[j]) : 0.f;
                    sm.A[r][j] = (j < r) ? br * dec * kk[i][jj] : 0.f;
                    sm.P[r][j] = dec * qk[i][jj];
                }
            }
        }
        __syncthreads();

        // ---- 3. T = (I + A)^-1, one column per thread (forward substitution)
        {
            float x[kChunk];
            if (tid < kChunk) {
#pragma unroll
                for (int r = 0; r < kChunk; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < r; ++j) acc = fmaf(sm.A[r][j], x[j], acc);
                    x[r] = (r == tid) ? 1.f : ((r < tid) ? 0.f : -acc);
                }
            }
            __syncthreads();
            if (tid < kChunk) {
#pragma unroll
                for (int r = 0; r < kChunk; ++r) sm.A[r][tid] = x[r];
            }
        }
        __syncthreads();

        // ---- 4. W = T diag(b gam) K  (64 x 128),  U = T diag(b) V  (64 x 32)
        {
            float w[4][8], u[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) w[i][cc] = 0.f;
                u[i][0] = 0.f; u[i][1] = 0.f;
            }
#pragma unroll 2
            for (int j = 0; j < kChunk; ++j) {
                const float bj = sm.b[j], bgj = bj * sm.gam[j];
                float kj[8], vj[2];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) kj[cc] = sm.Kn[j][tx + 16 * cc];
                vj[0] = sm.V[j][tx];
                vj[1] = sm.V[j][tx + 16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float t = sm.A[ty + 16 * i][j];
                    const float tw = t * bgj, tu = t * bj;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) w[i][cc] = fmaf(tw, kj[cc], w[i][cc]);
                    u[i][0] = fmaf(tu, vj[0], u[i][0]);
                    u[i][1] = fmaf(tu, vj[1], u[i][1]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) sm.W[ty + 16 * i][tx + 16 * cc] = w[i][cc];
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sm.V[ty + 16 * i][tx] = u[i][0];
                sm.V[ty + 16 * i][tx + 16] = u[i][1];
            }
        }
        __syncthreads();

        // ---- 5. X = W S^T, Y = Q S^T; Delta = U - X (64 x 32 each)
        float y[4][2];
        {
            float xw[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) { xw[i][0] = xw[i][1] = 0.f; y[i][0] = y[i][1] = 0.f; }
#pragma unroll 4
            for (int cc = 0; cc < kD; ++cc) {
                const float s0v = sm.St[tx][cc], s1v = sm.St[tx + 16][cc];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float wv = sm.W[ty + 16 * i][cc], qv = sm.Qn[ty + 16 * i][cc];
                    xw[i][0] = fmaf(wv, s0v, xw[i][0]);
                    xw[i][1] = fmaf(wv, s1v, xw[i][1]);
                    y[i][0] = fmaf(qv, s0v, y[i][0]);
                    y[i][1] = fmaf(qv, s1v, y[i][1]);
                }
            }
            float dl[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dl[i][0] = sm.V[ty + 16 * i][tx] - xw[i][0];
                dl[i][1] = sm.V[ty + 16 * i][tx + 16] - xw[i][1];
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sm.V[ty + 16 * i][tx] = dl[i][0];
                sm.V[ty + 16 * i][tx + 16] = dl[i][1];
            }
        }
        __syncthreads();

        // ---- 6. O = diag(gam) Y + P Delta  -> out
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 16 * i;
            float o0 = sm.gam[r] * y[i][0], o1 = sm.gam[r] * y[i][1];
#pragma unroll 8
            for (int j = 0; j < kChunk; ++j) {
                const float p = sm.P[r][j];
                o0 = fmaf(p, sm.V[j][tx], o0);
                o1 = fmaf(p, sm.V[j][tx + 16], o1);
            }
            if (r < L) {
                IO* orow = out + ((size_t)(t0 + r) * hv + h) * kD + cv0;
                orow[tx] = from_f32<IO>(o0);
                orow[tx + 16] = from_f32<IO>(o1);
            }
        }

        // ---- 7. S <- gam_L S + Delta^T diag(c) K   (32 x 128)
        {
            const float gl = sm.gam[L - 1];
            float acc[2][8];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) acc[i][cc] = gl * sm.St[ty + 16 * i][tx + 16 * cc];
#pragma unroll 2
            for (int j = 0; j < L; ++j) {
                const float cj = sm.c[j];
                const float d0 = sm.V[j][ty] * cj, d1 = sm.V[j][ty + 16] * cj;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const float kv = sm.Kn[j][tx + 16 * cc];
                    acc[0][cc] = fmaf(d0, kv, acc[0][cc]);
                    acc[1][cc] = fmaf(d1, kv, acc[1][cc]);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) sm.St[ty + 16 * i][tx + 16 * cc] = acc[i][cc];
            if (cstates) {
                float* cs_row = cstates + ((size_t)(s_chunk0 + chunk_no) * hv + h) * kD * kD + (size_t)cv0 * kD;
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) cs_row[(size_t)(ty + 16 * i) * kD + tx + 16 * cc] = acc[i][cc];
            }
        }
    }
    __syncthreads();
    if (sT) {
        for (int idx = tid; idx < kSlice * kD; idx += kSimtThreads) {
            const int i = idx / kD, j = idx % kD;
            sT[state_base + (size_t)i * kD + j] = sm.St[i][j];
        }
    }
}

template <typename IO>
cudaError_t launch_typed(const IO* q, const IO* k, const IO* v, const float* g,
                         const float* beta, const float* s0, const int32_t* cu, IO* out,
                         float* sT, StateSlots map, float* cstates, int num_seqs, int hk, int hv,
                         GateAct act, cudaStream_t stream)
{
    const size_t smem = sizeof(SimtSmem);
    cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<IO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)num_seqs * (unsigned)hv * kSlices);
    prefill_simt_kernel<IO><<<grid, kSimtThreads, smem, stream>>>(q, k, v, g, beta, s0, cu, out,
                                                                   sT, map, cstates, hk, hv, act);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* s0, const int32_t* cu,
                                void* out, float* sT, StateSlots map, float* cstates, int num_seqs, int hk,
                                int hv, gdn_dtype io, GateAct act, cudaStream_t stream)
{
    if (num_seqs == 0) return cudaSuccess;
    if (io == GDN_BF16) {
        using T = __nv_bfloat16;
        return launch_typed<T>((const T*)q, (const T*)k, (const T*)v, g, beta, s0, cu, (T*)out,
                               sT, map, cstates, num_seqs, hk, hv, act, stream);
    }
    return launch_typed<float>((const float*)q, (const float*)k, (const float*)v, g, beta, s0, cu,
                               (float*)out, sT, map, cstates, num_seqs, hk, hv, act, stream);
}

}  // namespace gdn
