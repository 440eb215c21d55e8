// decode.cu -- memory-bound decode / multi-token-verify step of the Gated DeltaNet
// layer (gated delta rule; Qwen3-Next-80B-A3B model card, "Model Overview": 16 QK /
// 32 V heads, head dim 128; multi-token prediction serving verifies up to 4 draft
// tokens per step, Qwen3-Next model card "Deployment" and the vLLM blog post,
// "Multi-Token Prediction").
//
// Each (sequence n, V head h) streams that head's 128x128 fp32 state (64 KiB) once from
// HBM and once back, whatever the number of tokens m = 1..4.  The m tokens
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
// (n, h).
//
// Two kernels evaluate this.  decode_kernel (the 1-token step, every verify, and fp32 I/O)
// is described here; decode_mma_kernel (2..4 tokens in place with bf16 I/O) runs the same
// closed form with its two contractions on warp MMAs and is described at its definition.
//
// decode_kernel, one CTA per (sequence n, V head h).
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
#include <cuda.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {

__device__ unsigned int g_decode_error;  // set when a bounded wait of a decode kernel gives up

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
              int hk, int hv, GateAct act)
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
            acc += load_g(g, gi, act, h);
            G[t] = acc;
            bt[t] = load_beta(beta, gi, act);
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

// ---------------------------------------------------------------- multi-token step on warp MMAs (bf16 I/O)
// For 2..4 tokens in place with bf16 q, k, v.  The two contractions of the closed form are
// small matrix products:  the raw products X = S [k_0..k_{m-1} q_0..q_{m-1}]^T (128 x 8, K =
// 128) and the rank-m update S <- Gam_m S + W K (W: 128 x m per-row coefficients).  Here they
// run as m16n8k8 tf32 warp MMAs with fp32 accumulation, which takes the multiply-adds, the
// reductions over the 128 columns and the row update off the CUDA cores (about a third of the
// instructions of the SIMT kernel).  tf32 keeps 10 mantissa bits, so every fp32 operand x goes
// in as two terms, x = hi + lo with hi = x rounded to tf32 and lo = x - hi (together about 21
// bits); bf16 values (q, k, v) are exact in tf32 and need no split.
//
// One CTA of 4 warps per (sequence, V head), three CTAs per SM, so that the copies of one CTA
// overlap the arithmetic of the others.  At entry one thread issues the whole head's state as
// eight 2-D tensor copies (64 rows x 32 columns, 128-byte swizzle) and the item's q, k, v rows
// as bulk copies; rows 0..63 and the vectors complete one barrier, rows 64..127 a second, so
// that each warp starts on its first 16-row tile (rows 16 w ..) while its second (rows 16 (w +
// 4) ..) is still arriving.  Within a tile, MMA rows g = 0..7 are state rows 16 tile + 2 g and
// MMA rows g + 8 are 16 tile + 2 g + 1, which with the swizzle makes every fragment load free of
// bank conflicts.  The columns are permuted the same way in both products: in k-step / n-tile
// p, slot t of the MMA is column 8p + 2t and slot t + 4 is column 8p + 2t + 1, so the A
// fragments of S for the first product are exactly the accumulator fragments of S for the
// second.  The new rows go straight to HBM (each 8-byte store completes a 32-byte sector with
// its three neighbours).
constexpr int kCtaWarps = 4;
constexpr int kVecStride = 272;  // bytes between staged q / k / v rows (bank-conflict padding)
constexpr int kHalfRows = kD / 2;

template <int NTOK>
struct MmaLayout {
    static constexpr int kStateBytes = kD * kD * 4;                     // 4 column boxes of 128 rows
    static constexpr int kHalfBytes = kStateBytes / 2;
    static constexpr int kVec = kStateBytes;                            // rows k_0.., q_0.., v_0..
    static constexpr int kTx0 = kHalfBytes + 3 * NTOK * kD * 2;         // rows 0..63 and the vectors
    static constexpr int kGate = kVec + 3 * NTOK * kVecStride;          // g_t, beta_t, a_h, b_h
    static constexpr int kDots = (kGate + 16 * 4 + 15) / 16 * 16;       // per warp [8][8] floats
    static constexpr int kBar = kDots + kCtaWarps * 64 * 4;             // two barriers
    static constexpr int kSmem = kBar + 16 + 1024;                      // + alignment of the base
};

template <int NTOK>
__global__ void __launch_bounds__(kCtaWarps * 32, 3)
decode_mma_kernel(const __grid_constant__ CUtensorMap tm_state, const __nv_bfloat16* __restrict__ q,
                  const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                  StateSlots map, __nv_bfloat16* __restrict__ out, int hk, int hv, GateAct act) {
    using namespace sm100;
    using Lay = MmaLayout<NTOK>;
    constexpr int NV = 2 * NTOK;
    constexpr int NG = 2 * NTOK + 2;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sl =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    float* dots = reinterpret_cast<float*>(sl + Lay::kDots) + warp * 64;
    uint64_t* full = reinterpret_cast<uint64_t*>(sl + Lay::kBar);  // [0] rows 0..63 + vectors, [1] rows 64..127
    const int n = blockIdx.x / hv, h = blockIdx.x % hv, qh = h / (hv / hk);
    bool has;
    const int sidx = state_index(map, n, has);
    if (!has) return;  // a sequence without a state slot is skipped (whole CTA)
    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(full + 1, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(full, Lay::kTx0);
        mbar_arrive_expect_tx(full + 1, Lay::kHalfBytes);
        const int row0 = (sidx * hv + h) * kD;
        // box (column block cb, half hf) lands at cb * 16 KiB + hf * 8 KiB: the same bytes as
        // one 128-row box, so the swizzled addressing below does not depend on the split
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tma_load_2d(sl + cb * 16384, &tm_state, cb * 32, row0, full);
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            const size_t tok = (size_t)n * NTOK + t;
            bulk_g2s(sl + Lay::kVec + t * kVecStride, k + (tok * hk + qh) * kD, kD * 2, full);
            bulk_g2s(sl + Lay::kVec + (NTOK + t) * kVecStride, q + (tok * hk + qh) * kD, kD * 2, full);
            bulk_g2s(sl + Lay::kVec + (2 * NTOK + t) * kVecStride, v + (tok * hv + h) * kD, kD * 2, full);
        }
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
            tma_load_2d(sl + cb * 16384 + kHalfRows * 128, &tm_state, cb * 32, row0 + kHalfRows, full + 1);
    }
    if (tid >= 32 && tid < 32 + NG) {  // the gates, by plain loads while the copies fly
        const int e = tid - 32, t = e % NTOK;
        float val = 0.f;
        if (e < NTOK) val = g[((size_t)n * NTOK + t) * hv + h];
        else if (e < 2 * NTOK) val = beta[((size_t)n * NTOK + t) * hv + h];
        else if (act.a) val = (e == 2 * NTOK ? act.a : act.b)[h];
        reinterpret_cast<float*>(sl + Lay::kGate)[e] = val;
    }
    __syncthreads();  // the barriers are armed and the gates stored; no block barrier follows
    // Each warp waits (bounded) for what it reads; a warp whose wait gives up records the error
    // and leaves.  Nothing after this point synchronises the whole CTA.
    if (!mbar_wait(full, 0)) {
        if (lane == 0) atomicOr(&g_decode_error, 1u);
        return;
    }
    const unsigned char* vec = sl + Lay::kVec;

    // ---- this thread's vector n = gq at columns 8p + 2t, 8p + 2t + 1 and key t at 8p + gq
    uint32_t vb0[16], vb1[16];
    float kb[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        if (gq < NV) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vec + gq * kVecStride + (8 * p + 2 * tq) * 2);
            vb0[p] = w << 16;
            vb1[p] = w & 0xffff0000u;
        } else {
            vb0[p] = 0u;
            vb1[p] = 0u;
        }
        kb[p] = tq < NTOK ? to_f32(reinterpret_cast<const __nv_bfloat16*>(vec + tq * kVecStride)[8 * p + gq]) : 0.f;
    }
    {   // products among the vectors
        float dv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < 16; ++p) mma_tf32(dv, vb0[p], 0u, vb1[p], 0u, vb0[p], vb1[p]);
        dots[gq * 8 + 2 * tq] = dv[0];
        dots[gq * 8 + 2 * tq + 1] = dv[1];
    }
    __syncwarp();
    float bt[NTOK], Gm[NTOK], rk[NTOK], rq[NTOK], Et[NTOK][NTOK];
    {
        const float* gs = reinterpret_cast<const float*>(sl + Lay::kGate);
        const float ga = gs[2 * NTOK], gb = gs[2 * NTOK + 1];
        float G[NTOK], acc = 0.f;
#pragma unroll
        for (int t = 0; t < NTOK; ++t) {
            acc += act.a ? act_g(gs[t], ga, gb) : gs[t];
            G[t] = acc;
            bt[t] = act.a ? act_beta(gs[NTOK + t]) : gs[NTOK + t];
            Gm[t] = expf(G[t]);
            rk[t] = rsqrtf(dots[t * 8 + t] + kNormEps);
            rq[t] = rsqrtf(dots[(NTOK + t) * 8 + NTOK + t] + kNormEps) * kInvSqrtD;
        }
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
#pragma unroll
            for (int j = 0; j <= t; ++j) Et[t][j] = (j == t) ? 1.f : expf(G[t] - G[j]);
    }
    const __nv_bfloat16* vrow = reinterpret_cast<const __nv_bfloat16*>(vec + 2 * NTOK * kVecStride);
    const float gl = Gm[NTOK - 1];
#pragma unroll 1
    for (int tt = 0; tt < 2; ++tt) {
        if (tt == 1 && !mbar_wait(full + 1, 0)) {
            if (lane == 0) atomicOr(&g_decode_error, 1u);
            return;
        }
        const int tile = warp + kCtaWarps * tt;
        const int rowA = 16 * tile + 2 * gq, rowB = rowA + 1;
        // the rows' fragments are read from shared memory twice (here and in the update), which
        // keeps them out of registers across the recurrence
        auto frag = [&](int p, int row) {
            const int chunk = 2 * (p & 3) + (tq >> 1);
            return *reinterpret_cast<const float2*>(sl + (p >> 2) * 16384 + row * 128 +
                                                    ((chunk ^ (row & 7)) << 4) + 8 * (tq & 1));
        };
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const float2 sa = frag(p, rowA), sb = frag(p, rowB);
            const uint32_t a0 = tf32_hi(sa.x), a1 = tf32_hi(sb.x);
            const uint32_t a2 = tf32_hi(sa.y), a3 = tf32_hi(sb.y);
            mma_tf32(d, a0, a1, a2, a3, vb0[p], vb1[p]);
            mma_tf32(d, __float_as_uint(sa.x - __uint_as_float(a0)), __float_as_uint(sb.x - __uint_as_float(a1)),
                     __float_as_uint(sa.y - __uint_as_float(a2)), __float_as_uint(sb.y - __uint_as_float(a3)),
                     vb0[p], vb1[p]);
        }
        float xa[8], xb[8];
#pragma unroll
        for (int src = 0; src < 4; ++src) {
            const int from = (lane & ~3) | src;
            xa[2 * src] = __shfl_sync(0xffffffffu, d[0], from);
            xa[2 * src + 1] = __shfl_sync(0xffffffffu, d[1], from);
            xb[2 * src] = __shfl_sync(0xffffffffu, d[2], from);
            xb[2 * src + 1] = __shfl_sync(0xffffffffu, d[3], from);
        }
        float wa = 0.f, wb = 0.f;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const float* xr = rr ? xb : xa;
            const int row = rr ? rowB : rowA;
            float delta[NTOK];
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                float x = Gm[t] * (rk[t] * xr[t]);
#pragma unroll
                for (int j = 0; j < t; ++j) x = fmaf(Et[t][j] * dots[j * 8 + t] * rk[j] * rk[t], delta[j], x);
                delta[t] = bt[t] * (to_f32(vrow[t * (kVecStride / 2) + row]) - x);
                float o = Gm[t] * (rq[t] * xr[NTOK + t]);
#pragma unroll
                for (int j = 0; j <= t; ++j) o = fmaf(Et[t][j] * dots[j * 8 + NTOK + t] * rk[j] * rq[t], delta[j], o);
                if (t == tq) out[(((size_t)n * NTOK + t) * hv + h) * kD + row] = from_f32<__nv_bfloat16>(o);
            }
#pragma unroll
            for (int j = 0; j < NTOK; ++j)
                if (j == tq) (rr ? wb : wa) = Et[NTOK - 1][j] * rk[j] * delta[j];
        }
        const uint32_t wa_hi = tf32_hi(wa), wb_hi = tf32_hi(wb);
        const uint32_t wa_lo = __float_as_uint(wa - __uint_as_float(wa_hi));
        const uint32_t wb_lo = __float_as_uint(wb - __uint_as_float(wb_hi));
        float* dstA = state + ((size_t)sidx * hv + h) * kD * kD + rowA * kD + 2 * tq;
        float* dstB = dstA + kD;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const float2 sa = frag(p, rowA), sb = frag(p, rowB);
            float y[4] = {gl * sa.x, gl * sa.y, gl * sb.x, gl * sb.y};
            const uint32_t kbits = __float_as_uint(kb[p]);
            mma_tf32(y, wa_hi, wb_hi, wa_lo, wb_lo, kbits, kbits);
            __stcs(reinterpret_cast<float2*>(dstA + 8 * p), make_float2(y[0], y[1]));
            __stcs(reinterpret_cast<float2*>(dstB + 8 * p), make_float2(y[2], y[3]));
        }
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

template <int NTOK>
cudaError_t launch_mma(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const float* g,
                       const float* beta, float* state, StateSlots map, __nv_bfloat16* out, int num_seqs, int hk,
                       int hv, GateAct act, cudaStream_t stream) {
    using Lay = MmaLayout<NTOK>;
    static_assert(3 * (Lay::kSmem + 1024) <= 228 * 1024, "three CTAs per SM");
    // The states as a 2-D fp32 tensor [slots * HV * 128 rows][128], boxes of 64 rows x 32
    // columns (128 bytes, the swizzle width).
    const long long slots = map.slots ? map.num_slots : num_seqs;
    if (slots <= 0) return cudaSuccess;  // no sequence has a state: nothing to do
    if (slots * hv * kD > INT32_MAX) return cudaErrorInvalidValue;  // row numbers are 32-bit
    const long long items = (long long)num_seqs * hv;
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)(slots * hv * kD)};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)kHalfRows};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, state, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kernel = decode_mma_kernel<NTOK>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
    if (e != cudaSuccess) return e;
    kernel<<<dim3((unsigned)items), dim3(kCtaWarps * 32), Lay::kSmem, stream>>>(tm, q, k, v, g, beta, state, map,
                                                                                out, hk, hv, act);
    return cudaGetLastError();
}

template <typename IO, int NTOK, int R, bool SNAP>
cudaError_t launch_one(const IO* q, const IO* k, const IO* v, const float* g, const float* beta,
                       float* state, StateSlots map, IO* out, float* snap, int num_seqs, int hk, int hv,
                       GateAct act, cudaStream_t stream)
{
    auto kernel = decode_kernel<IO, NTOK, R, SNAP>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<dim3((unsigned)num_seqs * (unsigned)hv), dim3(kDecodeThreads), kStateSmemBytes,
             stream>>>(q, k, v, g, beta, state, map, out, snap, hk, hv, act);
    return cudaGetLastError();
}

template <typename IO, bool SNAP>
cudaError_t launch_typed(const IO* q, const IO* k, const IO* v, const float* g,
                         const float* beta, float* state, StateSlots map, IO* out, float* snap, int ntok,
                         int num_seqs, int hk, int hv, GateAct act, cudaStream_t stream)
{
    if constexpr (!SNAP) {  // in place
        if constexpr (sizeof(IO) == 2) {  // bf16: 2..4 tokens on warp MMAs
            switch (ntok) {
            case 2: return launch_mma<2>(q, k, v, g, beta, state, map, out, num_seqs, hk, hv, act, stream);
            case 3: return launch_mma<3>(q, k, v, g, beta, state, map, out, num_seqs, hk, hv, act, stream);
            case 4: return launch_mma<4>(q, k, v, g, beta, state, map, out, num_seqs, hk, hv, act, stream);
            default: break;
            }
        }
        switch (ntok) {  // one token, and fp32 I/O: one CTA per (sequence, V head)
        case 1: return launch_one<IO, 1, 8, false>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        case 2: return launch_one<IO, 2, 4, false>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        case 3: return launch_one<IO, 3, 2, false>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        default: return launch_one<IO, 4, 2, false>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        }
    } else {  // verify: one CTA per (sequence, V head)
        switch (ntok) {
        case 1: return launch_one<IO, 1, 8, true>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        case 2: return launch_one<IO, 2, 4, true>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        case 3: return launch_one<IO, 3, 2, true>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        default: return launch_one<IO, 4, 2, true>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
        }
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
                          int num_tokens, int num_seqs, int hk, int hv, gdn_dtype io, GateAct act,
                          cudaStream_t stream)
{
    if (num_seqs == 0) return cudaSuccess;
    if (io == GDN_BF16) {
        using T = __nv_bfloat16;
        if (snap)
            return launch_typed<T, true>((const T*)q, (const T*)k, (const T*)v, g, beta, state, map, (T*)out, snap,
                                         num_tokens, num_seqs, hk, hv, act, stream);
        return launch_typed<T, false>((const T*)q, (const T*)k, (const T*)v, g, beta, state, map, (T*)out, nullptr,
                                      num_tokens, num_seqs, hk, hv, act, stream);
    }
    if (snap)
        return launch_typed<float, true>((const float*)q, (const float*)k, (const float*)v, g, beta, state,
                                         map, (float*)out, snap, num_tokens, num_seqs, hk, hv, act, stream);
    return launch_typed<float, false>((const float*)q, (const float*)k, (const float*)v, g, beta, state,
                                      map, (float*)out, nullptr, num_tokens, num_seqs, hk, hv, act, stream);
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

// Reads and clears the streaming decode kernel's device error word on the current device.
extern "C" gdn_status gdn_get_decode_device_error(void* stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, gdn::g_decode_error, sizeof word, 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (word == 0) return GDN_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(gdn::g_decode_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_ERR_DEVICE_TIMEOUT;
}
