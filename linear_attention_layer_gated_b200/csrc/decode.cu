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
#include "sm100.cuh"

namespace gdn {

__device__ unsigned int g_decode_error;  // set when a bounded wait of the streaming kernel gives up

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

// ---------------------------------------------------------------- streaming multi-token step
// For 2..4 tokens the per-row work is several times the 1-token step's.  This kernel keeps
// one 512-thread CTA per SM and streams (sequence, V head) items through a ring of three
// shared-memory slots, so that while item i is computed the states of items i+1 and i+2 are
// on their way.  Each state (64 KiB, contiguous in HBM) arrives by one bulk asynchronous copy
// that completes on the slot's mbarrier; the small per-item vectors (q, k, v rows and the
// gates) come by cp.async.  The updated rows go back by bulk copies too (one 4 KiB copy per
// warp), so the threads issue only shared-memory accesses and arithmetic.
//
// Per item, with three CTA barriers:
//   B1  the item's state and vectors have landed;
//       the raw dot products among k_0.., q_0.. (8 lanes per product) and
//   pass 1: the 2m raw products s.k_t, s.q_t of every state row (a half-warp per R rows,
//       the transposing butterfly);
//   B2  the next free slot is refilled (item i+2);
//   pass 2: one thread per row turns the raw products into the norms, decays and
//       coefficients and runs the scalar recurrence of the m tokens;
//   B3
//   pass 3: the row update s <- Gam_m s + sum_j Et[m-1][j] delta_j k_j / |k_j|, written
//       back into the slot and copied to HBM by each warp for its 8 rows (with SNAP, every
//       intermediate state s_t goes straight to the snapshots instead and the state is left
//       alone; the last snapshot is computed with the same operations as the in-place state).
constexpr int kStrThreads = 512;

template <typename IO, int NTOK, bool SNAP>
struct StrLayout {
    static constexpr int kTokBytes = kD * (int)sizeof(IO);   // one q, k or v row
    static constexpr int kStateBytes = kD * kD * 4;
    static constexpr int kVec = kStateBytes;                  // q_0.., k_0.., v_0.. rows
    static constexpr int kG = kVec + 3 * NTOK * kTokBytes;    // g[NTOK], beta[NTOK], a_h, b_h
    static constexpr int kSlot = (kG + (2 * NTOK + 2) * 4 + 127) / 128 * 128;
    static constexpr int kCoefStride = SNAP ? 16 : 4;          // per row: [t][j] with SNAP, else [j]
    static constexpr int kSums = 3 * kSlot;                    // [128][8] raw products
    static constexpr int kCoef = kSums + 128 * 8 * 4;          // [128][kCoefStride]
    static constexpr int kOst = kCoef + 128 * kCoefStride * 4;  // [4][128] outputs
    static constexpr int kDots = kOst + 4 * 128 * 4;           // [8][8] raw vector products
    static constexpr int kGam = kDots + 64 * 4;                // Gam_t
    static constexpr int kBar = kGam + 16;                     // full[3], abort flag
    static constexpr int kSmem = kBar + 32;
};

template <typename IO>
__device__ __forceinline__ void load16f(const IO* p, float* x) {  // 16 consecutive elements
    if constexpr (sizeof(IO) == 4) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 v = reinterpret_cast<const float4*>(p)[c];
            x[4 * c] = v.x; x[4 * c + 1] = v.y; x[4 * c + 2] = v.z; x[4 * c + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 u = reinterpret_cast<const uint4*>(p)[c];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // a bf16 value is the upper half of the fp32 with its bits
                x[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
                x[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
        }
    }
}

__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
                 "l"(src)
                 : "memory");
}

template <typename IO, int NTOK, bool SNAP>
__global__ void __launch_bounds__(kStrThreads, 1)
decode_stream_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                     const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                     StateSlots map, IO* __restrict__ out, float* __restrict__ snap, int num_seqs, int hk,
                     int hv, GateAct act) {
    using namespace sm100;
    using Lay = StrLayout<IO, NTOK, SNAP>;
    constexpr int NT = NTOK == 3 ? 4 : NTOK;  // sums per kind, padded to a power of two
    constexpr int VR = 2 * NT;                // sums per row: x_0.., y_0..
    constexpr int R = 16 / VR;                // rows per half-warp per butterfly
    constexpr int kIters = 8 / (2 * R);       // a warp owns 8 rows
    constexpr int NV = 2 * NTOK;              // vectors k_0.., q_0..
    constexpr int ND = NV * (NV + 1) / 2;     // products among them
    constexpr int kDotWarps = (ND * 8 + 31) / 32;
    constexpr int CS = Lay::kCoefStride;
    extern __shared__ __align__(128) unsigned char smem[];
    float* sums = reinterpret_cast<float*>(smem + Lay::kSums);
    float* coefr = reinterpret_cast<float*>(smem + Lay::kCoef);
    float* ostage = reinterpret_cast<float*>(smem + Lay::kOst);
    float* dots = reinterpret_cast<float*>(smem + Lay::kDots);
    float* gam = reinterpret_cast<float*>(smem + Lay::kGam);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kBar + 24);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, half = lane >> 4, l = lane & 15;
    const int items = num_seqs * hv;
    const int first = blockIdx.x, stride = gridDim.x;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 3; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // The vectors of an item: cp.async by the threads, one group per item (empty past the end
    // or without a state slot, so that every thread's group count stays aligned with the items).
    auto issue_vectors = [&](int item, int slot) {
        if (item < items) {
            const int n = item / hv, h = item % hv, qh = h / (hv / hk);
            bool has;
            state_index(map, n, has);
            if (has) {
                unsigned char* base = smem + slot * Lay::kSlot;
                constexpr int kRowChunks = Lay::kTokBytes / 16;
                for (int c = tid; c < 3 * NTOK * kRowChunks; c += kStrThreads) {
                    const int which = c / (NTOK * kRowChunks), rem = c % (NTOK * kRowChunks);
                    const int t = rem / kRowChunks, ch = rem % kRowChunks;
                    const IO* src = which == 0   ? q + (((size_t)n * NTOK + t) * hk + qh) * kD
                                    : which == 1 ? k + (((size_t)n * NTOK + t) * hk + qh) * kD
                                                 : v + (((size_t)n * NTOK + t) * hv + h) * kD;
                    cp_async16(base + Lay::kVec + (which * NTOK + t) * Lay::kTokBytes + ch * 16,
                               reinterpret_cast<const unsigned char*>(src) + ch * 16);
                }
                if (tid >= kStrThreads - 2 * NTOK - 2) {  // the gates (and a_h, b_h for raw gates)
                    const int e = tid - (kStrThreads - 2 * NTOK - 2), t = e % NTOK;
                    if (e < 2 * NTOK)
                        cp_async4(base + Lay::kG + e * 4, (e < NTOK ? g : beta) + ((size_t)n * NTOK + t) * hv + h);
                    else if (act.a)
                        cp_async4(base + Lay::kG + e * 4, (e == 2 * NTOK ? act.a : act.b) + h);
                }
            }
        }
        cp_async_commit();
    };
    // The state of an item: one bulk copy issued by thread 0 that completes on full[slot]
    // (a plain arrival completes the phase for an item without a state slot).
    auto issue_state = [&](int item, int slot) {
        if (tid == 0 && item < items) {
            bool has;
            const int sidx = state_index(map, item / hv, has);
            if (has) {
                mbar_arrive_expect_tx(&full[slot], Lay::kStateBytes);
                bulk_g2s(smem + slot * Lay::kSlot, state + ((size_t)sidx * hv + item % hv) * kD * kD,
                         Lay::kStateBytes, &full[slot]);
            } else {
                mbar_arrive(&full[slot]);
            }
        }
    };

    issue_vectors(first, 0);
    issue_state(first, 0);
    issue_vectors(first + stride, 1);
    issue_state(first + stride, 1);
    int i = 0;
    for (;; ++i) {
        const int item = first + i * stride;
        if (item >= items) break;
        const int slot = i % 3;
        const uint32_t parity = (i / 3) & 1;
        cp_async_wait<1>();  // this thread's vectors of item i (item i+1's may still be in flight)
        if (tid == 0 && !mbar_wait(&full[slot], parity)) {
            *abort_flag = 1;
            atomicOr(&g_decode_error, 1u);
        }
        __syncthreads();  // B1
        if (*abort_flag) break;
        mbar_try_wait(&full[slot], parity);  // completed: makes the bulk copy's data visible here too
        const int n = item / hv, h = item % hv;
        bool has;
        const int sidx = state_index(map, n, has);
        issue_vectors(item + 2 * stride, (i + 2) % 3);  // the slot item i-1 used, free since B1

        unsigned char* base = smem + slot * Lay::kSlot;
        float* Ss = reinterpret_cast<float*>(base);
        const IO* vecs = reinterpret_cast<const IO*>(base + Lay::kVec);  // q_0.. k_0.. v_0.. rows
        float2 kv[NTOK][4];
        if (has) {
            // ---- raw products among k_0.. (vectors 0..NTOK-1) and q_0.. (NTOK..), 8 lanes each
            if (warp < kDotWarps) {
                const int d = tid >> 3, part = tid & 7;
                float acc = 0.f;
                int a = 0, b = 0;
                if (d < ND) {
                    int rem = d;
                    while (rem >= NV - a) { rem -= NV - a; ++a; }
                    b = a + rem;
                    auto vec = [&](int idx) { return vecs + (idx < NTOK ? NTOK + idx : idx - NTOK) * kD; };
                    float xa[16], xb[16];
                    load16f<IO>(vec(a) + 16 * part, xa);
                    load16f<IO>(vec(b) + 16 * part, xb);
                    float2 s2 = __fmul2_rn(make_float2(xa[0], xa[1]), make_float2(xb[0], xb[1]));
#pragma unroll
                    for (int e = 2; e < 16; e += 2)
                        s2 = __ffma2_rn(make_float2(xa[e], xa[e + 1]), make_float2(xb[e], xb[e + 1]), s2);
                    acc = s2.x + s2.y;
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                if (d < ND && part == 0) {
                    dots[a * 8 + b] = acc;
                    dots[b * 8 + a] = acc;
                }
            }
            // ---- pass 1: raw products of every state row with k_t and q_t
            float2 qv[NTOK][4];
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                load_cols(vecs + (NTOK + t) * kD, l, kv[t]);
                load_cols(vecs + t * kD, l, qv[t]);
            }
#pragma unroll
            for (int it = 0; it < kIters; ++it) {
                const int row0 = 8 * warp + it * 2 * R + half * R;
                float a[16];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float2 s2[4];
                    load_cols(Ss + (row0 + r) * kD, l, s2);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        a[r * VR + t] = t < NTOK ? dot8(s2, kv[t < NTOK ? t : 0]) : 0.f;
                        a[r * VR + NT + t] = t < NTOK ? dot8(s2, qv[t < NTOK ? t : 0]) : 0.f;
                    }
                }
                xpose_reduce<16, 8>(a, l);
                sums[(row0 + l / VR) * 8 + l % VR] = a[0];
            }
        }
        if (lane == 0) bulk_wait_read_all();  // this warp's copies of item i-1's rows have left the slot
        __syncthreads();                      // B2
        issue_state(item + 2 * stride, (i + 2) % 3);
        if (has) {
            // ---- pass 2: coefficients and the recurrence, one thread per row
            if (tid < kD) {
                const int row = tid;
                const float* gg = reinterpret_cast<const float*>(base + Lay::kG);
                const bool raw = act.a != nullptr;
                float G[NTOK], bt[NTOK], rk[NTOK], rq[NTOK], Gm[NTOK], Et[NTOK][NTOK];
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < NTOK; ++t) {
                    acc += raw ? act_g(gg[t], gg[2 * NTOK], gg[2 * NTOK + 1]) : gg[t];
                    bt[t] = raw ? act_beta(gg[NTOK + t]) : gg[NTOK + t];
                    G[t] = acc;
                    rk[t] = rsqrtf(dots[t * 8 + t] + kNormEps);
                    rq[t] = rsqrtf(dots[(NTOK + t) * 8 + NTOK + t] + kNormEps) * kInvSqrtD;
                    Gm[t] = expf(G[t]);
                }
#pragma unroll
                for (int t = 0; t < NTOK; ++t)
#pragma unroll
                    for (int j = 0; j <= t; ++j) Et[t][j] = (j == t) ? 1.f : expf(G[t] - G[j]);
                if (row == 0) {
#pragma unroll
                    for (int t = 0; t < NTOK; ++t) gam[t] = Gm[t];
                }
                float delta[NTOK];
#pragma unroll
                for (int t = 0; t < NTOK; ++t) {
                    float x = Gm[t] * (rk[t] * sums[row * 8 + t]);
#pragma unroll
                    for (int j = 0; j < t; ++j) x = fmaf(Et[t][j] * dots[j * 8 + t] * rk[j] * rk[t], delta[j], x);
                    delta[t] = bt[t] * (to_f32(vecs[(2 * NTOK + t) * kD + row]) - x);
                    float o = Gm[t] * (rq[t] * sums[row * 8 + NT + t]);
#pragma unroll
                    for (int j = 0; j <= t; ++j)
                        o = fmaf(Et[t][j] * dots[j * 8 + NTOK + t] * rk[j] * rq[t], delta[j], o);
                    ostage[t * kD + row] = o;
                }
#pragma unroll
                for (int t = SNAP ? 0 : NTOK - 1; t < NTOK; ++t)
#pragma unroll
                    for (int j = 0; j <= t; ++j)
                        coefr[row * CS + (SNAP ? t * 4 : 0) + j] = Et[t][j] * rk[j] * delta[j];
            }
            __syncthreads();  // B3
            // ---- pass 3: the new rows (or the snapshots); the outputs
#pragma unroll
            for (int it = 0; it < kIters; ++it) {
                const int row0 = 8 * warp + it * 2 * R + half * R;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int row = row0 + r;
                    float2 s2[4];
                    load_cols(Ss + row * kD, l, s2);
#pragma unroll
                    for (int t = SNAP ? 0 : NTOK - 1; t < NTOK; ++t) {
                        const float2 gt = make_float2(gam[t], gam[t]);
                        float2 y[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) y[c] = __fmul2_rn(gt, s2[c]);
#pragma unroll
                        for (int j = 0; j <= t; ++j) {
                            const float w = coefr[row * CS + (SNAP ? t * 4 : 0) + j];
#pragma unroll
                            for (int c = 0; c < 4; ++c) y[c] = __ffma2_rn(make_float2(w, w), kv[j][c], y[c]);
                        }
                        float* dst = SNAP ? snap + (((size_t)n * NTOK + t) * hv + h) * kD * kD + row * kD
                                          : Ss + row * kD;
                        const float4 lo = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
                        const float4 hi = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
                        if constexpr (SNAP) {
                            __stcs(reinterpret_cast<float4*>(dst + 4 * l), lo);
                            __stcs(reinterpret_cast<float4*>(dst + 64 + 4 * l), hi);
                        } else {
                            *reinterpret_cast<float4*>(dst + 4 * l) = lo;
                            *reinterpret_cast<float4*>(dst + 64 + 4 * l) = hi;
                        }
                    }
                }
            }
            if constexpr (!SNAP) {  // this warp's 8 rows, 4 KiB contiguous in HBM
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    bulk_s2g(state + ((size_t)sidx * hv + h) * kD * kD + 8 * warp * kD, Ss + 8 * warp * kD,
                             8 * kD * 4);
                    bulk_commit();
                }
            }
            if (tid < NTOK * kD) {
                const int t = tid / kD, row = tid % kD;
                out[(((size_t)n * NTOK + t) * hv + h) * kD + row] = from_f32<IO>(ostage[t * kD + row]);
            }
        }
    }
    // Drain: the state copies this CTA still has in flight, then the vectors.
    if (lane == 0) bulk_wait_all();
    if (tid == 0 && *abort_flag) {  // loads issued for items i (gave up) and i+1
        const int nxt = i + 1;
        if (first + nxt * stride < items) mbar_wait(&full[nxt % 3], (nxt / 3) & 1);
    }
    cp_async_wait<0>();
}

template <typename IO, int NTOK, bool SNAP>
cudaError_t launch_stream(const IO* q, const IO* k, const IO* v, const float* g, const float* beta, float* state,
                          StateSlots map, IO* out, float* snap, int num_seqs, int hk, int hv, GateAct act,
                          cudaStream_t stream) {
    auto kernel = decode_stream_kernel<IO, NTOK, SNAP>;
    using Lay = StrLayout<IO, NTOK, SNAP>;
    static_assert(Lay::kSmem <= 227 * 1024, "shared memory");
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int items = num_seqs * hv;
    kernel<<<dim3((unsigned)(items < sms ? items : sms)), dim3(kStrThreads), Lay::kSmem, stream>>>(
        q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act);
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
    switch (ntok) {  // one token: one CTA per head; 2..4 tokens: the streaming kernel
    case 1: return launch_one<IO, 1, 8, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
    case 2: return launch_stream<IO, 2, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
    case 3: return launch_stream<IO, 3, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
    default: return launch_stream<IO, 4, SNAP>(q, k, v, g, beta, state, map, out, snap, num_seqs, hk, hv, act, stream);
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
