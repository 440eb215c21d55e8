// prefill_tc.cu -- chunked prefill of the Gated DeltaNet layer on sm_100a tensor cores.
//
// The chunked form of the gated delta rule (chunks of 64 tokens; Gated DeltaNet per the
// Qwen3-Next-80B-A3B model card, "Model Overview": 16 QK heads, 32 V heads, head dim
// 128).  For a chunk entering with state S (d_v x d_k), normalised Q, K (rows = tokens),
// values V, in-chunk inclusive gate sums G_r, gam_r = exp(G_r), c_j = exp(G_L - G_j):
//   A = strictly_lower(b_r exp(G_r - G_j) K K^T),  T = (I + A)^-1
//   W = T diag(b gam) K,   U = T diag(b) V,   P = lower(exp(G_r - G_j) Q K^T)
//   Delta = U - W S^T,   O = diag(gam) Q S^T + P Delta,   S <- gam_L S + Delta^T diag(c) K
//
// Three kernels, all on the caller's stream:
//  K0 chunk_table_kernel  cu_seqlens -> per-sequence first chunk id and a (seq, start,
//                         length) entry per chunk, on the device (no host read).
//  K1 chunk_prep_kernel   one CTA per (chunk, QK head), all chunks in parallel, both V
//                         heads of the QK head:
//                         - normalisation; K K^T and Q K^T as one M=128 MMA [K; Q] K^T;
//                         - decay masks A and P; T = (I + A)^-1 in fp32 by 16x16 blocks:
//                           diagonal inverses by forward substitution, then the blocks below
//                           the diagonal as dense 16x16 products (64 threads per V head);
//                         - W and U of both heads as M=128 MMAs [T_0 D_0; T_1 D_1] x (K or V),
//                           so each thread owns one output row and writes 16-byte chunks;
//                         - bf16 operand images, already in the 128-byte swizzled layout the
//                           state kernel's MMAs read, go to the workspace, with the gate
//                           factors (c, gam) of each V head.
//  K2 chunk_state_kernel  one CTA per (sequence, V head, half of d_v), sequential over the
//                         sequence's chunks.  Warp 8 issues the MMAs, warp 9 the bulk copies
//                         (two chunks ahead, three buffers); warps 0-7 compute, each warp on
//                         32 of the 64 d_v columns of its TMEM lane quarter.  Per chunk:
//                           [X; Y] = [W; Q] S^T          (M=128)            <- on the chain
//                           Delta = U - X, c Delta       (lanes 0-63: token rows)
//                           K^T diag(c) Delta            (M=128: d_k rows)  <- on the chain
//                           S^T <- gam_L S^T + K^T diag(c) Delta   (fp32 in registers)
//                           P Delta                      (M=128 operand [U; P]: rows 64..127)
//                           O = diag(gam) Y + P Delta    (lanes 64-127, one chunk later)
//                         Hand-offs between the issuing and the compute warps are mbarriers;
//                         the output accumulators are triple-buffered in Tensor Memory so
//                         the output epilogue stays off the state chain.
// Every mbarrier wait is bounded (1 s) and, in the state kernel, also gives up as soon as
// another thread of the CTA has given up; the kernel then records an error in the
// workspace header, drains its own copies and MMAs (bounded), frees Tensor Memory and
// returns.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

// Operand image sizes (bytes)
constexpr uint32_t kWBytes = 16384;    // W: 64 token rows x 128 d_k, K-major, [K-block][64 rows]
constexpr uint32_t kQBytes = 16384;    // normalised Q, same layout (per QK head)
constexpr uint32_t kUBytes = 16384;    // U: [d_v half][64 rows][64]
constexpr uint32_t kPBytes = 8192;     // P: 64 token rows x 64, K-major
constexpr uint32_t kCvecBytes = 1024;  // c_j at [0,64), gam_r at [64,128), gam_L at [128]
constexpr uint32_t kCvecLoad = 528;    // the bytes of a gate-factor record the state kernel reads
constexpr uint32_t kKTBytes = 16384;   // K, [d_k block][64 token rows] (MN-major A operand)
constexpr uint32_t kChunkLoadBytes = kWBytes + kQBytes + kKTBytes + kUBytes / 2 + kPBytes + kCvecLoad;

struct WsLayout {
    size_t seq_chunk0, table, w, u, p, cvec, kt, qn, total;
    long long max_chunks;
};

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int num_seqs, int total_tokens, int hk, int hv) {
    WsLayout L;
    L.max_chunks = (long long)total_tokens / kChunk + num_seqs;
    size_t off = 256;  // header: [0] device error word, [1] number of chunks
    L.seq_chunk0 = off;
    off = round_up(off + (size_t)(num_seqs + 1) * 4, 1024);
    L.table = off;
    off = round_up(off + (size_t)L.max_chunks * 16, 1024);
    L.w = off;
    off += (size_t)L.max_chunks * hv * kWBytes;
    L.u = off;
    off += (size_t)L.max_chunks * hv * kUBytes;
    L.p = off;
    off += (size_t)L.max_chunks * hv * kPBytes;
    L.cvec = off;
    off += (size_t)L.max_chunks * hv * kCvecBytes;
    L.kt = off;
    off += (size_t)L.max_chunks * hk * kKTBytes;
    L.qn = off;
    off += (size_t)L.max_chunks * hk * kQBytes;
    L.total = round_up(off, 1024);
    return L;
}

// ===================================================================== K0
__global__ void __launch_bounds__(1024)
chunk_table_kernel(const int32_t* __restrict__ cu, int num_seqs, unsigned char* ws) {
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const WsLayout L = ws_layout(num_seqs, 0, 1, 1);  // seq_chunk0 and table do not depend on T
    int32_t* seq_chunk0 = reinterpret_cast<int32_t*>(ws + L.seq_chunk0);
    int4* table = reinterpret_cast<int4*>(ws + L.table);
    __shared__ int32_t scan[1024];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + threadIdx.x;
        const int cnt = (n < num_seqs) ? (cu[n + 1] - cu[n] + kChunk - 1) / kChunk : 0;
        scan[threadIdx.x] = cnt;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {  // inclusive Hillis-Steele scan
            const int add = (threadIdx.x >= o) ? scan[threadIdx.x - o] : 0;
            __syncthreads();
            scan[threadIdx.x] += add;
            __syncthreads();
        }
        if (n < num_seqs) seq_chunk0[n] = carry + scan[threadIdx.x] - cnt;
        __syncthreads();
        if (threadIdx.x == 1023) carry += scan[1023];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        seq_chunk0[num_seqs] = carry;
        header[1] = carry;
    }
    __syncthreads();
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        const int t0 = cu[n], len = cu[n + 1] - cu[n];
        const int first = seq_chunk0[n];
        for (int kk = 0; kk * kChunk < len; ++kk)
            table[first + kk] = make_int4(n, t0 + kk * kChunk, min(kChunk, len - kk * kChunk), 0);
    }
}

// bf16 packing helpers
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* x) {
    return make_uint4(pack2(x[0], x[1]), pack2(x[2], x[3]), pack2(x[4], x[5]), pack2(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float* x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        float2 f = __bfloat1622float2(h);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ float sum8(float x) {  // over groups of 8 consecutive lanes
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
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

// fp32 64x64 matrices in shared memory: rows padded to 68 floats, so that 8 threads writing
// float4s to 8 consecutive rows hit different banks and row reads stay contiguous.
constexpr int kLdA = 68;
constexpr int kAfHead = kChunk * kLdA;   // floats per head

// 2^x on the special-function unit (PTX ex2.approx); callers pass arguments <= 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// ===================================================================== K1
// Shared memory map (bytes from a 1024-aligned base):
constexpr uint32_t kP_GR = 0;        // [K; Q] K-major (32 KB)  | after the Gram MMA: V images of both heads
constexpr uint32_t kP_KT = 32768;    // K MN-major (16 KB)
constexpr uint32_t kP_AF = 49152;    // A / T fp32, 2 heads (2 x 17 KB) | then [T0 D0; T1 D1] images for W and U
constexpr uint32_t kP_XS = 49152 + 2 * kAfHead * 4;  // block-solve scratch, 2 heads x 768 floats (6 KB)
constexpr uint32_t kP_SMALL = kP_XS + 2 * 768 * 4;   // gates, barrier, TMEM address
constexpr uint32_t kPrepSmem = kP_SMALL + 2048 + 1024;

struct PrepSmall {
    float G[2][kChunk];   // in-chunk gate sums, pre-scaled by log2(e)
    float b[2][kChunk];
    float gam[2][kChunk];
    uint64_t bar_mma;
    uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 2)
chunk_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                  const float* __restrict__ beta, unsigned char* ws, int num_seqs,
                  int total_tokens, int hk, int hv) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    PrepSmall& ss = *reinterpret_cast<PrepSmall*>(sm + kP_SMALL);
    float* af = reinterpret_cast<float*>(sm + kP_AF);   // [head][64][kLdA]
    float* xs = reinterpret_cast<float*>(sm + kP_XS);   // [head][768]

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int cid = blockIdx.x / hk;
    const int jq = blockIdx.x % hk;
    if (cid >= header[1]) return;
    const int4 ent = reinterpret_cast<const int4*>(ws + L.table)[cid];
    const int t0 = ent.y, len = ent.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h0 = jq * 2;  // the two V heads of this QK head

    // Thread's slice of a row for the row loads: 16 elements = 2 chunks of one 64-wide block.
    const int sub = tid & 7, kb = sub >> 2, c0 = (sub & 3) * 2;
    int err = 0;
    bool ok;

    // ---- 0. issue the q, k row loads (4 passes of 16 rows), gates, TMEM, barrier
    uint4 kr[4][2], qr[4][2];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int r = pass * 16 + (tid >> 3);
        if (r < len) {
            const size_t base = ((size_t)(t0 + r) * hk + jq) * kD + sub * 16;
            kr[pass][0] = *reinterpret_cast<const uint4*>(k + base);
            kr[pass][1] = *reinterpret_cast<const uint4*>(k + base + 8);
            qr[pass][0] = *reinterpret_cast<const uint4*>(q + base);
            qr[pass][1] = *reinterpret_cast<const uint4*>(q + base + 8);
        } else {
            kr[pass][0] = kr[pass][1] = qr[pass][0] = qr[pass][1] = make_uint4(0, 0, 0, 0);
        }
    }
    if (warp < 2) {
        const int h = h0 + warp;
        const float g0 = (lane < len) ? g[(size_t)(t0 + lane) * hv + h] : 0.f;
        const float g1 = (lane + 32 < len) ? g[(size_t)(t0 + lane + 32) * hv + h] : 0.f;
        const float G0 = warp_inclusive_scan(g0, lane);
        const float G1 = warp_inclusive_scan(g1, lane) + __shfl_sync(0xffffffffu, G0, 31);
        ss.G[warp][lane] = G0 * kLog2e;
        ss.G[warp][lane + 32] = G1 * kLog2e;
        ss.gam[warp][lane] = expf(G0);
        ss.gam[warp][lane + 32] = expf(G1);
        ss.b[warp][lane] = (lane < len) ? beta[(size_t)(t0 + lane) * hv + h] : 0.f;
        ss.b[warp][lane + 32] = (lane + 32 < len) ? beta[(size_t)(t0 + lane + 32) * hv + h] : 0.f;
    }
    if (warp == 3) {
        tmem_alloc(&ss.tmem_base, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&ss.bar_mma, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;

    // ---- 1. normalise; [K; Q] K-major and K MN-major in smem; K and Q images to the workspace
    {
        unsigned char* kt_img = ws + L.kt + ((size_t)cid * hk + jq) * kKTBytes;
        unsigned char* qn_img = ws + L.qn + ((size_t)cid * hk + jq) * kQBytes;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
            const int r = pass * 16 + (tid >> 3);
            float kv[16], qv[16];
            unpack8(kr[pass][0], kv);
            unpack8(kr[pass][1], kv + 8);
            unpack8(qr[pass][0], qv);
            unpack8(qr[pass][1], qv + 8);
            float ssk = 0.f, ssq = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) { ssk = fmaf(kv[e], kv[e], ssk); ssq = fmaf(qv[e], qv[e], ssq); }
            const float rk = rsqrtf(sum8(ssk) + kNormEps);
            const float rq = rsqrtf(sum8(ssq) + kNormEps) * kInvSqrtD;
#pragma unroll
            for (int e = 0; e < 16; ++e) { kv[e] *= rk; qv[e] *= rq; }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int ch = c0 + cc;
                const uint4 kp8 = pack8(kv + 8 * cc), qp8 = pack8(qv + 8 * cc);
                *reinterpret_cast<uint4*>(sm + kP_GR + kb * 16384 + sw128(r, ch)) = kp8;
                *reinterpret_cast<uint4*>(sm + kP_GR + kb * 16384 + sw128(64 + r, ch)) = qp8;
                *reinterpret_cast<uint4*>(sm + kP_KT + kb * 8192 + sw128(r, ch)) = kp8;
                *reinterpret_cast<uint4*>(kt_img + kb * 8192 + sw128(r, ch)) = kp8;
                *reinterpret_cast<uint4*>(qn_img + kb * 8192 + sw128(r, ch)) = qp8;
            }
        }
    }
    fence_async_smem();
    __syncthreads();

    // ---- 2. Gram: TMEM[0:128, 0:64] = [K; Q] K^T  (M=128, N=64, K=128); V loads meanwhile
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t a = sb + kP_GR + (s >> 2) * 16384 + (s & 3) * 32;
            mma_bf16(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idesc, s > 0);
        }
        mma_commit(&ss.bar_mma);
    }
    {
        uint4 vr[2][4][2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int pass = 0; pass < 4; ++pass) {
                const int r = pass * 16 + (tid >> 3);
                if (r < len) {
                    const uint4* vp = reinterpret_cast<const uint4*>(v + ((size_t)(t0 + r) * hv + h0 + hh) * kD + sub * 16);
                    vr[hh][pass][0] = vp[0];
                    vr[hh][pass][1] = vp[1];
                } else {
                    vr[hh][pass][0] = vr[hh][pass][1] = make_uint4(0, 0, 0, 0);
                }
            }
        // gate factors of both heads to the workspace (warps 2-3; token row r)
        if (warp >= 2) {
            const int r = tid - 64;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float* cv = reinterpret_cast<float*>(ws + L.cvec + ((size_t)cid * hv + h0 + hh) * kCvecBytes);
                const float Gl = ss.G[hh][len - 1], Gr = ss.G[hh][r];
                cv[r] = (r < len) ? fast_exp2(Gl - Gr) : 0.f;
                cv[64 + r] = ss.gam[hh][r];
                if (r == 0) cv[128] = ss.gam[hh][len - 1];
            }
        }
        ok = mbar_wait(&ss.bar_mma, 0);
        if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
        tc_fence_after();

        // ---- 3. decay masks from the Gram rows: A (fp32, smem) from K K^T (warps 0-1),
        //         P = lower(exp(G_r - G_j) Q K^T) of both heads to the workspace (warps 2-3)
        {
            float row[64];
            tmem_ld64(tmem, warp, 0, row);
            const int r = tid & 63;
            if (warp < 2) {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const float Gr = ss.G[hh][r], br = ss.b[hh][r];
                    const float4* g4 = reinterpret_cast<const float4*>(ss.G[hh]);
                    float4* a4 = reinterpret_cast<float4*>(af + hh * kAfHead + r * kLdA);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float4 gi = g4[m];
                        const float gg[4] = {gi.x, gi.y, gi.z, gi.w};
                        float t4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 4 * m + e;
                            t4[e] = (i < r) ? br * fast_exp2(fminf(Gr - gg[e], 0.f)) * row[i] : 0.f;
                        }
                        a4[m] = make_float4(t4[0], t4[1], t4[2], t4[3]);
                    }
                }
            } else {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const float Gr = ss.G[hh][r];
                    const float4* g4 = reinterpret_cast<const float4*>(ss.G[hh]);
                    unsigned char* pimg = ws + L.p + ((size_t)cid * hv + h0 + hh) * kPBytes;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const float4 ga = g4[2 * ch], gb = g4[2 * ch + 1];
                        const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                        float p8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = 8 * ch + e;
                            p8[e] = (i <= r) ? fast_exp2(fminf(Gr - gg[e], 0.f)) * row[i] : 0.f;
                        }
                        *reinterpret_cast<uint4*>(pimg + sw128(r, ch)) = pack8(p8);
                    }
                }
            }
        }
        // V images (MN-major: token row, d_v contiguous) into the dead [K; Q] region
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int pass = 0; pass < 4; ++pass) {
                const int rr = pass * 16 + (tid >> 3);
                *reinterpret_cast<uint4*>(sm + kP_GR + hh * 16384 + kb * 8192 + sw128(rr, c0)) = vr[hh][pass][0];
                *reinterpret_cast<uint4*>(sm + kP_GR + hh * 16384 + kb * 8192 + sw128(rr, c0 + 1)) = vr[hh][pass][1];
            }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- 4. T = (I + A)^-1 per head, by 16x16 blocks, in place.  Each head uses 64 threads.
    //         (a) diagonal blocks: D_b = (I + A_bb)^-1 by forward substitution, one column
    //             per thread; (b) below the diagonal, block row by block row,
    //             T_ij = -D_i (sum_{k=j}^{i-1} A_ik T_kj), as dense 16x16 products.
    {
        const int hh = tid >> 6, l = tid & 63;
        float* A = af + hh * kAfHead;
        float* X = xs + hh * 768;
        {
            const int base = 16 * (l >> 4), j = l & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float* arow = A + (base + r) * kLdA + base;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < r; ++k) acc = fmaf(arow[k], x[k], acc);
                x[r] = (r == j) ? 1.f : ((r < j) ? 0.f : -acc);
            }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < 16; ++r) A[(base + r) * kLdA + base + j] = x[r];
        }
        __syncthreads();
        // Output mapping inside a 16x16 block: column cc = l & 15, rows rr0 + 4 q for q = 0..3.
        const int cc = l & 15, rr0 = l >> 4;
        // Block rows i = 1, 2, 3 in order.  Row i reads only its own A blocks (still intact)
        // and blocks of rows < i (already T); it is overwritten only after all its X_ij are formed.
        // The block loops stay rolled (small code); each 16-term dot product is unrolled.
#pragma unroll 1
        for (int i = 1; i < 4; ++i) {
            const float* arow[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) arow[q] = A + (16 * i + rr0 + 4 * q) * kLdA;
#pragma unroll 1
            for (int j = 0; j < i; ++j) {              // X_ij = sum_{k=j}^{i-1} A_ik T_kj
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
                for (int k = j; k < i; ++k) {
                    const float* tc = A + (16 * k) * kLdA + 16 * j + cc;
                    float tcol[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) tcol[m] = tc[m * kLdA];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4* ar = reinterpret_cast<const float4*>(arow[q] + 16 * k);
#pragma unroll
                        for (int m4 = 0; m4 < 4; ++m4) {
                            const float4 a = ar[m4];
                            acc[q] = fmaf(a.x, tcol[4 * m4 + 0], acc[q]);
                            acc[q] = fmaf(a.y, tcol[4 * m4 + 1], acc[q]);
                            acc[q] = fmaf(a.z, tcol[4 * m4 + 2], acc[q]);
                            acc[q] = fmaf(a.w, tcol[4 * m4 + 3], acc[q]);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) X[j * 256 + (rr0 + 4 * q) * 16 + cc] = acc[q];
            }
            __syncthreads();
#pragma unroll 1
            for (int j = 0; j < i; ++j) {              // T_ij = -D_i X_ij
                float xcol[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) xcol[m] = X[j * 256 + m * 16 + cc];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4* dr = reinterpret_cast<const float4*>(arow[q] + 16 * i);
                    float acc = 0.f;
#pragma unroll
                    for (int m4 = 0; m4 < 4; ++m4) {
                        const float4 d = dr[m4];
                        acc = fmaf(d.x, xcol[4 * m4 + 0], acc);
                        acc = fmaf(d.y, xcol[4 * m4 + 1], acc);
                        acc = fmaf(d.z, xcol[4 * m4 + 2], acc);
                        acc = fmaf(d.w, xcol[4 * m4 + 3], acc);
                    }
                    A[(16 * i + rr0 + 4 * q) * kLdA + 16 * j + cc] = -acc;
                }
            }
            __syncthreads();
        }
    }

    // ---- 5. MMA operand images [T_0 diag(b_0 gam_0); T_1 diag(b_1 gam_1)] and [T_0 diag(b_0); ...]
    {
        const int hh = tid >> 6, r = tid & 63;
        const float4* t4 = reinterpret_cast<const float4*>(af + hh * kAfHead + r * kLdA);
        uint4 wrow[8], urow[8];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            float w8[8], u8[8];
#pragma unroll
            for (int half4 = 0; half4 < 2; ++half4) {
                const int m = 2 * ch + half4;   // float4 group: columns 4m .. 4m+3
                const float4 tv = t4[m];
                const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * m + e;
                    u8[4 * half4 + e] = tt[e] * ss.b[hh][j];
                    w8[4 * half4 + e] = u8[4 * half4 + e] * ss.gam[hh][j];
                }
            }
            wrow[ch] = pack8(w8);
            urow[ch] = pack8(u8);
        }
        __syncthreads();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            *reinterpret_cast<uint4*>(sm + kP_AF + sw128(tid, ch)) = wrow[ch];
            *reinterpret_cast<uint4*>(sm + kP_AF + 16384 + sw128(tid, ch)) = urow[ch];
        }
    }
    fence_async_smem();
    __syncthreads();

    // ---- 6. W (both heads) and U of head 0:  D[:, 0:128] = A_W K,  D[:, 128:256] = A_U V_0
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            mma_bf16(tmem, sdesc_sw128(sb + kP_AF + s * 32, 16, 1024),
                     sdesc_sw128(sb + kP_KT + s * 2048, 8192, 1024), idesc, s > 0);
            mma_bf16(tmem + 128, sdesc_sw128(sb + kP_AF + 16384 + s * 32, 16, 1024),
                     sdesc_sw128(sb + kP_GR + s * 2048, 8192, 1024), idesc, s > 0);
        }
        mma_commit(&ss.bar_mma);
    }
    ok = mbar_wait(&ss.bar_mma, 1);
    if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
    tc_fence_after();

    // ---- 7. epilogue: accumulator row r' is row r' % 64 of head r' / 64
    {
        const int hh = tid >> 6, r = tid & 63, h = h0 + hh;
        unsigned char* wimg = ws + L.w + ((size_t)cid * hv + h) * kWBytes;
        unsigned char* uimg = ws + L.u + ((size_t)cid * hv + h) * kUBytes;
        float col[64];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tmem_ld64(tmem, warp, 64 * half, col);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(wimg + half * 8192 + sw128(r, ch)) = pack8(col + 8 * ch);
        }
        if (hh == 0) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld64(tmem, warp, 128 + 64 * half, col);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(uimg + half * 8192 + sw128(r, ch)) = pack8(col + 8 * ch);
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // U of head 1: D[:, 128:256] = A_U V_1 (rows 64..127 are head 1's)
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem + 128, sdesc_sw128(sb + kP_AF + 16384 + s * 32, 16, 1024),
                         sdesc_sw128(sb + kP_GR + 16384 + s * 2048, 8192, 1024), idesc, s > 0);
            mma_commit(&ss.bar_mma);
        }
        ok = mbar_wait(&ss.bar_mma, 0);
        if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
        tc_fence_after();
        if (hh == 1) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld64(tmem, warp, 128 + 64 * half, col);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(uimg + half * 8192 + sw128(r, ch)) = pack8(col + 8 * ch);
            }
        }
    }

cleanup:
    if (err && tid == 0) {
        atomicOr(header, 1);
        mma_commit(&ss.bar_mma);  // MMAs issued so far complete before TMEM is freed
        mbar_wait(&ss.bar_mma, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ===================================================================== K2
constexpr int kStateThreads = 320;                  // warps 0-7 compute, warp 8 MMAs, warp 9 bulk copies
constexpr int kStages = 3;                          // chunk buffers (loads run two chunks ahead)
constexpr uint32_t kS_A1 = 0;                       // [W; Q] K-major, 2 K-blocks of 128 rows (32 KB)
constexpr uint32_t kS_KT = 32768;                   // K, MN-major A operand (16 KB)
constexpr uint32_t kS_U = 49152;                    // U, this CTA's d_v half (8 KB)
constexpr uint32_t kS_P = 57344;                    // P (8 KB); [U; P] is the A operand of P Delta
constexpr uint32_t kS_BUF = 65536;                  // one chunk buffer (64 KB)
constexpr uint32_t kS_B1 = kStages * kS_BUF;        // S slice bf16, MN-major (16 KB)
constexpr uint32_t kS_B2 = kS_B1 + 16384;           // Delta, MN-major (8 KB)
constexpr uint32_t kS_B3 = kS_B2 + 8192;            // diag(c) Delta, MN-major (8 KB)
constexpr uint32_t kS_CV = kS_B3 + 8192;            // gate factors of each stage (3 x 528 B)
constexpr uint32_t kS_SMALL = kS_CV + kStages * kCvecLoad;
constexpr uint32_t kStateSmem = kS_SMALL + 128;     // needs a 1024-aligned dynamic base (checked)
// Tensor Memory columns
constexpr int kTBufs = 3;        // output accumulators of three consecutive chunks stay live
constexpr uint32_t kT_XY = 0;     // [X; Y] of chunk c at kT_XY + 64 (c % 3)
constexpr uint32_t kT_PD = 192;   // P Delta of chunk c at kT_PD + 64 (c % 3) (rows 64..127)
constexpr uint32_t kT_SA = 384;   // K^T diag(c) Delta

struct StateSmall {
    uint64_t full[kStages];   // stage loaded
    uint64_t empty[kStages];  // stage consumed: 256 compute-thread arrivals + the MMAs' commit
    uint64_t mma2[kTBufs];    // P Delta of chunk c done, on mma2[c % 3] (a waiter may lag one chunk)
    uint64_t b1, b3, b2, mma1, mma3;
    uint32_t tmem_base;
    int abort_flag;
};

// Bounded wait that also returns (false) as soon as another thread has given up.  The
// waiting thread is suspended by the hardware between checks (it resumes when the phase
// completes), so idle waiters neither spin on issue slots nor oversleep.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int32_t* header) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(header, 1);
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 32 consecutive TMEM columns of this warp's lane quarter.
__device__ __forceinline__ void tmem_ld32(uint32_t tmem_base, int warp, uint32_t col, float* v) {
    const uint32_t a = tmem_base + ((uint32_t)(warp & 3) * 32u << 16) + col;
    tmem_ld16(a, v);
    tmem_ld16(a + 16, v + 16);
    tmem_ld_wait();
}

__device__ __forceinline__ void issue_chunk_loads(unsigned char* buf, unsigned char* cv, uint64_t* bar,
                                                  const unsigned char* ws, const WsLayout& L, int cid, int h,
                                                  int jq, int half, int hk, int hv) {
    mbar_arrive_expect_tx(bar, kChunkLoadBytes);
    const unsigned char* w = ws + L.w + ((size_t)cid * hv + h) * kWBytes;
    const unsigned char* qn = ws + L.qn + ((size_t)cid * hk + jq) * kQBytes;
    bulk_g2s(buf + kS_A1, w, 8192, bar);                  // W rows, d_k 0..63
    bulk_g2s(buf + kS_A1 + 8192, qn, 8192, bar);          // Q rows, d_k 0..63
    bulk_g2s(buf + kS_A1 + 16384, w + 8192, 8192, bar);   // W rows, d_k 64..127
    bulk_g2s(buf + kS_A1 + 24576, qn + 8192, 8192, bar);  // Q rows, d_k 64..127
    bulk_g2s(buf + kS_KT, ws + L.kt + ((size_t)cid * hk + jq) * kKTBytes, kKTBytes, bar);
    bulk_g2s(buf + kS_U, ws + L.u + ((size_t)cid * hv + h) * kUBytes + half * (kUBytes / 2), kUBytes / 2, bar);
    bulk_g2s(buf + kS_P, ws + L.p + ((size_t)cid * hv + h) * kPBytes, kPBytes, bar);
    bulk_g2s(cv, ws + L.cvec + ((size_t)cid * hv + h) * kCvecBytes, kCvecLoad, bar);
}

__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_kernel(const float* s0, const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out,
                   float* sT, unsigned char* ws, int num_seqs, int total_tokens, int hk, int hv) {
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sb = smem_u32(sm);
    StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + kS_SMALL);
    volatile int* abort_flag = &ss.abort_flag;

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int half = blockIdx.x & 1;
    const int h = (blockIdx.x >> 1) % hv;
    const int n = (blockIdx.x >> 1) / hv;
    const int jq = h / (hv / hk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t* seq_chunk0 = reinterpret_cast<const int32_t*>(ws + L.seq_chunk0);
    const int cs = seq_chunk0[n], nch = seq_chunk0[n + 1] - cs;
    const int t_begin = cu[n], t_end = cu[n + 1];
    if (sb & 1023u) {  // the swizzled operand layouts need a 1024-byte-aligned base
        if (tid == 0) atomicOr(header, 2);
        return;
    }

    if (warp == 0) {
        tmem_alloc(&ss.tmem_base, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ss.full[s], 1);
            mbar_init(&ss.empty[s], 257);
        }
        mbar_init(&ss.b1, 256);
        mbar_init(&ss.b3, 128);
        mbar_init(&ss.b2, 128);
        mbar_init(&ss.mma1, 1);
        for (int s = 0; s < kTBufs; ++s) mbar_init(&ss.mma2[s], 1);
        mbar_init(&ss.mma3, 1);
        ss.abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;

    if (warp == 8) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_xy = idesc_bf16(128, 64, 0, 1);  // A K-major, B MN-major
            const uint32_t id_s = idesc_bf16(128, 64, 1, 1);   // A MN-major, B MN-major
            const uint64_t d_b1 = sdesc_sw128(sb + kS_B1, 16384, 1024);
            const uint64_t d_b2 = sdesc_sw128(sb + kS_B2, 8192, 1024);
            const uint64_t d_b3 = sdesc_sw128(sb + kS_B3, 8192, 1024);
            int c = 0;
            for (; c < nch; ++c) {
                const int b = c % kStages, par = c & 1, tb = c % kTBufs;
                const uint32_t bufa = sb + b * kS_BUF;
                const uint64_t d_a1 = sdesc_sw128(bufa + kS_A1, 16, 1024);
                const uint64_t d_kt = sdesc_sw128(bufa + kS_KT, 8192, 1024);
                const uint64_t d_up = sdesc_sw128(bufa + kS_U, 16, 1024);  // rows 0..63 U (unused), 64..127 P
                // the operands normally land long before the state does: check them first
                if (!wait_or_abort(&ss.full[b], (c / kStages) & 1, abort_flag, header)) break;
                if (!wait_or_abort(&ss.b1, par, abort_flag, header)) break;   // S(c) in B1
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s)  // descriptor start addresses advance in 16-byte units
                    mma_bf16(tmem + kT_XY + 64 * tb, d_a1 + (((s >> 2) * 16384 + (s & 3) * 32) >> 4),
                             d_b1 + ((s * 2048) >> 4), id_xy, s > 0);
                mma_commit(&ss.mma1);
                if (!wait_or_abort(&ss.b3, par, abort_flag, header)) break;   // diag(c) Delta(c) written
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kT_SA, d_kt + ((s * 2048) >> 4), d_b3 + ((s * 2048) >> 4), id_s, s > 0);
                mma_commit(&ss.mma3);
                if (!wait_or_abort(&ss.b2, par, abort_flag, header)) break;   // Delta(c) written
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + kT_PD + 64 * tb, d_up + ((s * 32) >> 4), d_b2 + ((s * 2048) >> 4), id_xy, s > 0);
                mma_commit(&ss.mma2[tb]);
                mma_commit(&ss.empty[b]);  // every MMA reading stage b has completed
            }
            if (*abort_flag) {  // drain: every MMA issued so far completes before TMEM is freed
                mma_commit(&ss.mma1);
                mbar_wait(&ss.mma1, c & 1);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------ bulk copies, two chunks ahead
        if (lane == 0) {
            int issued = 0;
            for (; issued < nch; ++issued) {
                const int st = issued % kStages;
                if (issued >= kStages &&
                    !wait_or_abort(&ss.empty[st], ((issued / kStages) - 1) & 1, abort_flag, header))
                    break;
                issue_chunk_loads(sm + st * kS_BUF, sm + kS_CV + st * kCvecLoad, &ss.full[st], ws, L,
                                  cs + issued, h, jq, half, hk, hv);
            }
            if (*abort_flag) {  // drain: copies in flight land before the CTA exits
                for (int j = max(0, issued - kStages); j < issued; ++j)
                    mbar_wait(&ss.full[j % kStages], (j / kStages) & 1);
            }
        }
    } else {
        // ------------------------------------------------ compute warps 0-7
        // warp w: TMEM lane quarter q4 = w & 3, column half ch2 = w >> 2 of this CTA's 64 d_v
        const int q4 = warp & 3, ch2 = warp >> 2;
        const int t = q4 * 32 + lane;       // d_k row of S^T this thread owns (state update)
        const int r = (q4 & 1) * 32 + lane; // token row (Delta: quarters 0-1; outputs: quarters 2-3)
        const bool delta_warp = q4 < 2;
        // fp32 state: S[half*64 + 32*ch2 + m][t], m = 0..31
        float S[32];
        const size_t sbase = ((size_t)n * hv + h) * kD * kD + (size_t)(half * 64 + 32 * ch2) * kD + t;
#pragma unroll
        for (int m = 0; m < 32; ++m) S[m] = s0 ? s0[sbase + (size_t)m * kD] : 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            *reinterpret_cast<uint4*>(sm + kS_B1 + sw128(t, 4 * ch2 + cc)) = pack8(S + 8 * cc);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&ss.b1);

        // Outputs of chunk c are written one chunk later (after the state update of c+1), so
        // that their global stores are not still in flight at the next shared-memory proxy
        // fence on the state chain.  Three TMEM accumulator sets keep chunk c's [X; Y] and
        // P Delta alive until then.
        float prev_gam = 0.f;
        auto write_outputs = [&](int cp, float gam_r) {
            const int tb = cp % kTBufs;
            if (!wait_or_abort(&ss.mma2[tb], (cp / kTBufs) & 1, abort_flag, header)) return false;
            tc_fence_after();
            const int t0 = t_begin + cp * kChunk;
            const int len = min(kChunk, t_end - t0);
            float y[32], pd[32];
            tmem_ld32(tmem, warp, kT_XY + 64 * tb + 32 * ch2, y);
            tmem_ld32(tmem, warp, kT_PD + 64 * tb + 32 * ch2, pd);
            if (r < len) {
                uint4* op = reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * hv + h) * kD + half * 64 + 32 * ch2);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float o8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o8[e] = fmaf(gam_r, y[8 * cc + e], pd[8 * cc + e]);
                    op[cc] = pack8(o8);
                }
            }
            tc_fence_before();
            return true;
        };
        int c = 0;
        for (; c < nch; ++c) {
            const int b = c % kStages, par = c & 1, tb = c % kTBufs;
            unsigned char* buf = sm + b * kS_BUF;
            if (!wait_or_abort(&ss.full[b], (c / kStages) & 1, abort_flag, header)) break;
            const float* cvec = reinterpret_cast<const float*>(sm + kS_CV + b * kCvecLoad);
            const float gl = cvec[128];
            const float crow = delta_warp ? cvec[r] : cvec[64 + r];  // c_r, or gam_r for outputs
            uint4 u4[4];  // this row's U values (Delta warps)
            if (delta_warp) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) u4[cc] = *reinterpret_cast<const uint4*>(buf + kS_U + sw128(r, 4 * ch2 + cc));
            }
            mbar_arrive(&ss.empty[b]);  // this thread's reads of stage b are done (values in registers)

            if (delta_warp) {  // Delta = U - X for token row r, columns 32*ch2 .. +32
                if (c >= 1 && !wait_or_abort(&ss.mma2[(c - 1) % kTBufs], ((c - 1) / kTBufs) & 1, abort_flag, header))
                    break;  // B2 and B3 are free once P Delta of c-1 is done
                if (!wait_or_abort(&ss.mma1, par, abort_flag, header)) break;
                tc_fence_after();
                float x[32];
                tmem_ld32(tmem, warp, kT_XY + 64 * tb + 32 * ch2, x);
                float d[32];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float u8[8];
                    unpack8(u4[cc], u8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) d[8 * cc + e] = u8[e] - x[8 * cc + e];
                }
                // diag(c) Delta first: it feeds the state update, the next link of the chain
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float c8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) c8[e] = d[8 * cc + e] * crow;
                    *reinterpret_cast<uint4*>(sm + kS_B3 + sw128(r, 4 * ch2 + cc)) = pack8(c8);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&ss.b3);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    *reinterpret_cast<uint4*>(sm + kS_B2 + sw128(r, 4 * ch2 + cc)) = pack8(d + 8 * cc);
                fence_async_smem();
                mbar_arrive(&ss.b2);
            }
            // state update S^T <- gam_L S^T + K^T diag(c) Delta (d_k row t, 32 d_v columns)
            if (!wait_or_abort(&ss.mma3, par, abort_flag, header)) break;
            tc_fence_after();
            {
                float acc[32];
                tmem_ld32(tmem, warp, kT_SA + 32 * ch2, acc);
#pragma unroll
                for (int m = 0; m < 32; ++m) S[m] = fmaf(gl, S[m], acc[m]);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    *reinterpret_cast<uint4*>(sm + kS_B1 + sw128(t, 4 * ch2 + cc)) = pack8(S + 8 * cc);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&ss.b1);

            if (!delta_warp) {  // outputs of the previous chunk: O = gam_r Y + P Delta
                if (c >= 1 && !write_outputs(c - 1, prev_gam)) break;
                prev_gam = crow;
            }
        }
        if (!delta_warp && c == nch && nch > 0 && !*abort_flag) write_outputs(nch - 1, prev_gam);
        if (!*abort_flag && sT) {
#pragma unroll
            for (int m = 0; m < 32; ++m) sT[sbase + (size_t)m * kD] = S[m];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

size_t tc_workspace_bytes(int num_seqs, int total_tokens, int hk, int hv) {
    return ws_layout(num_seqs, total_tokens, hk, hv).total;
}

cudaError_t launch_prefill_tc_prep(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const int32_t* cu, int num_seqs,
                                   int total_tokens, int hk, int hv, void* workspace,
                                   cudaStream_t stream) {
    if (num_seqs == 0) return cudaSuccess;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kPrepSmem);
    if (e != cudaSuccess) return e;
    chunk_table_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, ws);
    if (L.max_chunks > 0 && total_tokens > 0) {
        chunk_prep_kernel<<<(unsigned)(L.max_chunks * hk), kThreads, kPrepSmem, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, g, beta, ws,
            num_seqs, total_tokens, hk, hv);
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc_state(const float* s0, const int32_t* cu, void* out, float* sT,
                                    int num_seqs, int total_tokens, int hk, int hv,
                                    void* workspace, cudaStream_t stream) {
    if (num_seqs == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateSmem);
    if (e != cudaSuccess) return e;
    chunk_state_kernel<<<(unsigned)num_seqs * hv * 2, kStateThreads, kStateSmem, stream>>>(
        s0, cu, (__nv_bfloat16*)out, sT, static_cast<unsigned char*>(workspace), num_seqs,
        total_tokens, hk, hv);
    return cudaGetLastError();
}

}  // namespace gdn
