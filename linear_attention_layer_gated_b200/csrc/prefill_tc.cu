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
//  K1 chunk_prep_kernel   one CTA per (chunk, QK head), all chunks in parallel:
//                         normalisation, K K^T and Q K^T on tcgen05 (M=128: [K; Q] x K^T),
//                         decay masks, T by fp32 forward substitution, W^T = K^T (T diag(b gam))^T
//                         and U^T = V^T (T diag(b))^T on tcgen05, for both V heads of the QK
//                         head.  Writes bf16 operand images, already in the 128-byte
//                         swizzled layout the state kernel's MMAs read, to the workspace.
//  K2 chunk_state_kernel  one CTA per (sequence, V head, half of d_v), sequential over the
//                         sequence's chunks: [X; Y] = [W; diag(gam) Q] S^T (M=128),
//                         Delta = U - X, O = Y + P Delta (M=128 with a zero upper half),
//                         S^T <- gam_L S^T + K^T diag(c) Delta; the fp32 state slice lives in
//                         registers (one d_k row per thread), its bf16 copy in shared memory
//                         as the next chunk's MMA operand.  Chunk operands stream in with
//                         double-buffered bulk copies.
// Every mbarrier wait is bounded (1 s); on expiry the kernel records an error in the
// workspace header, drains its own copies and MMAs (again bounded), frees Tensor Memory
// and returns.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

// Operand image sizes (bytes)
constexpr uint32_t kA1Bytes = 32768;   // [W; diag(gam) Q]: 128 rows x 128 (K-major, 2 K-blocks)
constexpr uint32_t kUBytes = 16384;    // U: 2 halves of d_v, 64 rows x 64 each
constexpr uint32_t kPBytes = 8192;     // P: 64 rows x 64 (K-major)
constexpr uint32_t kCvecBytes = 512;   // c_j (64 floats) and gam_L at [64]
constexpr uint32_t kKTBytes = 16384;   // K as an MN-major operand (d_k x chunk)
constexpr uint32_t kChunkLoadBytes = kA1Bytes + kKTBytes + kPBytes + kUBytes / 2 + kCvecBytes;

struct WsLayout {
    size_t seq_chunk0, table, a1, u, p, cvec, kt, total;
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
    L.a1 = off;
    off += (size_t)L.max_chunks * hv * kA1Bytes;
    L.u = off;
    off += (size_t)L.max_chunks * hv * kUBytes;
    L.p = off;
    off += (size_t)L.max_chunks * hv * kPBytes;
    L.cvec = off;
    off += (size_t)L.max_chunks * hv * kCvecBytes;
    L.kt = off;
    off += (size_t)L.max_chunks * hk * kKTBytes;
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
__device__ __forceinline__ void st_shared_b16(uint32_t addr, float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(*reinterpret_cast<uint16_t*>(&h)) : "memory");
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

// ===================================================================== K1
// Shared memory map (bytes from a 1024-aligned base):
constexpr uint32_t kP_GRAM = 0;          // [K; Q] K-major, 32 KB   | later: V images (2 x 16 KB)
constexpr uint32_t kP_KT = 32768;        // K MN-major, 16 KB
constexpr uint32_t kP_AF = 49152;        // A fp32, 2 heads x 16 KB | later: W/U staging, head 0
constexpr uint32_t kP_B = 81920;         // T images: Bw0, Bu0, Bw1, Bu1 (8 KB each) | later: staging, head 1
constexpr uint32_t kP_SMALL = 114688;    // gates and barriers
constexpr uint32_t kPrepSmem = kP_SMALL + 2048 + 1024;

struct PrepSmall {
    float G[2][kChunk];
    float b[2][kChunk];
    float gam[2][kChunk];
    uint64_t bar_mma;
    uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 1)
chunk_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                  const float* __restrict__ beta, unsigned char* ws, int num_seqs,
                  int total_tokens, int hk, int hv) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    PrepSmall& ss = *reinterpret_cast<PrepSmall*>(sm + kP_SMALL);

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int cid = blockIdx.x / hk;
    const int jq = blockIdx.x % hk;
    if (cid >= header[1]) return;
    const int4 ent = reinterpret_cast<const int4*>(ws + L.table)[cid];
    const int t0 = ent.y, len = ent.z;
    const int group = hv / hk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- gates of the two V heads, barrier, TMEM
    if (warp < 2) {
        const int h = jq * group + warp;
        const float g0 = (lane < len) ? g[(size_t)(t0 + lane) * hv + h] : 0.f;
        const float g1 = (lane + 32 < len) ? g[(size_t)(t0 + lane + 32) * hv + h] : 0.f;
        const float G0 = warp_inclusive_scan(g0, lane);
        const float G1 = warp_inclusive_scan(g1, lane) + __shfl_sync(0xffffffffu, G0, 31);
        ss.G[warp][lane] = G0;
        ss.G[warp][lane + 32] = G1;
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
    int32_t err = 0;

    unsigned char* a1_base[2];
    for (int hh = 0; hh < 2; ++hh)
        a1_base[hh] = ws + L.a1 + ((size_t)cid * hv + jq * group + hh) * kA1Bytes;

    // ---- 1. normalise K and Q rows; K-major [K; Q], MN-major K, diag(gam) Q rows of A1
    {
        const int sub = tid & 7;             // 16 consecutive elements of a row
        const int kb = sub >> 2;             // 64-wide block of the row
        const int c0 = (sub & 3) * 2;        // first of two 16-byte chunks in the block
        for (int pass = 0; pass < 4; ++pass) {
            const int r = pass * 16 + (tid >> 3);
            float kv[16], qv[16];
            if (r < len) {
                const size_t base = ((size_t)(t0 + r) * hk + jq) * kD + sub * 16;
                const uint4* kp = reinterpret_cast<const uint4*>(k + base);
                const uint4* qp = reinterpret_cast<const uint4*>(q + base);
                unpack8(kp[0], kv);
                unpack8(kp[1], kv + 8);
                unpack8(qp[0], qv);
                unpack8(qp[1], qv + 8);
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) { kv[e] = 0.f; qv[e] = 0.f; }
            }
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
                *reinterpret_cast<uint4*>(sm + kP_GRAM + kb * 16384 + sw128(r, ch)) = kp8;
                *reinterpret_cast<uint4*>(sm + kP_GRAM + kb * 16384 + sw128(64 + r, ch)) = qp8;
                *reinterpret_cast<uint4*>(sm + kP_KT + kb * 8192 + sw128(r, ch)) = kp8;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float gm = ss.gam[hh][r];
                    float t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t8[e] = qv[8 * cc + e] * gm;
                    *reinterpret_cast<uint4*>(a1_base[hh] + kb * 16384 + sw128(64 + r, ch)) = pack8(t8);
                }
            }
        }
    }
    fence_async_smem();
    __syncthreads();

    // ---- 2. Gram: D[0:128, 0:64] = [K; Q] K^T  (M=128, N=64, K=128)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t a = sb + kP_GRAM + (s >> 2) * 16384 + (s & 3) * 32;
            mma_bf16(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), idesc, s > 0);
        }
        mma_commit(&ss.bar_mma);
        // K as MN-major operand image -> workspace (read by the state kernel)
        bulk_s2g(ws + L.kt + ((size_t)cid * hk + jq) * kKTBytes, sm + kP_KT, kKTBytes);
        bulk_commit();
    }
    bool ok = mbar_wait(&ss.bar_mma, 0);
    if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
    tc_fence_after();

    // ---- 3. decay masks: A (fp32, smem) from K K^T rows; P (bf16, workspace) from Q K^T rows
    {
        float row[64];
        tmem_ld64(tmem, warp, 0, row);
        const int r = tid & 63;
        if (warp < 2) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float Gr = ss.G[hh][r], br = ss.b[hh][r];
                float4* af = reinterpret_cast<float4*>(sm + kP_AF + hh * 16384);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    float a4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * m + e;
                        a4[e] = (i < r) ? br * expf(Gr - ss.G[hh][i]) * row[i] : 0.f;
                    }
                    af[r * 16 + (m ^ (r & 15))] = make_float4(a4[0], a4[1], a4[2], a4[3]);
                }
            }
        } else {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int h = jq * group + hh;
                const float Gr = ss.G[hh][r];
                unsigned char* pimg = ws + L.p + ((size_t)cid * hv + h) * kPBytes;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float p8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 8 * ch + e;
                        p8[e] = (i <= r) ? expf(Gr - ss.G[hh][i]) * row[i] : 0.f;
                    }
                    *reinterpret_cast<uint4*>(pimg + sw128(r, ch)) = pack8(p8);
                }
                float* cv = reinterpret_cast<float*>(ws + L.cvec + ((size_t)cid * hv + h) * kCvecBytes);
                const float Gl = ss.G[hh][len - 1];
                cv[r] = (r < len) ? expf(Gl - Gr) : 0.f;
                if (r == 0) cv[64] = expf(Gl);
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- 4. V images (MN-major, into the dead [K; Q] region), then T = (I + A)^-1
    {
        const int sub = tid & 7, kb = sub >> 2, c0 = (sub & 3) * 2;
        for (int hh = 0; hh < 2; ++hh) {
            const int h = jq * group + hh;
            for (int pass = 0; pass < 4; ++pass) {
                const int r = pass * 16 + (tid >> 3);
                uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
                if (r < len) {
                    const uint4* vp = reinterpret_cast<const uint4*>(v + ((size_t)(t0 + r) * hv + h) * kD + sub * 16);
                    u0 = vp[0];
                    u1 = vp[1];
                }
                *reinterpret_cast<uint4*>(sm + kP_GRAM + hh * 16384 + kb * 8192 + sw128(r, c0)) = u0;
                *reinterpret_cast<uint4*>(sm + kP_GRAM + hh * 16384 + kb * 8192 + sw128(r, c0 + 1)) = u1;
            }
        }
    }
    {
        const int hh = tid >> 6, i = tid & 63;
        const float4* af = reinterpret_cast<const float4*>(sm + kP_AF + hh * 16384);
        float x[kChunk];
#pragma unroll
        for (int r = 0; r < kChunk; ++r) x[r] = 0.f;
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int m = 0; m < (r + 3) / 4; ++m) {
                const float4 av = af[r * 16 + (m ^ (r & 15))];
                a0 = fmaf(av.x, x[4 * m + 0], a0);
                a1 = fmaf(av.y, x[4 * m + 1], a1);
                a2 = fmaf(av.z, x[4 * m + 2], a2);
                a3 = fmaf(av.w, x[4 * m + 3], a3);
            }
            x[r] = (r == i) ? 1.f : ((r < i) ? 0.f : -((a0 + a1) + (a2 + a3)));
        }
        // B operands (K-major, row r, K index i): T diag(b gam) for W, T diag(b) for U
        const float bi = ss.b[hh][i], bgi = bi * ss.gam[hh][i];
        const uint32_t bw = sb + kP_B + hh * 16384, bu = bw + 8192;
        const uint32_t colo = (uint32_t)(i & 7) * 2;
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
            const uint32_t o = sw128(r, i >> 3) + colo;
            st_shared_b16(bw + o, x[r] * bgi);
            st_shared_b16(bu + o, x[r] * bi);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- 5. W^T = K^T (T diag(b gam))^T, U^T = V^T (T diag(b))^T  (M=128, N=64, K=64 each)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, 1, 0);
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t bw = sb + kP_B + hh * 16384, bu = bw + 8192;
            const uint32_t vimg = sb + kP_GRAM + hh * 16384;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                mma_bf16(tmem + 128 * hh, sdesc_sw128(sb + kP_KT + s * 2048, 8192, 1024),
                         sdesc_sw128(bw + s * 32, 16, 1024), idesc, s > 0);
                mma_bf16(tmem + 128 * hh + 64, sdesc_sw128(vimg + s * 2048, 8192, 1024),
                         sdesc_sw128(bu + s * 32, 16, 1024), idesc, s > 0);
            }
        }
        mma_commit(&ss.bar_mma);
    }
    ok = mbar_wait(&ss.bar_mma, 1);
    if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
    tc_fence_after();

    // ---- 6. epilogue: W rows 0..63 of A1 and U, staged K-major, bulk-stored
    for (int hh = 0; hh < 2; ++hh) {
        const int h = jq * group + hh;
        unsigned char* stage = sm + (hh == 0 ? kP_AF : kP_B);
        const int t = tid;  // TMEM lane = d_k (for W) or d_v (for U) index
        const uint32_t so = (uint32_t)(t >> 6) * 8192, ch = (uint32_t)(t & 63) >> 3, colo = (uint32_t)(t & 7) * 2;
        float col[64];
        tmem_ld64(tmem, warp, 128 * hh, col);
#pragma unroll
        for (int r = 0; r < kChunk; ++r) st_shared_b16(smem_u32(stage) + so + sw128(r, ch) + colo, col[r]);
        tmem_ld64(tmem, warp, 128 * hh + 64, col);
#pragma unroll
        for (int r = 0; r < kChunk; ++r) st_shared_b16(smem_u32(stage) + 16384 + so + sw128(r, ch) + colo, col[r]);
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            unsigned char* a1 = ws + L.a1 + ((size_t)cid * hv + h) * kA1Bytes;
            bulk_s2g(a1, stage, 8192);              // W rows, d_k 0..63
            bulk_s2g(a1 + 16384, stage + 8192, 8192);  // W rows, d_k 64..127
            bulk_s2g(ws + L.u + ((size_t)cid * hv + h) * kUBytes, stage + 16384, kUBytes);
            bulk_commit();
        }
    }

cleanup:
    if (err) {
        if (tid == 0) {
            atomicOr(header, 1);
            mma_commit(&ss.bar_mma);  // all MMAs issued so far complete before TMEM is freed
        }
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ===================================================================== K2
constexpr uint32_t kS_A1 = 0, kS_KT = 32768, kS_A2 = 49152, kS_U = 65536, kS_CV = 73728;
constexpr uint32_t kS_BUF = 74752;                  // one chunk buffer (73 KB)
constexpr uint32_t kS_B1 = 2 * kS_BUF;              // S slice bf16, MN-major (16 KB)
constexpr uint32_t kS_B2 = kS_B1 + 16384;           // Delta, MN-major (8 KB)
constexpr uint32_t kS_B3 = kS_B2 + 8192;            // diag(c) Delta, MN-major (8 KB)
constexpr uint32_t kS_SMALL = kS_B3 + 8192;
constexpr uint32_t kStateSmem = kS_SMALL + 256 + 1024;

struct StateSmall {
    uint64_t full[2];
    uint64_t bar_mma1, bar_mma23;
    uint32_t tmem_base;
};

__device__ __forceinline__ void issue_chunk_loads(unsigned char* buf, uint64_t* bar, const unsigned char* ws,
                                                  const WsLayout& L, int cid, int h, int jq, int half,
                                                  int hk, int hv) {
    mbar_arrive_expect_tx(bar, kChunkLoadBytes);
    bulk_g2s(buf + kS_A1, ws + L.a1 + ((size_t)cid * hv + h) * kA1Bytes, kA1Bytes, bar);
    bulk_g2s(buf + kS_KT, ws + L.kt + ((size_t)cid * hk + jq) * kKTBytes, kKTBytes, bar);
    bulk_g2s(buf + kS_A2 + 8192, ws + L.p + ((size_t)cid * hv + h) * kPBytes, kPBytes, bar);
    bulk_g2s(buf + kS_U, ws + L.u + ((size_t)cid * hv + h) * kUBytes + half * (kUBytes / 2), kUBytes / 2, bar);
    bulk_g2s(buf + kS_CV, ws + L.cvec + ((size_t)cid * hv + h) * kCvecBytes, kCvecBytes, bar);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_state_kernel(const float* s0, const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out,
                   float* sT, unsigned char* ws, int num_seqs, int total_tokens, int hk, int hv) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + kS_SMALL);

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int half = blockIdx.x & 1;
    const int h = (blockIdx.x >> 1) % hv;
    const int n = (blockIdx.x >> 1) / hv;
    const int jq = h / (hv / hk);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int32_t* seq_chunk0 = reinterpret_cast<const int32_t*>(ws + L.seq_chunk0);
    const int cs = seq_chunk0[n], nch = seq_chunk0[n + 1] - cs;
    const int t_begin = cu[n], t_end = cu[n + 1];

    // zero the upper (unused) 64 rows of both P operands
    for (int i = tid; i < 2 * 512; i += kThreads) {
        const int b = i >> 9, o = (i & 511) * 16;
        *reinterpret_cast<uint4*>(sm + b * kS_BUF + kS_A2 + o) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 0) {
        tmem_alloc(&ss.tmem_base, 128);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&ss.full[0], 1);
        mbar_init(&ss.full[1], 1);
        mbar_init(&ss.bar_mma1, 1);
        mbar_init(&ss.bar_mma23, 1);
        fence_mbar_init();
    }

    // fp32 state slice: thread t owns S[half*64 + m][t], m = 0..63 (column t of S)
    const int t = tid;
    float S[64];
    const size_t sbase = ((size_t)n * hv + h) * kD * kD + (size_t)(half * 64) * kD + t;
#pragma unroll
    for (int m = 0; m < 64; ++m) S[m] = s0 ? s0[sbase + (size_t)m * kD] : 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(sm + kS_B1 + sw128(t, ch)) = pack8(S + 8 * ch);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;
    if (tid == 0) {
        for (int kk = 0; kk < 2 && kk < nch; ++kk)
            issue_chunk_loads(sm + kk * kS_BUF, &ss.full[kk], ws, L, cs + kk, h, jq, half, hk, hv);
    }

    const uint32_t id_xy = idesc_bf16(128, 64, 0, 1);   // A K-major, B MN-major
    const uint32_t id_s = idesc_bf16(128, 64, 1, 1);    // A MN-major, B MN-major
    int err = 0;
    int kk = 0;
    for (; kk < nch; ++kk) {
        const int b = kk & 1;
        unsigned char* buf = sm + b * kS_BUF;
        const uint32_t bufa = sb + b * kS_BUF;
        const int t0 = t_begin + kk * kChunk;
        const int len = min(kChunk, t_end - t0);
        bool ok = mbar_wait(&ss.full[b], (kk >> 1) & 1);
        if (__syncthreads_or(!ok)) { err = 1; break; }
        const float* cvec = reinterpret_cast<const float*>(buf + kS_CV);
        const float gl = cvec[64];

        // [X; Y] = [W; diag(gam) Q] S^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tmem, sdesc_sw128(bufa + kS_A1 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         sdesc_sw128(sb + kS_B1 + s * 2048, 16384, 1024), id_xy, s > 0);
            mma_commit(&ss.bar_mma1);
        }
        ok = mbar_wait(&ss.bar_mma1, kk & 1);
        if (__syncthreads_or(!ok)) { err = 1; break; }
        tc_fence_after();

        if (warp < 2) {  // Delta = U - X for token row r; write Delta and diag(c) Delta
            const int r = tid;
            float x[64];
            tmem_ld64(tmem, warp, 0, x);
            const float cr = cvec[r];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float u8[8], d8[8], c8[8];
                unpack8(*reinterpret_cast<const uint4*>(buf + kS_U + sw128(r, ch)), u8);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    d8[e] = u8[e] - x[8 * ch + e];
                    c8[e] = d8[e] * cr;
                }
                *reinterpret_cast<uint4*>(sm + kS_B2 + sw128(r, ch)) = pack8(d8);
                *reinterpret_cast<uint4*>(sm + kS_B3 + sw128(r, ch)) = pack8(c8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // Y += P Delta (rows 64..127 of the accumulator), S-update = K^T diag(c) Delta
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem, sdesc_sw128(bufa + kS_A2 + s * 32, 16, 1024),
                         sdesc_sw128(sb + kS_B2 + s * 2048, 8192, 1024), id_xy, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem + 64, sdesc_sw128(bufa + kS_KT + s * 2048, 8192, 1024),
                         sdesc_sw128(sb + kS_B3 + s * 2048, 8192, 1024), id_s, s > 0);
            mma_commit(&ss.bar_mma23);
        }
        ok = mbar_wait(&ss.bar_mma23, kk & 1);
        if (__syncthreads_or(!ok)) { err = 1; break; }
        tc_fence_after();
        if (tid == 0 && kk + 2 < nch)
            issue_chunk_loads(buf, &ss.full[b], ws, L, cs + kk + 2, h, jq, half, hk, hv);

        if (warp >= 2) {  // outputs of token row r
            const int r = tid - 64;
            float y[64];
            tmem_ld64(tmem, warp, 0, y);
            if (r < len) {
                uint4* op = reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * hv + h) * kD + half * 64);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) op[ch] = pack8(y + 8 * ch);
            }
        }
        {
            float acc[64];
            tmem_ld64(tmem, warp, 64, acc);
#pragma unroll
            for (int m = 0; m < 64; ++m) S[m] = fmaf(gl, S[m], acc[m]);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4*>(sm + kS_B1 + sw128(t, ch)) = pack8(S + 8 * ch);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (err) {
        if (tid == 0) {
            atomicOr(header, 1);
            // drain: MMAs issued so far, and chunk loads still in flight (bounded waits)
            mma_commit(&ss.bar_mma1);
            mbar_wait(&ss.bar_mma1, kk & 1);
            for (int j = kk; j < nch && j < kk + 2; ++j) mbar_wait(&ss.full[j & 1], (j >> 1) & 1);
        }
    } else if (sT) {
#pragma unroll
        for (int m = 0; m < 64; ++m) sT[sbase + (size_t)m * kD] = S[m];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
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
    chunk_state_kernel<<<(unsigned)num_seqs * hv * 2, kThreads, kStateSmem, stream>>>(
        s0, cu, (__nv_bfloat16*)out, sT, static_cast<unsigned char*>(workspace), num_seqs,
        total_tokens, hk, hv);
    return cudaGetLastError();
}

}  // namespace gdn
