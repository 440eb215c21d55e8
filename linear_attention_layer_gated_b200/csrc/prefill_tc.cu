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
//  K0 chunk_table_kernel  clears the workspace's device error word; cu_seqlens -> per-sequence
//                         first chunk id and a (seq, start, length) entry per chunk, on the
//                         device (no host read).
//  K1 chunk_prep_kernel   one CTA (256 threads) per (chunk, QK head), all chunks in
//                         parallel, both V heads of the QK head:
//                         - normalisation; Q K^T, K K^T and the cross Gram K K_prev^T with
//                           the previous chunk's keys as one M=128, N=128 MMA;
//                         - decay masks A and P; T = (I + A)^-1 in fp32 by 32x32 blocks
//                           (forward substitution per diagonal block, then one off-diagonal
//                           block as two dense products);
//                         - W and U of both heads as M=128 MMAs [T_0 D_0; T_1 D_1] x (K or V),
//                           and M~ = [T D] (K K_prev^T) diag(c_prev);
//                         - bf16 operand images, already in the 128-byte swizzled layout the
//                           state kernel's MMAs read, go to the workspace: W~ = gam_L,prev W,
//                           U, P, M~, diag(c) K per V head and Q per QK head, with the gate
//                           factors (c, gam) of each V head.
//  K2 chunk_state_kernel  one CTA per (sequence, V head, quarter of d_v), sequential over the
//                         sequence's chunks, in the look-ahead form described at the kernel.
// Every mbarrier wait is bounded (1 s) and, in the state kernel, also gives up as soon as
// another thread of the CTA has given up; the kernel then records an error in the
// workspace header, drains its own copies and MMAs (bounded), frees Tensor Memory and
// returns.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

// Operand image sizes (bytes)
constexpr uint32_t kWBytes = 16384;    // W: 64 token rows x 128 d_k, K-major, [K-block][64 rows]
constexpr uint32_t kQBytes = 16384;    // normalised Q, same layout (per QK head)
constexpr uint32_t kUBytes = 16384;    // U: [d_v half][64 rows][64]
constexpr uint32_t kPBytes = 8192;     // P: 64 token rows x 64, K-major
constexpr uint32_t kCvecBytes = 1024;  // c_j at [0,64), gam_r at [64,128), gam_L at [128]
constexpr uint32_t kCvecLoad = 528;    // the bytes of a gate-factor record the state kernel reads
constexpr uint32_t kKTBytes = 16384;   // diag(c) K (per V head), [d_k block][64 token rows] (MN-major A operand)
constexpr uint32_t kMBytes = 8192;     // M = W K_prev^T diag(c_prev): 64 token rows x 64 previous-chunk tokens,
                                       // K-major

struct WsLayout {
    size_t seq_chunk0, table, w, u, p, cvec, kt, qn, m, total;
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
    off += (size_t)L.max_chunks * hv * kKTBytes;
    L.qn = off;
    off += (size_t)L.max_chunks * hk * kQBytes;
    L.m = off;
    off += (size_t)L.max_chunks * hv * kMBytes;
    L.total = round_up(off, 1024);
    return L;
}

// ===================================================================== K0
__global__ void __launch_bounds__(1024)
chunk_table_kernel(const int32_t* __restrict__ cu, int num_seqs, unsigned char* ws) {
    allow_dependent_launch();
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    if (threadIdx.x == 0) header[0] = 0;  // the device error word of this call
    const WsLayout L = ws_layout(num_seqs, 0, 1, 1);  // seq_chunk0 and table do not depend on T
    int32_t* seq_chunk0 = reinterpret_cast<int32_t*>(ws + L.seq_chunk0);
    int4* table = reinterpret_cast<int4*>(ws + L.table);
    __shared__ int32_t scan[1024];
    __shared__ int32_t carry;
    // up to 1024 sequences: chunk starts and cu_seqlens stay in shared memory for the entries
    __shared__ int32_t start_s[1025], cu_s[1025];
    const bool small = num_seqs <= 1024;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + threadIdx.x;
        const int c0n = (n < num_seqs) ? cu[n] : 0, c1n = (n < num_seqs) ? cu[n + 1] : 0;
        const int cnt = (n < num_seqs) ? (c1n - c0n + kChunk - 1) / kChunk : 0;
        if (small && n < num_seqs) {
            cu_s[n] = c0n;
            if (n == num_seqs - 1) cu_s[num_seqs] = c1n;
        }
        scan[threadIdx.x] = cnt;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {  // inclusive Hillis-Steele scan
            const int add = (threadIdx.x >= o) ? scan[threadIdx.x - o] : 0;
            __syncthreads();
            scan[threadIdx.x] += add;
            __syncthreads();
        }
        if (n < num_seqs) {
            seq_chunk0[n] = carry + scan[threadIdx.x] - cnt;
            if (small) start_s[n] = carry + scan[threadIdx.x] - cnt;
        }
        __syncthreads();
        if (threadIdx.x == 1023) carry += scan[1023];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        seq_chunk0[num_seqs] = carry;
        header[1] = carry;
        if (small) start_s[num_seqs] = carry;
    }
    __syncthreads();
    // one entry per thread: chunk c belongs to the last sequence n with seq_chunk0[n] <= c
    const int total = carry;
    const int32_t* starts = small ? start_s : seq_chunk0;
    const int32_t* cus = small ? cu_s : cu;
    for (int c = threadIdx.x; c < total; c += blockDim.x) {
        int lo = 0, hi = num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= c) lo = mid;
            else hi = mid - 1;
        }
        const int n = lo, kk = c - starts[n];
        const int t0 = cus[n], len = cus[n + 1] - t0;
        table[c] = make_int4(n, t0 + kk * kChunk, min(kChunk, len - kk * kChunk), 0);
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
//   kP_GR  per d_k block b (b = 0, 1) at b * kP_GRB: rows of Q | K | K_prev (8 KB each), K-major.
//          The Gram MMA reads A = [Q; K] and B = [K; K_prev] (128 rows each) from it.  After
//          the Gram, the Q and K_prev slots take the V images of both heads; the K slot stays
//          (it is the MN-major B operand of W = [T D] K).
//   kP_GX  K K_prev^T in bf16, MN-major B operand of M = [T D] (K K_prev^T) (8 KB)
//   kP_AF  at entry: raw K_prev rows (16 KB); then A / T fp32 (2 heads x 17 KB); then the
//          [T0 D0; T1 D1] and [T0 B0; T1 B1] operand images (2 x 16 KB)
constexpr uint32_t kP_GR = 0;
constexpr uint32_t kP_GRB = 24576;
constexpr uint32_t kP_GX = 2 * kP_GRB;
constexpr uint32_t kP_AF = kP_GX + 8192;
constexpr uint32_t kP_SMALL = kP_AF + 2 * kAfHead * 4;  // gates, barrier, TMEM address
constexpr uint32_t kPrepSmem = kP_SMALL + 3072 + 1024;  // small struct + alignment slack

struct PrepSmall {
    float G[2][kChunk];   // in-chunk gate sums, pre-scaled by log2(e)
    float b[2][kChunk];
    float gam[2][kChunk];
    float cprev[2][kChunk];  // c of the previous chunk, exp(G_L - G_j), or 0 (16-byte aligned)
    float gprev[2];       // exp(total gate sum of the previous chunk of the sequence), or 1
    uint64_t bar_mma;
    uint32_t tmem_base;
};
static_assert(sizeof(PrepSmall) <= 3072, "PrepSmall fits its region");

// 256 threads: warp w reads Tensor Memory lane quarter w % 4; the two warps of a quarter
// split the columns (column half hf = w / 4).
constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads, 2)
chunk_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                  const float* __restrict__ beta, unsigned char* ws, int num_seqs,
                  int total_tokens, int hk, int hv, int resident) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    PrepSmall& ss = *reinterpret_cast<PrepSmall*>(sm + kP_SMALL);
    float* af = reinterpret_cast<float*>(sm + kP_AF);   // [head][64][kLdA]

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int cid = blockIdx.x / hk;
    const int jq = blockIdx.x % hk;
    grid_dependency_wait();    // the chunk table is written
    allow_dependent_launch();  // the state kernel may be scheduled as SMs free up
    const int nchunks = header[1];
    if (cid >= nchunks) return;
    const int4 ent = reinterpret_cast<const int4*>(ws + L.table)[cid];
    // The CTA that takes this one's place on the SM (CTAs start in index order, `resident`
    // at a time): its chunk entry, for the L2 prefetch of its inputs in phase 3.
    const int nb = blockIdx.x + resident;
    const int ncid = nb / hk, njq = nb % hk;
    const int4 nent = (ncid < nchunks) ? reinterpret_cast<const int4*>(ws + L.table)[ncid] : make_int4(0, 0, 0, 0);
    const int t0 = ent.y, len = ent.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qw = warp & 3, hf = warp >> 2;  // TMEM lane quarter, column half
    const int h0 = jq * 2;  // the two V heads of this QK head
    // The previous chunk (always a full one) belongs to the same sequence unless this chunk
    // is the sequence's first.
    const bool has_prev = cid > reinterpret_cast<const int32_t*>(ws + L.seq_chunk0)[ent.x];

    // Row loads: 8 threads per row, 16 elements (2 chunks of one 64-wide block) each;
    // 32 rows per pass.
    const int sub = tid & 7, kb = sub >> 2, c0 = (sub & 3) * 2;
    int err = 0;
    bool ok;

    // ---- 0. loads: each thread stages (async) exactly the K_prev pieces it normalises
    //         below, and loads its q, k rows (2 passes); warps 0-1 the gates; TMEM; barrier
    if (has_prev) {
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int r = pass * 32 + (tid >> 3);
            const __nv_bfloat16* src = k + ((size_t)(t0 - kChunk + r) * hk + jq) * kD + sub * 16;
            cp_async16(sm + kP_AF + r * 256 + sub * 32, src);
            cp_async16(sm + kP_AF + r * 256 + sub * 32 + 16, src + 8);
        }
        cp_async_commit();
    }
    uint4 kr[2][2], qr[2][2];
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const int r = pass * 32 + (tid >> 3);
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
        const float gp0 = has_prev ? g[(size_t)(t0 - kChunk + lane) * hv + h] : 0.f;
        const float gp1 = has_prev ? g[(size_t)(t0 - kChunk + 32 + lane) * hv + h] : 0.f;
        const float b0 = (lane < len) ? beta[(size_t)(t0 + lane) * hv + h] : 0.f;
        const float b1 = (lane + 32 < len) ? beta[(size_t)(t0 + lane + 32) * hv + h] : 0.f;
        const float G0 = warp_inclusive_scan(g0, lane);
        const float G1 = warp_inclusive_scan(g1, lane) + __shfl_sync(0xffffffffu, G0, 31);
        ss.G[warp][lane] = G0 * kLog2e;
        ss.G[warp][lane + 32] = G1 * kLog2e;
        ss.gam[warp][lane] = expf(G0);
        ss.gam[warp][lane + 32] = expf(G1);
        ss.b[warp][lane] = b0;
        ss.b[warp][lane + 32] = b1;
        const float Gp0 = warp_inclusive_scan(gp0, lane);
        const float Gp1 = warp_inclusive_scan(gp1, lane) + __shfl_sync(0xffffffffu, Gp0, 31);
        const float GpL = __shfl_sync(0xffffffffu, Gp1, 31);
        ss.cprev[warp][lane] = has_prev ? expf(GpL - Gp0) : 0.f;
        ss.cprev[warp][lane + 32] = has_prev ? expf(GpL - Gp1) : 0.f;
        if (lane == 0) ss.gprev[warp] = has_prev ? expf(GpL) : 1.f;
    }
    if (warp == 3) {
        tmem_alloc(&ss.tmem_base, 256);
        tmem_relinquish();
    }
    if (tid == 64) {
        mbar_init(&ss.bar_mma, 1);
        fence_mbar_init();
    }

    // ---- 1. normalise q, k and K_prev rows into their K-major smem slots (no dependency on
    //         the gates, so no barrier before it).  (Global stores wait until after the proxy
    //         fences below: a fence.proxy.async also waits for the thread's stores in flight,
    //         so each phase writes shared memory, fences, and only then stores to the
    //         workspace.)
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const int r = pass * 32 + (tid >> 3);
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
            *reinterpret_cast<uint4*>(sm + kP_GR + kb * kP_GRB + sw128(r, ch)) = pack8(qv + 8 * cc);
            *reinterpret_cast<uint4*>(sm + kP_GR + kb * kP_GRB + 8192 + sw128(r, ch)) = pack8(kv + 8 * cc);
        }
    }
    if (has_prev) cp_async_wait_all();  // this thread's own staged pieces
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int r = pass * 32 + (tid >> 3);
        float kv[16];
        if (has_prev) {
            const uint4* src = reinterpret_cast<const uint4*>(sm + kP_AF + r * 256 + sub * 32);
            unpack8(src[0], kv);
            unpack8(src[1], kv + 8);
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) kv[e] = 0.f;
        }
        float ssk = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) ssk = fmaf(kv[e], kv[e], ssk);
        const float rk = rsqrtf(sum8(ssk) + kNormEps);
#pragma unroll
        for (int e = 0; e < 16; ++e) kv[e] *= rk;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
            *reinterpret_cast<uint4*>(sm + kP_GR + kb * kP_GRB + 16384 + sw128(r, c0 + cc)) = pack8(kv + 8 * cc);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // gates, TMEM address, barrier and the three row slots are ready
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;

    // ---- 2. Gram: TMEM[0:128, 0:128] = [Q; K] [K; K_prev]^T  (M=128, N=128, K=128); V loads
    //         meanwhile.  Rows 0..63: Q K^T | Q K_prev^T (unused); rows 64..127: K K^T | K K_prev^T.
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t a = sb + kP_GR + (s >> 2) * kP_GRB + (s & 3) * 32;
            mma_bf16(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(a + 8192, 16, 1024), idesc, s > 0);
        }
        mma_commit(&ss.bar_mma);
    }
    if (tid == 32) {  // the Q image is the Q slot as it stands: two 8 KB bulk stores
        unsigned char* qn_img = ws + L.qn + ((size_t)cid * hk + jq) * kQBytes;
        bulk_s2g(qn_img, sm + kP_GR, 8192);
        bulk_s2g(qn_img + 8192, sm + kP_GR + kP_GRB, 8192);
        bulk_commit();
    }
    {
        uint4 vr[2][2][2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                const int r = pass * 32 + (tid >> 3);
                if (r < len) {
                    const uint4* vp = reinterpret_cast<const uint4*>(v + ((size_t)(t0 + r) * hv + h0 + hh) * kD + sub * 16);
                    vr[hh][pass][0] = vp[0];
                    vr[hh][pass][1] = vp[1];
                } else {
                    vr[hh][pass][0] = vr[hh][pass][1] = make_uint4(0, 0, 0, 0);
                }
            }
        // gate factors of both heads to the workspace (warps 0-1; token row r)
        if (warp < 2) {
            const int r = tid;
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
        if (tid == 32) bulk_wait_read_all();  // the Q slot is read before V overwrites it
        if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
        tc_fence_after();

        // ---- 3. from the Gram rows, columns 32 hf .. 32 hf + 31 of each block:
        //         warps of quarters 0-1 (Q rows): P = lower(exp(G_r - G_j) Q K^T) of both heads
        //         to the workspace; quarters 2-3 (K rows): A = strictly_lower(b_r exp(G_r - G_j)
        //         K K^T) in fp32 -- the two 32x32 diagonal blocks stored transposed, for the
        //         forward substitution -- and the bf16 image of K K_prev^T.
        float row[32];
        const uint32_t ta = tmem + ((uint32_t)qw * 32u << 16) + 32u * hf;
        const int r = (qw & 1) * 32 + lane;  // token row
        const int j0 = 32 * hf;              // first column of this thread
        if (qw >= 2) {
            tmem_ld16(ta, row);
            tmem_ld16(ta + 16, row + 16);
            tmem_ld_wait();
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const float Gr = ss.G[hh][r], br = ss.b[hh][r];
                const float* gj = ss.G[hh] + j0;
                float* A = af + hh * kAfHead;
                float a[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    a[e] = (j0 + e < r) ? br * fast_exp2(fminf(Gr - gj[e], 0.f)) * row[e] : 0.f;
                if ((r >> 5) == hf) {  // diagonal block, transposed: A^T[j][r]
#pragma unroll
                    for (int e = 0; e < 32; ++e) A[(j0 + e) * kLdA + r] = a[e];
                } else if (hf < (r >> 5)) {  // A21, row-major
                    float4* a4 = reinterpret_cast<float4*>(A + r * kLdA + j0);
#pragma unroll
                    for (int m = 0; m < 8; ++m) a4[m] = make_float4(a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3]);
                }
            }
            tmem_ld16(ta + 64, row);
            tmem_ld16(ta + 80, row + 16);
            tmem_ld_wait();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                *reinterpret_cast<uint4*>(sm + kP_GX + sw128(r, 4 * hf + ch)) = pack8(row + 8 * ch);
        }
        // V images (MN-major: token row, d_v contiguous; d_v blocks kP_GRB apart) into the
        // dead Q (head 0) and K_prev (head 1) slots
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                const int rr = pass * 32 + (tid >> 3);
                unsigned char* vb = sm + kP_GR + hh * 16384 + kb * kP_GRB;
                *reinterpret_cast<uint4*>(vb + sw128(rr, c0)) = vr[hh][pass][0];
                *reinterpret_cast<uint4*>(vb + sw128(rr, c0 + 1)) = vr[hh][pass][1];
            }
        fence_async_smem();
        // This CTA's own loads are done: ask L2 for the next CTA's q, k (one 128-byte line per
        // thread), v of both heads (four lines per token) and gates.  Its K_prev rows and
        // previous gates belong to the chunk before it, which a CTA now running has just read.
        if (nent.z > 0) {
            const int nt0 = nent.y, nlen = nent.z;
            const int pr = tid >> 1, pl = tid & 1;
            if ((pr & 63) < nlen) {
                const __nv_bfloat16* src = (pr < 64 ? q : k) + ((size_t)(nt0 + (pr & 63)) * hk + njq) * kD + pl * 64;
                prefetch_l2(src);
            }
            const int vrow = tid >> 2, vl = tid & 3;
            if (vrow < nlen) prefetch_l2(v + ((size_t)(nt0 + vrow) * hv + 2 * njq) * kD + vl * 64);
            if (tid < 128 && (tid & 63) < nlen)
                prefetch_l2((tid < 64 ? g : beta) + (size_t)(nt0 + (tid & 63)) * hv + 2 * njq);
        }
        if (qw < 2) {  // P rows, after the fence: these stores may stay in flight
            tmem_ld16(ta, row);
            tmem_ld16(ta + 16, row + 16);
            tmem_ld_wait();
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const float Gr = ss.G[hh][r];
                const float* gj = ss.G[hh] + j0;
                unsigned char* pimg = ws + L.p + ((size_t)cid * hv + h0 + hh) * kPBytes;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    float p8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = j0 + 8 * ch + e;
                        p8[e] = (i <= r) ? fast_exp2(fminf(Gr - gj[8 * ch + e], 0.f)) * row[8 * ch + e] : 0.f;
                    }
                    *reinterpret_cast<uint4*>(pimg + sw128(r, 4 * hf + ch)) = pack8(p8);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- 4. T = (I + A)^-1 per head, by 32x32 blocks, in place; 128 threads per head.
    //         With A = [A11 0; A21 A22]:  T = [T1 0; T21 T2], T1 = (I + A11)^-1,
    //         T2 = (I + A22)^-1, T21 = -T2 (A21 T1).
    //         (a) T1 and T2 by forward substitution, one warp per block, lane = column j,
    //             column-oriented: once x_k is known every later row's partial sum takes its
    //             term (independent updates), reading row k of the transposed block;
    //         (b) Y = A21 T1 into the (zero) upper-right block, then T21 = -T2 Y, each thread
    //             a 4x2 tile; the upper-right block is cleared again afterwards.
    {
        const int hh = tid >> 7, l = tid & 127;
        float* A = af + hh * kAfHead;
        if (l < 64) {
            const int base = 32 * (l >> 5), j = l & 31;
            float acc[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) acc[r] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
                const float xk = (kk == j) ? 1.f : ((kk < j) ? 0.f : -acc[kk]);
                acc[kk] = xk;
                const float4* at = reinterpret_cast<const float4*>(A + (base + kk) * kLdA + base);  // A^T row kk
#pragma unroll
                for (int r4 = (kk + 1) / 4; r4 < 8; ++r4) {
                    const float4 a = at[r4];
                    const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * r4 + e > kk) acc[4 * r4 + e] = fmaf(av[e], xk, acc[4 * r4 + e]);
                }
            }
            __syncwarp();  // every lane of this block's warp is done reading A^T
#pragma unroll
            for (int r = 0; r < 32; ++r) A[(base + r) * kLdA + base + j] = acc[r];
        } else {
            // meanwhile the other 64 threads of the head write its diag(c) K image from the
            // K slot, rows scaled by c_r = exp(G_L - G_r) (0 beyond the chunk's length); eight
            // lanes cover one 128-byte image row, so every store instruction writes whole lines
            const int lk = l - 64, pc = lk & 7;
            unsigned char* kt_img = ws + L.kt + ((size_t)cid * hv + h0 + hh) * kKTBytes;
            const float GL = ss.G[hh][len - 1];
#pragma unroll 2
            for (int i = 0; i < 16; ++i) {  // 16 passes of 8 rows: (d_k block, row) pairs
                const int rowi = i * 8 + (lk >> 3);
                const int kb2 = rowi >> 6, r = rowi & 63;
                const float cr = (r < len) ? fast_exp2(GL - ss.G[hh][r]) : 0.f;
                const uint32_t off = kb2 * 8192 + r * 128 + pc * 16;  // same swizzled position
                float kv8[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + kP_GR + kb2 * kP_GRB + 8192 + r * 128 + pc * 16), kv8);
#pragma unroll
                for (int e = 0; e < 8; ++e) kv8[e] *= cr;
                *reinterpret_cast<uint4*>(kt_img + off) = pack8(kv8);
            }
        }
        __syncthreads();
        const int tr = l >> 4, tc = l & 15;  // 4x2 output tile: rows 4 tr .., columns 2 tc ..
        float2 acc2[4];
        auto tile_product = [&](const float* Lm, const float* Rm) {  // acc2 = Lm (32x32) Rm (32x32)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc2[i] = make_float2(0.f, 0.f);
#pragma unroll 2
            for (int k4 = 0; k4 < 8; ++k4) {
                float4 a[4];
                float2 b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(Lm + (4 * tr + i) * kLdA + 4 * k4);
#pragma unroll
                for (int e = 0; e < 4; ++e) b[e] = *reinterpret_cast<const float2*>(Rm + (4 * k4 + e) * kLdA + 2 * tc);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc2[i] = __ffma2_rn(make_float2(a[i].x, a[i].x), b[0], acc2[i]);
                    acc2[i] = __ffma2_rn(make_float2(a[i].y, a[i].y), b[1], acc2[i]);
                    acc2[i] = __ffma2_rn(make_float2(a[i].z, a[i].z), b[2], acc2[i]);
                    acc2[i] = __ffma2_rn(make_float2(a[i].w, a[i].w), b[3], acc2[i]);
                }
            }
        };
        tile_product(A + 32 * kLdA, A);  // Y = A21 T1
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<float2*>(A + (4 * tr + i) * kLdA + 32 + 2 * tc) = acc2[i];
        __syncthreads();
        tile_product(A + 32 * kLdA + 32, A + 32);  // T2 Y
        __syncthreads();  // every thread is done reading Y and A21
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            *reinterpret_cast<float2*>(A + (32 + 4 * tr + i) * kLdA + 2 * tc) = make_float2(-acc2[i].x, -acc2[i].y);
            *reinterpret_cast<float2*>(A + (4 * tr + i) * kLdA + 32 + 2 * tc) = make_float2(0.f, 0.f);
        }
    }
    __syncthreads();

    // ---- 5. MMA operand images [T_0 diag(b_0 gam_0); T_1 diag(b_1 gam_1)] and [T_0 diag(b_0); ...]
    //         (two threads per row, 32 columns each)
    {
        const int hh = tid >> 7, r = (tid & 127) >> 1, hc = tid & 1;
        const float4* t4 = reinterpret_cast<const float4*>(af + hh * kAfHead + r * kLdA + 32 * hc);
        const float* bj = ss.b[hh] + 32 * hc;
        const float* gj = ss.gam[hh] + 32 * hc;
        uint4 wrow[4], urow[4];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float w8[8], u8[8];
#pragma unroll
            for (int half4 = 0; half4 < 2; ++half4) {
                const float4 tv = t4[2 * ch + half4];
                const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int jj = 8 * ch + 4 * half4 + e;
                    u8[4 * half4 + e] = tt[e] * bj[jj];
                    w8[4 * half4 + e] = u8[4 * half4 + e] * gj[jj];
                }
            }
            wrow[ch] = pack8(w8);
            urow[ch] = pack8(u8);
        }
        __syncthreads();
        const int row = hh * 64 + r;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            *reinterpret_cast<uint4*>(sm + kP_AF + sw128(row, 4 * hc + ch)) = wrow[ch];
            *reinterpret_cast<uint4*>(sm + kP_AF + 16384 + sw128(row, 4 * hc + ch)) = urow[ch];
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
                     sdesc_sw128(sb + kP_GR + 8192 + s * 2048, kP_GRB, 1024), idesc, s > 0);
            mma_bf16(tmem + 128, sdesc_sw128(sb + kP_AF + 16384 + s * 32, 16, 1024),
                     sdesc_sw128(sb + kP_GR + s * 2048, kP_GRB, 1024), idesc, s > 0);
        }
        mma_commit(&ss.bar_mma);
    }
    ok = mbar_wait(&ss.bar_mma, 1);
    if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
    tc_fence_after();

    // ---- 7. epilogue: accumulator row r' (lane quarter qw) is row r' % 64 of head r' / 64;
    //         each warp takes 64 of the 128 columns.  The W image is stored pre-scaled by the
    //         previous chunk's total decay (W~ = gam_L,prev W).  Images are assembled in
    //         shared memory that is free by then, in their final (swizzled) layout, and leave
    //         as 8 KB bulk copies: batch 1 W~ of both heads (K and Q slots), batch 2 U of head
    //         1 and M~ of both heads (the same four 8 KB pieces).  U of head 0 goes straight to
    //         the workspace (its accumulator is reused before batch 2).
    {
        const int hh = qw >> 1, r = (qw & 1) * 32 + lane, h = h0 + hh;
        const uint32_t tq = tmem + ((uint32_t)qw * 32u << 16);
        // piece i: the Q (i even) or K (i odd) slot of d_k block i / 2, 8 KB each
        auto piece = [&](int i) { return sm + kP_GR + (i >> 1) * kP_GRB + (i & 1) * 8192; };
        unsigned char* uimg = ws + L.u + ((size_t)cid * hv + h) * kUBytes;
        const float gp = ss.gprev[hh];
        float col[32];
        auto store32 = [&](unsigned char* img, uint32_t tcol, int chunk0, float scale) {
            tmem_ld16(tq + tcol, col);
            tmem_ld16(tq + tcol + 16, col + 16);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) col[e] *= scale;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                *reinterpret_cast<uint4*>(img + sw128(r, chunk0 + ch)) = pack8(col + 8 * ch);
        };
        // W columns 64 hf .. 64 hf + 63 = d_k block hf (8 KB image half) -> piece 2 hh + hf
        store32(piece(2 * hh + hf), 64 * hf, 0, gp);
        store32(piece(2 * hh + hf), 64 * hf + 32, 4, gp);
        if (hh == 0) {  // U of head 0: columns 128 + 64 hf ..
            store32(uimg + hf * 8192, 128 + 64 * hf, 0, 1.f);
            store32(uimg + hf * 8192, 128 + 64 * hf + 32, 4, 1.f);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // U of head 1: D[:, 128:256] = A_U V_1 (rows 64..127 are head 1's)
            tc_fence_after();  // and M = [T0 D0; T1 D1] (K K_prev^T): D[:, 0:64]
            const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
            const uint32_t idesc_m = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                mma_bf16(tmem + 128, sdesc_sw128(sb + kP_AF + 16384 + s * 32, 16, 1024),
                         sdesc_sw128(sb + kP_GR + 16384 + s * 2048, kP_GRB, 1024), idesc, s > 0);
                mma_bf16(tmem, sdesc_sw128(sb + kP_AF + s * 32, 16, 1024),
                         sdesc_sw128(sb + kP_GX + s * 2048, 8192, 1024), idesc_m, s > 0);
            }
            mma_commit(&ss.bar_mma);
        }
        if (tid == 32) {  // batch 1 out: W~ of both heads
            unsigned char* w0 = ws + L.w + ((size_t)cid * hv + h0) * kWBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i) bulk_s2g(w0 + (i >> 1) * kWBytes + (i & 1) * 8192, piece(i), 8192);
            bulk_commit();
            bulk_wait_read_all();  // the pieces are read before batch 2 refills them
        }
        ok = mbar_wait(&ss.bar_mma, 0);
        if (__syncthreads_or(!ok)) { err = 1; goto cleanup; }
        tc_fence_after();
        if (hh == 1) {  // U of head 1 -> pieces 0 (d_v block 0) and 1 (d_v block 1)
            store32(piece(hf), 128 + 64 * hf, 0, 1.f);
            store32(piece(hf), 128 + 64 * hf + 32, 4, 1.f);
        }
        {   // M~ = M diag(c_prev): columns 32 hf .. 32 hf + 31 of head hh -> piece 2 + hh
            tmem_ld16(tq + 32 * hf, col);
            tmem_ld16(tq + 32 * hf + 16, col + 16);
            tmem_ld_wait();
            const float* cp = ss.cprev[hh] + 32 * hf;
#pragma unroll
            for (int e = 0; e < 32; ++e) col[e] *= cp[e];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                *reinterpret_cast<uint4*>(piece(2 + hh) + sw128(r, 4 * hf + ch)) = pack8(col + 8 * ch);
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 32) {  // batch 2 out: U of head 1, M~ of both heads
            unsigned char* u1 = ws + L.u + ((size_t)cid * hv + h0 + 1) * kUBytes;
            unsigned char* m0 = ws + L.m + ((size_t)cid * hv + h0) * kMBytes;
            bulk_s2g(u1, piece(0), 8192);
            bulk_s2g(u1 + 8192, piece(1), 8192);
            bulk_s2g(m0, piece(2), 8192);
            bulk_s2g(m0 + kMBytes, piece(3), 8192);
            bulk_commit();
            bulk_wait_read_all();  // shared memory is read before the CTA exits
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
// Look-ahead form of the chunk recurrence.  With S_c the state entering chunk c and
// X_c = W_c S_c^T, the state update of chunk c-1 gives
//   X_c = gam_L,c-1 W_c S_{c-1}^T + (W_c K_{c-1}^T diag(c_{c-1})) Delta_{c-1}
//       = W~_c S_{c-1}^T            + M~_c Delta_{c-1},
// with W~ and M~ from the prep kernel.  The K = 128 product W~_c S_{c-1}^T (together with
// Y_{c-1} = Q_{c-1} S_{c-1}^T, as one M = 128 MMA) is issued one chunk ahead; only the
// K = 64 product M~_c Delta_{c-1} separates Delta_{c-1} from Delta_c, and it shares its
// B operand with P_{c-1} Delta_{c-1} (the outputs of chunk c-1): [M~_c; P_{c-1}] Delta_{c-1}
// is one M = 128 MMA.  The state update S_c = gam_L S_{c-1} + (K~_{c-1}^T Delta_{c-1})^T,
// with K~ = diag(c) K from the prep kernel, reads the same B operand.  At these sizes every
// tcgen05.mma costs the issuing thread about the same time whatever its N, so the schedule
// is built around that one thread (16 MMAs per chunk).  In step c it waits for
// Delta_{c-1}, issues (a) and (b) back to back, and (d) once S_c is written:
//   (a) SA  = K~_{c-1}^T B2           (B2 = Delta_{c-1}, bf16)             -> state warps
//   (b) CH  = [M~_c; P_{c-1}] B2      (rows 0..63 -> Delta warps; rows 64..127 -> outputs)
//   (d) ZY  = [W~_{c+1}; Q_c] B1      (B1 = S_c, written by the state warps after (a))
// Operand slot k (k = 0 .. nch) holds W~_k, M~_k and Q, P, K~ and the gate factors of chunk
// k-1; step c reads slots c and c+1.  A slot is released in step k once (b) has completed;
// the copy warp refills it two steps ahead of use and asks L2 for the slot after that.
// Completion of (a) in step c+1 implies completion of everything issued before it, so the
// outputs of chunk c-1 need no barrier of their own.
//
// Warps (TMEM lane quarter = warp % 4, 16-column half of the 32 d_v = (warp / 4) % 2):
//   0, 1, 4, 5     Delta warps: token rows 0..63 of X_c, Delta_c and B2
//   2, 3, 6, 7     state rows (d_k) 64..127 and the outputs (token rows of Y and PD)
//   8, 9, 12, 13   state rows (d_k) 0..63
//   10             MMA issuer;  11  bulk copies
constexpr int kStateThreads = 448;
constexpr int kIssuerWarp = 10, kCopyWarp = 11;
constexpr int kStages = 3;                          // operand slots
constexpr uint32_t kS_A1 = 0;                       // [W~_k; Q_{k-1}] K-major, 2 d_k blocks of 128 rows (32 KB)
constexpr uint32_t kS_M = 32768;                    // M~_k (8 KB); [M~; P] is the A operand of (b)
constexpr uint32_t kS_P = 40960;                    // P_{k-1} (8 KB)
constexpr uint32_t kS_KT = 49152;                   // K~_{k-1}, MN-major A operand (16 KB)
constexpr uint32_t kS_BUF = 65536;                  // one slot (64 KB)
constexpr int kSlices = 4;                          // CTAs per (sequence, V head)
constexpr int kSliceW = kD / kSlices;               // d_v columns per CTA (the MMAs' N)
constexpr uint32_t kS_B1 = kStages * kS_BUF;        // S slice bf16, MN-major, 64-byte swizzle (8 KB)
constexpr uint32_t kS_B2 = kS_B1 + 8192;            // Delta, two buffers (2 x 4 KB)
constexpr uint32_t kS_CV = kS_B2 + 8192;            // gate factors of each slot (3 x 528 B)
constexpr uint32_t kS_SMALL = kS_CV + kStages * kCvecLoad;
constexpr uint32_t kStateSmem = kS_SMALL + 256;     // needs a 1024-aligned dynamic base (checked)
constexpr uint32_t kEmptyArrivals = 257;            // state/output warps and the MMA commit (step k)
// Tensor Memory columns
constexpr uint32_t kT_ZY = 0;     // [Z~_c; Y_{c-1}] at 32 (c % 3)
constexpr uint32_t kT_CH = 96;    // [M~_c Delta_{c-1}; P_{c-1} Delta_{c-1}] at 96 + 32 (c % 3)
constexpr uint32_t kT_SA = 192;   // K~^T Delta
constexpr uint32_t kTmemCols = 256;

struct StateSmall {
    uint64_t full[kStages];   // slot loaded
    uint64_t empty[kStages];  // slot consumed (kEmptyArrivals arrivals)
    uint64_t b2[2];           // Delta_c in B2[c & 1], on b2[c & 1]
    uint64_t b1, mx, msa, fin, drain;
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

// 16 consecutive TMEM columns of this warp's lane quarter.
__device__ __forceinline__ void tmem_ld16w(uint32_t tmem_base, int warp, uint32_t col, float* v) {
    tmem_ld16(tmem_base + ((uint32_t)(warp & 3) * 32u << 16) + col, v);
    tmem_ld_wait();
}

// Operand slot k of a sequence whose chunks are cs .. cs + nch - 1.
__device__ __forceinline__ void issue_slot_loads(unsigned char* buf, unsigned char* cv, uint64_t* bar,
                                                 const unsigned char* ws, const WsLayout& L, int cs, int k,
                                                 int nch, int h, int jq, int hk, int hv) {
    const bool w_k = k < nch, m_k = k >= 1 && k < nch, prev = k >= 1;
    uint32_t bytes = 0;
    if (w_k) bytes += kWBytes;
    if (m_k) bytes += kMBytes;
    if (prev) bytes += kQBytes + kPBytes + kKTBytes + kCvecLoad;
    mbar_arrive_expect_tx(bar, bytes);
    if (w_k) {
        const unsigned char* w = ws + L.w + ((size_t)(cs + k) * hv + h) * kWBytes;
        bulk_g2s(buf + kS_A1, w, 8192, bar);                  // W~ rows, d_k 0..63
        bulk_g2s(buf + kS_A1 + 16384, w + 8192, 8192, bar);   // W~ rows, d_k 64..127
    }
    if (m_k) bulk_g2s(buf + kS_M, ws + L.m + ((size_t)(cs + k) * hv + h) * kMBytes, kMBytes, bar);
    if (prev) {
        const int cp = cs + k - 1;
        const unsigned char* qn = ws + L.qn + ((size_t)cp * hk + jq) * kQBytes;
        bulk_g2s(buf + kS_A1 + 8192, qn, 8192, bar);          // Q rows, d_k 0..63
        bulk_g2s(buf + kS_A1 + 24576, qn + 8192, 8192, bar);  // Q rows, d_k 64..127
        bulk_g2s(buf + kS_P, ws + L.p + ((size_t)cp * hv + h) * kPBytes, kPBytes, bar);
        bulk_g2s(buf + kS_KT, ws + L.kt + ((size_t)cp * hv + h) * kKTBytes, kKTBytes, bar);
        bulk_g2s(cv, ws + L.cvec + ((size_t)cp * hv + h) * kCvecBytes, kCvecLoad, bar);
    }
}

// The same bytes as issue_slot_loads, into L2 only.
__device__ __forceinline__ void prefetch_slot(const unsigned char* ws, const WsLayout& L, int cs, int k, int nch,
                                              int h, int jq, int hk, int hv) {
    if (k < nch) bulk_prefetch_l2(ws + L.w + ((size_t)(cs + k) * hv + h) * kWBytes, kWBytes);
    if (k >= 1 && k < nch) bulk_prefetch_l2(ws + L.m + ((size_t)(cs + k) * hv + h) * kMBytes, kMBytes);
    if (k >= 1) {
        const int cp = cs + k - 1;
        bulk_prefetch_l2(ws + L.qn + ((size_t)cp * hk + jq) * kQBytes, kQBytes);
        bulk_prefetch_l2(ws + L.p + ((size_t)cp * hv + h) * kPBytes, kPBytes);
        bulk_prefetch_l2(ws + L.kt + ((size_t)cp * hv + h) * kKTBytes, kKTBytes);
        bulk_prefetch_l2(ws + L.cvec + ((size_t)cp * hv + h) * kCvecBytes, kCvecLoad);
    }
}

__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_kernel(const float* s0, const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out,
                   float* sT, StateSlots map, float* cstates, unsigned char* ws, int num_seqs, int total_tokens,
                   int hk, int hv) {
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sb = smem_u32(sm);
    StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + kS_SMALL);
    volatile int* abort_flag = &ss.abort_flag;

    const WsLayout L = ws_layout(num_seqs, total_tokens, hk, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int slice = blockIdx.x % kSlices;
    const int h = (blockIdx.x / kSlices) % hv;
    const int n = (blockIdx.x / kSlices) / hv;
    const int jq = h / (hv / hk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (sb & 1023u) {  // the swizzled operand layouts need a 1024-byte-aligned base
        grid_dependency_wait();
        if (tid == 0) atomicOr(header, 2);
        return;
    }

    // Set-up that needs nothing from the prep kernel runs before the dependency wait (a
    // CTA of this kernel never shares an SM with a prep CTA: their shared memory does not
    // fit together, so the Tensor Memory columns are free).
    if (warp == 0) {
        tmem_alloc(&ss.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ss.full[s], 1);
            mbar_init(&ss.empty[s], kEmptyArrivals);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&ss.b2[s], 128);
        mbar_init(&ss.b1, 256);
        mbar_init(&ss.mx, 1);
        mbar_init(&ss.msa, 1);
        mbar_init(&ss.fin, 1);
        mbar_init(&ss.drain, 1);
        ss.abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;
    grid_dependency_wait();  // the prep kernel's workspace is complete and visible
    const int32_t* seq_chunk0 = reinterpret_cast<const int32_t*>(ws + L.seq_chunk0);
    const int cs = seq_chunk0[n], nch = seq_chunk0[n + 1] - cs;
    const int t_begin = cu[n], t_end = cu[n + 1];

    if (warp == kIssuerWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && nch > 0) {
            const uint32_t id_xy = idesc_bf16(128, kSliceW, 0, 1);  // A K-major, B MN-major
            const uint32_t id_s = idesc_bf16(128, kSliceW, 1, 1);   // A MN-major, B MN-major
            // B operands: one 32-wide atom along N (the N-block stride is never used), 8-K-row
            // groups of 512 bytes
            const uint64_t d_b1 = sdesc_sw64(sb + kS_B1, 512, 512);
            auto issue_zy = [&](int k) {  // [W~_k; Q_{k-1}] S^T -> ZY buffer k % 3
                const uint64_t d_a1 = sdesc_sw128(sb + (k % kStages) * kS_BUF + kS_A1, 16, 1024);
#pragma unroll
                for (int s = 0; s < 8; ++s)  // descriptor start addresses advance in 16-byte units
                    mma_bf16(tmem + kT_ZY + kSliceW * (k % 3), d_a1 + (((s >> 2) * 16384 + (s & 3) * 32) >> 4),
                             d_b1 + ((s * 1024) >> 4), id_xy, s > 0);
            };
            int c = -1;
            bool ok = wait_or_abort(&ss.full[0], 0, abort_flag, header) &&
                      wait_or_abort(&ss.b1, 0, abort_flag, header);
            if (ok) {  // X_0 = W_0 S_0^T
                tc_fence_after();
                issue_zy(0);
                mma_commit(&ss.mx);
                for (c = 0; c <= nch; ++c) {
                    const int sc = c % kStages, sn = (c + 1) % kStages;
                    const uint32_t bufc = sb + sc * kS_BUF;
                    if (c >= 1) {
                        const int pb = (c - 1) & 1;
                        if (!wait_or_abort(&ss.b2[pb], ((c - 1) >> 1) & 1, abort_flag, header)) break;
                        tc_fence_after();
                        const uint64_t d_b2 = sdesc_sw64(sb + kS_B2 + 4096 * pb, 512, 512);
                        const uint64_t d_kt = sdesc_sw128(bufc + kS_KT, 8192, 1024);
#pragma unroll
                        for (int s = 0; s < 4; ++s)  // (a)
                            mma_bf16(tmem + kT_SA, d_kt + ((s * 2048) >> 4), d_b2 + ((s * 1024) >> 4), id_s, s > 0);
                        mma_commit(&ss.msa);
                        const uint64_t d_mp = sdesc_sw128(bufc + kS_M, 16, 1024);
#pragma unroll
                        for (int s = 0; s < 4; ++s)  // (b)
                            mma_bf16(tmem + kT_CH + kSliceW * (c % 3), d_mp + ((s * 32) >> 4), d_b2 + ((s * 1024) >> 4),
                                     id_xy, s > 0);
                        mma_commit(&ss.mx);
                    }
                    mma_commit(&ss.empty[sc]);  // every MMA reading slot c has been issued
                    if (c < nch) {  // (d)
                        if (!wait_or_abort(&ss.full[sn], ((c + 1) / kStages) & 1, abort_flag, header)) break;
                        if (!wait_or_abort(&ss.b1, c & 1, abort_flag, header)) break;
                        tc_fence_after();
                        issue_zy(c + 1);
                    }
                }
                if (c == nch + 1) mma_commit(&ss.fin);  // P Delta of the last chunk
            }
            if (*abort_flag) {  // drain: every MMA issued so far completes before TMEM is freed
                mma_commit(&ss.drain);
                mbar_wait(&ss.drain, 0);
            }
        }
    } else if (warp == kCopyWarp) {
        // ------------------------------------------------ bulk copies, two slots ahead
        if (lane == 0 && nch > 0) {
            int issued = 0;
            for (; issued <= nch; ++issued) {
                const int st = issued % kStages;
                if (issued >= kStages &&
                    !wait_or_abort(&ss.empty[st], ((issued / kStages) - 1) & 1, abort_flag, header))
                    break;
                issue_slot_loads(sm + st * kS_BUF, sm + kS_CV + st * kCvecLoad, &ss.full[st], ws, L, cs, issued,
                                 nch, h, jq, hk, hv);
                if (issued + kStages <= nch) prefetch_slot(ws, L, cs, issued + kStages, nch, h, jq, hk, hv);
            }
            if (*abort_flag) {  // drain: copies in flight land before the CTA exits
                for (int j = max(0, issued - kStages); j < issued; ++j)
                    mbar_wait(&ss.full[j % kStages], (j / kStages) & 1);
            }
        }
    } else {
        const int q4 = warp & 3, ch2 = (warp >> 2) & 1;
        const int dv0 = slice * kSliceW + 16 * ch2;  // first d_v column of this thread
        const int r = (q4 & 1) * 32 + lane;         // token row (Delta warps; output warps)
        const bool delta_warp = warp < 8 && q4 < 2;
        const bool out_warp = warp < 8 && q4 >= 2;
        if (delta_warp) {
            // ------------------------------------------------ Delta warps
            // U rows of a chunk straight from the workspace (U image: [d_v half][64 rows][128 B])
            auto load_u = [&](int cidx, uint4* u) {
                const unsigned char* ub =
                    ws + L.u + ((size_t)(cs + cidx) * hv + h) * kUBytes + (dv0 >> 6) * (kUBytes / 2);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    u[cc] = *reinterpret_cast<const uint4*>(ub + sw128(r, (dv0 & 63) / 8 + cc));
            };
            uint4 u_next[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
            if (nch > 0) load_u(0, u_next);
            for (int c = 0; c < nch; ++c) {
                // Delta_c = U_c - X_c,  X_c = Z~_c + M~_c Delta_{c-1}  (token row r)
                uint4 u4[2] = {u_next[0], u_next[1]};
                if (c + 1 < nch) load_u(c + 1, u_next);
                if (!wait_or_abort(&ss.mx, c & 1, abort_flag, header)) break;
                tc_fence_after();
                float x[16];
                tmem_ld16w(tmem, warp, kT_ZY + kSliceW * (c % 3) + 16 * ch2, x);
                if (c >= 1) {
                    float xc[16];
                    tmem_ld16w(tmem, warp, kT_CH + kSliceW * (c % 3) + 16 * ch2, xc);
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] += xc[e];
                }
                float d[16];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float u8[8];
                    unpack8(u4[cc], u8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) d[8 * cc + e] = u8[e] - x[8 * cc + e];
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    *reinterpret_cast<uint4*>(sm + kS_B2 + 4096 * (c & 1) + sw64(r, 2 * ch2 + cc)) = pack8(d + 8 * cc);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&ss.b2[c & 1]);
            }
        } else {
            // ------------------------------------------------ state warps (and outputs)
            const int t = q4 * 32 + lane;  // d_k row of S^T this thread owns
            // fp32 state: S[dv0 + m][t], m = 0..15
            float S[16];
            bool has_state;
            const int sidx = state_index(map, n, has_state);
            if (!has_state) { s0 = nullptr; sT = nullptr; }  // no slot: start from zeros, keep no state
            const size_t sbase = ((size_t)sidx * hv + h) * kD * kD + (size_t)dv0 * kD + t;
#pragma unroll
            for (int m = 0; m < 16; ++m) S[m] = s0 ? s0[sbase + (size_t)m * kD] : 0.f;
            auto write_b1 = [&]() {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    *reinterpret_cast<uint4*>(sm + kS_B1 + sw64(t, 2 * ch2 + cc)) = pack8(S + 8 * cc);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&ss.b1);
            };
            write_b1();  // S_0: phase 0 of b1
            if (nch > 0) mbar_arrive(&ss.empty[0]);  // slot 0 has no gate factors to read

            // O_c = gam_r Y_c + P_c Delta_c, with Y_c in the ZY buffer of c+1 and P_c Delta_c in
            // the CH buffer of c+1 (rows 64..127).  Written in step c+2, after the state update
            // (whose wait on (a) of step c+2 covers (b) of step c+1), so that the global stores
            // are not still in flight at the next proxy fence.
            float prev_gam = 0.f;  // gam_r of the chunk whose outputs are written next
            auto write_outputs = [&](int cpo, float gam_r) {
                const int t0 = t_begin + cpo * kChunk;
                const int len = min(kChunk, t_end - t0);
                float y[16], pd[16];
                tmem_ld16w(tmem, warp, kT_ZY + kSliceW * ((cpo + 1) % 3) + 16 * ch2, y);
                tmem_ld16w(tmem, warp, kT_CH + kSliceW * ((cpo + 1) % 3) + 16 * ch2, pd);
                if (r < len) {
                    uint4* op = reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * hv + h) * kD + dv0);
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float o8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o8[e] = fmaf(gam_r, y[8 * cc + e], pd[8 * cc + e]);
                        op[cc] = pack8(o8);
                    }
                }
                tc_fence_before();
            };
            int c = 1;
            for (; c <= nch; ++c) {
                // S_c = gam_L S_{c-1} + SA  (gate factors of chunk c-1 are in slot c)
                const int sc = c % kStages;
                if (!wait_or_abort(&ss.full[sc], (c / kStages) & 1, abort_flag, header)) break;
                const float* cvp = reinterpret_cast<const float*>(sm + kS_CV + sc * kCvecLoad);
                const float gl = cvp[128];
                const float gr = cvp[64 + r];
                mbar_arrive(&ss.empty[sc]);
                if (!wait_or_abort(&ss.msa, (c - 1) & 1, abort_flag, header)) break;
                tc_fence_after();
                float acc[16];
                tmem_ld16w(tmem, warp, kT_SA + 16 * ch2, acc);
#pragma unroll
                for (int m = 0; m < 16; ++m) S[m] = fmaf(gl, S[m], acc[m]);
                if (c < nch) write_b1();
                if (cstates) {  // the state after chunk c-1, after the proxy fence (stores may stay in flight)
                    float* cr = cstates + ((size_t)(cs + c - 1) * hv + h) * kD * kD + (size_t)dv0 * kD + t;
#pragma unroll
                    for (int m = 0; m < 16; ++m) cr[(size_t)m * kD] = S[m];
                }
                if (out_warp) {
                    if (c >= 2) write_outputs(c - 2, prev_gam);
                    prev_gam = gr;
                }
            }
            if (out_warp && nch > 0 && c == nch + 1 && wait_or_abort(&ss.fin, 0, abort_flag, header)) {
                tc_fence_after();
                write_outputs(nch - 1, prev_gam);
            }
            if (!*abort_flag && sT) {
#pragma unroll
                for (int m = 0; m < 16; ++m) sT[sbase + (size_t)m * kD] = S[m];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Launch with programmatic stream serialization: the kernel may begin (and run its set-up)
// while the previous kernel on the stream finishes; it waits with grid_dependency_wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
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
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_prep_kernel, kPrepThreads, kPrepSmem)) !=
        cudaSuccess)
        return e;
    chunk_table_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, ws);
    if (L.max_chunks > 0 && total_tokens > 0) {
        e = launch_dependent(chunk_prep_kernel, dim3((unsigned)(L.max_chunks * hk)), dim3(kPrepThreads),
                             kPrepSmem, stream, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                             (const __nv_bfloat16*)v, g, beta, ws, num_seqs, total_tokens, hk, hv,
                             sms * per_sm);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc_state(const float* s0, const int32_t* cu, void* out, float* sT,
                                    StateSlots map, float* cstates, int num_seqs, int total_tokens, int hk,
                                    int hv, void* workspace, cudaStream_t stream) {
    if (num_seqs == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kStateSmem);
    if (e != cudaSuccess) return e;
    e = launch_dependent(chunk_state_kernel, dim3((unsigned)num_seqs * hv * kSlices), dim3(kStateThreads),
                         kStateSmem, stream, s0, cu, (__nv_bfloat16*)out, sT, map, cstates,
                         static_cast<unsigned char*>(workspace), num_seqs, total_tokens, hk, hv);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
