// prefill_tc.cu -- chunked prefill of the Gated DeltaNet layer on sm_100a tensor cores.
//
// The chunked form of the gated delta rule (Gated DeltaNet per the Qwen3-Next-80B-A3B model
// card, "Model Overview": 16 QK heads, 32 V heads, head dim 128), chunks of 64 tokens.  For a
// chunk of one V head entering with state S (d_v x d_k), raw keys K, queries Q and values V
// (rows = tokens), norms r_k = 1/|k|, r_q = 1/(|q| sqrt(128)), in-chunk inclusive gate sums
// G_r, gam_r = exp(G_r), c_r = exp(G_L - G_r) with L the chunk's last row:
//   A = strictly_lower(b_r exp(G_r - G_j) r_k,r r_k,j K K^T),  T = (I + A)^-1
//   P = lower(exp(G_r - G_j) r_q,r r_k,j Q K^T)
//   W = T diag(b gam r_k) K,         Delta = T diag(b) V - W S^T
//   O = diag(gam r_q) Q S^T + P Delta
//   S <- gam_L S + (diag(c r_k) Delta)^T K
// The keys, queries and values enter every product as the exact bf16 inputs; normalisation,
// gates and beta live in fp32 coefficient matrices.  The output is taken in resolved form,
//   O = Qt S^T + At V,  Qt = diag(gam r_q) Q - P T diag(b gam r_k) K,  At = P T diag(b),
// so that the sums over the chunk whose terms cancel (repeated or colinear keys with b near 1
// make T's rows alternate in sign) are formed in fp32 before anything is rounded to bf16.
// Where a product of that kind must still pass through bf16 MMA operands (T diag(b gam r_k)
// for W, [T diag(b); At] for U and At V, and diag(c r_k) Delta for the state update), the
// operand is split into a bf16 high part and a bf16 remainder and both are multiplied, which
// keeps about 16 significant bits.
//
// The state update runs as a tf32 product: it reads Delta^T (fp32) straight out of the
// accumulator of the previous product and Kt = diag(c r_k) K in fp32, so Delta never passes
// through the CUDA cores or bf16 (tf32 keeps 10 bits of each operand).
//
// Three kernels, all on the caller's stream:
//  K0 chunk_table_kernel  clears the workspace's device error word; cu_seqlens -> per-sequence
//                         first chunk id and a (seq, start, length) entry per chunk.
//  K1 chunk_prep_kernel   one CTA (256 threads) per (chunk, pair of V heads sharing a QK head),
//                         all chunks in parallel: q and k tiles by TMA; the Gram [Q;K][Q;K]^T
//                         (tcgen05), whose diagonal gives the norms; decay masks A and P;
//                         T = (I + A)^-1 in 32 x 32 blocks (the diagonal blocks by row
//                         substitution in fp32, T21 = -T22 A21 T11) and P T, the products on
//                         warp tf32 MMAs with both factors split high / low; then per V head the
//                         coefficient rows are written to Tensor Memory and W and
//                         diag(gam r_q) Q - (P T diag(b gam r_k)) K come out of one tcgen05
//                         product with K; -W, Qt, the split [T diag(b); At] images, Kt in fp32
//                         and gam_L go to the workspace.
//  K2 chunk_state_kernel  one CTA per (sequence, V head), sequential over the sequence's chunks:
//                         the state is the A operand of its MMAs, held in Tensor Memory (M =
//                         d_v = 128 rows), so every product reads only its B operand from shared
//                         memory; V and K tiles come by TMA, the workspace images by bulk copy.
// Every mbarrier wait is bounded (1 s); a wait that gives up records an error in the workspace
// header, the kernel drains its own copies and MMAs (bounded), frees Tensor Memory and returns.
#include <cuda.h>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)
constexpr float kLog2e = 1.4426950408889634f;

// Workspace record per (chunk, V head), images in the 128-byte-swizzled layouts the state
// kernel's MMAs read:
//   WQ     [-W; Qt] bf16, K-major: per d_k block b (64 columns) at b * 16384, 64 rows of -W then
//          64 rows of Qt
//   TA_hi  [T diag(b); At] bf16 high part, K-major: 128 rows (64 of T diag(b), 64 of At) x 64
//          tokens
//   TA_lo  the remainders of the same
//   KT     Kt = diag(c r_k) K in fp32 (the tf32 B operand of the state update), K-major: per
//          32-token block b at b * 16384, 128 d_k rows of 128 bytes (32 tokens)
//   F      gam_L
constexpr uint32_t kWQBytes = 32768;
constexpr uint32_t kTABytes = 16384;
constexpr uint32_t kKTOff = kWQBytes + 2 * kTABytes;  // 65536
constexpr uint32_t kKTBytes = 32768;
constexpr uint32_t kFacOff = kKTOff + kKTBytes;       // 98304
constexpr uint32_t kFacLoad = 16;                     // bytes of F the state kernel reads
constexpr uint32_t kRecBytes = kFacOff + 1024;        // 99,328
// The one-launch pass keeps the records of at most kRing chunks (a ring: 14 x 32 heads x 99 KB =
// 44.5 MB at 32 V heads, which stays in L2, so the records rarely reach DRAM) instead of one
// slot per chunk.  Its prep workers run about 14.5 chunks ahead of the state passes at B = 1
// (232 workers, 16 items per chunk); a larger ring lets L2 evict records to DRAM before they
// are overwritten, a smaller one stalls the workers.
constexpr int kRing = 14;

struct WsLayout {
    size_t seq_chunk0, table, flags, rec, total;
    long long max_chunks;
};

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int num_seqs, int total_tokens, int hv) {
    WsLayout L;
    L.max_chunks = (long long)total_tokens / kChunk + num_seqs;
    size_t off = 256;  // header: [0] device error word, [1] number of chunks
    L.seq_chunk0 = off;
    off = round_up(off + (size_t)(num_seqs + 1) * 4, 1024);
    L.table = off;
    off = round_up(off + (size_t)L.max_chunks * 16, 1024);
    L.flags = off;  // the one-launch pass: per (chunk, pair of V heads) "records complete" flags,
                    // then per (ring slot, V head) the last chunk consumed + 1
    off = round_up(off + ((size_t)L.max_chunks * (hv / 2 > 0 ? hv / 2 : 1) + (size_t)kRing * hv) * 4, 1024);
    L.rec = off;
    off += (size_t)L.max_chunks * hv * kRecBytes;
    L.total = round_up(off, 1024);
    return L;
}

// ===================================================================== K0
__global__ void __launch_bounds__(1024)
chunk_table_kernel(const int32_t* __restrict__ cu, int num_seqs, int total_tokens, int hv, unsigned char* ws) {
    allow_dependent_launch();
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    if (threadIdx.x == 0) header[0] = 0;  // the device error word of this call
    const WsLayout L = ws_layout(num_seqs, total_tokens, hv);
    {
        int32_t* flags = reinterpret_cast<int32_t*>(ws + L.flags);
        const long long nflags = L.max_chunks * (hv / 2) + (long long)kRing * hv;
        for (long long i = threadIdx.x; i < nflags; i += blockDim.x) flags[i] = 0;
    }
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
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): two bf16 words carrying ~16 bits.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ float warp_inclusive_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// 2^x on the special-function unit (PTX ex2.approx); callers pass arguments <= 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp32 64x64 matrices in shared memory: rows padded to 68 floats, so that 8 threads writing
// float4s to 8 consecutive rows hit different banks and row reads stay contiguous.
constexpr int kLdA = 68;
constexpr int kMat = kChunk * kLdA;  // floats per matrix

// ===================================================================== K1
// Shared memory (bytes from a 1024-aligned base):
//   kP_QK  per d_k block b at b * 16384: 64 rows of Q then 64 rows of K (TMA, 128-byte swizzle).
//          The Gram reads it as A = B = [Q; K] (K-major); the W product reads the K rows as an
//          MN-major B operand (tokens along K, d_k along N).
//   kP_AT  per head: A, then T (fp32, row-major)
//   kP_PP  per head: P, then P T (fp32, row-major)
// Tensor Memory (256 columns): 0..127 the Gram, later the [W; -P T diag(b gam r_k) K] product of
// one head at a time; 128 + 64 h .. : head h's A operand rows (32 columns high part, 32 low).
constexpr uint32_t kP_QK = 0;
constexpr uint32_t kP_AT = 32768;
constexpr uint32_t kP_PP = kP_AT + 2 * kMat * 4;
constexpr uint32_t kP_SMALL = kP_PP + 2 * kMat * 4;
constexpr uint32_t kPrepSmem = kP_SMALL + 4096 + 1024;  // small struct + alignment slack
constexpr int kPrepThreads = 256;

struct PrepSmall {
    float G[2][kChunk];    // in-chunk gate sums, pre-scaled by log2(e) (constant past the length)
    float b[2][kChunk];    // beta, 0 past the chunk's length
    float gam[2][kChunk];  // exp(G)
    float c[2][kChunk];    // exp(G_L - G_r), 0 past the chunk's length
    float rq[kChunk];      // 1 / (sqrt(|q|^2 + eps) sqrt(128))
    float rk[kChunk];      // 1 / sqrt(|k|^2 + eps)
    float fw[2][kChunk];   // b gam r_k per column (the W / P T coefficient scaling)
    float fk[2][kChunk];   // c r_k per token (Kt's row scaling)
    uint64_t bar_tma, bar_mma, bar_drain;
    uint32_t tmem_base;
};
static_assert(sizeof(PrepSmall) <= 4096, "PrepSmall fits its region");
constexpr uint32_t kPrepRegion = kP_SMALL + 4096;  // one prep item's shared memory (1024-aligned)

// Everything one prep item needs besides its place in the CTA.
struct PrepArgs {
    const CUtensorMap* tm_q;
    const CUtensorMap* tm_k;
    const float* g;
    const float* beta;
    unsigned char* ws;
    int num_seqs, total_tokens, hk, hv;
    GateAct act;
    int32_t* ready;  // per (chunk, pair of V heads): set once the item's records are complete, or nullptr
    const int32_t* consumed;  // per (ring slot, V head): last chunk whose records a state pass has taken + 1
    int ring;                 // records go to ring slot chunk % ring (0: to slot chunk, no ring)
};

// The barriers of a prep item's 256 threads, initialised once (thread 32 of the item).
__device__ __forceinline__ void prep_init_barriers(PrepSmall& ss) {
    mbar_init(&ss.bar_tma, 1);
    mbar_init(&ss.bar_mma, 1);
    mbar_init(&ss.bar_drain, 1);
    fence_mbar_init();
}

// Bounded wait (one thread) until both V heads' state passes have taken chunk `need` - 1 from
// a ring slot: marks[0] and marks[1] reach `need`.  Gives up (false, recording the error) after
// the wait limit, or at once when another CTA has recorded an error in the header.
__device__ bool wait_consumed(const int32_t* marks, int need, int32_t* header) {
    if (wait_marks_reach(marks, need, header, kWaitLimitNs)) return true;
    atomicOr(header, 1);
    return false;
}

// One prep item, the chunk cid for the V heads 2 pair and 2 pair + 1, by 256 threads (tid
// 0..255, their warps a multiple-of-4-aligned group of the CTA) that synchronise on named
// barrier bid.  sm is the item's 1024-aligned shared memory (kPrepRegion bytes), tmem its 256
// Tensor Memory columns; j counts the items these threads have run before, so that the
// mbarrier phases continue across items.  Returns false (on all 256 threads) if a bounded wait
// gave up; the caller then records the error and drains.
__device__ bool prep_item(const PrepArgs& a, int cid, int pair, unsigned char* sm, uint32_t tmem, int tid,
                          uint32_t bid, uint32_t j) {
    const uint32_t sb = smem_u32(sm);
    PrepSmall& ss = *reinterpret_cast<PrepSmall*>(sm + kP_SMALL);
    float* AT = reinterpret_cast<float*>(sm + kP_AT);  // [head][64][kLdA]
    float* PP = reinterpret_cast<float*>(sm + kP_PP);
    const int hv = a.hv;
    const GateAct act = a.act;
    const float* g = a.g;
    const float* beta = a.beta;
    unsigned char* ws = a.ws;
    const WsLayout L = ws_layout(a.num_seqs, a.total_tokens, hv);
    const int h0 = 2 * pair;             // the two V heads of this item
    const size_t rslot = a.ring ? (size_t)(cid % a.ring) : (size_t)cid;  // the item's record slot
    const int jq = h0 / (hv / a.hk);     // their QK head
    const int lane = tid & 31, warp = tid >> 5;
    const int qw = warp & 3, hf = warp >> 2;  // TMEM lane quarter, column half
    const int4 ent = reinterpret_cast<const int4*>(ws + L.table)[cid];
    const int t0 = ent.y, len = ent.z;
    const uint32_t ph = j & 1;  // parity of this item's first completion of each barrier
    bool ok;

    // ---- 0. q and k tiles by TMA; warps 0-1 the gates of one head each
    if (tid == 32) {
        fence_async_smem();  // a previous item's reads of the tiles come first
        mbar_arrive_expect_tx(&ss.bar_tma, 32768);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tma_load_2d(sm + kP_QK + b * 16384, a.tm_q, jq * kD + b * 64, t0, &ss.bar_tma);
            tma_load_2d(sm + kP_QK + b * 16384 + 8192, a.tm_k, jq * kD + b * 64, t0, &ss.bar_tma);
        }
    }
    if (warp < 2) {
        const int h = h0 + warp;
        const float g0 = (lane < len) ? load_g(g, (size_t)(t0 + lane) * hv + h, act, h) : 0.f;
        const float g1 = (lane + 32 < len) ? load_g(g, (size_t)(t0 + lane + 32) * hv + h, act, h) : 0.f;
        const float b0 = (lane < len) ? load_beta(beta, (size_t)(t0 + lane) * hv + h, act) : 0.f;
        const float b1 = (lane + 32 < len) ? load_beta(beta, (size_t)(t0 + lane + 32) * hv + h, act) : 0.f;
        const float G0 = warp_inclusive_scan(g0, lane);
        const float G1 = warp_inclusive_scan(g1, lane) + __shfl_sync(0xffffffffu, G0, 31);
        const float GL = __shfl_sync(0xffffffffu, G1, 31);  // g = 0 past the length: the last row's sum
        ss.G[warp][lane] = G0 * kLog2e;
        ss.G[warp][lane + 32] = G1 * kLog2e;
        ss.gam[warp][lane] = expf(G0);
        ss.gam[warp][lane + 32] = expf(G1);
        ss.b[warp][lane] = b0;
        ss.b[warp][lane + 32] = b1;
        ss.c[warp][lane] = (lane < len) ? expf(GL - G0) : 0.f;
        ss.c[warp][lane + 32] = (lane + 32 < len) ? expf(GL - G1) : 0.f;
    }
    tc_fence_before();
    hbar(bid, 256);
    tc_fence_after();

    // ---- 1. Gram: TMEM[0:128, 0:128] = [Q; K] [Q; K]^T  (M = N = 128, K = 128)
    if (tid == 0) {
        if (mbar_wait(&ss.bar_tma, ph)) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t d = sdesc_sw128(sb + kP_QK + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                mma_bf16(tmem, d, d, idesc, s > 0);
            }
            mma_commit(&ss.bar_mma);
        }
    }
    ok = mbar_wait(&ss.bar_mma, ph);
    if (hbar_or(bid, 256, !ok)) return false;
    tc_fence_after();

    // ---- 2. norms from the Gram's diagonal: row R = 32 qw + lane has q_R.q_R (R < 64) or
    //         k_{R-64}.k_{R-64} at column R
    {
        const uint32_t trow = tmem + ((uint32_t)qw * 32u << 16);
        if (hf == 0) {
            float d[32];
            tmem_ld32(trow + 32 * qw, d);
            tmem_ld_wait();
            float x = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) x = (e == lane) ? d[e] : x;
            if (qw < 2) ss.rq[32 * qw + lane] = rsqrtf(x + kNormEps) * kInvSqrtD;
            else ss.rk[32 * (qw - 2) + lane] = rsqrtf(x + kNormEps);
        }
        hbar(bid, 256);

        // ---- 3. decay masks from the Gram's key columns (64 + 32 hf ..): quarters 0-1 (Q rows)
        //         P = lower(exp(G_r - G_j) r_q r_k Q K^T) of both heads, row-major; quarters 2-3
        //         (K rows) A = strictly_lower(b_r exp(G_r - G_j) r_k r_k K K^T), row-major.
        float row[32];
        const int r = (qw & 1) * 32 + lane;  // token row
        const int j0 = 32 * hf;              // first key column of this thread
        tmem_ld32(trow + 64 + j0, row);
        tmem_ld_wait();
        const float* rkj = ss.rk + j0;
        if (qw < 2) {
            const float sr = ss.rq[r];
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const float Gr = ss.G[hh][r];
                const float* gj = ss.G[hh] + j0;
                float4* Pm = reinterpret_cast<float4*>(PP + hh * kMat + r * kLdA + j0);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    float p4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * m + e;
                        p4[e] = (j0 + i <= r) ? fast_exp2(fminf(Gr - gj[i], 0.f)) * sr * rkj[i] * row[i] : 0.f;
                    }
                    Pm[m] = make_float4(p4[0], p4[1], p4[2], p4[3]);
                }
            }
        } else {
            const float sr = ss.rk[r];
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const float Gr = ss.G[hh][r], br = ss.b[hh][r] * sr;
                const float* gj = ss.G[hh] + j0;
                float4* a4 = reinterpret_cast<float4*>(AT + hh * kMat + r * kLdA + j0);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    float x4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * m + e;
                        x4[e] = (j0 + i < r) ? br * fast_exp2(fminf(Gr - gj[i], 0.f)) * rkj[i] * row[i] : 0.f;
                    }
                    a4[m] = make_float4(x4[0], x4[1], x4[2], x4[3]);
                }
            }
        }
    }
    tc_fence_before();
    hbar(bid, 256);

    // ---- 4. T = (I + A)^-1 per head in 32 x 32 blocks.  With A11, A22 the diagonal blocks and
    //         A21 the lower-left one (A strictly lower triangular),
    //           T11 = (I + A11)^-1,  T22 = (I + A22)^-1,  T21 = -T22 A21 T11,  T12 = 0.
    //  (a) T11 and T22 one row per thread (warps 0-3): row r of a diagonal block satisfies
    //      x (I + Abb) = e_r, so x_j = [j == r] - sum_{i > j} x_i A_ij within the block.  Taking i
    //      from the top down, x_i is final when reached and its terms go to every lower x_j at
    //      once (row i of A, read by all threads of the head as broadcasts); every chain is at
    //      most 31 steps long.
    {
        if (tid < 128) {
            const int hh = warp >> 1, c0 = 32 * (warp & 1);  // head, first row / column of the block
            const int rr = c0 + lane;
            const float* A = AT + hh * kMat + c0;
            float2 x[16];  // x_{c0 + 2m}, x_{c0 + 2m + 1}
#pragma unroll
            for (int m = 0; m < 16; ++m) x[m] = make_float2(2 * m == lane ? 1.f : 0.f, 2 * m + 1 == lane ? 1.f : 0.f);
#pragma unroll
            for (int i = 31; i >= 1; --i) {  // block-local row i
                const float xi = (i & 1) ? x[i >> 1].y : x[i >> 1].x;
                const float2 nx = make_float2(-xi, -xi);
                const float4* ar = reinterpret_cast<const float4*>(A + (c0 + i) * kLdA);
                // highest columns first: x_{i-1} is final soonest, so the next step can start
                // while this one's other terms are still in flight
#pragma unroll
                for (int m = (i - 1) / 4; m >= 0; --m) {
                    const float4 av = ar[m];
                    // pairs (4m, 4m+1) and (4m+2, 4m+3); only columns below i take the term
                    if (4 * m + 3 < i) x[2 * m + 1] = __ffma2_rn(nx, make_float2(av.z, av.w), x[2 * m + 1]);
                    else if (4 * m + 2 < i) x[2 * m + 1].x = fmaf(-xi, av.z, x[2 * m + 1].x);
                    if (4 * m + 1 < i) x[2 * m] = __ffma2_rn(nx, make_float2(av.x, av.y), x[2 * m]);
                    else x[2 * m].x = fmaf(-xi, av.x, x[2 * m].x);
                }
            }
            hbar(bid, 256);  // every thread is done reading A11 and A22
            // the block's row, columns c0 .. c0 + 31; A21 (rows 32.., columns 0..31) stays
            float4* dst = reinterpret_cast<float4*>(AT + hh * kMat + rr * kLdA + c0);
#pragma unroll
            for (int m = 0; m < 8; ++m) dst[m] = make_float4(x[2 * m].x, x[2 * m].y, x[2 * m + 1].x, x[2 * m + 1].y);
        } else {
            hbar(bid, 256);
        }
    }
    hbar(bid, 256);  // T11 and T22 are complete

    // The products below run on the warp tensor cores (m16n8k8, tf32).  Each fp32 factor goes in
    // as a tf32 high part and its remainder, and hi hi + hi lo + lo hi keep about 21 bits, more
    // than the bf16 splits downstream take.  Matrices are the row-major fp32 blocks above (row
    // stride kLdA); lane (gq, tq) = (lane / 4, lane % 4).
    const int gq = lane >> 2, tq = lane & 3;
    auto frag_a = [&](const float* M, int r0, int k0, uint32_t* hi, uint32_t* lo) {
        const float* pr = M + (r0 + gq) * kLdA + k0 + tq;
        const float v4[4] = {pr[0], pr[8 * kLdA], pr[4], pr[8 * kLdA + 4]};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            hi[e] = tf32_hi(v4[e]);
            lo[e] = __float_as_uint(v4[e] - __uint_as_float(hi[e]));
        }
    };
    // d += hi hi, e += hi lo + lo hi: two accumulators halve the chain of dependent MMAs
    auto mma3 = [&](float* d, float* e, const uint32_t* ah, const uint32_t* al, const float* M, int k0, int n0) {
        const float* pr = M + (k0 + tq) * kLdA + n0 + gq;
        const float b0 = pr[0], b1 = pr[4 * kLdA];
        const uint32_t bh0 = tf32_hi(b0), bh1 = tf32_hi(b1);
        const uint32_t bl0 = __float_as_uint(b0 - __uint_as_float(bh0));
        const uint32_t bl1 = __float_as_uint(b1 - __uint_as_float(bh1));
        mma_tf32(e, ah[0], ah[1], ah[2], ah[3], bl0, bl1);
        mma_tf32(d, ah[0], ah[1], ah[2], ah[3], bh0, bh1);
        mma_tf32(e, al[0], al[1], al[2], al[3], bh0, bh1);
    };
    //  (b) Y = T22 A21 (rows 32..63, columns 0..31; T22 is lower triangular, so row block rb sums
    //      k over 32 .. 32 + 16 rb + 15) and then T21 = -Y T11 (T11 lower triangular: column tile
    //      nt sums k over 8 nt .. 31).  Warp w: head w / 4, row block (w / 2) % 2, and column
    //      tiles {0, 3} or {1, 2} of the four, which gives every warp the same number of steps
    //      of the second product.
    {
        const int hh = warp >> 2, rb = (warp >> 1) & 1, nh = warp & 1;
        const int ntA = nh ? 1 : 0, ntB = nh ? 2 : 3;
        float* M = AT + hh * kMat;
        float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float ye[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            if (s <= 2 * rb + 1) {
                uint32_t ah[4], al[4];
                frag_a(M, 32 + 16 * rb, 32 + 8 * s, ah, al);
                mma3(y[0], ye[0], ah, al, M, 32 + 8 * s, 8 * ntA);
                mma3(y[1], ye[1], ah, al, M, 32 + 8 * s, 8 * ntB);
            }
        }
        hbar(bid, 256);  // every warp is done reading A21
        float* yr = M + (32 + 16 * rb + gq) * kLdA + 2 * tq;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int nt = j ? ntB : ntA;
            *reinterpret_cast<float2*>(yr + 8 * nt) = make_float2(y[j][0] + ye[j][0], y[j][1] + ye[j][1]);
            *reinterpret_cast<float2*>(yr + 8 * kLdA + 8 * nt) = make_float2(y[j][2] + ye[j][2], y[j][3] + ye[j][3]);
        }
        hbar(bid, 256);  // Y is complete (in A21's place)
        float t21[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float te[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            if (s >= ntA) {  // ntA <= ntB
                uint32_t ah[4], al[4];
                frag_a(M, 32 + 16 * rb, 8 * s, ah, al);
                mma3(t21[0], te[0], ah, al, M, 8 * s, 8 * ntA);
                if (s >= ntB) mma3(t21[1], te[1], ah, al, M, 8 * s, 8 * ntB);
            }
        }
        hbar(bid, 256);  // every warp is done reading Y
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int nt = j ? ntB : ntA;
            *reinterpret_cast<float2*>(yr + 8 * nt) = make_float2(-(t21[j][0] + te[j][0]), -(t21[j][1] + te[j][1]));
            *reinterpret_cast<float2*>(yr + 8 * kLdA + 8 * nt) =
                make_float2(-(t21[j][2] + te[j][2]), -(t21[j][3] + te[j][3]));
        }
    }
    hbar(bid, 256);  // T is complete

    // ---- 5. P T = P (I + A)^-1 per head.  Both factors are lower triangular, so tile (row block
    //         ab of 16, column tile nt of 8) sums k over 8 nt .. 16 ab + 15 only (2 ab + 2 - nt
    //         steps of 8), and the tiles past the block diagonal stay as P left them (zero).  The
    //         70 tile-steps of a head go to its 4 warps as runs of column tiles of one row block,
    //         17 or 18 steps each (one A fragment serves all tiles of a run):
    //           warp 0: (3, tiles 0-1), (0, 0-1)      warp 1: (3, 2-3), (1, 0-1)
    //           warp 2: (3, 4-7), (1, 2-3), (2, 4-5)  warp 3: (2, 0-3)
    {
        const int hh = warp >> 2, q = warp & 3;
        const float* Pm = PP + hh * kMat;
        const float* Tm = AT + hh * kMat;
        // runs (row block, first tile, last tile); a row block of -1 marks no run
        int run[3][3];
        switch (q) {
            case 0: run[0][0] = 3; run[0][1] = 0; run[0][2] = 1; run[1][0] = 0; run[1][1] = 0; run[1][2] = 1; run[2][0] = -1; break;
            case 1: run[0][0] = 3; run[0][1] = 2; run[0][2] = 3; run[1][0] = 1; run[1][1] = 0; run[1][2] = 1; run[2][0] = -1; break;
            case 2: run[0][0] = 3; run[0][1] = 4; run[0][2] = 7; run[1][0] = 1; run[1][1] = 2; run[1][2] = 3; run[2][0] = 2; break;
            default: run[0][0] = 2; run[0][1] = 0; run[0][2] = 3; run[1][0] = -1; run[2][0] = -1; break;
        }
        if (q == 2) { run[2][1] = 4; run[2][2] = 5; }
        float d[8][4], e[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t) d[t][0] = d[t][1] = d[t][2] = d[t][3] = e[t][0] = e[t][1] = e[t][2] = e[t][3] = 0.f;
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const int ab = run[u][0], n0 = run[u][1], n1 = run[u][2];
            if (ab < 0) continue;  // warp-uniform
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                if (s >= n0 && s <= 2 * ab + 1) {
                    uint32_t ah[4], al[4];
                    frag_a(Pm, 16 * ab, 8 * s, ah, al);
#pragma unroll
                    for (int j = 0; j < (u == 0 ? 4 : 2); ++j)  // accumulator slots: run 0 -> 0..3, 1 -> 4..5, 2 -> 6..7
                        if (n0 + j <= n1 && n0 + j <= s) mma3(d[2 * u + (u > 0 ? 2 : 0) + j], e[2 * u + (u > 0 ? 2 : 0) + j], ah, al, Tm, 8 * s, 8 * (n0 + j));
                }
            }
        }
        hbar(bid, 256);  // every warp is done reading P
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const int ab = run[u][0], n0 = run[u][1], n1 = run[u][2];
            if (ab < 0) continue;
            float* dst = PP + hh * kMat + (16 * ab + gq) * kLdA + 2 * tq;
#pragma unroll
            for (int j = 0; j < (u == 0 ? 4 : 2); ++j) {
                if (n0 + j <= n1) {
                    const float* dj = d[2 * u + (u > 0 ? 2 : 0) + j];
                    const float* ej = e[2 * u + (u > 0 ? 2 : 0) + j];
                    *reinterpret_cast<float2*>(dst + 8 * (n0 + j)) = make_float2(dj[0] + ej[0], dj[1] + ej[1]);
                    *reinterpret_cast<float2*>(dst + 8 * kLdA + 8 * (n0 + j)) = make_float2(dj[2] + ej[2], dj[3] + ej[3]);
                }
            }
        }
    }
    if (tid < 128) {  // per-column factors of step 6, once
        const int hh = tid >> 6, i = tid & 63;
        ss.fw[hh][i] = ss.b[hh][i] * ss.gam[hh][i] * ss.rk[i];
        ss.fk[hh][i] = ss.c[hh][i] * ss.rk[i];
    }
    // With a ring, the slot's previous chunk (cid - ring) must have been taken by the state
    // passes of both heads before its records are overwritten.
    ok = true;
    if (a.ring && cid >= a.ring && tid == 0) {
        ok = wait_consumed(a.consumed + rslot * hv + h0, cid - a.ring + 1, reinterpret_cast<int32_t*>(ws));
        if (ok) fence_async_global();
    }
    if (hbar_or(bid, 256, !ok)) return false;

    // ---- 6. per head, 128 threads.
    //   (a) thread l takes row l & 63 of T (l < 64) or of P T (l >= 64) and writes Tensor Memory
    //       A-operand row l: T diag(b gam r_k) split high / low (l < 64), or -P T diag(b gam r_k)
    //       with a zero low part (l >= 64); thread 0 also writes gam_L.
    //   (b) the [T diag(b); At = P T diag(b)] images, split high / low, straight to the
    //       workspace: thread l takes the 16-byte chunk l & 7 of rows l / 8 + 16 m, so that a
    //       warp's store covers four whole 128-byte rows.
    {
        const int hh = tid >> 7, l = tid & 127, rr = l & 63;
        const bool trow = l < 64;
        const int h = h0 + hh;
        unsigned char* rec = ws + L.rec + (rslot * hv + h) * kRecBytes;
        const float* bb = ss.b[hh];
        const float* fw = ss.fw[hh];
        {
            const float* src = (trow ? AT : PP) + hh * kMat + rr * kLdA;
            const uint32_t ta = tmem + ((uint32_t)(l & ~31) << 16) + 128 + 64 * hh;
            uint32_t whi[32], wlo[32];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const float4 x0 = *reinterpret_cast<const float4*>(src + 8 * ch);
                const float4 x1 = *reinterpret_cast<const float4*>(src + 8 * ch + 4);
                const float4 f0 = *reinterpret_cast<const float4*>(fw + 8 * ch);
                const float4 f1 = *reinterpret_cast<const float4*>(fw + 8 * ch + 4);
                const float sg = trow ? 1.f : -1.f;
                const float cw[8] = {sg * x0.x * f0.x, sg * x0.y * f0.y, sg * x0.z * f0.z, sg * x0.w * f0.w,
                                     sg * x1.x * f1.x, sg * x1.y * f1.y, sg * x1.z * f1.z, sg * x1.w * f1.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint32_t hi, lo;
                    split2(cw[2 * e], cw[2 * e + 1], hi, lo);
                    whi[4 * ch + e] = hi;
                    wlo[4 * ch + e] = trow ? lo : 0u;
                }
            }
            tmem_st16(ta, whi);
            tmem_st16(ta + 16, whi + 16);
            tmem_st16(ta + 32, wlo);
            tmem_st16(ta + 48, wlo + 16);
            if (l == 0) {
                float* fac = reinterpret_cast<float*>(rec + kFacOff);
                fac[0] = ss.gam[hh][kChunk - 1];  // gam_L (G is constant past the length)
            }
        }
        {
            unsigned char* ta_hi = rec + kWQBytes;
            unsigned char* ta_lo = ta_hi + kTABytes;
            const int ch = l & 7;
            float b8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) b8[e] = bb[8 * ch + e];
#pragma unroll 2
            for (int m = 0; m < 8; ++m) {
                const int row = (l >> 3) + 16 * m;  // image row: T rows 0..63, then P T rows
                const float* src = (row < 64 ? AT + row * kLdA : PP + (row - 64) * kLdA) + hh * kMat + 8 * ch;
                const float4 x0 = *reinterpret_cast<const float4*>(src);
                const float4 x1 = *reinterpret_cast<const float4*>(src + 4);
                const float v[8] = {x0.x * b8[0], x0.y * b8[1], x0.z * b8[2], x0.w * b8[3],
                                    x1.x * b8[4], x1.y * b8[5], x1.z * b8[6], x1.w * b8[7]};
                uint32_t th[4], tl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) split2(v[2 * e], v[2 * e + 1], th[e], tl[e]);
                *reinterpret_cast<uint4*>(ta_hi + sw128(row, ch)) = make_uint4(th[0], th[1], th[2], th[3]);
                *reinterpret_cast<uint4*>(ta_lo + sw128(row, ch)) = make_uint4(tl[0], tl[1], tl[2], tl[3]);
            }
        }
        {   // (c) Kt = diag(c r_k) K in fp32, K-major (tokens contiguous).  Thread item i = l + 128 m:
            //     token block i / 256, d_k rows 4 ((i / 8) % 32) .. + 3, tokens 32 (i / 256) + 4 (i % 8)
            //     .. + 3: four 8-byte reads of K rows, four 16-byte chunks of Kt rows -- a warp's store
            //     covers four whole 128-byte rows
            unsigned char* kt = rec + kKTOff;
            const float* fk = ss.fk[hh];
#pragma unroll 2
            for (int m = 0; m < 4; ++m) {
                const int i = l + 128 * m;
                const int kb = i >> 8, dk = 4 * ((i >> 3) & 31), tc = i & 7;
                const int t = 32 * kb + 4 * tc;  // first of the 4 tokens
                const unsigned char* kblk = sm + kP_QK + (dk >> 6) * 16384 + 8192 + (dk & 7) * 2;
                float v[4][4];  // [token][d_k]
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint2 kr = *reinterpret_cast<const uint2*>(kblk + sw128(t + e, (dk & 63) >> 3));
                    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.x));
                    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.y));
                    const float sc = fk[t + e];
                    v[e][0] = a.x * sc; v[e][1] = a.y * sc; v[e][2] = b.x * sc; v[e][3] = b.y * sc;
                }
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    *reinterpret_cast<float4*>(kt + kb * 16384 + sw128(dk + d, tc)) =
                        make_float4(v[0][d], v[1][d], v[2][d], v[3][d]);
            }
        }
        tmem_st_wait();
    }
    tc_fence_before();
    hbar(bid, 256);

    // ---- 7. per head: TMEM[0:128, 0:128] = A_hi K + A_lo K (rows 0-63: W, rows 64-127:
    //         -P T diag(b gam r_k) K); the -W and Qt = diag(gam r_q) Q + (rows 64-127) images are
    //         assembled in the (now free) fp32 region in their final swizzled layout and leave
    //         as one 32 KB bulk copy per head.
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 128, 0, 1);  // A from TMEM (K-major), B MN-major
            const uint32_t a = tmem + 128 + 64 * hh;
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16_tmem_a(tmem, a + 8 * (s & 3) + 32 * (s >> 2),
                                sdesc_sw128(sb + kP_QK + 8192 + (s & 3) * 2048, 16384, 1024), idesc, s > 0);
            mma_commit(&ss.bar_mma);
        }
        ok = mbar_wait(&ss.bar_mma, (ph + 1 + hh) & 1);
        if (hbar_or(bid, 256, !ok)) return false;
        tc_fence_after();
        {
            unsigned char* img = sm + kP_AT + hh * kWQBytes;  // staging image of this head
            const uint32_t trow = tmem + ((uint32_t)qw * 32u << 16);
            const int r = (qw & 1) * 32 + lane;
            const float sq = (qw >= 2) ? ss.gam[hh][r] * ss.rq[r] : 0.f;
            float col[32];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(trow + 64 * hf + 32 * half, col);
                tmem_ld_wait();
                if (qw < 2) {  // -W row r, d_k block hf
#pragma unroll
                    for (int e = 0; e < 32; ++e) col[e] = -col[e];
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        *reinterpret_cast<uint4*>(img + hf * 16384 + sw128(r, 4 * half + ch)) = pack8(col + 8 * ch);
                } else {  // Qt row r = gam_r r_q,r q_r + (the product row), d_k block hf
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float q8[8];
                        unpack8(*reinterpret_cast<const uint4*>(sm + kP_QK + hf * 16384 + sw128(r, 4 * half + ch)), q8);
#pragma unroll
                        for (int e = 0; e < 8; ++e) q8[e] = fmaf(sq, q8[e], col[8 * ch + e]);
                        *reinterpret_cast<uint4*>(img + hf * 16384 + 8192 + sw128(r, 4 * half + ch)) = pack8(q8);
                    }
                }
            }
            fence_async_smem();
        }
        tc_fence_before();
        hbar(bid, 256);  // the product is read before the next head's MMA overwrites it
        if (tid == 32) {
            bulk_s2g(ws + L.rec + (rslot * hv + h0 + hh) * kRecBytes, sm + kP_AT + hh * kWQBytes, kWQBytes);
            bulk_commit();
        }
    }
    // The item's records are complete when the image copies have finished (not only read shared
    // memory, whose regions the next item reuses) and every thread's direct stores are visible.
    if (a.ready) {
        __threadfence();
        if (tid == 32) {
            bulk_wait_all();
            fence_async_global();
        }
        hbar(bid, 256);
        if (tid == 0) st_release_gpu(a.ready + (size_t)cid * (hv / 2) + pair, 1);
    } else if (tid == 32) {
        bulk_wait_read_all();
    }
    return true;
}

// After a failed item: this item's MMAs complete before its Tensor Memory is freed or reused
// (thread 0 of the item; d counts the drains these threads have done before).
__device__ __forceinline__ void prep_drain(PrepSmall& ss, int tid, uint32_t d) {
    if (tid == 0) {
        mma_commit(&ss.bar_drain);
        mbar_wait(&ss.bar_drain, d & 1);
    }
    if (tid == 32) bulk_wait_all();
}

__global__ void __launch_bounds__(kPrepThreads, 2)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const float* __restrict__ g, const float* __restrict__ beta, unsigned char* ws,
                  int num_seqs, int total_tokens, int hk, int hv, GateAct act) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    PrepSmall& ss = *reinterpret_cast<PrepSmall*>(sm + kP_SMALL);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int npairs = hv / 2;
    const int cid = blockIdx.x / npairs;
    const int tid = threadIdx.x, warp = tid >> 5;
    grid_dependency_wait();    // the chunk table is written
    allow_dependent_launch();  // the state kernel may be scheduled as SMs free up
    if (cid >= header[1]) return;
    if (warp == 0) {
        tmem_alloc(&ss.tmem_base, 256);
        tmem_relinquish();
    }
    if (tid == 32) prep_init_barriers(ss);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;
    const PrepArgs a{&tm_q, &tm_k, g, beta, ws, num_seqs, total_tokens, hk, hv, act, nullptr, nullptr, 0};
    if (!prep_item(a, cid, blockIdx.x % npairs, sm, tmem, tid, 1, 0)) {
        if (tid == 0) atomicOr(header, 1);
        prep_drain(ss, tid, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ===================================================================== K2
// State pass, one CTA per (sequence, V head).  With S the fp32 state entering chunk c (held in
// registers by the row workers, its bf16 copy in Tensor Memory as the A operand), per chunk
// three groups of eight N = 128 MMAs (an MMA instruction costs the issuing thread about the
// same whatever its N up to 128, so the products are merged into as few as possible):
//   (2) D_c  = V^T [Tb; At]_hi^T + V^T [Tb; At]_lo^T   D_c = [U^T | O^T]    (no dependence on S)
//   (1) D_c += S [-W; Qt]^T  (bf16)                   D_c = [Delta^T | O^T]
//   (3) SA   = Delta^T Kt    (tf32, A = D_c's first 64 columns, Kt = diag(c r_k) K in fp32)
//   S <- gam_L S + SA
// (1) and (3) follow each other in the tensor pipe with no thread in between; the chain per
// chunk is S -> (1) -> (3) -> S.  D is double-buffered so that (2) of chunk c+1 runs while the
// row workers update the state; the tensor-pipe order is (1)_c (3)_c (2)_{c+1}.
//
// Warps: 0 loads (bulk copies and TMA), 1 issues MMAs, 2..9 row workers (the state: lane
// quarter warp % 4 = d_v rows 32 q .. 32 q + 31, half (warp - 2) / 4 of the d_k columns),
// 10..13 output warps (lane quarter warp % 4, all 64 tokens).  The outputs of a full chunk are
// staged in the slot's V tile, which (2) has finished with, and leave by TMA store.
constexpr int kStateThreads = 448;
constexpr int kRowThreads = 256;
constexpr int kOutWarp0 = 10;
constexpr uint32_t kSl_WQ = 0;          // [-W; Qt] image (32 KB)
constexpr uint32_t kSl_TA = 32768;      // TA_hi (16 KB) then TA_lo (16 KB)
constexpr uint32_t kSl_V = 65536;       // V tile: 2 d_v blocks x 64 tokens x 128 B (TMA); later the outputs
constexpr uint32_t kSl_KT = 81920;      // Kt^T, fp32, K-major (32 KB)
constexpr uint32_t kSlotBytes = 114688; // 112 KB, a multiple of 1024
constexpr uint32_t kSlotTx = 65536 + 16384 + kKTBytes + kFacLoad;
constexpr uint32_t kS_SMALL = 2 * kSlotBytes;
constexpr uint32_t kStateSmem = kS_SMALL + 256 + 1024;  // small struct + alignment slack
constexpr uint32_t kEmptyArrivals = 5;                  // the MMA commit and the 4 output warps
// Tensor Memory columns
constexpr uint32_t kT_D = 0;     // D buffers at 0 and 128: [Delta^T | O^T] (2 x 128)
constexpr uint32_t kT_SA = 256;  // state update (128)
constexpr uint32_t kT_SB = 384;  // S in bf16, the A operand of (1) (64)
constexpr uint32_t kTmemCols = 512;

struct StateSmall {
    alignas(16) float gl[2][4];  // gam_L of the chunk in each slot (a 16-byte bulk-copy target)
    uint64_t full[2], empty[2];
    uint64_t s_ready;            // row workers -> issuer (256 arrivals)
    uint64_t o_done;             // output warps -> issuer (128 arrivals)
    uint64_t mo, msa;            // MMA commits -> output warps, row workers
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(StateSmall) <= 256, "StateSmall fits its region");

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

// Bounded wait (one thread) for a flag another CTA of the same launch raises; returns false
// (and raises the CTA's abort flag, recording the error) if it gave up, or at once if another
// CTA has recorded an error.
__device__ bool wait_flag(const int32_t* flag, volatile int* abort_flag, int32_t* header) {
    if (wait_flag_set(flag, header, kWaitLimitNs)) return true;
    *abort_flag = 1;
    atomicOr(header, 1);
    return false;
}

// The state pass of sequence n, V head h, by the CTA's threads 0..447 (any further threads of
// the CTA take part in its barriers only).  sm is the CTA's 1024-aligned shared memory
// (kStateSmem bytes), tmem its kTmemCols Tensor Memory columns.  With `ready` set, the loads of
// chunk c first wait (bounded) for that chunk's flag: the records are then produced while this
// pass runs, by the other CTAs of the same launch.
__device__ void state_body(const CUtensorMap* tm_v_p, const CUtensorMap* tm_out_p, const float* s0,
                           const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out, float* sT,
                           StateSlots map, float* cstates, unsigned char* ws, int num_seqs, int total_tokens,
                           int hv, int n, int h, unsigned char* sm, uint32_t tmem, const int32_t* ready,
                           int32_t* consumed, int ring) {
    const uint32_t sb = smem_u32(sm);
    StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + kS_SMALL);
    volatile int* abort_flag = &ss.abort_flag;
    const CUtensorMap& tm_v = *tm_v_p;
    const CUtensorMap& tm_out = *tm_out_p;

    const WsLayout L = ws_layout(num_seqs, total_tokens, hv);
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 32) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ss.full[s], 1);
            mbar_init(&ss.empty[s], kEmptyArrivals);
        }
        mbar_init(&ss.s_ready, kRowThreads);
        mbar_init(&ss.o_done, 128);
        mbar_init(&ss.mo, 1);
        mbar_init(&ss.msa, 1);
        mbar_init(&ss.drain, 1);
        ss.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_out);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dependency_wait();  // (two-phase launch) the prep kernel's workspace is complete and visible
    const int32_t* seq_chunk0 = reinterpret_cast<const int32_t*>(ws + L.seq_chunk0);
    const int cs = seq_chunk0[n], nch = seq_chunk0[n + 1] - cs;
    const int t_begin = cu[n], t_end = cu[n + 1];
    auto rec_of = [&](int c) {
        const size_t slot_c = ring ? (size_t)((cs + c) % ring) : (size_t)(cs + c);
        return ws + L.rec + (slot_c * hv + h) * kRecBytes;
    };

    if (warp == 0) {
        // ------------------------------------------------ loads, one slot ahead
        if (lane == 0 && nch > 0) {
            // chunk j's workspace record and V tile into L2, kAhead chunks before its slot load,
            // so that the slot fills are L2 hits
            auto prefetch = [&](int j) {
                if (j >= nch) return;
                const unsigned char* rec = rec_of(j);
                if (!ready) bulk_prefetch_l2(rec, kFacOff + kFacLoad);  // fused: not written yet
                const int tj = t_begin + j * kChunk;
                tma_prefetch_l2_2d(&tm_v, h * kD, tj);
                tma_prefetch_l2_2d(&tm_v, h * kD + 64, tj);
            };
            constexpr int kAhead = 4;
            for (int j = 2; j < kAhead; ++j) prefetch(j);
            int k = 0;
            for (; k < nch; ++k) {
                prefetch(k + kAhead);
                const int st = k & 1;
                if (k >= 2 && !wait_or_abort(&ss.empty[st], ((k >> 1) - 1) & 1, abort_flag, header)) break;
                unsigned char* slot = sm + st * kSlotBytes;
                const unsigned char* rec = rec_of(k);
                const int tk = t_begin + k * kChunk;
                if (ready && !wait_flag(ready + (size_t)(cs + k) * (hv / 2) + h / 2, abort_flag, header)) break;
                mbar_arrive_expect_tx(&ss.full[st], kSlotTx);
                bulk_g2s(slot + kSl_WQ, rec, 65536, &ss.full[st]);
                bulk_g2s(slot + kSl_KT, rec + kKTOff, kKTBytes, &ss.full[st]);
                bulk_g2s(&ss.gl[st][0], rec + kFacOff, kFacLoad, &ss.full[st]);
                tma_load_2d(slot + kSl_V, &tm_v, h * kD, tk, &ss.full[st]);
                tma_load_2d(slot + kSl_V + 8192, &tm_v, h * kD + 64, tk, &ss.full[st]);
            }
            if (*abort_flag) {  // drain: copies in flight land before the CTA exits
                for (int j = max(0, k - 2); j < k; ++j) mbar_wait(&ss.full[j & 1], (j >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && nch > 0) {
            const uint32_t id_s = idesc_bf16(128, 128, 0, 0);   // (1): A TMEM, B K-major
            const uint32_t id_v = idesc_bf16(128, 128, 1, 0);   // (2): A (V^T) MN-major, B K-major
            const uint32_t id_k = idesc_tf32(128, 128, 0, 0);   // (3): A TMEM (fp32), B (Kt) K-major
            auto issue_2 = [&](int c) {  // D_c = V^T [Tb; At]^T, high then low part
                const uint32_t slot = sb + (c & 1) * kSlotBytes;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + kT_D + 128 * (c & 1), sdesc_sw128(slot + kSl_V + (s & 3) * 2048, 8192, 1024),
                             sdesc_sw128(slot + kSl_TA + (s >> 2) * kTABytes + (s & 3) * 32, 16, 1024), id_v, s > 0);
            };
            bool ok = wait_or_abort(&ss.full[0], 0, abort_flag, header);
            if (ok) {
                tc_fence_after();
                issue_2(0);
            }
            for (int c = 0; ok && c < nch; ++c) {
                const uint32_t slot = sb + (c & 1) * kSlotBytes;
                const uint32_t dcol = tmem + kT_D + 128 * (c & 1);
                // (1) once S_c is in Tensor Memory.  The output warps released D_{c-1} (o_done);
                // waiting for it here, before the commit below, keeps the wait from ever falling
                // two phases behind.
                if (!(ok = wait_or_abort(&ss.s_ready, c & 1, abort_flag, header))) break;
                if (c >= 1 && !(ok = wait_or_abort(&ss.o_done, (c - 1) & 1, abort_flag, header))) break;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_tmem_a(dcol, tmem + kT_SB + 8 * s,
                                    sdesc_sw128(slot + kSl_WQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), id_s, 1);
                mma_commit(&ss.mo);
                // (3): SA = Delta^T Kt, Delta^T from the first 64 columns of D_c
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_tf32_tmem_a(tmem + kT_SA, dcol + 8 * s,
                                    sdesc_sw128(slot + kSl_KT + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), id_k, s > 0);
                mma_commit(&ss.msa);
                mma_commit(&ss.empty[c & 1]);  // every MMA reading slot c has been issued
                // (2) of the next chunk into the other D buffer (released with D_{c-1} above); it
                // runs while the row workers update the state
                if (c + 1 < nch) {
                    if (!(ok = wait_or_abort(&ss.full[(c + 1) & 1], ((c + 1) >> 1) & 1, abort_flag, header))) break;
                    tc_fence_after();
                    issue_2(c + 1);
                }
            }
            if (*abort_flag) {  // drain: every MMA issued so far completes before TMEM is freed
                mma_commit(&ss.drain);
                mbar_wait(&ss.drain, 0);
            }
        }
    } else if (warp < kOutWarp0) {
        // ------------------------------------------------ row workers: the state
        const int q4 = warp & 3, hf = (warp - 2) >> 2;
        const int dv = 32 * q4 + lane;  // d_v row of S this thread owns, d_k columns 64 hf ..
        const uint32_t trow = tmem + ((uint32_t)q4 * 32u << 16);
        bool has_state;
        const int sidx = state_index(map, n, has_state);
        if (!has_state) { s0 = nullptr; sT = nullptr; }  // no slot: start from zeros, keep no state
        float* srow_out = sT ? sT + ((size_t)sidx * hv + h) * kD * kD + (size_t)dv * kD + 64 * hf : nullptr;
        float S[64];
        if (s0) {
            const float4* src = reinterpret_cast<const float4*>(s0 + ((size_t)sidx * hv + h) * kD * kD + (size_t)dv * kD + 64 * hf);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float4 x = src[m];
                S[4 * m] = x.x; S[4 * m + 1] = x.y; S[4 * m + 2] = x.z; S[4 * m + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int m = 0; m < 64; ++m) S[m] = 0.f;
        }
        auto write_sb = [&]() {  // bf16 copy of this thread's 64 state columns -> the A operand
            uint32_t w[32];
#pragma unroll
            for (int m = 0; m < 32; ++m) w[m] = pack2(S[2 * m], S[2 * m + 1]);
            tmem_st16(trow + kT_SB + 32 * hf, w);
            tmem_st16(trow + kT_SB + 32 * hf + 16, w + 16);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&ss.s_ready);
        };
        if (nch > 0) write_sb();
        bool alive = true;
        for (int c = 0; c < nch && alive; ++c) {
            if (!(alive = wait_or_abort(&ss.full[c & 1], (c >> 1) & 1, abort_flag, header))) break;
            if (consumed && warp == 2 && lane == 0)  // the chunk's records are in shared memory: its ring slot is free
                st_release_gpu(consumed + (size_t)((cs + c) % ring) * hv + h, cs + c + 1);
            const float gl = ss.gl[c & 1][0];
            if (!(alive = wait_or_abort(&ss.msa, c & 1, abort_flag, header))) break;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float sa[32];
                tmem_ld32(trow + kT_SA + 64 * hf + 32 * half, sa);
                tmem_ld_wait();
#pragma unroll
                for (int m = 0; m < 32; ++m) S[32 * half + m] = fmaf(gl, S[32 * half + m], sa[m]);
            }
            if (c + 1 < nch) write_sb();
            if (cstates) {  // the state after this chunk
                float4* cr = reinterpret_cast<float4*>(cstates + ((size_t)(cs + c) * hv + h) * kD * kD + (size_t)dv * kD + 64 * hf);
#pragma unroll
                for (int m = 0; m < 16; ++m) cr[m] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
            }
        }
        if (alive && !*abort_flag && srow_out) {
            float4* dst = reinterpret_cast<float4*>(srow_out);
#pragma unroll
            for (int m = 0; m < 16; ++m) dst[m] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
        }
    } else if (warp < kOutWarp0 + 4) {
        // ------------------------------------------------ output warps
        const int q4 = warp & 3;
        const int dv = 32 * q4 + lane;  // d_v row of O^T this thread reads, all 64 tokens
        const uint32_t trow = tmem + ((uint32_t)q4 * 32u << 16);
        for (int c = 0; c < nch; ++c) {
            if (!wait_or_abort(&ss.mo, c & 1, abort_flag, header)) break;
            tc_fence_after();
            const uint32_t dcol = kT_D + 128 * (c & 1) + 64;
            float o[64];
            tmem_ld32(trow + dcol, o);
            tmem_ld32(trow + dcol + 32, o + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&ss.o_done);  // D_c has been read
            const int t0 = t_begin + c * kChunk;
            const int len = min(kChunk, t_end - t0);
            if (len == kChunk) {
                // a 64-token x 32-d_v tile, row-major in the slot's V area (its (2) is complete:
                // (1) of this chunk, which follows it in the pipe, has completed), one TMA store
                unsigned char* st = sm + (c & 1) * kSlotBytes + kSl_V + q4 * 4096;
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    *reinterpret_cast<__nv_bfloat16*>(st + e * 64 + lane * 2) = __float2bfloat16_rn(o[e]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tm_out, h * kD + 32 * q4, t0, st);
                    bulk_commit();
                    bulk_wait_read_all();  // the tile is read before the slot is released
                }
            } else {
                __nv_bfloat16* op = out + ((size_t)t0 * hv + h) * kD + dv;
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (e < len) op[(size_t)e * hv * kD] = __float2bfloat16_rn(o[e]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ss.empty[c & 1]);
        }
        if (lane == 0) bulk_wait_all();  // this warp's output TMA stores have completed
    }
}

__global__ void __launch_bounds__(kStateThreads, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                   const float* s0, const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out, float* sT,
                   StateSlots map, float* cstates, unsigned char* ws, int num_seqs, int total_tokens, int hk,
                   int hv) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + kS_SMALL);
    (void)hk;
    // Set-up that needs nothing from the prep kernel runs before the dependency wait (a CTA of
    // this kernel never shares an SM with a prep CTA: their shared memory does not fit
    // together, so the Tensor Memory columns are free).
    if (threadIdx.x < 32) {
        tmem_alloc(&ss.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss.tmem_base;
    state_body(&tm_v, &tm_out, s0, cu, out, sT, map, cstates, ws, num_seqs, total_tokens, hv, blockIdx.x / hv,
               blockIdx.x % hv, sm, tmem, nullptr, nullptr, 0);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ===================================================================== K1 + K2 in one launch
// For a batch with few (sequence, V head) chains the state pass occupies few SMs and the prep
// pass must finish before it starts.  This cooperative launch runs both at once: CTAs
// 0 .. nstate-1 are the state passes (one per chain), every other CTA runs two prep workers of
// 256 threads (halves of the CTA, named barriers 1 and 2, 256 Tensor Memory columns each) that
// take the (chunk, pair) items in chunk order and raise each item's flag once its records are
// complete; a state pass waits for a chunk's flag before it loads the chunk.  All CTAs are
// resident at once (cooperative launch, one CTA per SM), and no prep worker waits for a state
// pass, so every flag is eventually raised; all waits are bounded and give up when another CTA
// has recorded an error.
constexpr int kFusedThreads = 512;
constexpr uint32_t kFusedSmem = (kStateSmem > 2 * kPrepRegion + 1024) ? kStateSmem : 2 * kPrepRegion + 1024;

__global__ void __launch_bounds__(kFusedThreads, 1)
chunk_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                   const float* __restrict__ g, const float* __restrict__ beta, const float* s0,
                   const int32_t* __restrict__ cu, __nv_bfloat16* __restrict__ out, float* sT, StateSlots map,
                   float* cstates, unsigned char* ws, int num_seqs, int total_tokens, int hk, int hv, GateAct act,
                   int nstate) {
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    __shared__ uint32_t tmem_s;
    const int tid = threadIdx.x, warp = tid >> 5;
    int32_t* header = reinterpret_cast<int32_t*>(ws);
    const WsLayout L = ws_layout(num_seqs, total_tokens, hv);
    int32_t* ready = reinterpret_cast<int32_t*>(ws + L.flags);
    int32_t* consumed = ready + L.max_chunks * (hv / 2);
    const int ring = L.max_chunks > kRing ? kRing : 0;
    const bool is_state = (int)blockIdx.x < nstate;
    if (warp == 0) {
        tmem_alloc(&tmem_s, 512);
        tmem_relinquish();
    }
    if (!is_state && (tid & 255) == 32) prep_init_barriers(*reinterpret_cast<PrepSmall*>(sm + (tid >> 8) * kPrepRegion + kP_SMALL));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_s;
    if (is_state) {
        state_body(&tm_v, &tm_out, s0, cu, out, sT, map, cstates, ws, num_seqs, total_tokens, hv, blockIdx.x / hv,
                   blockIdx.x % hv, sm, tmem, ready, ring ? consumed : nullptr, ring);
    } else {
        const int half = tid >> 8, ltid = tid & 255;
        const uint32_t bid = 1 + half;
        unsigned char* hsm = sm + half * kPrepRegion;
        PrepSmall& ss = *reinterpret_cast<PrepSmall*>(hsm + kP_SMALL);
        const int npairs = hv / 2;
        const long long items = (long long)header[1] * npairs;
        const long long worker = (long long)(blockIdx.x - nstate) * 2 + half;
        const long long nworkers = (long long)(gridDim.x - nstate) * 2;
        const PrepArgs a{&tm_q, &tm_k, g, beta, ws, num_seqs, total_tokens, hk, hv, act, ready, consumed, ring};
        uint32_t j = 0;
        for (long long it = worker; it < items; it += nworkers, ++j) {
            if (hbar_or(bid, 256, *reinterpret_cast<volatile int32_t*>(header) != 0)) break;  // another CTA gave up
            if (!prep_item(a, (int)(it / npairs), (int)(it % npairs), hsm, tmem + 256u * half, ltid, bid, j)) {
                if (ltid == 0) atomicOr(header, 1);
                prep_drain(ss, ltid, 0);
                break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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

// ---- TMA descriptors: a bf16 [rows][heads * 128] tensor, boxes of box_y rows x box_x elements
//      (64 x 64 by default: 128 bytes, the 128-byte swizzle width); loads read rows past the end
//      as zeros, stores do not write them.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

cudaError_t encode_rows(CUtensorMap* m, const void* base, int rows, int heads,
                        CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B, unsigned box_x = 64,
                        unsigned box_y = 64) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)heads * kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)heads * kD * 2};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

size_t tc_workspace_bytes(int num_seqs, int total_tokens, int hk, int hv) {
    (void)hk;
    return ws_layout(num_seqs, total_tokens, hv).total;
}

size_t tc_fused_workspace_bytes(int num_seqs, int total_tokens, int hk, int hv) {
    (void)hk;
    const WsLayout L = ws_layout(num_seqs, total_tokens, hv);
    const long long slots = L.max_chunks > kRing ? kRing : L.max_chunks;  // the record ring
    return round_up(L.rec + (size_t)slots * hv * kRecBytes, 1024);
}

cudaError_t launch_prefill_tc_prep(const void* q, const void* k, const float* g, const float* beta,
                                   const int32_t* cu, int num_seqs, int total_tokens, int hk, int hv,
                                   void* workspace, GateAct act, cudaStream_t stream) {
    if (num_seqs == 0) return cudaSuccess;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const WsLayout L = ws_layout(num_seqs, total_tokens, hv);
    chunk_table_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total_tokens, hv, ws);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || L.max_chunks == 0 || total_tokens == 0) return e;
    CUtensorMap tq, tk;
    if ((e = encode_rows(&tq, q, total_tokens, hk)) != cudaSuccess) return e;
    if ((e = encode_rows(&tk, k, total_tokens, hk)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrepSmem)) !=
        cudaSuccess)
        return e;
    e = launch_dependent(chunk_prep_kernel, dim3((unsigned)(L.max_chunks * (hv / 2))), dim3(kPrepThreads), kPrepSmem,
                         stream, tq, tk, g, beta, ws, num_seqs, total_tokens, hk, hv, act);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc_state(const void* k, const void* v, const float* s0, const int32_t* cu, void* out,
                                    float* sT, StateSlots map, float* cstates, int num_seqs, int total_tokens, int hk,
                                    int hv, void* workspace, cudaStream_t stream) {
    (void)k;  // the keys reach the state pass as Kt, in the workspace
    if (num_seqs == 0) return cudaSuccess;
    // a zero-token batch still hands every initial state through; the descriptors then cover
    // one (never read) row of the caller's buffers
    const int rows = total_tokens > 0 ? total_tokens : 1;
    CUtensorMap tv, to;
    cudaError_t e;
    if ((e = encode_rows(&tv, v ? v : workspace, rows, v ? hv : 1)) != cudaSuccess) return e;
    // the outputs leave row-major (unswizzled) staging tiles of 64 tokens x 32 d_v
    if ((e = encode_rows(&to, out ? out : workspace, rows, out ? hv : 1, CU_TENSOR_MAP_SWIZZLE_NONE, 32, 64)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem)) !=
        cudaSuccess)
        return e;
    e = launch_dependent(chunk_state_kernel, dim3((unsigned)num_seqs * hv), dim3(kStateThreads), kStateSmem, stream, tv,
                         to, s0, cu, (__nv_bfloat16*)out, sT, map, cstates, static_cast<unsigned char*>(workspace),
                         num_seqs, total_tokens, hk, hv);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

bool fused_prefill_applies(int num_seqs, int total_tokens, int hv) {
    if (num_seqs <= 0 || total_tokens <= 0) return false;
    int dev = 0, sms = 0, coop = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop) return false;
    return 2LL * num_seqs * hv <= sms;
}

cudaError_t launch_prefill_tc_fused(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                   const float* s0, const int32_t* cu, void* out, float* sT, StateSlots map,
                                   float* cstates, int num_seqs, int total_tokens, int hk, int hv, void* workspace,
                                   GateAct act, cudaStream_t stream) {
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    chunk_table_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total_tokens, hv, ws);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv, to;
    if ((e = encode_rows(&tq, q, total_tokens, hk)) != cudaSuccess) return e;
    if ((e = encode_rows(&tk, k, total_tokens, hk)) != cudaSuccess) return e;
    if ((e = encode_rows(&tv, v, total_tokens, hv)) != cudaSuccess) return e;
    if ((e = encode_rows(&to, out, total_tokens, hv, CU_TENSOR_MAP_SWIZZLE_NONE, 32, 64)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(chunk_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmem)) !=
        cudaSuccess)
        return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_fused_kernel, kFusedThreads, kFusedSmem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int nstate = num_seqs * hv;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms);  // one CTA per SM, all resident (cooperative launch)
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = kFusedSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, chunk_fused_kernel, tq, tk, tv, to, g, beta, s0, cu, (__nv_bfloat16*)out, sT, map,
                           cstates, ws, num_seqs, total_tokens, hk, hv, act, nstate);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
