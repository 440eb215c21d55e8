/*
 * gdn.h -- C ABI of libgdn.so, the B200 (sm_100a) Gated DeltaNet layer.
 *
 * The layer.  Gated DeltaNet is the linear-attention layer of Qwen3-Next
 * (Qwen3-Next-80B-A3B model card, "Highlights": Hybrid Attention; "Model Overview":
 * Gated DeltaNet with 32 linear-attention heads for V and 16 for QK, head dimension
 * 128; the layout puts it in 36 of the 48 layers).  Per sequence and per V head h it
 * keeps a fixed-size fp32 state S (d_v x d_k = 128 x 128) and applies the gated delta
 * rule to every token:
 *
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * where k_t = k / sqrt(|k|^2 + 1e-6), q_t = q / sqrt(|q|^2 + 1e-6) / sqrt(128)
 * (normalisation and scaling happen inside the library: pass raw q and k), g_t <= 0
 * and 0 < beta_t < 1 (already activated gates; documented preconditions, not checked
 * on the device).  V head h reads QK head h / (num_v_heads / num_qk_heads), i.e. V
 * heads 2j and 2j+1 share QK head j in the 16/32 layout.
 *
 * Layouts (all contiguous, row-major, token-major; T = total packed tokens,
 * N = num_seqs, HK = num_qk_heads, HV = num_v_heads, D = head_dim = 128):
 *   q, k          [T][HK][D]   io dtype (bf16 or fp32)
 *   v, out        [T][HV][D]   io dtype
 *   g, beta       [T][HV]      fp32
 *   states        [N][HV][D][D] fp32, S[n][h][i][j] with i the d_v (row) index
 *   cu_seqlens    [N+1] int32, DEVICE memory, cu_seqlens[0] = 0, non-decreasing,
 *                 cu_seqlens[N] = T; sequence n owns tokens [cu[n], cu[n+1]).
 * For decode the token axis is [N][num_tokens] flattened (sequence-major).
 *
 * Ownership and behaviour common to all entry points:
 *   - Every pointer except `shape` is a device pointer owned by the caller; the
 *     library never allocates, frees, synchronises or reads device memory on the
 *     host inside gdn_chunk_prefill / gdn_decode_step.  Work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = legacy default stream).  Both calls are
 *     therefore stream-ordered and can be captured into CUDA graphs.
 *   - Device pointers must be 16-byte aligned (GDN_ERR_ALIGN otherwise).
 *   - The return value reports host-side validation and launch errors only.  Device
 *     side faults surface through the CUDA runtime (GDN_ERR_CUDA from a later call or
 *     cudaStreamSynchronize); a bounded device wait that gave up is recorded in the
 *     workspace and read back by gdn_get_device_error.
 *   - `out` must not alias any input.  initial_state and final_state may alias each
 *     other (in-place state carry).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 2

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = 1,           /* a required pointer is NULL */
    GDN_ERR_SHAPE = 2,          /* unsupported or inconsistent sizes */
    GDN_ERR_ALIGN = 3,          /* a device pointer is not 16-byte aligned */
    GDN_ERR_DTYPE = 4,          /* io_dtype not one of gdn_dtype */
    GDN_ERR_NUM_TOKENS = 5,     /* decode num_tokens outside [1, 4] */
    GDN_ERR_WORKSPACE = 6,      /* workspace missing or smaller than required */
    GDN_ERR_CUDA = 7,           /* the CUDA runtime reported an error */
    GDN_ERR_DEVICE_TIMEOUT = 8, /* a bounded device-side wait expired */
    GDN_ERR_UNSUPPORTED = 9     /* requested algorithm not available for these inputs */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* Prefill algorithm selection (gdn_shape.algo). */
typedef enum {
    GDN_ALGO_AUTO = 0,          /* tensor-core path where it applies, else the SIMT fp32 path */
    GDN_ALGO_SIMT = 1,          /* chunked form on CUDA cores in fp32 (any io dtype) */
    GDN_ALGO_TENSOR = 2         /* chunked form on tcgen05 tensor cores: bf16 I/O and an even
                                   number of V heads per QK head only */
} gdn_algo;

typedef struct {
    int32_t num_seqs;      /* N >= 0 (prefill: sequences; decode: batch) */
    int32_t total_tokens;  /* T >= 0 (prefill only; decode ignores it) */
    int32_t max_seqlen;    /* optional hint, 0 = unknown; if > 0 must be <= total_tokens */
    int32_t num_qk_heads;  /* HK >= 1 */
    int32_t num_v_heads;   /* HV, a multiple of HK */
    int32_t head_dim;      /* must be 128 (d_k = d_v) */
    int32_t io_dtype;      /* gdn_dtype of q, k, v, out */
    int32_t algo;          /* gdn_algo (prefill only) */
} gdn_shape;

/*
 * Workspace the caller must provide to gdn_chunk_prefill (and its _slots, _chunk_states,
 * _raw_gates variants) for `shape` (bytes, a multiple of 256).  It depends on
 * total_tokens, num_seqs, the head counts, the algorithm and the current device: when the
 * (sequence, V head) chains fill at most half of the device's SMs the tensor-core prefill
 * runs both of its passes in one cooperative launch and keeps its per-chunk operands in
 * a ring of a few chunks (about 46 MB at 32 V heads, whatever the length); otherwise the
 * workspace holds the operands of every chunk (about 50 KB per token at 16/32 heads).
 * Query it with the device current that will run the call: a call whose path needs more
 * than it is given returns GDN_ERR_WORKSPACE.  Returns 0 if the shape is invalid.
 */
size_t gdn_prefill_workspace_bytes(const gdn_shape *shape);

/*
 * Workspace of the two-phase entry points gdn_chunk_prefill_prep / gdn_chunk_prefill_state
 * (the operands of every chunk; at least gdn_prefill_workspace_bytes).  Returns 0 if the
 * shape is invalid or does not take the tensor-core path.
 */
size_t gdn_prefill_phase_workspace_bytes(const gdn_shape *shape);

/*
 * Chunked prefill over a packed varlen batch.  The chunked form of the gated delta
 * rule processes each sequence in chunks of 64 tokens: per chunk it builds the
 * cumulative-gate-weighted intra-chunk UT representation (the unit lower-triangular
 * system I + strictly_lower(beta * K K^T * decay)), applies it to the entering state
 * and carries the fp32 state to the next chunk.  Chunks restart at each sequence
 * start; the last chunk of a sequence may be partial; empty sequences are allowed
 * (their final state equals their initial state).
 *
 *   q, k, v, g, beta   inputs, layouts above
 *   initial_state      [N][HV][D][D] fp32, or NULL for zero states
 *   cu_seqlens         [N+1] int32 device array
 *   out                [T][HV][D] written for every token
 *   final_state        [N][HV][D][D] fp32, or NULL (not written); may alias initial_state
 *   shape              host pointer
 *   workspace          device scratch of >= gdn_prefill_workspace_bytes(shape) bytes,
 *                      256-byte aligned; its contents on entry do not matter; it must
 *                      not be shared by calls that overlap on the device
 *   stream             cudaStream_t
 */
gdn_status gdn_chunk_prefill(const void *q, const void *k, const void *v,
                             const float *g, const float *beta,
                             const float *initial_state, const int32_t *cu_seqlens,
                             void *out, float *final_state, const gdn_shape *shape,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * The tensor-core prefill in two phases, for callers that want to schedule or time
 * them separately (gdn_chunk_prefill is exactly prep followed by state on one stream).
 *
 * gdn_chunk_prefill_prep: builds the chunk table from cu_seqlens and, for every chunk and
 *   V head in parallel, the chunk's coefficient images into `workspace`: the solved UT
 *   system T = (I + strictly_lower(beta K K^T decay))^-1 applied to the keys (W) and folded
 *   into the queries, T diag(beta) and its product with the decay-masked Q K^T, and the gate
 *   factors.  Reads q, k, g, beta, cu_seqlens.
 * gdn_chunk_prefill_state: carries each sequence's fp32 state across its chunks using the
 *   workspace written by the prep phase of the same shape, reading the raw keys and values
 *   again, and writes out and final_state.  Reads k, v, initial_state, cu_seqlens.
 * Both require io_dtype == GDN_BF16, an even number of V heads per QK head and an algo of
 * GDN_ALGO_AUTO or GDN_ALGO_TENSOR (GDN_ERR_UNSUPPORTED otherwise); arguments as for
 * gdn_chunk_prefill.  The workspace header is cleared by the prep phase.
 */
gdn_status gdn_chunk_prefill_prep(const void *q, const void *k, const float *g, const float *beta,
                                  const int32_t *cu_seqlens, const gdn_shape *shape,
                                  void *workspace, size_t workspace_bytes, void *stream);
gdn_status gdn_chunk_prefill_state(const void *k, const void *v, const float *initial_state,
                                   const int32_t *cu_seqlens, void *out, float *final_state,
                                   const gdn_shape *shape, void *workspace, size_t workspace_bytes,
                                   void *stream);

/*
 * Decode / multi-token verify step: advances every sequence's state by num_tokens
 * (1..4) tokens in place and writes the output of every token.  This is the memory
 * bound step a speculative-decoding verifier uses (the pages' multi-token prediction
 * serving, up to 4 draft tokens).
 *
 *   q, k            [N][num_tokens][HK][D] io dtype (raw; normalised inside)
 *   v               [N][num_tokens][HV][D] io dtype
 *   g, beta         [N][num_tokens][HV] fp32
 *   state_inout     [N][HV][D][D] fp32, read and overwritten with the state after
 *                   the last token
 *   out             [N][num_tokens][HV][D] io dtype
 *   num_tokens      1..4, the same for every sequence (GDN_ERR_NUM_TOKENS otherwise)
 *   shape           uses num_seqs, num_qk_heads, num_v_heads, head_dim, io_dtype
 */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *g, const float *beta, float *state_inout,
                           void *out, int32_t num_tokens, const gdn_shape *shape,
                           void *stream);

/*
 * Speculative verify with per-token state snapshots (the multi-token prediction
 * serving of the pages -- vLLM blog post, "Multi-Token Prediction"; Qwen3-Next model
 * card, "Deployment" -- checks up to 4 draft tokens per step and keeps only the
 * accepted ones, so the state must be recoverable after any prefix of the drafts).
 *
 * gdn_decode_verify: same inputs and outputs as gdn_decode_step, except that `state`
 *   is only read, and the state after each token t (t = 0 .. num_tokens-1) is written
 *   to `snapshots`:
 *     state       [N][HV][D][D] fp32, read only
 *     snapshots   [N][num_tokens][HV][D][D] fp32, written; snapshots[n][t] is the state
 *                 after tokens 0..t of sequence n (must not overlap state, inputs or out)
 *   The outputs are those gdn_decode_step gives for the same tokens.
 * gdn_decode_commit: for every sequence n with 1 <= accepted[n] <= num_tokens, copies
 *   snapshots[n][accepted[n] - 1] into state[n]; a sequence with any other count (0:
 *   every draft rejected) keeps its state.
 *     accepted    [N] int32, DEVICE memory (typically written by the sampler on the GPU)
 *   num_tokens must be the value the snapshots were written with.
 * Errors as for gdn_decode_step (GDN_ERR_NULL for a missing snapshots or accepted
 * pointer); the commit reads num_seqs, num_v_heads and head_dim of `shape`.  Bytes moved: verify reads the state once and writes num_tokens states;
 * commit reads and writes one state per sequence that accepted a draft.
 */
gdn_status gdn_decode_verify(const void *q, const void *k, const void *v,
                             const float *g, const float *beta, const float *state,
                             void *out, float *snapshots, int32_t num_tokens,
                             const gdn_shape *shape, void *stream);
gdn_status gdn_decode_commit(float *state, const float *snapshots, const int32_t *accepted,
                             int32_t num_tokens, const gdn_shape *shape, void *stream);

/*
 * Gates from raw projections.  The entry points above take the activated gates g <= 0 and
 * beta in (0, 1).  These three take instead, per token and V head, the raw projections x
 * (decay) and y (write strength) and per V head a decay rate a > 0 and a bias b, and apply
 *
 *     g = -a[h] * softplus(x + b[h]),   softplus(z) = log(1 + exp(z)),
 *     beta = sigmoid(y) = 1 / (1 + exp(-y))
 *
 * in fp32 where the kernels load the gates (no separate pass, nothing written back).  The
 * pages give only the activated gates; this activation is the usual parameterisation of
 * the decay and write strength of gated delta rules, offered as an option.
 *   x, y        same layout as g and beta of the corresponding call ([T][HV], or
 *               [N][num_tokens][HV] for decode), fp32
 *   a, b        [HV] fp32, DEVICE memory, 16-byte aligned (GDN_ERR_NULL / GDN_ERR_ALIGN)
 * Everything else, and every error, as for gdn_chunk_prefill, gdn_decode_step and
 * gdn_decode_verify.
 */
gdn_status gdn_chunk_prefill_raw_gates(const void *q, const void *k, const void *v,
                                       const float *x, const float *y, const float *a,
                                       const float *b, const float *initial_state,
                                       const int32_t *cu_seqlens, void *out, float *final_state,
                                       const gdn_shape *shape, void *workspace,
                                       size_t workspace_bytes, void *stream);
gdn_status gdn_decode_step_raw_gates(const void *q, const void *k, const void *v,
                                     const float *x, const float *y, const float *a,
                                     const float *b, float *state_inout, void *out,
                                     int32_t num_tokens, const gdn_shape *shape, void *stream);
gdn_status gdn_decode_verify_raw_gates(const void *q, const void *k, const void *v,
                                       const float *x, const float *y, const float *a,
                                       const float *b, const float *state, void *out,
                                       float *snapshots, int32_t num_tokens,
                                       const gdn_shape *shape, void *stream);

/*
 * Prefill that also keeps the state at every chunk boundary (for prefix caching: the
 * pages' roadmap lists automatic prefix caching for hybrid models -- vLLM blog post,
 * "Future Work" -- which needs the linear-attention state at cached prefix lengths).
 * Same arguments and results as gdn_chunk_prefill, plus
 *     chunk_states  [C][HV][D][D] fp32, C = sum over sequences of ceil(T_n / 64): the
 *                   state after chunk c of sequence n (after token min(64 (c+1), T_n) - 1)
 *                   is row sum_{m<n} ceil(T_m / 64) + c.  The last row of a sequence equals
 *                   its final state.  Must not overlap the other buffers.
 * GDN_ERR_NULL if chunk_states is missing while there are tokens.  Bytes: one extra state
 * write per chunk (2 MiB per 64 tokens at 32 V heads).
 */
gdn_status gdn_chunk_prefill_chunk_states(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta,
                                          const float *initial_state, const int32_t *cu_seqlens,
                                          void *out, float *final_state, float *chunk_states,
                                          const gdn_shape *shape, void *workspace,
                                          size_t workspace_bytes, void *stream);

/*
 * State-slot indirection (the pages' hybrid cache manager keeps the linear-attention
 * states of running requests in one preallocated pool -- vLLM blog post, "Hybrid KV
 * Cache Management"): the same prefill, decode, verify and commit on states held in
 *     state_pool    [num_slots][HV][D][D] fp32
 * where sequence n's state is state_pool[state_slots[n]].
 *     state_slots   [N] int32, DEVICE memory.  A slot outside [0, num_slots) marks a
 *                   sequence without a state: decode and verify skip it (its outputs and
 *                   snapshots are not written) and commit leaves the pool unchanged for it;
 *                   prefill runs it from a zero state and writes no final state.
 * gdn_chunk_prefill_slots reads each sequence's initial state from its slot and writes
 * the final state back to the same slot (in place); otherwise the arguments are those of
 * gdn_chunk_prefill.  Two sequences of one call must not share a valid slot.
 * GDN_ERR_NULL for a missing pool or slot table, GDN_ERR_SHAPE for num_slots < 0; the
 * rest as for the dense entry points.
 */
gdn_status gdn_chunk_prefill_slots(const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, float *state_pool,
                                   const int32_t *state_slots, int32_t num_slots,
                                   const int32_t *cu_seqlens, void *out, const gdn_shape *shape,
                                   void *workspace, size_t workspace_bytes, void *stream);
gdn_status gdn_decode_step_slots(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta, float *state_pool,
                                 const int32_t *state_slots, int32_t num_slots, void *out,
                                 int32_t num_tokens, const gdn_shape *shape, void *stream);
gdn_status gdn_decode_verify_slots(const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, const float *state_pool,
                                   const int32_t *state_slots, int32_t num_slots, void *out,
                                   float *snapshots, int32_t num_tokens, const gdn_shape *shape,
                                   void *stream);
gdn_status gdn_decode_commit_slots(float *state_pool, const int32_t *state_slots,
                                   int32_t num_slots, const float *snapshots,
                                   const int32_t *accepted, int32_t num_tokens,
                                   const gdn_shape *shape, void *stream);

/*
 * Reads the device error word of a prefill workspace (synchronises `stream`; meant for
 * tests and debugging).  Returns GDN_ERR_DEVICE_TIMEOUT if a bounded device wait of a
 * previous prefill gave up, GDN_ERR_CUDA if the runtime reports an error, else GDN_OK.
 */
gdn_status gdn_get_device_error(void *workspace, void *stream);

/*
 * Prefill that allocates nothing, for callers that cannot allocate device memory where
 * they run (for example a plugin whose host framework owns every device allocation and
 * hands it only fixed input and output buffers, or code that must not block on an
 * allocation on its hot path).  The paper has no counterpart: this is a library
 * convenience, not part of the method.
 *
 * Same arguments and results as gdn_chunk_prefill on the tensor-core path, minus the
 * workspace: the scratch is a static device array of GDN_NOALLOC_SCRATCH_BYTES bytes
 * inside libgdn.so, which every GPU that loads the library holds until exit.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Workloads whose gdn_prefill_workspace_bytes(shape) exceeds the maximum are rejected
 *     with GDN_ERR_WORKSPACE.  With 16 QK / 32 V heads on a 148-SM device one or two
 *     sequences of any length fit (their operands live in a ring of a few chunks); larger
 *     batches fit up to about 21 chunks of 64 tokens in all.  fp32 I/O or GDN_ALGO_SIMT give
 *     GDN_ERR_UNSUPPORTED.
 *   - The first call on each device (with that device current) looks up the array's
 *     device address and caches it with the identity of the device's current context;
 *     make that first call before any stream capture.  If the context changes (after
 *     cudaDeviceReset, for instance) the next call looks the address up again, so make
 *     the first call after a reset before any capture as well.
 *   - Every call on a device shares the one array, which keeps the previous call's
 *     contents; each call clears what must start at zero.  Calls that overlap on the GPU
 *     (e.g. on unordered streams) race on the array.
 *   - A bounded device wait that gave up is recorded in the array's header; read it with
 *     gdn_get_noalloc_device_error.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
gdn_status gdn_chunk_prefill_noalloc(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     void *out, float *final_state, const gdn_shape *shape,
                                     void *stream);

/*
 * The device error word of gdn_chunk_prefill_noalloc's static scratch on the current
 * device (its callers never see the array's address, so gdn_get_device_error cannot be
 * given it).  Synchronises `stream` and returns GDN_ERR_DEVICE_TIMEOUT if a bounded
 * device wait of the last allocation-free prefill on this device gave up, GDN_ERR_CUDA
 * if the runtime reports an error, else GDN_OK.  Meant for tests and debugging.
 */
gdn_status gdn_get_noalloc_device_error(void *stream);

/*
 * The device error word of the decode and verify kernels on the current device.  The
 * multi-token kernels (num_tokens 2..4) wait on asynchronous copies with a bounded wait;
 * if one gives up, the kernel stops early (the results of that call are undefined) and
 * records it here.  Synchronises `stream`, returns GDN_ERR_DEVICE_TIMEOUT if a wait gave up
 * since the last read (and clears the word), GDN_ERR_CUDA if the runtime reports an error,
 * else GDN_OK.  Meant for tests and debugging.
 */
gdn_status gdn_get_decode_device_error(void *stream);

/*
 * Failure-path self-test.  Clears the workspace header, then launches a kernel that runs
 * each kind of bounded wait the kernels use -- on a flag another CTA would raise, on a pair
 * of marks, and on an mbarrier phase -- against something nothing completes, with a limit
 * of `limit_us` microseconds each (1 .. 2,000,000).  When the limits expire the kernel
 * records the timeout in the header and returns normally; a following
 * gdn_get_device_error(workspace, stream) then returns GDN_ERR_DEVICE_TIMEOUT and the
 * CUDA context remains usable.  `workspace` needs >= 256 bytes, 256-byte aligned.
 */
gdn_status gdn_selftest_wait_timeout(void *workspace, size_t workspace_bytes, uint32_t limit_us,
                                     void *stream);

/* Static, human-readable name of a status code. */
const char *gdn_status_string(gdn_status status);

/* GDN_ABI_VERSION of the loaded library. */
int32_t gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
