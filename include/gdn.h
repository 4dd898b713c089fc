/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta rule library, libgdn.so.
 *
 * The operation (state S in R^{d_v x d_k} per sequence and head, o_t = S_t q_t):
 *   Gated DeltaNet (scalar decay alpha_t in (0,1), one beta_t for erase and
 *   write):   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   KDA (channel-wise decay Diag(alpha_t), alpha_t in R^{d_k}):
 *             S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 * Sources: "FG2-GDN: Enhancing Long-Context Gated Delta Networks with Doubly
 * Fine-Grained Control", section 1 (GDN, then KDA's Diag(alpha_t) as a tied
 * diagonal-plus-rank-1 transition), section 3.6 (the chunkwise WY / UT
 * algorithm), section 5 (the unified view S_t = A_t S_{t-1} + k_t v_t^T,
 * o_t = S_t^T q_t, i.e. this map transposed); "Gated Delta Networks: Improving
 * Mamba2 with Delta Rule", section 3.1 (one beta_t in both terms) and 3.3
 * (scalar cumulative decay inside a chunk).
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers to contiguous row-major memory,
 *     owned by the caller; the library keeps no pointer after a call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns after launch.  Nothing is allocated.
 *   - Layouts are token-major: q, k [B, T, H, d_k]; v, o [B, T, H, d_v];
 *     log_alpha [B, T, H] (scalar decay) or [B, T, H, d_k] (channel decay),
 *     fp32, natural log of alpha (so <= 0 for a decay); beta [B, T, H] fp32.
 *     For a packed variable-length batch B = 1, T = total tokens and
 *     cu_seqlens holds the N+1 int32 sequence offsets.
 *   - States are fp32 [N, H, d_v, d_k] (row i = output channel i, d_k
 *     contiguous), N = number of sequences.
 *   - q, k, v and o share one dtype (gdn_dtype).  No scale is applied to q:
 *     a caller that wants 1/sqrt(d_k) scales q first.
 *   - Supported head sizes: d_k, d_v in {64, 128}.
 *   - Errors: argument errors are detected on the host before any launch and
 *     return a status without touching the device.  A failed launch returns
 *     GDN_ERR_CUDA.  Errors only the device can see (inconsistent cu_seqlens
 *     contents, an expired bounded wait) set a sticky error word in the
 *     workspace, read and cleared by gdn_workspace_status().  No call traps.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque stream handle; pass a cudaStream_t (the same pointer type). */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID = 1,      /* bad argument (null, shape, alignment, size)    */
    GDN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d_k = 96)       */
    GDN_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed           */
    GDN_ERR_TIMEOUT = 4,      /* a device-side bounded wait expired             */
    GDN_ERR_DEVICE_INPUT = 5  /* the device found bad cu_seqlens contents       */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_FP32 = 1 } gdn_dtype;
typedef enum { GDN_DECAY_SCALAR = 0, GDN_DECAY_CHANNEL = 1 } gdn_decay;

/* Kernel selection flags (gdn_dims.flags).  0 = the library's choice: for bf16
 * with d_k = d_v = 128, channel decay on the two-CTA tensor-core kernel; scalar
 * decay on the pool kernel when the sequences hold 2048 tokens or more on average
 * (B * T / n_seqs) and there are at most SMs / 4 (sequence, head) chains, else on
 * the two-CTA kernel from 2048 tokens on average and on the single-CTA kernel
 * below; the fp32 CUDA-core kernel for every other shape.  GDN_FLAG_POOL,
 * GDN_FLAG_PAIR and GDN_FLAG_ONE_CTA select one of the three tensor-core kernels
 * (at most one of them; GDN_FLAG_POOL and GDN_FLAG_ONE_CTA take scalar decay only,
 * else GDN_ERR_INVALID).  The pool kernel is one persistent grid over all SMs:
 * a few CTAs run the sequential state pass of all chains while the others work
 * through the chunk-local steps of every chunk, so one long sequence uses the
 * whole GPU.  The two-CTA kernel runs one thread-block cluster per sequence and
 * head (one SM for the chunk-local steps, one for the state pass); it is exact
 * for any decay (a channel that decays by more than e^-80 over 16 tokens has its
 * within-block terms taken directly).  Both need a larger workspace (see below).
 * GDN_FLAG_CUDA_CORES forces the fp32 CUDA-core kernel.  The tests use the flags
 * to compare the device paths. */
enum { GDN_FLAG_CUDA_CORES = 1, GDN_FLAG_PAIR = 2, GDN_FLAG_ONE_CTA = 4, GDN_FLAG_POOL = 8,
       GDN_FLAG_BETA_CHANNEL = 16, GDN_FLAG_VALUE_RATE = 32 };
/* GDN_FLAG_BETA_CHANNEL (prefill, channel decay): FG2-GDN's writing rate per key
 * channel (FG2-GDN paper, section 3.2 "FG2-GDN Update Rule" and 3.6 "Chunkwise
 * Parallel Training").  beta is then [B, T, H, d_k] fp32 (per-channel rates in
 * (0, 1]) and the update is
 *     S_t = S_{t-1} Diag(alpha_t) (I - k~_t k~_t^T) + v_t k~_t^T,  k~_t = sqrt(beta_t) . k_t,
 * KDA's update with unit rate on the square-root-scaled keys.  It runs on the
 * two-CTA kernel (bf16, d_k = d_v = 128): GDN_ERR_UNSUPPORTED for every other
 * shape, with GDN_FLAG_CUDA_CORES, for gdn_recurrent_step and on the
 * no-allocation entry point; GDN_ERR_INVALID with scalar decay,
 * GDN_FLAG_ONE_CTA or GDN_FLAG_POOL.
 * GDN_FLAG_VALUE_RATE (with GDN_FLAG_BETA_CHANNEL): FG2-GDN+'s value-side rate
 * (section 3.4 "FG2-GDN+ Variant"), v~_t = sqrt(beta^v_t) . v_t in place of v_t
 * in the update above; the call is gdn_chunk_fwd_value_rate, whose workspace
 * (gdn_chunk_fwd_workspace_size with this flag) also holds v~. */

typedef struct {
    int32_t B;       /* batch (1 for a packed batch)                           */
    int32_t T;       /* tokens per batch row (total tokens when packed)         */
    int32_t H;       /* heads                                                   */
    int32_t d_k;     /* key / query head size                                   */
    int32_t d_v;     /* value head size                                         */
    int32_t n_seqs;  /* sequences: B, or len(cu_seqlens) - 1 when packed         */
    int32_t dtype;   /* gdn_dtype of q, k, v, o                                 */
    int32_t decay;   /* gdn_decay                                               */
    int32_t flags;   /* GDN_FLAG_* (0 = default)                                */
} gdn_dims;

/* Bytes of device workspace gdn_chunk_fwd needs for `dims` (always >= 256),
 * on the current device.  The first 256 bytes are a header: word 0 (bytes
 * 0-3) is the sticky error word; word 1 (bytes 4-7), when nonzero, replaces
 * the default limit of the tensor-core kernels' bounded waits on data (2^31 SM
 * clock cycles, about a second) -- a test-only control: set to a few hundred
 * cycles it makes those waits run out on purpose, and the kernels then record
 * GDN_ERR_TIMEOUT, drain their own copies and MMAs, free their tensor memory
 * and return.  Zero the header once before the workspace's first use
 * (gdn_workspace_init).  The
 * two-CTA tensor-core kernel adds a ring of four 64 KiB slots for each SM index
 * of the device (2 x its SM count), through which the chunk-local SM hands each
 * chunk's matrices to the state SM, and (packed batches of up to 4096
 * sequences) the sequences' longest-first order, 4 bytes each, which a small
 * kernel before it writes; both are written before they are read and need no
 * initialisation.  The pool kernel adds eight 73 KiB ring slots per chain
 * CTA, its hand-off flags and (packed batches) a table of round offsets, which
 * a small kernel before it writes.  The other kernels need only the header.  Returns 0 for
 * invalid dims. */
size_t gdn_chunk_fwd_workspace_size(const gdn_dims *dims);

/* Chunkwise (WY / UT-transform) prefill, chunk size C = 64
 * (FG2-GDN section 3.6).  Per sequence and head, over chunks of 64 tokens:
 * cumulative log decay; the strictly lower beta- and decay-scaled K K^T (A);
 * T = (I + A)^{-1}; W = T diag(beta)(decayed K), U = T diag(beta) V; the
 * sequential inter-chunk state pass V' = U - W S^T, S <- decayed S + V'^T K^;
 * and the output (decayed Q) S^T + (causal decayed Q K^T) V'.
 *   q, k, v          inputs, layouts above, dtype dims->dtype
 *   log_alpha, beta  fp32 gates
 *   initial_state    fp32 [N,H,d_v,d_k], or NULL for zeros
 *   cu_seqlens       device int32 [N+1] offsets (0, ..., T, non-decreasing),
 *                    or NULL for B fixed-length rows of T tokens; chunks never
 *                    cross a sequence boundary
 *   o                output [B,T,H,d_v], dtype dims->dtype (rounded once,
 *                    to nearest even, from fp32)
 *   final_state      fp32 [N,H,d_v,d_k] or NULL; may alias initial_state
 *   workspace        device scratch of >= gdn_chunk_fwd_workspace_size bytes,
 *                    16-byte aligned, zeroed before first use; one call at a
 *                    time may use a given workspace
 * q, k, v, o and the states must be 16-byte aligned. */
gdn_status gdn_chunk_fwd(const gdn_dims *dims, const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         const float *initial_state, const int32_t *cu_seqlens,
                         void *o, float *final_state,
                         void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/* gdn_chunk_fwd with the input prologue fused into the kernel: the queries
 * and keys arrive unnormalised and the gates as logits, and the kernel applies
 * (FG2-GDN section 3.5, "Gate Parameterization")
 *   q_t <- q_t / ||q_t||,  k_t <- k_t / ||k_t||   (per token and head, norms in
 *                                                  fp32, clamped below at 1e-12)
 *   beta_t = sigmoid(beta_logit_t)
 *   log alpha_t = -softplus(alpha_logit_t + alpha_bias[h])
 * before the chunkwise pass, without writing the normalised inputs or the
 * gates anywhere: the norms become row and column scales of the chunk
 * products.  The result equals gdn_chunk_fwd on the prologue's outputs up to
 * rounding (the normalised vectors are never rounded to bf16 here).
 *   q_raw, k_raw     [B,T,H,d_k] bf16, unnormalised
 *   alpha_logit      [B,T,H] fp32;  alpha_bias [H] fp32 or NULL (zero)
 *   beta_logit       [B,T,H] fp32
 *   everything else  as for gdn_chunk_fwd; the workspace is that of
 *                    gdn_chunk_fwd_workspace_size for the same dims with
 *                    flags = GDN_FLAG_POOL
 * Scalar decay, bf16, d_k = d_v = 128 only (the pool kernel); other shapes
 * return GDN_ERR_UNSUPPORTED.  dims->flags must be 0 or GDN_FLAG_POOL. */
gdn_status gdn_chunk_fwd_raw(const gdn_dims *dims, const void *q_raw, const void *k_raw,
                             const void *v, const float *alpha_logit, const float *alpha_bias,
                             const float *beta_logit, const float *initial_state,
                             const int32_t *cu_seqlens, void *o, float *final_state,
                             void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/* One recurrent decode step for N = dims->B sequences (dims->T is ignored,
 * one token each): for every (sequence, head), with the state updated in place,
 *   S <- S Diag(alpha) (I - beta k k^T) + beta v k^T   (scalar alpha for GDN)
 *   o  = S q   (read with the updated state)
 * The state's constant size is what makes decoding constant-memory (FG2-GDN
 * abstract and "Inference Challenges"; Gated DeltaNet-2 abstract).
 *   q, k [N,H,d_k], v [N,H,d_v] (dtype dims->dtype); log_alpha [N,H] or
 *   [N,H,d_k]; beta [N,H]; state_inout fp32 [N,H,d_v,d_k]; o [N,H,d_v].
 * No workspace; touches no memory other than these. */
gdn_status gdn_recurrent_step(const gdn_dims *dims, const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              float *state_inout, void *o, gdn_stream_t stream);

/* Multi-token verification for speculative decoding (a chain of K drafts; the
 * TreeWY finding on the Gated DeltaNet-2 page: no per-node state snapshots).
 * For N = dims->B sequences of K = dims->T draft tokens each, the recurrence of
 * gdn_recurrent_step runs through the K tokens from state_inout:
 *   o_t = S_t q_t for t = 0..K-1 (if o is not null);
 *   state_inout <- S_c, the state after the first c = n_commit[n] tokens of
 *   sequence n (n_commit: device int32 [N], values clamped to [0, K]; c = 0, or a
 *   null n_commit, leaves the state untouched).
 * Speculative decoding peeks at a draft (o, n_commit = null), picks the accepted
 * length j per sequence, then commits it (o = null, n_commit = j): the state after
 * j tokens is recomputed from the state before them, so nothing per position is
 * kept.  Layouts are token-major: q, k [N,K,H,d_k]; v, o [N,K,H,d_v]; log_alpha
 * [N,K,H] or [N,K,H,d_k]; beta [N,K,H]; state_inout fp32 [N,H,d_v,d_k].  No
 * workspace.  GDN_FLAG_BETA_CHANNEL is GDN_ERR_UNSUPPORTED. */
gdn_status gdn_recurrent_verify(const gdn_dims *dims, const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta, float *state_inout,
                                const int32_t *n_commit, void *o, gdn_stream_t stream);

/* Tree-shaped drafts (the TreeWY setting on the Gated DeltaNet-2 page): the K =
 * dims->T draft tokens of sequence n form a tree through parent [N,K] int32
 * (device): node j follows node parent[n][j] in [0, j - 1], or the current state
 * when parent[n][j] = -1 (any other value is taken as -1).  o_j = S_j q_j, S_j the
 * state after the path from the current state to node j; n_commit[n] = c >= 1
 * commits the state after node c - 1's path (0 or a null n_commit: untouched), so
 * a chain (parent[n][j] = j - 1) behaves as gdn_recurrent_verify.  K <= 64
 * (GDN_ERR_UNSUPPORTED above).  Layouts and the rest as gdn_recurrent_verify. */
gdn_status gdn_recurrent_verify_tree(const gdn_dims *dims, const void *q, const void *k,
                                     const void *v, const float *log_alpha, const float *beta,
                                     float *state_inout, const int32_t *parent,
                                     const int32_t *n_commit, void *o, gdn_stream_t stream);

/* FG2-GDN+ prefill: gdn_chunk_fwd with dims->flags holding GDN_FLAG_BETA_CHANNEL
 * and GDN_FLAG_VALUE_RATE, and the value-side rate beta_v [B,T,H,d_v] fp32 (16-byte
 * aligned), rates in (0, 1].  A small kernel first writes v~ = sqrt(beta_v) . v
 * (bf16) into the workspace; the prefill then runs on (k~, v~) with unit rate.
 * Without both flags: GDN_ERR_INVALID; gdn_chunk_fwd refuses GDN_FLAG_VALUE_RATE. */
gdn_status gdn_chunk_fwd_value_rate(const gdn_dims *dims, const void *q, const void *k,
                                    const void *v, const float *log_alpha, const float *beta,
                                    const float *beta_v, const float *initial_state,
                                    const int32_t *cu_seqlens, void *o, float *final_state,
                                    void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Segment state maps, for sharding one long sequence over GPUs (the exchange of
 * per-segment affine maps).  Over a segment the recurrence is affine in the state
 * it starts from (FG2-GDN section 1: S_t = S_{t-1} A_t + beta_t v_t k_t^T with
 * A_t = Diag(alpha_t)(I - beta_t k_t k_t^T)):
 *   S_end = S_start M + B,   M = A_1 ... A_n,   B = S_end when S_start = 0.
 * B is gdn_chunk_fwd's final state from a null initial state; M is its final
 * state from the identity (gdn_state_identity) with v = 0 of width d_k (every
 * state row a probe vector, so the state is d_k x d_k).  Consecutive segments
 * compose: S_start(r + 1) = S_start(r) M_r + B_r, after which each segment is
 * rerun from its true start.
 *
 * gdn_state_compose: out = s m + b for every (sequence, head), fp32:
 *   s, b, out [N,H,d_v,d_k]; m [N,H,d_k,d_k]; N = dims->B, H = dims->H.
 *   b may be null (out = s m).  out may alias b, not s or m.  d_v and d_k are
 *   64 or 128; all pointers 16-byte aligned device memory.
 * gdn_state_identity: out [N,H,d_k,d_k] = I (requires d_v == d_k). */
gdn_status gdn_state_compose(const gdn_dims *dims, const float *s, const float *m, const float *b,
                             float *out, gdn_stream_t stream);
gdn_status gdn_state_identity(const gdn_dims *dims, float *out, gdn_stream_t stream);

/* Size of the device array that gdn_chunk_fwd_noalloc uses in place of a
 * caller workspace: 256 KiB, held by every GPU that loads the library until
 * the process exits. */
#define GDN_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/* gdn_chunk_fwd without a workspace argument and without allocating anything.
 * The paper has no counterpart: this is a deployment convenience.
 *
 * Who needs it: code that is handed only its input and output buffers and has
 * no way to get more device memory -- a plugin inside another framework whose
 * allocator it may not call, a serving loop that forbids allocation once it
 * has started, or a process whose device memory is already fully reserved by
 * another allocator, so that a cudaMalloc would fail or fragment it.
 *
 * Instead of a caller workspace it uses one fixed device array of
 * GDN_NOALLOC_SCRATCH_BYTES compiled into the library.  Where the selected
 * kernel's workspace (gdn_chunk_fwd_workspace_size) does not fit in it -- the
 * rings of the pool and two-CTA tensor-core kernels never do -- the call runs
 * the single-CTA tensor-core kernel (scalar decay) or the CUDA-core kernel
 * (channel decay) instead, whose workspace is the header alone.
 * Problems whose workspace exceeds the array even then return
 * GDN_ERR_UNSUPPORTED before anything is launched.  All other arguments,
 * layouts and results are those of gdn_chunk_fwd.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array.  Each call clears its
 *     header on `stream` before the kernels run, so calls that overlap on the
 *     GPU (other streams, other host threads) race: serialise them.
 *   - Device-detected errors (inconsistent cu_seqlens contents, whose
 *     sequences are skipped without any out-of-bounds access; an expired
 *     bounded wait) are recorded in the array's header: read them with
 *     gdn_noalloc_status after the call.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine. */
gdn_status gdn_chunk_fwd_noalloc(const gdn_dims *dims, const void *q, const void *k,
                                 const void *v, const float *log_alpha, const float *beta,
                                 const float *initial_state, const int32_t *cu_seqlens,
                                 void *o, float *final_state, gdn_stream_t stream);

/* Synchronise `stream`, then read and clear the error word of the array that
 * gdn_chunk_fwd_noalloc uses on the current device; the codes are those of
 * gdn_workspace_status.  Since every gdn_chunk_fwd_noalloc call clears the
 * word before its kernels run, this reports the errors of the last call on
 * the device.  The paper has no counterpart either. */
gdn_status gdn_noalloc_status(gdn_stream_t stream);

/* Zero the workspace header (the sticky error word) on `stream`. */
gdn_status gdn_workspace_init(void *workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Synchronise `stream`, read and clear the workspace's sticky error word.
 * GDN_OK if no device-side error was recorded since the last read;
 * GDN_ERR_TIMEOUT, GDN_ERR_DEVICE_INPUT, or GDN_ERR_CUDA (a kernel found no
 * ring slot for the SM it ran on) otherwise. */
gdn_status gdn_workspace_status(void *workspace, gdn_stream_t stream);

/* Name of the prefill kernel gdn_chunk_fwd selects for `dims` (static
 * storage): "tensor_core_pool" (pool tcgen05 kernel), "tensor_core_pair"
 * (two-CTA tcgen05 kernel), "tensor_core" (single-CTA tcgen05 kernel) or
 * "cuda_core" (fp32 CUDA cores); NULL for invalid dims. */
const char *gdn_chunk_fwd_path(const gdn_dims *dims);

/* Human-readable name of a status code (static storage). */
const char *gdn_status_string(gdn_status status);

/* Number of kernels this library has launched in this process (all calls,
 * all threads); used to count device work in benchmarks. */
uint64_t gdn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
