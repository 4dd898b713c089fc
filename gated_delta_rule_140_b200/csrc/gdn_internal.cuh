// gdn_internal.cuh -- definitions shared by the kernels of libgdn.so (not part
// of the public ABI, which is include/gdn.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// A named NVTX range over one C-ABI call (host side; a few instructions unless a
// profiler is attached), so that timelines show which entry point issued a launch.
struct ApiRange {
    explicit ApiRange(const char *name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange &) = delete;
    ApiRange &operator=(const ApiRange &) = delete;
};

constexpr int kChunk = 64;  // chunk size C of the chunkwise form

// Sticky error bits kept in the first word of the workspace.
enum : uint32_t { kErrBadSeqlens = 1u, kErrTimeout = 2u, kErrInternal = 4u };
constexpr size_t kWorkspaceHeader = 256;
// Bounded waits of the tensor-core kernels (SM clock cycles, ~1 s at 2 GHz).
// The second word of the workspace header, when nonzero, replaces this limit
// for the waits on data (tiles, products, hand-offs); the waits that drain a
// kernel's own copies and MMAs after an abort always use the default.
constexpr long long kDefaultWaitLimit = 1LL << 31;

// Everything a prefill kernel needs, in device pointers.  Token-major layouts
// (see gdn.h).  `seq_start` is null for fixed-length rows of T tokens.
struct PrefillArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    const float *s0;          // [N,H,dv,dk] or null
    const int32_t *cu_seqlens;  // [N+1] or null
    void *o;
    float *s_final;           // [N,H,dv,dk] or null
    uint32_t *err;            // sticky error word (workspace)
    void *scratch;            // workspace after the header
    int B, T, H, dk, dv, n_seqs;
    int channel;              // 1 = KDA channel-wise decay
    int bf16;                 // 1 = bf16 q/k/v/o, 0 = fp32
    // fused input prologue (pool kernel): q, k unnormalised, log_alpha and beta
    // hold the decay and writing-rate logits, alpha_bias [H] (or null) is added
    // to the decay logit
    int raw;
    const float *alpha_bias;
    // FG2-GDN (two-CTA kernel, channel decay): beta is [tokens, H, d_k], the
    // writing rate per key channel; keys are scaled by its square root and the
    // rate is 1 in the delta-rule step
    int beta_channel;
};

struct DecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *state;
    void *o;
    int N, H, dk, dv;
    int channel, bf16;
};

// Multi-token verification: K draft tokens per sequence, token-major [N, K, H].
constexpr int kMaxTreeNodes = 64;  // tree-shaped drafts per sequence (gdn_recurrent_verify_tree)

struct VerifyArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *state;
    const int32_t *n_commit;  // device [N] or null (no commit)
    const int32_t *parent;    // device [N, K] (tree-shaped drafts) or null (a chain)
    void *o;                  // [N, K, H, dv] or null (no outputs)
    int N, K, H, dk, dv;
    int channel, bf16;
};

// Host launchers (each returns cudaGetLastError() of its launches).
cudaError_t launch_verify(const VerifyArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_chunk_simt(const PrefillArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_chunk_pair(const PrefillArgs &a, cudaStream_t s, int *launches);
cudaError_t launch_chunk_pool(const PrefillArgs &a, cudaStream_t s, int *launches);
size_t chunk_pool_scratch_bytes(const gdn_dims &d);
// bf16 d_k = d_v = 128 scalar-decay shapes the pool kernel takes (fixed rows)
bool chunk_pool_supported(const gdn_dims &d);
bool chunk_pool_preferred(const gdn_dims &d);
size_t chunk_tc_scratch_bytes(const gdn_dims &d);
size_t chunk_pair_scratch_bytes(const gdn_dims &d);
// state maps of sequence segments (gdn_state.cu): out = s m (+ b), out = I
cudaError_t launch_state_compose(const float *s, const float *m, const float *b, float *out,
                                 long long nh, int dv, int dk, cudaStream_t st, int *launches);
cudaError_t launch_state_identity(float *out, long long nh, int d, cudaStream_t st, int *launches);
// FG2-GDN+ (gdn_state.cu): out = sqrt(beta_v) . v, bf16, n elements (a multiple of 8)
cudaError_t launch_value_rate(const void *v, const float *beta_v, void *out, long long n,
                              cudaStream_t st, int *launches);
// bf16 d_k = d_v = 128 shapes (either decay) the two-CTA kernel takes
bool chunk_pair_supported(const gdn_dims &d);
// bf16 d_k = d_v = 128 scalar-decay shapes the tensor-core kernels take
bool chunk_tc_supported(const gdn_dims &d);
// [tokens, H, d] bf16 as a 3-D TMA tensor map (d, H, tokens), box 64 x 1 x 64,
// 128-byte swizzle (defined with the single-CTA tensor-core kernel).
bool make_tile_map(CUtensorMap *m, const void *base, int d, int H, long long ntok);
// [tokens, H, 128] bf16 as a 4-D tensor map (64, tokens, 2, H), box 64 x 64 x 2 x 1:
// both 64-wide halves of a 64-token tile in one load, two consecutive 8 KB tiles.
bool make_halves_map(CUtensorMap *m, const void *base, int H, long long ntok);

__device__ __forceinline__ long long data_wait_limit(const uint32_t *hdr) {
    const uint32_t w = hdr[1];
    return w ? (long long)w : kDefaultWaitLimit;
}

// Token range of sequence n for fixed rows or packed sequences, validated on
// the device: a bad range records kErrBadSeqlens and yields an empty range.
__device__ __forceinline__ void seq_range(const PrefillArgs &a, int n, long long *t0,
                                          long long *t1) {
    if (a.cu_seqlens == nullptr) {
        *t0 = (long long)n * a.T;
        *t1 = *t0 + a.T;
        return;
    }
    long long s = a.cu_seqlens[n], e = a.cu_seqlens[n + 1];
    if (s < 0 || e < s || e > (long long)a.T || (n == 0 && s != 0)) {
        atomicOr(a.err, kErrBadSeqlens);
        s = e = 0;
    }
    *t0 = s;
    *t1 = e;
}

__device__ __forceinline__ float load_elem(const void *p, long long i, int bf16) {
    return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i])
                : reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void store_elem(void *p, long long i, float x, int bf16) {
    if (bf16)
        reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<float *>(p)[i] = x;
}

}  // namespace gdn
