// gdn_api.cu -- the extern "C" entry points of libgdn.so (declared in
// include/gdn.h): host-side argument validation, workspace bookkeeping and
// kernel selection.  Every step of the computation runs in the kernels of the
// other translation units; this file only checks and launches.
#include <atomic>

#include "gdn_internal.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host validation of the dims shared by both calls.
gdn_status check_dims(const gdn_dims *d, bool prefill) {
    if (!d) return GDN_ERR_INVALID;
    if (d->B < 0 || d->H <= 0 || d->T < 0) return GDN_ERR_INVALID;
    if (d->dtype != GDN_BF16 && d->dtype != GDN_FP32) return GDN_ERR_INVALID;
    if (d->decay != GDN_DECAY_SCALAR && d->decay != GDN_DECAY_CHANNEL) return GDN_ERR_INVALID;
    if (d->d_k <= 0 || d->d_v <= 0) return GDN_ERR_INVALID;
    if ((d->d_k != 64 && d->d_k != 128) || (d->d_v != 64 && d->d_v != 128))
        return GDN_ERR_UNSUPPORTED;
    if ((d->flags & ~(GDN_FLAG_CUDA_CORES | GDN_FLAG_PAIR | GDN_FLAG_ONE_CTA | GDN_FLAG_POOL |
                      GDN_FLAG_BETA_CHANNEL | GDN_FLAG_VALUE_RATE)) != 0)
        return GDN_ERR_INVALID;
    // FG2-GDN+: the value-side rate comes with the key-side one
    if ((d->flags & GDN_FLAG_VALUE_RATE) && !(d->flags & GDN_FLAG_BETA_CHANNEL))
        return GDN_ERR_INVALID;
    if (d->flags & GDN_FLAG_BETA_CHANNEL) {
        // FG2-GDN: a writing rate per key channel rides on KDA's decay, prefill only,
        // on the two-CTA tensor-core kernel
        if (d->decay != GDN_DECAY_CHANNEL || (d->flags & (GDN_FLAG_ONE_CTA | GDN_FLAG_POOL)))
            return GDN_ERR_INVALID;
        if (!prefill || (d->flags & GDN_FLAG_CUDA_CORES) || !gdn::chunk_pair_supported(*d))
            return GDN_ERR_UNSUPPORTED;
    }
    const int kernel_flags = d->flags & (GDN_FLAG_PAIR | GDN_FLAG_ONE_CTA | GDN_FLAG_POOL);
    if (kernel_flags & (kernel_flags - 1)) return GDN_ERR_INVALID;  // at most one
    if ((d->flags & (GDN_FLAG_ONE_CTA | GDN_FLAG_POOL)) && d->decay == GDN_DECAY_CHANNEL)
        return GDN_ERR_INVALID;
    if (prefill && d->n_seqs < 0) return GDN_ERR_INVALID;
    // every index the kernels form must fit in 63 bits; keep the token axis sane
    if ((long long)d->B * d->T * d->H * (d->d_k > d->d_v ? d->d_k : d->d_v) > (1LL << 40))
        return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

enum class Path { kPool, kPair, kOneCta, kCudaCores };

// The prefill kernel a call runs.  bf16, d_k = d_v = 128: KDA (and FG2-GDN) the
// two-CTA kernel; GDN the pool kernel for few long sequences, else the two-CTA
// kernel from 2048 tokens per sequence on average and the single-CTA kernel below
// (the flags choose one); every other case, or GDN_FLAG_CUDA_CORES, the fp32
// CUDA-core kernel.
constexpr long long kPairMinMeanTokens = 2048;

Path select_path(const gdn_dims &d) {
    if ((d.flags & GDN_FLAG_CUDA_CORES) || !gdn::chunk_pair_supported(d)) return Path::kCudaCores;
    if (d.decay == GDN_DECAY_CHANNEL || (d.flags & GDN_FLAG_PAIR)) return Path::kPair;
    if (!gdn::chunk_tc_supported(d)) return Path::kCudaCores;
    if (d.flags & GDN_FLAG_ONE_CTA) return Path::kOneCta;
    if ((d.flags & GDN_FLAG_POOL) && gdn::chunk_pool_supported(d))
        return Path::kPool;
    if (gdn::chunk_pool_preferred(d)) return Path::kPool;
    // scalar decay: the two-CTA kernel's steady state is faster per chunk, its
    // start-up (the first chunk through both SMs) longer; measured, it is ahead
    // from sequences of about 32 chunks on (16 chunks: 3% behind; 64: 3% ahead;
    // 128: 10% ahead)
    const long long seqs = d.n_seqs > 0 ? d.n_seqs : (d.B > 0 ? d.B : 1);
    return (long long)d.B * d.T >= kPairMinMeanTokens * seqs ? Path::kPair : Path::kOneCta;
}

// the selected prefill kernel's scratch after the header (256-byte multiple)
size_t kernel_scratch_bytes(const gdn_dims &d) {
    const Path p = select_path(d);
    const size_t extra = p == Path::kPool     ? gdn::chunk_pool_scratch_bytes(d)
                         : p == Path::kPair   ? gdn::chunk_pair_scratch_bytes(d)
                         : p == Path::kOneCta ? gdn::chunk_tc_scratch_bytes(d)
                                              : 0;
    return (extra + 255) & ~size_t(255);
}

// FG2-GDN+: v~ (bf16, the layout of v) after the kernel scratch
size_t value_rate_bytes(const gdn_dims &d) {
    if (!(d.flags & GDN_FLAG_VALUE_RATE)) return 0;
    return ((size_t)d.B * d.T * d.H * d.d_v * 2 + 255) & ~size_t(255);
}

int prefill_seqs(const gdn_dims &d, const int32_t *cu_seqlens) {
    return cu_seqlens ? d.n_seqs : d.B;
}

}  // namespace

extern "C" {

size_t gdn_chunk_fwd_workspace_size(const gdn_dims *dims) {
    if (check_dims(dims, true) != GDN_OK) return 0;
    return gdn::kWorkspaceHeader + kernel_scratch_bytes(*dims) + value_rate_bytes(*dims);
}

}  // extern "C"

namespace {

// The prefill entry points: validate on the host, fill the device arguments,
// launch the selected kernel.  raw = 1: the fused input prologue (pool kernel).
gdn_status chunk_fwd_impl(const gdn_dims *dims, const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta, const float *alpha_bias,
                          int raw, const float *initial_state, const int32_t *cu_seqlens,
                          void *o, float *final_state, void *workspace, size_t workspace_bytes,
                          gdn_stream_t stream) {
    gdn_status st = check_dims(dims, true);
    if (st != GDN_OK) return st;
    const gdn_dims &d = *dims;
    if (cu_seqlens) {
        if (d.B != 1 || d.n_seqs < 1) return GDN_ERR_INVALID;
    } else if (d.n_seqs != 0 && d.n_seqs != d.B) {
        return GDN_ERR_INVALID;
    }
    const int n_seqs = prefill_seqs(d, cu_seqlens);
    const bool any_tokens = (long long)d.B * d.T > 0;
    if (any_tokens && (!q || !k || !v || !log_alpha || !beta || !o)) return GDN_ERR_INVALID;
    if (!workspace || workspace_bytes < gdn_chunk_fwd_workspace_size(dims)) return GDN_ERR_INVALID;
    for (const void *p : {q, k, v, (const void *)o, (const void *)initial_state,
                          (const void *)final_state, (const void *)workspace})
        if (p && !aligned16(p)) return GDN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(log_alpha) | reinterpret_cast<uintptr_t>(beta) |
         reinterpret_cast<uintptr_t>(alpha_bias) | reinterpret_cast<uintptr_t>(cu_seqlens)) & 3u)
        return GDN_ERR_INVALID;
    const Path p = select_path(d);
    if (raw && p != Path::kPool) return GDN_ERR_UNSUPPORTED;

    gdn::PrefillArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.log_alpha = log_alpha; a.beta = beta;
    a.s0 = initial_state; a.cu_seqlens = cu_seqlens;
    a.o = o; a.s_final = final_state;
    a.err = reinterpret_cast<uint32_t *>(workspace);
    a.scratch = reinterpret_cast<char *>(workspace) + gdn::kWorkspaceHeader;
    a.B = d.B; a.T = d.T; a.H = d.H; a.dk = d.d_k; a.dv = d.d_v; a.n_seqs = n_seqs;
    a.channel = d.decay == GDN_DECAY_CHANNEL;
    a.bf16 = d.dtype == GDN_BF16;
    a.raw = raw;
    a.beta_channel = (d.flags & GDN_FLAG_BETA_CHANNEL) != 0;
    a.alpha_bias = alpha_bias;

    // Nothing to compute and nothing to write: an empty batch is a no-op.
    if (n_seqs == 0) return GDN_OK;
    int launches = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = p == Path::kPool     ? gdn::launch_chunk_pool(a, s, &launches)
                    : p == Path::kPair   ? gdn::launch_chunk_pair(a, s, &launches)
                    : p == Path::kOneCta ? gdn::launch_chunk_tc(a, s, &launches)
                                         : gdn::launch_chunk_simt(a, s, &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

gdn_status gdn_chunk_fwd(const gdn_dims *dims, const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         const float *initial_state, const int32_t *cu_seqlens,
                         void *o, float *final_state,
                         void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_chunk_fwd");
    if (dims && (dims->flags & GDN_FLAG_VALUE_RATE)) return GDN_ERR_INVALID;
    return chunk_fwd_impl(dims, q, k, v, log_alpha, beta, nullptr, 0, initial_state, cu_seqlens,
                          o, final_state, workspace, workspace_bytes, stream);
}

gdn_status gdn_chunk_fwd_value_rate(const gdn_dims *dims, const void *q, const void *k,
                                    const void *v, const float *log_alpha, const float *beta,
                                    const float *beta_v, const float *initial_state,
                                    const int32_t *cu_seqlens, void *o, float *final_state,
                                    void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_chunk_fwd_value_rate");
    if (!dims) return GDN_ERR_INVALID;
    const int both = GDN_FLAG_BETA_CHANNEL | GDN_FLAG_VALUE_RATE;
    if ((dims->flags & both) != both) return GDN_ERR_INVALID;
    gdn_status st = check_dims(dims, true);
    if (st != GDN_OK) return st;
    const long long n = (long long)dims->B * dims->T * dims->H * dims->d_v;
    if (n > 0 && (!v || !beta_v || !aligned16(v) || !aligned16(beta_v))) return GDN_ERR_INVALID;
    if (!workspace || !aligned16(workspace) || workspace_bytes < gdn_chunk_fwd_workspace_size(dims))
        return GDN_ERR_INVALID;
    void *vt = reinterpret_cast<char *>(workspace) + gdn::kWorkspaceHeader + kernel_scratch_bytes(*dims);
    int launches = 0;
    cudaError_t e = gdn::launch_value_rate(v, beta_v, vt, n, reinterpret_cast<cudaStream_t>(stream),
                                           &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    return chunk_fwd_impl(dims, q, k, vt, log_alpha, beta, nullptr, 0, initial_state, cu_seqlens,
                          o, final_state, workspace, workspace_bytes, stream);
}

gdn_status gdn_chunk_fwd_raw(const gdn_dims *dims, const void *q_raw, const void *k_raw,
                             const void *v, const float *alpha_logit, const float *alpha_bias,
                             const float *beta_logit, const float *initial_state,
                             const int32_t *cu_seqlens, void *o, float *final_state,
                             void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_chunk_fwd_raw");
    if (!dims) return GDN_ERR_INVALID;
    if (dims->decay != GDN_DECAY_SCALAR || (dims->flags & ~GDN_FLAG_POOL) != 0)
        return dims->decay == GDN_DECAY_CHANNEL ? GDN_ERR_UNSUPPORTED : GDN_ERR_INVALID;
    gdn_dims d = *dims;
    d.flags = GDN_FLAG_POOL;
    return chunk_fwd_impl(&d, q_raw, k_raw, v, alpha_logit, beta_logit, alpha_bias, 1,
                          initial_state, cu_seqlens, o, final_state, workspace, workspace_bytes,
                          stream);
}

gdn_status gdn_recurrent_step(const gdn_dims *dims, const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              float *state_inout, void *o, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_recurrent_step");
    gdn_status st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    const gdn_dims &d = *dims;
    if (d.B == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !state_inout || !o) return GDN_ERR_INVALID;
    // 16-byte state rows; 8-byte (bf16 x4) or 16-byte (fp32 x4) token vectors
    if (!aligned16(state_inout)) return GDN_ERR_INVALID;
    for (const void *p : {q, k, v, (const void *)o})
        if (reinterpret_cast<uintptr_t>(p) & (d.dtype == GDN_BF16 ? 7u : 15u)) return GDN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(log_alpha) | reinterpret_cast<uintptr_t>(beta)) & 3u)
        return GDN_ERR_INVALID;
    gdn::DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.state = state_inout; a.o = o;
    a.N = d.B; a.H = d.H; a.dk = d.d_k; a.dv = d.d_v;
    a.channel = d.decay == GDN_DECAY_CHANNEL;
    a.bf16 = d.dtype == GDN_BF16;
    int launches = 0;
    cudaError_t e = gdn::launch_decode(a, reinterpret_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

namespace {
gdn_status verify_impl(const gdn_dims *dims, const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta, float *state_inout,
                       const int32_t *parent, const int32_t *n_commit, void *o,
                       gdn_stream_t stream);
}  // namespace

gdn_status gdn_recurrent_verify(const gdn_dims *dims, const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta, float *state_inout,
                                const int32_t *n_commit, void *o, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_recurrent_verify");
    return verify_impl(dims, q, k, v, log_alpha, beta, state_inout, nullptr, n_commit, o, stream);
}

gdn_status gdn_recurrent_verify_tree(const gdn_dims *dims, const void *q, const void *k,
                                     const void *v, const float *log_alpha, const float *beta,
                                     float *state_inout, const int32_t *parent,
                                     const int32_t *n_commit, void *o, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_recurrent_verify_tree");
    if (!dims) return GDN_ERR_INVALID;
    if (dims->T > gdn::kMaxTreeNodes) return GDN_ERR_UNSUPPORTED;
    if ((long long)dims->B * dims->T > 0 && (!parent || (reinterpret_cast<uintptr_t>(parent) & 3u)))
        return GDN_ERR_INVALID;
    return verify_impl(dims, q, k, v, log_alpha, beta, state_inout, parent, n_commit, o, stream);
}

}  // extern "C"

namespace {
gdn_status verify_impl(const gdn_dims *dims, const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta, float *state_inout,
                       const int32_t *parent, const int32_t *n_commit, void *o,
                       gdn_stream_t stream) {
    gdn_status st = check_dims(dims, false);
    if (st != GDN_OK) return st;
    const gdn_dims &d = *dims;
    if (d.B == 0 || d.T == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !state_inout) return GDN_ERR_INVALID;
    if (!aligned16(state_inout)) return GDN_ERR_INVALID;
    for (const void *p : {q, k, (const void *)o})
        if (p && (reinterpret_cast<uintptr_t>(p) & (d.dtype == GDN_BF16 ? 7u : 15u))) return GDN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(log_alpha) |
         reinterpret_cast<uintptr_t>(beta) | reinterpret_cast<uintptr_t>(n_commit)) & 3u)
        return GDN_ERR_INVALID;
    gdn::VerifyArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.state = state_inout; a.n_commit = n_commit; a.o = o; a.parent = parent;
    a.N = d.B; a.K = d.T; a.H = d.H; a.dk = d.d_k; a.dv = d.d_v;
    a.channel = d.decay == GDN_DECAY_CHANNEL;
    a.bf16 = d.dtype == GDN_BF16;
    int launches = 0;
    cudaError_t e = gdn::launch_verify(a, reinterpret_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
}  // namespace

extern "C" {

gdn_status gdn_state_compose(const gdn_dims *dims, const float *s, const float *m, const float *b,
                             float *out, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_state_compose");
    if (!dims || dims->B < 0 || dims->H <= 0) return GDN_ERR_INVALID;
    const int dk = dims->d_k, dv = dims->d_v;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GDN_ERR_UNSUPPORTED;
    if (dims->B == 0) return GDN_OK;
    if (!s || !m || !out) return GDN_ERR_INVALID;
    for (const void *p : {(const void *)s, (const void *)m, (const void *)out})
        if (!aligned16(p)) return GDN_ERR_INVALID;
    if (b && !aligned16(b)) return GDN_ERR_INVALID;
    if (out == s || out == m) return GDN_ERR_INVALID;
    int launches = 0;
    cudaError_t e = gdn::launch_state_compose(s, m, b, out, (long long)dims->B * dims->H, dv, dk,
                                              reinterpret_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_state_identity(const gdn_dims *dims, float *out, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_state_identity");
    if (!dims || dims->B < 0 || dims->H <= 0) return GDN_ERR_INVALID;
    if (dims->d_k != dims->d_v || (dims->d_k != 64 && dims->d_k != 128)) return GDN_ERR_UNSUPPORTED;
    if (dims->B == 0) return GDN_OK;
    if (!out || !aligned16(out)) return GDN_ERR_INVALID;
    int launches = 0;
    cudaError_t e = gdn::launch_state_identity(out, (long long)dims->B * dims->H, dims->d_k,
                                               reinterpret_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_workspace_init(void *workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (!workspace || workspace_bytes < gdn::kWorkspaceHeader || !aligned16(workspace))
        return GDN_ERR_INVALID;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kWorkspaceHeader,
                                    reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_workspace_status(void *workspace, gdn_stream_t stream) {
    if (!workspace || !aligned16(workspace)) return GDN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (word == 0) return GDN_OK;
    if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (word & gdn::kErrInternal) return GDN_ERR_CUDA;
    return (word & gdn::kErrTimeout) ? GDN_ERR_TIMEOUT : GDN_ERR_DEVICE_INPUT;
}

const char *gdn_chunk_fwd_path(const gdn_dims *dims) {
    if (check_dims(dims, true) != GDN_OK) return nullptr;
    switch (select_path(*dims)) {
        case Path::kPool: return "tensor_core_pool";
        case Path::kPair: return "tensor_core_pair";
        case Path::kOneCta: return "tensor_core";
        default: return "cuda_core";
    }
}

const char *gdn_status_string(gdn_status status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID: return "GDN_ERR_INVALID: invalid argument";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: unsupported shape or dtype";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA runtime or launch failure";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a device-side bounded wait expired";
        case GDN_ERR_DEVICE_INPUT: return "GDN_ERR_DEVICE_INPUT: bad cu_seqlens contents";
    }
    return "unknown gdn_status";
}

uint64_t gdn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
