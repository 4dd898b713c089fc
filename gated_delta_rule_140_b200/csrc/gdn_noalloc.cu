// gdn_noalloc.cu -- gdn_chunk_fwd_noalloc: the chunkwise prefill for callers
// that cannot allocate device memory (see include/gdn.h).  The workspace the
// prefill kernels need is a fixed array compiled into the library instead of a
// caller buffer; nothing here allocates.
#include <mutex>

#include "gdn_internal.cuh"

// The scratch array.  In host code this name is only a host-side stand-in for
// the symbol: its device address comes from cudaGetSymbolAddress below and is
// what the kernels receive.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device (the first call on a device does it, with that device current).
cudaError_t scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_noalloc(const gdn_dims *dims, const void *q, const void *k,
                                            const void *v, const float *log_alpha,
                                            const float *beta, const float *initial_state,
                                            const int32_t *cu_seqlens, void *o,
                                            float *final_state, gdn_stream_t stream) {
    gdn::ApiRange range("gdn_chunk_fwd_noalloc");
    size_t need = gdn_chunk_fwd_workspace_size(dims);
    if (need == 0) return GDN_ERR_INVALID;
    gdn_dims d = *dims;
    if (need > GDN_NOALLOC_SCRATCH_BYTES) {
        // the two-CTA kernel's ring does not fit: GDN runs the single-CTA
        // tensor-core kernel, KDA the CUDA-core kernel
        d.flags &= ~(GDN_FLAG_PAIR | GDN_FLAG_POOL);
        d.flags |= d.decay == GDN_DECAY_CHANNEL ? GDN_FLAG_CUDA_CORES : GDN_FLAG_ONE_CTA;
        need = gdn_chunk_fwd_workspace_size(&d);
    }
    if (need > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess) return GDN_ERR_CUDA;
    // The array keeps the previous call's contents: clear the header (the
    // error word), which the kernels expect to start at zero.
    if (cudaMemsetAsync(scratch, 0, gdn::kWorkspaceHeader,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDN_ERR_CUDA;
    return gdn_chunk_fwd(&d, q, k, v, log_alpha, beta, initial_state, cu_seqlens, o,
                         final_state, scratch, GDN_NOALLOC_SCRATCH_BYTES, stream);
}

// The error word of the array's header on the current device, read and
// cleared like a caller workspace's (gdn_workspace_status).
extern "C" gdn_status gdn_noalloc_status(gdn_stream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_workspace_status(scratch, stream);
}
