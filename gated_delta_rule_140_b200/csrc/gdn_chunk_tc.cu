// gdn_chunk_tc.cu -- tensor-core (tcgen05) chunkwise prefill for bf16,
// d_k = d_v = 128.  Not yet enabled: the library selects the fp32 CUDA-core
// kernel for every shape until this path passes its parity tests.
#include "gdn_internal.cuh"

namespace gdn {

bool chunk_tc_supported(const gdn_dims &) { return false; }

size_t chunk_tc_scratch_bytes(const gdn_dims &) { return 0; }

cudaError_t launch_chunk_tc(const PrefillArgs &, cudaStream_t, int *) {
    return cudaErrorNotSupported;
}

}  // namespace gdn
