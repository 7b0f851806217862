// chunk_fwd_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) chunk forward for bf16.
#include "common.cuh"

namespace gdn {

bool chunk_fwd_tc_supported(int, int, int) { return false; }

cudaError_t launch_chunk_fwd_tc(const ChunkParams&, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdn
