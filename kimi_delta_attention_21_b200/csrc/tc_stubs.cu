// Tensor-core engines not yet wired in this build: report "unsupported" so the
// dispatcher takes the SIMT kernels.
#include "kda_internal.cuh"

namespace kda {

bool chunk_tc_supported(const kda_chunk_args &, int) { return false; }
bool chunk_tc_aligned(const kda_chunk_args &) { return false; }
size_t chunk_tc_workspace(const kda_chunk_args &) { return 0; }
kda_status_t launch_chunk_tc(const kda_chunk_args &, cudaStream_t) {
    return fail(KDA_ERR_UNSUPPORTED, "tensor-core chunk engine not built");
}

}  // namespace kda
