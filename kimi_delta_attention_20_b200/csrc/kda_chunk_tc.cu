// Tensor-core (tcgen05) chunkwise forward for bf16 inputs. Not built yet:
// every request falls to the fp32 CUDA-core kernel.
#include "kda_common.cuh"

namespace kda {

bool chunk_tc_supported(bool, int, int, int) { return false; }

size_t chunk_tc_workspace_bytes(int, int, int, int) { return 0; }

cudaError_t launch_chunk_tc(const ChunkParams &, int, int, void *, size_t, const int32_t *,
                            cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace kda
