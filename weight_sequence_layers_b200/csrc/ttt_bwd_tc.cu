// tcgen05 backward of the chunkwise TTT layer (bf16 storage, fp32 state).
#include "common.cuh"
#include "kernels.h"

namespace tttk {
bool tc_bwd_supported(const LayerArgs&) { return false; }
size_t tc_bwd_workspace(const LayerArgs&) { return 0; }
cudaError_t tc_bwd(const LayerArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace tttk
