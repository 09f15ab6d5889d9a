// Tensor-core (tcgen05) lightning-indexer kernel: not yet enabled.
#include "internal.h"

namespace dsa {
cudaError_t launch_indexer_tc(const IndexerProblem &, cudaStream_t, bool *taken) {
    *taken = false;
    return cudaSuccess;
}
}  // namespace dsa
