// tcgen05 / TMEM lightning-indexer scorer (filled in by the tensor-core path).
#include "kernels.cuh"

namespace lidx {

bool score_tc_supported(const lidx_score_args &) { return false; }

cudaError_t launch_score_tc(const lidx_score_args &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace lidx
