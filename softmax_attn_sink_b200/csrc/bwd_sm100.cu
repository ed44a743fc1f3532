// Tensor-core (tcgen05) sink-attention backward for sm_100a.
#include "common.cuh"

namespace attn_sink {

bool bwd_sm100_supported(const BwdArgs&, int) { return false; }
cudaError_t launch_bwd_sm100(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace attn_sink
