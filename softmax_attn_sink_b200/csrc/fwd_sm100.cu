// Tensor-core (tcgen05) sink-attention forward for sm_100a.
#include "common.cuh"

namespace attn_sink {

bool fwd_sm100_supported(const FwdArgs&, int) { return false; }
cudaError_t launch_fwd_sm100(const FwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace attn_sink
