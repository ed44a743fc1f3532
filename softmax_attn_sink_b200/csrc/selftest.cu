// Diagnostics: exercise the bounded-wait path of the tensor-core kernels on purpose.
//
// One thread initialises an mbarrier that expects one arrival and then waits for its first
// phase, which nothing ever completes.  The wait is the same bounded helper the kernels use
// (a 2 s limit on the global timer, plus a poll-count limit), so it gives up, records the
// timeout bit in the per-device status word and the kernel returns normally.  The GPU
// context stays usable; attn_sink_get_device_status() then reports ATTN_SINK_ERR_TIMEOUT.
#include "attn_sink.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

__global__ void wait_timeout_kernel(unsigned* status) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = sm100::smem_addr(&bar);
  sm100::mbar_init(b, 1);
  sm100::fence_mbar_init();
  (void)sm100::mbar_wait(b, 0, status);   // no arrival will ever come
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* status, cudaStream_t s) {
  wait_timeout_kernel<<<1, 1, 0, s>>>(status);
  return cudaGetLastError();
}

}  // namespace attn_sink
