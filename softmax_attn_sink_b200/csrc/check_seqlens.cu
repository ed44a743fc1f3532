// Device-side check of the cu_seqlens contract: start at 0, never decrease, end at the
// total row count, and no sequence longer than the max_seqlen the caller announced (CANN
// ops-transformer flash_attn doc, "SeqLengths Parameter Group" and the max_seqlen rows of
// its parameter table).  The arrays live on the device, so the host cannot check them
// without a synchronisation; this kernel reads them and sets a bit in the status word.
#include "common.cuh"

namespace attn_sink {
namespace {

__device__ __forceinline__ bool cu_ok(const int32_t* cu, int batch, int total, int max_len, int b) {
  // entry b and the length of sequence b (entries 0 .. batch)
  if (b == 0 && cu[0] != 0) return false;
  if (b == batch) return cu[batch] == total;
  const long long len = (long long)cu[b + 1] - cu[b];
  return len >= 0 && len <= max_len;
}

__global__ void __launch_bounds__(256) check_seqlens_kernel(const int32_t* cu_q, const int32_t* cu_k, int batch,
                                                           int total_q, int total_k, int max_sq, int max_sk,
                                                           unsigned* status) {
  bool ok = true;
  for (int b = threadIdx.x; b <= batch; b += blockDim.x) {
    if (cu_q) ok = ok && cu_ok(cu_q, batch, total_q, max_sq, b);
    ok = ok && cu_ok(cu_k, batch, total_k, max_sk, b);
  }
  if (!__syncthreads_and(ok) && threadIdx.x == 0) set_status(status, kStatusBadSeqlens);
}

}  // namespace

cudaError_t launch_check_seqlens(const int32_t* cu_q, const int32_t* cu_k, int batch, int total_q, int total_k,
                                 int max_sq, int max_sk, unsigned* status, cudaStream_t s) {
  check_seqlens_kernel<<<1, 256, 0, s>>>(cu_q, cu_k, batch, total_q, total_k, max_sq, max_sk, status);
  return cudaGetLastError();
}

}  // namespace attn_sink
