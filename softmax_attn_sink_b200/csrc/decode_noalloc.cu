// Split-KV decode for callers that cannot allocate device memory.
//
// attn_sink_decode needs a workspace for its per-chunk partials (max, sum and the
// unnormalised output of every key chunk).  Some callers have no way to provide one:
// a plugin or custom-op host that hands the library only the tensors of the call and
// exposes no allocator, a process whose device memory is entirely reserved by another
// framework's pool, or a latency-critical loop where an allocation (and the
// synchronisation cudaMalloc can imply) is not acceptable.  For them this file keeps the
// partials in a fixed, file-scope device array that is part of the library image: it is
// created when the library's module is loaded on a device and stays there, on every
// device that loads the library, until the process exits.  Nothing here calls
// cudaMalloc, cudaFree or any other allocating routine.
//
// The entry point runs exactly the kernels attn_sink_decode runs (split + merge), with
// its workspace pointed at that array.  Every call shares the array, so two calls whose
// kernels overlap on the GPU (different streams without ordering, or different host
// threads) race on the partials and produce wrong results; calls in one stream are
// ordered and safe.  No part of the array needs to start at zero: the split kernel
// writes every (sequence, head, chunk) slot that the merge kernel then reads, so the
// previous call's leftovers are never read.
#include <stdint.h>

#include "attn_sink.h"

namespace {

// Size of the fixed scratch array on every device that loads the library.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];

// Device address of g_decode_scratch on the current device.  The array's name in host
// code is only a host-side stand-in for the symbol, never a device address, so the
// address is looked up once per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_SINK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_SINK_ERR_UNSUPPORTED;
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return ATTN_SINK_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ATTN_SINK_OK;
}

}  // namespace

extern "C" int attn_sink_decode_noalloc(const attn_sink_params* params, const void* q,
                                        const void* k, const void* v,
                                        const int32_t* cu_seqlens_k, const float* sink,
                                        int num_splits, void* out, float* lse,
                                        attn_sink_stream_t stream) {
  if (num_splits < 0) return ATTN_SINK_ERR_INVALID_ARG;
  int splits = num_splits;
  if (splits == 0) {
    splits = attn_sink_decode_num_splits(params);
    if (splits < 0) return ATTN_SINK_ERR_INVALID_ARG;  // params rejected
    // shrink the automatic split count until the partials fit the fixed array
    while (splits > 1 && attn_sink_decode_workspace_size(params, splits) > kNoAllocScratchBytes) {
      const size_t need = attn_sink_decode_workspace_size(params, splits);
      int next = (int)((double)splits * (double)kNoAllocScratchBytes / (double)need);
      splits = next < splits ? (next > 0 ? next : 1) : splits - 1;
    }
  }
  const size_t need = attn_sink_decode_workspace_size(params, splits);
  if (need == SIZE_MAX) return ATTN_SINK_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return ATTN_SINK_ERR_WORKSPACE;  // beyond the fixed maximum
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != ATTN_SINK_OK) return st;
  return attn_sink_decode(params, q, k, v, cu_seqlens_k, sink, splits, out, lse, scratch,
                          kNoAllocScratchBytes, stream);
}
