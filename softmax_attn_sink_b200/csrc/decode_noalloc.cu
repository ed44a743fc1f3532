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

#include <atomic>

#include "attn_sink.h"

namespace {

// Size of the fixed scratch array on every device that loads the library.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
// Last address looked up per device, for calls made while the stream is being captured.
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_decode_scratch in the current device's context, for a call on
// `stream`.  The array's name in host code is only a host-side stand-in for the symbol,
// never a device address, so the address comes from cudaGetSymbolAddress with the device
// current.  It is looked up afresh on every call made outside stream capture: the module
// holding the array is loaded per context, so after cudaDeviceReset (or in another context
// of the same device) the array may sit elsewhere, and a cached address would then point
// at memory this context does not own.  While `stream` is being captured no lookup is
// made (it could load a module in the middle of a capture); the address recorded by the
// device's last uncaptured call is used, and a capture that comes before any uncaptured
// call on the device is refused.  The per-device record is atomic, so first calls from
// several host threads at once do not race.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_SINK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_SINK_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return ATTN_SINK_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) {
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) return ATTN_SINK_ERR_CUDA;  // no uncaptured call on this device yet
    *out = p;
    return ATTN_SINK_OK;
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) return ATTN_SINK_ERR_CUDA;
  g_scratch_addr[dev].store(p, std::memory_order_release);
  *out = p;
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
    // the automatic count, or the largest count below it whose partials fit the fixed
    // array (the workspace size grows with the split count)
    if (attn_sink_decode_workspace_size(params, splits) > kNoAllocScratchBytes) {
      int lo = 1, hi = splits;  // invariant: hi does not fit; the answer is in [1, hi)
      while (hi - lo > 1) {
        const int mid = lo + (hi - lo) / 2;
        if (attn_sink_decode_workspace_size(params, mid) <= kNoAllocScratchBytes) lo = mid;
        else hi = mid;
      }
      splits = lo;
    }
  }
  const size_t need = attn_sink_decode_workspace_size(params, splits);
  if (need == SIZE_MAX) return ATTN_SINK_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return ATTN_SINK_ERR_WORKSPACE;  // beyond the fixed maximum
  void* scratch = nullptr;
  const int st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (st != ATTN_SINK_OK) return st;
  return attn_sink_decode(params, q, k, v, cu_seqlens_k, sink, splits, out, lse, scratch,
                          kNoAllocScratchBytes, stream);
}
