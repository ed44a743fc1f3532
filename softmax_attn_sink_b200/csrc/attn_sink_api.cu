// Host side of the C ABI declared in include/attn_sink.h: argument validation, workspace
// layout, kernel dispatch and the per-device status word.  No allocation, no
// synchronisation (except attn_sink_get_device_status, which exists to synchronise).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "attn_sink.h"
#include "launch.h"

using namespace attn_sink;

namespace {

// Bits set by kernels: a bounded wait ran out (kStatusTimeout), an index or length outside
// its table was skipped (kStatusBadIndex), cu_seqlens broke their contract
// (kStatusBadSeqlens), a debug build skipped a store outside its output (kStatusDebugBounds).
__device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;
unsigned* g_status_ptr[kMaxDevices];

unsigned* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// (dk, dv): 64 or 128 with 32, 64 or 128; and 256 with 256 (the CANN flash_attn doc lists
// head dims 64, 128 and 256)
// Forward workspace: one counter word of the persistent kernel's work queue, padded to 256
// bytes.
constexpr size_t kFwdWorkspaceBytes = 256;

bool dims_supported(int dk, int dv) {
  return ((dk == 64 || dk == 128) && (dv == 32 || dv == 64 || dv == 128)) || (dk == 256 && dv == 256);
}

int validate_params(const attn_sink_params* p, bool decode) {
  if (!p) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->dtype != ATTN_SINK_BF16 && p->dtype != ATTN_SINK_FP32 && p->dtype != ATTN_SINK_FP16)
    return ATTN_SINK_ERR_UNSUPPORTED;
  if (p->batch <= 0 || p->total_q <= 0 || p->total_k <= 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->num_heads_q <= 0 || p->num_heads_kv <= 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->num_heads_q % p->num_heads_kv != 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->max_seqlen_q < 1 || p->max_seqlen_k < 1) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->max_seqlen_q > p->total_q || p->max_seqlen_k > p->total_k) return ATTN_SINK_ERR_INVALID_ARG;
  if (p->window_left < -1 || p->window_right < -1) return ATTN_SINK_ERR_INVALID_ARG;
  if (!isfinite(p->softmax_scale)) return ATTN_SINK_ERR_INVALID_ARG;
  if (!dims_supported(p->head_dim_qk, p->head_dim_v)) return ATTN_SINK_ERR_UNSUPPORTED;
  if (decode && (p->total_q != p->batch || p->max_seqlen_q != 1)) return ATTN_SINK_ERR_INVALID_ARG;
  return ATTN_SINK_OK;
}

void effective_window(const attn_sink_params* p, int& left, int& right) {
  left = p->window_left < 0 ? kUnbounded : p->window_left;
  right = p->window_right < 0 ? kUnbounded : p->window_right;
  if (p->causal && right > 0) right = 0;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? ATTN_SINK_OK : ATTN_SINK_ERR_CUDA; }

// workspace layout of the backward: D, lse_tot, the preprocess blocks' d_sink partials
// ([hq][ceil(total_q / 64)]), then the fp32 dQ accumulator of the tensor-core path
struct BwdLayout {
  size_t D, lse_tot, dsink_part, dq_acc, total;
};
BwdLayout bwd_layout(const attn_sink_params* p) {
  BwdLayout l{};
  const size_t rows = (size_t)p->num_heads_q * p->total_q;
  const size_t parts = (size_t)p->num_heads_q * ((p->total_q + 63) / 64);
  l.D = 0;
  l.lse_tot = align_up(l.D + rows * 4, 256);
  l.dsink_part = align_up(l.lse_tot + rows * 4, 256);
  l.dq_acc = align_up(l.dsink_part + parts * 4, 256);
  size_t end = l.dq_acc;
  if (p->dtype != ATTN_SINK_FP32) end += (size_t)p->total_q * p->num_heads_q * p->head_dim_qk * 4;
  l.total = align_up(end, 256);
  return l;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int decode_auto_splits(const attn_sink_params* p) {
  const int group = p->num_heads_q / p->num_heads_kv;
  const long long units = (long long)p->num_heads_kv * ((group + 15) / 16);
  const long long target = 4LL * sm_count();
  long long chunk = (long long)p->total_k * units / target;
  if (chunk < 256) chunk = 256;
  if (chunk > 2048) chunk = 2048;
  chunk = (chunk + 63) / 64 * 64;
  long long splits = (p->max_seqlen_k + chunk - 1) / chunk;
  if (splits < 1) splits = 1;
  if (splits > 1024) splits = 1024;
  return (int)splits;
}

size_t decode_ws(const attn_sink_params* p, int splits) {
  if (p->dtype == ATTN_SINK_FP32) return 0;
  const size_t rows = (size_t)p->batch * p->num_heads_q * splits;
  return align_up(rows * p->head_dim_v * 4, 256) + align_up(rows * 2 * 4, 256);
}

// Split + merge launch shared by the packed and paged decode entry points: workspace check,
// partial-buffer layout and the remaining DecodeArgs fields.
int launch_decode(const attn_sink_params* p, DecodeArgs& a, int num_splits, void* workspace,
                  size_t workspace_bytes, int left, int right, cudaStream_t s) {
  const int splits = num_splits == 0 ? decode_auto_splits(p) : num_splits;
  const size_t need = decode_ws(p, splits);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return ATTN_SINK_ERR_WORKSPACE;
  const size_t rows = (size_t)p->batch * p->num_heads_q * splits;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  a.part_o = reinterpret_cast<float*>(ws);
  a.part_ml = reinterpret_cast<float*>(ws + align_up(rows * p->head_dim_v * 4, 256));
  a.batch = p->batch; a.total_k = p->total_k; a.max_sk = p->max_seqlen_k;
  a.hq = p->num_heads_q; a.hkv = p->num_heads_kv; a.dk = p->head_dim_qk; a.dv = p->head_dim_v;
  a.splits = splits; a.scale = p->softmax_scale; a.left = left; a.right = right;
  a.status = status_ptr();
  return from_cuda(launch_decode_split(a, p->dtype, s));
}

// Keep threshold and scale of a dropout request: T = floor(256 (1 - p) + 1/2) from the float
// p, evaluated exactly in double (halves round up), in [1, 256]; false when p is outside
// that range.
bool dropout_of(const attn_sink_dropout* d, Dropout& out) {
  out = Dropout{};
  if (!d) return true;
  if (!(d->p >= 0.f) || !isfinite(d->p)) return false;
  const long t = (long)floor(256.0 * (1.0 - (double)d->p) + 0.5);
  if (t < 1 || t > 256) return false;
  out.threshold = (uint32_t)t;
  out.seed_lo = (uint32_t)(d->seed & 0xFFFFFFFFu);
  out.seed_hi = (uint32_t)(d->seed >> 32);
  out.offset = d->offset;
  out.scale = 256.f / (float)t;
  return true;
}

int run_fwd(const attn_sink_params* p, const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
            const int32_t* cu_seqlens_k, const float* sink, const attn_sink_dropout* dropout, void* out, float* lse,
            void* workspace, size_t workspace_bytes, attn_sink_stream_t stream) {
  int st = validate_params(p, false);
  if (st != ATTN_SINK_OK) return st;
  if (!q || !k || !v || !cu_seqlens_q || !cu_seqlens_k || !out) return ATTN_SINK_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (!aligned16(ptr)) return ATTN_SINK_ERR_INVALID_ARG;
  if ((lse && !aligned16(lse)) || (sink && !aligned16(sink))) return ATTN_SINK_ERR_INVALID_ARG;
  FwdArgs a{};
  if (!dropout_of(dropout, a.drop)) return ATTN_SINK_ERR_INVALID_ARG;
  a.q = q; a.k = k; a.v = v; a.cu_q = cu_seqlens_q; a.cu_k = cu_seqlens_k; a.sink = sink;
  a.out = out; a.lse = lse;
  a.batch = p->batch; a.total_q = p->total_q; a.total_k = p->total_k;
  a.max_sq = p->max_seqlen_q; a.max_sk = p->max_seqlen_k;
  a.hq = p->num_heads_q; a.hkv = p->num_heads_kv; a.dk = p->head_dim_qk; a.dv = p->head_dim_v;
  a.scale = p->softmax_scale;
  effective_window(p, a.left, a.right);
  a.status = status_ptr();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dt = p->dtype;   // 0 bf16, 1 fp32, 2 fp16
  if (fwd_sm100_supported(a, dt)) {
    // the persistent kernel's CTAs take their work items from a counter in the workspace
    if (!workspace || workspace_bytes < kFwdWorkspaceBytes || !aligned16(workspace)) return ATTN_SINK_ERR_WORKSPACE;
    a.work_counter = static_cast<unsigned*>(workspace);
    return from_cuda(launch_fwd_sm100(a, dt, s));
  }
  if (fwd_d256_sm100_supported(a, dt)) return from_cuda(launch_fwd_d256_sm100(a, dt, s));
  if (a.drop.threshold) return ATTN_SINK_ERR_UNSUPPORTED;   // dropout runs on the tensor-core path only
  return from_cuda(launch_fwd_simt(a, dt, s));
}

// The backward, with dQ reduced by fp32 atomics into a workspace accumulator (fast) or, in
// the deterministic mode, computed by a query-stationary pass that adds the key tiles'
// contributions in a fixed order.
int run_bwd(const attn_sink_params* p, const void* q, const void* k, const void* v, const void* out,
            const void* dout, const float* lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
            const float* sink, void* dq, void* dk, void* dv, float* dsink, void* workspace,
            size_t workspace_bytes, attn_sink_stream_t stream, bool deterministic,
            const attn_sink_dropout* dropout = nullptr) {
  int st = validate_params(p, false);
  if (st != ATTN_SINK_OK) return st;
  if (!q || !k || !v || !out || !dout || !lse || !cu_seqlens_q || !cu_seqlens_k || !dq || !dk || !dv)
    return ATTN_SINK_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, out, dout, (const void*)lse, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return ATTN_SINK_ERR_INVALID_ARG;
  if ((sink && !aligned16(sink)) || (dsink && !aligned16(dsink))) return ATTN_SINK_ERR_INVALID_ARG;
  const BwdLayout lay = bwd_layout(p);
  if (!workspace || workspace_bytes < lay.total || !aligned16(workspace)) return ATTN_SINK_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  BwdArgs a{};
  if (!dropout_of(dropout, a.drop)) return ATTN_SINK_ERR_INVALID_ARG;
  if (a.drop.threshold) deterministic = true;   // dropout runs on the query-stationary dQ path
  a.q = q; a.k = k; a.v = v; a.out = out; a.dout = dout; a.lse = lse;
  a.cu_q = cu_seqlens_q; a.cu_k = cu_seqlens_k; a.sink = sink;
  a.grad_q = dq; a.grad_k = dk; a.grad_v = dv; a.dsink = dsink;
  a.D = reinterpret_cast<float*>(ws + lay.D);
  a.lse_tot = reinterpret_cast<float*>(ws + lay.lse_tot);
  a.dsink_part = reinterpret_cast<float*>(ws + lay.dsink_part);
  a.dq_acc = (p->dtype != ATTN_SINK_FP32 && !deterministic) ? reinterpret_cast<float*>(ws + lay.dq_acc) : nullptr;
  a.batch = p->batch; a.total_q = p->total_q; a.total_k = p->total_k;
  a.max_sq = p->max_seqlen_q; a.max_sk = p->max_seqlen_k;
  a.hq = p->num_heads_q; a.hkv = p->num_heads_kv; a.dk = p->head_dim_qk; a.dv = p->head_dim_v;
  a.scale = p->softmax_scale;
  effective_window(p, a.left, a.right);
  a.status = status_ptr();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dt = p->dtype;   // 0 bf16, 1 fp32, 2 fp16
  if (bwd_d256_sm100_supported(a, dt)) {   // head dim 256: no atomics in either mode
    cudaError_t e = launch_bwd_preprocess(a, dt, s);
    if (e == cudaSuccess) e = launch_bwd_d256_sm100(a, dt, s);
    return from_cuda(e);
  }
  if (!deterministic) {
    if (bwd_sm100_supported(a, dt)) return from_cuda(launch_bwd_sm100(a, dt, s));
    return from_cuda(launch_bwd_simt(a, dt, s));
  }
  // deterministic: dK / dV on the key-stationary tensor-core kernel without its dQ part,
  // then dQ query-stationary; the CUDA-core path has no atomics to begin with
  const bool tc = bwd_sm100_supported(a, dt) && bwd_dq_sm100_supported(a, dt);
  if (a.drop.threshold && !tc) return ATTN_SINK_ERR_UNSUPPORTED;   // dropout: tensor-core kernels only
  if (tc) {
    cudaError_t e = launch_bwd_sm100(a, dt, s);
    if (e == cudaSuccess) e = launch_bwd_dq_sm100(a, dt, s);
    return from_cuda(e);
  }
  return from_cuda(launch_bwd_simt(a, dt, s));
}

}  // namespace

extern "C" {

int attn_sink_version(void) { return 0x000100; }

const char* attn_sink_status_string(int status) {
  switch (status) {
    case ATTN_SINK_OK: return "ok";
    case ATTN_SINK_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_SINK_ERR_UNSUPPORTED: return "unsupported dtype or head dims";
    case ATTN_SINK_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_SINK_ERR_CUDA: return "CUDA error";
    case ATTN_SINK_ERR_TIMEOUT: return "a bounded on-chip wait timed out";
    case ATTN_SINK_ERR_BAD_INDEX: return "an index or length outside its table was skipped on the device";
    default: return "unknown status";
  }
}

size_t attn_sink_fwd_workspace_size(const attn_sink_params* p) {
  if (validate_params(p, false) != ATTN_SINK_OK) return SIZE_MAX;
  return kFwdWorkspaceBytes;
}

size_t attn_sink_bwd_workspace_size(const attn_sink_params* p) {
  if (validate_params(p, false) != ATTN_SINK_OK) return SIZE_MAX;
  return bwd_layout(p).total;
}

int attn_sink_decode_num_splits(const attn_sink_params* p) {
  if (validate_params(p, true) != ATTN_SINK_OK) return -1;
  return decode_auto_splits(p);
}

size_t attn_sink_decode_workspace_size(const attn_sink_params* p, int num_splits) {
  if (validate_params(p, true) != ATTN_SINK_OK || num_splits < 0) return SIZE_MAX;
  return decode_ws(p, num_splits == 0 ? decode_auto_splits(p) : num_splits);
}

int attn_sink_fwd(const attn_sink_params* p, const void* q, const void* k, const void* v,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                  void* out, float* lse, void* workspace, size_t workspace_bytes,
                  attn_sink_stream_t stream) {
  return run_fwd(p, q, k, v, cu_seqlens_q, cu_seqlens_k, sink, nullptr, out, lse, workspace, workspace_bytes,
                 stream);
}

int attn_sink_fwd_dropout(const attn_sink_params* p, const void* q, const void* k, const void* v,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                          const attn_sink_dropout* dropout, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, attn_sink_stream_t stream) {
  if (!dropout) return ATTN_SINK_ERR_INVALID_ARG;
  return run_fwd(p, q, k, v, cu_seqlens_q, cu_seqlens_k, sink, dropout, out, lse, workspace, workspace_bytes,
                 stream);
}


int attn_sink_bwd(const attn_sink_params* p, const void* q, const void* k, const void* v,
                  const void* out, const void* dout, const float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                  void* dq, void* dk, void* dv, float* dsink, void* workspace,
                  size_t workspace_bytes, attn_sink_stream_t stream) {
  return run_bwd(p, q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, sink, dq, dk, dv, dsink, workspace,
                 workspace_bytes, stream, false);
}

int attn_sink_bwd_deterministic(const attn_sink_params* p, const void* q, const void* k, const void* v,
                                const void* out, const void* dout, const float* lse,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                                void* dq, void* dk, void* dv, float* dsink, void* workspace,
                                size_t workspace_bytes, attn_sink_stream_t stream) {
  return run_bwd(p, q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, sink, dq, dk, dv, dsink, workspace,
                 workspace_bytes, stream, true);
}

int attn_sink_bwd_dropout(const attn_sink_params* p, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, const float* lse, const int32_t* cu_seqlens_q,
                          const int32_t* cu_seqlens_k, const float* sink, const attn_sink_dropout* dropout,
                          void* dq, void* dk, void* dv, float* dsink, void* workspace, size_t workspace_bytes,
                          attn_sink_stream_t stream) {
  if (!dropout) return ATTN_SINK_ERR_INVALID_ARG;
  return run_bwd(p, q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, sink, dq, dk, dv, dsink, workspace,
                 workspace_bytes, stream, true, dropout);
}

int attn_sink_decode(const attn_sink_params* p, const void* q, const void* k, const void* v,
                     const int32_t* cu_seqlens_k, const float* sink, int num_splits, void* out,
                     float* lse, void* workspace, size_t workspace_bytes,
                     attn_sink_stream_t stream) {
  int st = validate_params(p, true);
  if (st != ATTN_SINK_OK) return st;
  if (num_splits < 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (!q || !k || !v || !cu_seqlens_k || !out) return ATTN_SINK_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (!aligned16(ptr)) return ATTN_SINK_ERR_INVALID_ARG;
  if ((lse && !aligned16(lse)) || (sink && !aligned16(sink))) return ATTN_SINK_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int left, right;
  effective_window(p, left, right);
  if (p->dtype == ATTN_SINK_FP32) {
    FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.cu_q = nullptr; a.cu_k = cu_seqlens_k; a.sink = sink;
    a.out = out; a.lse = lse;
    a.batch = p->batch; a.total_q = p->total_q; a.total_k = p->total_k;
    a.max_sq = 1; a.max_sk = p->max_seqlen_k;
    a.hq = p->num_heads_q; a.hkv = p->num_heads_kv; a.dk = p->head_dim_qk; a.dv = p->head_dim_v;
    a.scale = p->softmax_scale; a.left = left; a.right = right;
    a.status = status_ptr();
    return from_cuda(launch_fwd_simt(a, 1, s));
  }
  DecodeArgs a{};
  a.q = q; a.k = k; a.v = v; a.cu_k = cu_seqlens_k; a.sink = sink; a.out = out; a.lse = lse;
  return launch_decode(p, a, num_splits, workspace, workspace_bytes, left, right, s);
}

int attn_sink_decode_paged(const attn_sink_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_table, const int32_t* seqused_k,
                           int num_blocks, int block_size, int max_blocks_per_seq, const float* sink,
                           int num_splits, void* out, float* lse, void* workspace,
                           size_t workspace_bytes, attn_sink_stream_t stream) {
  int st = validate_params(p, true);
  if (st != ATTN_SINK_OK) return st;
  if (p->dtype == ATTN_SINK_FP32) return ATTN_SINK_ERR_UNSUPPORTED;
  if (num_splits < 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !block_table || !seqused_k || !out) return ATTN_SINK_ERR_INVALID_ARG;
  if (block_size < 16 || block_size > 1024 || block_size % 16 != 0) return ATTN_SINK_ERR_INVALID_ARG;
  if (num_blocks <= 0 || max_blocks_per_seq <= 0) return ATTN_SINK_ERR_INVALID_ARG;
  if ((long long)num_blocks * block_size != p->total_k) return ATTN_SINK_ERR_INVALID_ARG;
  for (const void* ptr : {q, k_cache, v_cache, (const void*)out})
    if (!aligned16(ptr)) return ATTN_SINK_ERR_INVALID_ARG;
  if ((lse && !aligned16(lse)) || (sink && !aligned16(sink))) return ATTN_SINK_ERR_INVALID_ARG;
  int left, right;
  effective_window(p, left, right);
  DecodeArgs a{};
  a.q = q; a.k = k_cache; a.v = v_cache; a.cu_k = nullptr; a.sink = sink; a.out = out; a.lse = lse;
  a.block_table = block_table; a.seqused_k = seqused_k;
  a.block_size = block_size; a.max_blocks = max_blocks_per_seq; a.num_blocks = num_blocks;
  return launch_decode(p, a, num_splits, workspace, workspace_bytes, left, right,
                       static_cast<cudaStream_t>(stream));
}

int attn_sink_selftest_wait_timeout(attn_sink_stream_t stream) {
  unsigned* sp = status_ptr();
  if (!sp) return ATTN_SINK_ERR_CUDA;
  return from_cuda(launch_wait_timeout_selftest(sp, static_cast<cudaStream_t>(stream)));
}

int attn_sink_get_device_status(attn_sink_stream_t stream, uint32_t* bits) {
  unsigned* sp = status_ptr();
  if (!sp) return ATTN_SINK_ERR_CUDA;
  unsigned host = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&host, sp, sizeof(unsigned), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ATTN_SINK_ERR_CUDA;
  if (cudaMemsetAsync(sp, 0, sizeof(unsigned), s) != cudaSuccess) return ATTN_SINK_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_SINK_ERR_CUDA;
  if (bits) *bits = host;
  if (host & kStatusTimeout) return ATTN_SINK_ERR_TIMEOUT;
  return host ? ATTN_SINK_ERR_BAD_INDEX : ATTN_SINK_OK;
}

int attn_sink_check_seqlens(const attn_sink_params* p, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            attn_sink_stream_t stream) {
  if (!p || !cu_seqlens_k || p->batch <= 0) return ATTN_SINK_ERR_INVALID_ARG;
  unsigned* sp = status_ptr();
  if (!sp) return ATTN_SINK_ERR_CUDA;
  return from_cuda(launch_check_seqlens(cu_seqlens_q, cu_seqlens_k, p->batch, p->total_q, p->total_k,
                                        p->max_seqlen_q, p->max_seqlen_k, sp, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
