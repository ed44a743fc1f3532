// Internal launcher interface between the C-ABI host code and the kernels.
// Not part of the public ABI (that is include/attn_sink.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace attn_sink {

// A window side at or above this value is unbounded.
constexpr int kUnbounded = 1 << 30;

// Bits of the per-device status word.
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadIndex = 2u;  // a paged block id or key count outside its table
constexpr unsigned kStatusBadSeqlens = 4u;  // cu_seqlens broke its contract (attn_sink_check_seqlens)
constexpr unsigned kStatusDebugBounds = 8u;  // debug builds: a store outside its tensor was skipped

// Dropout keep decisions: key j of packed query row r and q head h is kept when byte j % 16
// of Philox4x32-10(counter = (j / 16, r, h, offset), key = (seed_lo, seed_hi)) is below the
// threshold T (keep probability T / 256); kept values are scaled by 256 / T.  Byte t is bits
// 8 (t % 4) .. +7 of output word t / 4.
struct Dropout {
  uint32_t threshold;   // T in [1, 256]; 0 = no dropout
  uint32_t seed_lo, seed_hi, offset;
  float scale;          // 256 / T
};

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu_q;   // nullptr in decode mode: sequence b owns exactly q row b
  const int32_t* cu_k;
  const float* sink;     // nullptr = -inf
  void* out;
  float* lse;            // may be nullptr
  int batch, total_q, total_k, max_sq, max_sk, hq, hkv, dk, dv;
  float scale;
  int left, right;       // effective window (causal folded into right), kUnbounded = none
  unsigned* status;
  Dropout drop;          // threshold 0 = none (tensor-core path only)
  unsigned* work_counter;  // workspace word the persistent forward's CTAs take items from (zeroed per launch)
};

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const void* dout;
  const float* lse;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* sink;
  void* grad_q;          // dq [total_q, hq, dk]
  void* grad_k;          // dk [total_k, hkv, dk]
  void* grad_v;          // dv [total_k, hkv, dv]
  float* dsink;          // may be nullptr
  float* D;              // workspace [hq, total_q]: rowsum(dout * out)
  float* lse_tot;        // workspace [hq, total_q]: logaddexp(lse, sink)
  float* dq_acc;         // workspace [total_q, hq, dk] fp32 (tensor-core path; nullptr = no dQ there)
  float* dsink_part;     // workspace [hq, preprocess blocks] fp32: per-block d_sink partials
  int batch, total_q, total_k, max_sq, max_sk, hq, hkv, dk, dv;
  float scale;
  int left, right;
  unsigned* status;
  int band_groups;       // tensor-core path: (sequence, kv head) groups whose key tiles run together
  Dropout drop;          // threshold 0 = none (deterministic tensor-core path only)
};

struct DecodeArgs {
  const void* q;         // [batch, hq, dk]
  const void* k;
  const void* v;
  const int32_t* cu_k;
  const float* sink;
  void* out;             // [batch, hq, dv]
  float* lse;            // [hq, batch] or nullptr
  float* part_o;         // workspace [batch, hq, splits, dv]
  float* part_ml;        // workspace [batch, hq, splits, 2] (max, sum)
  int batch, total_k, max_sk, hq, hkv, dk, dv, splits;
  float scale;
  int left, right;
  unsigned* status;
  // Paged K/V (block_table != nullptr): k/v are caches [num_blocks, block_size, hkv, d];
  // key t of sequence b is row t % block_size of block block_table[b * max_blocks +
  // t / block_size]; sequence b has seqused_k[b] keys and cu_k is unused.
  const int32_t* block_table;
  const int32_t* seqused_k;
  int block_size, max_blocks, num_blocks;
};

// dtype: 0 = bf16, 1 = fp32, 2 = fp16.  Each returns cudaSuccess or the launch error.
cudaError_t launch_fwd_simt(const FwdArgs& a, int dtype, cudaStream_t s);
bool fwd_sm100_supported(const FwdArgs& a, int dtype);
cudaError_t launch_fwd_sm100(const FwdArgs& a, int dtype, cudaStream_t s);
// head dim 256 (dk = dv = 256), bf16 / fp16
bool fwd_d256_sm100_supported(const FwdArgs& a, int dtype);
cudaError_t launch_fwd_d256_sm100(const FwdArgs& a, int dtype, cudaStream_t s);

// D, lse_tot and dsink (dsink cleared first); shared by both backward paths.
cudaError_t launch_bwd_preprocess(const BwdArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_bwd_simt(const BwdArgs& a, int dtype, cudaStream_t s);
bool bwd_sm100_supported(const BwdArgs& a, int dtype);
// With a.dq_acc == nullptr the tensor-core backward computes dK and dV only.
cudaError_t launch_bwd_sm100(const BwdArgs& a, int dtype, cudaStream_t s);
// Query-stationary dQ without atomics (the deterministic backward's dQ pass).
bool bwd_dq_sm100_supported(const BwdArgs& a, int dtype);
cudaError_t launch_bwd_dq_sm100(const BwdArgs& a, int dtype, cudaStream_t s);
// head dim 256 (dk = dv = 256), bf16 / fp16: dQ, dK and dV kernels after the preprocess;
// deterministic (no atomics)
bool bwd_d256_sm100_supported(const BwdArgs& a, int dtype);
cudaError_t launch_bwd_d256_sm100(const BwdArgs& a, int dtype, cudaStream_t s);
// Contract check of cu_seqlens_q (may be nullptr) and cu_seqlens_k; sets kStatusBadSeqlens.
cudaError_t launch_check_seqlens(const int32_t* cu_q, const int32_t* cu_k, int batch, int total_q, int total_k,
                                 int max_sq, int max_sk, unsigned* status, cudaStream_t s);
// d_sink from the preprocess pass's per-block partials, summed in a fixed order.
cudaError_t launch_dsink_reduce(const BwdArgs& a, cudaStream_t s);

cudaError_t launch_decode_split(const DecodeArgs& a, int dtype, cudaStream_t s);

// A one-thread kernel whose bounded mbarrier wait is made to run out (diagnostics).
cudaError_t launch_wait_timeout_selftest(unsigned* status, cudaStream_t s);
bool decode_split_supported(int dk, int dv, int dtype);

}  // namespace attn_sink
