/*
 * attn_sink.h -- C ABI of the B200 (sm_100a) sink-attention library, libattn_sink.so.
 *
 * The operation (Huawei CANN ops-transformer "flash_attn" doc, section "Function",
 * the formula after "After adding sink"):
 *
 *     S   = scale * Q K^T                       per (sequence, q head)
 *     m   = max(sink, max_j S_j)
 *     out = sum_j e^{S_j - m} V_j / (sum_j e^{S_j - m} + e^{sink - m})
 *
 * sink is a per-q-head fp32 logit in post-scale units.  It is the learnable softmax
 * offset of slime's learnable_softmax_attention.py (module docstring: an appended
 * logit column, equivalently softmax(S) * sigmoid(lse - offset)) and softmax_n of the
 * Flash-Attention-Softmax-N README with sink = log n.  A NULL sink means -inf, i.e.
 * plain softmax attention.
 *
 * Conventions shared by every entry point
 *   - Layout: packed THD, row-major, contiguous.
 *       q   [total_q, num_heads_q,  head_dim_qk]
 *       k   [total_k, num_heads_kv, head_dim_qk]
 *       v   [total_k, num_heads_kv, head_dim_v ]
 *       out [total_q, num_heads_q,  head_dim_v ]
 *       lse [num_heads_q, total_q] fp32   (CANN doc, softmax_lse note: (Q_N, Q_T) for TND)
 *       sink [num_heads_q] fp32
 *     Sequence b owns q rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and k/v rows
 *     [cu_seqlens_k[b], cu_seqlens_k[b+1]); both arrays are int32 [batch + 1], start
 *     at 0, never decrease, end at total_q / total_k (slime wrapper docstring; CANN doc,
 *     "SeqLengths Parameter Group").  Zero-length sequences are allowed.
 *   - GQA: num_heads_q % num_heads_kv == 0; q head h reads kv head
 *     h / (num_heads_q / num_heads_kv) (CANN doc, "Common Parameter Group").
 *   - Masking: query row i of a sequence with sq queries and sk keys sits at key
 *     position i + (sk - sq) (bottom-right alignment, PyTorch issue #108108,
 *     "Proposal").  It sees key j iff  pos - window_left <= j <= pos + window_right,
 *     where -1 means unbounded (slime wrapper docstring "window_size"; CANN doc,
 *     "Mask Parameter Group") and causal sets window_right = min(window_right, 0).
 *     A row that sees no key outputs 0 (issue #108108) and has lse = -inf.
 *   - lse is the vanilla log-sum-exp of the visible scaled scores, natural log,
 *     WITHOUT the sink (CANN doc, softmax_lse formula).
 *   - dtype: ATTN_SINK_BF16 or ATTN_SINK_FP16 (16-bit q/k/v/out/dout/dq/dk/dv, fp32
 *     accumulation, P and dS rounded to the same 16-bit type for the tensor cores, outputs
 *     rounded once to nearest-even; the CANN doc lists both BFLOAT16 and FLOAT16 for
 *     q / k / v) or ATTN_SINK_FP32 (fp32 everywhere, no tensor cores).
 *   - Supported head dims: head_dim_qk in {64, 128} with head_dim_v in {32, 64, 128}, and
 *     head_dim_qk = head_dim_v = 256 (the CANN flash_attn doc lists 64, 128 and 256).
 *   - Ownership: the caller allocates every buffer (inputs, outputs, workspace).  The
 *     library never allocates, frees or synchronises; every pointer except `params`
 *     is a device pointer and must be 16-byte aligned.  Calls are asynchronous on
 *     `stream` (a cudaStream_t; NULL = the legacy default stream).
 *   - Errors: the return value is an attn_sink_status.  Arguments the host can see
 *     are validated before anything is launched (ATTN_SINK_ERR_INVALID_ARG,
 *     ATTN_SINK_ERR_UNSUPPORTED, ATTN_SINK_ERR_WORKSPACE); a failed launch returns
 *     ATTN_SINK_ERR_CUDA.  The contents of cu_seqlens are the caller's contract (as in
 *     the CANN doc's "Declaration"): they are not read on the host.  Kernels that wait
 *     on on-chip barriers give every wait an iteration limit; a wait that runs out
 *     sets a bit in a per-device status word and the kernel returns early, leaving
 *     the outputs undefined.  attn_sink_get_device_status() reads and clears it.
 */
#ifndef ATTN_SINK_H
#define ATTN_SINK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_SINK_BF16 = 0, ATTN_SINK_FP32 = 1, ATTN_SINK_FP16 = 2 } attn_sink_dtype;

typedef enum {
  ATTN_SINK_OK = 0,
  ATTN_SINK_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, ... */
  ATTN_SINK_ERR_UNSUPPORTED = 2,   /* head dims / dtype outside the supported set     */
  ATTN_SINK_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required      */
  ATTN_SINK_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed            */
  ATTN_SINK_ERR_TIMEOUT = 5,       /* device status: a bounded on-chip wait ran out   */
  ATTN_SINK_ERR_BAD_INDEX = 6      /* device status: a paged block id, a key count or a
                                      sequence length fell outside what the call's
                                      tables and sizes allow; those keys were skipped  */
} attn_sink_status;

/* Problem description shared by the three entry points (plain struct, by pointer). */
typedef struct {
  int batch;            /* B > 0: number of sequences                                  */
  int total_q;          /* rows of q / out (> 0); decode: must equal batch             */
  int total_k;          /* rows of k / v (> 0)                                         */
  int max_seqlen_q;     /* >= every sequence's query length (decode: 1)                */
  int max_seqlen_k;     /* >= every sequence's key length                              */
  int num_heads_q;      /* Hq > 0                                                      */
  int num_heads_kv;     /* Hkv > 0, Hq % Hkv == 0                                      */
  int head_dim_qk;      /* 64 or 128; or 256 with head_dim_v = 256                     */
  int head_dim_v;       /* 32, 64 or 128; or 256 with head_dim_qk = 256                */
  float softmax_scale;  /* multiplies QK^T; finite.  The slime wrapper's default is
                           1/sqrt(head_dim_qk); here the caller passes it explicitly   */
  int causal;           /* nonzero: bottom-right causal                                */
  int window_left;      /* >= -1; -1 = unbounded                                       */
  int window_right;     /* >= -1; -1 = unbounded                                       */
  attn_sink_dtype dtype;
} attn_sink_params;

/* Opaque stream handle: pass a cudaStream_t. */
typedef void* attn_sink_stream_t;

/*
 * Dropout on the attention probabilities (slime wrapper's `dropout_p`, which it passes to
 * flash attention before the sigmoid(lse - offset) scaling, i.e. dropout acts on the
 * sink-normalised probabilities).  Key j of packed query row r and q head h is kept when
 * byte j % 16 of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 * Easy as 1, 2, 3", SC 2011) with counter (j / 16, r, h, offset) and key (seed low 32 bits,
 * seed high 32 bits) is below T = floor(256 (1 - p) + 1/2) (p as passed, evaluated
 * exactly); byte t is bits 8 (t % 4) .. +7 of
 * output word t / 4.  Kept probabilities are scaled by 256 / T (keep probability T / 256),
 * so the output's expectation is the output without dropout; lse is not affected.
 * 1 <= T <= 256 is required (0 <= p < 1 - 1/512).  The backward draws the same decisions.
 */
typedef struct {
  float p;          /* dropout probability                                          */
  uint64_t seed;    /* Philox key                                                   */
  uint32_t offset;  /* fourth counter word, e.g. a step counter for fresh masks     */
} attn_sink_dropout;

/*
 * Forward (CANN doc, "Function" formula and softmax_lse formula; slime
 * learnable_softmax_flash_attn_varlen).  Writes out [total_q, Hq, dv] (dtype) and, when
 * `lse` is not NULL, lse [Hq, total_q] fp32.  sink may be NULL (= -inf).  The workspace
 * (attn_sink_fwd_workspace_size() bytes, 16-byte aligned, contents ignored) holds the work
 * counter the bf16/fp16 tensor-core forward's CTAs take their items from; the call zeroes
 * it on `stream` first, so two forwards that overlap on the GPU need two workspaces.  A
 * missing or smaller workspace returns ATTN_SINK_ERR_WORKSPACE on that path (the fp32 and
 * head-dim-256 forwards do not read it).
 */
int attn_sink_fwd(const attn_sink_params* params, const void* q, const void* k, const void* v,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                  void* out, float* lse, void* workspace, size_t workspace_bytes,
                  attn_sink_stream_t stream);

/*
 * Backward of the forward above for the loss sum(dout * out) (the gradient the slime
 * class docstring describes: dS = P * s * (D - s * di) with s = sigmoid(lse - sink),
 * and d_offset = -sum_i (dout_i . out_vanilla_i) s_i (1 - s_i)).
 * Inputs: q, k, v, the forward's out and lse (lse REQUIRED), dout [total_q, Hq, dv].
 * Outputs (all overwritten): dq [total_q, Hq, dk], dk [total_k, Hkv, dk],
 * dv [total_k, Hkv, dv] (dtype; dk / dv sum over the q heads of each group) and
 * dsink [Hq] fp32 (may be NULL when sink is NULL or not wanted).
 */
int attn_sink_bwd(const attn_sink_params* params, const void* q, const void* k, const void* v,
                  const void* out, const void* dout, const float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                  void* dq, void* dk, void* dv, float* dsink, void* workspace,
                  size_t workspace_bytes, attn_sink_stream_t stream);

/*
 * Forward and backward with dropout (see attn_sink_dropout); otherwise the arguments of
 * attn_sink_fwd / attn_sink_bwd.  Tensor-core paths only: bf16 or fp16 with head_dim_qk in
 * {64, 128} and head_dim_v in {32, 64, 128}, or 256 / 256 (ATTN_SINK_ERR_UNSUPPORTED
 * otherwise; ATTN_SINK_ERR_INVALID_ARG for a NULL dropout or p out of range).  The backward
 * takes the deterministic path (bit-identical results from run to run) and the workspace
 * attn_sink_bwd_workspace_size() gives.
 */
int attn_sink_fwd_dropout(const attn_sink_params* params, const void* q, const void* k,
                          const void* v, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          const float* sink, const attn_sink_dropout* dropout, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, attn_sink_stream_t stream);
int attn_sink_bwd_dropout(const attn_sink_params* params, const void* q, const void* k,
                          const void* v, const void* out, const void* dout, const float* lse,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const float* sink,
                          const attn_sink_dropout* dropout, void* dq, void* dk, void* dv, float* dsink,
                          void* workspace, size_t workspace_bytes, attn_sink_stream_t stream);

/*
 * Deterministic backward: the same arguments, results and workspace size as
 * attn_sink_bwd, and bit-identical outputs from run to run (the slime wrapper exposes a
 * `deterministic` flag for the same purpose).  attn_sink_bwd adds the dQ contributions of
 * different key tiles with fp32 atomics, whose order varies; here dQ is computed by a
 * query-stationary pass that adds them in a fixed order (dK, dV and dsink are reduced in a
 * fixed order by both entry points).  Slower than attn_sink_bwd: Q K^T and dout V^T are
 * computed twice.
 */
int attn_sink_bwd_deterministic(const attn_sink_params* params, const void* q, const void* k,
                                const void* v, const void* out, const void* dout, const float* lse,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                const float* sink, void* dq, void* dk, void* dv, float* dsink,
                                void* workspace, size_t workspace_bytes, attn_sink_stream_t stream);

/*
 * Decode: one query per sequence, q [batch, Hq, dk] (cu_seqlens_q = 0, 1, ..., batch is
 * implied; total_q == batch, max_seqlen_q == 1).  K/V are packed with cu_seqlens_k.
 * The keys of each (sequence, kv head) are cut into num_splits chunks (0 = choose
 * automatically), each chunk produces (max, sum, unnormalised output) without the sink,
 * and a merge combines them and applies the sink exactly once (CANN doc, softmax_lse
 * note on combining partial results).  Writes out [batch, Hq, dv] and, when not NULL,
 * lse [Hq, batch].  The workspace holds the partials.  fp32 problems are computed
 * without splitting.
 */
int attn_sink_decode(const attn_sink_params* params, const void* q, const void* k, const void* v,
                     const int32_t* cu_seqlens_k, const float* sink, int num_splits, void* out,
                     float* lse, void* workspace, size_t workspace_bytes,
                     attn_sink_stream_t stream);

/*
 * Paged decode: attn_sink_decode with K/V in a block cache (CANN doc, "Paged Attention
 * Parameter Group", and the PA_BBND layout of k / v in its parameter table).
 *   k_cache [num_blocks, block_size, Hkv, dk], v_cache [num_blocks, block_size, Hkv, dv]
 *     (dtype; contiguous).  Key t of sequence b is row t % block_size of block
 *     block_table[b * max_blocks_per_seq + t / block_size].
 *   block_table int32 [batch, max_blocks_per_seq]: block ids in [0, num_blocks).  Only the
 *     first ceil(seqused_k[b] / block_size) entries of row b are read; blocks may be shared
 *     between sequences and appear in any order.
 *   seqused_k int32 [batch]: keys of each sequence, 0 <= seqused_k[b] <=
 *     max_blocks_per_seq * block_size, and <= params->max_seqlen_k.
 *   16 <= block_size <= 1024 and block_size % 16 == 0 (the CANN doc's range).
 * params: total_q == batch, max_seqlen_q == 1 as for attn_sink_decode; total_k must equal
 * num_blocks * block_size; max_seqlen_k bounds every seqused_k[b] (it sizes the chunks).
 * The query of sequence b sits at key position seqused_k[b] - 1 (bottom-right), so causal
 * decode sees all of its keys and a window keeps the last window_left + 1 of them.
 * Writes out [batch, Hq, dv] and, when not NULL, lse [Hq, batch]; the workspace is the one
 * attn_sink_decode_workspace_size() gives for the same params and num_splits.  bf16 or fp16
 * (ATTN_SINK_ERR_UNSUPPORTED for fp32).  Table contents are the caller's contract: a
 * block id outside [0, num_blocks) or a seqused_k beyond its table row is not read (those
 * keys count as zero vectors) and sets the device status that
 * attn_sink_get_device_status() reports as ATTN_SINK_ERR_BAD_INDEX.
 */
int attn_sink_decode_paged(const attn_sink_params* params, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_table, const int32_t* seqused_k,
                           int num_blocks, int block_size, int max_blocks_per_seq, const float* sink,
                           int num_splits, void* out, float* lse, void* workspace,
                           size_t workspace_bytes, attn_sink_stream_t stream);

/*
 * Decode that allocates nothing and takes no workspace.  None of the pages this library
 * follows has a counterpart: it exists for callers that cannot allocate device memory
 * (a plugin or custom-op host that passes only the call's tensors and offers no
 * allocator, a process whose device memory is all held by another framework's pool, or a
 * latency-critical loop that must not allocate).  Same arguments, results and kernels as
 * attn_sink_decode, minus the workspace: the chunk partials live in a fixed 16 MiB
 * device array inside the library, present on every GPU that loads the library until the
 * process exits.  No cudaMalloc, cudaFree or other allocating routine is called.
 *   - num_splits == 0 picks the automatic split count of attn_sink_decode_num_splits(),
 *     or, when its partials need more than 16 MiB, the largest smaller count whose
 *     partials fit; an explicit num_splits whose partials need more than 16 MiB, or a
 *     problem that does not fit even with one split, returns ATTN_SINK_ERR_WORKSPACE
 *     before any launch.
 *   - Each call made outside stream capture looks up the array's device address
 *     (cudaGetSymbolAddress with the device current), so the address stays right after a
 *     cudaDeviceReset or in another context of the device.  A call made while `stream`
 *     is being captured reuses the address of the device's last uncaptured call; make at
 *     least one uncaptured call on a device before capturing (otherwise
 *     ATTN_SINK_ERR_CUDA).
 *   - All calls share the one array and it keeps the last call's contents.  Nothing in
 *     it has to start at zero (each call writes every slot it later reads), but calls
 *     whose kernels overlap on the GPU race on it: order them on one stream.
 */
int attn_sink_decode_noalloc(const attn_sink_params* params, const void* q, const void* k,
                             const void* v, const int32_t* cu_seqlens_k, const float* sink,
                             int num_splits, void* out, float* lse, attn_sink_stream_t stream);

/* Workspace bytes each entry point needs for `params` (0 = none; SIZE_MAX = params invalid). */
size_t attn_sink_fwd_workspace_size(const attn_sink_params* params);
size_t attn_sink_bwd_workspace_size(const attn_sink_params* params);
size_t attn_sink_decode_workspace_size(const attn_sink_params* params, int num_splits);

/* The split count attn_sink_decode uses for num_splits == 0. */
int attn_sink_decode_num_splits(const attn_sink_params* params);

/* Static text for a status code. */
const char* attn_sink_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the calling device's status word.
 * Returns ATTN_SINK_OK, ATTN_SINK_ERR_TIMEOUT (a bounded wait ran out; bit 0),
 * ATTN_SINK_ERR_BAD_INDEX (an index or length outside its table was skipped, bit 1;
 * attn_sink_check_seqlens found a broken cu_seqlens, bit 2; or, in the debug build
 * libattn_sink_debug.so only, a kernel skipped a store whose index range left the output
 * it writes, bit 3) or ATTN_SINK_ERR_CUDA.  *bits (if not NULL) receives the raw word.
 */
int attn_sink_get_device_status(attn_sink_stream_t stream, uint32_t* bits);

/*
 * Debug check of the cu_seqlens contract, which the other entry points take on trust (the
 * CANN doc leaves invalid values undefined; "SeqLengths Parameter Group"): both arrays
 * start at 0, never decrease and end at total_q / total_k, and no sequence is longer than
 * max_seqlen_q / max_seqlen_k.  cu_seqlens_q may be NULL (decode).  One small kernel on
 * `stream`, asynchronous; a violation sets the device status, which
 * attn_sink_get_device_status() then reports as ATTN_SINK_ERR_BAD_INDEX (bit 2).  Returns
 * ATTN_SINK_ERR_INVALID_ARG for a NULL params / cu_seqlens_k or batch <= 0, else the launch
 * status.
 */
int attn_sink_check_seqlens(const attn_sink_params* params, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, attn_sink_stream_t stream);

/*
 * Diagnostics, with no counterpart on the pages: launches a one-thread kernel whose bounded
 * on-chip wait is made to run out (it waits for an mbarrier phase nothing completes), so the
 * timeout path of the tensor-core kernels can be exercised without faulting or hanging the
 * GPU.  Takes about 2 s of GPU time.  Afterwards attn_sink_get_device_status() returns
 * ATTN_SINK_ERR_TIMEOUT (and clears the word); the context stays usable.  Returns the
 * launch status.
 */
int attn_sink_selftest_wait_timeout(attn_sink_stream_t stream);

/* Library version, e.g. 0x000100 for 0.1.0. */
int attn_sink_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_SINK_H */
