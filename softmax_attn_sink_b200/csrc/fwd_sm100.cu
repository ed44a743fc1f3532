// Sink-attention forward on the sm_100a tensor cores (bf16 in, fp32 accumulation).
//
// What it computes (Huawei CANN ops-transformer flash_attn doc, "Function", the formula
// after "After adding sink"; softmax_lse formula of the same section):
//   S = scale * Q K^T,  m = max(sink, max S),
//   out = sum e^{S-m} V / (sum e^{S-m} + e^{sink-m}),   lse = log sum e^{S}  (no sink).
//
// A work item is two 128-row query units, A and B, that read the same K/V tiles: two q heads
// of one GQA group at the same row tile when the group size is even (identical key ranges),
// otherwise two adjacent row tiles of one head.  Keys are streamed in 128-key tiles over the
// union of the two units' visible ranges (bottom-right causal / sliding window, PyTorch
// issue #108108 "Proposal"; slime wrapper docstring "window_size"); each unit only takes the
// tiles that meet its own range.  The kernel is persistent: one CTA per SM walks a
// longest-first list of items (built in shared memory from cu_seqlens_q by every CTA), and
// the K/V ring, the TMEM buffers and the mbarrier phases carry over from one item to the
// next, so an item's Q load and first QK overlap the previous item's last tiles.  Warp roles:
//   warp 0      TMA producer: Q_A, Q_B per item (once the previous item's last QK has read
//               Q), then K and V tiles into a 2-stage ring; a stage's K and V are released
//               together once both PVs of its tile are issued (one commit per tile).
//   warp 1      TMEM allocation and the MMA issuer, in the order
//                 PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1)
//               Without dropout the whole warp runs the loop in step and elect.sync over the
//               full warp picks the issuing lane (the same lane every time, so every MMA and
//               commit still comes from one thread); with dropout lane 0 alone runs it.
//               so the tensor core works for one unit while the other unit's softmax runs;
//               on an item's last tile the QKs of the next item's first tile follow the
//               PVs directly.  QK: S_U = Q_U K^T (A, B from shared memory); PV: O_U += P_U V
//               (P from TMEM).  An MMA issue returns only once the tensor core takes it, so
//               the thread waits for the next tile's V while earlier MMAs are still queued.
//   warp 2      the scheduler: builds the item list, then decodes the CTA's items one by one
//               into a 2-slot shared-memory ring that the other roles read (warp 3 idles).
//   warps 4-7   softmax and epilogue of unit A, warps 8-11 of unit B: thread t owns query row
//               t (TMEM lane t).  The running max starts at the sink (log2 domain, the sink is
//               in post-scale units); the running sum counts keys only and e^{sink-m} joins
//               the denominator in the epilogue, so the vanilla lse is m + log sum.  O is
//               rescaled lazily, only when a row's max grows by more than 2^8 (exact: O and
//               the sum share the stale reference).  An item's epilogue runs after the
//               unit's next first softmax has read O out of TMEM (without dropout), and its
//               rows go out through a per-warp shared-memory stage as whole row segments.
// TMEM columns: S_A [0,128) O_A [128,256) S_B [256,384) O_B [384,512); P_U (bf16) is written
// over the first 64 columns of S_U once S_U has been read; the next QK_U into S_U is issued
// after the PV_U that reads it, and MMAs from one thread execute in issue order.  Because a
// commit tracks every earlier MMA of the thread, S_U(j) being ready also means PV_U(j-1) is
// done: the lazy rescale of O needs no other wait, and pv_done is committed only after a
// unit's last PV of an item, for its epilogue.  Every mbarrier wait is bounded; a timeout sets the status word and the CTA drains
// and frees its TMEM instead of hanging.
#include <cuda.h>

#include "sm100_ptx.cuh"
#include "tma_map.h"

namespace attn_sink {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per unit
constexpr int kBN = 128;       // keys per tile
constexpr int kStages = 2;     // K / V ring depth
constexpr int kThreads = 384;  // 3 warpgroups
constexpr int kItemSlots = 2;  // scheduled items in flight
constexpr int kItemReaders = 10;  // item slot readers: producer, MMA thread, 8 softmax warps
// Registers: launched at 168 per thread (384 x 168 = 64512); the TMA/MMA warpgroup gives
// back down to 72 and the two softmax warpgroups take 216: 128 x 72 + 256 x 216 = 64512.
constexpr int kRegsLaunch = 168, kRegsProducer = 72, kRegsSoftmax = 216;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__host__ __device__ constexpr uint32_t col_S(int u) { return u ? 256u : 0u; }
__host__ __device__ constexpr uint32_t col_O(int u) { return u ? 384u : 128u; }

template <int DK, int DV>
struct Layout {
  static constexpr int KH = DK / 64, VH = DV / 64;           // 64-element (128-byte) column halves
  static constexpr int kHalfBytes = kBM * 128;               // one 128-row x 64-column box
  static constexpr int kQBytes = KH * kHalfBytes;
  static constexpr int kKBytes = KH * kHalfBytes;
  static constexpr int kVBytes = VH * kHalfBytes;
  static constexpr int kOffQ = 0;                             // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffBar = kOffV + kStages * kVBytes;
  // q_full, q_empty, k_full[S], kv_empty[S], v_full[S], s_full[2], p_full[2], pv_done[2],
  // drain, item_full[I], item_empty[I]
  static constexpr int kNumBars = 2 + 3 * kStages + 7 + 2 * kItemSlots;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffItems = (kOffTmemSlot + 16 + 127) / 128 * 128;  // ItemDesc[kItemSlots]
  static constexpr int kOffTable = kOffItems + kItemSlots * 128;           // item list of a persistent launch
  // Output staging after the table: 32 rows x 64 columns (128 B) per softmax warp.
  static constexpr int kStageBytes = 32 * 128;
  static constexpr long long stage_offset(long long table_ints) { return (kOffTable + 4 * table_ints + 127) / 128 * 128; }
  // bytes for a table of `table_ints` ints (and the staging area), + slack to align the base
  // to 1 KB; at least 116 KB so that two CTAs never share an SM (each CTA holds all 512 TMEM
  // columns)
  static constexpr long long smem_bytes(long long table_ints, bool staged) {
    const long long b = (staged ? stage_offset(table_ints) + 8LL * kStageBytes : kOffTable + 4 * table_ints) + 1024;
    return b > 118784 ? b : 118784;
  }
};

// mbarrier addresses, laid out back to back from `base`.
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t q_full() const { return base; }
  __device__ __forceinline__ uint32_t q_empty() const { return base + 8u; }
  __device__ __forceinline__ uint32_t k_full(int s) const { return base + 8u * (2 + s); }
  // K and V of a stage are released together, after the tile's last PV
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return base + 8u * (2 + kStages + s); }
  __device__ __forceinline__ uint32_t v_full(int s) const { return base + 8u * (2 + 2 * kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int u) const { return base + 8u * (2 + 3 * kStages + u); }
  __device__ __forceinline__ uint32_t p_full(int u) const { return base + 8u * (4 + 3 * kStages + u); }
  __device__ __forceinline__ uint32_t pv_done(int u) const { return base + 8u * (6 + 3 * kStages + u); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (8 + 3 * kStages); }
  __device__ __forceinline__ uint32_t item_full(int s) const { return base + 8u * (9 + 3 * kStages + s); }
  __device__ __forceinline__ uint32_t item_empty(int s) const {
    return base + 8u * (9 + 3 * kStages + kItemSlots + s);
  }
};

// ---- work schedule -----------------------------------------------------------------------
//
// A work item is one CTA's worth of work: a sequence b, a unit pair x (a head pair of a GQA
// group when the group size is even, otherwise a head) and a level z (the row tile, or the
// pair of row tiles, that the two units take).  In a persistent launch items are numbered
// sequence by sequence, longest sequence first, and within a sequence from its deepest level
// down, then by unit pair; the CTAs take them in that order from a shared counter, each
// taking the next item as soon as it has room for one.  Under a causal mask an item's cost
// grows with its level, so the first items are the longest and the ones that finish the
// launch are short; and the CTAs working at any time read the K/V of one or two sequences,
// which stay in L2 while every level of those sequences reads them.
struct Sched {
  int zmax;        // levels of the longest sequence (bounded by max_seqlen_q)
  int width;       // unit pairs per (sequence, level)
  int persistent;  // 1: the grid's CTAs take items from the counter; 0: CTA i runs item i of the dense grid
  int stage_off;   // byte offset of the output staging area from the aligned base; 0: none
};

// Levels of sequence b: its row tiles (two q heads per item) or row-tile pairs (one head per item).
__device__ __forceinline__ int levels_of(const FwdArgs& a, const Sched& sc, bool even, int b) {
  const int sq = a.cu_q[b + 1] - a.cu_q[b];
  const int nt = sq > 0 ? (sq + kBM - 1) / kBM : 0;
  const int nz = even ? nt : (nt + 1) / 2;
  return nz < sc.zmax ? nz : sc.zmax;
}

// In-place inclusive suffix sum over v[0, n) by one warp: v[i] becomes sum_{k >= i} v[k].
__device__ __forceinline__ void warp_suffix_sum(int* v, int n, int lane) {
  const int C = (n + 31) / 32;
  const int b0 = lane * C, b1 = (b0 + C < n) ? b0 + C : n;
  int tot = 0;
  for (int i = b0; i < b1; ++i) tot += v[i];
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += y;
  }
  int run = incl - tot;  // totals of the chunks above this lane's
  for (int i = b1 - 1; i >= b0; --i) {
    run += v[i];
    v[i] = run;
  }
  __syncwarp();
}

// Item table of a persistent launch, built by one warp of every CTA (identical in all of them):
//   start[j] = number of the first item of the j-th sequence of perm (start[j] = the total
//              item count for j >= the number of sequences with rows),
//   perm[j]  = the j-th sequence by descending level count (ties by index); sequences
//              without rows are left out,
// followed by two scratch arrays of the counting sort, cnt[z] (sequences with more than z
// levels) and run[z].  Table ints: (B + 1) + B + 2 Z.
constexpr long long table_ints(long long zmax, long long batch) { return 2 * batch + 1 + 2 * zmax; }
__device__ void build_table(const FwdArgs& a, const Sched& sc, bool even, int* tbl, int lane) {
  const int Z = sc.zmax, B = a.batch, W = sc.width;
  int* start = tbl;
  int* perm = tbl + B + 1;
  int* cnt = perm + B;
  int* run = cnt + Z;
  for (int i = lane; i < Z; i += 32) cnt[i] = run[i] = 0;
  __syncwarp();
  for (int b = lane; b < B; b += 32) {
    const int nz = levels_of(a, sc, even, b);
    if (nz > 0) atomicAdd(&cnt[nz - 1], 1);  // histogram: cnt[n - 1] = sequences with n levels
  }
  __syncwarp();
  warp_suffix_sum(cnt, Z, lane);             // cnt[z] = sequences with more than z levels
  // stable counting sort of the sequences by descending level count
  for (int c0 = 0; c0 < B; c0 += 32) {
    const int b = c0 + lane;
    const int nz = b < B ? levels_of(a, sc, even, b) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, nz);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (nz > 0) perm[(nz < Z ? cnt[nz] : 0) + run[nz - 1] + rank] = b;
    __syncwarp();
    if (nz > 0 && rank == 0) run[nz - 1] += __popc(peers);
    __syncwarp();
  }
  // start[]: exclusive prefix sums of the sorted sequences' item counts, from an inclusive
  // suffix sum: start[j] = total - sum_{k >= j} items(perm[k])
  const int P = Z > 0 ? cnt[0] : 0;          // sequences with rows
  for (int j = lane; j < P; j += 32) start[j] = W * levels_of(a, sc, even, perm[j]);
  __syncwarp();
  warp_suffix_sum(start, P, lane);
  const int total = P > 0 ? start[0] : 0;
  __syncwarp();
  for (int j = lane; j <= B; j += 32) start[j] = j < P ? total - start[j] : total;
  __syncwarp();
}

// The next item for this CTA: in a persistent launch the next number of the shared counter
// (every CTA's scheduler takes its items one at a time, so they come in increasing order);
// in grid mode CTA i runs item i only.
__device__ __forceinline__ long long next_item(const Sched& sc, unsigned* counter, int r) {
  if (!sc.persistent) return r == 0 ? (long long)blockIdx.x : -1;
  return (long long)atomicAdd(counter, 1u);
}

// Decodes item t into (b, x, z).  `cur` is a per-thread cursor over perm (the items of one
// CTA come in increasing order, so it only moves forward; start at 0).  Returns false past
// the last item, or for a grid-mode item whose sequence has no such level.
__device__ __forceinline__ bool decode_item(const FwdArgs& a, const Sched& sc, bool even, const int* tbl,
                                            long long t, int& cur, int& b, int& x, int& z) {
  if (t < 0) return false;
  const int W = sc.width;
  if (sc.persistent) {
    const int B = a.batch;
    const int* start = tbl;
    const int* perm = tbl + B + 1;
    if (t >= (long long)start[B]) return false;
    while (t >= (long long)start[cur + 1]) ++cur;
    const int r = (int)(t - start[cur]);
    const int lv = r / W;
    x = r - lv * W;
    b = perm[cur];
    z = levels_of(a, sc, even, b) - 1 - lv;
    return true;
  }
  const long long per_level = (long long)a.batch * W;
  const long long zr = t / per_level;
  if (zr >= sc.zmax) return false;
  const int rem = (int)(t - zr * per_level);
  z = sc.zmax - 1 - (int)zr;
  b = rem / W;
  x = rem - b * W;
  return z < levels_of(a, sc, even, b);
}

// One query unit of an item: q head, first row, rows, visible key range and the tiles of the
// item's key loop that meet it, [j0, j1).  Rows and keys are below 2^31 (packed totals are int).
struct Unit {
  int h, m0, nrows, lo, hi, j0, j1;
  bool valid;
};

// Everything a role needs about an item.
struct Item {
  int g;                  // kv head
  int q0, sq, k0, sk;     // sequence offsets and lengths
  int lo;                 // first key of the item's key loop
  int n_tiles;            // 128-key tiles in the loop (the union of the units' ranges)
  Unit un[2];
};

// align16: start the key loop at a multiple of 16 keys (dropout draws its keep bytes for
// 16-key blocks; the extra leading keys are masked like any invisible key).
__device__ __forceinline__ void setup_item(const FwdArgs& a, bool even, int group, int b, int x, int z,
                                           Item& it, bool align16 = false) {
  int hA, hB, mA, mB;
  if (even) {
    const int g_ = x / (group / 2), p_ = x % (group / 2);
    hA = g_ * group + 2 * p_;
    hB = hA + 1;
    mA = mB = z;
  } else {
    hA = hB = x;
    mA = 2 * z;
    mB = 2 * z + 1;
  }
  it.q0 = a.cu_q[b];
  it.sq = a.cu_q[b + 1] - it.q0;
  it.k0 = a.cu_k[b];
  it.sk = a.cu_k[b + 1] - it.k0;
  it.g = hA / group;
  const int hs[2] = {hA, hB}, ms[2] = {mA, mB};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    Unit& y = it.un[u];
    y.h = hs[u];
    y.m0 = ms[u] * kBM;
    y.valid = y.m0 < it.sq;
    y.nrows = y.valid ? ((it.sq - y.m0 < kBM) ? it.sq - y.m0 : kBM) : 0;
    y.lo = y.hi = 0;
    if (y.valid) {
      long long l1, h1, l2, h2;
      row_key_range(y.m0, it.sq, it.sk, a.left, a.right, l1, h1);
      row_key_range(y.m0 + y.nrows - 1, it.sq, it.sk, a.left, a.right, l2, h2);
      y.lo = (int)l1;
      y.hi = (int)(h2 < l1 ? l1 : h2);  // ranges move right with the row: the union is [lo(first), hi(last))
    }
  }
  int lo = it.un[0].lo, hi = it.un[0].hi;
  if (it.un[1].valid && it.un[1].hi > it.un[1].lo) {
    if (hi <= lo) { lo = it.un[1].lo; hi = it.un[1].hi; }
    else { lo = lo < it.un[1].lo ? lo : it.un[1].lo; hi = hi > it.un[1].hi ? hi : it.un[1].hi; }
  }
  if (align16 && hi > lo) lo &= ~15;
  it.lo = lo;
  it.n_tiles = hi > lo ? (hi - lo + kBN - 1) / kBN : 0;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    Unit& y = it.un[u];
    if (y.valid && y.hi > y.lo) {
      y.j0 = (y.lo - lo) / kBN;
      y.j1 = (y.hi - lo + kBN - 1) / kBN;
    } else {
      y.j0 = y.j1 = 0;
    }
  }
}

// An item as the scheduler warp hands it to the other roles (one 128-byte shared-memory slot).
struct ItemDesc {
  int kind;                  // 1: an item, 0: no more items
  int q0, sq, k0, sk;        // sequence offsets and lengths
  int lo, n_tiles, g;        // first key and 128-key tiles of the key loop, kv head
  int h[2], m0[2], j0[2], j1[2], valid[2];  // units A and B
  int pad[14];
};
static_assert(sizeof(ItemDesc) == 128, "item slot size");

// DV is the width of the PV product and of V's shared-memory tile (64 or 128); DVO <= DV is
// the width of v and out in memory.  With DVO = 32, V is loaded as a 64-column box over a
// 32-column tensor, whose columns 32-63 the copy fills with zeros, so O's columns 32-63 stay
// zero and only the first 32 are stored.
template <typename T, int DK, int DV, int DVO, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
fwd_sm100_kernel(const FwdArgs a, const Sched sc, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  using L = Layout<DK, DV>;
  extern __shared__ unsigned char smem_raw[];

  const int group = a.hq / a.hkv;
  const bool even = (group & 1) == 0;
  if (!sc.persistent) {
    // grid mode: a CTA whose item does not exist leaves before taking any resource
    int cur = 0, b, x, z;
    if (!decode_item(a, sc, even, nullptr, blockIdx.x, cur, b, x, z)) return;
  }
  const uint32_t base_u32 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base_u32 - smem_addr(smem_raw));
  const uint32_t sQ = base_u32 + L::kOffQ, sK = base_u32 + L::kOffK, sV = base_u32 + L::kOffV;
  const Bars bar{base_u32 + L::kOffBar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmemSlot);
  ItemDesc* items = reinterpret_cast<ItemDesc*>(smem + L::kOffItems);
  int* tbl = reinterpret_cast<int*>(smem + L::kOffTable);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full(), 1);
    mbar_init(bar.q_empty(), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar.k_full(s), 1);
      mbar_init(bar.kv_empty(s), 1);
      mbar_init(bar.v_full(s), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar.s_full(u), 1);
      mbar_init(bar.p_full(u), 4);   // one arrival per softmax warp of the unit
      mbar_init(bar.pv_done(u), 1);
    }
    for (int s = 0; s < kItemSlots; ++s) {
      mbar_init(bar.item_full(s), 1);
      mbar_init(bar.item_empty(s), kItemReaders);
    }
    mbar_init(bar.drain(), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2 && sc.persistent) build_table(a, sc, even, tbl, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0) {
    // ================================ TMA producer ======================================
    regs_dec<kRegsProducer>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int kv = 0, qn = 0;
      for (int r = 0;; ++r) {
        const int slot = r % kItemSlots;
        if (!mbar_wait(bar.item_full(slot), (r / kItemSlots) & 1, a.status)) break;
        const ItemDesc& d = items[slot];
        const int kind = d.kind, n = d.n_tiles, q0 = d.q0, k0 = d.k0, lo = d.lo, g = d.g;
        const int hA = d.h[0], hB = d.h[1], mA = d.m0[0], mB = d.m0[1], nq = d.valid[1] ? 2 : 1;
        mbar_arrive(bar.item_empty(slot));
        if (kind == 0) break;
        if (n == 0) continue;
        // the previous item's last QK has read Q
        if (!mbar_wait(bar.q_empty(), (qn & 1) ^ 1, a.status)) break;
        mbar_arrive_expect_tx(bar.q_full(), nq * L::kQBytes);
        for (int hf = 0; hf < L::KH; ++hf)
          tma_load_3d(sQ + hf * L::kHalfBytes, &tm_q, bar.q_full(), hf * 64, hA, q0 + mA);
        if (nq == 2)
          for (int hf = 0; hf < L::KH; ++hf)
            tma_load_3d(sQ + L::kQBytes + hf * L::kHalfBytes, &tm_q, bar.q_full(), hf * 64, hB, q0 + mB);
        ++qn;
        bool ok = true;
        for (int j = 0; j < n; ++j, ++kv) {
          const int st = kv % kStages;
          const uint32_t par = ((kv / kStages) & 1) ^ 1;
          const int row = k0 + lo + j * kBN;
          if (!(ok = mbar_wait(bar.kv_empty(st), par, a.status))) break;
          mbar_arrive_expect_tx(bar.k_full(st), L::kKBytes);
          for (int hf = 0; hf < L::KH; ++hf)
            tma_load_3d(sK + st * L::kKBytes + hf * L::kHalfBytes, &tm_k, bar.k_full(st), hf * 64, g, row);
          mbar_arrive_expect_tx(bar.v_full(st), L::kVBytes);
          for (int hf = 0; hf < L::VH; ++hf)
            tma_load_3d(sV + st * L::kVBytes + hf * L::kHalfBytes, &tm_v, bar.v_full(st), hf * 64, g, row);
        }
        if (!ok) break;
      }
      // make sure no copy is still landing in shared memory when the CTA exits
      if (qn > 0) mbar_wait(bar.q_full(), (qn - 1) & 1, a.status);
      for (int p = kv - kStages < 0 ? 0 : kv - kStages; p < kv; ++p) {
        mbar_wait(bar.k_full(p % kStages), (p / kStages) & 1, a.status);
        mbar_wait(bar.v_full(p % kStages), (p / kStages) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =========================================
    regs_dec<kRegsProducer>();
    // Without dropout the whole warp runs the issue loop in step (every lane computes the same
    // values and waits on the same barriers) and elect.sync picks the lane that issues each
    // MMA and commit, which costs the warp far less per MMA than a lone lane of a diverged
    // warp: +3% on the forward.  The dropout variant, whose softmax warps are busy with the
    // Philox draws, measured 1-7% slower that way and keeps the lone issuing lane.
    constexpr bool kElect = !DROP;
    if (kElect || lane == 0) {
      auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
        const bool done = mbar_wait(b, par, a.status);
        return kElect ? __all_sync(0xffffffffu, done) : done;
      };
      auto mma_ss_ = [&](uint32_t d, uint32_t al, uint32_t bl, uint32_t hi, uint32_t id, uint32_t acc) {
        if constexpr (kElect) mma_ss_lo_elect(d, al, bl, hi, id, acc);
        else mma_ss_lo(d, al, bl, hi, id, acc);
      };
      auto mma_ts_ = [&](uint32_t d, uint32_t at, uint32_t bl, uint32_t hi, uint32_t id, uint32_t acc) {
        if constexpr (kElect) mma_ts_lo_elect(d, at, bl, hi, id, acc);
        else mma_ts_lo(d, at, bl, hi, id, acc);
      };
      auto commit_ = [&](uint32_t b) {
        if constexpr (kElect) mma_commit_elect(b);
        else mma_commit(b);
      };
      constexpr uint32_t idesc_qk = idesc_of<T>(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_of<T>(kBM, DV, 0, 1);
      // Shared-memory descriptors, built once: an address offset is an addition to the start
      // field (addresses stay below 2^18 bytes, so the 14-bit field never carries).
      // All three share the high word (1024-byte stride, SW128), kept once in desc_hi.
      const uint64_t dQ0_ = smem_desc(sQ, 16, 1024, kLayoutSwizzle128B);
      const uint32_t desc_hi = (uint32_t)(dQ0_ >> 32);
      const uint32_t dQ0 = (uint32_t)dQ0_, dQ1 = dQ0 + (uint32_t)(L::kQBytes >> 4);
      const uint32_t dK0 = (uint32_t)smem_desc(sK, 16, 1024, kLayoutSwizzle128B);
      const uint32_t dV0 = (uint32_t)smem_desc(sV, L::kHalfBytes, 1024, kLayoutSwizzle128B);
      int kv = 0, qn = 0;
      int pcA = 0, pcB = 0;  // P tiles taken so far per unit (p_full phases)
      // Look-ahead across items: on an item's last tile the MMA thread peeks at the next item
      // (without releasing its ring slot, so the descriptor stays in place) and issues each
      // unit's QK of its tile 0 right after that unit's last PV; a unit's next S then does
      // not wait for the other unit's last softmax.  That Q was loaded once every QK of the
      // item had read Q; its K is the ring's next tile.
      bool qk0_issued = false;
      for (int r = 0;; ++r) {
        const int slot = r % kItemSlots;
        if (!wait_all(bar.item_full(slot), (r / kItemSlots) & 1)) break;
        const ItemDesc& d = items[slot];
        const int kind = d.kind, n = d.n_tiles;
        const int jA0 = d.j0[0], jA1 = d.j1[0], jB0 = d.j0[1], jB1 = d.j1[1];
        if (kElect) __syncwarp();
        if (lane == 0) mbar_arrive(bar.item_empty(slot));
        if (kind == 0) break;
        if (n == 0) continue;
        if (!qk0_issued) {
          if (!wait_all(bar.q_full(), qn & 1)) break;
          ++qn;
        }
        bool ok = true, nx_qk = false;
        int k_waited = -1;  // last tile of this item whose K load was waited for
        auto wait_k = [&](int j) -> bool {
          if (k_waited >= j) return true;
          const int p = kv + j;
          if (!wait_all(bar.k_full(p % kStages), (p / kStages) & 1)) return false;
          k_waited = j;
          return true;
        };
        // S_u(j) = Q_u K_j^T (j = n: tile 0 of the next item, whose K is ring tile kv + n).
        // S_u is overwritten while P_u (inside S_u) was read by the previous PV_u: MMAs issued
        // by one thread execute in issue order, so that read is done before this write.
        auto issue_qk = [&](int u, int j) -> bool {
          if (!wait_k(j)) return false;
          tc_fence_after();
          const int st = (kv + j) % kStages;
          const uint32_t dq = u ? dQ1 : dQ0, dk = dK0 + (uint32_t)(st * (L::kKBytes >> 4));
          const uint32_t dS = tmem + col_S(u);
#pragma unroll
          for (int ks = 0; ks < DK / 16; ++ks) {
            const uint32_t off16 = ((ks >> 2) * L::kHalfBytes + (ks & 3) * 32) >> 4;
            mma_ss_(dS, dq + off16, dk + off16, desc_hi, idesc_qk, ks > 0);
          }
          commit_(bar.s_full(u));
          return true;
        };
        // O_u += P_u(j) V_j (the first tile of the unit overwrites O_u)
        auto issue_pv = [&](int u, int j) -> bool {
          const int ph = u ? pcB + (j - jB0) : pcA + (j - jA0);
          if (!wait_all(bar.p_full(u), ph & 1)) return false;
          tc_fence_after();
          const int st = (kv + j) % kStages;
          const bool first = j == (u ? jB0 : jA0);
          const uint32_t dv = dV0 + (uint32_t)(st * (L::kVBytes >> 4));
          const uint32_t dO = tmem + col_O(u), aP = tmem + col_S(u);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts_(dO, aP + kk * 8, dv + (uint32_t)(kk * (2048 >> 4)), desc_hi, idesc_pv,
                            (!first || kk > 0) ? 1u : 0u);
          if (j + 1 == (u ? jB1 : jA1)) commit_(bar.pv_done(u));
          return true;
        };
        auto active = [&](int u, int j) { return u ? (j >= jB0 && j < jB1) : (j >= jA0 && j < jA1); };
        if (!qk0_issued)
          for (int u = 0; u < 2 && ok; ++u)
            if (active(u, 0)) ok = issue_qk(u, 0);
        if (!ok) break;
        qk0_issued = false;
        if (n == 1) commit_(bar.q_empty());  // every QK of the item is issued
        // V(j) is waited for one step ahead (while the previous QKs are still queued), so a
        // unit's P arrival finds this thread already waiting for it.
        if (!(ok = wait_all(bar.v_full(kv % kStages), (kv / kStages) & 1))) break;
        for (int j = 0; j < n && ok; ++j) {
          const int p = kv + j, st = p % kStages;
          for (int u = 0; u < 2 && ok; ++u) {
            if (active(u, j)) ok = issue_pv(u, j);
            if (!ok) break;
            if (u == 1) {
              commit_(bar.kv_empty(st));   // both PVs of tile j are issued: K and V of tile j are free
              if (j + 1 < n && !(ok = wait_all(bar.v_full((p + 1) % kStages), ((p + 1) / kStages) & 1))) break;
            }
            if (j + 1 < n) {
              if (active(u, j + 1)) ok = issue_qk(u, j + 1);
            } else {
              const int ns = (r + 1) % kItemSlots;
              if (u == 0) {
                if (!(ok = wait_all(bar.item_full(ns), ((r + 1) / kItemSlots) & 1))) break;
                nx_qk = items[ns].kind != 0 && items[ns].n_tiles > 0;
                // the next item's Q (loaded once this item's QKs completed)
                if (nx_qk && !(ok = wait_all(bar.q_full(), qn & 1))) break;
                qn += nx_qk ? 1 : 0;
              }
              if (nx_qk && items[ns].j0[u] == 0 && items[ns].j1[u] > 0) ok = issue_qk(u, n);
            }
          }
          if (!ok) break;
          if (j + 2 == n) commit_(bar.q_empty());  // the last QKs are issued
          if (j + 1 < n) {
            // a tile no unit needs still has to be consumed for the producer's accounting
            if (!(ok = wait_k(j + 1))) break;
          }
        }
        if (!ok) break;
        kv += n;
        pcA += jA1 - jA0;
        pcB += jB1 - jB0;
        qk0_issued = nx_qk;
      }
      // every MMA must be complete before the TMEM is freed
      commit_(bar.drain());
      wait_all(bar.drain(), 0);
    }
  } else if (warp == 2) {
    // ================================ scheduler ===========================================
    regs_dec<kRegsProducer>();
    if (lane == 0) {
      int cur = 0;
      for (int r = 0;; ++r) {
        const int slot = r % kItemSlots;
        if (!mbar_wait(bar.item_empty(slot), ((r / kItemSlots) & 1) ^ 1, a.status)) break;
        int b, x, z;
        const bool more = decode_item(a, sc, even, tbl, next_item(sc, a.work_counter, r), cur, b, x, z);
        ItemDesc& d = items[slot];
        d.kind = more ? 1 : 0;
        if (more) {
          Item it;
          setup_item(a, even, group, b, x, z, it, DROP);
          d.q0 = it.q0;
          d.sq = it.sq;
          d.k0 = it.k0;
          d.sk = it.sk;
          d.lo = it.lo;
          d.n_tiles = it.n_tiles;
          d.g = it.g;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            d.h[u] = it.un[u].h;
            d.m0[u] = it.un[u].m0;
            d.j0[u] = it.un[u].j0;
            d.j1[u] = it.un[u].j1;
            d.valid[u] = it.un[u].valid ? 1 : 0;
          }
        }
        mbar_arrive(bar.item_full(slot));  // release: the slot's writes are visible to the readers
        if (!more) break;
      }
    }
  } else if (warp == 3) {
    regs_dec<kRegsProducer>();   // no role, but part of the first warpgroup
  } else {
    // ================================ softmax warpgroups =================================
    regs_inc<kRegsSoftmax>();
    const int u = warp < 8 ? 0 : 1;
    const int lg = warp & 3;                      // TMEM lane quarter this warp may access
    const int r = lg * 32 + lane;                 // row within the unit
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_S(u), tO = tmem + lane_off + col_O(u);
    const float scale2 = a.scale * kLog2e;
    // the staged store moves 64-column (128-byte) row segments
    const uint32_t stg = (DVO % 64 == 0 && sc.stage_off) ? base_u32 + (uint32_t)sc.stage_off + (uint32_t)(warp - 4) * L::kStageBytes : 0u;
    int sc_u = 0;  // S tiles of this unit taken so far (s_full phases)
    int ic_u = 0;  // items in which this unit had tiles (pv_done phases)
    constexpr int kChunks = DVO / 32;
    // Epilogue of an item: out = O / (l + 2^{sink2 - m}),  lse = (m + log2 l) ln 2.  Without
    // dropout it is deferred to the unit's next item: after that item's first softmax the
    // warps read O (its first S being ready means every earlier PV of the unit is complete),
    // then announce P, and scale and store the old O while the next PV and QK run.
    constexpr bool kDefer = !DROP;
    bool pend = false;                        // an item's O waits in TMEM for its epilogue
    int e_h = 0, e_nrow = 0;                  // its head, rows of this warp that exist
    long long e_grow = 0;                     // packed row of this thread's query
    bool e_row = false;
    float e_inv = 0.f, e_lse = 0.f;
    T* const out = static_cast<T*>(a.out);
    // scale, convert and store 32 output columns (chunk cc) of the item in e_*
    auto emit = [&](const uint32_t (&o)[32], int cc) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack2<T>(__uint_as_float(o[2 * e]) * e_inv, __uint_as_float(o[2 * e + 1]) * e_inv);
      if (stg) {
        // Staged: the warp's 32 rows x 64 columns go through shared memory (16-byte chunk k
        // of row r at chunk k ^ (r % 8): no bank conflicts either way), and each store then
        // writes 4 rows x 128 contiguous bytes instead of 32 rows x 16 bytes.
#pragma unroll
        for (int v = 0; v < 4; ++v)
          st_shared_v4(stg + lane * 128 + ((((cc & 1) * 4 + v) ^ (lane & 7)) << 4), pk[4 * v], pk[4 * v + 1],
                       pk[4 * v + 2], pk[4 * v + 3]);
        if (cc & 1) {
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rr = 4 * k + (lane >> 3), ch = lane & 7;
            const uint4 w = ld_shared_v4(stg + rr * 128 + ((ch ^ (rr & 7)) << 4));
            const long long o0 = ((e_grow - lane + rr) * a.hq + e_h) * DVO + (cc >> 1) * 64 + ch * 8;
            if (rr < e_nrow && store_ok(o0, o0 + 7, (long long)a.total_q * a.hq * DVO, a.status))
              *reinterpret_cast<uint4*>(out + o0) = w;
          }
          __syncwarp();
        }
      } else if (e_row && store_ok((e_grow * a.hq + e_h) * DVO + cc * 32, (e_grow * a.hq + e_h) * DVO + cc * 32 + 31,
                                   (long long)a.total_q * a.hq * DVO, a.status)) {
        uint4* orow = reinterpret_cast<uint4*>(out + (e_grow * a.hq + e_h) * DVO);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          orow[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    };
    auto emit_lse = [&]() {
      // lse is [Hq, total_q]: the row itself must lie inside total_q
      if (e_row && a.lse && store_ok(e_grow, e_grow, a.total_q, a.status))
        a.lse[(long long)e_h * a.total_q + e_grow] = e_lse;
    };
    // The pending epilogue, when the next item does not take its deferred path: wait for the
    // unit's last PV (pv_done is committed once per item, after the unit's last PV), then
    // read O and store it.
    auto flush = [&]() -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(bar.pv_done(u), (ic_u - 1) & 1, a.status))) return false;
      tc_fence_after();
      uint32_t o[kChunks][32];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) tmem_ld32(tO + c * 32, o[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < kChunks; ++c) emit(o[c], c);
      emit_lse();
      tc_fence_before();
      pend = false;
      return true;
    };
    for (int it = 0;; ++it) {
      const int slot = it % kItemSlots;
      if (!__all_sync(0xffffffffu, mbar_wait(bar.item_full(slot), (it / kItemSlots) & 1, a.status))) break;
      const ItemDesc& d = items[slot];
      const int kind = d.kind, valid = d.valid[u], h = d.h[u], j0 = d.j0[u], j1 = d.j1[u];
      const int q0 = d.q0, sq = d.sq, sk = d.sk, klo0 = d.lo, i = d.m0[u] + r;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.item_empty(slot));
      if (kDefer && pend && (kind == 0 || !valid || j1 == j0) && !flush()) break;
      if (kind == 0) break;
      if (!valid) continue;
      const bool row_ok = i < sq;
      // this row's visible keys relative to the item's first key: [rlo, rhi) (empty if no row)
      int rlo = 0, rhi = 0;
      if (row_ok) {
        long long l_, h_;
        row_key_range(i, sq, sk, a.left, a.right, l_, h_);
        rlo = (int)(l_ - klo0);
        rhi = (int)(h_ - klo0);
      }
      float m = a.sink ? a.sink[h] * kLog2e : kNegInf, l = 0.f;
      const int ph = sc_u - j0;                   // s_full phase of tile j is ph + j
      bool ok = true;

      for (int j = j0; j < j1; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar.s_full(u), (ph + j) & 1, a.status))) { ok = false; break; }
        tc_fence_after();
        const int klo = rlo - j * kBN, khi = rhi - j * kBN;   // visible columns [klo, khi)
        const bool full = klo <= 0 && khi >= kBN;
        // the whole S row in one read (one TMEM round trip on the critical path)
        uint32_t sr[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        if (!full) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c < klo || c >= khi) sr[c] = __float_as_uint(kNegInf);
        }
        // row max over 8 independent chains of three-input maxima (a single chain would be
        // 128 dependent steps)
        float mxv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mxv[e] = fmaxf(__uint_as_float(sr[e]), __uint_as_float(sr[8 + e]));
#pragma unroll
        for (int c = 16; c < kBN; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            mxv[e] = fmax3(mxv[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e]));
        const float mx = fmax3(fmax3(mxv[0], mxv[1], mxv[2]), fmax3(mxv[3], mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7]));
        const float m_tile = mx * scale2;
        const bool need = m_tile > m + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = (m == kNegInf) ? 0.f : ex2(m - m_tile);
          m = m_tile;
        }
        const bool any_rescale = __any_sync(0xffffffffu, need);
        // P = 2^{S scale log2e - m} as bf16, over S columns already read, 64 keys at a time.
        // Masked scores are -inf and 2^-inf = +0, so they need no test; m = -inf only when
        // every score is -inf (then neg_m = 0 keeps the argument -inf, not NaN).
        const float neg_m = (m == kNegInf) ? 0.f : -m;
        // two columns per packed multiply-add and per packed sum update
        const float2 sc2 = make_float2(scale2, scale2), nm2 = make_float2(neg_m, neg_m);
        const uint32_t t4 = (a.drop.threshold - 1u) * 0x01010101u, t4h = t4 | 0x80808080u;
        float2 sv[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[32];
          // dropout: drop flags of this half's four 16-key blocks (the key loop starts at a
          // multiple of 16); the row sum keeps every probability, the P V operand only the
          // kept ones (the 256 / T scale is applied to the output)
          uint32_t fl[DROP ? 16 : 1];
          if constexpr (DROP) {
            const uint32_t kb0 = (uint32_t)(klo0 + j * kBN + hh * 64) >> 4;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
              const uint4 w = dropout_bytes(a.drop, kb0 + gq, (uint32_t)(q0 + i), (uint32_t)h);
              fl[4 * gq] = drop_flags4(w.x, t4, t4h);
              fl[4 * gq + 1] = drop_flags4(w.y, t4, t4h);
              fl[4 * gq + 2] = drop_flags4(w.z, t4, t4h);
              fl[4 * gq + 3] = drop_flags4(w.w, t4, t4h);
            }
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 x = ffma2(make_float2(__uint_as_float(sr[hh * 64 + 2 * c]), __uint_as_float(sr[hh * 64 + 2 * c + 1])),
                                   sc2, nm2);
            const float2 pp = make_float2(ex2(x.x), ex2(x.y));
            sv[c & 1] = fadd2(sv[c & 1], pp);
            pk[c] = pack2<T>(pp.x, pp.y);
            if constexpr (DROP) {
              // keys 2c, 2c + 1 are bytes 0-1 (c even) or 2-3 (c odd) of flag word c / 2:
              // widen their flags to the two 16-bit halves and clear the dropped ones
              const uint32_t mask = (c & 1) ? prmt_sign<0xBBAA>(fl[c >> 1]) : prmt_sign<0x9988>(fl[c >> 1]);
              pk[c] &= ~mask;
            }
          }
          tmem_st32(tS + hh * 32, pk);
        }
        const float sum = (sv[0].x + sv[0].y) + (sv[1].x + sv[1].y);
        l = l * alpha + sum;

        if (any_rescale && j > j0) {
          // O holds sum of the earlier P V: wait for the last of those MMAs, then scale rows
          // S(j) being ready means PV(j - 1) is complete (one issuing thread, commits in order)
#pragma unroll
          for (int c = 0; c < DVO / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        if (kDefer && pend) {
          // the previous item's O, before this announcement lets PV(j0) overwrite it
          uint32_t o[kChunks][32];
#pragma unroll
          for (int c = 0; c < kChunks; ++c) tmem_ld32(tO + c * 32, o[c]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.p_full(u));
#pragma unroll
          for (int c = 0; c < kChunks; ++c) emit(o[c], c);
          emit_lse();
          pend = false;
          continue;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(u));
      }
      if (!ok) break;

      // ---- epilogue (see emit): record this item's output state -------------------------
      const bool have_o = j1 > j0;
      sc_u += j1 - j0;
      ic_u += have_o ? 1 : 0;
      {
        const float sink2 = a.sink ? a.sink[h] * kLog2e : kNegInf;
        const float e_sink = (sink2 == kNegInf || m == kNegInf) ? 0.f : ex2(sink2 - m);
        const float den = l + e_sink;
        // with dropout, O summed the kept probabilities unscaled: the 256 / T factor goes here
        e_inv = den > 0.f ? (DROP ? a.drop.scale : 1.f) / den : 0.f;
        e_lse = l > 0.f ? (m + __log2f(l)) * kLn2 : kNegInf;
        e_h = h;
        e_grow = (long long)q0 + i;
        e_row = row_ok;
        e_nrow = sq - (i - lane);   // rows of this warp (queries i - lane ..) that exist
      }
      if (kDefer && have_o) {
        pend = true;
        continue;
      }
      if (have_o) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar.pv_done(u), (ic_u - 1) & 1, a.status))) break;
        tc_fence_after();
      }
      // O 32 columns at a time with dropout (whose flag words take the room), else at once
      constexpr int kPer = DROP ? 1 : kChunks;
#pragma unroll
      for (int c0 = 0; c0 < kChunks; c0 += kPer) {
        uint32_t o[kPer][32];
        if (have_o) {
#pragma unroll
          for (int c = 0; c < kPer; ++c) tmem_ld32(tO + (c0 + c) * 32, o[c]);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < kPer; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) o[c][e] = 0u;
        }
#pragma unroll
        for (int c = 0; c < kPer; ++c) emit(o[c], c0 + c);
      }
      emit_lse();
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host: tensor maps and launch ----------------------------------------------------------

// Multiprocessors and opt-in shared memory per block of the current device (cached per device).
struct DeviceShape {
  int sms = 0, smem_optin = 0;
};
constexpr int kMaxDevices = 64;
DeviceShape g_shape[kMaxDevices];

cudaError_t device_shape(DeviceShape& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceShape& d = g_shape[dev];
  if (d.sms == 0) {
    int sms = 0, optin = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    d.smem_optin = optin;
    d.sms = sms;
  }
  out = d;
  return cudaSuccess;
}

// Levels of the longest sequence and unit pairs per level (see Sched).
void schedule_shape(const FwdArgs& a, int& zmax, int& width) {
  const int mtiles = (a.max_sq + kBM - 1) / kBM;
  const int group = a.hq / a.hkv;
  const bool even = group % 2 == 0;
  zmax = even ? mtiles : (mtiles + 1) / 2;
  width = even ? a.hq / 2 : a.hq;
}


template <typename T, int DK, int DV, int DVO = DV>
cudaError_t launch_typed(const FwdArgs& a, cudaStream_t s) {
  using L = Layout<DK, DV>;
  int zmax, width;
  schedule_shape(a, zmax, width);
  if (zmax <= 0) return cudaSuccess;  // no query rows
  DeviceShape dev;
  cudaError_t e = device_shape(dev);
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  constexpr CUtensorMapDataType dt = tma_dtype<T>();
  if (!make_map_3d(&tq, a.q, DK, a.hq, a.total_q, 128, dt) || !make_map_3d(&tk, a.k, DK, a.hkv, a.total_k, 128, dt) ||
      !make_map_3d(&tv, a.v, DVO, a.hkv, a.total_k, 128, dt))
    return cudaErrorInvalidValue;
  // Persistent launch (one CTA per SM walking the item list) when the item table fits in
  // shared memory; otherwise one CTA per item of the dense (level, sequence, unit pair) grid.
  const long long items_ub = (long long)zmax * a.batch * width;
  // The output staging area goes in when it fits beside the table (else rows are stored
  // directly from registers).
  const long long tbl = table_ints(zmax, a.batch);
  Sched sc{zmax, width, 1, 0};
  long long smem;
  constexpr bool kStageable = DVO % 64 == 0;
  if (kStageable && L::smem_bytes(tbl, true) <= dev.smem_optin) {
    sc.stage_off = (int)L::stage_offset(tbl);
    smem = L::smem_bytes(tbl, true);
  } else if (L::smem_bytes(tbl, false) <= dev.smem_optin) {
    smem = L::smem_bytes(tbl, false);
  } else {
    sc.persistent = 0;
    const bool st = kStageable && L::smem_bytes(0, true) <= dev.smem_optin;
    sc.stage_off = st ? (int)L::stage_offset(0) : 0;
    smem = L::smem_bytes(0, st);
  }
  const long long grid = sc.persistent ? (items_ub < dev.sms ? items_ub : dev.sms) : items_ub;
  if (sc.persistent) {
    // the shared item counter starts at zero for every launch
    if (a.work_counter == nullptr) return cudaErrorInvalidValue;
    if ((e = cudaMemsetAsync(a.work_counter, 0, sizeof(unsigned), s)) != cudaSuccess) return e;
  }
  auto kernel = a.drop.threshold ? fwd_sm100_kernel<T, DK, DV, DVO, true> : fwd_sm100_kernel<T, DK, DV, DVO, false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kernel<<<(unsigned)grid, kThreads, (size_t)smem, s>>>(a, sc, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace

bool fwd_sm100_supported(const FwdArgs& a, int dtype) {
  if ((dtype != 0 && dtype != 2) || a.cu_q == nullptr) return false;
  if (!((a.dk == 64 || a.dk == 128) && (a.dv == 32 || a.dv == 64 || a.dv == 128))) return false;
  int zmax, width;
  schedule_shape(a, zmax, width);
  if ((long long)zmax * a.batch * width > 0x7fffffffLL) return false;  // item numbers are 32-bit
  return encode_fn() != nullptr;
}

namespace {
template <typename T>
cudaError_t launch_dims(const FwdArgs& a, cudaStream_t s) {
  if (a.dk == 128 && a.dv == 128) return launch_typed<T, 128, 128>(a, s);
  if (a.dk == 128 && a.dv == 64) return launch_typed<T, 128, 64>(a, s);
  if (a.dk == 64 && a.dv == 64) return launch_typed<T, 64, 64>(a, s);
  if (a.dk == 64 && a.dv == 128) return launch_typed<T, 64, 128>(a, s);
  // dv = 32: a 64-wide PV over zero-filled V columns
  if (a.dk == 64 && a.dv == 32) return launch_typed<T, 64, 64, 32>(a, s);
  if (a.dk == 128 && a.dv == 32) return launch_typed<T, 128, 64, 32>(a, s);
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_fwd_sm100(const FwdArgs& a, int dtype, cudaStream_t s) {
  return dtype == 2 ? launch_dims<__half>(a, s) : launch_dims<__nv_bfloat16>(a, s);
}

}  // namespace attn_sink
