// Attention decoding against a paged KV cache for sm_100a.
//
// The new tokens of each sequence attend to its cached keys and values, which
// live in fixed-size pages reached through a per-sequence page table
// ("Efficient attention: long context and sub-quadratic variants",
// stanleyjacob.dev, section "FlashAttention: exact attention, IO-aware",
// PagedAttention paragraph; "Efficient Attention", giftedprocrastinator.com,
// section "What it does", KV-cache paragraph).  The result is the same exact
// masked softmax attention as the forward; only the new tokens are queries.
//
// A decoding step streams every visible cached key and value once and does
// little arithmetic per byte, so the kernel is built to keep HBM busy:
//
// * Work item = (sequence b, KV head, chunk of the group's query rows, split
//   s of the visible key range).  Splits spread one long sequence over many
//   SMs; a second kernel merges the splits' partial results by their
//   log-sum-exp.  One persistent CTA per SM takes items from a shared
//   counter as it finishes the previous one, so sequences of different
//   lengths balance across SMs.
// * The group's query rows (Hq/Hkv heads x Nq new tokens, at most 128) form
//   the 128-lane M dimension of the tcgen05 MMAs.  With R rows the rows are
//   replicated into 128 / (32 * WC) copies (WC = warps per copy = ceil(R/32)
//   rounded to a power of two), and copy c handles only key columns
//   [c*C, c*C + C) of every 128-key tile (C = 32 * WC): each copy runs its own
//   online softmax over its share of the keys, so the exponentials of a step
//   are spread over all four softmax warps even for one query row.  The
//   copies' partial (max, sum, O) are merged in shared memory at the end of
//   the item.  P of a copy is written only into its own key columns of a P
//   buffer whose other columns stay zero, so one O += P V MMA sums exactly
//   each copy's own keys.
// * K and V tiles are gathered page by page with TMA (one box of
//   min(page_size, 128) rows per page and 64-column chunk), issued by the
//   loader warp's lanes in parallel; the page-table entries are read one tile
//   ahead.  Boxes that hold no position of the step's visible range are not
//   loaded at all; under a sliding window the pages wholly before the oldest
//   visible key are never looked up, so a caller may recycle them (a rolling
//   window buffer).  Rows of an edge tile outside the visible range are
//   cleared in shared memory before the P V MMA (those slots may hold
//   anything), and masked scores are replaced by -inf.
//
// CTA organisation (224 threads): warps 0-3 softmax (thread = TMEM lane),
// warp 4 TMA loader for the work items, Q and K, warp 5 tcgen05 issuer, warp 6
// TMA loader for V (small pages cost one TMA box each; two issuing warps keep
// the K and V boxes of a tile going out together).  TMEM: S double buffer at columns
// [0,128) and [128,256), P double buffer (bf16 pairs) at [256,320) and
// [320,384), O at [384, 384 + d).  All waits are bounded like the forward's.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace attn_sm100_dec {
using namespace attn_sm100;

constexpr int kKeys = 128;           // keys per K/V tile
constexpr int kLanes = 128;          // query-row lanes of one work item
constexpr int kDecThreads = 224;
constexpr int kDecLoaderWarp = 4;   // work items, Q and K
constexpr int kDecMmaWarp = 5;
constexpr int kDecVLoaderWarp = 6;  // V
constexpr uint32_t kDecTmemCols = 512;
constexpr float kDecLn2 = 0.6931471805599453f;
// A lane's running max moves only when it grows by more than 2^32 (as in the
// forward): P may then exceed 1 by up to 2^32, which bf16 P and fp32 sums and
// accumulators carry without loss, and the final merge uses the same maxima.
constexpr float kDecRescaleThreshold = 32.0f;
// Work items are handed out by a counter in global memory; the loader fetches
// them and passes each index to the other roles through this many slots.
constexpr int kItemSlots = 4;

enum : int { kDMaskFull = 0, kDMaskCausal = 1, kDMaskWindow = 2 };
enum : int { kDRoleLoader = 1, kDRoleMma = 2, kDRoleSoftmax = 3 };
// Data errors recorded in the error word (bits 20..21; low bits: sequence index).
constexpr int kDErrSeqLen = 1 << 20;   // seq_lens[b] < Nq or beyond the page table
constexpr int kDErrPage = 2 << 20;     // a page-table entry the step needs is out of range

struct DecParams {
  CUtensorMap tm_q;       // [1, B*Hq*Nq, d] bf16, box 64 x rows_chunk, 128-byte swizzle
  CUtensorMap tm_k;       // [num_pages*Hkv][d/64][page_size][64] view, box 64 x rows_per_load x d/64 x 1
  CUtensorMap tm_v;
  const int* block_table; // [B, max_pages]
  const int* seq_lens;    // [B]
  __nv_bfloat16* out;     // [B*Hq*Nq, d]
  float* lse;             // [B*Hq*Nq]
  float* part_o;          // [B*Hq*Nq, num_splits, d] (num_splits > 1)
  float* part_lse;        // [B*Hq*Nq, num_splits], base-2 units (num_splits > 1)
  int* err;
  int B, Hq, Hkv, Nq, group;
  int rows_total;         // group * Nq query rows per (b, KV head)
  int rows_chunk;         // query rows per work item (<= 128)
  int row_chunks;         // ceil(rows_total / rows_chunk)
  int page_size, rows_per_load, loads_per_tile, max_pages, num_pages;
  int mask_kind, window;
  int num_splits, num_items;
  float scale_log2;       // scale * log2(e)
  unsigned long long timeout_ns;
  unsigned int* sched;    // [0] next work item, [1] CTAs finished; zero between launches
};

template <int D>
struct DecSmem {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kChunkBytes = kKeys * 128;           // 128 rows x 128 B
  static constexpr uint32_t kTileBytes = kChunks * kChunkBytes;  // Q, K or V tile
  static constexpr int kStages = (D == 128) ? 5 : 10;            // K/V ring slots
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kRingOff = kTileBytes;
  static constexpr uint32_t kScratchOff = kRingOff + kStages * kTileBytes;  // [128 lanes][33] fp32
  static constexpr uint32_t kLaneOff = kScratchOff + 33 * kLanes * 4;       // m, l per lane
  static constexpr uint32_t kRowOff = kLaneOff + 2 * kLanes * 4;            // M, l_total per row
  static constexpr uint32_t kBarOff = kRowOff + 2 * kLanes * 4;
  static constexpr int kQFull = 0;
  static constexpr int kQEmpty = 1;
  static constexpr int kKVFull = 2;
  static constexpr int kKVEmpty = kKVFull + kStages;
  static constexpr int kSFull = kKVEmpty + kStages;   // x2
  static constexpr int kPFull = kSFull + 2;           // x2
  static constexpr int kPVDone = kPFull + 2;          // every P V (waited on only before an O rescale)
  static constexpr int kODone = kPVDone + 1;          // an item's last P V
  static constexpr int kOFree = kODone + 1;
  static constexpr int kEpi = kOFree + 1;             // softmax warps' own barrier
  static constexpr int kFin = kEpi + 1;
  static constexpr int kItemFull = kFin + 1;          // x kItemSlots
  static constexpr int kItemEmpty = kItemFull + kItemSlots;
  static constexpr int kNumBars = kItemEmpty + kItemSlots;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kItemOff = kMiscOff + 16;  // kItemSlots work-item indices
  static constexpr uint32_t kBytes = kItemOff + 4 * kItemSlots;
  static constexpr uint32_t kAlloc = kBytes + 1024;   // slack to align the base to 1024 B
  static constexpr uint32_t kSCol = 0;                // + 128 * buffer
  static constexpr uint32_t kPCol = 256;              // + 64 * buffer
  static constexpr uint32_t kOCol = 384;
};

// ------------------------------------------------------------ work items
struct DecItem {
  int b, hkv, rc, s;
  int L;        // cached keys of the sequence
  int lo_pos;   // oldest position any query of the step can see
  int t0, t1;   // tile range of this split (empty when t1 < t0)
  int row0;     // first query row of the group handled here
  int rows;     // rows handled here
  bool bad;     // seq_lens[b] unusable: the item is empty and reports an error
};

__device__ __forceinline__ DecItem dec_item(const DecParams& p, int idx) {
  DecItem it;
  it.s = idx % p.num_splits;
  idx /= p.num_splits;
  it.rc = idx % p.row_chunks;
  idx /= p.row_chunks;
  it.hkv = idx % p.Hkv;
  it.b = idx / p.Hkv;
  it.L = __ldg(p.seq_lens + it.b);
  it.bad = it.L < p.Nq || it.L > p.max_pages * p.page_size;
  it.row0 = it.rc * p.rows_chunk;
  it.rows = min(p.rows_chunk, p.rows_total - it.row0);
  it.lo_pos = 0;
  it.t0 = 0;
  it.t1 = -1;
  if (!it.bad) {
    if (p.mask_kind == kDMaskWindow) it.lo_pos = max(0, it.L - p.Nq - p.window + 1);
    const int first = it.lo_pos / kKeys, last = (it.L - 1) / kKeys;
    const int chunk = (last - first + p.num_splits) / p.num_splits;  // ceil(tiles / splits)
    it.t0 = first + it.s * chunk;
    it.t1 = min(last, it.t0 + chunk - 1);
  }
  return it;
}

// Bounded mbarrier waits (same contract as the forward's).
struct DecWaiter {
  uint64_t limit_ns;
  volatile int* abort_flag;
  int* err;
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, int code) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
      if (mbar_try_wait(bar, parity)) return true;
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        atomicCAS(err, 0, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
  __device__ __forceinline__ bool drain(uint32_t bar, uint32_t parity, int code) const {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (global_timer_ns() - t0 > limit_ns) {
        atomicCAS(err, 0, code);
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  }
  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, int code) const {
    return __all_sync(0xffffffffu, wait(bar, parity, code));
  }
};

// 4-D tiled load global -> shared (one page box: both 64-column halves of
// rows_per_load rows), completing its bytes on the mbarrier.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z,
                                            int w, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w), "l"(policy)
      : "memory");
}

__device__ __forceinline__ float dec_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t dec_pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Next work item of this CTA for a consuming role (every lane of the warp
// calls it): the index the loader published in the next slot, or -1 if the
// CTA aborts.  One lane per warp frees the slot after the warp has read it.
template <int D>
__device__ __forceinline__ int dec_take_item(uint32_t sbase, const uint8_t* smem, const DecWaiter& w, uint32_t& k,
                                             int code) {
  using L = DecSmem<D>;
  const uint32_t slot = k % kItemSlots;
  const uint32_t full = sbase + L::kBarOff + 8u * (L::kItemFull + slot);
  if (!w.wait_warp(full, (k / kItemSlots) & 1, code | (L::kItemFull + slot))) return -1;
  const int idx = *reinterpret_cast<const volatile int*>(smem + L::kItemOff + 4 * slot);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(sbase + L::kBarOff + 8u * (L::kItemEmpty + slot));
  ++k;
  return idx;
}

// ------------------------------------------------------------ roles
// Loader warps: tile t of the CTA's g-th tile overall goes to ring index 2g
// (K, loader warp 4) and 2g + 1 (V, loader warp 6).  Lane i < loads_per_tile
// copies the tile's rows [i*R, i*R + R) (R = rows_per_load) from the page
// holding them; lane 0 sets the expected bytes.  Warp 4 also fetches the work
// items and loads Q; warp 6 takes the items from it like the other roles.
template <int D, int WC, bool kV>
__device__ __forceinline__ uint32_t dec_loader(const DecParams& p, uint32_t sbase, uint8_t* smem, const DecWaiter& w) {
  using L = DecSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const int lane = threadIdx.x & 31;
  const uint64_t pol = l2_policy_evict_first();  // every cached byte is read once per step
  if (lane == 0) {
    tma_prefetch_map(&p.tm_q);
    tma_prefetch_map(&p.tm_k);
    tma_prefetch_map(&p.tm_v);
  }
  const int code = kDRoleLoader << 8;
  constexpr int kCopies = 4 / WC;   // replicas of the item's query rows
  constexpr int kRpc = 32 * WC;     // TMEM lanes per replica
  uint32_t gt = 0, q_n = 0, k_item = 0;  // tiles this CTA has loaded, Q loads, items taken
  bool ok = true;
  // Work items come from the shared counter, one ahead of use so that the
  // atomic's latency overlaps the current item; each index is published to
  // the other roles before the item's loads start.
  int next = 0;
  if (!kV && lane == 0) next = static_cast<int>(atomicAdd(p.sched, 1u));
  while (ok) {
    int idx;
    if constexpr (kV) {
      idx = dec_take_item<D>(sbase, smem, w, k_item, code);
      if (idx < 0) break;
    } else {
      const uint32_t slot_i = k_item % kItemSlots;
      if (k_item >= (uint32_t)kItemSlots &&
          !w.wait_warp(bar(L::kItemEmpty + slot_i), ((k_item / kItemSlots) - 1) & 1, code | (L::kItemEmpty + slot_i)))
        break;
      idx = __shfl_sync(0xffffffffu, next, 0);
      if (lane == 0) {
        *reinterpret_cast<volatile int*>(smem + L::kItemOff + 4 * slot_i) = idx < p.num_items ? idx : -2;
        mbar_arrive(bar(L::kItemFull + slot_i));
      }
      ++k_item;
      if (idx >= p.num_items) break;
      if (lane == 0) next = static_cast<int>(atomicAdd(p.sched, 1u));
    }
    const DecItem it = dec_item(p, idx);
    if (it.t1 < it.t0) continue;
    const int* trow = p.block_table + static_cast<size_t>(it.b) * p.max_pages;
    // Page-table entry of this lane's box in tile t, or -1 when the box holds
    // no position of [lo_pos, L) (then nothing is loaded and the table entry
    // is not read).  The entries are read two tiles ahead and checked only
    // when used, so the table's load latency stays off the issue path.
    auto box_entry = [&](int t) -> int {
      if (t > it.t1 || lane >= p.loads_per_tile) return -1;
      const int pos0 = t * kKeys + lane * p.rows_per_load;
      if (pos0 >= it.L || pos0 + p.rows_per_load <= it.lo_pos) return -1;
      return __ldg(trow + pos0 / p.page_size);
    };
    auto checked = [&](int t, int entry) -> int {
      const int pos0 = t * kKeys + lane * p.rows_per_load;
      if (lane >= p.loads_per_tile || pos0 >= it.L || pos0 + p.rows_per_load <= it.lo_pos) return -1;
      if (entry < 0 || entry >= p.num_pages) {
        atomicCAS(p.err, 0, kDErrPage | (it.b & 0xFFFFF));
        return 0;  // stand-in inside the pool; the step's result is then undefined
      }
      return entry;
    };
    auto issue = [&](int t, int kv, int page) -> bool {
      const uint32_t ring_idx = 2 * gt + kv;
      const uint32_t slot = ring_idx % L::kStages;
      if (ring_idx >= (uint32_t)L::kStages &&
          !w.wait_warp(bar(L::kKVEmpty + slot), ((ring_idx / L::kStages) - 1) & 1, code | (L::kKVEmpty + slot)))
        return false;
      const unsigned boxes = __ballot_sync(0xffffffffu, page >= 0);
      if (lane == 0)
        mbar_arrive_expect_tx(bar(L::kKVFull + slot),
                              __popc(boxes) * static_cast<uint32_t>(p.rows_per_load) * 128u * L::kChunks);
      __syncwarp();
      if (page >= 0) {
        const int y = (t * kKeys + lane * p.rows_per_load) % p.page_size;  // 0 unless pages exceed a tile
        const int z = page * p.Hkv + it.hkv;
        const uint32_t tile = sbase + L::kRingOff + slot * L::kTileBytes;
        if (kv) {
          // V: one box per page, both column halves, stored half after half
          // ([half][R rows][128 B], the page's block of the tile).
          tma_load_4d(tile + lane * p.rows_per_load * 128 * L::kChunks, &p.tm_v, bar(L::kKVFull + slot), 0, y, 0, z,
                      pol);
        } else {
          // K: one box per page and column half into the [half][128 rows]
          // tile that a single N = 128 product reads.
#pragma unroll
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(tile + c * L::kChunkBytes + lane * p.rows_per_load * 128, &p.tm_k, bar(L::kKVFull + slot), 0,
                        y, c, z, pol);
        }
      }
      return true;
    };
    int e0 = box_entry(it.t0), e1 = box_entry(it.t0 + 1);
    for (int t = it.t0; t <= it.t1; ++t) {
      const int e2 = box_entry(t + 2);
      const int pg = checked(t, e0);
      if (!issue(t, kV ? 1 : 0, pg)) {
        ok = false;
        break;
      }
      ++gt;
      if (!kV && t == it.t0) {
        // Q of the item, once the previous item's last S has read the buffer:
        // one box of rows_chunk rows per copy and 64-column chunk.
        if (q_n > 0 && !w.wait_warp(bar(L::kQEmpty), (q_n - 1) & 1, code | L::kQEmpty)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(L::kQFull), kCopies * L::kChunks * static_cast<uint32_t>(p.rows_chunk) * 128u);
          const int y = (it.b * p.Hq + it.hkv * p.group) * p.Nq + it.row0;
          for (int cp = 0; cp < kCopies; ++cp)
#pragma unroll
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_3d(sbase + L::kQOff + c * L::kChunkBytes + cp * kRpc * 128, &p.tm_q, bar(L::kQFull), c * 64, y,
                          0, pol);
        }
        __syncwarp();
        ++q_n;
      }
      e0 = e1;
      e1 = e2;
    }
  }
  // Drain this warp's Q copies; the K/V ring is drained after both loaders
  // are done (dec_drain_ring), since the two warps take turns on every slot.
  if (lane == 0 && q_n > 0) w.drain(bar(L::kQFull), (q_n - 1) & 1, code | L::kQFull);
  __syncwarp();
  return gt;
}

// Every K/V copy must land before the CTA exits.  A slot is loaded again only
// after its previous load landed and was consumed, so at most its last load
// can still be in flight: wait for that one (ring index 2g for K, 2g + 1 for V).
template <int D>
__device__ __forceinline__ void dec_drain_ring(uint32_t sbase, const DecWaiter& w, uint32_t gt_k, uint32_t gt_v) {
  using L = DecSmem<D>;
  for (uint32_t s = 0; s < (uint32_t)L::kStages; ++s) {
    int64_t last = -1;
    for (uint32_t back = 0; back < (uint32_t)L::kStages; ++back) {
      if (back < gt_k && (2 * (gt_k - 1 - back)) % L::kStages == s) last = max(last, int64_t(2 * (gt_k - 1 - back)));
      if (back < gt_v && (2 * (gt_v - 1 - back) + 1) % L::kStages == s)
        last = max(last, int64_t(2 * (gt_v - 1 - back) + 1));
    }
    if (last >= 0)
      w.drain(sbase + L::kBarOff + 8u * (L::kKVFull + s), (uint32_t(last) / L::kStages) & 1,
              (kDRoleLoader << 8) | (L::kKVFull + s));
  }
}

// MMA warp: per item S_0, then for each tile j: S_{j+1} (look-ahead into the
// other S buffer) and O += P_j V_j once the softmax has published P_j.  S_j is
// always issued after P V of tile j-2 (in-order completion then makes "S_j
// done" imply "P V_{j-2} done"), whichever of S_{j+1} and P V_j goes first.
template <int D>
__device__ __forceinline__ void dec_mma(const DecParams& p, uint32_t sbase, const uint8_t* smem, uint32_t tmem,
                                        const DecWaiter& w) {
  using L = DecSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr uint32_t idesc_s = idesc_bf16_f32(kLanes, kKeys, false);
  constexpr uint32_t idesc_o = idesc_bf16_f32(kLanes, D, true);
  const uint64_t q_desc = smem_desc_sw128(sbase + L::kQOff, 16, 1024);
  // A K tile is [half][128 rows][128 B]; a V tile is 128 / R page blocks of
  // [half][R rows][128 B] (R = rows_per_load), which for one column half or
  // R = 128 is the same thing.
  const int R = p.rows_per_load;
  const uint32_t box_bytes = static_cast<uint32_t>(R) * 128u * L::kChunks;
  const uint64_t k_desc0 = smem_desc_sw128(sbase + L::kRingOff, 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(sbase + L::kRingOff, static_cast<uint32_t>(R) * 128u, 1024);
  const uint32_t o_tmem = tmem + L::kOCol;
  const int code = kDRoleMma << 8;
  uint32_t g = 0, q_n = 0, items = 0, k_item = 0;
  bool ok = true;
  while (ok) {
    const int idx = dec_take_item<D>(sbase, smem, w, k_item, code);
    if (idx < 0) break;
    const DecItem it = dec_item(p, idx);
    if (it.t1 < it.t0) continue;
    const int n = it.t1 - it.t0 + 1;
    if (!w.wait_warp(bar(L::kQFull), q_n & 1, code | L::kQFull)) break;
    ++q_n;
    tc_fence_after_sync();
    auto issue_s = [&](int j) -> bool {
      const uint32_t gi = g + j, kidx = 2 * gi, kslot = kidx % L::kStages;
      if (!w.wait_warp(bar(L::kKVFull + kslot), (kidx / L::kStages) & 1, code | (L::kKVFull + kslot))) return false;
      tc_fence_after_sync();
      const uint32_t s_tmem = tmem + L::kSCol + 128 * (gi & 1);
      const uint64_t kd = k_desc0 + ((kslot * L::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
        mma_bf16_ss_elect(s_tmem, q_desc + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
      }
      tc_commit_elect(bar(L::kSFull + (gi & 1)));
      tc_commit_elect(bar(L::kKVEmpty + kslot));
      if (j == n - 1) tc_commit_elect(bar(L::kQEmpty));
      return true;
    };
    if (!issue_s(0)) break;
    for (int j = 0; j < n; ++j) {
      // S of the next tile goes first when its K has landed (the softmax can
      // then start that tile as soon as it finishes this one); otherwise this
      // tile's P V goes first, so its V slot is not held while K is awaited.
      bool s_next_done = j + 1 >= n;
      if (!s_next_done) {
        const uint32_t kidx = 2 * (g + j + 1);
        if (__all_sync(0xffffffffu, mbar_try_wait(bar(L::kKVFull + kidx % L::kStages), (kidx / L::kStages) & 1))) {
          if (!issue_s(j + 1)) {
            ok = false;
            break;
          }
          s_next_done = true;
        }
      }
      const uint32_t gi = g + j, vidx = 2 * gi + 1, vslot = vidx % L::kStages;
      if (!w.wait_warp(bar(L::kPFull + (gi & 1)), (gi >> 1) & 1, code | (L::kPFull + (gi & 1))) ||
          !w.wait_warp(bar(L::kKVFull + vslot), (vidx / L::kStages) & 1, code | (L::kKVFull + vslot)) ||
          (j == 0 && items > 0 && !w.wait_warp(bar(L::kOFree), (items - 1) & 1, code | L::kOFree))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t p_tmem = tmem + L::kPCol + 64 * (gi & 1);
      const uint64_t vd = v_desc0 + ((vslot * L::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        // keys 16 kk .. 16 kk + 15: box block (16 kk) / R, rows from (16 kk) % R
        const uint32_t voff = ((16 * kk) / R * box_bytes + ((16 * kk) % R) * 128) >> 4;
        mma_bf16_ts_elect(o_tmem, p_tmem + kk * 8, vd + voff, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit_elect(bar(L::kPVDone));
      if (j == n - 1) tc_commit_elect(bar(L::kODone));
      tc_commit_elect(bar(L::kKVEmpty + vslot));
      if (!s_next_done && !issue_s(j + 1)) {
        ok = false;
        break;
      }
    }
    g += n;
    ++items;
  }
  // Drain: every MMA this warp issued must complete before TMEM is freed.
  tc_commit_elect(bar(L::kFin));
  w.drain(bar(L::kFin), 0, code | L::kFin);
}

// Softmax warps: thread = TMEM lane.  Warp w belongs to replica c = w / WC,
// holds row r = (w % WC) * 32 + lane of the item's query rows, and handles key
// columns [c*C, c*C + C) of every tile (C = 32 * WC) with its own running
// (max, sum); at the end of the item the replicas are merged through shared
// memory and the rows written (final output, or one split's partial result).
template <int D, int WC>
__device__ __forceinline__ void dec_softmax(const DecParams& p, uint32_t sbase, uint8_t* smem, uint32_t tmem,
                                            const DecWaiter& w) {
  using L = DecSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr int C = 32 * WC;      // key columns per replica
  constexpr int kRpc = 32 * WC;   // lanes per replica
  constexpr int kCopies = 4 / WC;
  const int tid = threadIdx.x;    // 0..127, the TMEM lane
  const int warp = tid >> 5;
  const int copy = warp / WC;
  const int r = tid - copy * kRpc;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  float* scratch = reinterpret_cast<float*>(smem + L::kScratchOff);  // [lane][33]
  float* lane_m = reinterpret_cast<float*>(smem + L::kLaneOff);
  float* lane_l = lane_m + kLanes;
  float* row_M = reinterpret_cast<float*>(smem + L::kRowOff);
  float* row_L = row_M + kLanes;
  const int code = kDRoleSoftmax << 8;
  const int S = p.num_splits;

  {  // Both P buffers start at zero; a replica only ever writes its own columns.
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
    for (int c = 0; c < 128; c += 32) tmem_store_32cols(lane_addr + L::kPCol + c, z);
    tmem_store_wait();
  }

  uint32_t g = 0, items = 0, epi = 0, k_item = 0;
  bool ok = true;
  // Barrier of the 128 softmax threads (bounded, unlike bar.sync).
  auto epi_sync = [&]() -> bool {
    mbar_arrive(bar(L::kEpi));
    const bool got = w.wait(bar(L::kEpi), epi & 1, code | L::kEpi);
    ++epi;
    return __all_sync(0xffffffffu, got);
  };

  while (ok) {
    const int idx = dec_take_item<D>(sbase, smem, w, k_item, code);
    if (idx < 0) break;
    const DecItem it = dec_item(p, idx);
    const size_t grow0 = (static_cast<size_t>(it.b) * p.Hq + static_cast<size_t>(it.hkv) * p.group) * p.Nq + it.row0;
    if (it.t1 < it.t0) {
      // Nothing to read: a split past the end of a short sequence (its
      // partial result has weight zero) or an unusable sequence length.
      if (it.bad && tid == 0) atomicCAS(p.err, 0, kDErrSeqLen | (it.b & 0xFFFFF));
      for (int e = tid; e < it.rows; e += kLanes) {
        if (S > 1) {
          p.part_lse[(grow0 + e) * S + it.s] = -INFINITY;
        } else {
          p.lse[grow0 + e] = -INFINITY;
          for (int c = 0; c < D; ++c) p.out[(grow0 + e) * D + c] = __float2bfloat16_rn(0.f);
        }
      }
      continue;
    }
    const int n = it.t1 - it.t0 + 1;
    int lo_vis = 0, hi_vis = -1;  // visible key positions of this lane's row
    if (r < it.rows) {
      const int qpos = it.L - p.Nq + (it.row0 + r) % p.Nq;
      hi_vis = (p.mask_kind == kDMaskFull) ? it.L - 1 : qpos;
      lo_vis = (p.mask_kind == kDMaskWindow) ? max(0, qpos - p.window + 1) : 0;
    }
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < n; ++j) {
      const uint32_t gi = g + j;
      const int base = (it.t0 + j) * kKeys;
      if (!w.wait_warp(bar(L::kSFull + (gi & 1)), (gi >> 1) & 1, code | (L::kSFull + (gi & 1)))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      float x[C];
      {
        uint32_t sr[C];
        const uint32_t s_addr = lane_addr + L::kSCol + 128 * (gi & 1) + copy * C;
        if constexpr (C == 32) {
          tmem_load_32cols(s_addr, sr);
        } else if constexpr (C == 64) {
          tmem_load_64cols(s_addr, sr);
        } else {
          tmem_load_128cols(s_addr, sr);
        }
        const int key0 = base + copy * C;
#pragma unroll
        for (int c = 0; c < C; ++c) x[c] = __uint_as_float(sr[c]) * p.scale_log2;
        if (!(key0 >= lo_vis && key0 + C - 1 <= hi_vis)) {
          // Masked scores are replaced (not offset), so whatever an unloaded
          // or stale slot produced never reaches P.
#pragma unroll
          for (int c = 0; c < C; ++c) x[c] = (key0 + c >= lo_vis && key0 + c <= hi_vis) ? x[c] : -INFINITY;
        }
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c + 1 < C; c += 2) mx = max3f(mx, x[c], x[c + 1]);
      mx = fmaxf(mx, x[C - 1]);
      const float m_new = fmaxf(m, mx);
      bool resc = false;
      float f = 1.f;
      if (m == -INFINITY) {
        m = m_new;  // nothing accumulated yet for this lane
      } else if (m_new > m + kDecRescaleThreshold) {
        f = dec_exp2(m - m_new);
        l *= f;
        m = m_new;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O holds this item's tiles before j: wait for the P V of tile j-1.
        // A parity wait needs the barrier within one phase of the target:
        // S_j completing implies P V of tile j-2 completed (it was issued
        // before S_j), and P V of tile j cannot start before this P is
        // published, so P V phases gi-1 or gi are the only ones possible here.
        if (!w.wait_warp(bar(L::kPVDone), (gi - 1) & 1, code | L::kPVDone)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_load_32cols(lane_addr + L::kOCol + cc * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
          tmem_store_32cols(lane_addr + L::kOCol + cc * 32, o);
        }
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[C / 2];
#pragma unroll
      for (int c = 0; c < C / 2; ++c) {
        const float lo = dec_exp2(x[2 * c] - mu), hi = dec_exp2(x[2 * c + 1] - mu);
        l += lo + hi;
        pk[c] = dec_pack_bf16x2(lo, hi);
      }
      const uint32_t p_addr = lane_addr + L::kPCol + 64 * (gi & 1) + copy * (C / 2);
      if constexpr (C == 32) {
        tmem_store_16cols(p_addr, pk);
      } else {
#pragma unroll
        for (int c = 0; c < C / 2; c += 32) {
          uint32_t part[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) part[i] = pk[c + i];
          tmem_store_32cols(p_addr + c, part);
        }
      }
      if (base < it.lo_pos || base + kKeys > it.L) {
        // Edge tile: V rows outside [lo_pos, L) were not loaded or hold
        // slots past the sequence end; P is zero there, and they are cleared
        // so that 0 * (whatever they hold) cannot reach O.
        const uint32_t vidx = 2 * gi + 1, vslot = vidx % L::kStages;
        if (!w.wait_warp(bar(L::kKVFull + vslot), (vidx / L::kStages) & 1, code | (L::kKVFull + vslot))) {
          ok = false;
          break;
        }
        const int z0 = max(0, min(kKeys, it.lo_pos - base));  // rows [0, z0)
        const int z1 = max(0, min(kKeys, it.L - base));       // rows [z1, 128)
        const int nrows = z0 + (kKeys - z1);
        uint4* vt = reinterpret_cast<uint4*>(smem + L::kRingOff + vslot * L::kTileBytes);
        for (int e = tid; e < nrows * 8 * L::kChunks; e += kLanes) {
          const int rr = e / (8 * L::kChunks), rem = e - rr * (8 * L::kChunks);
          const int row = rr < z0 ? rr : z1 + (rr - z0);
          const int R = p.rows_per_load;
          vt[((row / R) * R * 128 * L::kChunks + (rem >> 3) * R * 128 + (row % R) * 128) / 16 + (rem & 7)] =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(bar(L::kPFull + (gi & 1)));
    }
    if (!ok) break;

    // ---- epilogue: merge the replicas, write the rows.  The item's own
    // barrier (one phase per item) says its last P V is done; the per-tile
    // one could be two phases behind here, where a parity wait is ambiguous.
    if (!w.wait_warp(bar(L::kODone), items & 1, code | L::kODone)) break;
    tc_fence_after_sync();
    lane_m[tid] = m;
    lane_l[tid] = l;
    if (!epi_sync()) break;
    if (tid < kRpc) {
      float M = -INFINITY;
#pragma unroll
      for (int cp = 0; cp < kCopies; ++cp) M = fmaxf(M, lane_m[cp * kRpc + tid]);
      float lt = 0.f;
#pragma unroll
      for (int cp = 0; cp < kCopies; ++cp) {
        const float mc = lane_m[cp * kRpc + tid];
        if (mc != -INFINITY) lt += dec_exp2(mc - M) * lane_l[cp * kRpc + tid];
      }
      row_M[tid] = M;
      row_L[tid] = lt;
    }
    if (!epi_sync()) break;
    const float f_self = (m == -INFINITY) ? 0.f : dec_exp2(m - row_M[r]);
#pragma unroll 1
    for (int cc = 0; cc < D / 32 && ok; ++cc) {
      uint32_t o[32];
      tmem_load_32cols(lane_addr + L::kOCol + cc * 32, o);
      if (cc == D / 32 - 1) {
        tc_fence_before_sync();
        mbar_arrive(bar(L::kOFree));  // O may now take the next item's P V
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) scratch[tid * 33 + c] = __uint_as_float(o[c]) * f_self;
      if (!epi_sync()) {
        ok = false;
        break;
      }
      for (int e = tid; e < it.rows * 32; e += kLanes) {
        const int row = e >> 5, c = e & 31;
        float acc = 0.f;
#pragma unroll
        for (int cp = 0; cp < kCopies; ++cp) acc += scratch[(cp * kRpc + row) * 33 + c];
        const float lt = row_L[row];
        const float val = lt > 0.f ? acc / lt : 0.f;
        const size_t grow = grow0 + row;
        if (S > 1) {
          p.part_o[(grow * S + it.s) * D + cc * 32 + c] = val;
        } else {
          p.out[grow * D + cc * 32 + c] = __float2bfloat16_rn(val);
        }
      }
      if (!epi_sync()) {
        ok = false;
        break;
      }
    }
    if (!ok) break;
    for (int row = tid; row < it.rows; row += kLanes) {
      const float lt = row_L[row];
      const float l2 = lt > 0.f ? row_M[row] + __log2f(lt) : -INFINITY;
      if (S > 1) {
        p.part_lse[(grow0 + row) * S + it.s] = l2;
      } else {
        p.lse[grow0 + row] = lt > 0.f ? l2 * kDecLn2 : -INFINITY;
      }
    }
    g += n;
    ++items;
  }
  tmem_store_wait();
}

template <int D, int WC>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const __grid_constant__ DecParams p) {
  using L = DecSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile uint32_t* loaded = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff + 8);  // tiles per loader

  // Query-buffer rows that no Q box covers must read as zero.
  for (uint32_t i = threadIdx.x; i < L::kTileBytes / 16; i += kDecThreads)
    reinterpret_cast<uint4*>(smem + L::kQOff)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
    mbar_init(bar(L::kQFull), 1);
    mbar_init(bar(L::kQEmpty), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kKVFull + s), 1);
      mbar_init(bar(L::kKVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::kSFull + b), 1);
      mbar_init(bar(L::kPFull + b), 4);       // one arrival per softmax warp
    }
    mbar_init(bar(L::kPVDone), 1);
    mbar_init(bar(L::kODone), 1);
    mbar_init(bar(L::kOFree), kLanes);
    mbar_init(bar(L::kEpi), kLanes);
    mbar_init(bar(L::kFin), 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(bar(L::kItemFull + i), 1);
      mbar_init(bar(L::kItemEmpty + i), 6);  // the MMA warp, the four softmax warps and the V loader
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDecMmaWarp) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const DecWaiter w{p.timeout_ns, abort_flag, p.err};

  if (warp < 4) {
    dec_softmax<D, WC>(p, sbase, smem, tmem, w);
  } else if (warp == kDecLoaderWarp) {
    const uint32_t gt = dec_loader<D, WC, false>(p, sbase, smem, w);
    if ((threadIdx.x & 31) == 0) loaded[0] = gt;
  } else if (warp == kDecVLoaderWarp) {
    const uint32_t gt = dec_loader<D, WC, true>(p, sbase, smem, w);
    if ((threadIdx.x & 31) == 0) loaded[1] = gt;
  } else {
    dec_mma<D>(p, sbase, smem, tmem, w);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == kDecLoaderWarp * 32) dec_drain_ring<D>(sbase, w, loaded[0], loaded[1]);
  if (warp == kDecMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kDecTmemCols);
  }
  // The last CTA to finish puts the work counter back to zero for the next
  // launch (every CTA has taken its last index by now).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
  }
}

// ------------------------------------------------------------ split merge
// One warp per query row: out = sum_s w_s O_s / sum_s w_s with
// w_s = 2^(lse2_s - max lse2), lse = ln sum_s 2^lse2_s.
struct DecMergeParams {
  const float* part_o;
  const float* part_lse;
  __nv_bfloat16* out;
  float* lse;
  int rows;
  int num_splits;
};

template <int D>
__global__ void __launch_bounds__(128) attn_decode_merge_kernel(const DecMergeParams p) {
  constexpr int V = D / 32;  // columns per lane
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const int S = p.num_splits;
  const float* pl = p.part_lse + static_cast<size_t>(row) * S;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, pl[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float wgt = dec_exp2(pl[s] - M);
      if (wgt > 0.f) {
        wsum += wgt;
        const float* src = p.part_o + (static_cast<size_t>(row) * S + s) * D + lane * V;
        if constexpr (V == 4) {
          const float4 o = *reinterpret_cast<const float4*>(src);
          acc[0] += wgt * o.x;
          acc[1] += wgt * o.y;
          acc[2] += wgt * o.z;
          acc[3] += wgt * o.w;
        } else {
          const float2 o = *reinterpret_cast<const float2*>(src);
          acc[0] += wgt * o.x;
          acc[1] += wgt * o.y;
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = p.out + static_cast<size_t>(row) * D + lane * V;
#pragma unroll
  for (int v = 0; v < V; v += 2) {
    const uint32_t pk = dec_pack_bf16x2(acc[v] * inv, acc[v + 1] * inv);
    *reinterpret_cast<uint32_t*>(dst + v) = pk;
  }
  if (lane == 0) p.lse[row] = wsum > 0.f ? (M + __log2f(wsum)) * kDecLn2 : -INFINITY;
}

}  // namespace attn_sm100_dec
