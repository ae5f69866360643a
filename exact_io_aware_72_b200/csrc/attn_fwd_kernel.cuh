// Exact attention forward for sm_100a: one persistent, warp-specialised kernel.
//
// What it computes is masked softmax attention with an online softmax
// ("Efficient attention: long context and sub-quadratic variants",
// stanleyjacob.dev, sections "Implementation, twice" and "FlashAttention: exact
// attention, IO-aware"): scores are formed tile by tile on chip, folded into a
// running (max, sum) per query row, and the N x N matrix never reaches HBM.
//
// CTA organisation (384 threads = 3 warpgroups, one CTA per SM, persistent):
//   warps 0-3   softmax for query tile 0 (thread = one query row = one TMEM lane)
//   warps 4-7   softmax for query tile 1
//   warp  8     TMA loader: Q tiles once per work item, K/V tiles through a ring
//   warps 9-10  tcgen05 issuers, one warp per query tile: S = Q K^T and
//               O += P V; warp 9 also owns the TMEM allocation; with bf16
//               inputs each also converts a quarter of every V tile to fp16
//   warp  11    bf16 inputs: converts the other half of every V tile to fp16
// Registers: launched at 168 per thread; the softmax warpgroups raise theirs to
// 208 and the third warpgroup drops to 88 (2*128*208 + 128*88 = 384*168).
// A work item is two 128-row query tiles that read the same K/V tiles: two query
// heads of one KV group (GQA with an even group size) or two consecutive query
// blocks of one head.  The two tiles ping-pong: while the softmax warps of one
// tile work, the tensor core runs the other tile's matmuls.
//
// TMEM (512 columns x 128 lanes, fp32): S0 [0,128) S1 [128,256) O0 and O1 after
// them.  P (fp16 with bf16 inputs, two per column; E4M3 with FP8 inputs, four per
// column) overwrites the first columns of its S tile.
//
// Precision (bf16 inputs): S = Q K^T is a bf16 product with fp32 accumulation;
// the softmax weights P are rounded to fp16 (11 significant bits) and V is
// converted to fp16 in shared memory for O += P V, so a row dominated by a few
// keys keeps its output within about 2^-12 of their spread before the one bf16
// rounding of out.  (bf16 P, 8 bits, is kept for V values beyond the fp16 range
// by request: F16P = false.)
//
// Every mbarrier wait is bounded by a global-timer limit; a wait that gives up
// records a code in the device error word and raises a CTA-wide abort flag, and
// all roles then leave their loops, drain what they issued, and free TMEM.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kBlockM = 128;    // query rows per tile
constexpr int kBlockN = 128;    // keys per K/V tile
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSoftmaxRegs = 208;
constexpr uint32_t kOtherRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * 168, "register split exceeds launch");
constexpr float kLn2 = 0.6931471805599453f;
// bf16 inputs: P goes to the tensor core as fp16 (11 significant bits, against
// bf16's 8), so its rounding adds about 2^-12 relative per weight instead of 2^-9;
// V is converted to fp16 in shared memory for the P V product (kind::f16 takes
// one type for both operands).  The running max is only moved when a row's max
// grows by more than kRescaleThresholdF16 powers of two, so P <= 2^15 < 65504, the
// largest fp16 value; the final O / l and log-sum-exp use the same max, so the
// result is unchanged, and the margin keeps O rescales (a TMEM round trip on the
// softmax critical path) rare.
constexpr float kRescaleThresholdF16 = 15.0f;
// bf16 P (inputs with V beyond the fp16 range, by request): P is packed to bf16
// by truncating p * (1 + 2^-9) -- with the factor folded into the exponent
// (x + log2(1 + 2^-9)), truncation lands within 3/4 of a bf16 ulp of p at the
// cost of one byte permute per pair -- and O is normalised by the sum of the
// bf16 values written, so a row dominated by one key returns that key's v.  The
// factor is common to every p of a row; the log-sum-exp (from the fp32 sum)
// subtracts it.  The running max may lag the row max by up to 2^32 there.
constexpr float kP16Bias = 0.0028150156f;  // log2(1 + 2^-9)
constexpr float kRescaleThresholdBF16 = 32.0f;
// E4M3 P (FP8 inputs): p is stored times 2^8, so weights down to 2^-14 of
// the row max stay normal E4M3 numbers; the running max then moves whenever a
// row's max grows by more than half a power of two (P <= 2^8.5 < 448, the
// largest E4M3 value).  The factor is common to the row: O / l is unaffected
// and the log-sum-exp subtracts it.
constexpr float kP8Bias = 8.0f;
constexpr float kRescaleThresholdE4M3 = 0.5f;
// V tiles converted to fp16 are signalled on a ring of this many barriers,
// indexed by the K/V step (see softmax_role).
constexpr int kConvRing = 4;
// Steps before the end of a work item at which the loader prefetches the next
// item's first tiles into L2 (each step is a few microseconds of work).
constexpr int kPrefetchSteps = 6;

enum : int { kMaskFull = 0, kMaskCausal = 1, kMaskWindow = 2 };

// Error codes: role in bits 8..11, barrier index in bits 0..7 for a wait that
// gave up; kErrRangeV (with the KV head in the low bits) for a V value that
// fp16 cannot hold.
enum : int { kRoleProducer = 1, kRoleMma = 2, kRoleSoftmax = 3, kRoleVConv = 4 };
constexpr int kErrRangeV = 1 << 20;

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq, N, d] bf16, box 64 x 128, 128B swizzle
  CUtensorMap tm_k;  // [B*Hkv, N, d]
  CUtensorMap tm_v;  // [B*Hkv, N, d]
  __nv_bfloat16* out;
  float* lse;
  int* err;          // device error word
  int B, Hq, Hkv, N;
  int group;         // Hq / Hkv
  int mask_kind;
  int window;
  int key_offset;    // query row i sits at key position i + key_offset (causal and window masks)
  float scale_log2;  // scale * log2(e)
  int pair_heads;    // 1: the two tiles are two heads of one KV group
  int num_mblk;      // ceil(N / 128)
  int row_units;     // row units per head unit (unit = one block, or a pair of blocks)
  int head_units;    // (b, head) or (b, head pair) units
  int num_items;     // row_units * head_units
  unsigned long long timeout_ns;
  int inject_stall;
  int out_v8;        // 1: out is 32-byte aligned, rows are written with 32-byte stores
  float v_scale;     // FP8 inputs: the V tensor's scale, applied to O in the epilogue
  unsigned int* item_visits;  // test hook: per work item, incremented once per visit (or null)
  float* out_f32;    // non-null: out is written here in fp32 (partial results to merge) instead of bf16
};

// EB = bytes per input element: 2 for bf16, 1 for E4M3 (head dim 128 only).
template <int D, int EB = 2>
struct SmemLayout {
  static_assert((EB == 2 && (D == 64 || D == 128)) || (EB == 1 && D == 128), "head dim and element size");
  static constexpr int kChunks = D * EB / 128;                   // 128-byte column chunks
  static constexpr int kChunkElems = 128 / EB;                   // elements in a 128-byte chunk row
  static constexpr uint32_t kChunkBytes = kBlockM * 128;         // 128 rows x 128 B
  static constexpr uint32_t kTileBytes = kChunks * kChunkBytes;  // one Q, K or V tile
  static constexpr int kStages = (kChunks == 2) ? 5 : 8;         // K/V ring slots
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKVOff = 2 * kTileBytes;
  static constexpr uint32_t kBarOff = kKVOff + kStages * kTileBytes;
  static constexpr int kQFull = 0;
  static constexpr int kQEmpty = 1;
  static constexpr int kKVFull = 2;
  static constexpr int kKVEmpty = kKVFull + kStages;
  static constexpr int kSFull = kKVEmpty + kStages;
  static constexpr int kPFull = kSFull + 2;
  static constexpr int kODone = kPFull + 2;
  static constexpr int kOFree = kODone + 2;
  static constexpr int kFin = kOFree + 2;
  static constexpr int kTurn = kFin + 2;
  static constexpr int kVConv = kTurn + 2;  // V tile of a step converted to fp16 (bf16 inputs)
  static constexpr int kNumBars = kVConv + kConvRing;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
  static constexpr uint32_t kSCol0 = 0, kSCol1 = 128;
  static constexpr uint32_t kOCol0 = 256, kOCol1 = 256 + D;
};

// ------------------------------------------------------------ work items
struct WorkItem {
  int b, hkv;
  int head[2];
  int mblk[2];
  int valid[2];
  int lo[2], hi[2];  // KV tile range of each query tile
  int lo_u, hi_u;    // union of the two ranges
};

// Row r sees keys [r + key_offset - window + 1, r + key_offset] (window), keys
// [0, r + key_offset] (causal), or every key (full), within [0, N).  A query
// block whose rows see no key at all (possible only with a key offset) gets one
// tile, fully masked: its rows then end with O = 0 and lse = -inf, and no work
// item is ever empty.
__device__ __forceinline__ void kv_range(const FwdParams& p, int m, int& lo, int& hi) {
  const int r0 = m * kBlockM;
  const int r1 = min(r0 + kBlockM - 1, p.N - 1);
  if (p.mask_kind == kMaskFull) {
    lo = 0;
    hi = p.num_mblk - 1;
  } else {
    hi = min(r1 + p.key_offset, p.N - 1) / kBlockN;
    lo = (p.mask_kind == kMaskWindow) ? min(max(0, r0 + p.key_offset - p.window + 1) / kBlockN, hi) : 0;
  }
}

// Work item (head unit hu, row unit r): head unit = (b, query head) or
// (b, query-head pair); row unit = one 128-row block (head pairs) or a pair of
// consecutive blocks of one head.
__device__ __forceinline__ WorkItem decode_item(const FwdParams& p, int hu, int r) {
  WorkItem it;
  if (p.pair_heads) {
    const int hpairs = p.Hq >> 1;
    it.b = hu / hpairs;
    const int hp = hu - it.b * hpairs;
    it.head[0] = 2 * hp;
    it.head[1] = 2 * hp + 1;
    it.mblk[0] = it.mblk[1] = r;
  } else {
    it.b = hu / p.Hq;
    it.head[0] = it.head[1] = hu - it.b * p.Hq;
    it.mblk[0] = 2 * r;
    it.mblk[1] = 2 * r + 1;
  }
  it.hkv = it.head[0] / p.group;
  it.lo_u = 0x7fffffff;
  it.hi_u = -1;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    it.valid[t] = it.mblk[t] < p.num_mblk;
    if (it.valid[t]) {
      kv_range(p, it.mblk[t], it.lo[t], it.hi[t]);
      it.lo_u = min(it.lo_u, it.lo[t]);
      it.hi_u = max(it.hi_u, it.hi[t]);
    } else {
      it.lo[t] = 1;
      it.hi[t] = 0;
    }
  }
  return it;
}

// Does KV tile j need element-wise masking for query block m?
__device__ __forceinline__ bool tile_is_partial(const FwdParams& p, int m, int j) {
  const int r0 = m * kBlockM + p.key_offset, c0 = j * kBlockN;
  bool partial = (c0 + kBlockN > p.N);
  if (p.mask_kind != kMaskFull) partial |= (c0 + kBlockN - 1 > r0);
  if (p.mask_kind == kMaskWindow) partial |= (c0 <= r0 + kBlockM - 1 - p.window);
  return partial;
}

// Static persistent schedule without any shared counter.  Row units r and
// R-1-r of one head form a super-item: under a causal mask their costs add up
// to the same total for every r, so dealing super-items round-robin (CTA c
// takes c, c+G, c+2G, ...) balances the load.  Super-items are numbered head
// unit by head unit, so the CTAs running at any moment share a few heads' K/V
// through L2 instead of each streaming its own head from HBM.  When the last,
// partial round has at most G/2 super-items, they are dealt as single row
// units instead (CTA c takes unit c of them), which halves that round's length.
struct Schedule {
  int g, sub, grid, total, per_head, R;
  int split_from;  // first super-item of the split last round (total if none)
  int tail;        // this CTA's row unit in the split round, -1 if none / taken
  __device__ Schedule(const FwdParams& p, int cta, int grid_)
      : g(cta), sub(0), grid(grid_), per_head((p.row_units + 1) >> 1), R(p.row_units) {
    total = p.head_units * per_head;
    const int rem = total % grid;
    const bool split = rem > 0 && 2 * rem <= grid;
    split_from = split ? total - rem : total;
    tail = (split && cta < 2 * rem) ? cta : -1;
  }
  // Next work item of this CTA (long row unit first); false when done.
  __device__ __forceinline__ bool next(int& hu, int& r) {
    if (g >= split_from) {
      if (tail < 0) return false;
      const int sidx = split_from + (tail >> 1);
      hu = sidx / per_head;
      const int s = sidx - hu * per_head;
      const bool second = (tail & 1) != 0;
      tail = -1;
      if (second && R - 1 - s == s) return false;  // middle unit of an odd R: one item only
      r = second ? s : R - 1 - s;
      return true;
    }
    hu = g / per_head;
    const int s = g - hu * per_head;
    if (sub == 0) {
      r = R - 1 - s;
      if (r == s) {
        g += grid;
      } else {
        sub = 1;
      }
    } else {
      r = s;
      sub = 0;
      g += grid;
    }
    return true;
  }
};

// ------------------------------------------------------------ bounded waits
struct Waiter {
  uint64_t limit_ns;
  volatile int* abort_flag;
  int* err;
  // Wait for the phase of `bar` with parity `parity`; false if the CTA aborts.
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
  // Wait for work this thread itself started (copies, MMAs) to finish, even
  // after an abort; still bounded by the time limit.
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
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------ V to fp16
// bf16 inputs: every V tile is converted to fp16 in place in shared memory for
// the fp16 P V product (element-wise, so the swizzled layout does not matter).
// Warp 11 converts the first half of each tile as soon as it lands; each MMA
// warp converts a quarter of the NEXT step's tile right after issuing its S
// product of a step, long before it next issues (after the softmax of its
// tile), so neither tile's P V waits on the other tile's progress.  The three
// arrive on kVConv[v % kConvRing] for K/V step v, and the P V of step v waits
// there.  A barrier of the ring is reused four steps later; by then both MMA
// warps have passed its previous phase, because V_{v+4} cannot land before the
// P V of step v has released ring space.
template <int D, int EB>
struct VConvSplit {
  static constexpr int kUnits = static_cast<int>(SmemLayout<D, EB>::kTileBytes / 16);  // 16-byte units
  static constexpr int kWarp11 = kUnits / 2;                                      // [0, kUnits / 2)
  static constexpr int kMma = kUnits / 4;                                          // then one quarter per MMA warp
};

// Units [u0, u0 + n) of the tile at tile_base, lane-strided: bf16 to fp16 in
// place.  Returns the per-half maximum of |v| seen (bf16 bits).
__device__ __forceinline__ uint32_t convert_v_units(uint32_t tile_base, int u0, int n, int lane) {
  uint32_t mag = 0;
#pragma unroll 4
  for (int i = lane; i < n; i += 32) {
    const uint32_t a = tile_base + static_cast<uint32_t>(u0 + i) * 16;
    uint32_t x0, x1, x2, x3;
    ld_shared_v4(a, x0, x1, x2, x3);
    mag = max_u16x2(max_u16x2(mag, x0 & 0x7fff7fffu), max_u16x2(x1 & 0x7fff7fffu, x2 & 0x7fff7fffu));
    mag = max_u16x2(mag, x3 & 0x7fff7fffu);
    st_shared_v4(a, bf16x2_to_f16x2(x0), bf16x2_to_f16x2(x1), bf16x2_to_f16x2(x2), bf16x2_to_f16x2(x3));
  }
  return mag;
}

// After a warp's part of a tile: make it visible to the tensor core's (async)
// proxy, record a magnitude of 2^16 or more (bf16 bits 0x4780 and up: beyond
// the largest fp16 value, or not finite) as kErrRangeV, arrive.
__device__ __forceinline__ void finish_v_part(uint32_t bar, uint32_t mag, int* err, int lane) {
  fence_proxy_async_smem();
  if (__any_sync(0xffffffffu, max(mag >> 16, mag & 0xffffu) >= 0x4780u) && lane == 0) atomicCAS(err, 0, kErrRangeV);
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Warp 11: the first half of every V tile of this CTA's work, in step order.
template <int D, int EB>
__device__ __forceinline__ void vconv_role(const FwdParams& p, uint32_t sbase, const Waiter& w, int lane) {
  using L = SmemLayout<D, EB>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  uint32_t v = 0;  // K/V steps so far; V of step v is load 2v + 1
  Schedule sched(p, blockIdx.x, gridDim.x);
  int hu, r;
  while (sched.next(hu, r)) {
    const WorkItem it = decode_item(p, hu, r);
    for (int j = it.lo_u; j <= it.hi_u; ++j, ++v) {
      const uint32_t vn = 2 * v + 1, slot = vn % L::kStages;
      const bool got = w.wait(bar(L::kKVFull + slot), (vn / L::kStages) & 1, (kRoleVConv << 8) | (L::kKVFull + slot));
      if (!__all_sync(0xffffffffu, got)) return;
      const uint32_t mag = convert_v_units(sbase + L::kKVOff + slot * L::kTileBytes, 0, VConvSplit<D, EB>::kWarp11, lane);
      finish_v_part(bar(L::kVConv + (v % kConvRing)), mag, w.err, lane);
    }
  }
}

// ------------------------------------------------------------ roles
// L2 prefetch of the next work item's Q tiles and of its first two K/V tiles
// (sched has already moved past the current item).
template <int D, int EB>
__device__ __forceinline__ void prefetch_next_item(const FwdParams& p, Schedule sched) {
  using L = SmemLayout<D, EB>;
  int hu, r;
  if (!sched.next(hu, r)) return;
  const WorkItem n = decode_item(p, hu, r);
#pragma unroll
  for (int c = 0; c < L::kChunks; ++c) {
    const int x = c * L::kChunkElems;
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (n.valid[t]) tma_prefetch_3d(&p.tm_q, x, n.mblk[t] * kBlockM, n.b * p.Hq + n.head[t]);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (n.lo_u + j > n.hi_u) break;
      tma_prefetch_3d(&p.tm_k, x, (n.lo_u + j) * kBlockN, n.b * p.Hkv + n.hkv);
      tma_prefetch_3d(&p.tm_v, x, (n.lo_u + j) * kBlockN, n.b * p.Hkv + n.hkv);
    }
  }
}

template <int D, int EB>
__device__ __forceinline__ void producer_role(const FwdParams& p, uint32_t sbase, const Waiter& w) {
  using L = SmemLayout<D, EB>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const uint64_t pol_kv = l2_policy_evict_last();
  const uint64_t pol_q = l2_policy_evict_first();
  tma_prefetch_map(&p.tm_q);
  tma_prefetch_map(&p.tm_k);
  tma_prefetch_map(&p.tm_v);

  uint32_t kv_n = 0;  // K/V loads issued so far
  uint32_t q_issued = 0;
  int items = 0;
  bool ok = !p.inject_stall;
  Schedule sched(p, blockIdx.x, gridDim.x);
  int hu, r;
  while (ok && sched.next(hu, r)) {
    const WorkItem it = decode_item(p, hu, r);
    if (p.item_visits) atomicAdd(p.item_visits + static_cast<size_t>(hu) * p.row_units + r, 1u);
    // Q of this item goes into the single Q buffer once the previous item's
    // last S has read it.  The item's first K and V tiles are issued before
    // that wait (their ring slots free up earlier), so they are already in
    // flight while the previous item drains.
    auto load_q = [&]() -> bool {
      if (items > 0 && !w.wait(bar(L::kQEmpty), (items - 1) & 1, (kRoleProducer << 8) | L::kQEmpty)) return false;
      const uint32_t qbytes = (it.valid[0] + it.valid[1]) * L::kTileBytes;
      mbar_arrive_expect_tx(bar(L::kQFull), qbytes);
      ++q_issued;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!it.valid[t]) continue;
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sbase + L::kQOff + t * L::kTileBytes + c * L::kChunkBytes, &p.tm_q, bar(L::kQFull),
                      c * L::kChunkElems, it.mblk[t] * kBlockM, it.b * p.Hq + it.head[t], pol_q);
      }
      return true;
    };
    // A few steps before the item ends, start pulling what the next item
    // reads first (its Q tiles and first K/V tiles) into L2, so the next
    // item's loads do not wait on DRAM.
    const int pf_step = max(it.lo_u, it.hi_u - kPrefetchSteps);
    for (int j = it.lo_u; j <= it.hi_u && ok; ++j) {
      if (j == pf_step) prefetch_next_item<D, EB>(p, sched);
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t slot = kv_n % L::kStages;
        if (kv_n >= (uint32_t)L::kStages &&
            !w.wait(bar(L::kKVEmpty + slot), ((kv_n / L::kStages) - 1) & 1,
                    (kRoleProducer << 8) | (L::kKVEmpty + slot))) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::kKVFull + slot), L::kTileBytes);
        const CUtensorMap* map = kv ? &p.tm_v : &p.tm_k;
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sbase + L::kKVOff + slot * L::kTileBytes + c * L::kChunkBytes, map,
                      bar(L::kKVFull + slot), c * L::kChunkElems, j * kBlockN, it.b * p.Hkv + it.hkv, pol_kv);
        ++kv_n;
        if (j == it.lo_u && kv == 1 && !load_q()) {
          ok = false;
          break;
        }
      }
    }
    ++items;
  }
  // Drain: every copy this thread started must land before the CTA exits.
  for (uint32_t s = 0; s < (uint32_t)L::kStages; ++s) {
    if (kv_n > s) {
      const uint32_t last = s + ((kv_n - 1 - s) / L::kStages) * L::kStages;  // last load into slot s
      w.drain(bar(L::kKVFull + s), (last / L::kStages) & 1, (kRoleProducer << 8) | (L::kKVFull + s));
    }
  }
  if (q_issued > 0) w.drain(bar(L::kQFull), (q_issued - 1) & 1, (kRoleProducer << 8) | L::kQFull);
}

// One issuing warp per query tile t: all lanes run the loop with warp-uniform
// values (descriptor arithmetic stays on the uniform datapath) and one elected
// lane issues each tcgen05 instruction.  For each KV tile j of the item:
//   O_t += P_t(j-1) V_{j-1}   (once the softmax has written P_t(j-1))
//   S_t  = Q_t K_j^T          (after that P V in issue order, since P aliases S)
// and releases K_j / V_{j-1} / Q with commits; the other tile's warp does the
// same, so each ring slot is freed after both warps' reads complete.
template <int D, int EB, bool F16P>
__device__ __forceinline__ void mma_role(const FwdParams& p, uint32_t sbase, uint32_t tmem, const Waiter& w,
                                         int t) {
  using L = SmemLayout<D, EB>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  // bf16 inputs: kind::f16; E4M3 inputs: kind::f8f6f4.  Either way one
  // product takes 32 bytes of K per row: 16 bf16 or 32 E4M3 elements.
  constexpr uint32_t idesc_s =
      EB == 2 ? idesc_bf16_f32(kBlockM, kBlockN, false) : idesc_e4m3_f32(kBlockM, kBlockN, false);
  // P V: fp16 P and the fp16 copy of V, bf16 both, or E4M3 both.
  constexpr bool kConvV = EB == 2 && F16P;
  constexpr uint32_t idesc_o = EB == 1 ? idesc_e4m3_f32(kBlockM, D, true)
                                       : (F16P ? idesc_f16_f32(kBlockM, D, true) : idesc_bf16_f32(kBlockM, D, true));
  constexpr int kKeysPerPv = 32 / EB;  // keys per P V product
  const uint32_t s_tmem = tmem + (t ? L::kSCol1 : L::kSCol0);
  const uint32_t o_tmem = tmem + (t ? L::kOCol1 : L::kOCol0);
  // Descriptor bases: Q_t (K-major), ring slot 0 as K (K-major) and as V
  // (MN-major, d chunks 16 KB apart).  Per-MMA offsets are added to the start
  // address field (16-byte units).
  const uint64_t q_desc = smem_desc_sw128(sbase + L::kQOff + t * L::kTileBytes, 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(sbase + L::kKVOff, 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(sbase + L::kKVOff, L::kChunkBytes, 1024);
  const int code = (kRoleMma << 8) | (t << 7);
  // Every lane waits; the warp proceeds only if all lanes saw the phase.
  auto wait_all = [&](uint32_t b, uint32_t parity, int c) -> bool {
    const bool got = w.wait(b, parity, c);
    return __all_sync(0xffffffffu, got);
  };

  // This warp's quarter of the V tile of K/V step v (load 2v + 1) to fp16.
  auto convert_quarter = [&](uint32_t v) -> bool {
    const uint32_t vn = 2 * v + 1, vslot = vn % L::kStages;
    if (!wait_all(bar(L::kKVFull + vslot), (vn / L::kStages) & 1, code | (L::kKVFull + vslot))) return false;
    const uint32_t mag = convert_v_units(sbase + L::kKVOff + vslot * L::kTileBytes,
                                         VConvSplit<D, EB>::kWarp11 + t * VConvSplit<D, EB>::kMma,
                                         VConvSplit<D, EB>::kMma, threadIdx.x & 31);
    finish_v_part(bar(L::kVConv + (v % kConvRing)), mag, w.err, threadIdx.x & 31);
    return true;
  };

  uint32_t kv_n = 0;
  uint32_t p_cnt = 0;
  int items = 0;
  bool ok = true;
  Schedule sched(p, blockIdx.x, gridDim.x);
  if constexpr (kConvV) {
    Schedule peek = sched;
    int h0, r0;
    if (peek.next(h0, r0)) ok = convert_quarter(0);
  }
  int hu, r;
  while (ok && sched.next(hu, r)) {
    const WorkItem it = decode_item(p, hu, r);
    bool more_items = false;  // a step follows this item's last one
    if constexpr (kConvV) {
      Schedule peek = sched;
      int h2, r2;
      more_items = peek.next(h2, r2);
    }
    const int valid = t ? it.valid[1] : it.valid[0];
    const int lo = t ? it.lo[1] : it.lo[0];
    const int hi = t ? it.hi[1] : it.hi[0];
    if (!wait_all(bar(L::kQFull), items & 1, code | L::kQFull)) break;
    tc_fence_after_sync();
    bool pend = false;
    bool first_pv = true;

    // The V tile with load index vn has landed (a tile this warp does not
    // read must still be seen before this warp releases it).
    auto wait_v_landed = [&](uint32_t vn) -> bool {
      const uint32_t vslot = vn % L::kStages;
      return wait_all(bar(L::kKVFull + vslot), (vn / L::kStages) & 1, code | (L::kKVFull + vslot));
    };
    // O_t += P_t V for the V tile with load index vn.
    auto issue_pv = [&](uint32_t vn) -> bool {
      if (first_pv && items > 0 && !wait_all(bar(L::kOFree + t), (items - 1) & 1, code | (L::kOFree + t)))
        return false;
      if (!wait_all(bar(L::kPFull + t), p_cnt & 1, code | (L::kPFull + t))) return false;
      ++p_cnt;
      const uint32_t vslot = vn % L::kStages;
      // With fp16 P the conversion barrier below implies the tile landed (its
      // converters waited for that), and the product reads only bytes they rewrote.
      if (!kConvV && !wait_all(bar(L::kKVFull + vslot), (vn / L::kStages) & 1, code | (L::kKVFull + vslot)))
        return false;
      if constexpr (kConvV) {
        // Warp 11 and both MMA warps have converted this V tile (K/V step vn / 2) to fp16.
        const uint32_t v = vn >> 1;
        if (!wait_all(bar(L::kVConv + (v % kConvRing)), (v / kConvRing) & 1, code | (L::kVConv + (v % kConvRing))))
          return false;
      }
      tc_fence_after_sync();
      const uint64_t vd = v_desc0 + ((vslot * L::kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBlockN / kKeysPerPv; ++kk) {
        // Next keys: 16 (bf16) or 32 (E4M3) rows of 128 B further into the V
        // tile; their P is the next 8 TMEM columns (32 bytes per row).
        const uint64_t vk = vd + ((kk * kKeysPerPv * 128) >> 4);
        if constexpr (EB == 2)
          mma_bf16_ts_elect(o_tmem, s_tmem + kk * 8, vk, idesc_o, (kk > 0 || !first_pv) ? 1u : 0u);  // kind::f16
        else
          mma_e4m3_ts_elect(o_tmem, s_tmem + kk * 8, vk, idesc_o, (kk > 0 || !first_pv) ? 1u : 0u);
      }
      first_pv = false;
      pend = false;
      return true;
    };

    for (int j = it.lo_u; j <= it.hi_u; ++j) {
      const uint32_t kslot = kv_n % L::kStages;
      // K_j is normally resident long before P_t(j-1) is ready; confirming it
      // first lets P V and the next S issue back to back once P arrives.
      if (!wait_all(bar(L::kKVFull + kslot), (kv_n / L::kStages) & 1, code | (L::kKVFull + kslot))) {
        ok = false;
        break;
      }
      if (pend) {
        if (!issue_pv(kv_n - 1)) {
          ok = false;
          break;
        }
      } else if (j > it.lo_u && !wait_v_landed(kv_n - 1)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      if (valid && j >= lo && j <= hi) {
        const uint64_t kd = k_desc0 + ((kslot * L::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D * EB / 32; ++kk) {
          // K-major operands: 32 B of a 128 B swizzled row per product, the
          // next 128-byte chunk of the rows 16 KB further.
          const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
          if constexpr (EB == 2)
            mma_bf16_ss_elect(s_tmem, q_desc + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
          else
            mma_e4m3_ss_elect(s_tmem, q_desc + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit_elect(bar(L::kSFull + t));
        pend = true;
      }
      // Each slot's empty barrier takes one arrival per MMA warp and phase.
      // A warp releases a tile only after it has seen that tile land (for a
      // tile this warp's MMAs do not read, wait_v_landed above), so its
      // arrival for a load can only come after the load was issued, i.e.
      // after the slot's previous phase completed: no warp ever arrives twice
      // in one phase, even when its own tile is idle and it runs ahead.
      if (j > it.lo_u) tc_commit_elect(bar(L::kKVEmpty + (kv_n - 1) % L::kStages));  // V_{j-1} read
      tc_commit_elect(bar(L::kKVEmpty + kslot));                                   // K_j read
      if (j == it.hi_u) tc_commit_elect(bar(L::kQEmpty));                          // Q read
      if constexpr (kConvV) {
        // This warp's quarter of the next step's V (its P V comes a step later).
        if ((j < it.hi_u || more_items) && !convert_quarter((kv_n >> 1) + 1)) {
          ok = false;
          break;
        }
      }
      kv_n += 2;
    }
    if (!ok) break;
    if (pend ? !issue_pv(kv_n - 1) : !wait_v_landed(kv_n - 1)) break;
    tc_commit_elect(bar(L::kKVEmpty + (kv_n - 1) % L::kStages));  // V_hi read
    if (first_pv && items > 0 && !wait_all(bar(L::kOFree + t), (items - 1) & 1, code | (L::kOFree + t))) break;
    tc_commit_elect(bar(L::kODone + t));
    ++items;
  }
  // Drain: every MMA this thread issued must complete before TMEM is freed.
  tc_commit_elect(bar(L::kFin + t));
  w.drain(bar(L::kFin + t), 0, code | (L::kFin + t));
}

// Eight softmax warps, one thread per query row of their tile.
template <int D, int EB, bool F16P>
__device__ __forceinline__ void softmax_role(const FwdParams& p, uint32_t sbase, uint32_t tmem,
                                             const Waiter& w, int warp, int lane) {
  using L = SmemLayout<D, EB>;
  constexpr float kBias = EB == 1 ? kP8Bias : (F16P ? 0.f : kP16Bias);
  constexpr float kThreshold = EB == 1 ? kRescaleThresholdE4M3 : (F16P ? kRescaleThresholdF16 : kRescaleThresholdBF16);
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const int t = warp >> 2;
  const int quarter = warp & 3;
  const int row_in_tile = quarter * 32 + lane;
  const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_bits + (t ? L::kSCol1 : L::kSCol0);
  const uint32_t tO = tmem + lane_bits + (t ? L::kOCol1 : L::kOCol0);
  const float c = p.scale_log2;

  uint32_t s_cnt = 0;
  uint32_t turn_cnt = 0;
  int items = 0;
  bool ok = true;
  Schedule sched(p, blockIdx.x, gridDim.x);
  int hu, r;
  while (ok && sched.next(hu, r)) {
    const WorkItem it = decode_item(p, hu, r);
    // This warp's tile, picked with selects so the item stays in registers.
    const int mblk = t ? it.mblk[1] : it.mblk[0];
    const int head = t ? it.head[1] : it.head[0];
    const int valid = t ? it.valid[1] : it.valid[0];
    const int lo = t ? it.lo[1] : it.lo[0];
    const int hi = t ? it.hi[1] : it.hi[0];
    const int row = mblk * kBlockM + row_in_tile;
    float m_run = -INFINITY;
    float l_run = 0.f;   // row sum that normalises O (bf16 P: of the bf16 values written)
    float l_lse = 0.f;   // fp32 row sum of p: the log-sum-exp (and O's normaliser otherwise)
    // Both softmax warpgroups walk the item's whole KV range so they can hand
    // the turn token back and forth: the exp loop of one tile runs while
    // the tensor core works on the other tile (the exp unit is the shared
    // bottleneck), whether or not a tile has work at a given step.
    for (int j = it.lo_u; j <= it.hi_u; ++j) {
      const bool active = valid && j >= lo && j <= hi;
      float s[128];
      if (active) {
        bool got = w.wait(bar(L::kSFull + t), s_cnt & 1, (kRoleSoftmax << 8) | (L::kSFull + t));
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after_sync();
        uint32_t sr[128];
        tmem_load_128cols(tS, sr);
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
        if (tile_is_partial(p, mblk, j)) {
          const int c0 = j * kBlockN;
          const int hi_i = ((p.mask_kind == kMaskFull) ? p.N - 1 : min(row + p.key_offset, p.N - 1)) - c0;
          const int lo_i = (p.mask_kind == kMaskWindow) ? row + p.key_offset - p.window + 1 - c0 : -1;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > hi_i || i < lo_i) s[i] = -INFINITY;
        }
      }
      bool need = false;
      float alpha = 1.f;
      float neg_base = 0.f;
      if (active) {
        // Row max: eight chains of three-input max (integer/ALU work, done
        // before taking the turn so it overlaps the other tile's exp loop).
        float mx[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = s[q];
#pragma unroll
        for (int i = 8; i < 128; i += 2) mx[(i >> 1) & 7] = max3f(mx[(i >> 1) & 7], s[i], s[i + 1]);
        const float tile_max = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float m_new = fmaxf(m_run, tile_max * c);
        need = m_new > m_run + kThreshold;
        if (need) {
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        neg_base = (m_run == -INFINITY) ? 0.f : -m_run;
      }
      {
        bool got = w.wait(bar(L::kTurn + t), turn_cnt & 1, (kRoleSoftmax << 8) | (L::kTurn + t));
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        ++turn_cnt;
      }
      if (active) {
        // p = 2^(s*c - m) on column pairs (packed fp32 FMA, MUFU ex2), rounded to
        // fp16 or bf16 (bf16 inputs) or E4M3 (FP8 inputs) and written to TMEM
        // over the first columns of the S tile.  The fp32 sum of p gives the
        // log-sum-exp and, except with bf16 P, normalises O.
        const uint64_t c2 = f32x2_pack(c, c);
        const uint64_t nb2 = f32x2_pack(neg_base + kBias, neg_base + kBias);
        uint64_t sl2 = 0, so2 = 0;  // (+0.f, +0.f)
#pragma unroll
        for (int chunk = 0; chunk < 4; ++chunk) {
          uint32_t pk[EB == 2 ? 16 : 8];   // P columns: two fp16 or four E4M3 values each
          float prev0 = 0.f, prev1 = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = chunk * 32 + 2 * i;
            const uint64_t x2 = f32x2_fma(f32x2_pack(s[e], s[e + 1]), c2, nb2);
            float x0, x1;
            f32x2_unpack(x2, x0, x1);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            if constexpr (EB == 2 && F16P) {
              pk[i] = pack_f16x2(p0, p1);  // round to nearest even
            } else if constexpr (EB == 2) {
              pk[i] = __byte_perm(__float_as_uint(p0), __float_as_uint(p1), 0x7632);  // truncate to bf16x2
              so2 = f32x2_add(so2, f32x2_pack(__uint_as_float(__float_as_uint(p0) & 0xffff0000u),
                                              __uint_as_float(__float_as_uint(p1) & 0xffff0000u)));
            } else {
              // Round to nearest E4M3; four consecutive keys share a column, lowest first.
              if (i & 1) {
                pk[i >> 1] = pack_e4m3x4(prev0, prev1, p0, p1);
              } else {
                prev0 = p0;
                prev1 = p1;
              }
            }
            sl2 = f32x2_add(sl2, f32x2_pack(p0, p1));
          }
          if constexpr (EB == 2)
            tmem_store_16cols(tS + chunk * 16, pk);
          else
            tmem_store_8cols(tS + chunk * 8, pk);
        }
        float sl_lo, sl_hi;
        f32x2_unpack(sl2, sl_lo, sl_hi);
        l_lse = l_lse * alpha + (sl_lo + sl_hi);
        if constexpr (EB == 2 && !F16P) {
          float so_lo, so_hi;
          f32x2_unpack(so2, so_lo, so_hi);
          l_run = l_run * alpha + (so_lo + so_hi);
        } else {
          l_run = l_lse;
        }
      }
      if (!active) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kTurn + (t ^ 1)));
      } else {
        if (j > lo && __any_sync(0xffffffffu, need)) {
          // O of this row was last written by the P V of the previous tile; that
          // MMA completed before this S tile did (in-order tcgen05 completion).
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_load_32cols(tO + cc * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_store_32cols(tO + cc * 32, o);
          }
        }
        tmem_store_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(L::kPFull + t));
          // Hand the turn to the other tile once P is published: its exp loop
          // then runs while the tensor core takes this tile's P V and next S.
          mbar_arrive(bar(L::kTurn + (t ^ 1)));
        }
      }
    }
    if (!ok) break;
    // Epilogue: O / l to bf16, log-sum-exp to fp32.
    bool got = w.wait(bar(L::kODone + t), items & 1, (kRoleSoftmax << 8) | (L::kODone + t));
    if (!__all_sync(0xffffffffu, got)) break;
    tc_fence_after_sync();
    if (valid && p.out_f32) {
      // fp32 out: O / l written unrounded, 128 bytes per 32 columns.
      const bool row_ok = row < p.N;
      const float inv_l = (l_run > 0.f) ? (EB == 2 ? 1.f : p.v_scale) / l_run : 0.f;
      const size_t head_row = (static_cast<size_t>(it.b) * p.Hq + head) * p.N + (row_ok ? row : 0);
      float4* dstf = reinterpret_cast<float4*>(p.out_f32 + head_row * D);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_load_32cols(tO + cc * 32, o);
        if (row_ok) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dstf[cc * 8 + v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                           __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
      }
      if (row_ok) p.lse[head_row] = (m_run + __log2f(l_lse) - kBias) * kLn2;
    } else if (valid) {
      const bool row_ok = row < p.N;
      const float inv_l = (l_run > 0.f) ? (EB == 2 ? 1.f : p.v_scale) / l_run : 0.f;
      const size_t head_row = (static_cast<size_t>(it.b) * p.Hq + head) * p.N + (row_ok ? row : 0);
      uint4* dst = reinterpret_cast<uint4*>(p.out + head_row * D);
      const uint64_t inv2 = f32x2_pack(inv_l, inv_l);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_load_32cols(tO + cc * 32, o);
        if (row_ok) {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a, b;
            f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), inv2), a, b);
            h[i] = pack_bf16x2(a, b);
          }
          // 32 columns = 64 bytes of the row: two 32-byte stores when the
          // output allows it (fewer store instructions and L1 wavefronts).
          if (p.out_v8) {
#pragma unroll
            for (int v = 0; v < 2; ++v)
              st_global_v8(dst + cc * 4 + 2 * v, h[8 * v], h[8 * v + 1], h[8 * v + 2], h[8 * v + 3], h[8 * v + 4],
                           h[8 * v + 5], h[8 * v + 6], h[8 * v + 7]);
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[cc * 4 + v] = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
          }
        }
      }
      if (row_ok) p.lse[head_row] = (m_run + __log2f(l_lse) - kBias) * kLn2;
    }
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kOFree + t));
    ++items;
  }
  tmem_store_wait();
}

// EB = bytes per input element (2: bf16, 1: E4M3); F16P (bf16 inputs): P and V
// go to the P V product as fp16 (true) or as bf16 (false).
template <int D, int EB = 2, bool F16P = true>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using L = SmemLayout<D, EB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
    mbar_init(bar(L::kQFull), 1);
    mbar_init(bar(L::kQEmpty), 2);             // one commit per MMA thread
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kKVFull + s), 1);
      mbar_init(bar(L::kKVEmpty + s), 2);      // one commit per MMA thread
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kSFull + t), 1);
      mbar_init(bar(L::kPFull + t), 4);        // one arrival per softmax warp
      mbar_init(bar(L::kODone + t), 1);
      mbar_init(bar(L::kOFree + t), 4);        // one arrival per softmax warp
      mbar_init(bar(L::kFin + t), 1);
      mbar_init(bar(L::kTurn + t), 4);         // one arrival per warp of the other warpgroup
    }
    for (int i = 0; i < kConvRing; ++i) mbar_init(bar(L::kVConv + i), 3);  // warp 11 and both MMA warps
    for (int i = 0; i < 4; ++i) mbar_arrive(bar(L::kTurn + 0));  // tile 0 starts with the turn
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const Waiter w{p.timeout_ns, abort_flag, p.err};

  if (warp < 8) {
    reg_alloc_raise<kSoftmaxRegs>();
    softmax_role<D, EB, F16P>(p, sbase, tmem, w, warp, lane);
  } else {
    reg_alloc_lower<kOtherRegs>();
  }
  if (warp == kProducerWarp) {
    if (lane == 0) producer_role<D, EB>(p, sbase, w);
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    mma_role<D, EB, F16P>(p, sbase, tmem, w, warp - kMmaWarp);
  } else if (warp == kMmaWarp + 2) {
    if constexpr (EB == 2 && F16P) vconv_role<D, EB>(p, sbase, w, lane);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_sm100
