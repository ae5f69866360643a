// Exact attention backward for sm_100a: the gradients of sum(dO * O) with
// respect to q, k and v, recomputing P from the forward's log-sum-exp instead
// of storing it ("Efficient attention: long context and sub-quadratic
// variants", stanleyjacob.dev, section "Against the real libraries": the
// production kernel line ships a recompute-based backward pass).
//
// For one (batch, query head) with S = scale q k^T (masked -inf) and
// P = exp(S - lse) (lse from the forward), the chain rule gives
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D) with D_i = dO_i . O_i,
//   dQ = scale dS K,  dK = scale dS^T Q,
// and grouped KV heads sum the gradients of the query heads that read them.
//
// Kernels, all on the caller's stream, after attn_bwd_delta_kernel (D =
// rowsum(dO * O) in fp32, in the caller's workspace).  A key-tile kernel takes
// one 128-key K/V tile per work item and walks the visible query tiles of every
// query head of its KV group: S^T = K Q^T, dP^T = V dO^T, P^T and dS^T by the
// elementwise warps, dV += P^T dO and dK += dS^T Q accumulated in TMEM over the
// item.  Two paths use it:
//   fused (d = 128, Hq == Hkv): the key-tile kernel works in 64-query halves
//            and also forms dQ^T = K^T dS^T for each half (dS^T staged in
//            shared memory); four more warps read it from TMEM and add it into
//            an fp32 dQ accumulator in the workspace with coalesced global
//            reductions, and attn_bwd_dq_convert_kernel scales and rounds the
//            sums to bf16.  P and dS are formed once per (query, key) pair:
//            five matmuls per pair.
//   two-kernel (d = 64, grouped heads, or on request): a query-tile kernel
//            (one 128-row query tile per work item, walking its visible K/V
//            tiles: S = Q K^T and dP = dO V^T recomputed, dS by the elementwise
//            warps, dQ += dS K in TMEM), then the key-tile kernel for dK and
//            dV; both on whole 128 x 128 tiles, seven matmuls per pair, no
//            atomics.
//
// CTA organisation of the tcgen05 kernels (one CTA per SM, persistent):
// warps 0-3 elementwise (thread = TMEM lane = one row of the work item's
// tile), warp 4 TMA loader, warp 5 tcgen05 issuer (one elected lane
// issues), and in the fused d = 128 kernel warps 6-9 reading dQ^T out of
// TMEM.  All waits are bounded like the forward's.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace attn_sm100_bwd {
using namespace attn_sm100;

constexpr int kTile = 128;  // rows of every Q / dO / K / V tile
constexpr int kHalf = 64;   // keys (dQ kernel) or queries (dK/dV kernel) per score half
constexpr int kBwdThreads = 192;
constexpr int kBwdThreadsFused = 320;
constexpr int kBwdLoaderWarp = 4;
constexpr int kBwdMmaWarp = 5;
constexpr int kBwdDqWarp0 = 6;  // fused kernel: warps 6-9 read dQ^T
constexpr uint32_t kBwdTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kBMaskFull = 0, kBMaskCausal = 1, kBMaskWindow = 2 };
enum : int { kBRoleLoader = 1, kBRoleMma = 2, kBRoleElem = 3, kBRoleDq = 4 };
enum : int { kBKernelDq = 0, kBKernelDkdv = 1, kBKernelFused = 2, kBKernelDkdvFull = 3, kBKernelDqFull = 4 };

struct BwdParams {
  CUtensorMap tm_q;   // [B*Hq, N, d] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap tm_k;   // [B*Hkv, N, d]
  CUtensorMap tm_v;   // [B*Hkv, N, d]
  CUtensorMap tm_do;  // [B*Hq, N, d]
  const float* lse;   // [B*Hq, N] natural-log LSE from the forward
  const float* delta; // [B*Hq, N] D = rowsum(dO * O)
  __nv_bfloat16* dq;  // [B*Hq, N, d]
  __nv_bfloat16* dk;  // [B*Hkv, N, d]
  __nv_bfloat16* dv;  // [B*Hkv, N, d]
  float* dq_acc;      // fused kernel: [B*Hq, N, d] fp32 dQ / scale, zeroed before the launch
  int* err;           // device error word (shared with the forward)
  int B, Hq, Hkv, N, group;
  int mask_kind, window;
  float scale;        // softmax scale (dQ, dK are scaled by it)
  float scale_log2;   // scale * log2(e)
  int num_blk;        // ceil(N / 128)
  int num_items;      // work items of the kernel being launched
  unsigned long long timeout_ns;
};

// Visible key range [lo, hi] (tile indices) of query tile m, and visible query
// tile range of key tile n (the transposed question), for the three masks.
__device__ __forceinline__ void key_tiles_of_query_tile(const BwdParams& p, int m, int& lo, int& hi) {
  const int r0 = m * kTile;
  const int r1 = min(r0 + kTile - 1, p.N - 1);
  if (p.mask_kind == kBMaskFull) {
    lo = 0;
    hi = p.num_blk - 1;
  } else {
    hi = r1 / kTile;
    lo = (p.mask_kind == kBMaskWindow) ? max(0, r0 - p.window + 1) / kTile : 0;
  }
}
__device__ __forceinline__ void query_tiles_of_key_tile(const BwdParams& p, int n, int& lo, int& hi) {
  const int c0 = n * kTile;
  const int c1 = min(c0 + kTile - 1, p.N - 1);
  if (p.mask_kind == kBMaskFull) {
    lo = 0;
    hi = p.num_blk - 1;
  } else {
    lo = c0 / kTile;  // query i sees key j only if j <= i
    // window: key j is seen by queries i with j <= i <= j + w - 1
    hi = (p.mask_kind == kBMaskWindow) ? min(p.num_blk - 1, (c1 + p.window - 1) / kTile) : p.num_blk - 1;
  }
}
// Does the (query tile m, key tile n) block need element masks?
__device__ __forceinline__ bool block_is_partial(const BwdParams& p, int m, int n) {
  const int r0 = m * kTile, c0 = n * kTile;
  bool partial = (c0 + kTile > p.N) || (r0 + kTile > p.N);
  if (p.mask_kind != kBMaskFull) partial |= (c0 + kTile - 1 > r0);
  if (p.mask_kind == kBMaskWindow) partial |= (c0 <= r0 + kTile - 1 - p.window);
  return partial;
}

// Bounded mbarrier waits (a wait that gives up records `code` in the error
// word and raises the CTA's abort flag; the roles then leave their loops).
struct BwdWaiter {
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
  // All 32 lanes wait; true only if every lane saw the phase.
  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, int code) const {
    return __all_sync(0xffffffffu, wait(bar, parity, code));
  }
};

// Two 32-column TMEM loads (32x32b shape: thread = lane, consecutive registers
// = consecutive columns) completed by one wait.
__device__ __forceinline__ void tmem_load_2x32cols(uint32_t ta, uint32_t tb, uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]),
        "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]),
        "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]),
        "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]), "=r"(b[0]),
        "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]),
        "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]),
        "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]),
        "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

// 4-byte asynchronous copy global -> shared; with src_bytes = 0 it writes zero.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float bexp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------ delta
// D[row] = sum_c dO[row, c] * O[row, c] in fp32 from bf16, one row per 16
// threads (8 elements each, 16-byte loads), rows = B * Hq * N.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ out,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            float* __restrict__ delta, int64_t rows) {
  constexpr int kThreadsPerRow = D / 8;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = t / kThreadsPerRow;
  const int part = static_cast<int>(t % kThreadsPerRow);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(out + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), acc);
      acc = fmaf(__uint_as_float(av[i] & 0xffff0000u), __uint_as_float(bv[i] & 0xffff0000u), acc);
    }
  }
#pragma unroll
  for (int o = kThreadsPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (row < rows && part == 0) delta[row] = acc;
}

// ------------------------------------------------------------------ layouts
// dQ kernel: Q and dO tiles of the work item, then a ring of (K_j, V_j) stages.
// dK/dV kernel: K and V tiles of the work item, then a ring of (Q_i, dO_i)
// stages, plus the per-step log-sum-exp and D vectors of the query tile.
template <int D>
struct BwdSmem {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kChunks = D / 64;                        // 128-byte column chunks
  static constexpr uint32_t kChunkBytes = kTile * 128;          // 128 rows x 128 B
  static constexpr uint32_t kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr uint32_t kFixOff = 0;                        // two fixed tiles
  static constexpr uint32_t kRingOff = 2 * kTileBytes;          // stages of two tiles
  // Per-step query vectors (log-sum-exp, D): 4 warps x 2 buffers x 2 x 128 floats.
  static constexpr uint32_t kVecOff = kRingOff + kStages * 2 * kTileBytes;
  // Fused kernel: dS^T of one 64-query half (128 key rows x 128 B, 128-byte
  // swizzle), the B operand of dQ^T = K^T dS^T.
  static constexpr uint32_t kDsOff = kVecOff + 4 * 2 * 2 * kTile * 4;
  static constexpr uint32_t kDsBytes = kTile * kHalf * 2;
  static constexpr uint32_t kBarOff = kDsOff + kDsBytes;
  static constexpr int kFixFull = 0;
  static constexpr int kFixEmpty = 1;
  static constexpr int kRingFull = 2;
  static constexpr int kRingEmpty = kRingFull + kStages;
  static constexpr int kSFull = kRingEmpty + kStages;  // two: one per score half
  static constexpr int kPFull = kSFull + 2;             // two: one per score half
  static constexpr int kAccDone = kPFull + 2;
  static constexpr int kAccFree = kAccDone + 1;
  static constexpr int kFin = kAccFree + 1;
  static constexpr int kDqFull = kFin + 1;    // two: dQ^T of a half is in TMEM
  static constexpr int kDqFree = kDqFull + 2; // two: the dQ warps have read it
  static constexpr int kDsFree = kDqFree + 2; // the dQ^T product has read the staged dS^T
  // Full-tile key-tile kernel: a slot's Q and dO tiles land and are released
  // separately (kRingFull / kRingEmpty then cover Q alone).
  static constexpr int kRing2Full = kDsFree + 1;
  static constexpr int kRing2Empty = kRing2Full + kStages;
  static constexpr int kNumBars = kRing2Empty + kStages;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack to align the base to 1024 B
  static_assert(kDsOff % 1024 == 0, "swizzled dS^T tile alignment");
  static_assert(kAlloc <= 232448, "shared memory per CTA");
  // TMEM columns: two buffers of 64-wide score halves, each S (or S^T) then
  // dP (or dP^T), then the accumulators.  The key-tile kernel writes P^T and
  // dS^T (bf16, 32 columns each) over the S^T half, which leaves the dP^T half
  // free for the fused kernel's dQ^T of that half (64 fp32 columns).
  static constexpr uint32_t kColAcc0 = 256, kColAcc1 = 256 + D;
  static __device__ __forceinline__ uint32_t col_s(int h) { return h * 128; }
  static __device__ __forceinline__ uint32_t col_p(int h) { return h * 128 + 64; }
};

// Operand descriptors of a tile stored as 128 rows x D (K-major: the D axis
// is the reduction axis) or read as the MN-major B operand of a TS MMA (the
// 128 rows are the reduction axis).
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  return smem_desc_sw128(saddr, 16, 1024);
}
template <int D>
__device__ __forceinline__ uint32_t kmajor_off(int kk) {
  return ((kk >> 2) * BwdSmem<D>::kChunkBytes + (kk & 3) * 32) >> 4;
}
template <int D>
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t saddr) {
  return smem_desc_sw128(saddr, BwdSmem<D>::kChunkBytes, 1024);
}

// Store one 128-column-or-less fp32 TMEM row segment (this thread's row) as
// bf16 times `mul` to a global row; TMEM columns [col0, col0 + D).
template <int D>
__device__ __forceinline__ void store_acc_row(uint32_t tacc, float mul, __nv_bfloat16* dst_row, bool ok) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_load_32cols(tacc + cc * 32, o);
    if (ok) {
      uint32_t h[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) h[i] = bf16x2_rn(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
      uint4* dst = reinterpret_cast<uint4*>(dst_row) + cc * 4;
#pragma unroll
      for (int v = 0; v < 4; ++v) dst[v] = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
    }
  }
}

// ------------------------------------------------------------------ query-tile work items and loader
struct DqItem {
  int b, hq, hkv, m, lo, hi;
};
__device__ __forceinline__ DqItem dq_item(const BwdParams& p, int i) {
  DqItem it;
  const int bh = i / p.num_blk;
  it.m = p.num_blk - 1 - (i - bh * p.num_blk);  // longest query tile of a head first
  it.b = bh / p.Hq;
  it.hq = bh - it.b * p.Hq;
  it.hkv = it.hq / p.group;
  key_tiles_of_query_tile(p, it.m, it.lo, it.hi);
  return it;
}

template <int D>
__device__ __forceinline__ void dq_loader(const BwdParams& p, uint32_t sbase, const BwdWaiter& w) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const uint64_t pol_kv = l2_policy_evict_last();
  const uint64_t pol_q = l2_policy_evict_first();
  uint32_t n = 0;         // ring loads issued
  uint32_t fix_issued = 0;  // Q / dO tile pairs issued
  int items = 0;
  bool ok = true;
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x, ++items) {
    const DqItem it = dq_item(p, i);
    if (items > 0 && !w.wait(bar(L::kFixEmpty), (items - 1) & 1, (kBKernelDq << 12) | (kBRoleLoader << 8) | L::kFixEmpty)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(bar(L::kFixFull), 2 * L::kTileBytes);
    ++fix_issued;
    const int zq = it.b * p.Hq + it.hq;
#pragma unroll
    for (int c = 0; c < L::kChunks; ++c) {
      tma_load_3d(sbase + L::kFixOff + c * L::kChunkBytes, &p.tm_q, bar(L::kFixFull), c * 64, it.m * kTile, zq, pol_q);
      tma_load_3d(sbase + L::kFixOff + L::kTileBytes + c * L::kChunkBytes, &p.tm_do, bar(L::kFixFull), c * 64,
                  it.m * kTile, zq, pol_q);
    }
    const int zk = it.b * p.Hkv + it.hkv;
    for (int j = it.lo; j <= it.hi; ++j, ++n) {
      const uint32_t slot = n % L::kStages;
      if (n >= (uint32_t)L::kStages &&
          !w.wait(bar(L::kRingEmpty + slot), ((n / L::kStages) - 1) & 1,
                  (kBKernelDq << 12) | (kBRoleLoader << 8) | (L::kRingEmpty + slot))) {
        ok = false;
        break;
      }
      const uint32_t dst = sbase + L::kRingOff + slot * 2 * L::kTileBytes;
      mbar_arrive_expect_tx(bar(L::kRingFull + slot), 2 * L::kTileBytes);
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c) {
        tma_load_3d(dst + c * L::kChunkBytes, &p.tm_k, bar(L::kRingFull + slot), c * 64, j * kTile, zk, pol_kv);
        tma_load_3d(dst + L::kTileBytes + c * L::kChunkBytes, &p.tm_v, bar(L::kRingFull + slot), c * 64, j * kTile, zk,
                    pol_kv);
      }
    }
  }
  // Drain: every copy this thread started must land before the CTA exits.
  for (uint32_t s = 0; s < (uint32_t)L::kStages; ++s) {
    if (n > s) {
      const uint32_t last = s + ((n - 1 - s) / L::kStages) * L::kStages;
      w.drain(bar(L::kRingFull + s), (last / L::kStages) & 1, (kBKernelDq << 12) | (kBRoleLoader << 8) | (L::kRingFull + s));
    }
  }
  if (fix_issued > 0)
    w.drain(bar(L::kFixFull), (fix_issued - 1) & 1, (kBKernelDq << 12) | (kBRoleLoader << 8) | L::kFixFull);
}

// ------------------------------------------------------------------ key-tile work items and loader; the fused kernel (64-query halves)
struct DkvItem {
  int b, hkv, n, qlo, qhi, steps;  // steps = group * (qhi - qlo + 1)
};
__device__ __forceinline__ DkvItem dkv_item(const BwdParams& p, int i) {
  DkvItem it;
  const int bk = i / p.num_blk;
  it.n = i - bk * p.num_blk;  // under a causal mask the first key tiles see the most queries
  it.b = bk / p.Hkv;
  it.hkv = bk - it.b * p.Hkv;
  query_tiles_of_key_tile(p, it.n, it.qlo, it.qhi);
  it.steps = p.group * (it.qhi - it.qlo + 1);
  return it;
}
// Step s of an item: query head hkv * group + s / (qhi - qlo + 1), query tile qlo + s % (...).
__device__ __forceinline__ void dkv_step(const BwdParams& p, const DkvItem& it, int s, int& hq, int& m) {
  const int per_head = it.qhi - it.qlo + 1;
  const int h = s / per_head;
  hq = it.hkv * p.group + h;
  m = it.qlo + (s - h * per_head);
}

// kSplit (the full-tile key-tile kernel): a slot's Q and dO tiles land and are
// released through their own barriers, so Q can be refilled as soon as the
// products that read it are done.
template <int D, bool kSplit>
__device__ __forceinline__ void dkv_loader(const BwdParams& p, uint32_t sbase, const BwdWaiter& w) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const uint64_t pol_kv = l2_policy_evict_first();
  const uint64_t pol_q = l2_policy_evict_last();
  const int code = (kBKernelDkdv << 12) | (kBRoleLoader << 8);
  uint32_t n = 0;
  uint32_t fix_issued = 0;  // K / V tile pairs issued
  int items = 0;
  bool ok = true;
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x, ++items) {
    const DkvItem it = dkv_item(p, i);
    if (items > 0 && !w.wait(bar(L::kFixEmpty), (items - 1) & 1, code | L::kFixEmpty)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(bar(L::kFixFull), 2 * L::kTileBytes);
    ++fix_issued;
    const int zk = it.b * p.Hkv + it.hkv;
#pragma unroll
    for (int c = 0; c < L::kChunks; ++c) {
      tma_load_3d(sbase + L::kFixOff + c * L::kChunkBytes, &p.tm_k, bar(L::kFixFull), c * 64, it.n * kTile, zk, pol_kv);
      tma_load_3d(sbase + L::kFixOff + L::kTileBytes + c * L::kChunkBytes, &p.tm_v, bar(L::kFixFull), c * 64,
                  it.n * kTile, zk, pol_kv);
    }
    for (int s = 0; s < it.steps; ++s, ++n) {
      int hq, m;
      dkv_step(p, it, s, hq, m);
      const uint32_t slot = n % L::kStages;
      const uint32_t dst = sbase + L::kRingOff + slot * 2 * L::kTileBytes;
      const int zq = it.b * p.Hq + hq;
      const int do_full = kSplit ? L::kRing2Full : L::kRingFull;
      if (n >= (uint32_t)L::kStages &&
          !w.wait(bar(L::kRingEmpty + slot), ((n / L::kStages) - 1) & 1, code | (L::kRingEmpty + slot))) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(bar(L::kRingFull + slot), (kSplit ? 1 : 2) * L::kTileBytes);
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(dst + c * L::kChunkBytes, &p.tm_q, bar(L::kRingFull + slot), c * 64, m * kTile, zq, pol_q);
      if constexpr (kSplit) {
        if (n >= (uint32_t)L::kStages &&
            !w.wait(bar(L::kRing2Empty + slot), ((n / L::kStages) - 1) & 1, code | (L::kRing2Empty + slot))) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(do_full + slot), L::kTileBytes);
      }
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(dst + L::kTileBytes + c * L::kChunkBytes, &p.tm_do, bar(do_full + slot), c * 64, m * kTile, zq,
                    pol_q);
    }
  }
  for (uint32_t s = 0; s < (uint32_t)L::kStages; ++s) {
    if (n > s) {
      const uint32_t last = s + ((n - 1 - s) / L::kStages) * L::kStages;
      w.drain(bar(L::kRingFull + s), (last / L::kStages) & 1, code | (L::kRingFull + s));
      if constexpr (kSplit) w.drain(bar(L::kRing2Full + s), (last / L::kStages) & 1, code | (L::kRing2Full + s));
    }
  }
  if (fix_issued > 0) w.drain(bar(L::kFixFull), (fix_issued - 1) & 1, code | L::kFixFull);
}

template <int D>
__device__ __forceinline__ void dkv_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w) {
  using L = BwdSmem<D>;
  static_assert(D == 128, "the fused dQ^T product has M = d = 128");
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr uint32_t idesc_ss = idesc_bf16_f32(kTile, kHalf, false);  // 128 keys x 64 queries
  constexpr uint32_t idesc_ts = idesc_bf16_f32(kTile, D, true);
  // dQ^T (d x 64 queries) = K^T dS^T: A = the K tile read MN-major (d is its
  // contiguous axis), B = the staged dS^T, MN-major (queries contiguous).
  constexpr uint32_t idesc_dq = idesc_bf16_f32(D, kHalf, true) | (1u << 15);
  const uint64_t kt_desc = mnmajor_desc<D>(sbase + L::kFixOff);
  const uint64_t ds_desc = smem_desc_sw128(sbase + L::kDsOff, L::kChunkBytes, 1024);
  uint32_t dq_cnt[2] = {0, 0};  // dQ^T products issued, per half
  const uint32_t t_dv = tmem + L::kColAcc0, t_dk = tmem + L::kColAcc1;
  const uint64_t k_desc = kmajor_desc<D>(sbase + L::kFixOff);
  const uint64_t v_desc = kmajor_desc<D>(sbase + L::kFixOff + L::kTileBytes);
  const int code = (kBKernelFused << 12) | (kBRoleMma << 8);
  uint32_t n = 0;
  uint32_t p_cnt0 = 0, p_cnt1 = 0;  // P / dS halves consumed, per half
  int items = 0;
  bool ok = true;
  // dV += P^T_h dO_h and dK += dS^T_h Q_h for query half h of ring slot `slot`.
  auto issue_dkv = [&](int h, uint32_t slot, bool first) -> bool {
    if (!w.wait_warp(bar(L::kPFull + h), (h ? p_cnt1 : p_cnt0) & 1, code | (L::kPFull + h))) return false;
    if (h) ++p_cnt1; else ++p_cnt0;
    if (first && items > 0 && !w.wait_warp(bar(L::kAccFree), (items - 1) & 1, code | L::kAccFree)) return false;
    tc_fence_after_sync();
    // dQ^T_h over this tile's 128 keys, into the dP^T columns of half h.  It goes
    // ahead of dV and dK so that the dQ warps read it out while those execute:
    // the next S^T into these columns waits for that read.
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      mma_bf16_ss_elect(tmem + L::col_p(h), kt_desc + ((kk * 2048) >> 4), ds_desc + ((kk * 2048) >> 4), idesc_dq,
                        kk > 0 ? 1u : 0u);
    tc_commit_elect(bar(L::kDqFull + h));
    tc_commit_elect(bar(L::kDsFree));
    ++dq_cnt[h];
    const uint32_t qaddr = sbase + L::kRingOff + slot * 2 * L::kTileBytes + h * kHalf * 128;
    const uint64_t qb = mnmajor_desc<D>(qaddr), dob = mnmajor_desc<D>(qaddr + L::kTileBytes);
#pragma unroll
    for (int kk = 0; kk < kHalf / 16; ++kk) {
      const uint32_t acc = (kk > 0 || !first) ? 1u : 0u;
      mma_bf16_ts_elect(t_dv, tmem + L::col_s(h) + kk * 8, dob + ((kk * 2048) >> 4), idesc_ts, acc);
      mma_bf16_ts_elect(t_dk, tmem + L::col_s(h) + 32 + kk * 8, qb + ((kk * 2048) >> 4), idesc_ts, acc);
    }
    return true;
  };
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x, ++items) {
    const DkvItem it = dkv_item(p, i);
    if (!w.wait_warp(bar(L::kFixFull), items & 1, code | L::kFixFull)) break;
    tc_fence_after_sync();
    uint32_t prev_slot = 0;
    bool first = true;
    for (int s = 0; s < it.steps && ok; ++s, ++n) {
      const uint32_t slot = n % L::kStages;
      const uint32_t qaddr = sbase + L::kRingOff + slot * 2 * L::kTileBytes;
      if (!w.wait_warp(bar(L::kRingFull + slot), (n / L::kStages) & 1, code | (L::kRingFull + slot))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        // The dQ warps have read the previous dQ^T_h out of these columns.
        if (dq_cnt[h] > 0 &&
            !w.wait_warp(bar(L::kDqFree + h), (dq_cnt[h] - 1) & 1, code | (L::kDqFree + h))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        // S^T_h = K Q_h^T and dP^T_h = V dO_h^T (queries 64h .. 64h+63 of the tile).
        const uint64_t q_desc = kmajor_desc<D>(qaddr + h * kHalf * 128);
        const uint64_t do_desc = kmajor_desc<D>(qaddr + L::kTileBytes + h * kHalf * 128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = kmajor_off<D>(kk);
          mma_bf16_ss_elect(tmem + L::col_s(h), k_desc + off, q_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
          mma_bf16_ss_elect(tmem + L::col_p(h), v_desc + off, do_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
        tc_commit_elect(bar(L::kSFull + h));
        if (h == 1 || s > 0) {
          if (!issue_dkv(1 - h, h == 1 ? slot : prev_slot, first)) {
            ok = false;
            break;
          }
          first = false;
          if (h == 0) tc_commit_elect(bar(L::kRingEmpty + prev_slot));  // previous Q, dO tile done
        }
      }
      prev_slot = slot;
    }
    if (!ok) break;
    if (!issue_dkv(1, prev_slot, first)) break;  // the item's last half
    tc_commit_elect(bar(L::kFixEmpty));  // K (read by the dQ^T products too), V
    tc_commit_elect(bar(L::kRingEmpty + prev_slot));
    tc_commit_elect(bar(L::kAccDone));
  }
}

template <int D>
__device__ __forceinline__ void dkv_elem(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w,
                                         int warp, int lane) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const int r = warp * 32 + lane;  // key row of the tile = TMEM lane
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t t_dv = tmem + lane_bits + L::kColAcc0, t_dk = tmem + lane_bits + L::kColAcc1;
  // This warp's two buffers of a step's per-query vectors: the log-sum-exp and D
  // of the 128 query rows, copied in (zero past the sequence) while the step
  // before is computed, then negated in place (the LSE also scaled by log2 e).
  const uint32_t vec_saddr = sbase + L::kVecOff + warp * 4 * kTile * 4;
  float* const vec_base = reinterpret_cast<float*>(__cvta_shared_to_generic(vec_saddr));
  auto fetch_vectors = [&](int b, int hq, int m, uint32_t buf) {
    const size_t bhq = (static_cast<size_t>(b) * p.Hq + hq) * p.N;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t, q = m * kTile + c;
      const bool in = q < p.N;
      const size_t idx = bhq + (in ? q : 0);
      const uint32_t dst = vec_saddr + (buf * 2 * kTile + c) * 4;
      cp_async_4(dst, p.lse + idx, in ? 4u : 0u);
      cp_async_4(dst + kTile * 4, p.delta + idx, in ? 4u : 0u);
    }
    cp_async_commit();
  };
  const float c2 = p.scale_log2;
  const uint64_t c2x2 = f32x2_pack(c2, c2);
  const int code = (kBKernelFused << 12) | (kBRoleElem << 8);
  uint32_t s_cnt = 0;
  uint32_t ds_cnt = 0;  // fused kernel: dS^T halves staged in shared memory
  bool fetched = false;  // the next step's vectors are already on their way
  int items = 0;
  for (int i = blockIdx.x; i < p.num_items; i += gridDim.x, ++items) {
    const DkvItem it = dkv_item(p, i);
    const int key = it.n * kTile + r;
    bool ok = true;
    for (int s = 0; s < it.steps && ok; ++s, ++s_cnt) {
      int hq, m;
      dkv_step(p, it, s, hq, m);
      const uint32_t buf = s_cnt & 1;
      float* const s_lse = vec_base + buf * 2 * kTile;
      float* const s_dlt = s_lse + kTile;
      {
        if (!fetched) fetch_vectors(it.b, hq, m, buf);
        cp_async_wait_all();
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = lane + 32 * t;
          s_lse[c] = -s_lse[c] * kLog2e;
          s_dlt[c] = -s_dlt[c];
        }
        __syncwarp();  // every lane's entries are in place; the other buffer's last reads are done
        // Start the next step's copies (the next item's first step after the last one).
        fetched = false;
        if (s + 1 < it.steps) {
          int hq2, m2;
          dkv_step(p, it, s + 1, hq2, m2);
          fetch_vectors(it.b, hq2, m2, buf ^ 1);
          fetched = true;
        } else if (i + static_cast<int>(gridDim.x) < p.num_items) {
          const DkvItem nx = dkv_item(p, i + gridDim.x);
          int hq2, m2;
          dkv_step(p, nx, 0, hq2, m2);
          fetch_vectors(nx.b, hq2, m2, buf ^ 1);
          fetched = true;
        }
      }
      const bool partial = block_is_partial(p, m, it.n);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (!w.wait_warp(bar(L::kSFull + h), s_cnt & 1, code | (L::kSFull + h))) {
          ok = false;
          break;
        }
        // The staged dS^T is rewritten below: the previous dQ^T product must have read it.
        if (ds_cnt > 0 && !w.wait_warp(bar(L::kDsFree), (ds_cnt - 1) & 1, code | L::kDsFree)) {
          ok = false;
          break;
        }
        ++ds_cnt;
        tc_fence_after_sync();
        // Query columns of this half that see the key: lo_c <= c <= hi_c
        // (applied on partial tiles, where masked scores become -inf).
        const int q0 = m * kTile + h * kHalf;
        const int hi_c =
            (key < p.N) ? min(p.N - 1, p.mask_kind == kBMaskWindow ? key + p.window - 1 : p.N - 1) - q0 : -1;
        const int lo_c = (p.mask_kind == kBMaskFull) ? 0 : key - q0;
        const uint32_t t_s = tmem + lane_bits + L::col_s(h), t_p = tmem + lane_bits + L::col_p(h);
        uint32_t pk[2][16], dk[2][16];
#pragma unroll
        for (int chunk = 0; chunk < 2; ++chunk) {
          uint32_t sv[32], pv[32];
          tmem_load_2x32cols(t_s + chunk * 32, t_p + chunk * 32, sv, pv);
          if (partial) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = chunk * 32 + e;
              if (c > hi_c || c < lo_c) sv[e] = 0xff800000u;  // -inf
            }
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            // Column pairs: x = s c - lse, p = 2^x, dS = p (dP - D), with the
            // pair's (-lse, -D) read as 8-byte loads and packed fp32 arithmetic.
            const int c = h * kHalf + chunk * 32 + e;  // query column within the tile (even)
            const float2 nl = *reinterpret_cast<const float2*>(s_lse + c);
            const float2 nd = *reinterpret_cast<const float2*>(s_dlt + c);
            float x0, x1, p0, p1, d0, d1;
            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2x2,
                                   f32x2_pack(nl.x, nl.y)),
                         x0, x1);
            p0 = bexp2(x0);
            p1 = bexp2(x1);
            f32x2_unpack(f32x2_mul(f32x2_pack(p0, p1), f32x2_add(f32x2_pack(__uint_as_float(pv[e]),
                                                                            __uint_as_float(pv[e + 1])),
                                                                f32x2_pack(nd.x, nd.y))),
                         d0, d1);
            pk[chunk][e >> 1] = bf16x2_rn(p0, p1);
            dk[chunk][e >> 1] = bf16x2_rn(d0, d1);
          }
        }
        // Stage dS^T for dQ^T = K^T dS^T: this key's row of 64 queries is 128 B
        // (eight 16-byte chunks, chunk c stored at c ^ (row & 7): the 128-byte
        // swizzle of an MN-major operand).
        const uint32_t row_addr = sbase + L::kDsOff + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(row_addr + ((c ^ (r & 7)) << 4), dk[c >> 2][(c & 3) * 4], dk[c >> 2][(c & 3) * 4 + 1],
                       dk[c >> 2][(c & 3) * 4 + 2], dk[c >> 2][(c & 3) * 4 + 3]);
        fence_proxy_async_smem();
        // P^T and dS^T (bf16, 32 columns each) over this half's S^T columns.
        tmem_store_16cols(t_s, pk[0]);
        tmem_store_16cols(t_s + 16, pk[1]);
        tmem_store_16cols(t_s + 32, dk[0]);
        tmem_store_16cols(t_s + 48, dk[1]);
        tmem_store_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kPFull + h));
      }
    }
    if (!ok) break;
    if (!w.wait_warp(bar(L::kAccDone), items & 1, code | L::kAccDone)) break;
    tc_fence_after_sync();
    const bool key_ok = key < p.N;
    const size_t krow = (static_cast<size_t>(it.b) * p.Hkv + it.hkv) * p.N + (key_ok ? key : 0);
    store_acc_row<D>(t_dv, 1.f, p.dv + krow * D, key_ok);
    store_acc_row<D>(t_dk, p.scale, p.dk + krow * D, key_ok);
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kAccFree));
  }
  cp_async_wait_all();  // no copy into shared memory outlives the CTA (a run that stopped early)
  tmem_store_wait();
}

// ------------------------------------------------------------------ dQ kernel, full tiles
// The query-tile kernel with whole 128-key products, arranged like the full-tile
// key-tile kernel: X = [0, 128) holds S = Q K^T; Y = [128, 256) holds dP = dO V^T,
// then dS (bf16, [128, 192)); dQ after them.  Per key tile g the issuer queues
//   S(g) -> X        once the elementwise warps have loaded S(g-1) out of X,
//   dQ += dS(g-1) K  once dS(g-1) is in Y,
//   dP(g) -> Y       behind it,
// so the exponentials of tile g run while the tensor core does dQ of tile g-1
// and dP of tile g.  P is kept as bf16 until dP arrives.
template <int D>
__device__ __forceinline__ void dqf_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr int kSFull = L::kSFull, kDpFull = L::kSFull + 1;
  constexpr int kPFull = L::kPFull, kXFree = L::kPFull + 1;
  constexpr uint32_t idesc_ss = idesc_bf16_f32(kTile, kTile, false);  // 128 queries x 128 keys
  constexpr uint32_t idesc_ts = idesc_bf16_f32(kTile, D, true);
  const uint32_t tX = tmem, tY = tmem + 128, t_acc = tmem + L::kColAcc0;
  const uint64_t q_desc = kmajor_desc<D>(sbase + L::kFixOff);
  const uint64_t do_desc = kmajor_desc<D>(sbase + L::kFixOff + L::kTileBytes);
  const int code = (kBKernelDqFull << 12) | (kBRoleMma << 8);
  uint32_t g = 0, b_cnt = 0;
  int acc_items = 0, items = 0;
  bool ok = true;
  bool pend = false, pend_first = false, pend_last = false;
  uint32_t pend_slot = 0;
  auto issue_b = [&]() -> bool {
    if (!w.wait_warp(bar(kPFull), b_cnt & 1, code | kPFull)) return false;
    if (pend_first && acc_items > 0 && !w.wait_warp(bar(L::kAccFree), (acc_items - 1) & 1, code | L::kAccFree))
      return false;
    tc_fence_after_sync();
    const uint64_t kb = mnmajor_desc<D>(sbase + L::kRingOff + pend_slot * 2 * L::kTileBytes);
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      mma_bf16_ts_elect(t_acc, tY + kk * 8, kb + ((kk * 2048) >> 4), idesc_ts, (kk > 0 || !pend_first) ? 1u : 0u);
    tc_commit_elect(bar(L::kRingEmpty + pend_slot));  // that tile's K (and V, read by its dP) are done
    if (pend_last) {
      tc_commit_elect(bar(L::kAccDone));
      ++acc_items;
    }
    ++b_cnt;
    pend = false;
    return true;
  };
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x, ++items) {
    const DqItem it = dq_item(p, i);
    if (!w.wait_warp(bar(L::kFixFull), items & 1, code | L::kFixFull)) break;
    tc_fence_after_sync();
    for (int j = it.lo; j <= it.hi; ++j, ++g) {
      const uint32_t slot = g % L::kStages;
      if (!w.wait_warp(bar(L::kRingFull + slot), (g / L::kStages) & 1, code | (L::kRingFull + slot)) ||
          (g > 0 && !w.wait_warp(bar(kXFree), (g - 1) & 1, code | kXFree))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t kaddr = sbase + L::kRingOff + slot * 2 * L::kTileBytes;
      const uint64_t k_desc = kmajor_desc<D>(kaddr), v_desc = kmajor_desc<D>(kaddr + L::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = kmajor_off<D>(kk);
        mma_bf16_ss_elect(tX, q_desc + off, k_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
      tc_commit_elect(bar(kSFull));
      if (pend && !issue_b()) {
        ok = false;
        break;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = kmajor_off<D>(kk);
        mma_bf16_ss_elect(tY, do_desc + off, v_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
      tc_commit_elect(bar(kDpFull));
      if (j == it.hi) tc_commit_elect(bar(L::kFixEmpty));  // Q and dO read by the item's last products
      pend = true;
      pend_slot = slot;
      pend_first = (j == it.lo);
      pend_last = (j == it.hi);
    }
  }
  if (ok && pend) issue_b();
}

template <int D>
__device__ __forceinline__ void dqf_elem(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w,
                                         int warp, int lane) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr int kSFull = L::kSFull, kDpFull = L::kSFull + 1;
  constexpr int kPFull = L::kPFull, kXFree = L::kPFull + 1;
  const int r = warp * 32 + lane;  // row of the query tile = TMEM lane
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tX = tmem + lane_bits, tY = tmem + lane_bits + 128, t_acc = tmem + lane_bits + L::kColAcc0;
  const float c2 = p.scale_log2;
  const int code = (kBKernelDqFull << 12) | (kBRoleElem << 8);
  uint32_t g = 0;
  int items = 0;
  for (int i = blockIdx.x; i < p.num_items; i += gridDim.x, ++items) {
    const DqItem it = dq_item(p, i);
    const int row = it.m * kTile + r;
    const bool row_ok = row < p.N;
    const size_t bhrow = (static_cast<size_t>(it.b) * p.Hq + it.hq) * p.N + (row_ok ? row : 0);
    const float lse2 = row_ok ? p.lse[bhrow] * kLog2e : 0.f;
    const float dlt = row_ok ? p.delta[bhrow] : 0.f;
    const uint64_t c2x2 = f32x2_pack(c2, c2), nlse2x2 = f32x2_pack(-lse2, -lse2), ndlt2 = f32x2_pack(-dlt, -dlt);
    bool ok = true;
    for (int j = it.lo; j <= it.hi && ok; ++j, ++g) {
      if (!w.wait_warp(bar(kSFull), g & 1, code | kSFull)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t sv[128];
      tmem_load_128cols(tX, sv);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kXFree));
      if (block_is_partial(p, it.m, j)) {
        // Visible key columns of this row: lo_c <= c <= hi_c.
        const int j0 = j * kTile;
        const int hi_c = row_ok ? min(p.N - 1, p.mask_kind == kBMaskFull ? p.N - 1 : row) - j0 : -1;
        const int lo_c = (p.mask_kind == kBMaskWindow) ? row - p.window + 1 - j0 : 0;
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c > hi_c || c < lo_c) sv[c] = 0xff800000u;  // -inf
      }
      uint32_t pk[kTile / 2];  // P, bf16 pairs of keys
#pragma unroll
      for (int c = 0; c < kTile; c += 2) {
        float x0, x1;
        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2, nlse2x2), x0,
                     x1);
        pk[c >> 1] = bf16x2_rn(bexp2(x0), bexp2(x1));
      }
      if (!w.wait_warp(bar(kDpFull), g & 1, code | kDpFull)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t ds[kTile / 2];
#pragma unroll
      for (int chunk = 0; chunk < 4; ++chunk) {
        uint32_t pv[32];
        tmem_load_32cols(tY + chunk * 32, pv);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t pw = pk[(chunk * 32 + e) >> 1];
          float d0, d1;
          f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(pw << 16), __uint_as_float(pw & 0xffff0000u)),
                                 f32x2_add(f32x2_pack(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])), ndlt2)),
                       d0, d1);
          ds[(chunk * 32 + e) >> 1] = bf16x2_rn(d0, d1);
        }
      }
      // dS over Y's first 64 columns (all of dP has been read).
      tmem_store_32cols(tY, *reinterpret_cast<const uint32_t(*)[32]>(&ds[0]));
      tmem_store_32cols(tY + 32, *reinterpret_cast<const uint32_t(*)[32]>(&ds[32]));
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kPFull));
    }
    if (!ok) break;
    if (!w.wait_warp(bar(L::kAccDone), items & 1, code | L::kAccDone)) break;
    tc_fence_after_sync();
    store_acc_row<D>(t_acc, p.scale, p.dq + bhrow * D, row_ok);
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kAccFree));
  }
  tmem_store_wait();
}

// ------------------------------------------------------------------ dK/dV kernel, full tiles
// The key-tile kernel with whole 128-query products: S^T and dP^T of a step are
// single M = 128, N = 128 products (narrower products keep the tensor pipe far
// from busy), and the elementwise warps still overlap the tensor core.  TMEM:
// X = [0, 128) holds S^T; Y = [128, 256) holds dP^T, then P^T (bf16, [128, 192))
// and dS^T ([192, 256)); dV and dK after them.  Per step g the issuer queues
//   S^T(g) -> X      once the elementwise warps have loaded S^T(g-1) out of X,
//   dV, dK (g-1)     once P^T(g-1) and dS^T(g-1) are in Y,
//   dP^T(g) -> Y     behind them (in issue order, so after they read Y),
// so the exponentials of step g run while the tensor core does dV, dK of step g-1
// and dP^T of step g.  P is kept as bf16 until dP arrives; dS = P (dP - D) is
// formed from that bf16 P.
template <int D>
__device__ __forceinline__ void dkvf_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr int kSFull = L::kSFull, kDpFull = L::kSFull + 1;  // barrier indices of this kernel
  constexpr int kPFull = L::kPFull, kXFree = L::kPFull + 1;
  constexpr uint32_t idesc_ss = idesc_bf16_f32(kTile, kTile, false);  // 128 keys x 128 queries
  constexpr uint32_t idesc_ts = idesc_bf16_f32(kTile, D, true);
  const uint32_t tX = tmem, tY = tmem + 128, t_dv = tmem + L::kColAcc0, t_dk = tmem + L::kColAcc1;
  const uint64_t k_desc = kmajor_desc<D>(sbase + L::kFixOff);
  const uint64_t v_desc = kmajor_desc<D>(sbase + L::kFixOff + L::kTileBytes);
  const int code = (kBKernelDkdvFull << 12) | (kBRoleMma << 8);
  uint32_t g = 0;        // steps whose S^T and dP^T are issued
  uint32_t b_cnt = 0;    // steps whose dV and dK are issued
  int acc_items = 0;     // items whose accumulators are complete (AccDone committed)
  int items = 0;
  bool ok = true;
  bool pend = false, pend_first = false, pend_last = false;  // step g-1's dV, dK still to issue
  uint32_t pend_slot = 0;
  auto issue_b = [&]() -> bool {
    if (!w.wait_warp(bar(kPFull), b_cnt & 1, code | kPFull)) return false;
    if (pend_first && acc_items > 0 && !w.wait_warp(bar(L::kAccFree), (acc_items - 1) & 1, code | L::kAccFree))
      return false;
    tc_fence_after_sync();
    const uint32_t qaddr = sbase + L::kRingOff + pend_slot * 2 * L::kTileBytes;
    const uint64_t qb = mnmajor_desc<D>(qaddr), dob = mnmajor_desc<D>(qaddr + L::kTileBytes);
    // dK first: the slot's Q, which the next S^T of that slot needs, is released first.
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      mma_bf16_ts_elect(t_dk, tY + 64 + kk * 8, qb + ((kk * 2048) >> 4), idesc_ts, (kk > 0 || !pend_first) ? 1u : 0u);
    tc_commit_elect(bar(L::kRingEmpty + pend_slot));  // that step's Q is read
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      mma_bf16_ts_elect(t_dv, tY + kk * 8, dob + ((kk * 2048) >> 4), idesc_ts, (kk > 0 || !pend_first) ? 1u : 0u);
    tc_commit_elect(bar(L::kRing2Empty + pend_slot));  // and its dO
    if (pend_last) {
      tc_commit_elect(bar(L::kAccDone));
      ++acc_items;
    }
    ++b_cnt;
    pend = false;
    return true;
  };
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x, ++items) {
    const DkvItem it = dkv_item(p, i);
    if (!w.wait_warp(bar(L::kFixFull), items & 1, code | L::kFixFull)) break;
    tc_fence_after_sync();
    for (int s = 0; s < it.steps; ++s, ++g) {
      const uint32_t slot = g % L::kStages;
      if (!w.wait_warp(bar(L::kRingFull + slot), (g / L::kStages) & 1, code | (L::kRingFull + slot)) ||
          (g > 0 && !w.wait_warp(bar(kXFree), (g - 1) & 1, code | kXFree))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t qaddr = sbase + L::kRingOff + slot * 2 * L::kTileBytes;
      const uint64_t q_desc = kmajor_desc<D>(qaddr), do_desc = kmajor_desc<D>(qaddr + L::kTileBytes);
      // (dO of this slot is waited for below, before dP^T.)
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = kmajor_off<D>(kk);
        mma_bf16_ss_elect(tX, k_desc + off, q_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
      tc_commit_elect(bar(kSFull));
      if (pend && !issue_b()) {
        ok = false;
        break;
      }
      if (!w.wait_warp(bar(L::kRing2Full + slot), (g / L::kStages) & 1, code | (L::kRing2Full + slot))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = kmajor_off<D>(kk);
        mma_bf16_ss_elect(tY, v_desc + off, do_desc + off, idesc_ss, kk > 0 ? 1u : 0u);
      }
      tc_commit_elect(bar(kDpFull));
      if (s == it.steps - 1) tc_commit_elect(bar(L::kFixEmpty));  // K and V read by the item's last products
      pend = true;
      pend_slot = slot;
      pend_first = (s == 0);
      pend_last = (s == it.steps - 1);
    }
  }
  if (ok && pend) issue_b();  // the last step's dV, dK
}

template <int D>
__device__ __forceinline__ void dkvf_elem(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w,
                                          int warp, int lane) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  constexpr int kSFull = L::kSFull, kDpFull = L::kSFull + 1;
  constexpr int kPFull = L::kPFull, kXFree = L::kPFull + 1;
  const int r = warp * 32 + lane;  // key row of the tile = TMEM lane
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tX = tmem + lane_bits, tY = tmem + lane_bits + 128;
  const uint32_t t_dv = tmem + lane_bits + L::kColAcc0, t_dk = tmem + lane_bits + L::kColAcc1;
  // Per-step query vectors, as in the half-tile kernel: copied a step ahead, then negated.
  const uint32_t vec_saddr = sbase + L::kVecOff + warp * 4 * kTile * 4;
  float* const vec_base = reinterpret_cast<float*>(__cvta_shared_to_generic(vec_saddr));
  auto fetch_vectors = [&](int b, int hq, int m, uint32_t buf) {
    const size_t bhq = (static_cast<size_t>(b) * p.Hq + hq) * p.N;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = lane + 32 * t, q = m * kTile + c;
      const bool in = q < p.N;
      const size_t idx = bhq + (in ? q : 0);
      const uint32_t dst = vec_saddr + (buf * 2 * kTile + c) * 4;
      cp_async_4(dst, p.lse + idx, in ? 4u : 0u);
      cp_async_4(dst + kTile * 4, p.delta + idx, in ? 4u : 0u);
    }
    cp_async_commit();
  };
  const float c2 = p.scale_log2;
  const uint64_t c2x2 = f32x2_pack(c2, c2);
  const int code = (kBKernelDkdvFull << 12) | (kBRoleElem << 8);
  uint32_t g = 0;
  bool fetched = false;
  int items = 0;
  for (int i = blockIdx.x; i < p.num_items; i += gridDim.x, ++items) {
    const DkvItem it = dkv_item(p, i);
    const int key = it.n * kTile + r;
    bool ok = true;
    for (int s = 0; s < it.steps && ok; ++s, ++g) {
      int hq, m;
      dkv_step(p, it, s, hq, m);
      const uint32_t buf = g & 1;
      float* const s_lse = vec_base + buf * 2 * kTile;
      float* const s_dlt = s_lse + kTile;
      {
        if (!fetched) fetch_vectors(it.b, hq, m, buf);
        cp_async_wait_all();
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = lane + 32 * t;
          s_lse[c] = -s_lse[c] * kLog2e;
          s_dlt[c] = -s_dlt[c];
        }
        __syncwarp();
        fetched = false;
        if (s + 1 < it.steps) {
          int hq2, m2;
          dkv_step(p, it, s + 1, hq2, m2);
          fetch_vectors(it.b, hq2, m2, buf ^ 1);
          fetched = true;
        } else if (i + static_cast<int>(gridDim.x) < p.num_items) {
          const DkvItem nx = dkv_item(p, i + gridDim.x);
          int hq2, m2;
          dkv_step(p, nx, 0, hq2, m2);
          fetch_vectors(nx.b, hq2, m2, buf ^ 1);
          fetched = true;
        }
      }
      // S^T of the step: load it, release X for the next step's product, mask.
      if (!w.wait_warp(bar(kSFull), g & 1, code | kSFull)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t sv[128];
      tmem_load_128cols(tX, sv);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kXFree));
      if (block_is_partial(p, m, it.n)) {
        // Query columns that see this key: lo_c <= c <= hi_c.
        const int q0 = m * kTile;
        const int hi_c =
            (key < p.N) ? min(p.N - 1, p.mask_kind == kBMaskWindow ? key + p.window - 1 : p.N - 1) - q0 : -1;
        const int lo_c = (p.mask_kind == kBMaskFull) ? 0 : key - q0;
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c > hi_c || c < lo_c) sv[c] = 0xff800000u;  // -inf
      }
      // P^T = 2^(S c - lse log2 e), rounded to bf16 (query pairs per 32-bit word).
      uint32_t pk[kTile / 2];
#pragma unroll
      for (int c = 0; c < kTile; c += 2) {
        const float2 nl = *reinterpret_cast<const float2*>(s_lse + c);
        float x0, x1;
        f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2,
                               f32x2_pack(nl.x, nl.y)),
                     x0, x1);
        pk[c >> 1] = bf16x2_rn(bexp2(x0), bexp2(x1));
      }
      // dS^T = P (dP - D) once dP^T is in Y, 32 queries at a time; P^T and dS^T go
      // over Y only where dP^T has been read.
      if (!w.wait_warp(bar(kDpFull), g & 1, code | kDpFull)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t dk[kTile / 2];
#pragma unroll
      for (int chunk = 0; chunk < 4; ++chunk) {
        uint32_t pv[32];
        tmem_load_32cols(tY + chunk * 32, pv);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int c = chunk * 32 + e;
          const float2 nd = *reinterpret_cast<const float2*>(s_dlt + c);
          const uint32_t pw = pk[c >> 1];
          float d0, d1;
          f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(pw << 16), __uint_as_float(pw & 0xffff0000u)),
                                 f32x2_add(f32x2_pack(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])),
                                           f32x2_pack(nd.x, nd.y))),
                       d0, d1);
          dk[c >> 1] = bf16x2_rn(d0, d1);
        }
        if (chunk == 1) tmem_store_32cols(tY, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));  // Y[0, 32) read
      }
      tmem_store_32cols(tY + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
      tmem_store_32cols(tY + 64, *reinterpret_cast<const uint32_t(*)[32]>(&dk[0]));
      tmem_store_32cols(tY + 96, *reinterpret_cast<const uint32_t(*)[32]>(&dk[32]));
      tmem_store_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kPFull));
    }
    if (!ok) break;
    if (!w.wait_warp(bar(L::kAccDone), items & 1, code | L::kAccDone)) break;
    tc_fence_after_sync();
    const bool key_ok = key < p.N;
    const size_t krow = (static_cast<size_t>(it.b) * p.Hkv + it.hkv) * p.N + (key_ok ? key : 0);
    store_acc_row<D>(t_dv, 1.f, p.dv + krow * D, key_ok);
    store_acc_row<D>(t_dk, p.scale, p.dk + krow * D, key_ok);
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kAccFree));
  }
  cp_async_wait_all();
  tmem_store_wait();
}

// Fused kernel, warps 6-9: after each dQ^T_h product, read it out of TMEM
// (thread = TMEM lane = column c of dQ, 64 query values) and add it into the
// fp32 accumulator: for each query, the warp's 32 lanes add 32 consecutive
// floats (one 128-byte reduction).
template <int D>
__device__ __forceinline__ void dkv_dq(const BwdParams& p, uint32_t sbase, uint32_t tmem, const BwdWaiter& w,
                                       int warp, int lane) {
  using L = BwdSmem<D>;
  auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
  const int quarter = warp & 3;  // TMEM lanes this warp may read
  const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
  const int col = quarter * 32 + lane;
  const int code = (kBKernelFused << 12) | (kBRoleDq << 8);
  uint32_t cnt[2] = {0, 0};
  bool ok = true;
  for (int i = blockIdx.x; ok && i < p.num_items; i += gridDim.x) {
    const DkvItem it = dkv_item(p, i);
    for (int s = 0; s < it.steps && ok; ++s) {
      int hq, m;
      dkv_step(p, it, s, hq, m);
      float* head_base = p.dq_acc + (static_cast<size_t>(it.b) * p.Hq + hq) * p.N * D + col;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (!w.wait_warp(bar(L::kDqFull + h), cnt[h] & 1, code | (L::kDqFull + h))) {
          ok = false;
          break;
        }
        ++cnt[h];
        tc_fence_after_sync();
        uint32_t a[32], b[32];
        tmem_load_2x32cols(tmem + lane_bits + L::col_p(h), tmem + lane_bits + L::col_p(h) + 32, a, b);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kDqFree + h));
        const int q0 = m * kTile + h * kHalf;
        const int nq = min(kHalf, p.N - q0);  // queries of this half inside the sequence
        float* dst = head_base + static_cast<size_t>(q0) * D;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nq) atomicAdd(dst + static_cast<size_t>(j) * D, __uint_as_float(a[j]));
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (32 + j < nq) atomicAdd(dst + static_cast<size_t>(32 + j) * D, __uint_as_float(b[j]));
      }
    }
  }
}

// dq = bf16(scale * the fp32 accumulator), eight elements per thread per
// iteration (two 16-byte loads, one 16-byte store), grid-stride.
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                 __nv_bfloat16* __restrict__ dq, float scale,
                                                                 int64_t groups8) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups8; g += stride) {
    const float4 x = reinterpret_cast<const float4*>(acc)[2 * g];
    const float4 y = reinterpret_cast<const float4*>(acc)[2 * g + 1];
    reinterpret_cast<uint4*>(dq)[g] = make_uint4(bf16x2_rn(x.x * scale, x.y * scale), bf16x2_rn(x.z * scale, x.w * scale),
                                                 bf16x2_rn(y.x * scale, y.y * scale), bf16x2_rn(y.z * scale, y.w * scale));
  }
}

// ------------------------------------------------------------------ entry
template <int KIND>
constexpr int bwd_threads() {
  return KIND == kBKernelFused ? kBwdThreadsFused : kBwdThreads;
}

template <int D, int KIND>
__global__ void __launch_bounds__(bwd_threads<KIND>(), 1) __maxnreg__(KIND == kBKernelFused ? 200 : 255) attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return sbase + L::kBarOff + 8u * i; };
    mbar_init(bar(L::kFixFull), 1);
    mbar_init(bar(L::kFixEmpty), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kRingFull + s), 1);
      mbar_init(bar(L::kRingEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(L::kSFull + h), 1);
      mbar_init(bar(L::kPFull + h), 4);  // one arrival per elementwise warp
    }
    mbar_init(bar(L::kAccDone), 1);
    mbar_init(bar(L::kAccFree), 4);  // one arrival per elementwise warp
    mbar_init(bar(L::kFin), 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(L::kDqFull + h), 1);
      mbar_init(bar(L::kDqFree + h), 4);  // one arrival per dQ warp
    }
    mbar_init(bar(L::kDsFree), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kRing2Full + s), 1);
      mbar_init(bar(L::kRing2Empty + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const BwdWaiter w{p.timeout_ns, abort_flag, p.err};
  if (warp < 4) {
    if constexpr (KIND == kBKernelDqFull) dqf_elem<D>(p, sbase, tmem, w, warp, lane);
    else if constexpr (KIND == kBKernelDkdvFull) dkvf_elem<D>(p, sbase, tmem, w, warp, lane);
    else dkv_elem<D>(p, sbase, tmem, w, warp, lane);
  } else if (warp >= kBwdDqWarp0) {
    if constexpr (KIND == kBKernelFused) dkv_dq<D>(p, sbase, tmem, w, warp, lane);
  } else if (warp == kBwdLoaderWarp) {
    if (lane == 0) {
      if (KIND == kBKernelDqFull) dq_loader<D>(p, sbase, w);
      else dkv_loader<D, KIND == kBKernelDkdvFull>(p, sbase, w);
    }
    __syncwarp();
  } else if (warp == kBwdMmaWarp) {
    if constexpr (KIND == kBKernelDqFull) dqf_mma<D>(p, sbase, tmem, w);
    else if constexpr (KIND == kBKernelDkdvFull) dkvf_mma<D>(p, sbase, tmem, w);
    else dkv_mma<D>(p, sbase, tmem, w);
    // Every MMA this warp issued must complete before TMEM is freed.
    tc_commit_elect(sbase + L::kBarOff + 8u * L::kFin);
    w.drain(sbase + L::kBarOff + 8u * L::kFin, 0, (KIND << 12) | (kBRoleMma << 8) | L::kFin);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

}  // namespace attn_sm100_bwd
