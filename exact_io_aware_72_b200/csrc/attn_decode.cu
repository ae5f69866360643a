// Host side of the decoding entry points declared in include/attn.h: argument
// checks, TMA tensor maps over the paged caches, the decoding launch and (with
// more than one split) the merge launch, all on the caller's stream.
#include "attn.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_decode_kernel.cuh"

using namespace attn_sm100_dec;

namespace attn_sm100_dec {
// Device error word of the decoding kernel (read and cleared by attn_decode_debug_error).
__device__ int g_attn_dec_error;
}  // namespace attn_sm100_dec

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxSplits = 4096;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

struct DecDevice {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  int* err_word = nullptr;
};
std::mutex g_dec_mutex;
DecDevice g_dec_dev[kMaxDevices];

template <int D, int WC>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(attn_decode_kernel<D, WC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              DecSmem<D>::kAlloc);
}

int dec_device_setup(DecDevice& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dec_mutex);
  DecDevice& info = g_dec_dev[dev];
  if (!info.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    info.supported = (major == 10 && minor == 0);
    info.sm_count = sms;
    if (info.supported) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_attn_dec_error) != cudaSuccess) return ATTN_ERR_CUDA;
      info.err_word = static_cast<int*>(addr);
      if (set_smem<64, 1>() != cudaSuccess || set_smem<64, 2>() != cudaSuccess || set_smem<64, 4>() != cudaSuccess ||
          set_smem<128, 1>() != cudaSuccess || set_smem<128, 2>() != cudaSuccess ||
          set_smem<128, 4>() != cudaSuccess)
        return ATTN_ERR_CUDA;
    }
    info.probed = true;
  }
  out = info;
  return info.supported ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (na == 0 || nb == 0) return false;
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Query rows of one (b, KV head) handled per work item, and warps per replica.
int rows_per_chunk(int64_t rows_total) { return static_cast<int>(std::min<int64_t>(rows_total, kLanes)); }
int warps_per_copy(int rows_chunk) { return rows_chunk <= 32 ? 1 : (rows_chunk <= 64 ? 2 : 4); }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: 256 bytes of work-item counters (zero between calls), then with
// more than one split the partial log-sum-exps and the partial outputs.
constexpr size_t kSchedBytes = 256;
size_t workspace_bytes(int64_t rows, int64_t d, int64_t splits) {
  if (splits <= 1) return kSchedBytes;
  return kSchedBytes + align_up(static_cast<size_t>(rows) * splits * 4, 256) +
         static_cast<size_t>(rows) * splits * d * 4;
}

template <int D, int WC>
cudaError_t launch_decode(const DecParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = DecSmem<D>::kAlloc;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, attn_decode_kernel<D, WC>, p);
}

template <int D>
cudaError_t launch_decode_wc(const DecParams& p, int wc, int grid, cudaStream_t stream) {
  if (wc == 1) return launch_decode<D, 1>(p, grid, stream);
  if (wc == 2) return launch_decode<D, 2>(p, grid, stream);
  return launch_decode<D, 4>(p, grid, stream);
}

}  // namespace

extern "C" size_t attn_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Nq, int64_t d, int64_t num_splits) {
  if (B < 1 || Hq < 1 || Nq < 1 || (d != 64 && d != 128) || num_splits < 1 || num_splits > kMaxSplits) return 0;
  if (B > (int64_t(1) << 30) || Hq > (int64_t(1) << 30) || Nq > (int64_t(1) << 30)) return 0;
  const int64_t rows = B * Hq * Nq;
  if (rows > 0x7fffffff) return 0;
  return workspace_bytes(rows, d, num_splits);
}

extern "C" int64_t attn_decode_num_splits(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t max_seq_len,
                                          int mask_kind, int64_t window) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || max_seq_len < Nq || Hq % Hkv != 0) return -1;
  if (mask_kind < ATTN_MASK_FULL || mask_kind > ATTN_MASK_SLIDING_WINDOW) return -1;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return -1;
  if (B > (int64_t(1) << 30) || Hq > (int64_t(1) << 30) || Nq > (int64_t(1) << 30)) return -1;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
  }
  const int64_t rows_total = (Hq / Hkv) * Nq;
  const int64_t chunks = (rows_total + kLanes - 1) / kLanes;
  const int64_t units = B * Hkv * chunks;
  int64_t keys = max_seq_len;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW) keys = std::min<int64_t>(keys, window + Nq - 1);
  const int64_t tiles = (keys + kKeys - 1) / kKeys + 1;
  // A batch smaller than the SM count is split into one wave of items (each
  // SM streams one item).  A larger batch takes several waves from the shared
  // counter; there no item is longer than kMaxItemTiles tiles, so the SMs
  // finish together even when sequence lengths differ.  Each split keeps at
  // least four tiles.
  constexpr int64_t kMaxItemTiles = 64;
  const int64_t s = units < sms ? sms / units : (tiles + kMaxItemTiles - 1) / kMaxItemTiles;
  return std::max<int64_t>(1, std::min<int64_t>({s, std::max<int64_t>(1, tiles / 4), kMaxSplits}));
}

extern "C" int attn_decode_ex(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                              const int32_t* seq_lens, void* out, float* lse, void* workspace,
                              size_t workspace_bytes_given, int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                              int64_t d, int64_t num_pages, int64_t page_size, int64_t max_pages_per_seq,
                              int64_t num_splits, float scale, int mask_kind, int64_t window,
                              cudaStream_t stream, const attn_fwd_options* opts) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out || !lse) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Hq % Hkv != 0 || num_pages < 1 || max_pages_per_seq < 1)
    return ATTN_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > kMaxSplits) return ATTN_ERR_INVALID_ARG;
  if (mask_kind < ATTN_MASK_FULL || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128 && page_size != 256)
    return ATTN_ERR_UNSUPPORTED;
  const int64_t lim = 0x7fffffff;
  if (B > (int64_t(1) << 30) || Hq > (int64_t(1) << 30) || Nq > (int64_t(1) << 30) || B * Hq > lim ||
      B * Hq * Nq > lim || num_pages > lim / Hkv || max_pages_per_seq > lim / page_size ||
      B > lim / max_pages_per_seq)
    return ATTN_ERR_INVALID_ARG;
  const int64_t rows = B * Hq * Nq;
  const int64_t rows_total = (Hq / Hkv) * Nq;
  const int rows_chunk = rows_per_chunk(rows_total);
  const int64_t row_chunks = (rows_total + rows_chunk - 1) / rows_chunk;
  if (B * Hkv > lim / row_chunks || B * Hkv * row_chunks > lim / num_splits) return ATTN_ERR_INVALID_ARG;
  const int64_t items = B * Hkv * row_chunks * num_splits;
  const size_t ws_need = workspace_bytes(rows, d, num_splits);
  if (!workspace || workspace_bytes_given < ws_need) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(workspace, 16))
    return ATTN_ERR_MISALIGNED;

  const size_t q_bytes = static_cast<size_t>(rows) * d * 2;
  const size_t cache_bytes = static_cast<size_t>(num_pages) * Hkv * page_size * d * 2;
  const size_t table_bytes = static_cast<size_t>(B) * max_pages_per_seq * 4;
  const size_t lens_bytes = static_cast<size_t>(B) * 4;
  const size_t lse_bytes = static_cast<size_t>(rows) * 4;
  const void* ins[5] = {q, k_cache, v_cache, block_table, seq_lens};
  const size_t in_sz[5] = {q_bytes, cache_bytes, cache_bytes, table_bytes, lens_bytes};
  const void* outs[3] = {out, lse, workspace};
  const size_t out_sz[3] = {q_bytes, lse_bytes, ws_need};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 5; ++i)
      if (overlaps(outs[o], out_sz[o], ins[i], in_sz[i])) return ATTN_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlaps(outs[o], out_sz[o], outs[o2], out_sz[o2])) return ATTN_ERR_INVALID_ARG;
  }

  DecDevice dev;
  const int st = dec_device_setup(dev);
  if (st != ATTN_OK) return st;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;

  DecParams p;
  std::memset(&p, 0, sizeof(p));
  const int rows_per_load = static_cast<int>(std::min<int64_t>(page_size, kKeys));
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), 1};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(rows * d * 2)};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows_chunk), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_CUDA;
  }
  for (int kv = 0; kv < 2; ++kv) {
    // 4-D view of a cache: (64 columns, page rows, d/64 column halves, page x KV head); a V box
    // brings both halves of a page's rows, half after half, a K box one half.
    cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(page_size), static_cast<cuuint64_t>(d / 64),
                          static_cast<cuuint64_t>(num_pages * Hkv)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(d * 2), 128, static_cast<cuuint64_t>(page_size * d * 2)};
    cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows_per_load), kv ? static_cast<cuuint32_t>(d / 64) : 1u, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(kv ? &p.tm_v : &p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(kv ? v_cache : k_cache),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_CUDA;
  }
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.sched = static_cast<unsigned int*>(workspace);
  if (num_splits > 1) {
    uint8_t* ws = static_cast<uint8_t*>(workspace) + kSchedBytes;
    p.part_lse = reinterpret_cast<float*>(ws);
    p.part_o = reinterpret_cast<float*>(ws + align_up(static_cast<size_t>(rows) * num_splits * 4, 256));
  }
  p.err = dev.err_word;
  p.B = static_cast<int>(B);
  p.Hq = static_cast<int>(Hq);
  p.Hkv = static_cast<int>(Hkv);
  p.Nq = static_cast<int>(Nq);
  p.group = static_cast<int>(Hq / Hkv);
  p.rows_total = static_cast<int>(rows_total);
  p.rows_chunk = rows_chunk;
  p.row_chunks = static_cast<int>(row_chunks);
  p.page_size = static_cast<int>(page_size);
  p.rows_per_load = rows_per_load;
  p.loads_per_tile = kKeys / rows_per_load;
  p.max_pages = static_cast<int>(max_pages_per_seq);
  p.num_pages = static_cast<int>(num_pages);
  p.mask_kind = mask_kind;
  p.window = static_cast<int>(std::min<int64_t>(window, int64_t(1) << 30));
  p.num_splits = static_cast<int>(num_splits);
  p.num_items = static_cast<int>(items);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;

  int grid = static_cast<int>(std::min<int64_t>(items, dev.sm_count));
  if (opts && opts->grid_ctas > 0) grid = std::min(grid, opts->grid_ctas);
  const int wc = warps_per_copy(rows_chunk);
  const cudaError_t e = (d == 64) ? launch_decode_wc<64>(p, wc, grid, stream) : launch_decode_wc<128>(p, wc, grid, stream);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  if (num_splits > 1) {
    DecMergeParams mp;
    mp.part_o = p.part_o;
    mp.part_lse = p.part_lse;
    mp.out = p.out;
    mp.lse = lse;
    mp.rows = static_cast<int>(rows);
    mp.num_splits = static_cast<int>(num_splits);
    const unsigned blocks = static_cast<unsigned>((rows + 3) / 4);
    if (d == 64) {
      attn_decode_merge_kernel<64><<<blocks, 128, 0, stream>>>(mp);
    } else {
      attn_decode_merge_kernel<128><<<blocks, 128, 0, stream>>>(mp);
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

extern "C" int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                           const int32_t* seq_lens, void* out, float* lse, void* workspace,
                           size_t workspace_bytes_given, int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t d,
                           int64_t num_pages, int64_t page_size, int64_t max_pages_per_seq, int64_t num_splits,
                           float scale, int mask_kind, int64_t window, cudaStream_t stream) {
  return attn_decode_ex(q, k_cache, v_cache, block_table, seq_lens, out, lse, workspace, workspace_bytes_given, B,
                        Hq, Hkv, Nq, d, num_pages, page_size, max_pages_per_seq, num_splits, scale, mask_kind,
                        window, stream, nullptr);
}

extern "C" int attn_decode_debug_error(cudaStream_t stream, int* device_code) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  DecDevice dev;
  const int st = dec_device_setup(dev);
  if (st != ATTN_OK) return st;
  int code = 0;
  if (cudaMemcpy(&code, dev.err_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(dev.err_word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  if (device_code) *device_code = code;
  if (code == 0) return ATTN_OK;
  return (code & (kDErrSeqLen | kDErrPage)) ? ATTN_ERR_INVALID_ARG : ATTN_ERR_TIMEOUT;
}

// ---------------------------------------------------------------- allocation-free variant
// attn_decode_static (include/attn.h): the decoding step with its scratch -- the work
// counter and the splits' partial results -- in this fixed device array instead of a
// caller workspace, for callers that cannot allocate device memory. Every device that
// loads the library holds the array until the process exits; all calls on a device
// share it.
static __device__ __align__(256) unsigned char g_dec_static_scratch[ATTN_DECODE_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_static_mutex;
void* g_static_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up once per device.
// In host code the array's name only stands in for it, so the address must come from the
// runtime with the device current.
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_dec_static_scratch) != cudaSuccess || !ptr) return ATTN_ERR_CUDA;
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_static(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                                  int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t d, int64_t num_pages,
                                  int64_t page_size, int64_t max_pages_per_seq, int64_t num_splits, float scale,
                                  int mask_kind, int64_t window, cudaStream_t stream) {
  const size_t need = attn_decode_workspace_bytes(B, Hq, Nq, d, num_splits);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > sizeof(g_dec_static_scratch)) return ATTN_ERR_UNSUPPORTED;  // larger than the fixed array
  DecDevice dev;
  const int st = dec_device_setup(dev);  // refuses devices other than sm_100
  if (st != ATTN_OK) return st;
  void* scratch = nullptr;
  const int sst = static_scratch_address(&scratch);
  if (sst != ATTN_OK) return sst;
  // The work counter must be zero when the kernel starts. A call that completes leaves it
  // zero, but one that gave up on a wait may not, so every call clears it.
  if (cudaMemsetAsync(scratch, 0, kSchedBytes, stream) != cudaSuccess) return ATTN_ERR_CUDA;
  return attn_decode_ex(q, k_cache, v_cache, block_table, seq_lens, out, lse, scratch, sizeof(g_dec_static_scratch),
                        B, Hq, Hkv, Nq, d, num_pages, page_size, max_pages_per_seq, num_splits, scale, mask_kind,
                        window, stream, nullptr);
}
