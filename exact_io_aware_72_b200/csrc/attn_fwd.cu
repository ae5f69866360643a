// Host side of the C ABI declared in include/attn.h: argument checks, TMA tensor
// maps, schedule parameters and the launch of the sm_100a forward kernel.
#include "attn.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_fwd_kernel.cuh"

using namespace attn_sm100;

namespace attn_sm100 {
// Device error word written by timed-out waits (read and cleared by attn_debug_error).
__device__ int g_attn_error;
}  // namespace attn_sm100

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
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

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  int* err_word = nullptr;
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

// Probe the current device once: sm_100 check, SM count, error-word address,
// and the dynamic shared-memory opt-in of every kernel instance.
int device_setup(int& dev, DeviceInfo& out_info) {
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& info = g_dev[dev];
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
      if (cudaGetSymbolAddress(&addr, g_attn_error) != cudaSuccess) return ATTN_ERR_CUDA;
      info.err_word = static_cast<int*>(addr);
      if (cudaFuncSetAttribute(attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SmemLayout<64>::kAlloc) != cudaSuccess ||
          cudaFuncSetAttribute(attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SmemLayout<128>::kAlloc) != cudaSuccess ||
          cudaFuncSetAttribute(attn_fwd_kernel<128, 1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SmemLayout<128, 1>::kAlloc) != cudaSuccess ||
          cudaFuncSetAttribute(attn_fwd_kernel<64, 2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SmemLayout<64>::kAlloc) != cudaSuccess ||
          cudaFuncSetAttribute(attn_fwd_kernel<128, 2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SmemLayout<128>::kAlloc) != cudaSuccess)
        return ATTN_ERR_CUDA;
    }
    info.probed = true;
  }
  out_info = info;
  return info.supported ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

struct Plan {
  int mask_kind;
  int64_t window;
  int pair_heads;
  int64_t num_mblk, row_units, head_units, num_items, super_items;
};

// Checks that need no device; fills the schedule plan.
int check_sizes(int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d, int mask_kind, int64_t window,
                Plan& plan, int64_t key_offset = 0) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (key_offset < 0 || key_offset > (int64_t(1) << 30)) return ATTN_ERR_INVALID_ARG;
  // Index arithmetic in the kernel is 32-bit for rows and heads.
  if (N > (int64_t(1) << 30) || B * Hq > (int64_t(1) << 30) || B * Hkv > (int64_t(1) << 30))
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // Byte counts (at most 4 bytes per element) must fit in 63 bits; B * Hq * N is
  // at most 2^60 after the checks above, so the product itself cannot wrap.
  if (B * Hq * N > (int64_t(1) << 61) / (d * 4)) return ATTN_ERR_INVALID_ARG;
  plan.mask_kind = mask_kind;
  plan.window = window;
  // A window covering every earlier key is plain causal attention.
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window >= N + key_offset) {
    plan.mask_kind = ATTN_MASK_CAUSAL;
    plan.window = N;
  }
  const int64_t group = Hq / Hkv;
  plan.pair_heads = (group % 2 == 0) ? 1 : 0;
  plan.num_mblk = (N + kBlockM - 1) / kBlockM;
  plan.row_units = plan.pair_heads ? plan.num_mblk : (plan.num_mblk + 1) / 2;
  plan.head_units = plan.pair_heads ? B * Hq / 2 : B * Hq;
  plan.num_items = plan.row_units * plan.head_units;
  plan.super_items = plan.head_units * ((plan.row_units + 1) / 2);  // row units r and R-1-r together
  if (plan.num_items > 0x7fffffff) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// [BH, N, d] tensor of eb-byte elements (2: bf16, 1: E4M3 codes), boxes of
// 128 rows x 128 bytes with the 128-byte swizzle.
CUresult encode_bhnd(EncodeTiledFn enc, CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t d,
                     int eb = 2) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * eb), static_cast<cuuint64_t>(N * d * eb)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(kBlockM), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Shared by the bf16 (eb = 2) and E4M3 (eb = 1) entry points: checks, tensor
// maps and the launch.  score_scale multiplies q.k of the stored values
// (softmax scale, times the q and k scales for E4M3); v_scale multiplies O.
int fwd_launch(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t Hq,
               int64_t Hkv, int64_t N, int64_t d, int eb, float score_scale, float v_scale, int mask_kind,
               int64_t window, cudaStream_t stream, const attn_fwd_options* opts) {
  if (!q || !k || !v || !out || !lse) return ATTN_ERR_INVALID_ARG;
  Plan plan{};
  const int64_t key_offset = opts ? opts->key_offset : 0;
  int st = check_sizes(B, Hq, Hkv, N, d, mask_kind, window, plan, key_offset);
  if (st != ATTN_OK) return st;
  if (eb == 1 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(score_scale) || !(score_scale > 0.f) || !std::isfinite(v_scale) || !(v_scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  const bool out_f32 = opts && opts->out_fp32;
  const size_t q_bytes = static_cast<size_t>(B * Hq * N * d) * eb;
  const size_t kv_bytes = static_cast<size_t>(B * Hkv * N * d) * eb;
  const size_t out_bytes = static_cast<size_t>(B * Hq * N * d) * (out_f32 ? 4 : 2);
  const size_t lse_bytes = static_cast<size_t>(B * Hq * N) * 4;
  if (overlaps(out, out_bytes, q, q_bytes) || overlaps(out, out_bytes, k, kv_bytes) ||
      overlaps(out, out_bytes, v, kv_bytes) || overlaps(lse, lse_bytes, out, out_bytes) ||
      overlaps(lse, lse_bytes, q, q_bytes) || overlaps(lse, lse_bytes, k, kv_bytes) ||
      overlaps(lse, lse_bytes, v, kv_bytes))
    return ATTN_ERR_INVALID_ARG;
  auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis16(q) || mis16(k) || mis16(v) || mis16(out) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_MISALIGNED;

  int dev = 0;
  DeviceInfo info;
  st = device_setup(dev, info);
  if (st != ATTN_OK) return st;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return ATTN_ERR_CUDA;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_bhnd(enc, &p.tm_q, q, B * Hq, N, d, eb) != CUDA_SUCCESS ||
      encode_bhnd(enc, &p.tm_k, k, B * Hkv, N, d, eb) != CUDA_SUCCESS ||
      encode_bhnd(enc, &p.tm_v, v, B * Hkv, N, d, eb) != CUDA_SUCCESS)
    return ATTN_ERR_CUDA;
  p.out = out_f32 ? nullptr : static_cast<__nv_bfloat16*>(out);
  p.out_f32 = out_f32 ? static_cast<float*>(out) : nullptr;
  p.lse = lse;
  p.err = info.err_word;
  p.B = static_cast<int>(B);
  p.Hq = static_cast<int>(Hq);
  p.Hkv = static_cast<int>(Hkv);
  p.N = static_cast<int>(N);
  p.group = static_cast<int>(Hq / Hkv);
  p.mask_kind = plan.mask_kind;
  p.window = static_cast<int>(plan.mask_kind == ATTN_MASK_SLIDING_WINDOW ? std::min<int64_t>(plan.window, 1 << 30) : N);
  p.key_offset = plan.mask_kind == ATTN_MASK_FULL ? 0 : static_cast<int>(key_offset);
  p.scale_log2 = score_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  p.pair_heads = plan.pair_heads;
  p.num_mblk = static_cast<int>(plan.num_mblk);
  p.row_units = static_cast<int>(plan.row_units);
  p.head_units = static_cast<int>(plan.head_units);
  p.num_items = static_cast<int>(plan.num_items);
  p.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;
  p.inject_stall = (opts && opts->inject_stall) ? 1 : 0;
  p.out_v8 = (reinterpret_cast<uintptr_t>(out) % 32 == 0) ? 1 : 0;
  p.item_visits = opts ? opts->item_visits : nullptr;
  const bool p_bf16 = opts && opts->p_bf16;

  int grid = info.sm_count;
  if (opts && opts->grid_ctas > 0) grid = opts->grid_ctas;
  if (grid > plan.super_items) grid = static_cast<int>(plan.super_items);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaError_t e;
  if (eb == 1) {
    cfg.dynamicSmemBytes = SmemLayout<128, 1>::kAlloc;
    e = cudaLaunchKernelEx(&cfg, attn_fwd_kernel<128, 1, false>, p);
  } else if (d == 128) {
    cfg.dynamicSmemBytes = SmemLayout<128>::kAlloc;
    e = p_bf16 ? cudaLaunchKernelEx(&cfg, attn_fwd_kernel<128, 2, false>, p)
               : cudaLaunchKernelEx(&cfg, attn_fwd_kernel<128, 2, true>, p);
  } else {
    cfg.dynamicSmemBytes = SmemLayout<64>::kAlloc;
    e = p_bf16 ? cudaLaunchKernelEx(&cfg, attn_fwd_kernel<64, 2, false>, p)
               : cudaLaunchKernelEx(&cfg, attn_fwd_kernel<64, 2, true>, p);
  }
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_RANGE: return "ATTN_ERR_RANGE";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

int64_t attn_fwd_num_work_items(int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d, int mask_kind,
                                int64_t window) {
  Plan plan{};
  if (check_sizes(B, Hq, Hkv, N, d, mask_kind, window, plan) != ATTN_OK) return -1;
  return plan.num_items;
}

int attn_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t Hq,
                int64_t Hkv, int64_t N, int64_t d, float scale, int mask_kind, int64_t window, cudaStream_t stream,
                const attn_fwd_options* opts) {
  return fwd_launch(q, k, v, out, lse, B, Hq, Hkv, N, d, 2, scale, 1.f, mask_kind, window, stream, opts);
}

int attn_fwd_fp8_ex(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                    void* out, float* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d, float scale,
                    int mask_kind, int64_t window, cudaStream_t stream, const attn_fwd_options* opts) {
  if (!std::isfinite(q_scale) || !(q_scale > 0.f) || !std::isfinite(k_scale) || !(k_scale > 0.f) ||
      !std::isfinite(scale) || !(scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  return fwd_launch(q, k, v, out, lse, B, Hq, Hkv, N, d, 1, scale * q_scale * k_scale, v_scale, mask_kind, window,
                    stream, opts);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                 void* out, float* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d, float scale,
                 int mask_kind, int64_t window, cudaStream_t stream) {
  return attn_fwd_fp8_ex(q, k, v, q_scale, k_scale, v_scale, out, lse, B, Hq, Hkv, N, d, scale, mask_kind, window,
                         stream, nullptr);
}

int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t Hq,
             int64_t Hkv, int64_t N, int64_t d, float scale, int mask_kind, int64_t window, cudaStream_t stream) {
  return attn_fwd_ex(q, k, v, out, lse, B, Hq, Hkv, N, d, scale, mask_kind, window, stream, nullptr);
}

int attn_debug_error(cudaStream_t stream, int* device_code) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  int code = 0;
  if (cudaMemcpyFromSymbol(&code, g_attn_error, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_attn_error, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (device_code) *device_code = code;
  if (code == 0) return ATTN_OK;
  return (code & kErrRangeV) ? ATTN_ERR_RANGE : ATTN_ERR_TIMEOUT;
}

}  // extern "C"
