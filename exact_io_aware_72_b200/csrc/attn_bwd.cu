// Host side of the backward entry points declared in include/attn.h: argument
// checks, TMA tensor maps and the launches on the caller's stream: D, then for
// d = 128 with Hq == Hkv the zeroed fp32 dQ accumulator, the fused key-tile
// kernel and the dQ conversion; otherwise (d = 64, grouped heads, or
// bwd_deterministic) the query-tile (dQ) and key-tile (dK, dV) kernels on whole
// 128 x 128 tiles.
#include "attn.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_bwd_kernel.cuh"

using namespace attn_sm100_bwd;

namespace attn_sm100_bwd {
// Device error word of the backward kernels (read and cleared by attn_bwd_debug_error).
__device__ int g_attn_bwd_error;
}  // namespace attn_sm100_bwd

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr int kMaxDevices = 64;

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

struct BwdDevice {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  int* err_word = nullptr;
};
std::mutex g_bwd_mutex;
BwdDevice g_bwd_dev[kMaxDevices];

template <int D, int KIND>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(attn_bwd_kernel<D, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwdSmem<D>::kAlloc);
}

int bwd_device_setup(BwdDevice& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_bwd_mutex);
  BwdDevice& info = g_bwd_dev[dev];
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
      if (cudaGetSymbolAddress(&addr, g_attn_bwd_error) != cudaSuccess) return ATTN_ERR_CUDA;
      info.err_word = static_cast<int*>(addr);
      if (set_smem<128, kBKernelFused>() != cudaSuccess || set_smem<64, kBKernelDkdvFull>() != cudaSuccess ||
          set_smem<128, kBKernelDkdvFull>() != cudaSuccess || set_smem<64, kBKernelDqFull>() != cudaSuccess ||
          set_smem<128, kBKernelDqFull>() != cudaSuccess)
        return ATTN_ERR_CUDA;
    }
    info.probed = true;
  }
  out = info;
  return info.supported ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

CUresult encode_bhnd(EncodeTiledFn enc, CUtensorMap* map, const void* base, int64_t BH, int64_t N, int64_t d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(N * d * 2)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

bool sizes_ok(int64_t B, int64_t Hq, int64_t Hkv, int64_t N) {
  return B >= 1 && Hq >= 1 && Hkv >= 1 && N >= 1 && Hq % Hkv == 0 && N <= (int64_t(1) << 30) &&
         B * Hq <= (int64_t(1) << 30) && B * Hq * ((N + kTile - 1) / kTile) <= 0x7fffffff;
}

template <int D, int KIND>
cudaError_t launch_bwd(const BwdParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(bwd_threads<KIND>());
  cfg.dynamicSmemBytes = BwdSmem<D>::kAlloc;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, attn_bwd_kernel<D, KIND>, p);
}

}  // namespace

namespace {
// Workspace of a backward: D (B*Hq*N floats), then for the fused path
// (acc_d = 128), from the next 256-byte boundary, the fp32 dQ accumulator
// (B*Hq*N*acc_d floats).  0 when the byte count would not fit in 62 bits.
size_t bwd_workspace_bytes(int64_t B, int64_t Hq, int64_t N, int64_t acc_d) {
  if (B < 1 || Hq < 1 || N < 1 || B > (int64_t(1) << 30) || Hq > (int64_t(1) << 30) || N > (int64_t(1) << 30) ||
      B * Hq > (int64_t(1) << 61) / (N * 4 * (1 + 128)))
    return 0;
  const size_t rows = static_cast<size_t>(B) * static_cast<size_t>(Hq) * static_cast<size_t>(N);
  const size_t delta = rows * sizeof(float);
  if (acc_d == 0) return delta;
  return ((delta + 255) & ~size_t(255)) + rows * static_cast<size_t>(acc_d) * sizeof(float);
}
}  // namespace

extern "C" {

size_t attn_bwd_workspace_bytes(int64_t B, int64_t Hq, int64_t N) {
  return bwd_workspace_bytes(B, Hq, N, 128);  // covers every supported head dimension
}

int attn_bwd_ex(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int64_t B, int64_t Hq,
                int64_t Hkv, int64_t N, int64_t d, float scale, int mask_kind, int64_t window, cudaStream_t stream,
                const attn_fwd_options* opts) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!sizes_ok(B, Hq, Hkv, N)) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // Byte counts must fit in 63 bits (B * Hq * N <= 2^60 after sizes_ok).
  if (B * Hq * N > (int64_t(1) << 61) / (d * 4)) return ATTN_ERR_INVALID_ARG;
  // The fused kernel where each KV head serves one query head. With grouped heads a key
  // tile's dQ partial sums go to every query head of its group, whose fp32 accumulators
  // (and Q, dO) then outgrow L2; there the two-kernel path measured faster.
  const bool fused = (d == 128) && Hq == Hkv && !(opts && opts->bwd_deterministic);
  const size_t ws = bwd_workspace_bytes(B, Hq, N, fused ? 128 : 0);
  if (ws == 0 || workspace_bytes < ws) return ATTN_ERR_INVALID_ARG;
  const size_t q_bytes = static_cast<size_t>(B * Hq * N * d) * 2;
  const size_t kv_bytes = static_cast<size_t>(B * Hkv * N * d) * 2;
  const size_t lse_bytes = static_cast<size_t>(B * Hq * N) * 4;
  const void* ins[6] = {q, k, v, out, lse, dout};
  const size_t in_bytes[6] = {q_bytes, kv_bytes, kv_bytes, q_bytes, lse_bytes, q_bytes};
  void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {q_bytes, kv_bytes, kv_bytes, ws};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], out_bytes[a], ins[b], in_bytes[b])) return ATTN_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], out_bytes[a], outs[b], out_bytes[b])) return ATTN_ERR_INVALID_ARG;
  }
  auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis16(q) || mis16(k) || mis16(v) || mis16(out) || mis16(dout) || mis16(dq) || mis16(dk) || mis16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & (fused ? 15u : 3u)) != 0)
    return ATTN_ERR_MISALIGNED;

  BwdDevice info;
  int st = bwd_device_setup(info);
  if (st != ATTN_OK) return st;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;

  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_bhnd(enc, &p.tm_q, q, B * Hq, N, d) != CUDA_SUCCESS ||
      encode_bhnd(enc, &p.tm_k, k, B * Hkv, N, d) != CUDA_SUCCESS ||
      encode_bhnd(enc, &p.tm_v, v, B * Hkv, N, d) != CUDA_SUCCESS ||
      encode_bhnd(enc, &p.tm_do, dout, B * Hq, N, d) != CUDA_SUCCESS)
    return ATTN_ERR_CUDA;
  int kind = mask_kind;
  int64_t w = window;
  if (kind == ATTN_MASK_SLIDING_WINDOW && w >= N) kind = ATTN_MASK_CAUSAL;  // a window covering everything
  p.lse = lse;
  p.delta = static_cast<const float*>(workspace);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.err = info.err_word;
  p.B = static_cast<int>(B);
  p.Hq = static_cast<int>(Hq);
  p.Hkv = static_cast<int>(Hkv);
  p.N = static_cast<int>(N);
  p.group = static_cast<int>(Hq / Hkv);
  p.mask_kind = kind;
  p.window = static_cast<int>(kind == ATTN_MASK_SLIDING_WINDOW ? w : N);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_blk = static_cast<int>((N + kTile - 1) / kTile);
  p.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;

  // D = rowsum(dO * O) into the workspace.
  const int64_t rows = B * Hq * N;
  const int64_t threads = rows * (d / 8);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  if (d == 128)
    attn_bwd_delta_kernel<128><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out),
                                                          static_cast<const __nv_bfloat16*>(dout),
                                                          static_cast<float*>(workspace), rows);
  else
    attn_bwd_delta_kernel<64><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(out),
                                                         static_cast<const __nv_bfloat16*>(dout),
                                                         static_cast<float*>(workspace), rows);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;

  int sms = info.sm_count;
  if (opts && opts->grid_ctas > 0) sms = opts->grid_ctas;
  cudaError_t e;
  if (fused) {
    // Fused: dK, dV and the fp32 dQ sums in one key-tile kernel, then dQ to bf16.
    const size_t acc_off = (static_cast<size_t>(rows) * sizeof(float) + 255) & ~size_t(255);
    float* acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + acc_off);
    const size_t acc_bytes = static_cast<size_t>(rows) * 128 * sizeof(float);
    if (cudaMemsetAsync(acc, 0, acc_bytes, stream) != cudaSuccess) return ATTN_ERR_CUDA;
    p.dq_acc = acc;
    p.num_items = static_cast<int>(B * Hkv * p.num_blk);  // one key tile per item
    const int grid = static_cast<int>(std::min<int64_t>(sms, p.num_items));
    if (launch_bwd<128, kBKernelFused>(p, grid, stream) != cudaSuccess) return ATTN_ERR_CUDA;
    const int64_t groups8 = rows * 128 / 8;
    const unsigned cblocks = static_cast<unsigned>(std::min<int64_t>((groups8 + 255) / 256, int64_t(info.sm_count) * 16));
    attn_bwd_dq_convert_kernel<<<cblocks, 256, 0, stream>>>(acc, static_cast<__nv_bfloat16*>(dq), scale, groups8);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  p.num_items = static_cast<int>(B * Hq * p.num_blk);  // dQ: one query tile per item
  int grid = static_cast<int>(std::min<int64_t>(sms, p.num_items));
  e = (d == 128) ? launch_bwd<128, kBKernelDqFull>(p, grid, stream) : launch_bwd<64, kBKernelDqFull>(p, grid, stream);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  p.num_items = static_cast<int>(B * Hkv * p.num_blk);  // dK, dV: one key tile per item
  grid = static_cast<int>(std::min<int64_t>(sms, p.num_items));
  e = (d == 128) ? launch_bwd<128, kBKernelDkdvFull>(p, grid, stream)
                 : launch_bwd<64, kBKernelDkdvFull>(p, grid, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int64_t B, int64_t Hq,
             int64_t Hkv, int64_t N, int64_t d, float scale, int mask_kind, int64_t window, cudaStream_t stream) {
  return attn_bwd_ex(q, k, v, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d, scale,
                     mask_kind, window, stream, nullptr);
}

int attn_bwd_debug_error(cudaStream_t stream, int* device_code) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  int code = 0;
  if (cudaMemcpyFromSymbol(&code, g_attn_bwd_error, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_attn_bwd_error, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (device_code) *device_code = code;
  return code ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

}  // extern "C"
