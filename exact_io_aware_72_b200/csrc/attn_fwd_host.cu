// Host-buffer forward (attn_fwd_host, attn_fwd_fp8_host in include/attn.h): the
// exact attention forward of attn_fwd on tensors in host memory, with the
// host<->device copies overlapped with the kernels.
//
// The (batch, key/value head) units are independent ("Attention Mechanism
// Variants Beyond Self-Attention", tempatgunting.com, section "Multi-Query and
// Grouped-Query Attention": each key/value head serves its own group of query
// heads), and a contiguous range of units is a contiguous range of every tensor
// (q holds the group's Hq/Hkv heads of each unit one after the other).  A range
// of n units is therefore itself a forward with B = 1, Hkv = n, Hq = n * group.
// The job is cut into such chunks: chunk c's upload runs on one copy stream, its
// forward on the caller's stream once it has arrived, and its download on a
// second copy stream once it has been computed, so that uploads, kernels and
// downloads of different chunks run at the same time (PCIe moves both
// directions at once).  Each chunk's forward is the public attn_fwd_ex /
// attn_fwd_fp8_ex call; nothing here touches the data.
#include "attn.h"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>

namespace {

constexpr int64_t kDefaultChunks = 8;
constexpr int kMaxDevices = 64;

struct CopyStreams {
  cudaStream_t up = nullptr, down = nullptr;
};
std::mutex g_copy_mutex;
CopyStreams g_copy[kMaxDevices];

// Two non-blocking copy streams per device, created on first use and kept.
// An unsupported device is refused here, before anything is enqueued.
int copy_streams(CopyStreams& out) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (major != 10 || minor != 0) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_copy_mutex);
  CopyStreams& cs = g_copy[dev];
  if (!cs.up && cudaStreamCreateWithFlags(&cs.up, cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
  if (!cs.down && cudaStreamCreateWithFlags(&cs.down, cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
  out = cs;
  return ATTN_OK;
}

// Events of one call; destroyed when the call returns (an event still pending
// in a stream is released by the runtime once the device reaches it).
struct EventSet {
  std::vector<cudaEvent_t> ev;
  EventSet() = default;
  EventSet(const EventSet&) = delete;
  EventSet& operator=(const EventSet&) = delete;
  ~EventSet() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev.push_back(e);
    return e;
  }
};

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

// The sizes of one tensor set: q (and out) per unit, k and v per unit, lse per unit.
struct Units {
  int64_t count, group;
  size_t q, kv, out, lse;
};

// The outputs of a set (out, lse) overlap neither each other nor the inputs.
bool outputs_overlap(const void* q, const void* k, const void* v, const void* out, const void* lse,
                     const Units& u) {
  const size_t nq = u.q * u.count, nkv = u.kv * u.count, no = u.out * u.count, nl = u.lse * u.count;
  return overlaps(out, no, q, nq) || overlaps(out, no, k, nkv) || overlaps(out, no, v, nkv) ||
         overlaps(lse, nl, out, no) || overlaps(lse, nl, q, nq) || overlaps(lse, nl, k, nkv) ||
         overlaps(lse, nl, v, nkv);
}

// Every check attn_fwd makes before enqueueing, made once for the whole job so
// that a bad argument enqueues nothing (each chunk's call checks again).
int validate(const void* const ptrs[10], int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d, int eb,
             float score_scale, float v_scale, int mask_kind, int64_t window, int64_t chunks, Units& u) {
  for (int i = 0; i < 10; ++i)
    if (!ptrs[i]) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (mask_kind != ATTN_MASK_FULL && mask_kind != ATTN_MASK_CAUSAL && mask_kind != ATTN_MASK_SLIDING_WINDOW)
    return ATTN_ERR_INVALID_ARG;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 30) || B * Hq > (int64_t(1) << 30)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // Byte counts below are int64 products: keep q's element count within 2^50.
  if (static_cast<double>(B * Hq) * static_cast<double>(N) * static_cast<double>(d) > 1125899906842624.0)
    return ATTN_ERR_INVALID_ARG;
  if (eb == 1 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(score_scale) || !(score_scale > 0.f) || !std::isfinite(v_scale) || !(v_scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  if (chunks < 0) return ATTN_ERR_INVALID_ARG;
  u.count = B * Hkv;
  u.group = Hq / Hkv;
  u.q = static_cast<size_t>(u.group * N * d) * eb;
  u.kv = static_cast<size_t>(N * d) * eb;
  u.out = static_cast<size_t>(u.group * N * d) * 2;
  u.lse = static_cast<size_t>(u.group * N) * 4;
  const void* const* h = ptrs;      // hq, hk, hv, hout, hlse
  const void* const* dv = ptrs + 5;  // dq, dk, dv, dout, dlse
  if (outputs_overlap(dv[0], dv[1], dv[2], dv[3], dv[4], u) || outputs_overlap(h[0], h[1], h[2], h[3], h[4], u))
    return ATTN_ERR_INVALID_ARG;
  // The uploads write the device staging inputs, so unlike attn_fwd's inputs
  // (which may alias, e.g. k == v) they must not overlap one another.
  const size_t nq = u.q * u.count, nkv = u.kv * u.count;
  if (overlaps(dv[0], nq, dv[1], nkv) || overlaps(dv[0], nq, dv[2], nkv) || overlaps(dv[1], nkv, dv[2], nkv))
    return ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (reinterpret_cast<uintptr_t>(dv[i]) & 15u) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(dv[4]) & 3u) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

char* at(const void* base, int64_t unit_index, size_t unit_bytes) {
  return static_cast<char*>(const_cast<void*>(base)) + static_cast<size_t>(unit_index) * unit_bytes;
}

// eb = 2: bf16 inputs through attn_fwd_ex; eb = 1: E4M3 codes through attn_fwd_fp8_ex.
int host_forward(const void* hq, const void* hk, const void* hv, void* hout, float* hlse, void* dq, void* dk,
                 void* dv, void* dout, float* dlse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                 int eb, float scale, float q_scale, float k_scale, float v_scale, int mask_kind, int64_t window,
                 int64_t chunks, cudaStream_t stream) {
  const void* const ptrs[10] = {hq, hk, hv, hout, hlse, dq, dk, dv, dout, dlse};
  Units u{};
  int st = validate(ptrs, B, Hq, Hkv, N, d, eb, scale * q_scale * k_scale, v_scale, mask_kind, window, chunks, u);
  if (st != ATTN_OK) return st;
  if (chunks == 0) chunks = kDefaultChunks;
  if (chunks > u.count) chunks = u.count;

  CopyStreams cs;
  st = copy_streams(cs);
  if (st != ATTN_OK) return st;
  EventSet events;
  // The join's two events are made before anything is enqueued, so a join never
  // lacks an event; if recording or waiting on them fails, both copy streams are
  // synchronised instead, which orders their copies before anything `stream` runs later.
  cudaEvent_t start = events.make(), join_up = events.make(), join_down = events.make();
  if (!start || !join_up || !join_down) return ATTN_ERR_CUDA;
  if (cudaEventRecord(start, stream) != cudaSuccess) return ATTN_ERR_CUDA;
  // Nothing is copied into the staging buffers before earlier work on `stream` is done.
  if (cudaStreamWaitEvent(cs.up, start, 0) != cudaSuccess || cudaStreamWaitEvent(cs.down, start, 0) != cudaSuccess)
    return ATTN_ERR_CUDA;
  // On every exit past this point `stream` waits for both copy streams, so that
  // whatever was enqueued is ordered before the caller's later work.
  auto join = [&](int status) -> int {
    if (cudaEventRecord(join_up, cs.up) != cudaSuccess || cudaEventRecord(join_down, cs.down) != cudaSuccess ||
        cudaStreamWaitEvent(stream, join_up, 0) != cudaSuccess ||
        cudaStreamWaitEvent(stream, join_down, 0) != cudaSuccess) {
      cudaStreamSynchronize(cs.up);
      cudaStreamSynchronize(cs.down);
      return ATTN_ERR_CUDA;
    }
    return status;
  };
  auto range = [&](int64_t c, int64_t& u0, int64_t& n) {
    u0 = u.count * c / chunks;
    n = u.count * (c + 1) / chunks - u0;
  };

  std::vector<cudaEvent_t> done(static_cast<size_t>(chunks), nullptr);
  for (int64_t c = 0; c < chunks; ++c) {
    int64_t u0 = 0, n = 0;
    range(c, u0, n);
    cudaEvent_t in = events.make();
    done[c] = events.make();
    if (!in || !done[c] ||
        cudaMemcpyAsync(at(dq, u0, u.q), at(hq, u0, u.q), n * u.q, cudaMemcpyDefault, cs.up) != cudaSuccess ||
        cudaMemcpyAsync(at(dk, u0, u.kv), at(hk, u0, u.kv), n * u.kv, cudaMemcpyDefault, cs.up) != cudaSuccess ||
        cudaMemcpyAsync(at(dv, u0, u.kv), at(hv, u0, u.kv), n * u.kv, cudaMemcpyDefault, cs.up) != cudaSuccess ||
        cudaEventRecord(in, cs.up) != cudaSuccess || cudaStreamWaitEvent(stream, in, 0) != cudaSuccess)
      return join(ATTN_ERR_CUDA);
    void* o = at(dout, u0, u.out);
    float* l = reinterpret_cast<float*>(at(dlse, u0, u.lse));
    if (eb == 2)
      st = attn_fwd_ex(at(dq, u0, u.q), at(dk, u0, u.kv), at(dv, u0, u.kv), o, l, 1, n * u.group, n, N, d, scale,
                       mask_kind, window, stream, nullptr);
    else
      st = attn_fwd_fp8_ex(at(dq, u0, u.q), at(dk, u0, u.kv), at(dv, u0, u.kv), q_scale, k_scale, v_scale, o, l, 1,
                           n * u.group, n, N, d, scale, mask_kind, window, stream, nullptr);
    if (st != ATTN_OK) return join(st);
    if (cudaEventRecord(done[c], stream) != cudaSuccess) return join(ATTN_ERR_CUDA);
  }
  // Downloads are enqueued after every upload and launch, so that a pageable
  // destination (whose copy the runtime may perform synchronously) does not
  // hold back the uploads and kernels of later chunks.
  for (int64_t c = 0; c < chunks; ++c) {
    int64_t u0 = 0, n = 0;
    range(c, u0, n);
    if (cudaStreamWaitEvent(cs.down, done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(at(hout, u0, u.out), at(dout, u0, u.out), n * u.out, cudaMemcpyDefault, cs.down) !=
            cudaSuccess ||
        cudaMemcpyAsync(at(hlse, u0, u.lse), at(dlse, u0, u.lse), n * u.lse, cudaMemcpyDefault, cs.down) !=
            cudaSuccess)
      return join(ATTN_ERR_CUDA);
  }
  return join(ATTN_OK);
}

}  // namespace

extern "C" {

int attn_fwd_host(const void* hq, const void* hk, const void* hv, void* hout, float* hlse, void* dq, void* dk,
                  void* dv, void* dout, float* dlse, int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t d,
                  float scale, int mask_kind, int64_t window, int64_t chunks, cudaStream_t stream) {
  return host_forward(hq, hk, hv, hout, hlse, dq, dk, dv, dout, dlse, B, Hq, Hkv, N, d, 2, scale, 1.f, 1.f, 1.f,
                      mask_kind, window, chunks, stream);
}

int attn_fwd_fp8_host(const void* hq, const void* hk, const void* hv, float q_scale, float k_scale, float v_scale,
                      void* hout, float* hlse, void* dq, void* dk, void* dv, void* dout, float* dlse, int64_t B,
                      int64_t Hq, int64_t Hkv, int64_t N, int64_t d, float scale, int mask_kind, int64_t window,
                      int64_t chunks, cudaStream_t stream) {
  if (!std::isfinite(q_scale) || !(q_scale > 0.f) || !std::isfinite(k_scale) || !(k_scale > 0.f) ||
      !std::isfinite(scale) || !(scale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  return host_forward(hq, hk, hv, hout, hlse, dq, dk, dv, dout, dlse, B, Hq, Hkv, N, d, 1, scale, q_scale, k_scale,
                      v_scale, mask_kind, window, chunks, stream);
}

}  // extern "C"
