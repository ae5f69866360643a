// Merge of partial attention results by their log-sum-exp, the combining step
// of ring attention ("Attention Mechanism Variants Beyond Self-Attention",
// tempatgunting.com, section "Ring Attention for Very Long Sequences": each GPU
// holds a chunk of the sequence and KV blocks rotate around a ring, so a query
// chunk meets the key chunks one at a time).  For one query row, attention over
// the union of two disjoint key sets with partial results (O_a, lse_a) and
// (O_b, lse_b) is
//   lse = ln(e^lse_a + e^lse_b),  O = (e^(lse_a - lse) O_a + e^(lse_b - lse) O_b),
// because each partial O is normalised by its own softmax sum e^lse.
// One warp per row; the accumulator is fp32, the partials are the forward's
// out (bf16, or fp32 with the forward's out_fp32 option) and fp32 lse.
#include "attn.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

namespace {

template <int D, typename Part>
__global__ void __launch_bounds__(256) attn_merge_kernel(float* acc_o, float* acc_lse, const Part* part_o,
                                                         const float* part_lse, __nv_bfloat16* out, int64_t rows,
                                                         int mode) {
  constexpr int V = D / 32;  // columns per lane (4 or 2)
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float* a = acc_o + row * D + lane * V;
  const Part* pp = part_o + row * D + lane * V;
  float p[V];
#pragma unroll
  for (int i = 0; i < V; i += 2) {
    if constexpr (sizeof(Part) == 4) {
      const float2 h = *reinterpret_cast<const float2*>(pp + i);
      p[i] = h.x;
      p[i + 1] = h.y;
    } else {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(pp + i);
      p[i] = __bfloat162float(h.x);
      p[i + 1] = __bfloat162float(h.y);
    }
  }
  const float lp = part_lse[row];
  float r[V];
  float lse;
  if ((mode & 1) == 0) {
#pragma unroll
    for (int i = 0; i < V; ++i) r[i] = p[i];
    lse = lp;
  } else {
    const float la = acc_lse[row];
    const float m = fmaxf(la, lp);
    if (m == -INFINITY) {  // neither part saw a key: keep the empty row
#pragma unroll
      for (int i = 0; i < V; ++i) r[i] = 0.f;
      lse = -INFINITY;
    } else {
      const float wa = expf(la - m), wp = expf(lp - m);
      const float s = wa + wp;
      const float ca = wa / s, cp = wp / s;
      float av[V];
      if constexpr (V == 4) {
        const float4 t = *reinterpret_cast<const float4*>(a);
        av[0] = t.x, av[1] = t.y, av[2] = t.z, av[3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(a);
        av[0] = t.x, av[1] = t.y;
      }
#pragma unroll
      for (int i = 0; i < V; ++i) r[i] = ca * av[i] + cp * p[i];
      lse = m + logf(s);
    }
  }
  if constexpr (V == 4) {
    *reinterpret_cast<float4*>(a) = make_float4(r[0], r[1], r[2], r[3]);
  } else {
    *reinterpret_cast<float2*>(a) = make_float2(r[0], r[1]);
  }
  if (lane == 0) acc_lse[row] = lse;
  if (out) {
    __nv_bfloat16* o = out + row * D + lane * V;
#pragma unroll
    for (int i = 0; i < V; i += 2) *reinterpret_cast<__nv_bfloat162*>(o + i) = __floats2bfloat162_rn(r[i], r[i + 1]);
  }
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

}  // namespace

extern "C" int attn_merge(float* acc_out, float* acc_lse, const void* part_out, const float* part_lse, void* out,
                          int64_t rows, int64_t d, int mode, cudaStream_t stream) {
  if (!acc_out || !acc_lse || !part_out || !part_lse) return ATTN_ERR_INVALID_ARG;
  if (rows < 1 || rows > (int64_t(1) << 33) || mode < 0 || mode > 3) return ATTN_ERR_INVALID_ARG;
  const bool part_f32 = (mode & 2) != 0;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const uintptr_t ua = reinterpret_cast<uintptr_t>(acc_out), up = reinterpret_cast<uintptr_t>(part_out),
                  uo = reinterpret_cast<uintptr_t>(out);
  if ((ua & 15u) || (up & (part_f32 ? 15u : 7u)) || (uo & 7u) || (reinterpret_cast<uintptr_t>(acc_lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return ATTN_ERR_MISALIGNED;
  const size_t acc_b = static_cast<size_t>(rows) * d * 4, out_b = static_cast<size_t>(rows) * d * 2,
               part_b = part_f32 ? acc_b : out_b, lse_b = static_cast<size_t>(rows) * 4;
  // Outputs (acc_out, acc_lse, out) must not overlap each other or the partial inputs.
  if (overlaps(acc_out, acc_b, acc_lse, lse_b) || overlaps(acc_out, acc_b, part_out, part_b) ||
      overlaps(acc_out, acc_b, part_lse, lse_b) || overlaps(acc_lse, lse_b, part_out, part_b) ||
      overlaps(acc_lse, lse_b, part_lse, lse_b) || overlaps(out, out_b, acc_out, acc_b) ||
      overlaps(out, out_b, acc_lse, lse_b) || overlaps(out, out_b, part_lse, lse_b))
    return ATTN_ERR_INVALID_ARG;
  // A bf16 out may alias a bf16 part_out (each element is read before the same
  // lane writes it); with an fp32 partial the rows have different widths, so no overlap.
  if (part_f32 && overlaps(out, out_b, part_out, part_b)) return ATTN_ERR_INVALID_ARG;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (part_f32) {
    const auto* p = static_cast<const float*>(part_out);
    if (d == 128)
      attn_merge_kernel<128><<<blocks, 256, 0, stream>>>(acc_out, acc_lse, p, part_lse, o, rows, mode);
    else
      attn_merge_kernel<64><<<blocks, 256, 0, stream>>>(acc_out, acc_lse, p, part_lse, o, rows, mode);
  } else {
    const auto* p = static_cast<const __nv_bfloat16*>(part_out);
    if (d == 128)
      attn_merge_kernel<128><<<blocks, 256, 0, stream>>>(acc_out, acc_lse, p, part_lse, o, rows, mode);
    else
      attn_merge_kernel<64><<<blocks, 256, 0, stream>>>(acc_out, acc_lse, p, part_lse, o, rows, mode);
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
