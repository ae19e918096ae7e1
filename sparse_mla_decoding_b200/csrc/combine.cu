// combine.cu -- LSE-weighted merge of split-KV partials.
//
// Source: "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路", section
// 合并与性能账本: every split leaves a partial output and its lse; the combine
// kernel normalises them into the final result using the lse values, and it
// is chained to the split kernel with Programmatic Dependent Launch so its
// launch overlaps the tail of the split kernel.
//
// For a request r with S_r = num_splits[r+1] - num_splits[r] > 1 splits and a
// head h: lse = ln(sum_s exp(lse_s)), o = sum_s exp(lse_s - lse) * o_s, with
// o_s already normalised within its split.  Every lse_s = -inf (no valid slot
// anywhere) gives o = 0, lse = -inf.  Requests with one split were finished
// by the split kernel and are skipped.
//
// The merge is bound by the latency of reading the fp32 partials, so the
// layout is chosen for memory-level parallelism: one warp per (request, head),
// lane l owning the 16 output columns [16 l, 16 l + 16) (four 16-byte loads
// per split), with the rows of the first two splits loaded before the lse
// reductions, so their round trip overlaps the lse loads'.
#include <cuda_bf16.h>

#include <cstdint>

#include "sm100.cuh"
#include "splitkv_mla.h"

namespace smla {

// grid: (batch*s_q, ceil(h_q / kCombineHeadsPerCta)); block: 32 * kCombineHeadsPerCta threads.
__global__ void __launch_bounds__(32 * kCombineHeadsPerCta) combine_kernel(const int32_t* __restrict__ num_splits,
                                                                           const float* __restrict__ o_accum,
                                                                           const float* __restrict__ lse_accum,
                                                                           int h_q, int max_splits,
                                                                           __nv_bfloat16* __restrict__ o,
                                                                           float* __restrict__ lse) {
  // Everything this kernel reads is produced by the split kernel: wait for it.
  pdl_wait_primary();
  const int r = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * kCombineHeadsPerCta + (threadIdx.x >> 5);
  const int s0 = num_splits[r];
  const int ns = num_splits[r + 1] - s0;
  // one split: written by the split kernel; out-of-range tables were flagged there
  if (h >= h_q || ns <= 1 || s0 < 0 || s0 + ns > max_splits) return;

  const float* lse_s = lse_accum + (size_t)s0 * h_q + h;   // split s at lse_s[s * h_q]
  const size_t split_stride = (size_t)h_q * 512;
  const float* base = o_accum + ((size_t)s0 * h_q + h) * 512 + 16 * lane;
  float4 va[4], vb[4];   // splits s and s + 1 of the loop below, the first pair loaded now
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    va[i] = reinterpret_cast<const float4*>(base)[i];
    vb[i] = reinterpret_cast<const float4*>(base + split_stride)[i];
  }
  float m = -INFINITY;
  for (int s = lane; s < ns; s += 32) m = fmaxf(m, lse_s[(size_t)s * h_q]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __nv_bfloat16* out = o + ((size_t)r * h_q + h) * 512 + 16 * lane;
  if (m == -INFINITY) {
    reinterpret_cast<uint4*>(out)[0] = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(out)[1] = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) lse[(size_t)r * h_q + h] = -INFINITY;
    return;
  }
  // Work in base 2: exp(x) = exp2(x * log2 e).
  const float kLog2e = 1.4426950408889634f;
  float sum = 0.f;
  for (int s = lane; s < ns; s += 32) sum += exp2f((lse_s[(size_t)s * h_q] - m) * kLog2e);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float lse_r = m + logf(sum);

  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < ns; s += 2) {
    const bool two = s + 1 < ns;
    if (s > 0) {
      const float4* a = reinterpret_cast<const float4*>(base + (size_t)s * split_stride);
      const float4* b = reinterpret_cast<const float4*>(base + (size_t)(two ? s + 1 : s) * split_stride);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        va[i] = a[i];
        vb[i] = b[i];
      }
    }
    const float wa = exp2f((lse_s[(size_t)s * h_q] - lse_r) * kLog2e);
    const float wb = two ? exp2f((lse_s[(size_t)(s + 1) * h_q] - lse_r) * kLog2e) : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[4 * i + 0] += wa * va[i].x + wb * vb[i].x;
      acc[4 * i + 1] += wa * va[i].y + wb * vb[i].y;
      acc[4 * i + 2] += wa * va[i].z + wb * vb[i].z;
      acc[4 * i + 3] += wa * va[i].w + wb * vb[i].w;
    }
  }
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    pk[i] = *reinterpret_cast<uint32_t*>(&v);
  }
  reinterpret_cast<uint4*>(out)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  reinterpret_cast<uint4*>(out)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0) lse[(size_t)r * h_q + h] = lse_r;
}

}  // namespace smla
