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
#include <cuda_bf16.h>

#include <cstdint>

#include "sm100.cuh"

namespace smla {

constexpr int kCombineThreads = 128;  // 128 threads x 4 values = one 512-wide head row

// grid: (batch*s_q, h_q); block: 128 threads, thread t owns o[4t .. 4t+3].
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const int32_t* __restrict__ num_splits,
                                                                  const float* __restrict__ o_accum,
                                                                  const float* __restrict__ lse_accum, int h_q,
                                                                  int max_splits,
                                                                  __nv_bfloat16* __restrict__ o,
                                                                  float* __restrict__ lse) {
  // Everything this kernel reads is produced by the split kernel: wait for it.
  pdl_wait_primary();
  const int r = blockIdx.x;
  const int h = blockIdx.y;
  const int s0 = num_splits[r];
  const int ns = num_splits[r + 1] - s0;
  if (ns <= 1 || s0 < 0 || s0 + ns > max_splits) return;   // out-of-range tables were flagged upstream

  float m = -INFINITY;
  for (int s = 0; s < ns; ++s) m = fmaxf(m, lse_accum[(size_t)(s0 + s) * h_q + h]);
  const int t = threadIdx.x;
  __nv_bfloat16* out = o + ((size_t)r * h_q + h) * 512 + 4 * t;
  if (m == -INFINITY) {
    *reinterpret_cast<uint2*>(out) = make_uint2(0u, 0u);
    if (t == 0) lse[(size_t)r * h_q + h] = -INFINITY;
    return;
  }
  // Work in base 2: exp(x) = exp2(x * log2 e).
  const float kLog2e = 1.4426950408889634f;
  float sum = 0.f;
  for (int s = 0; s < ns; ++s) sum += exp2f((lse_accum[(size_t)(s0 + s) * h_q + h] - m) * kLog2e);
  const float lse_r = m + logf(sum);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < ns; ++s) {
    const float w = exp2f((lse_accum[(size_t)(s0 + s) * h_q + h] - lse_r) * kLog2e);
    const float4 v = *reinterpret_cast<const float4*>(o_accum + ((size_t)(s0 + s) * h_q + h) * 512 + 4 * t);
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&lo);
  packed.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out) = packed;
  if (t == 0) lse[(size_t)r * h_q + h] = lse_r;
}

}  // namespace smla
