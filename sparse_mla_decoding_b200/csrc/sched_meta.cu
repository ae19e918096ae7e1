// sched_meta.cu -- tile-scheduler metadata kernel.
//
// Source: "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路", section
// 调度: before the main kernel, a small kernel spreads (request, KV-range) work
// units evenly over all SMs; the main kernel follows the table with no
// run-time arbitration; the table is reusable while shapes stay the same.
//
// In sparse decoding the work of a request is its index slots, cut into
// n = ceil(topk / 64) tiles.  The R*n tiles, in (request, tile) order, are cut
// into P consecutive ranges of L = ceil(R*n / P) tiles (part p owns
// [p*L, min((p+1)*L, R*n))).  Every output entry is computed independently
// from closed forms, so the kernel needs no scan:
//   first(r)      = floor(r*n / L)                        (part holding tile 0 of r)
//   num_splits[r] = sum_{r'<r} S_r' = floor(r*n/L) + r - floor(r*g/L),  g = gcd(n, L)
// (S_r' = first(r'+1) - first(r') + 1 - [L divides (r'+1)*n]; the bracket
// counts the j in [1, r] with L | j*n, i.e. the multiples of L/g.)
#include <cstdint>

#include "sm100.cuh"

namespace smla {

__device__ __forceinline__ int64_t gcd64(int64_t a, int64_t b) {
  while (b != 0) {
    int64_t t = a % b;
    a = b;
    b = t;
  }
  return a;
}

__global__ void __launch_bounds__(256) sched_meta_kernel(int R, int n, int P, int32_t* __restrict__ sched_meta,
                                                          int32_t* __restrict__ num_splits) {
  // Let the dependent split-KV kernel start its prologue early; it waits for
  // this grid's completion before it reads the table.
  pdl_launch_dependents();
  const int64_t total = (int64_t)R * n;
  const int64_t L = total > 0 ? (total + P - 1) / P : 1;
  const int64_t g = gcd64((int64_t)n, L);
  for (int r = threadIdx.x; r <= R; r += blockDim.x) {
    const int64_t v = ((int64_t)r * n) / L + r - ((int64_t)r * g) / L;
    num_splits[r] = (int32_t)v;
  }
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    int32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int64_t g0 = (int64_t)p * L;
    if (g0 >= total) {
      m[5] = 1;
    } else {
      int64_t g1 = g0 + L;
      if (g1 > total) g1 = total;
      const int64_t r0 = g0 / n;
      m[0] = (int32_t)r0;
      m[1] = (int32_t)(g0 % n);
      m[2] = (int32_t)(g1 / n);
      m[3] = (int32_t)(g1 % n);
      const int64_t first0 = (r0 * n) / L;
      const int64_t ns0 = (r0 * n) / L + r0 - (r0 * g) / L;
      m[4] = (int32_t)(ns0 + p - first0);
    }
    int4* dst = reinterpret_cast<int4*>(sched_meta + (size_t)p * 8);
    dst[0] = make_int4(m[0], m[1], m[2], m[3]);
    dst[1] = make_int4(m[4], m[5], m[6], m[7]);
  }
}

}  // namespace smla
