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
//
// Dense decoding (sched_meta_dense_kernel): request r = b * s_q + t covers its
// visible cache tokens, len_r = seqlen[b] (or seqlen[b] - (s_q - 1 - t) under
// the causal mask, where the s_q new tokens are the last s_q positions), in
// n_r = max(1, ceil(len_r / 64)) tiles.  The tile counts differ per request,
// so the kernel scans them into a tile prefix (tiles before request r), then
// lays out the parts exactly as above with tile positions counted within each
// request; each part finds its first and last request by binary search.
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

namespace {

// Exclusive prefix sums of value(r), r in [0, R), written to out[0..R-1] and
// out[R] = the total, by one CTA (whole block; blockDim.x a multiple of 32,
// at most 1024).  Sums are taken in int64 and stored as int32; the return
// value is the int64 total (a total past INT32_MAX means the stored values
// are not usable).  Integer sums: deterministic.
template <class F>
__device__ int64_t block_exclusive_scan(int R, F value, int32_t* out) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < R; base += blockDim.x) {
    const int r = base + threadIdx.x;
    const int64_t v = r < R ? value(r) : 0;
    int64_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int64_t w = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      if (lane < nwarps) warp_tot[lane] = w;
    }
    __syncthreads();
    const int64_t incl = x + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (r < R) out[r] = (int32_t)(carry + incl - v);
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += incl;
    __syncthreads();
  }
  const int64_t total = carry;
  if (threadIdx.x == 0) out[R] = (int32_t)total;
  __syncthreads();
  return total;
}

}  // namespace

// One CTA.  A schedule whose total tile count does not fit in int32 is
// written as invalid parts (begin request -1), which the decode kernel
// rejects and flags.
__global__ void __launch_bounds__(1024) sched_meta_dense_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                                 int s_q, int causal, int P,
                                                                 int32_t* __restrict__ sched_meta,
                                                                 int32_t* __restrict__ num_splits,
                                                                 int32_t* __restrict__ tile_prefix) {
  pdl_launch_dependents();
  const int R = batch * s_q;
  const int64_t total = block_exclusive_scan(R, [&](int r) -> int64_t {
    const int t = r % s_q;
    int64_t len = seqlens[r / s_q];
    if (causal) len -= (s_q - 1 - t);
    if (len < 0) len = 0;
    const int64_t n = (len + 63) / 64;
    return n > 0 ? n : 1;
  }, tile_prefix);
  const bool fits = total < 0x7FFFFFFFll;
  const int64_t L = total > 0 ? (total + P - 1) / P : 1;
  const int32_t* tp = tile_prefix;
  block_exclusive_scan(R, [&](int r) -> int64_t {
    return fits ? ((int64_t)tp[r + 1] - 1) / L - (int64_t)tp[r] / L + 1 : 0;
  }, num_splits);
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    int32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int64_t g0 = (int64_t)p * L;
    if (!fits) {
      m[0] = -1;
    } else if (g0 >= total) {
      m[5] = 1;
    } else {
      int64_t g1 = g0 + L;
      if (g1 > total) g1 = total;
      // the last request whose first tile is at or before global tile g
      auto owner = [&](int64_t g) {
        int lo = 0, hi = R - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (tp[mid] <= g) lo = mid;
          else hi = mid - 1;
        }
        return lo;
      };
      const int rb = owner(g0);
      const int re = g1 == total ? R : owner(g1);
      m[0] = rb;
      m[1] = (int32_t)(g0 - tp[rb]);
      m[2] = re;
      m[3] = re == R ? 0 : (int32_t)(g1 - tp[re]);
      m[4] = (int32_t)(num_splits[rb] + p - (int64_t)tp[rb] / L);
    }
    int4* dst = reinterpret_cast<int4*>(sched_meta + (size_t)p * 8);
    dst[0] = make_int4(m[0], m[1], m[2], m[3]);
    dst[1] = make_int4(m[4], m[5], m[6], m[7]);
  }
}

}  // namespace smla
