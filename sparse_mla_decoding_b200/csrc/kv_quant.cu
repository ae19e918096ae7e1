// kv_quant.cu -- write tokens into the 656-byte FP8 KV rows.
//
// Source: "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路", section
// 数据加载 (the first 512 dimensions of each token are quantised per 1x128 tile
// to float8_e4m3; the RoPE part stays bf16), and "deepseek-ai/FlashMLA"
// (gitgenius summary): the row holds 512 bytes of quantised values, 16 bytes
// of scale factors and 128 bytes of unquantised RoPE.
//
// Per tile: scale = amax / 448 in float32 (448 = largest e4m3 magnitude),
// byte = e4m3(x / scale) rounded to nearest even and saturated; an all-zero
// tile stores scale 0 and zero bytes.  One warp per token: lane l owns latent
// values [16l, 16l+16), so the 8 lanes 8q..8q+7 hold tile q.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "sm100.cuh"

namespace smla {

constexpr int kQuantWarps = 8;

__global__ void __launch_bounds__(32 * kQuantWarps) quantize_kv_kernel(const __nv_bfloat16* __restrict__ latent,
                                                                       const __nv_bfloat16* __restrict__ rope,
                                                                       int64_t n_tokens,
                                                                       const int64_t* __restrict__ slot_mapping,
                                                                       uint8_t* __restrict__ kvcache,
                                                                       int64_t num_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t token = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (token >= n_tokens) return;
  const int64_t row = slot_mapping ? slot_mapping[token] : token;
  if (row < 0 || row >= num_rows) return;
  uint8_t* dst = kvcache + row * 656;

  // 16 latent values of this lane (two 16-byte loads).
  const uint4* src = reinterpret_cast<const uint4*>(latent + token * 512 + lane * 16);
  uint4 raw[2] = {src[0], src[1]};
  float x[16];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
      float2 f = __bfloat1622float2(p);
      x[8 * i + 2 * j] = f.x;
      x[8 * i + 2 * j + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  // reduce over the 8 lanes of this tile
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = __fdiv_rn(amax, 448.0f);

  uint32_t packed[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t word = 0;
    if (scale != 0.f) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float2 pair = make_float2(__fdiv_rn(x[4 * j + 2 * k], scale), __fdiv_rn(x[4 * j + 2 * k + 1], scale));
        __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
        word |= (uint32_t)q << (16 * k);
      }
    }
    packed[j] = word;
  }
  *reinterpret_cast<uint4*>(dst + lane * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);

  // scales: lane 8q holds tile q's scale
  const float s0 = __shfl_sync(0xffffffffu, scale, 0);
  const float s1 = __shfl_sync(0xffffffffu, scale, 8);
  const float s2 = __shfl_sync(0xffffffffu, scale, 16);
  const float s3 = __shfl_sync(0xffffffffu, scale, 24);
  if (lane == 0) *reinterpret_cast<float4*>(dst + 512) = make_float4(s0, s1, s2, s3);
  // RoPE: 128 bytes, 8 lanes x 16 bytes
  if (lane < 8)
    *reinterpret_cast<uint4*>(dst + 528 + 16 * lane) =
        reinterpret_cast<const uint4*>(rope + token * 64)[lane];
}

}  // namespace smla
