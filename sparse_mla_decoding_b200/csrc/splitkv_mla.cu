// splitkv_mla.cu -- the split-KV sparse MLA decode kernel for sm_100a.
//
// Sources (cited by page title and section):
//   "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路":
//     调度 -- the main kernel takes its (request, KV-range) jobs from the
//             precomputed table with no run-time arbitration; long requests
//             are split over several SMs and merged afterwards;
//     数据加载 -- the 656-byte row: 512 e4m3 values dequantised to bf16 with
//             their 1x128 tile scales, concatenated with the 64 bf16 RoPE
//             values into the 576-wide key; bf16 MMAs with fp32 accumulation;
//     计算环节二 (Seesaw) -- the result is the FlashAttention online softmax;
//     合并与性能账本 -- each split leaves a partial output and its lse.
//   "deepseek-ai/FlashMLA" (agentlenshq), 技術的な詳細 -- -1 in indices marks
//     an entry the kernel ignores.
//
// Design on B200 (not the Hopper design of the pages):
//   * One CTA owns up to 64 query heads of one request at a time (M = 64 of
//     every tcgen05.mma); 128 heads use two CTAs per scheduler part.
//   * Per tile of 64 index slots: the slots are mapped through the block
//     table, the 656-byte rows are gathered with 16-byte coalesced loads (one
//     warp per row, one lane per 16 latent bytes), dequantised exactly
//     (e4m3 -> f16 -> f32, times the tile scale in f32, round to bf16) and
//     stored as a 64 x 576 bf16 K tile in the 128-byte-swizzled K-major
//     layout the tensor core reads.  The same tile, read MN-major, is V.
//   * S = Q K^T (M=64, N=64, K=576) and O += P V (M=64, N=256 twice, K=64)
//     run as tcgen05.mma with fp32 accumulators in tensor memory.  The
//     64 x 512 output accumulator takes 256 TMEM columns: its two 256-wide
//     halves sit in the same columns, in the lower and upper 16 lanes of each
//     32-lane sub-partition (the M=64 accumulator uses 16 lanes per
//     sub-partition), which leaves room for S.
//   * Online softmax in base 2 by the four warps that own the TMEM lanes;
//     P is rounded to bf16 once and the same rounded values feed both the PV
//     MMA and the running denominator.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "sm100.cuh"
#include "splitkv_mla.h"

namespace smla {

namespace {

constexpr int kRows = 64;              // index slots per tile
constexpr int kHeads = 64;             // heads per CTA (MMA M)
constexpr int kThreads = 256;
constexpr int kKBlocks = 9;            // 576 / 64 bf16 per 128-byte swizzle line
constexpr int kAtom = kRows * 128;     // bytes of one 64-row x 128-byte column block
constexpr int kQBytes = kKBlocks * kAtom;
constexpr int kKBytes = kKBlocks * kAtom;
constexpr int kPBytes = kAtom;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;          // O: columns [0, 256), halves at lane offsets 0 / 16
constexpr uint32_t kSCol = 256;        // S: columns [256, 320), lanes 0-15 of each sub-partition
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: no legitimate wait comes close

struct __align__(16) SmemTail {
  int64_t row_off[kRows];   // byte offset of each gathered row in the cache, -1 if invalid
  uint64_t bar_s;           // S MMA complete
  uint64_t bar_o;           // PV MMA complete
  uint32_t tmem_base;
  int32_t abort_flag;
};

constexpr int kSmemBytes = kQBytes + kKBytes + kPBytes + (int)sizeof(SmemTail) + 1024;

__device__ __forceinline__ uint32_t swz(int row, int chunk16) {
  // byte offset of 16-byte chunk `chunk16` (0..7) of `row` inside one column block
  return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// 16 e4m3 values (one 16-byte chunk) -> 16 bf16 = bf16(float(e4m3) * scale).
__device__ __forceinline__ void dequant16(const uint4& raw, float scale, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t out[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] & 0xFFFFu), __NV_E4M3);
    __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] >> 16), __NV_E4M3);
    float2 f01 = __half22float2(*reinterpret_cast<__half2*>(&h01));
    float2 f23 = __half22float2(*reinterpret_cast<__half2*>(&h23));
    out[2 * j] = bf162_bits(__floats2bfloat162_rn(__fmul_rn(f01.x, scale), __fmul_rn(f01.y, scale)));
    out[2 * j + 1] = bf162_bits(__floats2bfloat162_rn(__fmul_rn(f23.x, scale), __fmul_rn(f23.y, scale)));
  }
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) splitkv_mla_kernel(const SplitKVParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;
  uint8_t* sP = sK + kKBytes;
  SmemTail* tail = reinterpret_cast<SmemTail*>(sP + kPBytes);
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aP = smem_u32(sP);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int part = blockIdx.x;
  const int hg = blockIdx.y;                       // head group: heads [64*hg, 64*hg + 64)
  const int heads_here = min(kHeads, p.h_q - kHeads * hg);

  if (tid == 0) {
    mbar_init(&tail->bar_s, 1);
    mbar_init(&tail->bar_o, 1);
    tail->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tail->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  // The schedule is written by the metadata kernel that precedes us.
  pdl_wait_primary();
  const int4 m0 = *reinterpret_cast<const int4*>(p.sched_meta + (size_t)part * 8);
  const int4 m1 = *reinterpret_cast<const int4*>(p.sched_meta + (size_t)part * 8 + 4);
  // Metadata comes from the caller: check it against this call's shapes so a
  // mismatched table cannot send reads or writes out of bounds.
  bool empty = m1.y != 0;
  if (!empty) {
    const bool ok = m0.x >= 0 && m0.x < p.num_requests && m0.y >= 0 && m0.y < p.n_tiles && m0.z >= m0.x &&
                    m0.z <= p.num_requests && m0.w >= 0 && m0.w < p.n_tiles &&
                    (m0.z > m0.x || m0.w > m0.y) && (m0.z < p.num_requests || m0.w == 0);
    if (!ok) {
      if (tid == 0) report_status(p.status, kStatusBadSchedule);
      empty = true;
    }
  }

  uint32_t phase_s = 0, phase_o = 0;
  const uint32_t idesc_s = idesc_bf16_f32(kHeads, kRows, false);
  const uint32_t idesc_pv = idesc_bf16_f32(kHeads, 256, true);
  const float scale_log2 = p.scale_log2;

  // softmax row owned by this thread (warps 0-3, lanes 0-15)
  const bool softmax_warp = warp < 4;
  const int my_head = 16 * (warp & 3) + (lane & 15);   // row of the CTA's 64-head tile
  const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;

  int r = m0.x, tile = m0.y;
  const int end_r = m0.z, end_tile = m0.w;
  bool first_req = true;
  bool aborted = false;

  while (!empty && !aborted && (r < end_r || (r == end_r && tile < end_tile))) {
    const int tb = tile;
    const int te = (r == end_r) ? end_tile : p.n_tiles;
    const int ns_r = p.num_splits[r], ns_r1 = p.num_splits[r + 1];
    const int slot = first_req ? m1.x : ns_r;
    const int nsplit = ns_r1 - ns_r;
    if (ns_r < 0 || ns_r1 > p.max_splits || nsplit < 1 || slot < ns_r || slot >= ns_r1) {
      if (tid == 0) report_status(p.status, kStatusBadSchedule);
      break;
    }
    const int b = r / p.s_q;
    const int seqlen = p.seqlens[b];
    const int32_t* bt = p.block_table + (size_t)b * p.max_blocks;
    const int32_t* idx_row = p.indices + (size_t)r * p.topk;

    // ---- Q tile: rows = heads of this group, zero rows past h_q ----------
    {
      const __nv_bfloat16* qsrc = p.q + ((size_t)r * p.h_q + (size_t)kHeads * hg) * 576;
      for (int i = tid; i < kHeads * 72; i += kThreads) {
        const int row = i / 72, ch = i % 72;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < heads_here) v = ldg_v4(qsrc + (size_t)row * 576 + ch * 8);
        st_shared_v4(aQ + (ch >> 3) * kAtom + swz(row, ch & 7), v);
      }
    }

    float m_run = -INFINITY, l_run = 0.f;   // base-2 running max and denominator

    for (int t = tb; t < te && !aborted; ++t) {
      // ---- indices -> cache row offsets -----------------------------------
      if (tid < kRows) {
        const int j = t * kRows + tid;
        const int idx = (j < p.topk) ? idx_row[j] : -1;
        int64_t off = -1;
        if (idx >= 0 && idx < seqlen) {
          const int blk = idx >> 6;
          if (blk < p.max_blocks) {
            const int64_t phys = bt[blk];
            if (phys >= 0 && phys < p.num_blocks) off = (phys * 64 + (idx & 63)) * 656;
            else report_status(p.status, kStatusBadBlockTable);
          } else {
            report_status(p.status, kStatusBadBlockTable);
          }
        }
        tail->row_off[tid] = off;
      }
      __syncthreads();

      // ---- gather + dequantise: warp w takes rows w, w+8, ...; lane = 16-byte chunk
      {
        uint4 raw[8];
        float sc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t off = tail->row_off[warp + 8 * i];
          raw[i] = make_uint4(0u, 0u, 0u, 0u);
          sc[i] = 0.f;
          if (off >= 0) {
            raw[i] = ldg_v4(p.kv + off + 16 * lane);
            sc[i] = __ldg(reinterpret_cast<const float*>(p.kv + off + 512) + (lane >> 3));
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = warp + 8 * i;
          uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
          if (tail->row_off[row] >= 0) dequant16(raw[i], sc[i], lo, hi);
          const uint32_t base = aK + (lane >> 2) * kAtom;
          st_shared_v4(base + swz(row, 2 * (lane & 3)), lo);
          st_shared_v4(base + swz(row, 2 * (lane & 3) + 1), hi);
        }
        // RoPE: 64 rows x 8 chunks of 16 bytes, copied into column block 8
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int c = tid + kThreads * k;
          const int row = c >> 3, ch = c & 7;
          const int64_t off = tail->row_off[row];
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (off >= 0) v = ldg_v4(p.kv + off + 528 + 16 * ch);
          st_shared_v4(aK + 8 * kAtom + swz(row, ch), v);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();

      // ---- S = Q K^T -----------------------------------------------------
      if (tid == 0) {
        tc_fence_after();
#pragma unroll 1
        for (int kk = 0; kk < 36; ++kk) {
          const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
          mma_bf16_ss(tmem + kSCol, smem_desc_sw128(aQ + koff, 16, 1024), smem_desc_sw128(aK + koff, 16, 1024),
                      idesc_s, kk > 0);
        }
        mma_commit(&tail->bar_s);
      }
      {
        const bool ok = mbar_wait_bounded(&tail->bar_s, phase_s, kWaitLimitNs, p.status);
        phase_s ^= 1;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
      }
      tc_fence_after();

      // ---- online softmax (warps 0-3) ------------------------------------
      if (softmax_warp) {
        uint32_t s_lo[32], s_hi[32];
        tmem_ld32(tmem + t_lane + kSCol, s_lo);
        tmem_ld32(tmem + t_lane + kSCol + 32, s_hi);
        tmem_wait_ld();
        uint32_t s_raw[64];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          s_raw[j] = s_lo[j];
          s_raw[32 + j] = s_hi[j];
        }
        float alpha = 1.f;
        if (lane < 16) {
          float mt = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            float s = __uint_as_float(s_raw[j]) * scale_log2;
            s = (tail->row_off[j] >= 0) ? s : -INFINITY;
            s_raw[j] = __float_as_uint(s);
            mt = fmaxf(mt, s);
          }
          const float m_new = fmaxf(m_run, mt);
          uint32_t pw[32];
          float psum = 0.f;
          if (m_new == -INFINITY) {
#pragma unroll
            for (int j = 0; j < 32; ++j) pw[j] = 0u;
          } else {
            alpha = exp2f(m_run - m_new);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float p0 = exp2f(__uint_as_float(s_raw[2 * j]) - m_new);
              const float p1 = exp2f(__uint_as_float(s_raw[2 * j + 1]) - m_new);
              __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
              const float2 pr = __bfloat1622float2(pb);
              psum += pr.x + pr.y;
              pw[j] = bf162_bits(pb);
            }
            m_run = m_new;
          }
          l_run = l_run * alpha + psum;
          // P row (64 bf16 = 8 chunks) -> K-major swizzled A operand
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(aP + swz(my_head, c), make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]));
        }
        // rescale the running output when the max moved (O exists after the first tile)
        alpha = __shfl_sync(0xffffffffu, alpha, lane & 15);
        const bool need = __any_sync(0xffffffffu, alpha != 1.f) && (t > tb);
        if (need) {
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + t_lane + kOCol + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st32(tmem + t_lane + kOCol + 32 * c, o);
          }
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();

      // ---- O += P V ------------------------------------------------------
      if (tid == 0) {
        tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a_desc = smem_desc_sw128(aP + ks * 32, 16, 1024);
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            const uint64_t b_desc = smem_desc_sw128(aK + (4 * hh) * kAtom + ks * 16 * 128, kAtom, 1024);
            mma_bf16_ss(tmem + kOCol + ((uint32_t)(16 * hh) << 16), a_desc, b_desc, idesc_pv,
                        (ks > 0 || t > tb) ? 1u : 0u);
          }
        }
        mma_commit(&tail->bar_o);
      }
      {
        const bool ok = mbar_wait_bounded(&tail->bar_o, phase_o, kWaitLimitNs, p.status);
        phase_o ^= 1;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
      }
      tc_fence_after();
    }
    if (aborted) break;

    // ---- epilogue: normalise and write (warps 0-3) ------------------------
    if (softmax_warp) {
      const float l_me = __shfl_sync(0xffffffffu, l_run, lane & 15);
      const float m_me = __shfl_sync(0xffffffffu, m_run, lane & 15);
      const int half = lane >> 4;
      const int head = kHeads * hg + my_head;
      const bool live = my_head < heads_here;
      const float inv_l = (l_me > 0.f) ? 1.f / l_me : 0.f;
      const float lse_val = (l_me > 0.f) ? (m_me + log2f(l_me)) * 0.69314718055994531f : -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(tmem + t_lane + kOCol + 32 * c, o);
        tmem_wait_ld();
        const int col = half * 256 + 32 * c;
        if (!live) {
        } else if (nsplit == 1) {
          __nv_bfloat16* dst = p.o + ((size_t)r * p.h_q + head) * 512 + col;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l));
            w.y = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l));
            w.z = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l));
            w.w = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
            reinterpret_cast<uint4*>(dst)[v] = w;
          }
        } else {
          float* dst = p.o_accum + ((size_t)slot * p.h_q + head) * 512 + col;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            reinterpret_cast<float4*>(dst)[v] =
                make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                            __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
      }
      if (live && lane < 16) {
        if (nsplit == 1) p.lse[(size_t)r * p.h_q + head] = lse_val;
        else p.lse_accum[(size_t)slot * p.h_q + head] = lse_val;
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    r += 1;
    tile = 0;
    first_req = false;
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int splitkv_smem_bytes() { return kSmemBytes; }

}  // namespace smla
