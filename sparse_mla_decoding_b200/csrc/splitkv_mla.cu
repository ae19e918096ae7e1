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
//             loads carry an evict-first L2 hint;
//     计算环节一 (Crossover) -- the 128 query heads of a token read the same
//             K/V, so two CTAs of a cluster each own 64 heads, each
//             dequantises half of the rows and writes them into both CTAs'
//             shared memory;
//     计算环节二 (Seesaw) -- the result is the FlashAttention online softmax;
//     合并与性能账本 -- each split leaves a partial output and its lse.
//   "deepseek-ai/FlashMLA" (agentlenshq), 技術的な詳細 -- -1 in indices marks
//     an entry the kernel ignores.
//
// Design on B200:
//   * A CTA owns 64 query heads of one request at a time (M = 64 of every
//     tcgen05.mma); 16/32 heads are zero-padded to 64 in a single CTA.  128
//     heads run, by default, as two independent CTAs per part (one per
//     64-head group, grid.y), each gathering and dequantising every row of
//     a tile; the second CTA's reads of a row mostly hit L2.  The optional
//     two-CTA cluster form shares the dequantised tiles over distributed
//     shared memory instead (each CTA dequantises half of the rows, and the
//     copy engine sends them to the peer with bulk shared-to-shared copies):
//     it halves the dequantisation per CTA but couples every tile of the two
//     CTAs, and measured slower on B200.
//   * Warp roles (416 threads, 13 warps, at most 128 registers a thread: one
//     SM sub-partition holds 4 of the 13 warps):
//       warps 0-3   softmax: online softmax over S in TMEM (two threads per
//                   head row, 32 score columns each), P to shared memory,
//                   lazy O rescaling, epilogue (own TMEM lane quarters 0-3);
//       warps 4-11  producers: index -> page map, 16-byte coalesced gathers
//                   of the 656-byte rows (evict-first), exact dequantisation
//                   into a double-buffered 64 x 576 bf16 K ring (128-byte
//                   swizzled, K-major; the same tile read MN-major is V), and
//                   each request's Q into TMEM;
//       warp 12     S issuer: waits for each K tile and issues its score
//                   MMAs (one elected lane issues each MMA and commit); the
//                   warp owns TMEM.
//   * MMAs: S = Q K^T with Q (the A operand) in TMEM and K in shared memory,
//     issued by warp 12 as soon as a tile is in shared memory, so the tensor
//     core computes the next scores while the softmax warps work on the
//     current ones; PV = P V with P and V in shared memory, issued by the
//     softmax warpgroup itself right after it has written P (no hand-off to
//     another warp on the per-tile critical path).
//   * The producers run a five-stage software pipeline across tiles
//     (dequantise tile t, row loads of t+1, L2 prefetch of the rows of t+2,
//     block table of t+3, indices of t+4), so the dependent loads index ->
//     block table -> row never stall a tile, the rows of t+1 are in flight
//     while the ring slot drains, and they come from L2 rather than DRAM.
//   * TMEM (512 columns; an M = 64 operand or accumulator uses 16 lanes of
//     each 32-lane sub-partition): lanes 0-15 hold Q (64 x 576 bf16, two
//     values a column, columns [0, 288)) and the S double buffer (columns
//     [320, 384) and [384, 448)); lanes 16-31 hold O = 64 x 512 fp32 in
//     columns [0, 256) and [256, 512).
//   * Shared memory: the K ring (2 x 72 KB) and a double-buffered P
//     (2 x 8 KB), about 161 KB.
//     Keeping Q out of it leaves the SM more L1 for the row gathers in
//     flight and halves the shared-memory reads of the S MMAs.
//   * Online softmax in base 2.  The running max used for P only moves when a
//     tile's max exceeds it by more than 2^8 (then O and l are rescaled), so
//     P <= 256 and rescales are rare; lse = (m + log2 l) ln 2 at the end.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstddef>
#include <cstdint>
#include <cstring>

#include "sm100.cuh"
#include "splitkv_mla.h"

namespace smla {

namespace {

constexpr int kRows = 64;              // index slots per tile
constexpr int kHeads = 64;             // heads per CTA (MMA M)
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 4 + kProducerWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);   // 4 softmax + 8 producer warps + 1 MMA warp = 416
// Warps are spread over the 4 SM sub-partitions by index, so one of them
// holds 4 of the 13 warps: registers are capped at 16384 / (4 x 32) = 128 per
// thread (the launch bound below asks for that cap).
constexpr int kRegCapThreads = 512;
constexpr int kKBlocks = 9;            // 576 / 64 bf16 per 128-byte swizzle line
constexpr int kAtom = kRows * 128;     // bytes of one 64-row x 128-byte column block
constexpr int kTileBytes = kKBlocks * kAtom;
constexpr int kPBytes = 2 * kAtom;   // P double buffer
static_assert(kAtom == 8192 && kKBlocks == 9, "the MMA blocks below encode 64-row column blocks as literal offsets");
static_assert(2 * kTileBytes + kPBytes < (1 << 18), "descriptor start fields are 14 bits of (address >> 4)");
// TMEM (512 columns x 128 lanes; an M = 64 operand or accumulator uses 16
// lanes of each 32-lane sub-partition):
//   lanes 0-15 of each quarter: Q (64 x 576 bf16, two values per column) in
//     columns [kQCol, kQCol + 288), S double buffer at kSCol + 64 s;
//   lanes 16-31: O (64 x 512 fp32), columns [0, 256) and [256, 512).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kQCol = 0;
constexpr uint32_t kSCol = 320;        // S buffer s at kSCol + 64 s, lanes 0-15
constexpr uint32_t kOLane = 16;        // O in lanes 16-31
static_assert(kQCol + 288 <= kSCol && kSCol + 128 <= kTmemCols, "TMEM column map");
constexpr float kRescaleLog2 = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: no legitimate wait comes close

struct __align__(16) Tail {
  // per K buffer: bit k of byte g = row 4g+k holds a valid slot (read as
  // 8-byte words, so it stays first in the 16-byte aligned struct)
  uint8_t vmask[2][16];
  uint64_t kfull[2];   // K tile s written (producers of both CTAs of a pair)
  uint64_t kempty[2];  // K tile s consumed by PV (both CTAs of a pair)
  uint64_t sfull[2];   // S buffer s computed
  uint64_t ofree[2];   // PV(j) complete, for tile j in ring slot j % 2
  uint64_t pready[2];  // the four softmax warps stored P(j), for tile j in ring slot j % 2
  uint64_t qfull;      // Q tile loaded
  uint64_t qfree;      // last S of a request complete: sQ reusable
  uint32_t tmem_base;
};
static_assert(offsetof(Tail, vmask) % 16 == 0 && offsetof(Tail, kfull) % 8 == 0, "Tail field alignment");

// The source of a skipped slot's row loads: zeros (a __device__ array is
// zero-initialised when the module loads and nothing writes it), so a
// skipped slot dequantises to a zero row without predicated loads or
// register clears.  Sized for the widest row format.
__device__ __align__(128) uint8_t g_zero_row[1152];

constexpr int kOffK = 0;
constexpr int kOffP = 2 * kTileBytes;
constexpr int kOffTail = kOffP + kPBytes;
constexpr int kSmemBytes = kOffTail + (int)sizeof(Tail) + 1024;

__device__ __forceinline__ uint32_t swz(int row, int chunk16) {
  return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// One S tile: 36 MMAs (9 column blocks x 4 K-steps of 16) of M = 64, N = 64,
// issued by one elected lane of a converged warp.  A = Q in TMEM (a K-step
// is 8 columns, a column block 32); B = the K tile in shared memory (a K-step
// adds 32 bytes = 2 descriptor units, a column block kAtom = 8192 bytes =
// 512).  Operands: D column, Q TMEM address, K descriptor lower half, the
// shared upper half, the instruction descriptor.
#define SMLA_S_STEP(kb, k4, acc)                                       \
  "add.u32 la, %1, (" #kb "*32+" #k4 "*8);\n\t"                        \
  "add.u32 lb, %2, (" #kb "*512+" #k4 "*2);\n\t"                       \
  "mov.b64 db, {lb, %3};\n\t"                                          \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [la], db, %4, " acc ";\n\t"
#define SMLA_S_BLOCK(kb) \
  SMLA_S_STEP(kb, 0, "pt") SMLA_S_STEP(kb, 1, "pt") SMLA_S_STEP(kb, 2, "pt") SMLA_S_STEP(kb, 3, "pt")

__device__ __forceinline__ void issue_s_tile(uint32_t d_tmem, uint32_t q_tmem, uint32_t k_lo, uint32_t hi,
                                             uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred e, pt, pf;\n\t.reg .b32 la, lb;\n\t.reg .b64 db;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 pt, 1, 0;\n\t"
      "setp.eq.b32 pf, 1, 0;\n\t"
      SMLA_S_STEP(0, 0, "pf") SMLA_S_STEP(0, 1, "pt") SMLA_S_STEP(0, 2, "pt") SMLA_S_STEP(0, 3, "pt")
      SMLA_S_BLOCK(1) SMLA_S_BLOCK(2) SMLA_S_BLOCK(3) SMLA_S_BLOCK(4)
      SMLA_S_BLOCK(5) SMLA_S_BLOCK(6) SMLA_S_BLOCK(7) SMLA_S_BLOCK(8)
      "}" ::"r"(d_tmem), "r"(q_tmem), "r"(k_lo), "r"(hi), "r"(idesc)
      : "memory");
}

// One PV step set: O[:, 256 hh + (0..255)] += P[:, 16 ks + (0..15)] V[16 ks + (0..15), ...]
// for ks = 0..3, hh = 0..1 (8 MMAs of M = 64, N = 256; V read MN-major from
// the K tile).  A K-step of P adds 32 bytes (2); of V 16 rows x 128 bytes
// (128); the second 256 columns of V start 4 column blocks later (2048).
#define SMLA_PV_STEP(ks, hh, acc)                                      \
  "add.u32 la, %2, (" #ks "*2);\n\t"                                   \
  "add.u32 lb, %3, (" #hh "*2048+" #ks "*128);\n\t"                    \
  "mov.b64 da, {la, %4};\n\t"                                          \
  "mov.b64 db, {lb, %4};\n\t"                                          \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%" #hh "], da, db, %5, " acc ";\n\t"

__device__ __forceinline__ void issue_pv_tile(uint32_t d_lo16, uint32_t d_hi16, uint32_t p_lo, uint32_t v_lo,
                                              uint32_t hi, uint32_t idesc, uint32_t accumulate_first) {
  asm volatile(
      "{\n\t.reg .pred e, pt, pa;\n\t.reg .b32 la, lb;\n\t.reg .b64 da, db;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 pt, 1, 0;\n\t"
      "setp.ne.b32 pa, %6, 0;\n\t"
      SMLA_PV_STEP(0, 0, "pa") SMLA_PV_STEP(0, 1, "pa")
      SMLA_PV_STEP(1, 0, "pt") SMLA_PV_STEP(1, 1, "pt")
      SMLA_PV_STEP(2, 0, "pt") SMLA_PV_STEP(2, 1, "pt")
      SMLA_PV_STEP(3, 0, "pt") SMLA_PV_STEP(3, 1, "pt")
      "}" ::"r"(d_lo16), "r"(d_hi16), "r"(p_lo), "r"(v_lo), "r"(hi), "r"(idesc), "r"(accumulate_first)
      : "memory");
}

// (a.x * b + c, a.y * b + c) in one packed instruction, each a fused
// multiply-add rounded exactly as fmaf.
__device__ __forceinline__ float2 ffma2_rn(float2 a, float b, float c) {
  uint64_t v, bb, cc, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %1};" : "=l"(bb) : "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(v), "l"(bb), "l"(cc));
  float2 out;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(out.x), "=f"(out.y) : "l"(r));
  return out;
}

// 2^x on the special-function unit (P is rounded to bf16 right after).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two round-to-nearest f32 products in one packed instruction (sm_100):
// (a.x * s, a.y * s), each rounded exactly as a scalar multiply.
__device__ __forceinline__ float2 fmul2_rn(float2 a, float s) {
  uint64_t v, sc, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %1};" : "=l"(sc) : "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(v), "l"(sc));
  float2 out;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(out.x), "=f"(out.y) : "l"(r));
  return out;
}

// 16 e4m3 values (one 16-byte chunk) -> 16 bf16 = bf16(float(e4m3) * scale):
// hardware e4m3x2 -> f16x2 converts (exact), f16 -> f32 (exact), a
// round-to-nearest f32 multiply (two per instruction), then
// round-to-nearest-even to bf16.
__device__ __forceinline__ void dequant16(const uint4& raw, float scale, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t out[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] & 0xFFFFu), __NV_E4M3);
    __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] >> 16), __NV_E4M3);
    const float2 p01 = fmul2_rn(__half22float2(*reinterpret_cast<__half2*>(&h01)), scale);
    const float2 p23 = fmul2_rn(__half22float2(*reinterpret_cast<__half2*>(&h23)), scale);
    out[2 * j] = bf162_bits(__floats2bfloat162_rn(p01.x, p01.y));
    out[2 * j + 1] = bf162_bits(__floats2bfloat162_rn(p23.x, p23.y));
  }
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Store `sel ? a : b` at addr: two predicated stores (each lane executes one)
// instead of selecting 4 registers of data.
__device__ __forceinline__ void st_shared_v4_sel(uint32_t addr, bool sel, const uint4& a, const uint4& b) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %1, 0;\n\t"
      "@p st.shared.v4.u32 [%0], {%2, %3, %4, %5};\n\t"
      "@!p st.shared.v4.u32 [%0], {%6, %7, %8, %9};\n\t}" ::"r"(addr),
      "r"((uint32_t)sel), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
      : "memory");
}

__device__ __forceinline__ void st_shared_u8(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_u8(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_shared_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}


// Eight bytes, each holding 4 bits in its low nibble -> 32 packed bits.
__device__ __forceinline__ uint32_t nibbles_to_bits(uint64_t x) {
  x = (x | (x >> 4)) & 0x00FF00FF00FF00FFull;
  x = (x | (x >> 8)) & 0x0000FFFF0000FFFFull;
  x = (x | (x >> 16)) & 0x00000000FFFFFFFFull;
  return (uint32_t)x;
}

// Walks a part's (request, tile) range one tile at a time, without any
// division in the loop.
// Tiles of request r: the fixed count n_tiles, or (dense decode) the
// difference of the tile prefix, at least 1 (a table that says otherwise is
// not from the metadata kernel; clamping keeps every walk finite).
__device__ __forceinline__ int tiles_of(const SplitKVParams& p, int r) {
  if (p.tile_prefix == nullptr) return p.n_tiles;
  const int n = __ldg(p.tile_prefix + r + 1) - __ldg(p.tile_prefix + r);
  return n > 0 ? n : 1;
}

// Tiles before request r in the part's (request, tile) order.
__device__ __forceinline__ int64_t tile_start(const SplitKVParams& p, int r) {
  return p.tile_prefix == nullptr ? (int64_t)r * p.n_tiles : (int64_t)__ldg(p.tile_prefix + r);
}

struct Cursor {
  int r, t, n;   // request, tile within it, tiles of the request
  __device__ __forceinline__ void advance(const SplitKVParams& p) {
    if (++t == n) {
      t = 0;
      ++r;
      if (p.tile_prefix != nullptr && r < p.num_requests) n = tiles_of(p, r);
    }
  }
};

// The same walk that also tracks the batch entry b = r / s_q of the request
// (b and q = r % s_q advance with r, so the loop needs no division).
struct BatchCursor {
  int r, t, n, b, q;
  __device__ __forceinline__ void advance(const SplitKVParams& p) {
    if (++t == n) {
      t = 0;
      ++r;
      if (p.tile_prefix != nullptr && r < p.num_requests) n = tiles_of(p, r);
      if (++q == p.s_q) {
        q = 0;
        ++b;
      }
    }
  }
};

}  // namespace

template <bool kPair, int kMode>
__global__ void __launch_bounds__(kRegCapThreads, 1) splitkv_mla_kernel(const SplitKVParams p) {
  constexpr bool kDense = kMode != kSparseFp8;
  constexpr bool kBf16 = kMode == kDenseBf16;
  constexpr int kRowBytes = kBf16 ? 1152 : 656;     // one cache row
  constexpr int kRopeOff = kBf16 ? 1024 : 528;      // byte offset of its 64 bf16 RoPE values
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Tail* tail = reinterpret_cast<Tail*>(smem + kOffTail);
  const uint32_t aK0 = smem_u32(smem + kOffK);
  const uint32_t aP = smem_u32(smem + kOffP);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int part = blockIdx.x;
  const uint32_t crank = kPair ? cluster_ctarank() : 0u;
  const int hg = kPair ? (int)crank : (int)blockIdx.y;      // head group: heads [64*hg, 64*hg + 64)
  const int heads_here = min(kHeads, p.h_q - kHeads * hg);
  const uint32_t peer = crank ^ 1u;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tail->kfull[s], kPair ? 2 * kProducerWarps : kProducerWarps);
      mbar_init(&tail->kempty[s], kPair ? 2 : 1);
      mbar_init(&tail->sfull[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tail->ofree[s], 1);
      mbar_init(&tail->pready[s], 4);
    }
    mbar_init(&tail->qfull, 32 * kProducerWarps);
    mbar_init(&tail->qfree, 1);
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tail->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();       // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  // The schedule is written by the metadata kernel that precedes us.
  pdl_wait_primary();
  // Let the combine kernel launch now: its CTAs take whatever room is left
  // on the SMs (or that finished parts free) and wait in griddepcontrol.wait,
  // which returns only once this whole grid has completed, so the merge
  // starts without a launch gap.
  pdl_launch_dependents();
  const int4 m0 = *reinterpret_cast<const int4*>(p.sched_meta + (size_t)part * 8);
  const int4 m1 = *reinterpret_cast<const int4*>(p.sched_meta + (size_t)part * 8 + 4);
  // Metadata comes from the caller: check it against this call's shapes so a
  // mismatched table cannot send reads or writes out of bounds.
  bool empty = m1.y != 0;
  int n0 = 1;   // tiles of the part's first request
  if (!empty) {
    const int R = p.num_requests;
    bool ok = m0.x >= 0 && m0.x < R && m0.y >= 0 && m0.z >= m0.x && m0.z <= R && m0.w >= 0;
    if (ok) {
      n0 = tiles_of(p, m0.x);
      ok = m0.y < n0 && (m0.z < R ? m0.w < tiles_of(p, m0.z) : m0.w == 0) && (m0.z > m0.x || m0.w > m0.y);
    }
    if (!ok) {
      if (tid == 0) report_status(p.status, kStatusBadSchedule);
      empty = true;
    }
  }
  const int64_t g0 = empty ? 0 : tile_start(p, m0.x) + m0.y;
  const int64_t g1 = empty ? 0 : tile_start(p, m0.z) + m0.w;
  const int64_t ntile = g1 > g0 ? g1 - g0 : 0;

  if (warp >= 4 && warp < 4 + kProducerWarps) {
    // ======================= producers =====================================
    // Warp pw owns kRPW consecutive rows of every tile: 8 in the single-CTA
    // form, 4 in the two-CTA form (where a CTA dequantises 32 of the 64 rows
    // and sends them to its peer).  Tiles are software-pipelined over five
    // stages per iteration, in this order: dequantise tile t, load the rows
    // of tile t+1, prefetch the rows of tile t+2 into L2, load the
    // block-table entries of tile t+3 and the indices of tile t+4.  Each
    // stage reads what the next one produced an iteration earlier, before
    // that register is reloaded, so no load is waited on early; the rows of
    // tile t+1 are in flight while the warp waits for the next ring slot,
    // and the prefetch an iteration earlier has brought them from DRAM into
    // L2.  The loop body is kept small (one copy of each stage): the roles
    // share the SM's instruction caches.
    constexpr int kRPW = kPair ? 4 : 8;
    const int pw = warp - 4;
    const uint64_t pol = l2_evict_first_policy();
    const int rb = kPair ? (32 * (int)crank + kRPW * pw) : kRPW * pw;   // this warp's first row of a tile
    // Stores: lane l writes the two 16-byte halves of its 32-byte output in
    // an order that puts the 8 lanes of a quarter-warp on 8 distinct bank
    // groups (lanes with bit 2 set start with the upper half).
    const int kb = lane >> 2;
    const int swap = (lane >> 2) & 1;
    const int c_first = 2 * (lane & 3) + swap;
    const int c_second = 2 * (lane & 3) + 1 - swap;
    // tiles t+4 (indices), t+3 (block table), t (fill)
    BatchCursor ca{m0.x, m0.y, n0, m0.x / p.s_q, m0.x % p.s_q}, cb = ca;
    Cursor cf{m0.x, m0.y, n0};

    int idx = -1, sl = 0;        // index and request length of lane k's slot (lanes 0..kRPW-1)
    int sl_hidden = 0;           // dense causal decode: the request's last positions this token cannot see
    int phys = -1, off = 0;      // its cache block (-1: skip) and row within the block
    bool looked_up = false;      // lane k's slot is valid and its block-table entry was read
    int row_n = -1;              // cache row of lane k's slot in the tile being prefetched
    int row_c = -1;              // cache row of lane k's slot in the tile being dequantised
    uint4 lat[kRPW], rp[kRPW / 4];
    uint4 lat2[kBf16 ? kRPW : 1];  // BF16 rows: the second 16 bytes of each lane's 32
    float sc[kRPW];
#pragma unroll
    for (int k = 0; k < kRPW; ++k) {
      lat[k] = make_uint4(0u, 0u, 0u, 0u);
      sc[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < (kBf16 ? kRPW : 1); ++k) lat2[k] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kRPW / 4; ++i) rp[i] = make_uint4(0u, 0u, 0u, 0u);

    int req_ord = -1;
    bool ok = true;
#pragma unroll 1
    for (int64_t R = -4; R < ntile && ok; ++R) {
      // ---- dequantise and store tile R -------------------------------------
      if (R >= 0) {
        const int64_t j = R;
        const bool tile_first = (j == 0) || (cf.t == 0);
        const int s = (int)(j & 1);
        const uint32_t aK = aK0 + (uint32_t)s * kTileBytes;
        const uint32_t aKr = kPair ? mapa_shared(aK, peer) : 0u;      // the peer's copy of this slot
        if (tile_first) {
          ++req_ord;
          if (req_ord > 0 &&
              !mbar_wait_bounded_warp(&tail->qfree, (uint32_t)((req_ord - 1) & 1), kWaitLimitNs, p.status)) {
            ok = false;
            break;
          }
          // Q of this request into TMEM (lanes 0-15 of this warp's quarter):
          // thread i holds head 16 (warp % 4) + i % 16 and, per 32-column chunk
          // c, the 32 values [64 c + 32 (i / 16), +32) packed two to a column.
          // The two producer warps of a quarter take chunks 0-4 and 5-8.
          {
            const int qh = 16 * (warp & 3) + (lane & 15);
            const bool qlive = qh < heads_here;
            const __nv_bfloat16* qrow = p.q + ((size_t)cf.r * p.h_q + (size_t)kHeads * hg + (qlive ? qh : 0)) * 576;
            const uint32_t qaddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kQCol;
            const int c0 = (pw < 4) ? 0 : 5, c1 = (pw < 4) ? 5 : 9;
            // each chunk in two halves of 8 columns (the two 16-thread halves of
            // the warp write 16 columns apart); the loads of kQB halves are in
            // flight together, few enough registers to stay live beside the
            // pipeline's row data (BF16 rows hold twice the row data)
            constexpr int kQB = kBf16 ? 1 : 2;
#pragma unroll 1
            for (int h = 2 * c0; h < 2 * c1; h += kQB) {
              uint32_t v[kQB][8];
#pragma unroll
              for (int g = 0; g < kQB; ++g) {
                const int c = (h + g) >> 1, u0 = 2 * ((h + g) & 1);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                  uint4 x = make_uint4(0u, 0u, 0u, 0u);
                  ldg_v4_if(x, qrow + 64 * c + 32 * (lane >> 4) + 8 * (u0 + u), qlive);
                  v[g][4 * u] = x.x;
                  v[g][4 * u + 1] = x.y;
                  v[g][4 * u + 2] = x.z;
                  v[g][4 * u + 3] = x.w;
                }
              }
#pragma unroll
              for (int g = 0; g < kQB; ++g) {
                const int c = (h + g) >> 1, u0 = 2 * ((h + g) & 1);
                tmem_st16x2_8<16>(qaddr + 32 * c + 4 * u0, v[g]);
              }
            }
            // The next request's rows of Q into L2 now, so its staging (on the
            // pipeline's critical path: S waits for it) reads L2, not DRAM.
            // (Not with BF16 rows: their row data leaves no registers for it.)
            if (!kBf16 && cf.r + 1 < p.num_requests) {
              const char* qn = reinterpret_cast<const char*>(p.q + ((size_t)(cf.r + 1) * p.h_q + (size_t)kHeads * hg) * 576);
              const int nlines = heads_here * 576 * 2 / 128;
#pragma unroll 1
              for (int i = 32 * pw + lane; i < nlines; i += 32 * kProducerWarps) prefetch_l2_if(qn + 128 * i, true);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&tail->qfull);
        }
        // the ring slot is free once PV of tile j-2 finished in every CTA of the cluster
        if (!mbar_wait_bounded_warp(&tail->kempty[s], (uint32_t)(((j >> 1) & 1) ^ 1), kWaitLimitNs, p.status)) {
          ok = false;
          break;
        }
        const uint32_t vbits = __ballot_sync(0xffffffffu, row_c >= 0) & ((1u << kRPW) - 1u);
        // A skipped slot's registers were loaded from the zero row, so
        // dequantising (or copying) it unconditionally stores a zero row.  FP8 rows: lanes that store their upper half first swap the
        // two 8-byte halves of the input instead of the two 16-byte halves of
        // the output.  BF16 rows are stored as they are.
#pragma unroll
        for (int k = 0; k < kRPW; ++k) {
          const int row = rb + k;
          if constexpr (kBf16) {
            st_shared_v4_sel(aK + kb * kAtom + swz(row, c_first), swap, lat2[k], lat[k]);
            st_shared_v4_sel(aK + kb * kAtom + swz(row, c_second), swap, lat[k], lat2[k]);
          } else {
            const uint4 in = swap ? make_uint4(lat[k].z, lat[k].w, lat[k].x, lat[k].y) : lat[k];
            uint4 first, second;
            dequant16(in, sc[k], first, second);
            st_shared_v4(aK + kb * kAtom + swz(row, c_first), first);
            st_shared_v4(aK + kb * kAtom + swz(row, c_second), second);
          }
        }
#pragma unroll
        for (int i = 0; i < kRPW / 4; ++i) st_shared_v4(aK + 8 * kAtom + swz(rb + 4 * i + (lane >> 3), lane & 7), rp[i]);
        // validity: one byte per 4-row group, bit k = row 4g+k
        if (lane < kRPW / 4) {
          const uint32_t va = smem_u32(&tail->vmask[s][(rb >> 2) + lane]);
          const uint32_t nib = (vbits >> (4 * lane)) & 0xFu;
          st_shared_u8(va, nib);
          if (kPair) st_cluster_u8(mapa_shared(va, peer), nib);
        }
        cf.advance(p);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->kfull[s]);
        if (kPair) {
          // The copy engine sends this warp's rows (kRPW x 128 bytes in each
          // of the 9 column blocks, same offsets) to the peer's slot; the
          // peer's kfull counts the arrive and the completed bytes.
          const uint32_t rbar = mapa_shared(smem_u32(&tail->kfull[s]), peer);
          if (lane == 0) mbar_arrive_expect_tx_cluster(rbar, kKBlocks * kRPW * 128);
          if (lane < kKBlocks) {
            const uint32_t off = (uint32_t)(lane * kAtom + rb * 128);
            bulk_copy_to_peer(aKr + off, aK + off, kRPW * 128, rbar);
          }
        }
      }
      // ---- row loads of tile R+1 -------------------------------------------
      if (R + 1 >= 0 && R + 1 < ntile) {
        row_c = row_n;
        // For every row, lane l takes latent bytes [16l, 16l+16) and the scale
        // of its 128-value tile; the RoPE chunks (8 per row) are spread over
        // the lanes (row 4i + l/8, chunk l%8).  A skipped slot reads the zero
        // row instead.
#pragma unroll
        for (int k = 0; k < kRPW; ++k) {
          const int rk = __shfl_sync(0xffffffffu, row_c, k);
          const uint8_t* row = rk >= 0 ? p.kv + (int64_t)rk * kRowBytes : g_zero_row;
          if constexpr (kBf16) {
            // lane l: latent values [16 l, 16 l + 16) = bytes [32 l, 32 l + 32)
            ldg_v4_evict_first(lat[k], row + 32 * lane, pol);
            ldg_v4_evict_first(lat2[k], row + 32 * lane + 16, pol);
          } else {
            ldg_v4_evict_first(lat[k], row + 16 * lane, pol);
            ldg_f32_evict_first(sc[k], row + 512 + 4 * (lane >> 3), pol);
          }
        }
#pragma unroll
        for (int i = 0; i < kRPW / 4; ++i) {
          const int rk = __shfl_sync(0xffffffffu, row_c, 4 * i + (lane >> 3));
          const uint8_t* row = rk >= 0 ? p.kv + (int64_t)rk * kRowBytes : g_zero_row;
          ldg_v4_evict_first(rp[i], row + kRopeOff + 16 * (lane & 7), pol);
        }
      }
      // ---- L2 prefetch of the rows of tile R+2 --------------------------------
      if (R + 2 >= 0 && R + 2 < ntile) {
        // A valid slot whose block-table entry lies outside the cache
        // (negative or past num_blocks) is skipped and flagged.
        row_n = -1;
        if (phys >= 0 && phys < p.num_blocks) row_n = phys * 64 + off;
        else if (looked_up) report_status(p.status, kStatusBadBlockTable);
        // (row, line) pairs over the lanes: each row's 128-byte lines at
        // offsets 0, 128, ... and its last byte (a row may straddle one more)
        constexpr int kLines = (kRowBytes + 127) / 128 + 1;
#pragma unroll 1
        for (int e0 = 0; e0 < kRPW * kLines; e0 += 32) {
          const int e = e0 + lane;
          const int k = min(e / kLines, kRPW - 1);
          const int rk = __shfl_sync(0xffffffffu, row_n, k);
          const int li = e - k * kLines;
          prefetch_l2_if(p.kv + (int64_t)max(rk, 0) * kRowBytes + min(128 * li, kRowBytes - 1),
                         rk >= 0 && e < kRPW * kLines);
        }
      }
      // ---- block-table entry of tile R+3 -----------------------------------
      if (R + 3 >= 0 && R + 3 < ntile) {
        const bool valid = lane < kRPW && idx >= 0 && idx + sl_hidden < sl;
        const int blk = idx >> 6;
        if (valid && blk >= p.max_blocks) report_status(p.status, kStatusBadBlockTable);
        off = idx & 63;
        phys = -1;
        looked_up = valid && blk < p.max_blocks;
        ldg_s32_if(phys, p.block_table + (size_t)cb.b * p.max_blocks + blk, looked_up);
        cb.advance(p);
      }
      // ---- index and request length of tile R+4 ---------------------------
      if (R + 4 < ntile) {
        const int slot = ca.t * kRows + rb + lane;
        idx = -1;
        sl = 0;
        if constexpr (kDense) {
          // every position of the request, in order; the causal mask hides
          // the last s_q - 1 - t of them from token t
          if (lane < kRPW) idx = slot;
          sl_hidden = p.causal ? p.s_q - 1 - ca.q : 0;
        } else {
          ldg_s32_if(idx, p.indices + (size_t)ca.r * p.topk + slot, lane < kRPW && slot < p.topk);
        }
        ldg_s32_if(sl, p.seqlens + ca.b, lane < kRPW);
        ca.advance(p);
      }
    }
    // Every arrive aimed at this CTA's ring barriers (the peer's multicast
    // commits included) has landed before the CTA may exit: wait for the last
    // completion of each ring slot that was used.
    if (lane == 0) {
      for (int64_t j = ntile; j < ntile + 2; ++j) {
        if (j - 2 < 0) continue;
        (void)mbar_wait_bounded(&tail->kempty[j & 1], (uint32_t)(((j >> 1) & 1) ^ 1), kWaitLimitNs, p.status);
      }
    }
  } else if (warp == kMmaWarp) {
    // ======================= S issuer ======================================
    // The whole warp runs this loop (so the descriptor arithmetic is
    // warp-uniform); one elected lane issues each tcgen05 instruction.  S(j)
    // goes to TMEM buffer j % 2 as soon as K tile j is in shared memory: the
    // softmax warps read S(j - 2) from that buffer before they issued PV(j - 2),
    // and the producers refilled the ring slot of tile j only after PV(j - 2)
    // completed, so the buffer is free.
    const uint32_t idesc_s = idesc_bf16_f32(kHeads, kRows, false);
    const uint32_t k_lo0 = smem_desc_lo(aK0, 16);     // K-major: leading offset 16 bytes
    const uint32_t d_hi = smem_desc_hi_sw128(1024);
    int req_ord = -1;
    Cursor cm{m0.x, m0.y, n0};
#pragma unroll 1
    for (int64_t j = 0; j < ntile; ++j, cm.advance(p)) {
      const bool t_first = (j == 0) || (cm.t == 0);
      const bool t_last = (j == ntile - 1) || (cm.t == cm.n - 1);
      const int s = (int)(j & 1);
      if (t_first) {
        ++req_ord;
        if (!mbar_wait_bounded_warp(&tail->qfull, (uint32_t)(req_ord & 1), kWaitLimitNs, p.status)) break;
      }
      if (!mbar_spin_bounded_warp(&tail->kfull[s], (uint32_t)((j >> 1) & 1), kWaitLimitNs, p.status)) break;
      tc_fence_after();
      issue_s_tile(tmem + kSCol + 64 * s, tmem + kQCol, k_lo0 + (uint32_t)s * (kTileBytes >> 4), d_hi, idesc_s);
      if (t_last) mma_commit(&tail->qfree);
      mma_commit(&tail->sfull[s]);
    }
    // the last request's qfree arrive lands before the CTA may exit
    if (ntile > 0) (void)mbar_wait_bounded_warp(&tail->qfree, (uint32_t)(req_ord & 1), kWaitLimitNs, p.status);
  } else {
    // ======================= softmax / epilogue (warps 0-3) =================
    // Thread i of softmax warp w owns score row (head) 16 w + i % 16, columns
    // [32 (i / 16), 32 (i / 16) + 32) of each tile (the 16x32bx2 TMEM shape);
    // the two threads of a row combine their max and sum with one shuffle.
    // P(j) goes to shared-memory buffer j % 2, which PV(j - 2) read: that MMA
    // completed before the producers refilled the ring slot S(j) was computed
    // from, so only an O rescale waits for the previous PV.  Once the four
    // warps have stored P (named barrier), warp 0 issues PV(j) and commits
    // the ring slot and the O accumulator.  The rendezvous is an mbarrier
    // that only warp 0 waits on, with the usual time bound, so a warp that
    // gives up cannot leave the others blocked.  TMEM lane i of the O accumulator
    // holds the same head (its upper lanes hold the second 256 columns), so
    // the rescale factor is already in the right thread.
    const int my_head = 16 * warp + (lane & 15);
    const int half = lane >> 4;
    const uint32_t t_lane = (uint32_t)(32 * warp) << 16;
    const float scale_log2 = p.scale_log2;
    const uint32_t idesc_pv = idesc_bf16_f32(kHeads, 256, true);
    const uint32_t p_lo0 = smem_desc_lo(aP, 16);        // P K-major: leading offset 16 bytes
    const uint32_t v_lo0 = smem_desc_lo(aK0, kAtom);    // V read MN-major: leading offset one column block
    const uint32_t d_hi = smem_desc_hi_sw128(1024);
    float m_used = -INFINITY, l_half = 0.f;
    int req_ord = -1;
    int slot = 0, nsplit = 1;
    bool req_ok = true;
    Cursor cx{m0.x, m0.y, n0};
#pragma unroll 1
    for (int64_t j = 0; j < ntile; ++j, cx.advance(p)) {
      struct {
        int r;
        bool first, last;
      } tp{cx.r, (j == 0) || (cx.t == 0), (j == ntile - 1) || (cx.t == cx.n - 1)};
      const int s = (int)(j & 1);
      const uint32_t ph = (uint32_t)((j >> 1) & 1);
      if (tp.first) {
        ++req_ord;
        m_used = -INFINITY;
        l_half = 0.f;
        const int ns_r = p.num_splits[tp.r], ns_r1 = p.num_splits[tp.r + 1];
        slot = (req_ord == 0) ? m1.x : ns_r;
        nsplit = ns_r1 - ns_r;
        req_ok = !(ns_r < 0 || ns_r1 > p.max_splits || nsplit < 1 || slot < ns_r || slot >= ns_r1);
        if (!req_ok && tid == 0) report_status(p.status, kStatusBadSchedule);
      }
      // The tile's validity bytes are published with kfull, which completes
      // before S(j) is even issued: wait for it first, while S executes.
      if (!mbar_wait_bounded_warp(&tail->kfull[s], ph, kWaitLimitNs, p.status)) break;
      if (!mbar_wait_bounded_warp(&tail->sfull[s], ph, kWaitLimitNs, p.status)) break;
      tc_fence_after();
      // validity bits of this thread's 32 columns (one nibble per 4 rows)
      const uint32_t vh = nibbles_to_bits(ld_shared_u64(smem_u32(&tail->vmask[s][8 * half])));
      uint32_t sr[32];
      tmem_ld16x2_32(tmem + t_lane + kSCol + 64 * s, sr);
      tmem_wait_ld();
      // Tiles whose 64 slots are all valid (the usual case) skip the
      // per-column mask tests; the results are the same either way.
      const bool all_valid = __all_sync(0xffffffffu, vh == 0xFFFFFFFFu);
      float mt = -INFINITY;
      if (all_valid) {
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          mx[c] = fmaxf(fmaxf(__uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1])),
                        fmaxf(__uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3])));
        mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if ((vh >> c) & 1u) mt = fmaxf(mt, __uint_as_float(sr[c]));
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      float alpha = 1.f;
      mt = (mt == -INFINITY) ? -INFINITY : mt * scale_log2;
      if (mt > m_used + kRescaleLog2) {
        alpha = fast_exp2(m_used - mt);     // 0 when nothing was valid before
        l_half *= alpha;
        m_used = mt;
      }
      // P = 2^(s * scale_log2 - m) for valid slots (0 otherwise), rounded to bf16
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      float psum = 0.f;
      uint32_t pk[16];
      if (all_valid) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 t = ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale_log2,
                                    neg_m);
          const float p0 = fast_exp2(t.x), p1 = fast_exp2(t.y);
          psum += p0 + p1;
          pk[c] = bf162_bits(__floats2bfloat162_rn(p0, p1));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 =
              ((vh >> (2 * c)) & 1u) ? fast_exp2(fmaf(__uint_as_float(sr[2 * c]), scale_log2, neg_m)) : 0.f;
          const float p1 =
              ((vh >> (2 * c + 1)) & 1u) ? fast_exp2(fmaf(__uint_as_float(sr[2 * c + 1]), scale_log2, neg_m)) : 0.f;
          psum += p0 + p1;
          pk[c] = bf162_bits(__floats2bfloat162_rn(p0, p1));
        }
      }
      if (m_used != -INFINITY) l_half += psum;
      // An O rescale needs PV(j - 1) complete.  The PV barriers are per ring
      // slot, which makes every such wait unambiguous: a warp that sees S(j)
      // knows PV(j - 2) completed (its ring slot was refilled for tile j), so
      // ofree[slot of j - 1] is at most one phase short of PV(j - 1).  (With
      // one barrier for all tiles a warp running ahead could match the parity
      // of a phase two PVs old.)
      if (!tp.first && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!mbar_wait_bounded_warp(&tail->ofree[s ^ 1], (uint32_t)(((j - 1) >> 1) & 1), kWaitLimitNs, p.status))
          break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld16x2_32(tmem + t_lane + (kOLane << 16) + 64 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st16x2_32(tmem + t_lane + (kOLane << 16) + 64 * c, o);
        }
        tmem_wait_st();
      }
      const uint32_t aPs = aP + (uint32_t)s * kAtom;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        st_shared_v4(aPs + swz(my_head, 4 * half + c), make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->pready[s]);
      if (warp == 0) {
        if (!mbar_spin_bounded_warp(&tail->pready[s], (uint32_t)((j >> 1) & 1), kWaitLimitNs, p.status)) break;
        tc_fence_after();
        issue_pv_tile(tmem + (kOLane << 16), tmem + (kOLane << 16) + 256, p_lo0 + (uint32_t)s * (kAtom >> 4),
                      v_lo0 + (uint32_t)s * (kTileBytes >> 4), d_hi, idesc_pv, tp.first ? 0u : 1u);
        if (kPair) mma_commit_multicast(&tail->kempty[s], (uint16_t)0x3);
        else mma_commit(&tail->kempty[s]);
        mma_commit(&tail->ofree[s]);
      }

      if (tp.last) {
        if (!mbar_wait_bounded_warp(&tail->ofree[s], (uint32_t)((j >> 1) & 1), kWaitLimitNs, p.status)) break;
        tc_fence_after();
        const float l_me = l_half + __shfl_xor_sync(0xffffffffu, l_half, 16);
        const float m_me = m_used;
        const int head = kHeads * hg + my_head;
        const bool live = req_ok && (my_head < heads_here);
        const float inv_l = (l_me > 0.f) ? 1.f / l_me : 0.f;
        const float lse_val = (l_me > 0.f) ? (m_me + log2f(l_me)) * 0.69314718055994531f : -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          __syncwarp();
          tmem_ld16x2_32(tmem + t_lane + (kOLane << 16) + 64 * c, o);
          tmem_wait_ld();
          const int col = 64 * c + 32 * half;
          if (!live) {
          } else if (nsplit == 1) {
            __nv_bfloat16* dst = p.o + ((size_t)tp.r * p.h_q + head) * 512 + col;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 0]) * inv_l,
                                                     __uint_as_float(o[8 * v + 1]) * inv_l));
              w.y = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 2]) * inv_l,
                                                     __uint_as_float(o[8 * v + 3]) * inv_l));
              w.z = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 4]) * inv_l,
                                                     __uint_as_float(o[8 * v + 5]) * inv_l));
              w.w = bf162_bits(__floats2bfloat162_rn(__uint_as_float(o[8 * v + 6]) * inv_l,
                                                     __uint_as_float(o[8 * v + 7]) * inv_l));
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
          if (nsplit == 1) p.lse[(size_t)tp.r * p.h_q + head] = lse_val;
          else p.lse_accum[(size_t)slot * p.h_q + head] = lse_val;
        }
        // The next request's first PV (issued by warp 0 after the next named
        // barrier) overwrites O only after every warp's reads above.
        tc_fence_before();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int splitkv_smem_bytes() { return kSmemBytes; }

// Host launcher shared by the entry points: picks the single-CTA or the
// two-CTA cluster form and the key source, and chains the launch to the
// previous kernel of the stream with programmatic dependent launch.
template <bool kPair>
static cudaError_t launch_form(const cudaLaunchConfig_t& cfg, const SplitKVParams& p) {
  switch (p.kv_mode) {
    case kSparseFp8: return cudaLaunchKernelEx(&cfg, splitkv_mla_kernel<kPair, kSparseFp8>, p);
    case kDenseFp8: return cudaLaunchKernelEx(&cfg, splitkv_mla_kernel<kPair, kDenseFp8>, p);
    case kDenseBf16: return cudaLaunchKernelEx(&cfg, splitkv_mla_kernel<kPair, kDenseBf16>, p);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_splitkv(const SplitKVParams& p, cudaStream_t stream) {
  const bool pair = p.h_q > kHeads && p.cta_pairs != 0;
  cudaLaunchAttribute attrs[2];
  std::memset(attrs, 0, sizeof(attrs));
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;
  attrs[1].val.clusterDim.x = 1;
  attrs[1].val.clusterDim.y = 2;
  attrs[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(p.num_parts, pair ? 2 : (p.h_q + kHeads - 1) / kHeads);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attrs;
  cfg.numAttrs = pair ? 2 : 1;
  return pair ? launch_form<true>(cfg, p) : launch_form<false>(cfg, p);
}

template <bool kPair, int kMode>
static cudaError_t set_smem() {
  return cudaFuncSetAttribute(splitkv_mla_kernel<kPair, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSmemBytes);
}

cudaError_t configure_splitkv() {
  const cudaError_t e[6] = {set_smem<true, kSparseFp8>(), set_smem<false, kSparseFp8>(),
                            set_smem<true, kDenseFp8>(),  set_smem<false, kDenseFp8>(),
                            set_smem<true, kDenseBf16>(), set_smem<false, kDenseBf16>()};
  for (cudaError_t x : e)
    if (x != cudaSuccess) return x;
  return cudaSuccess;
}

}  // namespace smla
