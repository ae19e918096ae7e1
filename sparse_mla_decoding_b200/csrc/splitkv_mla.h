// splitkv_mla.h -- internal interface between the decode entry points and the
// split-KV sparse MLA decode kernels (device parameters, launchers and the
// host-side pieces every decode entry point shares).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace smla {

// What the split kernel reads for a request's keys.
enum KvMode : int {
  kSparseFp8 = 0,   // the indices tensor names the tokens; 656-byte FP8 rows
  kDenseFp8 = 1,    // every visible token (indices made in the kernel); 656-byte FP8 rows
  kDenseBf16 = 2,   // every visible token; 1152-byte BF16 rows (576 bf16 values)
};

struct SplitKVParams {
  const __nv_bfloat16* q;       // [R][h_q][576], R = batch * s_q
  const uint8_t* kv;            // [num_blocks][64][row bytes]
  int64_t num_blocks;
  const int32_t* block_table;   // [batch][max_blocks]
  int max_blocks;
  const int32_t* seqlens;       // [batch]
  const int32_t* indices;       // [R][topk] (sparse mode)
  const int32_t* tile_prefix;   // [R + 1] tiles before each request (dense modes), or nullptr
  int kv_mode;                  // KvMode
  int cta_pairs;                // 128 heads: 1 = two-CTA cluster sharing dequantised tiles, 0 = independent CTAs
  int causal;                   // dense modes: token t of s_q sees seqlen - (s_q - 1 - t) positions
  const int32_t* sched_meta;    // [num_parts][8]
  const int32_t* num_splits;    // [R + 1]
  int s_q, h_q, topk, n_tiles, num_parts;   // n_tiles: tiles per request when tile_prefix is nullptr
  int num_requests;             // R = batch * s_q
  int max_splits;               // split slots the workspace holds (R + num_parts)
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* o;             // [R][h_q][512]
  float* lse;                   // [R][h_q]
  float* o_accum;               // [splits][h_q][512]
  float* lse_accum;             // [splits][h_q]
  uint32_t* status;             // sticky status word
};

// Heads merged by one CTA of the combine kernel (one warp per head).
constexpr int kCombineHeadsPerCta = 4;

// Dynamic shared memory of the split kernel, its attribute set-up (for the
// current device) and its launch (one CTA per part and 64-head group, or for
// 128 heads with cta_pairs a two-CTA cluster per part; chained to the
// previous kernel with programmatic dependent launch).
int splitkv_smem_bytes();
cudaError_t configure_splitkv();
cudaError_t launch_splitkv(const SplitKVParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Host side shared by smla_flash_mla_with_kvcache and its allocation-free
// variant, so both size, check and launch the decode the same way.
// ---------------------------------------------------------------------------

// A decode call's arguments as the C ABI receives them.
struct DecodeCall {
  const void* q;
  const uint8_t* kvcache;
  int64_t num_blocks;
  const int32_t* block_table;
  int max_blocks;
  const int32_t* cache_seqlens;
  const int32_t* indices;
  const int32_t* sched_meta;
  const int32_t* num_splits;
  int num_sm_parts;
  float softmax_scale;
  int batch, s_q, h_q, topk;
  void* o;
  float* lse;
  // dense decode (left at their defaults by the sparse entry points)
  const int32_t* tile_prefix = nullptr;
  int kv_mode = kSparseFp8;
  int causal = 0;
};

// Records a failing CUDA runtime result for smla_last_cuda_error (one slot
// per host thread) and returns SMLA_ERR_CUDA.
int cuda_failure(cudaError_t e);
int g_last_cuda_error_value();

// The process-wide form of 128-head decodes (smla_set_head_pair_form).
int head_pair_form();

// Scratch layout of a decode: a 256-byte status header, then float32
// o_accum [max_splits][h_q][512] and lse_accum [max_splits][h_q], each
// starting 256-byte aligned, with max_splits = batch * s_q + num_sm_parts.
constexpr size_t kStatusHeaderBytes = 256;
struct WorkspaceLayout {
  size_t o_accum_off, lse_accum_off, total;
};
WorkspaceLayout workspace_layout(int batch, int s_q, int h_q, int num_sm_parts);

// Host-side checks of a decode call (everything but the scratch): an
// smla_status code, SMLA_OK when the call may be launched.  A call with
// batch == 0 passes and launches nothing.
int check_decode_call(const DecodeCall& c);

// The current CUDA context as an opaque handle (nullptr if it cannot be
// queried).  Module-level state (kernel attributes, the device address of a
// __device__ array) belongs to a context, which cudaDeviceReset replaces.
void* current_context();

// Makes the split kernel launchable on the current device (sm_100 check and
// the dynamic shared-memory attribute), once per device and CUDA context.
int ensure_decode_kernels();

// Launches the split kernel and, chained to it, the combine kernel, with
// the partials in `scratch` (laid out by workspace_layout) and the sticky
// status word at `status`.  The call must have passed check_decode_call.
int launch_decode(const DecodeCall& c, uint8_t* scratch, uint32_t* status, cudaStream_t stream);

}  // namespace smla
