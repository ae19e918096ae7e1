// splitkv_mla.h -- parameters of the split-KV sparse MLA decode kernel (device side).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace smla {

struct SplitKVParams {
  const __nv_bfloat16* q;       // [R][h_q][576], R = batch * s_q
  const uint8_t* kv;            // [num_blocks][64][656]
  int64_t num_blocks;
  const int32_t* block_table;   // [batch][max_blocks]
  int max_blocks;
  const int32_t* seqlens;       // [batch]
  const int32_t* indices;       // [R][topk]
  const int32_t* sched_meta;    // [num_parts][8]
  const int32_t* num_splits;    // [R + 1]
  int s_q, h_q, topk, n_tiles, num_parts;
  int num_requests;             // R = batch * s_q
  int max_splits;               // split slots the workspace holds (R + num_parts)
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* o;             // [R][h_q][512]
  float* lse;                   // [R][h_q]
  float* o_accum;               // [splits][h_q][512]
  float* lse_accum;             // [splits][h_q]
  uint32_t* status;             // sticky status word
};

// Dynamic shared memory of the split kernel, its one-time attribute set-up
// (per device) and its launch (single CTA for <= 64 heads, a two-CTA cluster
// for 128 heads; chained to the previous kernel with programmatic dependent
// launch).
int splitkv_smem_bytes();
cudaError_t configure_splitkv();
cudaError_t launch_splitkv(const SplitKVParams& p, cudaStream_t stream);

}  // namespace smla
