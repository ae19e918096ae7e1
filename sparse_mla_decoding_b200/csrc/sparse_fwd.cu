// sparse_fwd.cu -- sparse attention of many query tokens over one flat FP8
// cache (flash_mla_sparse_fwd).
//
// Source: "deepseek-ai/FlashMLA" (agentlenshq), section 使用方法 item 2: the
// sparse prefill entry takes the query tensor, the KV cache and a 3-D indices
// tensor saying which KV tokens each query token attends to; the same page
// (技術的な詳細) marks skipped entries with -1.  The computation per query
// token is the one of the sparse decode (row j of the cache instead of a
// block-table lookup), so this entry runs the decode path: a small kernel
// writes an identity block table (block b -> b) and the one request length
// into the workspace, then the scheduler, the split kernel and the combine
// run on batch 1 with s_q query tokens.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/smla.h"
#include "splitkv_mla.h"

namespace smla {

// The one request's length and an identity block table over nb blocks.
__global__ void sparse_fwd_setup_kernel(int32_t* seqlen, int32_t* block_table, int nb, int32_t s_kv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) *seqlen = s_kv;
  for (int b = i; b < nb; b += gridDim.x * blockDim.x) block_table[b] = b;
}

}  // namespace smla

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct SparseFwdLayout {
  size_t decode_bytes, sched_off, splits_off, seqlen_off, table_off, total;
};

// [decode workspace (status header + split partials)] [sched_meta] [num_splits]
// [request length] [identity block table]
SparseFwdLayout sparse_fwd_layout(int s_q, int h_q, int topk, int num_sm_parts, int nb) {
  SparseFwdLayout l;
  l.decode_bytes = smla_workspace_bytes(1, s_q, h_q, topk, num_sm_parts);
  l.sched_off = align_up(l.decode_bytes);
  l.splits_off = l.sched_off + align_up((size_t)num_sm_parts * 8 * sizeof(int32_t));
  l.seqlen_off = l.splits_off + align_up(((size_t)s_q + 1) * sizeof(int32_t));
  l.table_off = l.seqlen_off + kAlign;
  l.total = l.table_off + align_up((size_t)nb * sizeof(int32_t));
  return l;
}

bool valid_shape(int s_q, int h_q, int64_t s_kv, int topk, int num_sm_parts) {
  return s_q >= 1 && (h_q == 16 || h_q == 32 || h_q == 64 || h_q == 128) && topk >= 1 && num_sm_parts >= 1 &&
         s_kv >= 1 && s_kv <= (int64_t)(0x7FFFFFFF / SMLA_BLOCK_SIZE) * SMLA_BLOCK_SIZE;
}

}  // namespace

extern "C" {

size_t smla_sparse_fwd_workspace_bytes(int s_q, int h_q, int64_t s_kv, int topk, int num_sm_parts) {
  if (!valid_shape(s_q, h_q, s_kv, topk, num_sm_parts)) return 0;
  const int nb = (int)((s_kv + SMLA_BLOCK_SIZE - 1) / SMLA_BLOCK_SIZE);
  return sparse_fwd_layout(s_q, h_q, topk, num_sm_parts, nb).total;
}

int smla_flash_mla_sparse_fwd(const void* q, const uint8_t* kv, int64_t s_kv, const int32_t* indices, int s_q,
                              int h_q, int topk, int num_sm_parts, float softmax_scale, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (h_q != 16 && h_q != 32 && h_q != 64 && h_q != 128) return SMLA_ERR_UNSUPPORTED;
  if (!valid_shape(s_q, h_q, s_kv, topk, num_sm_parts)) return SMLA_ERR_INVALID_ARGUMENT;
  if (!q || !kv || !indices || !o || !lse || !workspace) return SMLA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return SMLA_ERR_INVALID_ARGUMENT;
  const int nb = (int)((s_kv + SMLA_BLOCK_SIZE - 1) / SMLA_BLOCK_SIZE);
  const SparseFwdLayout l = sparse_fwd_layout(s_q, h_q, topk, num_sm_parts, nb);
  if (l.decode_bytes == 0 || workspace_bytes < l.total) return SMLA_ERR_INVALID_ARGUMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* sched_meta = reinterpret_cast<int32_t*>(ws + l.sched_off);
  int32_t* num_splits = reinterpret_cast<int32_t*>(ws + l.splits_off);
  int32_t* seqlen = reinterpret_cast<int32_t*>(ws + l.seqlen_off);
  int32_t* table = reinterpret_cast<int32_t*>(ws + l.table_off);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  const int threads = 256;
  const int blocks = (nb + threads - 1) / threads < 1024 ? (nb + threads - 1) / threads : 1024;
  smla::sparse_fwd_setup_kernel<<<blocks, threads, 0, st>>>(seqlen, table, nb, (int32_t)s_kv);
  if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) return smla::cuda_failure(e);
  if (int rc = smla_get_mla_metadata(seqlen, 1, s_q, topk, h_q, num_sm_parts, sched_meta, num_splits, stream))
    return rc;
  return smla_flash_mla_with_kvcache(q, kv, nb, table, nb, seqlen, indices, sched_meta, num_splits, num_sm_parts,
                                     softmax_scale, 1, s_q, h_q, topk, o, lse, workspace, l.decode_bytes, stream);
}

}  // extern "C"
