/*
 * smla.h -- C ABI of libsmla.so: token-level sparse Multi-head Latent
 * Attention (MLA) decoding over a paged FP8 KV cache, for NVIDIA B200
 * (sm_100a).
 *
 * The operation (sources cited by page title and section):
 *   "FlashMLA 注意力内核源码走读：656 字节 KV 缓存背后的完整链路" -- sections
 *   调度 (a small kernel assigns (request, KV-range) work evenly to all SMs
 *   before the main kernel; the table can be reused while shapes stay the
 *   same), 解码阶段调用示例 (get_mla_metadata, then flash_mla_with_kvcache with
 *   the sparse indices, returning o and lse), 数据加载 (each token's 656-byte
 *   FP8 row; dequantise to bf16, concatenate the 64 RoPE values, bf16 MMAs
 *   with fp32 accumulation) and 合并与性能账本 (each split leaves a partial o
 *   and lse; a combine kernel merges them by lse; the two kernels are chained
 *   with Programmatic Dependent Launch).
 *   "deepseek-ai/FlashMLA" (agentlenshq), section 技術的な詳細: the indices
 *   tensor is 3-D and -1 marks an entry the kernel ignores.
 *   "FlashMLA：DeepSeek开源的高效MLA解码内核，专为NVIDIA Hopper GPU优化",
 *   section 主要功能特性: the paged KV cache uses blocks of 64 tokens.
 *
 * Shapes: MQA with one KV head; d_qk = 576 (512 latent + 64 RoPE); d_v = 512
 * (the latent part of the same row).  For query token (b, t) and head h:
 *   valid slots j: 0 <= indices[b][t][j] < cache_seqlens[b]
 *   row(j)       : block_table[b][idx / 64] * 64 + idx % 64
 *   k_j          : bf16(float(e4m3) * scale) for the 512 latent values (the
 *                  product rounded in float32, then to bf16), then the 64 RoPE
 *   s_j          : softmax_scale * <q[b][t][h], k_j>
 *   lse          : ln(sum_j exp(s_j))   (-inf when no slot is valid)
 *   o            : sum_j exp(s_j - lse) * k_j[0:512]   (0 when no slot is valid)
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must be device memory of the current device;
 *     "host" means host memory.  The caller owns every buffer; the library
 *     never allocates device memory, never synchronises a stream (except
 *     smla_get_device_status, which says so) and keeps no state beyond a
 *     per-device cache of kernel attributes.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Return value: an smla_status.  Argument errors are detected on the host
 *     before anything is launched.  SMLA_ERR_CUDA means a launch failed; an
 *     asynchronous device error surfaces at the caller's next synchronisation.
 *   - All tensors are dense, row-major, in the layouts given per argument.
 */
#ifndef SMLA_H_
#define SMLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SMLA_OK = 0,
  SMLA_ERR_INVALID_ARGUMENT = 1, /* a null pointer, a bad size or an inconsistent shape */
  SMLA_ERR_UNSUPPORTED = 2,      /* h_q not in {16, 32, 64, 128}, or a device that is not sm_100 */
  SMLA_ERR_CUDA = 3,             /* a CUDA runtime call or a kernel launch failed */
  SMLA_ERR_DEVICE_TIMEOUT = 4,   /* reported by smla_get_device_status: a bounded device wait gave up */
  SMLA_ERR_SCRATCH_LIMIT = 5     /* the call needs more than SMLA_STATIC_SCRATCH_BYTES of library scratch */
} smla_status;

/* Head dimensions fixed by the operation. */
#define SMLA_D_QK 576
#define SMLA_D_V 512
#define SMLA_D_ROPE 64
#define SMLA_KV_ROW_BYTES 656   /* 512 e4m3 | 4 x float32 scale | 64 x bf16 RoPE */
#define SMLA_BLOCK_SIZE 64      /* tokens per paged-cache block */
#define SMLA_INDEX_TILE 64      /* index slots per scheduling tile */
/* Size of the library-owned device scratch of smla_flash_mla_with_kvcache_static_scratch. */
#define SMLA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Human-readable name of a status code (static string, never NULL). */
const char* smla_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int smla_version(void);

/*
 * The CUDA runtime error (a cudaError_t value) behind the most recent
 * SMLA_ERR_CUDA that this host thread received, and its name (a static
 * string, never NULL).  0 / "cudaSuccess" before any such failure.
 */
int smla_last_cuda_error(void);
const char* smla_last_cuda_error_string(void);

/*
 * Default number of scheduler parts for h_q heads on `device`: one part per
 * CTA group that can be resident at once (the SM count for h_q <= 64; half of
 * it for h_q = 128, where a part is two CTAs that own 64 heads each).
 * Returns a value >= 1, or -1 if the device cannot be queried.
 */
int smla_default_num_sm_parts(int h_q, int device);

/*
 * How the two 64-head CTAs of a 128-head part share a tile ("FlashMLA
 * 注意力内核源码走读…", section 计算环节一, describes the shared form).
 *   enable = 0 (default): independent CTAs; each gathers and dequantises all
 *                64 rows of a tile (the second read of a row mostly hits L2).
 *   enable = 1: a two-CTA cluster; each CTA dequantises half of the rows and
 *                copies them into its peer's shared memory.
 * Both forms give bitwise identical results; on B200 the independent form
 * measured faster.  The setting is process-wide, takes effect at the next
 * decode call, and returns the previous setting.
 */
int smla_set_head_pair_form(int enable);

/*
 * Bytes of caller-provided device workspace that smla_flash_mla_with_kvcache
 * needs for the given shape: a 256-byte header (the sticky device status
 * word) followed by the split partials (float32 o_accum and lse_accum for at
 * most batch*s_q + num_sm_parts splits).  The header must be zeroed once when
 * the workspace is allocated (smla_reset_device_status does that).
 * Returns 0 for invalid arguments.
 */
size_t smla_workspace_bytes(int batch, int s_q, int h_q, int topk, int num_sm_parts);

/*
 * Tile-scheduler metadata ("FlashMLA 注意力内核源码走读…", section 调度).
 * Splits the R = batch*s_q requests x n = ceil(topk/64) index tiles evenly
 * over num_sm_parts parts, before the main kernel, on `stream`:
 *   L = ceil(R*n / P); part p covers the tiles [p*L, min((p+1)*L, R*n)) in
 *   (request, tile) order.
 *   sched_meta[p] = {begin_r, begin_tile, end_r, end_tile (exclusive end),
 *                    first_split_slot, is_empty, 0, 0}
 *   num_splits[r] = number of split slots before request r (exclusive prefix
 *                   sum of the splits per request); num_splits[R] = total.
 * In sparse mode the work of a request is set by its index slots, not by its
 * length, so cache_seqlens is accepted for interface parity and not read.
 * The output can be reused by every call (and layer) with the same batch,
 * s_q, topk and num_sm_parts.
 *   cache_seqlens : device int32 [batch] (may be NULL)
 *   sched_meta    : device int32 [num_sm_parts][8], written
 *   num_splits    : device int32 [batch*s_q + 1], written
 */
int smla_get_mla_metadata(const int32_t* cache_seqlens, int batch, int s_q, int topk, int h_q,
                          int num_sm_parts, int32_t* sched_meta, int32_t* num_splits, void* stream);

/*
 * Sparse MLA decode ("FlashMLA 注意力内核源码走读…", sections 解码阶段调用示例,
 * 数据加载, 合并与性能账本).  Launches the split-KV kernel (one CTA per
 * scheduler part and 64-head group, see smla_set_head_pair_form, each
 * walking its part's (request, tile) ranges from sched_meta) and, chained to
 * it with Programmatic Dependent Launch, the LSE combine kernel for requests
 * that were split.  Output is bitwise reproducible run to run (static
 * schedule, no floating-point atomics).
 *   q             : device bf16 [batch][s_q][h_q][576]
 *   kvcache       : device uint8 [num_blocks][64][656] (16-byte aligned);
 *                   num_blocks <= 33554431 (rows are numbered with 32 bits)
 *   block_table   : device int32 [batch][max_blocks]
 *   cache_seqlens : device int32 [batch]
 *   indices       : device int32 [batch][s_q][topk]; -1 (any negative) or a
 *                   value >= cache_seqlens[b] means "skip this slot"
 *   sched_meta, num_splits : from smla_get_mla_metadata with the same
 *                   batch, s_q, topk and num_sm_parts
 *   softmax_scale : <= 0 or NaN selects the default 1/sqrt(576)
 *   o             : device bf16 [batch][s_q][h_q][512], written
 *   lse           : device float32 [batch][s_q][h_q], natural log, written
 *   workspace     : device, >= smla_workspace_bytes(...) bytes, 256-byte aligned
 * A valid index whose block lies outside block_table or the cache is skipped
 * and sets a flag in the workspace status word (see smla_get_device_status).
 */
int smla_flash_mla_with_kvcache(const void* q, const uint8_t* kvcache, int64_t num_blocks,
                                const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                const int32_t* indices, const int32_t* sched_meta, const int32_t* num_splits,
                                int num_sm_parts, float softmax_scale, int batch, int s_q, int h_q, int topk,
                                void* o, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Row formats of a dense-decode cache. */
#define SMLA_KV_FP8 0           /* 656-byte rows as for the sparse decode                       */
#define SMLA_KV_BF16 1          /* 1152-byte rows: the 576-wide key as bf16 (latent, then RoPE) */

/*
 * Scheduler metadata of a dense decode ("FlashMLA：DeepSeek开源的高效MLA解码内核…",
 * sections 主要功能特性 and 基础用法示例: get_mla_metadata from the cache lengths,
 * then flash_mla_with_kvcache with causal=True; "FlashMLA 注意力内核源码走读…",
 * section 调度: the work is spread evenly over the SMs before the main kernel).
 * Request r = b * s_q + t attends to the len_r visible tokens of batch entry
 * b: len_r = cache_seqlens[b], or with the causal mask cache_seqlens[b] -
 * (s_q - 1 - t) (the s_q new tokens are the last s_q positions of the cache),
 * at least 0.  Its work is n_r = max(1, ceil(len_r / 64)) tiles, so the split
 * follows the lengths: tile_prefix[r] = tiles before request r (tile_prefix[R]
 * = the total, which must stay below 2^31), then the tiles in (request, tile)
 * order are cut into num_sm_parts ranges of L = ceil(total / P) as for
 * smla_get_mla_metadata, with tile positions counted within each request.
 *   cache_seqlens : device int32 [batch]
 *   sched_meta    : device int32 [num_sm_parts][8], written (16-byte aligned)
 *   num_splits    : device int32 [batch*s_q + 1], written
 *   tile_prefix   : device int32 [batch*s_q + 1], written
 * Launches one CTA on `stream`; reusable while cache_seqlens, s_q, causal and
 * num_sm_parts stay the same.
 */
int smla_get_mla_metadata_dense(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int causal,
                                int num_sm_parts, int32_t* sched_meta, int32_t* num_splits, int32_t* tile_prefix,
                                void* stream);

/*
 * Dense MLA decode: every query token attends to all its visible cache tokens
 * ("FlashMLA：DeepSeek开源的高效MLA解码内核…", sections 主要功能特性 (paged cache
 * with 64-token blocks, BF16) and 基础用法示例 (flash_mla_with_kvcache with
 * causal=True)).  The same split kernel and combine as the sparse decode run
 * with the index list of request r taken to be 0 .. len_r - 1 (len_r as in
 * smla_get_mla_metadata_dense), made in the kernel instead of read from
 * memory.  With kv_format SMLA_KV_FP8 the rows are the 656-byte FP8 rows of
 * the sparse decode; with SMLA_KV_BF16 they are 1152-byte rows of 576 bf16
 * values, used as they are.
 *   q             : device bf16 [batch][s_q][h_q][576]
 *   kvcache       : device uint8 [num_blocks][64][656 or 1152] (16-byte aligned)
 *   block_table   : device int32 [batch][max_blocks]
 *   cache_seqlens : device int32 [batch]
 *   sched_meta, num_splits, tile_prefix : from smla_get_mla_metadata_dense
 *                   with the same batch, s_q, causal and num_sm_parts
 *   causal        : 0 or 1, as for the metadata
 *   o, lse, workspace : as for smla_flash_mla_with_kvcache (the workspace
 *                   size is smla_workspace_bytes(batch, s_q, h_q, 1,
 *                   num_sm_parts))
 * A visible position whose block lies outside block_table or the cache is
 * skipped and flags the workspace status word, as in the sparse decode.
 */
int smla_flash_mla_dense_with_kvcache(const void* q, const uint8_t* kvcache, int kv_format, int64_t num_blocks,
                                      const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                      const int32_t* sched_meta, const int32_t* num_splits,
                                      const int32_t* tile_prefix, int num_sm_parts, float softmax_scale, int causal,
                                      int batch, int s_q, int h_q, void* o, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * Sparse attention of many query tokens over one flat (unpaged) FP8 cache
 * ("deepseek-ai/FlashMLA" (agentlenshq), section 使用方法 item 2:
 * flash_mla_sparse_fwd(q, kv, indices, ...) with a 3-D indices tensor that
 * names the KV tokens each query token attends to; 技術的な詳細: -1 marks a
 * skipped entry).  Query token t and head h attend to the rows
 * kv[indices[t][0][j]] with 0 <= indices[t][0][j] < s_kv, with the row
 * format, dequantisation, scores, o and lse of smla_flash_mla_with_kvcache.
 * Runs the decode path on batch 1 with s_q query tokens: a small kernel
 * writes an identity block table and the request length into the
 * workspace, then the scheduler, the split kernel and the combine run on
 * `stream`.
 *   q        : device bf16 [s_q][h_q][576] (16-byte aligned)
 *   kv       : device uint8 [s_kv][656] (16-byte aligned), one KV head;
 *              1 <= s_kv <= 2147483584
 *   indices  : device int32 [s_q][1][topk]; negative or >= s_kv = skip
 *   num_sm_parts : scheduler parts (smla_default_num_sm_parts(h_q, device))
 *   softmax_scale : <= 0 or NaN selects the default 1/sqrt(576)
 *   o        : device bf16 [s_q][h_q][512], written
 *   lse      : device float32 [s_q][h_q], natural log, written
 *   workspace: device, >= smla_sparse_fwd_workspace_bytes(...) bytes,
 *              256-byte aligned; its first 256 bytes are the status header
 *              (zero it once; read it with smla_get_device_status)
 */
int smla_flash_mla_sparse_fwd(const void* q, const uint8_t* kv, int64_t s_kv, const int32_t* indices, int s_q,
                              int h_q, int topk, int num_sm_parts, float softmax_scale, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes of smla_flash_mla_sparse_fwd: the decode workspace for
 * (batch 1, s_q, h_q, topk, num_sm_parts), the scheduler tables, the
 * request length and a block table of ceil(s_kv / 64) entries.  Returns 0
 * for invalid arguments.
 */
size_t smla_sparse_fwd_workspace_bytes(int s_q, int h_q, int64_t s_kv, int topk, int num_sm_parts);

/*
 * Write tokens into the 656-byte FP8 cache rows ("FlashMLA 注意力内核源码走读…",
 * section 数据加载: the first 512 dimensions are quantised per 1x128 tile):
 * per tile, scale = amax / 448 in float32, byte = e4m3(x / scale) rounded to
 * nearest even with saturation to +-448; an all-zero tile stores scale 0 and
 * zero bytes; the 64 RoPE values are copied as bf16.
 *   latent       : device bf16 [n_tokens][512]
 *   rope         : device bf16 [n_tokens][64]
 *   slot_mapping : device int64 [n_tokens], destination row of each token
 *                  (block * 64 + offset); NULL writes token i to row i.
 *                  Negative entries skip the token.
 *   kvcache      : device uint8 [num_rows][656], rows written
 */
int smla_quantize_kv(const void* latent, const void* rope, int64_t n_tokens, const int64_t* slot_mapping,
                     uint8_t* kvcache, int64_t num_rows, void* stream);

/*
 * Read the sticky status word in a workspace (synchronises `stream` first).
 * *status_out receives SMLA_OK, SMLA_ERR_DEVICE_TIMEOUT (a bounded wait in a
 * kernel gave up) or SMLA_ERR_INVALID_ARGUMENT (a valid index mapped past the
 * block table or the cache).  *raw_flags_out (may be NULL) receives the raw
 * flag bits.  The word stays set until smla_reset_device_status.
 *   workspace : device, as passed to smla_flash_mla_with_kvcache
 */
int smla_get_device_status(const void* workspace, int* status_out, uint32_t* raw_flags_out, void* stream);

/*
 * Allocation-free variant of smla_flash_mla_with_kvcache.  The pages
 * describe no counterpart; it exists for callers that cannot allocate device
 * memory -- allocator-less runtimes and embedders that hand the library only
 * their inputs and outputs, code where an allocation would synchronise or is
 * not allowed, hosts whose memory planner owns every device byte.  Instead of
 * a caller workspace it uses a fixed array of SMLA_STATIC_SCRATCH_BYTES
 * (64 MiB) in the library's own device memory, which every GPU that loads
 * the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *   Arguments as for smla_flash_mla_with_kvcache, without the workspace, plus
 *   status_out : device uint32 (may be NULL).  If given, the kernels OR their
 *                status flags (see smla_get_device_status) into it; the
 *                caller zeroes it and reads it after the call.  If NULL, the
 *                flags go to the scratch header, which each call clears
 *                first and which no API reads back: the caller then gives up
 *                device-side error detection, and after such an error (a bad
 *                block-table entry, inconsistent metadata, a wait that gave
 *                up) o and lse may be built from incomplete or stale partials
 *                while the call still returns SMLA_OK.
 * The scratch need is the same as smla_workspace_bytes(batch, s_q, h_q, topk,
 * num_sm_parts); a call that needs more returns SMLA_ERR_SCRATCH_LIMIT and
 * launches nothing.  Every call on a device shares the one array and it keeps
 * the last call's contents: calls whose kernels overlap on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller.  The first call on each device does a one-time set-up with that
 * device current (it looks up the array's device address and sets a kernel
 * attribute), repeated only if the device's CUDA context is re-created (for
 * instance after cudaDeviceReset, which loads the module anew); make that
 * first call before any stream capture.
 */
int smla_flash_mla_with_kvcache_static_scratch(const void* q, const uint8_t* kvcache, int64_t num_blocks,
                                               const int32_t* block_table, int max_blocks,
                                               const int32_t* cache_seqlens, const int32_t* indices,
                                               const int32_t* sched_meta, const int32_t* num_splits,
                                               int num_sm_parts, float softmax_scale, int batch, int s_q, int h_q,
                                               int topk, void* o, float* lse, uint32_t* status_out, void* stream);

/* Clear the workspace status word (asynchronously, on `stream`). */
int smla_reset_device_status(void* workspace, void* stream);

/*
 * Self-test of the bounded device wait: launches one CTA that waits on a
 * shared-memory barrier nobody arrives at, giving up after `limit_ns`
 * nanoseconds (1 .. 10^10) and setting the timeout flag in the workspace
 * status word.  It exercises the same wait routine the kernels use, without
 * hanging or faulting the GPU.
 *   workspace : device, at least 256 bytes
 */
int smla_selftest_bounded_wait(void* workspace, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SMLA_H_ */
