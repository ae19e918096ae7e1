// smla_api.cu -- the C ABI of libsmla.so (declared in include/smla.h): host-side
// argument checks, workspace layout and kernel launches.  No device memory is
// allocated and no stream is synchronised here (except where a function's
// contract says so).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/smla.h"
#include "sm100.cuh"
#include "splitkv_mla.h"

namespace smla {
__global__ void sched_meta_kernel(int R, int n, int P, int32_t* sched_meta, int32_t* num_splits);
__global__ void sched_meta_dense_kernel(const int32_t* seqlens, int batch, int s_q, int causal, int P,
                                        int32_t* sched_meta, int32_t* num_splits, int32_t* tile_prefix);
__global__ void combine_kernel(const int32_t* num_splits, const float* o_accum, const float* lse_accum, int h_q,
                               int max_splits, __nv_bfloat16* o, float* lse);
__global__ void quantize_kv_kernel(const __nv_bfloat16* latent, const __nv_bfloat16* rope, int64_t n_tokens,
                                   const int64_t* slot_mapping, uint8_t* kvcache, int64_t num_rows);
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns);
}  // namespace smla

namespace {

constexpr int kMaxDevices = 64;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_h_q(int h_q) { return h_q == 16 || h_q == 32 || h_q == 64 || h_q == 128; }

int head_groups(int h_q) { return (h_q + 63) / 64; }

int64_t n_tiles_of(int topk) { return ((int64_t)topk + SMLA_INDEX_TILE - 1) / SMLA_INDEX_TILE; }

cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  std::memset(&a, 0, sizeof(a));
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

std::mutex g_setup_mutex;
std::atomic<int> g_head_pair_form{0};
void* g_configured_ctx[kMaxDevices] = {nullptr};

}  // namespace

namespace smla {

// The current CUDA context as an opaque handle (the driver's cuCtxGetCurrent,
// looked up once through the runtime), or nullptr when it cannot be queried.
// Kernel attributes belong to a context: after cudaDeviceReset the device's
// primary context is a new one and the attributes must be set again.
void* current_context() {
  typedef int (*CtxGetCurrentFn)(void**);
  static CtxGetCurrentFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

namespace {
thread_local int g_last_cuda_error = 0;
}  // namespace

int g_last_cuda_error_value() { return g_last_cuda_error; }

int head_pair_form() { return g_head_pair_form.load(std::memory_order_relaxed); }

int cuda_failure(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return SMLA_ERR_CUDA;
}

WorkspaceLayout workspace_layout(int batch, int s_q, int h_q, int num_sm_parts) {
  const size_t max_splits = (size_t)batch * s_q + (size_t)num_sm_parts;
  WorkspaceLayout w;
  w.o_accum_off = kStatusHeaderBytes;
  const size_t o_bytes = max_splits * (size_t)h_q * SMLA_D_V * sizeof(float);
  w.lse_accum_off = w.o_accum_off + ((o_bytes + 255) & ~size_t(255));
  const size_t l_bytes = max_splits * (size_t)h_q * sizeof(float);
  w.total = w.lse_accum_off + ((l_bytes + 255) & ~size_t(255));
  return w;
}

int check_decode_call(const DecodeCall& c) {
  if (!valid_h_q(c.h_q)) return SMLA_ERR_UNSUPPORTED;
  // cache rows are addressed as 32-bit row numbers (block * 64 + offset)
  if (c.batch < 0 || c.s_q < 1 || c.topk < 1 || c.num_sm_parts < 1 || c.max_blocks < 1 || c.num_blocks < 1 ||
      c.num_blocks > (int64_t)(0x7FFFFFFF / SMLA_BLOCK_SIZE))
    return SMLA_ERR_INVALID_ARGUMENT;
  if (c.batch == 0) return SMLA_OK;
  const bool dense = c.kv_mode != kSparseFp8;
  if (!c.q || !c.kvcache || !c.block_table || !c.cache_seqlens || (!dense && !c.indices) || !c.sched_meta ||
      !c.num_splits || (dense && !c.tile_prefix) || !c.o || !c.lse)
    return SMLA_ERR_INVALID_ARGUMENT;
  if (c.kv_mode < kSparseFp8 || c.kv_mode > kDenseBf16 || (dense && c.causal != 0 && c.causal != 1))
    return SMLA_ERR_INVALID_ARGUMENT;
  if (!aligned(c.q, 16) || !aligned(c.kvcache, 16) || !aligned(c.o, 16) || !aligned(c.sched_meta, 16))
    return SMLA_ERR_INVALID_ARGUMENT;
  const int64_t R = (int64_t)c.batch * c.s_q;
  if (R > (1 << 28) || n_tiles_of(c.topk) > (1 << 24)) return SMLA_ERR_INVALID_ARGUMENT;
  return SMLA_OK;
}

int ensure_decode_kernels() {
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return smla::cuda_failure(e);
  if (dev < 0 || dev >= kMaxDevices) return SMLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  void* ctx = current_context();
  if (ctx != nullptr && g_configured_ctx[dev] == ctx) return SMLA_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return SMLA_ERR_UNSUPPORTED;
  if (const cudaError_t e = configure_splitkv(); e != cudaSuccess) return smla::cuda_failure(e);
  // the attribute call above made the context current if it was not yet
  g_configured_ctx[dev] = ctx != nullptr ? ctx : current_context();
  return SMLA_OK;
}

int launch_decode(const DecodeCall& c, uint8_t* scratch, uint32_t* status, cudaStream_t stream) {
  if (c.batch == 0) return SMLA_OK;
  const WorkspaceLayout wl = workspace_layout(c.batch, c.s_q, c.h_q, c.num_sm_parts);
  const int64_t R = (int64_t)c.batch * c.s_q;
  float scale = c.softmax_scale;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)SMLA_D_QK);

  SplitKVParams p;
  p.q = static_cast<const __nv_bfloat16*>(c.q);
  p.kv = c.kvcache;
  p.num_blocks = c.num_blocks;
  p.block_table = c.block_table;
  p.max_blocks = c.max_blocks;
  p.seqlens = c.cache_seqlens;
  p.indices = c.indices;
  p.tile_prefix = c.tile_prefix;
  p.kv_mode = c.kv_mode;
  p.cta_pairs = head_pair_form();
  p.causal = c.causal;
  p.sched_meta = c.sched_meta;
  p.num_splits = c.num_splits;
  p.s_q = c.s_q;
  p.h_q = c.h_q;
  p.topk = c.topk;
  p.n_tiles = c.tile_prefix ? 0 : (int)n_tiles_of(c.topk);
  p.num_parts = c.num_sm_parts;
  p.num_requests = (int)R;
  p.max_splits = (int)(R + c.num_sm_parts);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(c.o);
  p.lse = c.lse;
  p.o_accum = reinterpret_cast<float*>(scratch + wl.o_accum_off);
  p.lse_accum = reinterpret_cast<float*>(scratch + wl.lse_accum_off);
  p.status = status;
  if (const cudaError_t e = launch_splitkv(p, stream); e != cudaSuccess) return smla::cuda_failure(e);

  cudaLaunchAttribute attr = pdl_attribute();
  cudaLaunchConfig_t ccfg;
  std::memset(&ccfg, 0, sizeof(ccfg));
  ccfg.gridDim = dim3((unsigned)R, (unsigned)((c.h_q + kCombineHeadsPerCta - 1) / kCombineHeadsPerCta));
  ccfg.blockDim = dim3(32 * kCombineHeadsPerCta);
  ccfg.stream = stream;
  ccfg.attrs = &attr;
  ccfg.numAttrs = 1;
  if (const cudaError_t e = cudaLaunchKernelEx(&ccfg, combine_kernel, (const int32_t*)c.num_splits,
                                               (const float*)p.o_accum, (const float*)p.lse_accum, c.h_q,
                                               p.max_splits, p.o, c.lse);
      e != cudaSuccess)
    return cuda_failure(e);
  return SMLA_OK;
}

}  // namespace smla

extern "C" {

const char* smla_status_string(int status) {
  switch (status) {
    case SMLA_OK: return "SMLA_OK";
    case SMLA_ERR_INVALID_ARGUMENT: return "SMLA_ERR_INVALID_ARGUMENT";
    case SMLA_ERR_UNSUPPORTED: return "SMLA_ERR_UNSUPPORTED";
    case SMLA_ERR_CUDA: return "SMLA_ERR_CUDA";
    case SMLA_ERR_DEVICE_TIMEOUT: return "SMLA_ERR_DEVICE_TIMEOUT";
    case SMLA_ERR_SCRATCH_LIMIT: return "SMLA_ERR_SCRATCH_LIMIT";
    default: return "SMLA_UNKNOWN_STATUS";
  }
}

int smla_version(void) { return 102; }

int smla_set_head_pair_form(int enable) { return g_head_pair_form.exchange(enable != 0 ? 1 : 0); }

int smla_last_cuda_error(void) { return smla::g_last_cuda_error_value(); }

const char* smla_last_cuda_error_string(void) {
  return cudaGetErrorName(static_cast<cudaError_t>(smla::g_last_cuda_error_value()));
}

int smla_default_num_sm_parts(int h_q, int device) {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) return -1;
  const int per_part = head_groups(h_q > 0 ? h_q : 64);
  const int parts = sms / per_part;
  return parts > 0 ? parts : 1;
}

size_t smla_workspace_bytes(int batch, int s_q, int h_q, int topk, int num_sm_parts) {
  if (batch < 0 || s_q < 1 || !valid_h_q(h_q) || topk < 1 || num_sm_parts < 1) return 0;
  return smla::workspace_layout(batch, s_q, h_q, num_sm_parts).total;
}

int smla_get_mla_metadata(const int32_t* cache_seqlens, int batch, int s_q, int topk, int h_q, int num_sm_parts,
                          int32_t* sched_meta, int32_t* num_splits, void* stream) {
  (void)cache_seqlens;
  if (batch < 0 || s_q < 1 || topk < 1 || num_sm_parts < 1 || !sched_meta || !num_splits)
    return SMLA_ERR_INVALID_ARGUMENT;
  if (!valid_h_q(h_q)) return SMLA_ERR_UNSUPPORTED;
  if (!aligned(sched_meta, 16)) return SMLA_ERR_INVALID_ARGUMENT;
  const int64_t R = (int64_t)batch * s_q;
  if (R > (1 << 28) || R * n_tiles_of(topk) > ((int64_t)1 << 40)) return SMLA_ERR_INVALID_ARGUMENT;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(256);
  cfg.stream = static_cast<cudaStream_t>(stream);
  if (const cudaError_t e = cudaLaunchKernelEx(&cfg, smla::sched_meta_kernel, (int)R, (int)n_tiles_of(topk),
                                               num_sm_parts, sched_meta, num_splits);
      e != cudaSuccess)
    return smla::cuda_failure(e);
  return SMLA_OK;
}

int smla_flash_mla_with_kvcache(const void* q, const uint8_t* kvcache, int64_t num_blocks, const int32_t* block_table,
                                int max_blocks, const int32_t* cache_seqlens, const int32_t* indices,
                                const int32_t* sched_meta, const int32_t* num_splits, int num_sm_parts,
                                float softmax_scale, int batch, int s_q, int h_q, int topk, void* o, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream) {
  const smla::DecodeCall c{q,          kvcache, num_blocks, block_table, max_blocks, cache_seqlens,
                           indices,    sched_meta, num_splits, num_sm_parts, softmax_scale, batch,
                           s_q,        h_q,     topk,       o,           lse};
  if (int rc = smla::check_decode_call(c)) return rc;
  if (batch == 0) return SMLA_OK;
  if (!workspace || !aligned(workspace, 256)) return SMLA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < smla::workspace_layout(batch, s_q, h_q, num_sm_parts).total) return SMLA_ERR_INVALID_ARGUMENT;
  if (int rc = smla::ensure_decode_kernels()) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return smla::launch_decode(c, ws, reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

int smla_get_mla_metadata_dense(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int causal,
                                int num_sm_parts, int32_t* sched_meta, int32_t* num_splits, int32_t* tile_prefix,
                                void* stream) {
  if (batch < 0 || s_q < 1 || num_sm_parts < 1 || (causal != 0 && causal != 1) || !sched_meta || !num_splits ||
      !tile_prefix || (batch > 0 && !cache_seqlens))
    return SMLA_ERR_INVALID_ARGUMENT;
  if (!valid_h_q(h_q)) return SMLA_ERR_UNSUPPORTED;
  if (!aligned(sched_meta, 16)) return SMLA_ERR_INVALID_ARGUMENT;
  if ((int64_t)batch * s_q > (1 << 28)) return SMLA_ERR_INVALID_ARGUMENT;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1024);
  cfg.stream = static_cast<cudaStream_t>(stream);
  if (const cudaError_t e = cudaLaunchKernelEx(&cfg, smla::sched_meta_dense_kernel, cache_seqlens, batch, s_q, causal,
                                               num_sm_parts, sched_meta, num_splits, tile_prefix);
      e != cudaSuccess)
    return smla::cuda_failure(e);
  return SMLA_OK;
}

int smla_flash_mla_dense_with_kvcache(const void* q, const uint8_t* kvcache, int kv_format, int64_t num_blocks,
                                      const int32_t* block_table, int max_blocks, const int32_t* cache_seqlens,
                                      const int32_t* sched_meta, const int32_t* num_splits,
                                      const int32_t* tile_prefix, int num_sm_parts, float softmax_scale, int causal,
                                      int batch, int s_q, int h_q, void* o, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (kv_format != SMLA_KV_FP8 && kv_format != SMLA_KV_BF16) return SMLA_ERR_INVALID_ARGUMENT;
  smla::DecodeCall c{q,          kvcache, num_blocks, block_table, max_blocks, cache_seqlens,
                     nullptr,    sched_meta, num_splits, num_sm_parts, softmax_scale, batch,
                     s_q,        h_q,     1,          o,           lse};
  c.tile_prefix = tile_prefix;
  c.kv_mode = kv_format == SMLA_KV_BF16 ? smla::kDenseBf16 : smla::kDenseFp8;
  c.causal = causal;
  if (int rc = smla::check_decode_call(c)) return rc;
  if (batch == 0) return SMLA_OK;
  if (!workspace || !aligned(workspace, 256)) return SMLA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < smla::workspace_layout(batch, s_q, h_q, num_sm_parts).total) return SMLA_ERR_INVALID_ARGUMENT;
  if (int rc = smla::ensure_decode_kernels()) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return smla::launch_decode(c, ws, reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

int smla_quantize_kv(const void* latent, const void* rope, int64_t n_tokens, const int64_t* slot_mapping,
                     uint8_t* kvcache, int64_t num_rows, void* stream) {
  if (n_tokens < 0 || num_rows < 0) return SMLA_ERR_INVALID_ARGUMENT;
  if (n_tokens == 0) return SMLA_OK;
  if (!latent || !rope || !kvcache) return SMLA_ERR_INVALID_ARGUMENT;
  if (!aligned(latent, 16) || !aligned(rope, 16) || !aligned(kvcache, 16)) return SMLA_ERR_INVALID_ARGUMENT;
  if (!slot_mapping && n_tokens > num_rows) return SMLA_ERR_INVALID_ARGUMENT;
  const int64_t blocks = (n_tokens + 7) / 8;
  if (blocks > 0x7FFFFFFF) return SMLA_ERR_INVALID_ARGUMENT;
  smla::quantize_kv_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(latent), static_cast<const __nv_bfloat16*>(rope), n_tokens, slot_mapping,
      kvcache, num_rows);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SMLA_OK : smla::cuda_failure(e);
}

int smla_get_device_status(const void* workspace, int* status_out, uint32_t* raw_flags_out, void* stream) {
  if (!workspace || !status_out) return SMLA_ERR_INVALID_ARGUMENT;
  uint32_t flags = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (const cudaError_t e = cudaMemcpyAsync(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost, s);
      e != cudaSuccess)
    return smla::cuda_failure(e);
  if (const cudaError_t e = cudaStreamSynchronize(s); e != cudaSuccess) return smla::cuda_failure(e);
  if (raw_flags_out) *raw_flags_out = flags;
  if (flags & smla::kStatusTimeout) *status_out = SMLA_ERR_DEVICE_TIMEOUT;
  else if (flags & (smla::kStatusBadBlockTable | smla::kStatusBadSchedule)) *status_out = SMLA_ERR_INVALID_ARGUMENT;
  else *status_out = SMLA_OK;
  return SMLA_OK;
}

int smla_reset_device_status(void* workspace, void* stream) {
  if (!workspace) return SMLA_ERR_INVALID_ARGUMENT;
  if (const cudaError_t e = cudaMemsetAsync(workspace, 0, smla::kStatusHeaderBytes, static_cast<cudaStream_t>(stream));
      e != cudaSuccess)
    return smla::cuda_failure(e);
  return SMLA_OK;
}

int smla_selftest_bounded_wait(void* workspace, uint64_t limit_ns, void* stream) {
  if (!workspace || limit_ns < 1 || limit_ns > 10000000000ull) return SMLA_ERR_INVALID_ARGUMENT;
  smla::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace),
                                                                              limit_ns);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SMLA_OK : smla::cuda_failure(e);
}

}  // extern "C"
