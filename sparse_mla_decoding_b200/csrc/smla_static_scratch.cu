// smla_static_scratch.cu -- an allocation-free variant of the sparse MLA decode
// entry point, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) around the
// decode: allocator-less runtimes and embedders that hand the library only
// their input and output buffers, code running where a device allocation
// would synchronise or is forbidden, and hosts whose memory planner owns every
// device byte.  smla_flash_mla_with_kvcache needs a caller-provided workspace
// for the split-KV partials; this variant instead keeps that scratch in a
// fixed-size array in the library's own device memory (a file-scope
// `static __device__` array: the driver places it when the module loads, and
// every GPU that loads the library holds it until the process exits).
//
// The kernels are the same as the ones smla_flash_mla_with_kvcache launches;
// only the scratch pointer differs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/smla.h"
#include "splitkv_mla.h"

// The scratch array: a 256-byte header (status word) followed by the split
// partials.  Its size is the stated maximum SMLA_STATIC_SCRATCH_BYTES.
static __device__ __align__(256) uint8_t g_static_scratch[SMLA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ctx[kMaxDevices] = {nullptr};
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Set-up, once per device (and again if the device's context was re-created,
// e.g. after cudaDeviceReset, which loads the module anew): in host code
// g_static_scratch names a host-side stand-in, not device memory, so with the
// device current look up the array's device address and keep it.
int scratch_address(void** out) {
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return smla::cuda_failure(e);
  if (dev < 0 || dev >= kMaxDevices) return SMLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  void* ctx = smla::current_context();
  if (ctx == nullptr || ctx != g_scratch_ctx[dev] || g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch); e != cudaSuccess)
      return smla::cuda_failure(e);
    if (ptr == nullptr) return smla::cuda_failure(cudaErrorInvalidSymbol);
    g_scratch_addr[dev] = ptr;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return SMLA_OK;
}

}  // namespace

extern "C" int smla_flash_mla_with_kvcache_static_scratch(
    const void* q, const uint8_t* kvcache, int64_t num_blocks, const int32_t* block_table, int max_blocks,
    const int32_t* cache_seqlens, const int32_t* indices, const int32_t* sched_meta, const int32_t* num_splits,
    int num_sm_parts, float softmax_scale, int batch, int s_q, int h_q, int topk, void* o, float* lse,
    uint32_t* status_out, void* stream) {
  const smla::DecodeCall c{q,       kvcache,    num_blocks, block_table,  max_blocks,    cache_seqlens,
                           indices, sched_meta, num_splits, num_sm_parts, softmax_scale, batch,
                           s_q,     h_q,        topk,       o,            lse};
  if (int rc = smla::check_decode_call(c)) return rc;
  if (batch == 0) return SMLA_OK;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) % 4) != 0) return SMLA_ERR_INVALID_ARGUMENT;
  // The scratch need is exactly the regular entry point's workspace size.
  if (smla::workspace_layout(batch, s_q, h_q, num_sm_parts).total > (size_t)SMLA_STATIC_SCRATCH_BYTES)
    return SMLA_ERR_SCRATCH_LIMIT;
  if (int rc = smla::ensure_decode_kernels()) return rc;

  void* scratch = nullptr;
  if (int rc = scratch_address(&scratch)) return rc;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Nothing in the partials needs to start at zero (every slot the combine
  // reads is written first); the status word does when it is the library's.
  uint32_t* status = status_out;
  if (!status) {
    if (const cudaError_t e = cudaMemsetAsync(ws, 0, smla::kStatusHeaderBytes, st); e != cudaSuccess) return smla::cuda_failure(e);
    status = reinterpret_cast<uint32_t*>(ws);
  }
  return smla::launch_decode(c, ws, status, st);
}
