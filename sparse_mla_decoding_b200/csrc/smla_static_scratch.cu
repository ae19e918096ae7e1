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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/smla.h"
#include "sm100.cuh"
#include "splitkv_mla.h"

namespace smla {
__global__ void combine_kernel(const int32_t* num_splits, const float* o_accum, const float* lse_accum, int h_q,
                               int max_splits, __nv_bfloat16* o, float* lse);
}  // namespace smla

// The scratch array: a 256-byte header (status word) followed by the split
// partials.  Its size is the stated maximum SMLA_STATIC_SCRATCH_BYTES.
static __device__ __align__(256) uint8_t g_static_scratch[SMLA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kHeader = 256;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};
bool g_smem_set[kMaxDevices] = {false};

// Per-device set-up, done by the first call on each device with that device
// current: look up the device address of the scratch array (host code only
// sees a host-side stand-in for the symbol) and raise the split kernel's
// dynamic shared-memory limit.
int setup_device(int dev, void** scratch_out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return SMLA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  if (!g_smem_set[dev]) {
    if (smla::configure_splitkv() != cudaSuccess) return SMLA_ERR_CUDA;
    g_smem_set[dev] = true;
  }
  *scratch_out = g_scratch_addr[dev];
  return SMLA_OK;
}

}  // namespace

extern "C" int smla_flash_mla_with_kvcache_static_scratch(
    const void* q, const uint8_t* kvcache, int64_t num_blocks, const int32_t* block_table, int max_blocks,
    const int32_t* cache_seqlens, const int32_t* indices, const int32_t* sched_meta, const int32_t* num_splits,
    int num_sm_parts, float softmax_scale, int batch, int s_q, int h_q, int topk, void* o, float* lse,
    uint32_t* status_out, void* stream) {
  if (!(h_q == 16 || h_q == 32 || h_q == 64 || h_q == 128)) return SMLA_ERR_UNSUPPORTED;
  // cache rows are addressed as 32-bit row numbers (block * 64 + offset)
  if (batch < 0 || s_q < 1 || topk < 1 || num_sm_parts < 1 || max_blocks < 1 || num_blocks < 1 ||
      num_blocks > (int64_t)(0x7FFFFFFF / SMLA_BLOCK_SIZE))
    return SMLA_ERR_INVALID_ARGUMENT;
  if (batch == 0) return SMLA_OK;
  if (!q || !kvcache || !block_table || !cache_seqlens || !indices || !sched_meta || !num_splits || !o || !lse)
    return SMLA_ERR_INVALID_ARGUMENT;
  auto aligned = [](const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!aligned(q, 16) || !aligned(kvcache, 16) || !aligned(o, 16) || !aligned(sched_meta, 16) ||
      (status_out && !aligned(status_out, 4)))
    return SMLA_ERR_INVALID_ARGUMENT;
  const int64_t R = (int64_t)batch * s_q;
  const int64_t n_tiles = ((int64_t)topk + SMLA_INDEX_TILE - 1) / SMLA_INDEX_TILE;
  if (R > (1 << 28) || n_tiles > (1 << 24)) return SMLA_ERR_INVALID_ARGUMENT;

  // Scratch need: header + float32 partials for at most R + num_sm_parts splits.
  const size_t max_splits = (size_t)R + (size_t)num_sm_parts;
  const size_t o_bytes = max_splits * (size_t)h_q * SMLA_D_V * sizeof(float);
  const size_t o_off = kHeader;
  const size_t l_off = o_off + ((o_bytes + 255) & ~size_t(255));
  const size_t l_bytes = max_splits * (size_t)h_q * sizeof(float);
  const size_t need = l_off + ((l_bytes + 255) & ~size_t(255));
  if (need > (size_t)SMLA_STATIC_SCRATCH_BYTES) return SMLA_ERR_SCRATCH_LIMIT;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SMLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SMLA_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return SMLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (int rc = setup_device(dev, &scratch)) return rc;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // Nothing in the partials needs to start at zero (every slot read by the
  // combine is written first); the status word does, when it is ours.
  uint32_t* status = status_out;
  if (!status) {
    if (cudaMemsetAsync(ws, 0, kHeader, s) != cudaSuccess) return SMLA_ERR_CUDA;
    status = reinterpret_cast<uint32_t*>(ws);
  }

  float scale = softmax_scale;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)SMLA_D_QK);
  smla::SplitKVParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kv = kvcache;
  p.num_blocks = num_blocks;
  p.block_table = block_table;
  p.max_blocks = max_blocks;
  p.seqlens = cache_seqlens;
  p.indices = indices;
  p.sched_meta = sched_meta;
  p.num_splits = num_splits;
  p.s_q = s_q;
  p.h_q = h_q;
  p.topk = topk;
  p.n_tiles = (int)n_tiles;
  p.num_parts = num_sm_parts;
  p.num_requests = (int)R;
  p.max_splits = (int)max_splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_accum = reinterpret_cast<float*>(ws + o_off);
  p.lse_accum = reinterpret_cast<float*>(ws + l_off);
  p.status = status;

  cudaLaunchAttribute attr;
  std::memset(&attr, 0, sizeof(attr));
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  if (smla::launch_splitkv(p, s) != cudaSuccess) return SMLA_ERR_CUDA;
  cudaLaunchConfig_t ccfg;
  std::memset(&ccfg, 0, sizeof(ccfg));
  ccfg.gridDim = dim3((unsigned)R, h_q);
  ccfg.blockDim = dim3(128);
  ccfg.stream = s;
  ccfg.attrs = &attr;
  ccfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&ccfg, smla::combine_kernel, (const int32_t*)num_splits, (const float*)p.o_accum,
                         (const float*)p.lse_accum, h_q, p.max_splits, p.o, lse) != cudaSuccess)
    return SMLA_ERR_CUDA;
  return SMLA_OK;
}
