// The hybrid attention core for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) at
// the point where they run the core: code that runs inside another
// framework's memory pool, hard real-time or certified runtimes that forbid
// allocation after start-up, and plug-ins handed only the input and output
// buffers.  For them this file keeps the core's scratch in a fixed device
// array that the library owns, so the caller passes inputs and outputs only.
//
// The array has static storage on every GPU that loads the library and stays
// allocated until the process exits.  All calls share it and it keeps the
// previous call's contents: the status words are cleared by every call and
// every other scratch region is fully written before it is read.  Calls whose
// kernels overlap on the GPU (two streams, two host threads, two devices'
// worth of work aimed at one device) race on the array; serialise them.
#include "vdn_internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = VDN_NOALLOC_SCRATCH_BYTES;  // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the array in the current device's context.  In host code
// `g_noalloc_scratch` names a host-side stand-in, not device memory, so only
// this address may be given to a kernel.  It is looked up on every call
// rather than cached: after a device reset (or any teardown of the primary
// context) the module is loaded again and the array can move, and a cached
// address would then point at memory the library no longer owns.
vdn_status scratch_for_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return VDN_ERR_CUDA;
  *out = p;
  return VDN_OK;
}

}  // namespace

extern "C" vdn_status vdn_hybrid_attn_fwd_noalloc(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args,
                                                  vdn_stream_t stream) {
  if (!cfg || !args) return VDN_ERR_INVALID_ARG;
  if (args->workspace || args->workspace_bytes) return VDN_ERR_INVALID_ARG;
  const size_t need = vdn_hybrid_attn_workspace_size(cfg);
  if (need == 0) {
    vdn_workspace_layout tmp;
    return vdn_hybrid_workspace_layout(cfg, &tmp);  // the configuration's own error
  }
  if (need > kNoallocScratchBytes) return VDN_ERR_WORKSPACE;
  void* scratch = nullptr;
  vdn_status st = scratch_for_current_device(&scratch);
  if (st != VDN_OK) return st;
  vdn_hybrid_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = kNoallocScratchBytes;
  return vdn_hybrid_attn_fwd(cfg, &a, stream);
}

extern "C" vdn_status vdn_hybrid_noalloc_device_status(vdn_stream_t stream, unsigned* where) {
  void* scratch = nullptr;
  vdn_status st = scratch_for_current_device(&scratch);
  if (st != VDN_OK) return st;
  // the status words lead the workspace layout of every configuration
  uint32_t host[2] = {0, 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host, scratch, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return VDN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VDN_ERR_CUDA;
  if (where) *where = host[1];
  return host[0] ? VDN_ERR_TIMEOUT : VDN_OK;
}
