// minf_estimate_vs_noalloc: Vertical-Slash index estimation for callers that
// must not allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they run this step: code that executes while a stream is being
// captured into a CUDA graph under a capture mode that forbids allocation,
// engine plugins whose enqueue path must not allocate because the runtime
// planned all device memory ahead of time, and latency-critical services
// that must not take the device-wide synchronisation an allocation can cause.
// They still pass their own inputs and outputs; the scratch space the
// estimation needs comes from the fixed array below instead of a workspace.
//
// The array is a file-scope device variable of kNoAllocScratchBytes, so every
// GPU on which the library's module is loaded keeps it for the life of the
// process.  In host code its name is only a host-side stand-in for the device
// variable; every call fetches the device address with cudaGetSymbolAddress
// (while the device is current), which allocates nothing.  The first call on
// a device loads the module, so it should be made before any stream capture
// starts.  All calls share the array and it keeps the last call's contents:
// the status word at its head is cleared on every call (and by
// minf_noalloc_device_status, which reads it), the rest is fully rewritten
// before it is read.  Calls whose executions overlap on the GPU (different
// streams, or different host threads) race on the array; serialise them.

#include "minf_device.cuh"
#include "minf_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;  // 64 MiB

__device__ __align__(256) unsigned char g_vs_scratch[kNoAllocScratchBytes];

// Device address of g_vs_scratch on the current device.  Looked up on every
// call (a lookup allocates nothing), so that the address follows a reloaded
// module after cudaDeviceReset.
minf_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_vs_scratch) != cudaSuccess || p == nullptr) return MINF_ERR_CUDA;
  *out = p;
  return MINF_OK;
}

}  // namespace

extern "C" minf_status minf_estimate_vs_noalloc(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                                const int32_t* heads, int nh, int last_q, int k_v, int k_s,
                                                int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score,
                                                void* stream) {
  const size_t need = minf_workspace_size(MINF_OP_ESTIMATE_VS, shape, nh, k_v, k_s, 0);
  if (need == 0) return MINF_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return MINF_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  minf_status st = scratch_address(&scratch);
  if (st != MINF_OK) return st;
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return MINF_ERR_CUDA;
  return minf_estimate_vs(shape, Q, K, heads, nh, last_q, k_v, k_s, v_idx, s_idx, v_score, s_score, scratch,
                          kNoAllocScratchBytes, stream);
}

extern "C" minf_status minf_noalloc_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MINF_ERR_CUDA;
  int code = 0;  // the status block's first word: the first error code recorded
  if (cudaMemcpyFromSymbol(&code, g_vs_scratch, sizeof(code), 0, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MINF_ERR_CUDA;
  const int zero[2] = {0, 0};  // code and site
  if (code != 0 && cudaMemcpyToSymbol(g_vs_scratch, zero, sizeof(zero), 0, cudaMemcpyHostToDevice) != cudaSuccess)
    return MINF_ERR_CUDA;
  return (minf_status)code;
}
