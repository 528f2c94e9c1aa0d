// Boundary-state path that allocates nothing and takes no workspace.
//
// Some callers cannot allocate device memory at all: code running under a
// host framework that owns every device allocation and gives the library no
// allocator, plugins loaded into a process whose memory pools are already
// reserved, or hot paths that must never call cudaMalloc (it can synchronise
// the device and is not allowed while a stream is being captured).  For them,
// vdn_vda_boundary_states_noalloc runs the same kernels as
// vdn_vda_boundary_states with its scratch in a fixed device array compiled
// into this library, so the caller passes only inputs and outputs.
//
// The array is VDN_NOALLOC_SCRATCH_BYTES large; every GPU that loads the
// library holds it until the process exits.  All calls share it: calls that
// overlap on the GPU (different streams or threads without ordering) race on
// it.  Its first bytes hold the device status word of the last call (cleared
// when each call starts; read it with vdn_noalloc_device_status); every other
// byte the path reads is written first by the same call.
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {
size_t vda_scratch_bytes(const vdn_params& p);
vdn_status boundary_states_impl(const vdn_params* p, const void* k, const void* v,
                                const float* beta, const float* alpha, const void* text_k,
                                const void* text_v, float* F, float* G, void* workspace,
                                vdn_stream_t stream);

static __device__ __align__(256) unsigned char g_noalloc_scratch[VDN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device (the host-side
// name is only a stand-in, not a device pointer).  Looked up on every call,
// with the caller's device current, so that a context torn down and made
// again (cudaDeviceReset) never leaves a stale address behind; the lookup is a
// table read once the library's module is loaded on that device.
static void* scratch_address(vdn_status* err) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    *err = VDN_ERR_CUDA;
    return nullptr;
  }
  *err = VDN_OK;
  return p;
}
}  // namespace vdn

extern "C" vdn_status vdn_vda_boundary_states_noalloc(const vdn_params* p, const void* k,
                                                      const void* v, const float* beta,
                                                      const float* alpha, const void* text_k,
                                                      const void* text_v, float* F, float* G,
                                                      vdn_stream_t stream) {
  size_t need = 0;
  const vdn_status vs = vdn_workspace_bytes(p, &need);  // validates p
  if (vs != VDN_OK) return vs;
  if (vdn::vda_scratch_bytes(*p) > (size_t)VDN_NOALLOC_SCRATCH_BYTES) return VDN_ERR_WORKSPACE;
  vdn_status err = VDN_OK;
  void* scratch = vdn::scratch_address(&err);
  if (scratch == nullptr) return err;
  return vdn::boundary_states_impl(p, k, v, beta, alpha, text_k, text_v, F, G, scratch, stream);
}

extern "C" vdn_status vdn_noalloc_device_status(vdn_stream_t stream) {
  vdn_status err = VDN_OK;
  void* scratch = vdn::scratch_address(&err);
  if (scratch == nullptr) return err;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return VDN_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return VDN_ERR_CUDA;
  if (cudaMemset(scratch, 0, sizeof(int)) != cudaSuccess) return VDN_ERR_CUDA;
  if (word & vdn::kDevTimeout) return VDN_ERR_TIMEOUT;
  if (word & vdn::kDevRange) return VDN_ERR_RANGE;
  return VDN_OK;
}
