// Fault-free check of the bounded-wait path that every pipelined kernel uses.
//
// The tensor-core kernels never spin on an mbarrier without a time limit: a
// wait that runs past its limit raises the CTA's abort flag, records
// kDevTimeout in the caller's device status word and returns, and every other
// waiter of the CTA leaves through the abort flag; the CTA then frees its TMEM
// and exits.  This kernel runs exactly that sequence on a barrier that nothing
// ever arrives at, so the expiry, the status word, the flag hand-off and the
// TMEM release can be tested on a GPU without a hang or a fault:
//   warp 1        allocates 32 TMEM columns (as the real kernels do);
//   thread 0      waits with the caller's limit  -> expires, sets the flag;
//   lane 0 of the other warps wait with twice the limit -> leave on the flag;
//   all           barrier, then warp 1 frees the TMEM columns.
#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

__global__ void __launch_bounds__(128, 1)
selftest_wait_kernel(int* __restrict__ status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);  // expects one arrival that never comes
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_slot, 32);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0)
    ptx::wait_bounded(&bar, 0, &abort_flag, status, kDevTimeout, limit_ns);
  else if (lane == 0)
    ptx::wait_bounded(&bar, 0, &abort_flag, status, kDevTimeout, 2 * limit_ns);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 32);
  }
}

// y = 2^x through the FMA-pipe polynomial exponential the Softmax kernel
// uses for a share of its P values (ptx::exp2_poly2), two lanes at a time.
__global__ void __launch_bounds__(256) selftest_exp2_kernel(const float* __restrict__ x,
                                                            float* __restrict__ y, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x * 2;
  for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float y0, y1;
    ptx::f2_unpack(ptx::exp2_poly2(ptx::f2_pack(x0, x1)), y0, y1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
  }
}

}  // namespace vdn

extern "C" {

vdn_status vdn_selftest_exp2(const float* x, float* y, size_t n, vdn_stream_t stream) {
  if (x == nullptr || y == nullptr) return VDN_ERR_INVALID_ARG;
  if (n == 0) return VDN_OK;
  const size_t blocks = (n + 511) / 512;
  vdn::selftest_exp2_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0,
                              (cudaStream_t)stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

vdn_status vdn_selftest_bounded_wait(void* workspace, unsigned int limit_us,
                                     vdn_stream_t stream) {
  if (workspace == nullptr) return VDN_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return VDN_ERR_ALIGNMENT;
  if (limit_us < 100u || limit_us > 1000000u) return VDN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  int* status = (int*)workspace;
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return VDN_ERR_CUDA;
  vdn::selftest_wait_kernel<<<1, 128, 0, st>>>(status, 1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

}  // extern "C"
