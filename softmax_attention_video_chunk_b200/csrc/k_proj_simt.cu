// Gated dual output projection on CUDA cores, exact FP32 arithmetic.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method, the paragraph on the two output gates: the Softmax
// readout passes its sigmoid gate, the linear readout is RMS-normalised and
// passes its own sigmoid gate, each branch has its own output projection and
// the two projections are added:
//   out = concat_h(g_s * o_s) W_soft + concat_h(g_l * o_l / rms(o_l)) W_lin.
// Written as one GEMM with K = 2 * H * d over the concatenated, gated rows;
// the gates and the RMS factor are applied while the A tile is loaded.
#include <math.h>

#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

// rinv[row, h] = 1 / sqrt(mean_c o_l[row, h, c]^2 + eps); one warp per (row, h).
__global__ void rms_inv_kernel(const float* __restrict__ o_l, float* __restrict__ rinv,
                               size_t nrows, int D, float eps) {
  const size_t warp = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= nrows) return;
  const float* p = o_l + warp * D;
  float s = 0.f;
  for (int c = lane; c < D; c += 32) s = fmaf(p[c], p[c], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) rinv[warp] = 1.f / sqrtf(s / (float)D + eps);
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256)
proj_simt_kernel(const float* __restrict__ o_s, const float* __restrict__ o_l,
                 const TIn* __restrict__ gates, const float* __restrict__ rinv,
                 const TIn* __restrict__ Ws, const TIn* __restrict__ Wl,
                 TOut* __restrict__ out, size_t M, int Din, int Dout, int D) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const size_t m0 = (size_t)blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  const int K = 2 * Din;
  const TIn* gs = gates;
  const TIn* gl = gates + M * (size_t)Din;
  const int H = Din / D;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    __syncthreads();
    for (int e = tid; e < BM * BK; e += 256) {
      const int mm = e / BK, kk = e % BK;
      const size_t m = m0 + mm;
      const int kg = k0 + kk;
      float a = 0.f;
      if (m < M) {
        if (kg < Din) {
          a = to_f(gs[m * Din + kg]) * o_s[m * Din + kg];
        } else {
          const int k2 = kg - Din;
          a = to_f(gl[m * Din + k2]) * o_l[m * Din + k2] * rinv[m * H + k2 / D];
        }
      }
      As[kk][mm] = a;
    }
    for (int e = tid; e < BK * BN; e += 256) {
      const int kk = e / BN, nn = e % BN;
      const int kg = k0 + kk, n = n0 + nn;
      float w = 0.f;
      if (n < Dout) w = kg < Din ? to_f(Ws[(size_t)kg * Dout + n]) : to_f(Wl[(size_t)(kg - Din) * Dout + n]);
      Bs[kk][nn] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const size_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < Dout) out[m * Dout + n] = from_f<TOut>(acc[i][j]);
    }
  }
}

template <typename TIn, typename TOut>
static cudaError_t launch_proj_t(const ProjArgs& a, cudaStream_t st) {
  const size_t M = (size_t)a.B * a.L;
  const int Din = a.H * a.D;
  proj_simt_kernel<TIn, TOut><<<dim3((unsigned)((M + 63) / 64), (a.D_out + 63) / 64), 256, 0, st>>>(
      a.o_s, a.o_l, (const TIn*)a.gates, a.rinv, (const TIn*)a.W_soft, (const TIn*)a.W_lin,
      (TOut*)a.out, M, Din, a.D_out, a.D);
  return cudaGetLastError();
}

cudaError_t launch_rms_inv(const float* o_l, float* rinv, size_t rows, int D, float eps,
                           cudaStream_t st) {
  const size_t threads = rows * 32;
  rms_inv_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(o_l, rinv, rows, D, eps);
  return cudaGetLastError();
}

cudaError_t launch_proj_simt(const ProjArgs& a, cudaStream_t st) {
  cudaError_t e = launch_rms_inv(a.o_l, a.rinv, (size_t)a.B * a.L * a.H, a.D, a.eps, st);
  if (e != cudaSuccess) return e;
  const bool bf = a.dtype == VDN_BF16, obf = a.out_dtype == VDN_BF16;
  if (bf) return obf ? launch_proj_t<__nv_bfloat16, __nv_bfloat16>(a, st)
                     : launch_proj_t<__nv_bfloat16, float>(a, st);
  return obf ? launch_proj_t<float, __nv_bfloat16>(a, st) : launch_proj_t<float, float>(a, st);
}

}  // namespace vdn
