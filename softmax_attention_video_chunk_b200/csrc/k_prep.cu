// VDA-Prep: the linear branch's feature map of the raw Q, K, V projections.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method (the linear branch applies its own feature map: a
// separable short convolution of K and V -- a depthwise spatial filter and a
// five-tap temporal filter -- then SiLU, with L2 normalisation of Q and K) and
// implementation ("Fused VDA kernels": one pass does the convolution, SiLU, L2
// normalisation and the store in the layout the statistics read).
//
//   k_l = L2(SiLU(conv_t(conv_s(k)))),  v_l = SiLU(conv_t(conv_s(v))),
//   q_l = L2(q),   L2(x) = x / sqrt(sum_d x^2 + eps);
// conv_s: depthwise 3x3 over the frame's row-major grid_h x grid_w token grid,
// conv_t: depthwise 5 taps over frames t-2..t+2, both cross-correlations with
// zero padding.
//
// prep_conv_kernel: HBM-bound, every input element is read from DRAM once and
// every output written once.  One CTA owns a segment of 24 grid columns of
// one grid row, one head and one tensor (K or V) and walks the frames in order:
//   - thread 0 brings each frame's 3-row x 26-column x d-channel halo tile into
//     a ring of shared-memory stages by TMA (rows and columns outside the grid
//     arrive as zeros, which is the spatial padding);
//   - warp w owns 3 consecutive columns, lane l owns channels l*d/32 ..; the
//     spatial filter runs from shared memory, and the temporal filter runs on
//     a 5-frame window of spatial results kept in registers (frames outside
//     the clip are zeros), so no intermediate leaves the SM;
//   - SiLU, then for K the L2 norm over the head's d channels, which is one
//     warp-wide sum (a warp holds exactly one head).
// Waits on the TMA barriers are bounded; on expiry the CTA records
// VDN_ERR_TIMEOUT, all threads leave together, and thread 0 waits (bounded)
// for its copies in flight before the CTA exits.
//
// prep_l2_kernel: q_l = L2(q), one warp per (token, head) row.
#include <cuda_bf16.h>

#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

bool make_tmap_plain(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

namespace {

constexpr int kWarps = 8;
constexpr int kPos = 3;                // grid columns per warp
constexpr int kSeg = kWarps * kPos;    // grid columns per CTA
constexpr int kCols = kSeg + 2;        // with the left and right halo
constexpr int kTaps = 5;               // temporal taps

template <typename E, int CPL>
__device__ __forceinline__ void load_ch(const E* p, float (&x)[CPL]);
template <>
__device__ __forceinline__ void load_ch<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
template <>
__device__ __forceinline__ void load_ch<__nv_bfloat16, 2>(const __nv_bfloat16* p, float (&x)[2]) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  x[0] = a.x; x[1] = a.y;
}
template <>
__device__ __forceinline__ void load_ch<__nv_bfloat16, 1>(const __nv_bfloat16* p, float (&x)[1]) {
  x[0] = __bfloat162float(*p);
}
template <>
__device__ __forceinline__ void load_ch<float, 4>(const float* p, float (&x)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void load_ch<float, 2>(const float* p, float (&x)[2]) {
  const float2 a = *reinterpret_cast<const float2*>(p);
  x[0] = a.x; x[1] = a.y;
}
template <>
__device__ __forceinline__ void load_ch<float, 1>(const float* p, float (&x)[1]) {
  x[0] = *p;
}

template <typename E, int CPL>
__device__ __forceinline__ void store_ch(E* p, const float (&x)[CPL]);
template <>
__device__ __forceinline__ void store_ch<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&x)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
template <>
__device__ __forceinline__ void store_ch<__nv_bfloat16, 2>(__nv_bfloat16* p, const float (&x)[2]) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_ch<__nv_bfloat16, 1>(__nv_bfloat16* p, const float (&x)[1]) {
  *p = __float2bfloat16_rn(x[0]);
}
template <>
__device__ __forceinline__ void store_ch<float, 4>(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <>
__device__ __forceinline__ void store_ch<float, 2>(float* p, const float (&x)[2]) {
  *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_ch<float, 1>(float* p, const float (&x)[1]) {
  *p = x[0];
}

__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

template <int CPL>
__device__ __forceinline__ float warp_sum_sq(const float (&x)[CPL]) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < CPL; ++c) s = fmaf(x[c], x[c], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

}  // namespace

// grid: (ceil(grid_w / 24), grid_h, B * H * 2); z = ((b * H + h) * 2 + which),
// which 0: K (L2 after SiLU), 1: V.
template <typename E, int D, int NS>
__global__ void __launch_bounds__(256, 1)
prep_conv_kernel(const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const float* __restrict__ wk_s,
                 const float* __restrict__ wk_t, const float* __restrict__ wv_s,
                 const float* __restrict__ wv_t, E* __restrict__ k_out, E* __restrict__ v_out,
                 int H, int T, int gh, int gw, float eps, int* __restrict__ status) {
  constexpr int CPL = D / 32;
  constexpr int STAGE = 3 * kCols * D;  // elements of one halo tile
  constexpr int STAGE_BYTES = STAGE * (int)sizeof(E);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  E* tiles = reinterpret_cast<E*>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + NS * STAGE_BYTES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + NS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int x0 = blockIdx.x * kSeg, y = blockIdx.y;
  const int which = blockIdx.z & 1, bh = blockIdx.z >> 1;
  const int b = bh / H, h = bh % H;
  const CUtensorMap* map = which ? &map_v : &map_k;
  const float* ws = which ? wv_s : wk_s;
  const float* wt = which ? wv_t : wk_t;
  E* out = which ? v_out : k_out;
  const size_t N = (size_t)gh * gw;

  // this lane's channels of head h: c = h * D + lane * CPL + i
  float wsp[9][CPL], wtp[kTaps][CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const size_t c = (size_t)h * D + lane * CPL + i;
#pragma unroll
    for (int j = 0; j < 9; ++j) wsp[j][i] = __ldg(ws + c * 9 + j);
#pragma unroll
    for (int j = 0; j < kTaps; ++j) wtp[j][i] = __ldg(wt + c * kTaps + j);
  }

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) ptx::mbar_init(full + s, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  int issued = 0;  // thread 0 only
  if (tid == 0) {
    for (; issued < NS && issued < T; ++issued) {
      ptx::mbar_arrive_expect_tx(full + issued, STAGE_BYTES);
      ptx::tma_load_5d(tiles + issued * STAGE, map, full + issued, 0, h, x0 - 1, y - 1,
                       b * T + issued);
    }
  }

  // ring[f] = spatial result of frame j - 4 + f (f = 0..3); frames outside
  // the clip are zeros
  float ring[4][kPos][CPL];
#pragma unroll
  for (int f = 0; f < 4; ++f)
#pragma unroll
    for (int p = 0; p < kPos; ++p)
#pragma unroll
      for (int i = 0; i < CPL; ++i) ring[f][p][i] = 0.f;

  for (int j = 0; j < T + 2; ++j) {
    bool ok = true;
    if (j < T)
      ok = ptx::wait_bounded(full + j % NS, (j / NS) & 1, abort_flag, status, kDevTimeout);
    // every thread is done with frame j - 1: its stage may be refilled
    if (!__syncthreads_and(ok)) break;
    if (tid == 0 && j >= 1 && issued < T) {
      const int s = issued % NS;
      ptx::mbar_arrive_expect_tx(full + s, STAGE_BYTES);
      ptx::tma_load_5d(tiles + s * STAGE, map, full + s, 0, h, x0 - 1, y - 1, b * T + issued);
      ++issued;
    }
    float cur[kPos][CPL];
#pragma unroll
    for (int p = 0; p < kPos; ++p)
#pragma unroll
      for (int i = 0; i < CPL; ++i) cur[p][i] = 0.f;
    if (j < T) {
      const E* tile = tiles + (j % NS) * STAGE + lane * CPL;
#pragma unroll
      for (int r = 0; r < 3; ++r) {
#pragma unroll
        for (int cc = 0; cc < kPos + 2; ++cc) {  // tile columns warp*kPos + cc
          float xv[CPL];
          load_ch<E, CPL>(tile + (r * kCols + warp * kPos + cc) * D, xv);
#pragma unroll
          for (int p = 0; p < kPos; ++p) {
            const int dx = cc - p;  // filter column 0..2
            if (dx >= 0 && dx < 3) {
#pragma unroll
              for (int i = 0; i < CPL; ++i) cur[p][i] = fmaf(wsp[r * 3 + dx][i], xv[i], cur[p][i]);
            }
          }
        }
      }
    }
    const int t = j - 2;  // output frame
    if (t >= 0) {
#pragma unroll
      for (int p = 0; p < kPos; ++p) {
        float o[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
          float a = wtp[4][i] * cur[p][i];
          a = fmaf(wtp[3][i], ring[3][p][i], a);
          a = fmaf(wtp[2][i], ring[2][p][i], a);
          a = fmaf(wtp[1][i], ring[1][p][i], a);
          a = fmaf(wtp[0][i], ring[0][p][i], a);
          o[i] = silu(a);
        }
        if (which == 0) {
          const float rs = rsqrtf(warp_sum_sq<CPL>(o) + eps);
#pragma unroll
          for (int i = 0; i < CPL; ++i) o[i] *= rs;
        }
        const int x = x0 + warp * kPos + p;
        if (x < gw) {
          const size_t tok = (size_t)t * N + (size_t)y * gw + x;
          store_ch<E, CPL>(out + (((size_t)b * T * N + tok) * H + h) * D + lane * CPL, o);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < kPos; ++p)
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        ring[0][p][i] = ring[1][p][i];
        ring[1][p][i] = ring[2][p][i];
        ring[2][p][i] = ring[3][p][i];
        ring[3][p][i] = cur[p][i];
      }
  }
  if (tid == 0 && *abort_flag) {  // copies still in flight must land first
    const uint64_t t0 = ptx::globaltimer_ns();
    for (int f = issued > NS ? issued - NS : 0; f < issued; ++f)
      while (!ptx::mbar_try_wait(full + f % NS, (f / NS) & 1) &&
             ptx::globaltimer_ns() - t0 < 2000000000ull) {}
  }
}

// q_l = L2(q): one warp per (token, head) row of D channels.
template <typename E, int D>
__global__ void __launch_bounds__(256)
prep_l2_kernel(const E* __restrict__ q, E* __restrict__ q_out, size_t rows, float eps) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  const size_t nwarps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += nwarps) {
    float x[CPL];
    load_ch<E, CPL>(q + r * D + lane * CPL, x);
    const float rs = rsqrtf(warp_sum_sq<CPL>(x) + eps);
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] *= rs;
    store_ch<E, CPL>(q_out + r * D + lane * CPL, x);
  }
}

int sm_count();

template <typename E, int D>
static cudaError_t launch_prep_t(const PrepArgs& a, cudaStream_t st) {
  constexpr int NS = sizeof(E) == 2 ? 4 : 3;
  constexpr size_t STAGE_BYTES = 3ull * kCols * D * sizeof(E);
  const CUtensorMapDataType dt =
      sizeof(E) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const size_t es = sizeof(E);
  if (a.k != nullptr) {
    // dims (d, H, grid_w, grid_h, B*T); box: one head, 26 columns, 3 rows, 1 frame
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.gw, (uint64_t)a.gh,
                              (uint64_t)a.B * a.T};
    const uint64_t strides[4] = {D * es, (uint64_t)a.H * D * es, (uint64_t)a.gw * a.H * D * es,
                                 (uint64_t)a.gh * a.gw * a.H * D * es};
    const uint32_t box[5] = {(uint32_t)D, 1u, (uint32_t)kCols, 3u, 1u};
    CUtensorMap mk, mv;
    if (!make_tmap_plain(&mk, dt, 5, a.k, dims, strides, box) ||
        !make_tmap_plain(&mv, dt, 5, a.v, dims, strides, box))
      return cudaErrorInvalidValue;
    const size_t sm = NS * STAGE_BYTES + NS * 8 + 16;
    auto kern = prep_conv_kernel<E, D, NS>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.gw + kSeg - 1) / kSeg, a.gh, a.B * a.H * 2);
    kern<<<grid, 256, sm, st>>>(mk, mv, a.wk_s, a.wk_t, a.wv_s, a.wv_t, (E*)a.k_out,
                                (E*)a.v_out, a.H, a.T, a.gh, a.gw, a.eps, a.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.q != nullptr) {
    const size_t rows = (size_t)a.B * a.T * a.gh * a.gw * a.H;
    const size_t want = (rows + 7) / 8;
    const int blocks = (int)(want < (size_t)sm_count() * 8 ? want : (size_t)sm_count() * 8);
    prep_l2_kernel<E, D><<<blocks, 256, 0, st>>>((const E*)a.q, (E*)a.q_out, rows, a.eps);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  if (a.bf16) {
    if (a.D == 128) return launch_prep_t<__nv_bfloat16, 128>(a, st);
    if (a.D == 64) return launch_prep_t<__nv_bfloat16, 64>(a, st);
    if (a.D == 32) return launch_prep_t<__nv_bfloat16, 32>(a, st);
  } else {
    if (a.D == 128) return launch_prep_t<float, 128>(a, st);
    if (a.D == 64) return launch_prep_t<float, 64>(a, st);
    if (a.D == 32) return launch_prep_t<float, 32>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
