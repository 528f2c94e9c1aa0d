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
// every output written once.  One CTA owns a segment of 16 grid columns of
// one grid row, one head and one tensor (K or V) and walks the frames in order:
//   - each frame's 3-row x 18-column x d-channel halo tile comes into a ring of
//     shared-memory stages by TMA (rows and columns outside the grid arrive as
//     zeros, which is the spatial padding); one CTA barrier per frame tells
//     thread 0 that the previous frame's stage is free for the frame NS ahead;
//   - warp w owns 2 consecutive columns, lane l owns channels l*d/32 .. as
//     packed FP32 pairs (fma.rn.f32x2); the spatial filter reads the tile, and
//     the temporal filter adds each frame's spatial result into the running
//     sums of the 5 output frames it feeds (registers; the frame loop is
//     unrolled by 5 so the slots are fixed), so no intermediate leaves the SM;
//   - SiLU, then for K the L2 norm over the head's d channels, which is one
//     warp-wide sum (a warp holds exactly one head).
// Waits on the TMA barriers are bounded; on expiry the CTA records
// VDN_ERR_TIMEOUT, the per-frame barrier takes every thread out of the loop
// together, and thread 0 waits (bounded) for the copies still in flight.
//
// prep_l2_kernel: q_l = L2(q), one warp per (token, head) row.
#include <cuda_bf16.h>

#include <type_traits>

#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

bool make_tmap_plain(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

namespace {

constexpr int kWarps = 8;
constexpr int kTaps = 5;  // temporal taps
#ifndef VDN_PREP_POS
#define VDN_PREP_POS 2
#endif
constexpr int kPos = VDN_PREP_POS;  // grid columns per warp

// A lane's CPL channels as packed FP32 pairs (fma.rn.f32x2); for CPL = 1 the
// upper half of the single pair is unused.
template <int CPL>
struct Lane {
  static constexpr int NP = (CPL + 1) / 2;
  uint64_t p[NP];
};

__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  // bf16 -> fp32 is exact: the bf16 bits are the upper half of the fp32 bits
  return ptx::f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <typename E, int CPL>
__device__ __forceinline__ void load_lane(const E* p, Lane<CPL>& x) {
  if constexpr (sizeof(E) == 2) {
    if constexpr (CPL == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      x.p[0] = bf2_to_f2(u.x);
      x.p[1] = bf2_to_f2(u.y);
    } else if constexpr (CPL == 2) {
      x.p[0] = bf2_to_f2(*reinterpret_cast<const uint32_t*>(p));
    } else {
      const uint32_t w = *reinterpret_cast<const unsigned short*>(p);
      x.p[0] = ptx::f2_pack(__uint_as_float(w << 16), 0.f);
    }
  } else {
    if constexpr (CPL == 4) {
      const float4 a = *reinterpret_cast<const float4*>(p);
      x.p[0] = ptx::f2_pack(a.x, a.y);
      x.p[1] = ptx::f2_pack(a.z, a.w);
    } else if constexpr (CPL == 2) {
      const float2 a = *reinterpret_cast<const float2*>(p);
      x.p[0] = ptx::f2_pack(a.x, a.y);
    } else {
      x.p[0] = ptx::f2_pack(*reinterpret_cast<const float*>(p), 0.f);
    }
  }
}

template <typename E, int CPL>
__device__ __forceinline__ void store_lane(E* p, const float (&x)[2 * Lane<CPL>::NP]) {
  if constexpr (sizeof(E) == 2) {
    if constexpr (CPL == 4) {
      __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
      __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&a);
      u.y = *reinterpret_cast<uint32_t*>(&b);
      *reinterpret_cast<uint2*>(p) = u;
    } else if constexpr (CPL == 2) {
      *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x[0], x[1]);
    } else {
      *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x[0]);
    }
  } else {
    if constexpr (CPL == 4) {
      *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (CPL == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
      *reinterpret_cast<float*>(p) = x[0];
    }
  }
}

__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

__device__ __forceinline__ float warp_sum(float s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// q_l rows: plain float arrays of CPL channels
template <typename E, int CPL>
__device__ __forceinline__ void load_ch(const E* p, float (&x)[CPL]) {
  Lane<CPL> l;
  load_lane<E, CPL>(p, l);
  float y[2 * Lane<CPL>::NP];
#pragma unroll
  for (int i = 0; i < Lane<CPL>::NP; ++i) ptx::f2_unpack(l.p[i], y[2 * i], y[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < CPL; ++i) x[i] = y[i];
}

}  // namespace

// Shared state of one prep_conv_kernel CTA besides the tile ring.
template <int NS>
struct PrepSync {
  uint64_t full[NS];  // TMA landed
  int issued;         // frames issued so far
  int abort_flag;
};

// grid: (ceil(grid_w / (8 * kPos)), grid_h, B * H * 2); z = ((b * H + h) * 2 + which),
// which 0: K (L2 after SiLU), 1: V.
template <typename E, int D, int NS>
__global__ void __launch_bounds__(256, kPos <= 2 ? 2 : 1)
prep_conv_kernel(const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const float* __restrict__ wk_s,
                 const float* __restrict__ wk_t, const float* __restrict__ wv_s,
                 const float* __restrict__ wv_t, E* __restrict__ k_out, E* __restrict__ v_out,
                 int H, int T, int gh, int gw, float eps, int* __restrict__ status) {
  constexpr int CPL = D / 32;
  constexpr int NP = Lane<CPL>::NP;
  constexpr int kCols = kWarps * kPos + 2;  // CTA columns with the left and right halo
  constexpr int STAGE = 3 * kCols * D;      // elements of one halo tile
  constexpr int STAGE_BYTES = STAGE * (int)sizeof(E);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  E* tiles = reinterpret_cast<E*>(smem_raw);
  PrepSync<NS>* sy = reinterpret_cast<PrepSync<NS>*>(smem_raw + NS * STAGE_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int x0 = blockIdx.x * kWarps * kPos, y = blockIdx.y;
  const int which = blockIdx.z & 1, bh = blockIdx.z >> 1;
  const int b = bh / H, h = bh % H;
  const CUtensorMap* map = which ? &map_v : &map_k;
  const float* ws = which ? wv_s : wk_s;
  const float* wt = which ? wv_t : wk_t;
  E* out = which ? v_out : k_out;
  const size_t N = (size_t)gh * gw;

  // this lane's channels of head h: c = h * D + lane * CPL + i, as pairs
  uint64_t wsp[9][NP], wtp[kTaps][NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const size_t c0 = (size_t)h * D + lane * CPL + 2 * i;
    const bool two = CPL >= 2;
#pragma unroll
    for (int j = 0; j < 9; ++j)
      wsp[j][i] = ptx::f2_pack(__ldg(ws + c0 * 9 + j), two ? __ldg(ws + (c0 + 1) * 9 + j) : 0.f);
#pragma unroll
    for (int j = 0; j < kTaps; ++j)
      wtp[j][i] = ptx::f2_pack(__ldg(wt + c0 * kTaps + j),
                               two ? __ldg(wt + (c0 + 1) * kTaps + j) : 0.f);
  }

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) ptx::mbar_init(&sy->full[s], 1);
    sy->abort_flag = 0;
    ptx::fence_mbar_init();
    int f = 0;
    for (; f < NS && f < T; ++f) {
      ptx::mbar_arrive_expect_tx(&sy->full[f], STAGE_BYTES);
      ptx::tma_load_5d(tiles + f * STAGE, map, &sy->full[f], 0, h, x0 - 1, y - 1, b * T + f);
    }
    sy->issued = f;
  }
  __syncthreads();

  // acc[t % 5]: temporal sum of output frame t, filled by frames t-2 .. t+2
  // (frame j adds w_t[tau] * spatial(j) to output j + 2 - tau); emitted and
  // cleared once frame t + 2 has been added.  The frame loop is unrolled by 5
  // so that every acc index is a compile-time constant.
  const uint64_t zero2 = ptx::f2_pack(0.f, 0.f);
  uint64_t acc[5][kPos][NP];
#pragma unroll
  for (int f = 0; f < 5; ++f)
#pragma unroll
    for (int p = 0; p < kPos; ++p)
#pragma unroll
      for (int i = 0; i < NP; ++i) acc[f][p][i] = zero2;

  // per-thread bases: this warp's tile columns and lane's channels; the
  // output rows of its positions (frame 0), advanced by one frame per output
  const E* tile_base = tiles + warp * kPos * D + lane * CPL;
  const size_t frame_stride = N * H * D;
  E* out_base[kPos];
#pragma unroll
  for (int p = 0; p < kPos; ++p) {
    const int x = x0 + warp * kPos + p;
    out_base[p] = x < gw ? out + (((size_t)b * T * N + (size_t)y * gw + x) * H + h) * D +
                               lane * CPL
                         : nullptr;
  }

  bool alive = true;
  auto step = [&](const int j, auto ph_const) {
    constexpr int PH = decltype(ph_const)::value;  // j % 5
    {  // one CTA barrier per frame: frame j landed, and frame j - 1 is free
      bool ok = true;
      if (j < T)
        ok = ptx::wait_bounded(&sy->full[j % NS], (j / NS) & 1, &sy->abort_flag, status,
                               kDevTimeout);
      if (!__syncthreads_and(ok)) {
        alive = false;
        return;
      }
      if (tid == 0 && j >= 1 && j - 1 + NS < T) {
        const int s1 = (j - 1) % NS;
        ptx::mbar_arrive_expect_tx(&sy->full[s1], STAGE_BYTES);
        ptx::tma_load_5d(tiles + s1 * STAGE, map, &sy->full[s1], 0, h, x0 - 1, y - 1,
                         b * T + j - 1 + NS);
        sy->issued = j + NS;
      }
    }
    if (j < T) {
      const int s = j % NS;
      uint64_t cur[kPos][NP];
#pragma unroll
      for (int p = 0; p < kPos; ++p)
#pragma unroll
        for (int i = 0; i < NP; ++i) cur[p][i] = zero2;
      const E* tile = tile_base + s * STAGE;
#pragma unroll
      for (int r = 0; r < 3; ++r) {
#pragma unroll
        for (int cc = 0; cc < kPos + 2; ++cc) {  // tile columns warp*kPos + cc
          Lane<CPL> xv;
          load_lane<E, CPL>(tile + (r * kCols + cc) * D, xv);
#pragma unroll
          for (int p = 0; p < kPos; ++p) {
            const int dx = cc - p;  // filter column 0..2
            if (dx >= 0 && dx < 3) {
#pragma unroll
              for (int i = 0; i < NP; ++i)
                cur[p][i] = ptx::f2_fma(wsp[r * 3 + dx][i], xv.p[i], cur[p][i]);
            }
          }
        }
      }
#pragma unroll
      for (int tau = 0; tau < kTaps; ++tau) {
        const int slot = (PH + 2 - tau + 5) % 5;  // (j + 2 - tau) % 5, compile-time
#pragma unroll
        for (int p = 0; p < kPos; ++p)
#pragma unroll
          for (int i = 0; i < NP; ++i)
            acc[slot][p][i] = ptx::f2_fma(wtp[tau][i], cur[p][i], acc[slot][p][i]);
      }
    }
    const int t = j - 2;  // output frame, complete now
    constexpr int slot = (PH + 3) % 5;  // (j - 2) % 5
    if (t < 0) {  // frames 0 and 1 also fed outputs -2 and -1: drop those sums
#pragma unroll
      for (int p = 0; p < kPos; ++p)
#pragma unroll
        for (int i = 0; i < NP; ++i) acc[slot][p][i] = zero2;
    } else {
#pragma unroll
      for (int p = 0; p < kPos; ++p) {
        float o[2 * NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          ptx::f2_unpack(acc[slot][p][i], o[2 * i], o[2 * i + 1]);
          acc[slot][p][i] = zero2;
        }
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[i] = silu(o[i]);
        if (which == 0) {
          float sq = 0.f;
#pragma unroll
          for (int i = 0; i < CPL; ++i) sq = fmaf(o[i], o[i], sq);
          const float rs = rsqrtf(warp_sum(sq) + eps);
#pragma unroll
          for (int i = 0; i < CPL; ++i) o[i] *= rs;
        }
        if (out_base[p] != nullptr) store_lane<E, CPL>(out_base[p] + t * frame_stride, o);
      }
    }
  };
  for (int j0 = 0; j0 < T + 2 && alive; j0 += 5) {
    step(j0, std::integral_constant<int, 0>());
    if (j0 + 1 < T + 2 && alive) step(j0 + 1, std::integral_constant<int, 1>());
    if (j0 + 2 < T + 2 && alive) step(j0 + 2, std::integral_constant<int, 2>());
    if (j0 + 3 < T + 2 && alive) step(j0 + 3, std::integral_constant<int, 3>());
    if (j0 + 4 < T + 2 && alive) step(j0 + 4, std::integral_constant<int, 4>());
  }
  __syncthreads();
  if (tid == 0 && sy->abort_flag) {  // copies still in flight must land first
    const uint64_t t0 = ptx::globaltimer_ns();
    const int issued = sy->issued;
    for (int f = issued > NS ? issued - NS : 0; f < issued; ++f)
      while (!ptx::mbar_try_wait(&sy->full[f % NS], (f / NS) & 1) &&
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
    float x[2 * Lane<CPL>::NP];
    load_ch<E, CPL>(q + r * D + lane * CPL, *reinterpret_cast<float(*)[CPL]>(x));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) s = fmaf(x[i], x[i], s);
    const float rs = rsqrtf(warp_sum(s) + eps);
#pragma unroll
    for (int i = 0; i < CPL; ++i) x[i] *= rs;
    store_lane<E, CPL>(q_out + r * D + lane * CPL, x);
  }
}

int sm_count();

template <typename E, int D>
static cudaError_t launch_prep_t(const PrepArgs& a, cudaStream_t st) {
#ifndef VDN_PREP_STAGES
#define VDN_PREP_STAGES 4
#endif
  constexpr int NS = sizeof(E) == 2 ? VDN_PREP_STAGES : 3;
  constexpr int kCols = kWarps * kPos + 2;
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
    const size_t sm = NS * STAGE_BYTES + sizeof(PrepSync<NS>);
    auto kern = prep_conv_kernel<E, D, NS>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.gw + kWarps * kPos - 1) / (kWarps * kPos), a.gh, a.B * a.H * 2);
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
