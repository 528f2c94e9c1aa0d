// Window + anchor Softmax attention on CUDA cores, exact FP32 arithmetic.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method, the paragraph on the local window: exact Softmax inside the
// chunk-aligned window (the query chunk and `radius` chunks on each side), the
// first and last latent frames visible to every query, and those two frames'
// queries seeing the whole clip; each key counted once.  The visible keys of a
// query group are at most three disjoint token ranges (see Geo::group), so the
// kernel walks those ranges and never builds a mask.
//
// One CTA = 32 query rows of one group, 128 threads; key tiles of 32 tokens;
// online softmax (running max / sum per row, FP32).  This is the exact-FP32
// path (fp32 inputs, and the cross-check of the tensor-core kernel).
#include <math.h>

#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

template <int D, typename TIn>
__global__ void __launch_bounds__(128)
attn_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                 const TIn* __restrict__ v, const TIn* __restrict__ tk,
                 const TIn* __restrict__ tv, int n_text, float* __restrict__ o, Geo geo,
                 int H, float scale, const TIn* __restrict__ qt) {
  constexpr int BQ = 32, BK = 32, QS = D + 4;
  constexpr int NO = D / 16;  // float4 output groups per thread
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = geo.T * geo.N;
  QGroup g;
  int row_start;
  if (qt != nullptr) {  // text queries: one dense group over every video key
    g.row0 = 0; g.nrows = n_text; g.nseg = 1;
    g.seg0[0] = 0; g.seg1[0] = L;
    g.seg0[1] = g.seg1[1] = g.seg0[2] = g.seg1[2] = 0;
    row_start = blockIdx.x * BQ;
    if (row_start >= n_text) return;
  } else if (!find_tile(geo, BQ, blockIdx.x, &g, &row_start)) {
    return;
  }
  const size_t rs = (size_t)H * D;
  const size_t base = (size_t)b * L * rs + (size_t)h * D;           // video tokens
  const size_t tbase = (size_t)b * n_text * rs + (size_t)h * D;     // text tokens
  const TIn* qsrc = qt != nullptr ? qt : q;
  const size_t qbase = qt != nullptr ? tbase : base;                 // query rows / output

  extern __shared__ __align__(16) float sm_attn[];
  float* Qs = sm_attn;         // [BQ][QS]
  float* Ks = Qs + BQ * QS;    // [BK][QS]
  float* Vs = Ks + BK * QS;    // [BK][D]
  float* Ps = Vs + BK * D;     // [BQ][BK + 1]

  const int row_end = g.row0 + g.nrows;
  for (int e = tid; e < BQ * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    const int row = min(row_start + r, row_end - 1);
    Qs[r * QS + c] = to_f(qsrc[qbase + (size_t)row * rs + c]) * scale;
  }

  const int r = tid >> 2, sub = tid & 3;
  float m_run = -INFINITY, l_run = 0.f;
  float acc[NO][4];
#pragma unroll
  for (int gq = 0; gq < NO; ++gq) acc[gq][0] = acc[gq][1] = acc[gq][2] = acc[gq][3] = 0.f;

  // key ranges of the group, then (optionally) the text tokens as one more range
  for (int s = 0; s < g.nseg + (n_text > 0 ? 1 : 0); ++s) {
    const bool text = s == g.nseg;
    const TIn* ks = text ? tk : k;
    const TIn* vs = text ? tv : v;
    const size_t kb = text ? tbase : base;
    const int s0 = text ? 0 : g.seg0[s], s1 = text ? n_text : g.seg1[s];
    for (int k0 = s0; k0 < s1; k0 += BK) {
      const int kend = min(BK, s1 - k0);
      __syncthreads();
      for (int e = tid; e < BK * D; e += blockDim.x) {
        const int rr = e / D, c = e % D;
        const int key = k0 + min(rr, kend - 1);
        Ks[rr * QS + c] = to_f(ks[kb + (size_t)key * rs + c]);
        Vs[rr * D + c] = to_f(vs[kb + (size_t)key * rs + c]);
      }
      __syncthreads();
      // scores for row r, keys sub + 4*m
      float sc[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) sc[m] = 0.f;
      for (int i = 0; i < D; i += 4) {
        const float4 a = *reinterpret_cast<const float4*>(Qs + r * QS + i);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float4 kk = *reinterpret_cast<const float4*>(Ks + (sub + 4 * m) * QS + i);
          sc[m] = fmaf(a.x, kk.x, sc[m]);
          sc[m] = fmaf(a.y, kk.y, sc[m]);
          sc[m] = fmaf(a.z, kk.z, sc[m]);
          sc[m] = fmaf(a.w, kk.w, sc[m]);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        if (sub + 4 * m >= kend) sc[m] = -INFINITY;
        mx = fmaxf(mx, sc[m]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float corr = expf(m_run - m_new);  // 0 on the first tile
      float ls = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float p = expf(sc[m] - m_new);
        ls += p;
        Ps[r * (BK + 1) + sub + 4 * m] = p;
      }
      ls += __shfl_xor_sync(0xffffffffu, ls, 1);
      ls += __shfl_xor_sync(0xffffffffu, ls, 2);
      l_run = l_run * corr + ls;
      m_run = m_new;
#pragma unroll
      for (int gq = 0; gq < NO; ++gq) {
        acc[gq][0] *= corr; acc[gq][1] *= corr; acc[gq][2] *= corr; acc[gq][3] *= corr;
      }
      __syncwarp();
      for (int kk = 0; kk < kend; ++kk) {
        const float p = Ps[r * (BK + 1) + kk];
#pragma unroll
        for (int gq = 0; gq < NO; ++gq) {
          const float4 vv = *reinterpret_cast<const float4*>(Vs + kk * D + sub * 4 + 16 * gq);
          acc[gq][0] = fmaf(p, vv.x, acc[gq][0]);
          acc[gq][1] = fmaf(p, vv.y, acc[gq][1]);
          acc[gq][2] = fmaf(p, vv.z, acc[gq][2]);
          acc[gq][3] = fmaf(p, vv.w, acc[gq][3]);
        }
      }
    }
  }
  if (row_start + r < row_end) {
    const float inv = 1.f / l_run;
    float* dst = o + qbase + (size_t)(row_start + r) * rs;
#pragma unroll
    for (int gq = 0; gq < NO; ++gq)
      *reinterpret_cast<float4*>(dst + sub * 4 + 16 * gq) =
          make_float4(acc[gq][0] * inv, acc[gq][1] * inv, acc[gq][2] * inv, acc[gq][3] * inv);
  }
}

template <int D, typename TIn>
static cudaError_t launch_t(const AttnArgs& a, float* o, cudaStream_t st) {
  Geo geo{a.T, a.N, a.C, a.R};
  const int tiles = a.text_q != nullptr ? (a.n_text_keys + 31) / 32 : count_tiles(geo, 32);
  const size_t sm = sizeof(float) * (2 * 32 * (D + 4) + 32 * D + 32 * 33);
  auto kern = attn_simt_kernel<D, TIn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  kern<<<dim3(tiles, a.H, a.B), 128, sm, st>>>(
      (const TIn*)a.q, (const TIn*)a.k, (const TIn*)a.v, (const TIn*)a.text_k,
      (const TIn*)a.text_v, a.n_text_keys, o, geo, a.H, a.scale, (const TIn*)a.text_q);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const AttnArgs& a, float* o, cudaStream_t st) {
  const bool bf = a.dtype == VDN_BF16;
  switch (a.D) {
    case 32: return bf ? launch_t<32, __nv_bfloat16>(a, o, st) : launch_t<32, float>(a, o, st);
    case 64: return bf ? launch_t<64, __nv_bfloat16>(a, o, st) : launch_t<64, float>(a, o, st);
    case 128: return bf ? launch_t<128, __nv_bfloat16>(a, o, st) : launch_t<128, float>(a, o, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
