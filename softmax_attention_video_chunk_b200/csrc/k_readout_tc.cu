// Linear-branch readout on the sm_100a tensor cores.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method: the query reads the forward state gathered just
// outside its window and the reverse state just outside the other edge, each
// carried across the skipped window span by the accumulated channel-wise
// decay, and the two readouts are added; the linear readout is then
// RMS-normalised and gated ("VDA-Gather" and "VDA-Epilogue" of the
// implementation section).
//
// One CTA per (b, h, frame t):
//   all warps   S_t = Diag(gf_t) F + Diag(gr_t) G (FP32; anchors: S_text), split
//               into bf16 hi + lo parts (S_hi + S_lo keeps ~16 significant bits
//               of the FP32 state) and stored as the K-major B operand;
//   warp 0      TMA producer: 128-token tiles of q (bf16), one buffer (two
//               CTAs share an SM and hide each other's load latency);
//   warp 1      MMA issuer: O = q S_hi + q S_lo (M = 128 tokens, N = d, FP32
//               in TMEM, two accumulators);
//   warps 2-5   epilogue, one token row per thread: RMS over the row, times
//               the linear gate, fp16 into the right half of the projection
//               operand x.
#include <math.h>

#include "mx_encode.cuh"
#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_tc.h"

namespace vdn {

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

template <int D>
__global__ void __launch_bounds__(192, 2)
readout_tc_kernel(const __grid_constant__ CUtensorMap map_q, const float* __restrict__ alpha,
                  const float* __restrict__ Rf, const float* __restrict__ FS,
                  const float* __restrict__ GS, const __nv_bfloat16* __restrict__ gl,
                  __half* __restrict__ x, uint8_t* __restrict__ xq, uint8_t* __restrict__ sfa,
                  int H, int T, int N, int C, int R, float init_scale,
                  float eps, int* __restrict__ status) {
  constexpr int BM = 128;
  constexpr int QT = BM * D * 2;      // bytes of a q tile
  constexpr int BTB = D * D * 2;      // bytes of one B operand (hi or lo)
  constexpr int NP = D / 64;          // 128-byte K panels
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nc = (T + C - 1) / C;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  const size_t L = (size_t)T * N;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sB = smem;                 // [hi | lo], each NP panels of [D rows][128 B]
  uint8_t* sQ = sB + 2 * BTB;         // 1 q tile
  uint64_t* q_full = (uint64_t*)(sQ + QT);
  uint64_t* q_empty = q_full + 2;
  uint64_t* acc_full = q_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  int* abort_flag = (int*)(tmem_slot + 1);
  __shared__ float gf[D], gr[D];

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(q_full + i, 1);
      ptx::mbar_init(q_empty + i, 1);
      ptx::mbar_init(acc_full + i, 1);
      ptx::mbar_init(acc_empty + i, 128);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 2 * D < 32 ? 32 : 2 * D);
    ptx::tmem_relinquish();
  }
  // ---- bridge decays and the combined state ----
  const bool anchor = (t == 0 || t == T - 1);
  const int c = t / C;
  const int jf = max(0, c - R), jr = min(nc, c + R + 1);
  const int w0 = max(0, (c - R) * C), w1 = min(T, (c + R + 1) * C);
  for (int i = tid; i < D; i += blockDim.x) {
    float a = 1.f, r = 1.f;
    if (alpha != nullptr && !anchor) {
      const float* al = alpha + bh * T * D;
      for (int j = w0; j <= t; ++j) a *= al[(size_t)j * D + i];
      for (int j = t; j < w1; ++j) r *= al[(size_t)j * D + i];
    }
    gf[i] = a;
    gr[i] = r;
  }
  __syncthreads();
  {
    const float* F = anchor ? Rf + (bh * (T + 1)) * mat : FS + (bh * (nc + 1) + jf) * mat;
    const float* G = anchor ? nullptr : GS + (bh * (nc + 1) + jr) * mat;
    for (int e = tid; e < D * D; e += blockDim.x) {
      const int i = e / D, j = e % D;  // S[i][j]: key channel i, value channel j
      const float s = anchor ? 2.f * init_scale * F[e] : gf[i] * F[e] + gr[i] * G[e];
      const __nv_bfloat16 hi = __float2bfloat16_rn(s);
      const __nv_bfloat16 lo = __float2bfloat16_rn(s - __bfloat162float(hi));
      // B[n = j][k = i], K-major with 128-byte swizzle
      const int panel = i >> 6, kk = i & 63;
      const uint32_t off = panel * (D * 128) + j * 128 + ((((kk >> 3) ^ (j & 7)) << 4)) +
                           (kk & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(sB + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sB + BTB + off) = lo;
    }
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntile = (N + BM - 1) / BM;

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&map_q);
      for (int m = 0; m < ntile; ++m) {
        if (m > 0 &&
            !ptx::wait_bounded(q_empty, (m - 1) & 1, abort_flag, status, kDevTimeout))
          break;
        ptx::mbar_arrive_expect_tx(q_full, QT);
        for (int p = 0; p < NP; ++p)
          ptx::tma_load_4d(sQ + p * BM * 128, &map_q, q_full, p * 64, h, t * N + m * BM, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16(128, D, 1);
      const uint32_t sQa = ptx::smem_u32(sQ), sBa = ptx::smem_u32(sB);
      for (int m = 0; m < ntile; ++m) {
        const int st = m & 1, use = m >> 1;
        if (!ptx::wait_bounded(q_full, m & 1, abort_flag, status, kDevTimeout)) break;
        if (use > 0 && !ptx::wait_bounded(acc_empty + st, (use - 1) & 1, abort_flag, status,
                                          kDevTimeout))
          break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + st * D;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;
            const uint64_t a = ptx::sdesc_k_sw128(sQa + (kk >> 2) * (BM * 128) + koff);
            const uint64_t bd =
                ptx::sdesc_k_sw128(sBa + part * BTB + (kk >> 2) * (D * 128) + koff);
            ptx::mma_ss(d, a, bd, idesc, (part > 0 || kk > 0) ? 1u : 0u);
          }
        ptx::mma_commit(q_empty);
        ptx::mma_commit(acc_full + st);
      }
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < 2000000000ull) {}
    }
  } else {
    // epilogue: warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    bool bad = false;
    for (int m = 0; m < ntile; ++m) {
      const int st = m & 1, use = m >> 1;
      if (!ptx::wait_bounded(acc_full + st, use & 1, abort_flag, status, kDevTimeout)) break;
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + lane_off + st * D;
      float ss = 0.f;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(taddr + 32 * cc, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
      }
      const float rinv = 1.f / sqrtf(ss / (float)D + eps);
      const int tok = m * BM + q * 32 + lane;
      const bool valid = tok < N;
      const size_t row = (size_t)b * L + (size_t)t * N + tok;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(taddr + 32 * cc, r);
        ptx::tmem_wait_ld();
        if (!valid) continue;
        const uint4* gp = reinterpret_cast<const uint4*>(gl + (row * H + h) * D + 32 * cc);
        uint32_t hw[16];  // g_l * RMS(o_l) of this 32-column block, fp16
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint4 gg = gp[v4];
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gg);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 gv = __bfloat1622float2(g2[e]);
            const float y0 = gv.x * __uint_as_float(r[8 * v4 + 2 * e]) * rinv;
            const float y1 = gv.y * __uint_as_float(r[8 * v4 + 2 * e + 1]) * rinv;
            bad |= !(fabsf(y0) <= 65504.f) || !(fabsf(y1) <= 65504.f);
            __half2 hv = __floats2half2_rn(y0, y1);
            hw[4 * v4 + e] = *reinterpret_cast<uint32_t*>(&hv);
          }
        }
        const size_t K = (size_t)(2 * H * D), col = (size_t)H * D + (size_t)h * D + 32 * cc;
        if (xq == nullptr) {
          uint4* xp = reinterpret_cast<uint4*>(x + row * K + col);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            xp[v4] = make_uint4(hw[4 * v4], hw[4 * v4 + 1], hw[4 * v4 + 2], hw[4 * v4 + 3]);
        } else {  // the same fp16 values, quantised to MXFP8 (one 32-element block)
          uint32_t cw[8];
          const uint32_t eb = mx::encode32(hw, cw);
          uint4* qp = reinterpret_cast<uint4*>(xq + row * K + col);
          qp[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          qp[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          sfa[mx::sf_offset(row, (int)(col / 32), (int)K)] = (uint8_t)eb;
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(acc_empty + st);
    }
    if (bad) atomicOr(status, kDevRange);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 2 * D < 32 ? 32 : 2 * D);
}

template <int D>
static cudaError_t launch_t(const TcFwdArgs& f, cudaStream_t st) {
  const VdaArgs& a = f.vda;
  CUtensorMap mq;
  const uint64_t L = (uint64_t)f.L, H = f.H, B = f.B;
  const uint64_t dims[4] = {(uint64_t)D, H, L, B};
  const uint64_t str[3] = {(uint64_t)D * 2, H * D * 2, L * H * D * 2};
  const uint32_t box[4] = {64, 1, 128, 1};
  if (!make_tmap(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, f.q, dims, str, box))
    return cudaErrorInvalidValue;
  const size_t sm = 1024 + 2 * (size_t)D * D * 2 + 128 * (size_t)D * 2 + 128;
  auto kern = readout_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const __nv_bfloat16* gl = (const __nv_bfloat16*)f.gates + (size_t)f.B * f.L * f.H * f.D;
  kern<<<dim3(a.T, a.H, a.B), 192, sm, st>>>(mq, a.alpha, a.Rf, a.FS, a.GS, gl, f.x, f.xq, f.sfa,
                                             a.H, a.T,
                                             a.N, a.C, a.R, a.init_scale, f.eps, f.status);
  return cudaGetLastError();
}

cudaError_t launch_readout_tc(const TcFwdArgs& f, cudaStream_t st) {
  if (f.D == 128) return launch_t<128>(f, st);
  if (f.D == 64) return launch_t<64>(f, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
