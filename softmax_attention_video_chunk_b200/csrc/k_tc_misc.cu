// Tensor-core path, other kernels:
//   convert_v   V [B, L, H, D] bf16 -> V^T [B*H][D][Lp] fp16 (keys contiguous:
//               the K-major B operand of O += P V); zero for keys >= L.
//   convert_w   [W_soft; W_lin] ([2*H*D][D_out] bf16) -> W^T [D_out][2*H*D] fp16.
//   readout     linear readout with the decay bridge (FP32), then the RMS
//               norm and sigmoid gate of the linear branch, written as fp16 into
//               the right half of the projection operand x.
//   gemm        out = x W^T on tcgen05 (fp16 operands, FP32 accumulation in
//               TMEM), TMA-fed 4-stage pipeline, 128 x 256 output tiles.
// fp16 (11-bit significand) is used for P, V, x and W because bf16 rounding of
// these operands alone would exceed the 2e-3 * RMS accuracy bar of the output;
// bf16 -> fp16 is exact for |value| in [2^-14, 65504], and any overflow is
// reported as VDN_ERR_RANGE through the device status word.
//
// Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method ("Both branches receive ..." paragraph: RMS norm and
// sigmoid gate on the linear readout, separate output projections summed) and
// implementation ("VDA-Gather", "VDA-Epilogue" fused kernels).
#include <math.h>

#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_tc.h"

namespace vdn {

// --------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link-time libcuda dependency)
// --------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// Tiled map with 128-byte swizzle; dims/box innermost first; strides of dims 1..
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, s, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// --------------------------------------------------------------------------
// sizes and argument builders
// --------------------------------------------------------------------------
static inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool use_tc(const vdn_params& p) {
  return p.dtype == VDN_BF16 && (p.d_k == 64 || p.d_k == 128) && !(p.flags & VDN_FLAG_SIMT);
}

TcSizes tc_sizes(const vdn_params& p) {
  TcSizes s;
  const size_t L = (size_t)p.T * p.N, Lp = round_up(L, 64);
  s.vt_bytes = (size_t)p.B * p.H * p.d_k * Lp * 2;
  s.wt_bytes = (size_t)p.D_out * 2 * p.H * p.d_k * 2;
  s.x_bytes = (size_t)p.B * L * 2 * p.H * p.d_k * 2;
  return s;
}

TcAttnArgs tc_attn_args(const vdn_params& p, const AttnArgs& a, void* vt, int* status) {
  TcAttnArgs t;
  t.B = p.B; t.H = p.H; t.T = p.T; t.N = p.N; t.D = p.d_k; t.C = p.chunk;
  t.R = p.window_radius; t.L = p.T * p.N; t.Lp = (int)round_up((size_t)t.L, 64);
  t.scale = a.scale; t.q = a.q; t.k = a.k; t.v = a.v; t.vt = (__half*)vt; t.status = status;
  return t;
}

TcFwdArgs tc_fwd_args(const vdn_params& p, const VdaArgs& va, const TcAttnArgs& t,
                      const void* W_soft, const void* W_lin, const void* gates, void* out,
                      void* wt, void* x) {
  TcFwdArgs f;
  f.B = p.B; f.H = p.H; f.T = p.T; f.N = p.N; f.D = p.d_k; f.L = p.T * p.N; f.D_out = p.D_out;
  f.out_dtype = p.out_dtype; f.eps = p.rms_eps; f.gates = gates; f.W_soft = W_soft;
  f.W_lin = W_lin; f.wt = (__half*)wt; f.x = (__half*)x; f.out = out; f.q = t.q; f.vda = va;
  f.status = t.status;
  return f;
}

// --------------------------------------------------------------------------
// conversions
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
convert_v_kernel(const __nv_bfloat16* __restrict__ v, __half* __restrict__ vt, int H, int L,
                 int Lp, int* __restrict__ status) {
  __shared__ float tile[64][D + 1];
  const int l0 = blockIdx.x * 64, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  for (int e = tid; e < 64 * D; e += blockDim.x) {
    const int r = e / D, c = e % D, l = l0 + r;
    tile[r][c] = l < L ? __bfloat162float(v[(((size_t)b * L + l) * H + h) * D + c]) : 0.f;
  }
  __syncthreads();
  bool bad = false;
  __half* dst = vt + ((size_t)b * H + h) * D * (size_t)Lp;
  for (int e = tid; e < 64 * D; e += blockDim.x) {
    const int c = e >> 6, r = e & 63, l = l0 + r;
    if (l < Lp) {
      const float xv = tile[r][c];
      bad |= !(fabsf(xv) <= 65504.f);
      dst[(size_t)c * Lp + l] = __float2half_rn(xv);
    }
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kDevRange);
}

__global__ void __launch_bounds__(256)
convert_w_kernel(const __nv_bfloat16* __restrict__ Ws, const __nv_bfloat16* __restrict__ Wl,
                 __half* __restrict__ wt, int Din, int Dout, int* __restrict__ status) {
  __shared__ float tile[32][33];
  const int n0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int kk = ty; kk < 32; kk += 8) {
    const int kg = k0 + kk, n = n0 + tx;
    float w = 0.f;
    if (n < Dout)
      w = __bfloat162float(kg < Din ? Ws[(size_t)kg * Dout + n] : Wl[(size_t)(kg - Din) * Dout + n]);
    tile[kk][tx] = w;
  }
  __syncthreads();
  bool bad = false;
  for (int nn = ty; nn < 32; nn += 8) {
    const int n = n0 + nn;
    if (n < Dout) {
      const float w = tile[tx][nn];
      bad |= !(fabsf(w) <= 65504.f);
      wt[(size_t)n * (2 * Din) + k0 + tx] = __float2half_rn(w);
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, kDevRange);
}

cudaError_t launch_convert_v(const TcAttnArgs& t, cudaStream_t st) {
  const dim3 grid(t.Lp / 64, t.H, t.B);
  if (t.D == 128)
    convert_v_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16*)t.v, t.vt, t.H, t.L, t.Lp, t.status);
  else if (t.D == 64)
    convert_v_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16*)t.v, t.vt, t.H, t.L, t.Lp, t.status);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_convert_w(const TcFwdArgs& f, cudaStream_t st) {
  const int Din = f.H * f.D;
  const dim3 grid((f.D_out + 31) / 32, 2 * Din / 32);
  convert_w_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)f.W_soft,
                                         (const __nv_bfloat16*)f.W_lin, f.wt, Din, f.D_out,
                                         f.status);
  return cudaGetLastError();
}

// --------------------------------------------------------------------------
// linear readout + bridge + RMS norm + gate -> x[:, H*D + h*D + c] (fp16)
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
readout_fused_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ alpha,
                     const float* __restrict__ Rf, const float* __restrict__ FS,
                     const float* __restrict__ GS, const __nv_bfloat16* __restrict__ gl,
                     __half* __restrict__ x, int H, int T, int N, int C, int R,
                     float init_scale, float eps, int* __restrict__ status) {
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int nc = (T + C - 1) / C;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  extern __shared__ float smem[];
  float* Sc = smem;        // [D][D]
  float* Qs = Sc + D * D;  // [32][D + 1]
  __shared__ float gf[D], gr[D];
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
  if (anchor) {
    const float* St = Rf + (bh * (T + 1)) * mat;
    for (int e = tid; e < D * D; e += blockDim.x) Sc[e] = 2.f * init_scale * St[e];
  } else {
    const float* F = FS + (bh * (nc + 1) + jf) * mat;
    const float* G = GS + (bh * (nc + 1) + jr) * mat;
    for (int e = tid; e < D * D; e += blockDim.x) {
      const int i = e / D;
      Sc[e] = gf[i] * F[e] + gr[i] * G[e];
    }
  }
  constexpr int NG = D / 32;
  const int tok = tid >> 3, cg = (tid & 7) * 4;
  const size_t rs = (size_t)H * D;
  const size_t L = (size_t)T * N;
  const size_t row0 = (size_t)b * L + (size_t)t * N;
  bool bad = false;
  for (int n0 = 0; n0 < N; n0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * D; e += blockDim.x) {
      const int rr = e / D, cc = e % D;
      Qs[rr * (D + 1) + cc] =
          (n0 + rr < N) ? __bfloat162float(q[(row0 + n0 + rr) * rs + (size_t)h * D + cc]) : 0.f;
    }
    __syncthreads();
    float acc[NG][4];
#pragma unroll
    for (int g = 0; g < NG; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
    for (int l = 0; l < D; ++l) {
      const float a = Qs[tok * (D + 1) + l];
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float4 sv = *reinterpret_cast<const float4*>(Sc + l * D + cg + 32 * g);
        acc[g][0] = fmaf(a, sv.x, acc[g][0]);
        acc[g][1] = fmaf(a, sv.y, acc[g][1]);
        acc[g][2] = fmaf(a, sv.z, acc[g][2]);
        acc[g][3] = fmaf(a, sv.w, acc[g][3]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) ss = fmaf(acc[g][e], acc[g][e], ss);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    const float rinv = 1.f / sqrtf(ss / (float)D + eps);
    if (n0 + tok < N) {
      const size_t row = row0 + n0 + tok;
      const __nv_bfloat16* gp = gl + (row * H + h) * D;
      __half* xp = x + row * (2 * rs) + rs + (size_t)h * D;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const int col = cg + 32 * g;
        const uint2 graw = *reinterpret_cast<const uint2*>(gp + col);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&graw);
        const float2 ga = __bfloat1622float2(g2[0]), gb = __bfloat1622float2(g2[1]);
        const float y0 = ga.x * acc[g][0] * rinv, y1 = ga.y * acc[g][1] * rinv;
        const float y2 = gb.x * acc[g][2] * rinv, y3 = gb.y * acc[g][3] * rinv;
        bad |= !(fabsf(y0) <= 65504.f) || !(fabsf(y1) <= 65504.f) || !(fabsf(y2) <= 65504.f) ||
               !(fabsf(y3) <= 65504.f);
        __half2 h01 = __floats2half2_rn(y0, y1), h23 = __floats2half2_rn(y2, y3);
        uint2 outv;
        outv.x = *reinterpret_cast<uint32_t*>(&h01);
        outv.y = *reinterpret_cast<uint32_t*>(&h23);
        *reinterpret_cast<uint2*>(xp + col) = outv;
      }
    }
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kDevRange);
}

cudaError_t launch_readout_tc(const TcFwdArgs& f, cudaStream_t st) {
  const VdaArgs& a = f.vda;
  const __nv_bfloat16* gl = (const __nv_bfloat16*)f.gates + (size_t)f.B * f.L * f.H * f.D;
  cudaError_t e;
  if (f.D == 128) {
    const size_t sm = sizeof(float) * (128 * 128 + 32 * 129);
    if ((e = cudaFuncSetAttribute(readout_fused_kernel<128>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
      return e;
    readout_fused_kernel<128><<<dim3(a.T, a.H, a.B), 256, sm, st>>>(
        (const __nv_bfloat16*)f.q, a.alpha, a.Rf, a.FS, a.GS, gl, f.x, a.H, a.T, a.N, a.C, a.R,
        a.init_scale, f.eps, f.status);
  } else if (f.D == 64) {
    const size_t sm = sizeof(float) * (64 * 64 + 32 * 65);
    if ((e = cudaFuncSetAttribute(readout_fused_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
      return e;
    readout_fused_kernel<64><<<dim3(a.T, a.H, a.B), 256, sm, st>>>(
        (const __nv_bfloat16*)f.q, a.alpha, a.Rf, a.FS, a.GS, gl, f.x, a.H, a.T, a.N, a.C, a.R,
        a.init_scale, f.eps, f.status);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// --------------------------------------------------------------------------
// out[M, Nout] = x[M, K] * W^T   (tcgen05, fp16 operands, FP32 accumulation)
// --------------------------------------------------------------------------
namespace {
constexpr uint64_t kGemmWaitNs = 2000000000ull;
__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, volatile int* flag,
                                      int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*flag) return false;
    if (ptx::globaltimer_ns() - t0 > kGemmWaitNs) {
      *flag = 1;
      atomicOr(status, kDevTimeout);
      return false;
    }
  }
}
}  // namespace

template <typename TOut>
__global__ void __launch_bounds__(192, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
               TOut* __restrict__ out, int M, int Nout, int K, int* __restrict__ status) {
  constexpr int BM = 128, BN = 256, BKK = 64, NS = 4;
  constexpr int AT = BM * BKK * 2, BT = BN * BKK * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + NS * AT;
  uint64_t* full = (uint64_t*)(sB + NS * BT);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  int* abort_flag = (int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int nkb = K / BKK;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(full + i, 1);
      ptx::mbar_init(empty + i, 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&map_x);
      ptx::prefetch_tmap(&map_w);
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int st = kb % NS, use = kb / NS;
        if (use > 0 && !gwait(empty + st, (use - 1) & 1, abort_flag, status)) break;
        ptx::mbar_arrive_expect_tx(full + st, AT + BT);
        ptx::tma_load_2d(sA + st * AT, &map_x, full + st, kb * BKK, m0);
        ptx::tma_load_2d(sB + st * BT, &map_w, full + st, kb * BKK, n0);
        issued = kb + 1;
      }
      if (*abort_flag) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int kb = max(0, issued - NS); kb < issued; ++kb)
          while (!ptx::mbar_try_wait(full + kb % NS, (kb / NS) & 1) &&
                 ptx::globaltimer_ns() - t0 < kGemmWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16(BM, BN, 0);
      const uint32_t sAa = ptx::smem_u32(sA), sBa = ptx::smem_u32(sB);
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        const int st = kb % NS;
        if (!(ok = gwait(full + st, (kb / NS) & 1, abort_flag, status))) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BKK / 16; ++kk) {
          const uint64_t a = ptx::sdesc_k_sw128(sAa + st * AT + kk * 32);
          const uint64_t bd = ptx::sdesc_k_sw128(sBa + st * BT + kk * 32);
          ptx::mma_ss(tmem, a, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(empty + st);
      }
      if (ok) ptx::mma_commit(acc_full);
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < kGemmWaitNs) {}
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters (warp % 4)
    const int wq = warp & 3;
    const int m = m0 + wq * 32 + lane;
    if (gwait(acc_full, 0, abort_flag, status)) {
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(taddr + 32 * c, r);
        ptx::tmem_wait_ld();
        const int n = n0 + 32 * c;
        if (m >= M) continue;
        if constexpr (sizeof(TOut) == 4) {
          float* op = reinterpret_cast<float*>(out) + (size_t)m * Nout + n;
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            if (n + 4 * v4 < Nout)
              *reinterpret_cast<float4*>(op + 4 * v4) =
                  make_float4(__uint_as_float(r[4 * v4]), __uint_as_float(r[4 * v4 + 1]),
                              __uint_as_float(r[4 * v4 + 2]), __uint_as_float(r[4 * v4 + 3]));
        } else {
          __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(out) + (size_t)m * Nout + n;
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8) {
            if (n + 8 * v8 >= Nout) continue;
            uint4 pk;
            uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(r[8 * v8 + 2 * e]),
                                                        __uint_as_float(r[8 * v8 + 2 * e + 1]));
              w[e] = *reinterpret_cast<uint32_t*>(&t2);
            }
            *reinterpret_cast<uint4*>(op + 8 * v8) = pk;
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 256);
}

cudaError_t launch_gemm_tc(const TcFwdArgs& f, cudaStream_t st) {
  const uint64_t M = (uint64_t)f.B * f.L, K = 2ull * f.H * f.D, Nout = f.D_out;
  CUtensorMap mx, mw;
  {
    const uint64_t dims[2] = {K, M};
    const uint64_t str[1] = {K * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, f.x, dims, str, box))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {K, Nout};
    const uint64_t str[1] = {K * 2};
    const uint32_t box[2] = {64, 256};
    if (!make_tmap(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, f.wt, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const size_t sm = 1024 + 4 * (128 * 64 * 2) + 4 * (256 * 64 * 2) + 128;
  const dim3 grid((unsigned)((Nout + 255) / 256), (unsigned)((M + 127) / 128));
  cudaError_t e;
  if (f.out_dtype == VDN_F32) {
    if ((e = cudaFuncSetAttribute(gemm_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm)) != cudaSuccess)
      return e;
    gemm_tc_kernel<float><<<grid, 192, sm, st>>>(mx, mw, (float*)f.out, (int)M, (int)Nout, (int)K,
                                                 f.status);
  } else {
    if ((e = cudaFuncSetAttribute(gemm_tc_kernel<__nv_bfloat16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
      return e;
    gemm_tc_kernel<__nv_bfloat16><<<grid, 192, sm, st>>>(mx, mw, (__nv_bfloat16*)f.out, (int)M,
                                                         (int)Nout, (int)K, f.status);
  }
  return cudaGetLastError();
}

}  // namespace vdn
