// Tensor-core path, other kernels:
//   convert_v   V [B, L, H, D] bf16 -> V^T [B*H][D][Lp] fp16 (keys contiguous:
//               the K-major B operand of O += P V); zero for keys >= L.
//   convert_w   [W_soft; W_lin] ([2*H*D][D_out] bf16) -> W^T [D_out][2*H*D] fp16.
//   gemm        out = x W^T on tcgen05 (fp16 operands, FP32 accumulation in
//               TMEM), TMA-fed 4-stage pipeline, 128 x 256 output tiles.
// fp16 (11-bit significand) is used for P, V, x and W because bf16 rounding of
// these operands alone would exceed the 2e-3 * RMS accuracy bar of the output;
// bf16 -> fp16 is exact for |value| in [2^-14, 65504], and any overflow is
// reported as VDN_ERR_RANGE through the device status word.
//
// Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", method (the paragraph on the two output gates: RMS norm and
// sigmoid gate on the linear readout, separate output projections summed) and
// implementation ("VDA-Gather", "VDA-Epilogue" fused kernels).
#include <math.h>

#include <atomic>
#include <mutex>

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

// Looked up once per process; std::call_once makes the first concurrent calls
// from several host threads safe.
static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// Tiled map with 128-byte swizzle; dims/box innermost first; strides of dims 1..
static bool make_tmap_sw(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                         const uint64_t* dims, const uint64_t* strides_bytes,
                         const uint32_t* box, CUtensorMapSwizzle swz) {
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
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 128-byte swizzled boxes (the tensor-core operand tiles).
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap_sw(map, dt, rank, base, dims, strides_bytes, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Row-major uint8 matrix [rows][cols] (cols a multiple of 16), 128-byte
// swizzled boxes of box_rows x box_cols bytes: the E4M3 operand tiles.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                  uint32_t box_cols, uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t str[1] = {cols};
  const uint32_t box[2] = {box_cols, box_rows};
  return make_tmap_sw(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, str, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

// Dense (unswizzled) boxes, laid out in shared memory in row-major box order.
bool make_tmap_plain(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap_sw(map, dt, rank, base, dims, strides_bytes, box, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  const size_t ntp = (p.flags & VDN_FLAG_TEXT_SOFTMAX) ? round_up((size_t)p.n_text, 64) : 0;
  s.vt_bytes = (size_t)p.B * p.H * p.d_k * (Lp + ntp) * 2;
  s.wt_bytes = (size_t)p.D_out * 2 * p.H * p.d_k * 2;
  s.x_bytes = (size_t)p.B * L * 2 * p.H * p.d_k * 2;
  return s;
}

TcAttnArgs tc_attn_args(const vdn_params& p, const AttnArgs& a, void* vt, int* status) {
  TcAttnArgs t;
  t.B = p.B; t.H = p.H; t.T = p.T; t.N = p.N; t.D = p.d_k; t.C = p.chunk;
  t.R = p.window_radius; t.L = p.T * p.N; t.Lp = (int)round_up((size_t)t.L, 64);
  t.scale = a.scale; t.q = a.q; t.k = a.k; t.v = a.v; t.vt = (__half*)vt; t.status = status;
  t.n_text_keys = a.n_text_keys;
  t.ntp = (int)round_up((size_t)a.n_text_keys, 64);
  t.text_k = a.text_k; t.text_v = a.text_v; t.text_q = a.text_q;
  t.vt_text = t.vt + (size_t)t.B * t.H * t.D * t.Lp;
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
// 64 tokens x D channels per CTA: 16-byte loads along channels into an fp16
// shared tile, 16-byte stores of 8 consecutive tokens per channel.
template <int D>
__global__ void __launch_bounds__(256)
convert_v_kernel(const __nv_bfloat16* __restrict__ v, __half* __restrict__ vt, int H, int L,
                 int Lp, int* __restrict__ status) {
  constexpr int TP = D + 8;  // padded row (halves) of the shared tile
  __shared__ __align__(16) __half tile[64 * TP];
  const int l0 = blockIdx.x * 64, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  bool bad = false;
  for (int e = tid; e < 64 * D / 8; e += blockDim.x) {
    const int r = e / (D / 8), c8 = (e % (D / 8)) * 8, l = l0 + r;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (l < L) raw = *reinterpret_cast<const uint4*>(v + (((size_t)b * L + l) * H + h) * D + c8);
    const __nv_bfloat162* in2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 outv;
    __half2* out2 = reinterpret_cast<__half2*>(&outv);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(in2[q]);
      bad |= !(fabsf(f.x) <= 65504.f) || !(fabsf(f.y) <= 65504.f);
      out2[q] = __floats2half2_rn(f.x, f.y);
    }
    *reinterpret_cast<uint4*>(&tile[r * TP + c8]) = outv;
  }
  __syncthreads();
  __half* dst = vt + ((size_t)b * H + h) * D * (size_t)Lp;
  for (int e = tid; e < D * 8; e += blockDim.x) {
    // consecutive threads take consecutive channels: conflict-free tile reads
    const int c = e % D, r8 = (e / D) * 8, l = l0 + r8;
    if (l < Lp) {
      uint4 outv;
      __half* o = reinterpret_cast<__half*>(&outv);
#pragma unroll
      for (int q = 0; q < 8; ++q) o[q] = tile[(r8 + q) * TP + c];
      *reinterpret_cast<uint4*>(dst + (size_t)c * Lp + l) = outv;
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

static cudaError_t convert_one(const void* src, __half* dst, int B, int H, int D, int L, int Lp,
                               int* status, cudaStream_t st) {
  const dim3 grid(Lp / 64, H, B);
  if (D == 128)
    convert_v_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16*)src, dst, H, L, Lp, status);
  else if (D == 64)
    convert_v_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16*)src, dst, H, L, Lp, status);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_convert_v(const TcAttnArgs& t, cudaStream_t st) {
  cudaError_t e = convert_one(t.v, t.vt, t.B, t.H, t.D, t.L, t.Lp, t.status, st);
  if (e != cudaSuccess || t.n_text_keys == 0) return e;
  return convert_one(t.text_v, t.vt_text, t.B, t.H, t.D, t.n_text_keys, t.ntp, t.status, st);
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

// Persistent: each CTA walks output tiles t = blockIdx.x, + gridDim.x, ...
// (n fastest, so consecutive tiles reuse the A row block from L2).  Two TMEM
// accumulators (2 x 256 columns): the epilogue of one tile overlaps the main
// loop of the next.
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
  uint64_t* acc_full = empty + NS;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2], 128 epilogue arrivals
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  int* abort_flag = (int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (Nout + BN - 1) / BN;
  const int ntiles = ((M + BM - 1) / BM) * tiles_n;
  const int nkb = K / BKK;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(full + i, 1);
      ptx::mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(acc_full + i, 1);
      ptx::mbar_init(acc_empty + i, 128);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
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
      int g = 0, issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int st = g % NS, use = g / NS;
          if (use > 0 &&
              !(ok = gwait(empty + st, (use - 1) & 1, abort_flag, status)))
            break;
          ptx::mbar_arrive_expect_tx(full + st, AT + BT);
          ptx::tma_load_2d(sA + st * AT, &map_x, full + st, kb * BKK, m0);
          ptx::tma_load_2d(sB + st * BT, &map_w, full + st, kb * BKK, n0);
          issued = g + 1;
        }
      }
      if (*abort_flag) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int q = max(0, issued - NS); q < issued; ++q)
          while (!ptx::mbar_try_wait(full + q % NS, (q / NS) & 1) &&
                 ptx::globaltimer_ns() - t0 < kGemmWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16(BM, BN, 0);
      const uint32_t sAa = ptx::smem_u32(sA), sBa = ptx::smem_u32(sB);
      bool ok = true;
      int g = 0, lt = 0;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++lt) {
        const int acc = lt & 1;
        if (lt >= 2 && !(ok = gwait(acc_empty + acc, ((lt >> 1) - 1) & 1, abort_flag, status)))
          break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int st = g % NS;
          if (!(ok = gwait(full + st, (g / NS) & 1, abort_flag, status))) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BKK / 16; ++kk) {
            const uint64_t a = ptx::sdesc_k_sw128(sAa + st * AT + kk * 32);
            const uint64_t bd = ptx::sdesc_k_sw128(sBa + st * BT + kk * 32);
            ptx::mma_ss(d, a, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(empty + st);
        }
        if (ok) ptx::mma_commit(acc_full + acc);
      }
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < kGemmWaitNs) {}
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters (warp % 4)
    const int wq = warp & 3;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      if (!gwait(acc_full + acc, (lt >> 1) & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m = (t / tiles_n) * BM + wq * 32 + lane, n0 = (t % tiles_n) * BN;
      const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + acc * BN;
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
      ptx::tc_fence_before();
      ptx::mbar_arrive(acc_empty + acc);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

// SM count of the current device (the per-device attribute cache; atomic
// entries, so concurrent first calls are safe).
int sm_count() {
  static std::atomic<int> cached[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
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
  const uint64_t ntiles = ((Nout + 255) / 256) * ((M + 127) / 128);
  const dim3 grid((unsigned)(ntiles < (uint64_t)sm_count() ? ntiles : (uint64_t)sm_count()));
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
