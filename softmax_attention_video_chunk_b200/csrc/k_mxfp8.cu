// MXFP8 output projection: quantisation of the fp16 operands and a
// block-scaled tcgen05 GEMM (kind::mxf8f6f4, E4M3 elements, UE8M0 scales).
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", implementation section ("Other optimizations": the QKV, output
// and feed-forward GEMMs run in MXFP8 while the recurrent state and the
// inverses stay FP32).  The format is the OCP Microscaling one: blocks of 32
// consecutive elements along the contraction dimension share a power-of-two
// scale 2^e, e = floor(log2(max |v|)) - 8 (8 = exponent of the largest normal
// E4M3 value, 448), stored as the unsigned exponent e + 127; each element is
// v / 2^e rounded to E4M3, ties to even, saturating at +-448.
//
// Scale factors are stored in 512-byte atoms, one per 128 rows x 4 blocks
// (128 contraction elements): byte 16 (r % 32) + 4 ((r % 128) / 32) + (j % 4)
// of atom (r / 128) * (K / 128) + j / 4 holds the scale of row r, block j.
// tcgen05.cp.32x128b.warpx4 moves one atom into 4 TMEM columns of lanes 0..31,
// repeated in every lane quarter; the MMA picks the byte of the K block it
// consumes (scale-factor id).
#include <cuda_fp8.h>
#include <math.h>

#include "mx_encode.cuh"
#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_tc.h"

namespace vdn {

bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                  uint32_t box_cols, uint32_t box_rows);

size_t mx_scale_bytes(long long rows_padded, int cols) {
  return (size_t)((rows_padded + 127) / 128) * (size_t)(cols / 128) * 512u;
}

// Each lane quantises 8 consecutive elements (one 16-byte load, one 8-byte
// store); the 4 lanes of a 32-element block share its maximum by shuffles, so
// a warp covers 256 columns (two scale atoms' worth of one row).  Grid-stride
// over (row, 256-column piece).  Rows in [rows, rows_padded) write the
// smallest scale only (their elements are never read: the GEMM's loads of them
// come back as zeros).
__global__ void __launch_bounds__(256)
mx_quant_rows_kernel(const __half* __restrict__ x, uint8_t* __restrict__ codes,
                     uint8_t* __restrict__ scales, long long rows, long long rows_padded,
                     int cols) {
  const int lane = threadIdx.x & 31;
  const int pieces = (cols + 255) / 256;
  const long long nwork = rows_padded * pieces;
  const long long wstride = (long long)gridDim.x * 8;
  for (long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); w < nwork; w += wstride) {
    const long long r = w / pieces;
    const int col = (int)(w % pieces) * 256 + 8 * lane;
    const bool in_cols = col < cols;  // uniform per 32-element block (cols % 128 == 0)
    const bool live = r < rows && in_cols;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    if (live) {
      const uint4 raw = *reinterpret_cast<const uint4*>(x + r * cols + col);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = mx::block_exp(amax);
    const float inv = mx::inv_scale(e);
    if (live) {
      const uint32_t lo = mx::e4m3x2(v[0] * inv, v[1] * inv) | (mx::e4m3x2(v[2] * inv, v[3] * inv) << 16);
      const uint32_t hi = mx::e4m3x2(v[4] * inv, v[5] * inv) | (mx::e4m3x2(v[6] * inv, v[7] * inv) << 16);
      *reinterpret_cast<uint2*>(codes + r * cols + col) = make_uint2(lo, hi);
    }
    if ((lane & 3) == 0 && in_cols)  // block index along the row: col / 32
      scales[mx::sf_offset((size_t)r, col / 32, cols)] = (uint8_t)(e + 127);
  }
}

int sm_count();

cudaError_t launch_mx_quant(const __half* x, uint8_t* codes, uint8_t* scales, long long rows,
                            long long rows_padded, int cols, cudaStream_t st) {
  const long long warps = rows_padded * ((cols + 255) / 256);
  long long blocks = (warps + 7) / 8;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  mx_quant_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, codes, scales, rows, rows_padded,
                                                         cols);
  return cudaGetLastError();
}

namespace {
constexpr uint64_t kMxWaitNs = 2000000000ull;
__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity, volatile int* flag,
                                      int* status) {
  return ptx::wait_bounded(bar, parity, flag, status, kDevTimeout, kMxWaitNs);
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(ptx::smem_u32(dst)), "l"(src), "r"(bytes), "r"(ptx::smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of one scale-factor atom for tcgen05.cp: K-major,
// no swizzle, core matrices of 8 rows x 16 bytes (rows 16 bytes apart), 8-row
// groups 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16 >> 4) << 16;   // leading byte offset (one 16-byte chunk per row)
  d |= (uint64_t)(128 >> 4) << 32;  // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;           // descriptor version (sm_100)
  return d;                         // layout type 0: no swizzle
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Instruction descriptor of kind::mxf8f6f4 with block scaling: E4M3 A and B
// (K-major), M x N, UE8M0 scales; scale-factor ids in bits [29,31) (A) and
// [4,6) (B) select the byte of the TMEM scale cells.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, uint32_t sf_id) {
  return (sf_id << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         (sf_id << 29);
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
}  // namespace

// out[M, Nout] = dequant(xq)[M, K] * dequant(wq)[Nout, K]^T.  Persistent CTAs
// walk 128 x 256 output tiles (n fastest); a 4-stage TMA ring of 128-element
// (128-byte) K panels of both operands plus their scale atoms; one TMEM
// accumulator (256 columns) and, per stage, 4 + 8 TMEM columns of scales.
template <typename TOut>
__global__ void __launch_bounds__(192, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
               const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
               TOut* __restrict__ out, int M, int Nout, int K, int* __restrict__ status) {
  constexpr int BM = 128, BN = 256, BK = 128, NS = 4;
  constexpr int AT = BM * BK, BT = BN * BK, SFAB = 512, SFBB = 1024;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + NS * AT;
  uint8_t* sSA = sB + NS * BT;
  uint8_t* sSB = sSA + NS * SFAB;
  uint64_t* full = (uint64_t*)(sSB + NS * SFBB);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;
  uint64_t* acc_empty = acc_full + 1;  // 128 epilogue arrivals
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  int* abort_flag = (int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (Nout + BN - 1) / BN;
  const int ntiles = ((M + BM - 1) / BM) * tiles_n;
  const int nkb = K / BK;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(full + i, 1);
      ptx::mbar_init(empty + i, 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 128);
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
        const int mb = t / tiles_n, nb = t % tiles_n;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int st = g % NS, use = g / NS;
          if (use > 0 && !(ok = mwait(empty + st, (use - 1) & 1, abort_flag, status))) break;
          ptx::mbar_arrive_expect_tx(full + st, AT + BT + SFAB + SFBB);
          ptx::tma_load_2d(sA + st * AT, &map_x, full + st, kb * BK, mb * BM);
          ptx::tma_load_2d(sB + st * BT, &map_w, full + st, kb * BK, nb * BN);
          bulk_g2s(sSA + st * SFAB, sfa + ((size_t)mb * nkb + kb) * 512, 512, full + st);
          bulk_g2s(sSB + st * SFBB, sfb + ((size_t)(2 * nb) * nkb + kb) * 512, 512, full + st);
          bulk_g2s(sSB + st * SFBB + 512, sfb + ((size_t)(2 * nb + 1) * nkb + kb) * 512, 512,
                   full + st);
          issued = g + 1;
        }
      }
      if (*abort_flag) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int q = max(0, issued - NS); q < issued; ++q)
          while (!ptx::mbar_try_wait(full + q % NS, (q / NS) & 1) &&
                 ptx::globaltimer_ns() - t0 < kMxWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t sAa = ptx::smem_u32(sA), sBa = ptx::smem_u32(sB);
      const uint32_t sSAa = ptx::smem_u32(sSA), sSBa = ptx::smem_u32(sSB);
      bool ok = true;
      int g = 0, lt = 0;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++lt) {
        if (lt >= 1 && !(ok = mwait(acc_empty, (lt - 1) & 1, abort_flag, status))) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int st = g % NS;
          if (!(ok = mwait(full + st, (g / NS) & 1, abort_flag, status))) break;
          ptx::tc_fence_after();
          const uint32_t ta = tmem + 256 + st * 16, tb = ta + 4;
          tmem_cp_sf(ta, sf_desc(sSAa + st * SFAB));
          tmem_cp_sf(tb, sf_desc(sSBa + st * SFBB));
          tmem_cp_sf(tb + 4, sf_desc(sSBa + st * SFBB + 512));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t a = ptx::sdesc_k_sw128(sAa + st * AT + kk * 32);
            const uint64_t b = ptx::sdesc_k_sw128(sBa + st * BT + kk * 32);
            const uint32_t sel = (uint32_t)kk << 30;  // byte of the scale cells
            mma_mx(tmem, a, b, idesc_mx(BM, BN, (uint32_t)kk), ta | sel, tb | sel,
                   (kb > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(empty + st);
        }
        if (ok) ptx::mma_commit(acc_full);
      }
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < kMxWaitNs) {}
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters (warp % 4)
    const int wq = warp & 3;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      if (!mwait(acc_full, lt & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m = (t / tiles_n) * BM + wq * 32 + lane, n0 = (t % tiles_n) * BN;
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
      ptx::tc_fence_before();
      ptx::mbar_arrive(acc_empty);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

// xq [M][K], wq [Nout][K] E4M3; sfa for M rows padded to 128, sfb for Nout
// rows padded to 256 (two atoms per 256-column output tile).
cudaError_t launch_mx_gemm(const uint8_t* xq, const uint8_t* sfa, const uint8_t* wq,
                           const uint8_t* sfb, void* out, vdn_dtype out_dtype, int M, int Nout,
                           int K, int* status, cudaStream_t st) {
  CUtensorMap mx, mw;
  if (!make_tmap_u8(&mx, xq, (uint64_t)K, (uint64_t)M, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_u8(&mw, wq, (uint64_t)K, (uint64_t)Nout, 128, 256)) return cudaErrorInvalidValue;
  const size_t sm = 1024 + 4 * (128 * 128 + 256 * 128 + 512 + 1024) + 128;
  const uint64_t ntiles = ((uint64_t)(Nout + 255) / 256) * ((uint64_t)(M + 127) / 128);
  const dim3 grid((unsigned)(ntiles < (uint64_t)sm_count() ? ntiles : (uint64_t)sm_count()));
  cudaError_t e;
  if (out_dtype == VDN_F32) {
    if ((e = cudaFuncSetAttribute(mx_gemm_kernel<float>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) !=
        cudaSuccess)
      return e;
    mx_gemm_kernel<float><<<grid, 192, sm, st>>>(mx, mw, sfa, sfb, (float*)out, M, Nout, K, status);
  } else {
    if ((e = cudaFuncSetAttribute(mx_gemm_kernel<__nv_bfloat16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) !=
        cudaSuccess)
      return e;
    mx_gemm_kernel<__nv_bfloat16><<<grid, 192, sm, st>>>(mx, mw, sfa, sfb, (__nv_bfloat16*)out, M,
                                                        Nout, K, status);
  }
  return cudaGetLastError();
}

}  // namespace vdn
