// Video Delta Attention frame transitions on the sm_100a tensor cores.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation": per frame, the statistics A_t = beta K_t^T K_t and
// W_t = beta K_t^T V_t (Video Delta Attention, frame statistics), then the
// inverse X_t = (I + A_t)^-1 in key-channel space (implementation section,
// "Small-matrix inverse": Gauss-Jordan elimination held in registers, FP32).
// The frame update is S_t = X_t (Diag(alpha_t) S_{t-1} + W_t); this kernel
// writes X_t and W_t and leaves the product with X_t to the scan, which needs
// one product per frame either way.  The text virtual frame writes its state
// X_0 W_0.
//
// One CTA per (b, h, frame); frame 0 is the text virtual frame.
//   warp 0      TMA producer: 64-token tiles of K and V (bf16, 5-D maps
//               that stop at the frame edge) into a 3-stage ring;
//   warp 1      MMA issuer: [K | V]^T-shaped products on tcgen05, both
//               operands MN-major straight from the TMA tiles:
//               D[128 x 2d] += K_t^T [K_t | V_t]  (FP32 in TMEM);
//   all warps   epilogue: D -> I + beta A in shared memory and beta W straight
//               to Rout, then the in-place Gauss-Jordan inversion of I + beta A
//               with each thread holding a (d/16) x (d/16) block in registers
//               (one barrier per pivot); X out (text frame: X beta W on CUDA
//               cores, W read back from Rout).
// For d = 64 the MMA computes [K|V]^T [K|V] (M = N = 128) and keeps the first
// 64 rows.  Anchor frames write X = I, W = 0 and exit.
// Frozen-state rule (comparison mode): X = I - beta A without the inversion
// and W = beta W; its update is S_t = X_t Diag(alpha_t) S_{t-1} + W_t.
// Per-token write gates: warps 2-7 turn every landed bf16 tile into an exact
// fp16 copy (the A operand, in place) and into beta_i-scaled fp16 hi and lo
// parts (two B operands: beta*x = hi + lo to ~22 bits); two MMA chains
// accumulate K^T (beta [K|V])_hi and K^T (beta [K|V])_lo in separate TMEM
// columns, summed in the epilogue.
#include "tc_ptx.cuh"
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);

template <int D>
__global__ void __launch_bounds__(256, 2)
vda_frame_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_tk,
                    const __grid_constant__ CUtensorMap map_tv, const float* __restrict__ beta,
                    const float* __restrict__ alpha, float* __restrict__ Mout,
                    float* __restrict__ Rout, int H, int T, int N, int n_text, bool beta_tok,
                    bool frozen,
                    int* __restrict__ status) {
  constexpr int BT = 64;                  // tokens per stage
  constexpr int NBLK = D / 32;            // 64-channel blocks of [K | V]
  constexpr int BLKB = BT * 128;          // bytes of one block (BT rows x 128 B)
  constexpr int STB = NBLK * BLKB;        // bytes of one landed tile
  // per-frame gates: 3 stages of one tile; per-token gates: 2 stages of three
  // tiles (A copy, B hi, B lo)
  const int NS = beta_tok ? 2 : 3;
  const int SSTR = beta_tok ? 3 * STB : STB;  // stage stride
  constexpr int NN = 2 * D;               // MMA N (columns of D)
  constexpr int SD = D + 1;               // padded row stride of I + beta A, then X
  constexpr int BL = D / 16;              // register block edge per thread

  const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  float* Mo = Mout + (bh * (T + 1) + f) * mat;
  float* Ro = Rout + (bh * (T + 1) + f) * mat;
  const int t = f - 1;

  if (f >= 1 && (t == 0 || t == T - 1)) {  // anchor: no write (X = I, W = 0)
    for (int e = tid; e < D * D; e += blockDim.x) {
      const int i = e / D, j = e % D;
      Mo[e] = (i == j) ? 1.f : 0.f;
      Ro[e] = 0.f;
    }
    return;
  }
  const int ntok = (f == 0) ? n_text : N;
  const CUtensorMap* mk = (f == 0) ? &map_tk : &map_k;
  const CUtensorMap* mv = (f == 0) ? &map_tv : &map_v;
  const int frame_coord = (f == 0) ? 0 : t;
  const float bt = beta_tok ? 1.f : beta[bh * (T + 1) + f];
  const float* btok = beta_tok ? beta + bh * ((size_t)n_text + (size_t)T * N) +
                                     (f == 0 ? 0 : (size_t)n_text + (size_t)t * N)
                               : nullptr;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // the first 1 KB: barriers; then phase 1: the TMA ring (3 x STB, or
  // 2 x 3 x STB with per-token gates); phase 2 (after the MMAs): I + beta A,
  // inverted in place.  beta W goes from TMEM straight to Rout.  With per-frame
  // gates this is under 100 KB, so two CTAs share an SM and one's inversion
  // overlaps the other's loads and MMAs.
  uint64_t* full = (uint64_t*)smem;
  uint8_t* stages = smem + 1024;
  float* Ash = (float*)stages;         // [D][SD]  I + beta A, then X
  uint64_t* empty = full + 3;
  uint64_t* conv_full = empty + 3;   // per-token gates: operands prepared
  uint64_t* acc_full = conv_full + 3;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  int* abort_flag = (int*)(tmem_slot + 1);
  __shared__ float prow[2][D], pcol[2][D];

  const int nst = (ntok + BT - 1) / BT;
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) {
      ptx::mbar_init(full + i, 1);
      ptx::mbar_init(empty + i, 1);
      ptx::mbar_init(conv_full + i, 192);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  // per-token gates at d = 128 hold two 256-column accumulators
  const uint32_t ncols = (beta_tok && 2 * NN > 256) ? 512u : 256u;
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, ncols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (nst > 0) {
    if (warp == 0 && lane == 0) {
      int issued = 0;
      for (int s = 0; s < nst; ++s) {
        const int st = s % NS, use = s / NS;
        if (use > 0 &&
            !ptx::wait_bounded(empty + st, (use - 1) & 1, abort_flag, status, kDevTimeout))
          break;
        ptx::mbar_arrive_expect_tx(full + st, STB);
        uint8_t* dst = stages + st * SSTR;
        for (int kb = 0; kb < D / 64; ++kb)
          ptx::tma_load_5d(dst + kb * BLKB, mk, full + st, kb * 64, h, s * BT, frame_coord, b);
        for (int vb = 0; vb < D / 64; ++vb)
          ptx::tma_load_5d(dst + (D / 64 + vb) * BLKB, mv, full + st, vb * 64, h, s * BT,
                           frame_coord, b);
        issued = s + 1;
      }
      if (*abort_flag) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int s = max(0, issued - NS); s < issued; ++s)
          while (!ptx::mbar_try_wait(full + s % NS, (s / NS) & 1) &&
                 ptx::globaltimer_ns() - t0 < 2000000000ull) {}
      }
    } else if (warp == 1 && lane == 0) {
      const uint32_t idesc = beta_tok ? ptx::idesc_f16(128, NN, 0, 1, 1)   // fp16 tiles
                                      : ptx::idesc_f16(128, NN, 1, 1, 1);  // bf16 tiles
      const uint32_t base = ptx::smem_u32(stages);
      bool ok = true;
      for (int s = 0; s < nst; ++s) {
        const int st = s % NS;
        if (!(ok = ptx::wait_bounded(beta_tok ? conv_full + st : full + st, (s / NS) & 1,
                                     abort_flag, status, kDevTimeout)))
          break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          const uint32_t a = base + st * SSTR + kk * 2048;  // 16 token rows of 128 B
          const uint64_t ad = ptx::sdesc_mn_sw128(a, BLKB);
          if (!beta_tok) {
            ptx::mma_ss(tmem, ad, ad, idesc, (s > 0 || kk > 0) ? 1u : 0u);
          } else {
            ptx::mma_ss(tmem, ad, ptx::sdesc_mn_sw128(a + STB, BLKB), idesc,
                        (s > 0 || kk > 0) ? 1u : 0u);
            ptx::mma_ss(tmem + NN, ad, ptx::sdesc_mn_sw128(a + 2 * STB, BLKB), idesc,
                        (s > 0 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::mma_commit(empty + st);
      }
      if (ok) ptx::mma_commit(acc_full);
      ptx::mma_commit(drain);
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(drain, 0) && ptx::globaltimer_ns() - t0 < 2000000000ull) {}
    } else if (beta_tok && warp >= 2) {
      // rescale each landed tile: row r of a 64-token block is token s*BT + r
      const int ct = tid - 64;  // 0..191
      bool bad = false;
      for (int s = 0; s < nst; ++s) {
        const int st = s % NS;
        if (!ptx::wait_bounded(full + st, (s / NS) & 1, abort_flag, status, kDevTimeout)) break;
        uint8_t* base = stages + st * SSTR;
        for (int ch = ct; ch < STB / 16; ch += 192) {
          const int off = ch * 16;
          const int row = (off % BLKB) / 128;
          const int tok = s * BT + row;
          const float bw = tok < ntok ? btok[tok] : 0.f;
          const uint4 raw = *reinterpret_cast<const uint4*>(base + off);
          const __nv_bfloat162* in2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          uint4 av, hv, lv;
          __half2* a2 = reinterpret_cast<__half2*>(&av);
          __half2* h2 = reinterpret_cast<__half2*>(&hv);
          __half2* l2 = reinterpret_cast<__half2*>(&lv);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 x = __bfloat1622float2(in2[q]);
            const float y0 = x.x * bw, y1 = x.y * bw;
            bad |= !(fabsf(x.x) <= 65504.f) || !(fabsf(x.y) <= 65504.f) ||
                   !(fabsf(y0) <= 65504.f) || !(fabsf(y1) <= 65504.f);
            a2[q] = __floats2half2_rn(x.x, x.y);  // exact for bf16 in the fp16 range
            h2[q] = __floats2half2_rn(y0, y1);
            const float2 hf = __half22float2(h2[q]);
            l2[q] = __floats2half2_rn(y0 - hf.x, y1 - hf.y);
          }
          *reinterpret_cast<uint4*>(base + off) = av;
          *reinterpret_cast<uint4*>(base + STB + off) = hv;
          *reinterpret_cast<uint4*>(base + 2 * STB + off) = lv;
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(conv_full + st);
      }
      if (bad) atomicOr(status, kDevRange);
    }
  }
  // ---- epilogue: D -> shared (all warps) ----
  bool have = true;
  if (nst > 0) have = ptx::wait_bounded(acc_full, 0, abort_flag, status, kDevTimeout);
  __syncthreads();  // every MMA done reading the stages: reuse them for Ash
  ptx::tc_fence_after();
  {
    const int q = warp & 3, part = warp >> 2;  // part 0: A columns, 1: W columns
    const int i = q * 32 + lane;               // row (key channel) = TMEM lane
    const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + part * D;
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      if (nst > 0 && have) {
        ptx::tmem_ld32(taddr + 32 * c, r);
        ptx::tmem_wait_ld();
        if (beta_tok) {  // add the lo-part accumulator
          uint32_t r2[32];
          ptx::tmem_ld32(taddr + NN + 32 * c, r2);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            r[e] = __float_as_uint(__uint_as_float(r[e]) + __uint_as_float(r2[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      if (i < D) {
        if (part == 0) {  // I + beta A (VDA), or I - beta A (frozen-state rule)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = 32 * c + e;
            const float x = bt * __uint_as_float(r[e]);
            Ash[i * SD + j] = (frozen ? -x : x) + (i == j ? 1.f : 0.f);
          }
        } else {          // beta W: row i, columns 32 c .. 32 c + 31
          float4* dst = reinterpret_cast<float4*>(Ro + (size_t)i * D + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(bt * __uint_as_float(r[4 * e]), bt * __uint_as_float(r[4 * e + 1]),
                                 bt * __uint_as_float(r[4 * e + 2]), bt * __uint_as_float(r[4 * e + 3]));
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, ncols);
  }

  // ---- in-place Gauss-Jordan inversion of I + beta A, in registers ----
  const int ty = tid >> 4, tx = tid & 15;
  float a[BL][BL];
#pragma unroll
  for (int i = 0; i < BL; ++i)
#pragma unroll
    for (int c = 0; c < BL; ++c) a[i][c] = Ash[(ty * BL + i) * SD + tx * BL + c];
  int buf = 0;
  for (int pb = 0; pb < (frozen ? 0 : 16); ++pb) {  // the frozen-state rule has no inverse
#pragma unroll
    for (int r = 0; r < BL; ++r) {
      const int p = pb * BL + r;
      if (ty == pb) {
#pragma unroll
        for (int c = 0; c < BL; ++c) prow[buf][tx * BL + c] = a[r][c];
      }
      if (tx == pb) {
#pragma unroll
        for (int i = 0; i < BL; ++i) pcol[buf][ty * BL + i] = a[i][r];
      }
      __syncthreads();
      const float piv = 1.f / prow[buf][p];
      float rp[BL], cp[BL];
#pragma unroll
      for (int c = 0; c < BL; ++c) rp[c] = prow[buf][tx * BL + c] * piv;
#pragma unroll
      for (int i = 0; i < BL; ++i) cp[i] = pcol[buf][ty * BL + i];
#pragma unroll
      for (int i = 0; i < BL; ++i)
#pragma unroll
        for (int c = 0; c < BL; ++c) a[i][c] = fmaf(-cp[i], rp[c], a[i][c]);
      if (ty == pb) {
#pragma unroll
        for (int c = 0; c < BL; ++c) a[r][c] = rp[c];
      }
      if (tx == pb) {
#pragma unroll
        for (int i = 0; i < BL; ++i) a[i][r] = -cp[i] * piv;
      }
      if (ty == pb && tx == pb) a[r][r] = piv;
      buf ^= 1;
    }
  }
  // ---- X (registers) -> Mout; video frames: beta W -> Rout; text frame:
  // X -> shared, R = X beta W -> Rout (the text state) ----
#pragma unroll
  for (int i = 0; i < BL; ++i) {
    float* dst = Mo + (size_t)(ty * BL + i) * D + tx * BL;
#pragma unroll
    for (int c = 0; c < BL; c += 4)
      *reinterpret_cast<float4*>(dst + c) = make_float4(a[i][c], a[i][c + 1], a[i][c + 2], a[i][c + 3]);
  }
  if (frozen || f >= 1) return;  // Rout already holds beta W (uniform over the CTA)
  __syncthreads();
#pragma unroll
  for (int i = 0; i < BL; ++i)
#pragma unroll
    for (int c = 0; c < BL; ++c) Ash[(ty * BL + i) * SD + tx * BL + c] = a[i][c];
  __syncthreads();
  // Text frame: R = X (beta W), W read back from Rout (written by this CTA's
  // epilogue before the inversion's barriers).  Thread (ty, tx) computes rows
  // ty*BL .. +BL-1 and the column groups {4 tx .. 4 tx + 3} + 4 D/4 g for
  // g < BL/4 (groups of four columns, D/4 apart), so that the sixteen threads
  // of a row group read W as consecutive float4.
  constexpr int NGR = BL / 4;
  float acc[BL][BL];
#pragma unroll
  for (int i = 0; i < BL; ++i)
#pragma unroll
    for (int c = 0; c < BL; ++c) acc[i][c] = 0.f;
#pragma unroll 4
  for (int l = 0; l < D; ++l) {
    float xv[BL], wv[BL];
#pragma unroll
    for (int i = 0; i < BL; ++i) xv[i] = Ash[(ty * BL + i) * SD + l];
#pragma unroll
    for (int g = 0; g < NGR; ++g) {
      const float4 w4 = *reinterpret_cast<const float4*>(Ro + (size_t)l * D + g * (D / NGR) + tx * 4);
      wv[4 * g] = w4.x;
      wv[4 * g + 1] = w4.y;
      wv[4 * g + 2] = w4.z;
      wv[4 * g + 3] = w4.w;
    }
#pragma unroll
    for (int i = 0; i < BL; ++i)
#pragma unroll
      for (int c = 0; c < BL; ++c) acc[i][c] = fmaf(xv[i], wv[c], acc[i][c]);
  }
  __syncthreads();  // every thread has read W before R overwrites it
#pragma unroll
  for (int i = 0; i < BL; ++i) {
    float* dst = Ro + (size_t)(ty * BL + i) * D + tx * 4;
#pragma unroll
    for (int g = 0; g < NGR; ++g)
      *reinterpret_cast<float4*>(dst + g * (D / NGR)) =
          make_float4(acc[i][4 * g], acc[i][4 * g + 1], acc[i][4 * g + 2], acc[i][4 * g + 3]);
  }
}

template <int D>
static cudaError_t launch_frame_tc_t(const VdaArgs& a, cudaStream_t st) {
  CUtensorMap mk, mv, mtk, mtv;
  const uint64_t Hh = a.H, B = a.B, N = a.N, T = a.T, nt = a.n_text > 0 ? a.n_text : 1;
  const uint32_t box[5] = {64, 1, 64, 1, 1};
  {
    const uint64_t dims[5] = {(uint64_t)D, Hh, N, T, B};
    const uint64_t str[4] = {(uint64_t)D * 2, Hh * D * 2, N * Hh * D * 2, T * N * Hh * D * 2};
    if (!make_tmap(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.k, dims, str, box) ||
        !make_tmap(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.v, dims, str, box))
      return cudaErrorInvalidValue;
  }
  {
    // text: one "frame" of n_text tokens; with no text the maps point at k
    // (never read: the text frame then issues no copy)
    const void* tk = a.n_text > 0 ? a.text_k : a.k;
    const void* tv = a.n_text > 0 ? a.text_v : a.v;
    const uint64_t dims[5] = {(uint64_t)D, Hh, nt, 1, B};
    const uint64_t str[4] = {(uint64_t)D * 2, Hh * D * 2, nt * Hh * D * 2, nt * Hh * D * 2};
    if (!make_tmap(&mtk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, tk, dims, str, box) ||
        !make_tmap(&mtv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, tv, dims, str, box))
      return cudaErrorInvalidValue;
  }
  constexpr int SD = D + 1;
  // alignment slack + barriers (1 KB) + the larger of the TMA ring and I + beta A
  const size_t stage_bytes = (a.beta_tok ? 6 : 3) * (size_t)(D / 32) * 64 * 128;
  const size_t mat_bytes = (size_t)D * SD * 4;
  const size_t sm = 1024 + 1024 + (stage_bytes > mat_bytes ? stage_bytes : mat_bytes);
  auto kern = vda_frame_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.T + 1, a.H, a.B), 256, sm, st>>>(mk, mv, mtk, mtv, a.beta, a.alpha, a.Mf, a.Rf,
                                                 a.H, a.T, a.N, a.n_text, a.beta_tok, a.frozen,
                                                 a.status);
  return cudaGetLastError();
}

cudaError_t launch_frame_tc(const VdaArgs& a, cudaStream_t st) {
  if (a.D == 128) return launch_frame_tc_t<128>(a, st);
  if (a.D == 64) return launch_frame_tc_t<64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
