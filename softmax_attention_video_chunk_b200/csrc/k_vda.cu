// Video Delta Attention state path on CUDA cores, exact FP32 arithmetic.
//
// "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation", Video Delta Attention paragraphs (joint objective, normal
// equation (I + A_t) S_t = Diag(alpha_t) S_{t-1} + W_t, inverse in key-channel
// space, FP32 state) and Implementation section ("Chunk-wise scans": each
// frame is an affine map S -> M_t S + R_t, frames are composed per chunk and
// the chunk sequence is scanned in both directions, keeping only the
// chunk-boundary states; "Small-matrix inverse": Gauss-Jordan elimination
// that emits the transition and injection terms directly).
//
//   vda_frame_solve  : per frame, A_t = beta K^T K, W_t = beta K^T V, then
//                      Gauss-Jordan on [I + A_t | I] -> X_t = (I + A_t)^-1;
//                      writes X_t and W_t (the affine map of frame t is
//                      S -> X_t (Diag(alpha_t) S + W_t)).  Frame index 0 is the
//                      text "virtual frame" (it writes S_text = X_0 W_0); anchor
//                      frames emit X = I, W = 0 (excluded from both scans, decay
//                      kept).
//   vda_frame_scan   : for short clips, the scan over frames directly, keeping
//                      only the chunk-boundary states.
//   vda_chunk_compose: per chunk and direction, the product of its frames'
//                      affine maps in scan order.
//   vda_chunk_scan   : per (b, h, direction, 32-column slice of S), the
//                      sequential scan over chunks from the text initial state;
//                      writes FS[j] (after chunks < j) and GS[j] (after chunks >= j).
//   vda_readout      : per frame, S_t = Diag(gf) FS + Diag(gr) GS with the
//                      decay bridge across the window, then o_l = q^T S_t.
#include "vdn_common.cuh"
#include "vdn_kernels.h"

namespace vdn {
int sm_count();

// ---------------------------------------------------------------------------
// S1 + S2: frame statistics and Gauss-Jordan solve.
// Per-frame maps (both frame kernels write the same): for video frame t,
// Mf[1 + t] = X_t and Rf[1 + t] = W_t, with X_t = (I + beta A_t)^-1 and the
// update S_t = X_t (Diag(alpha_t) S_{t-1} + W_t) (VDA), or X_t = I - beta A_t
// and S_t = X_t Diag(alpha_t) S_{t-1} + W_t (frozen-state rule); anchor
// frames write X = I, W = 0 (S_t = Diag(alpha_t) S_{t-1} under both).  The
// text virtual frame writes Mf[0] = X_0 and its state Rf[0] = X_0 W_0 (VDA)
// or W_0 (frozen).
// ---------------------------------------------------------------------------
template <int D, typename TIn>
__global__ void __launch_bounds__(256)
vda_frame_solve_kernel(const TIn* __restrict__ k, const TIn* __restrict__ v,
                       const TIn* __restrict__ text_k, const TIn* __restrict__ text_v,
                       const float* __restrict__ beta, const float* __restrict__ alpha,
                       float* __restrict__ Mout, float* __restrict__ Rout, int H, int T,
                       int N, int n_text, bool beta_tok, bool frozen) {
  constexpr int RT = D / 16;  // rows per thread
  constexpr int CT = D / 16;  // cols per thread
  constexpr int BN = 16;      // tokens per staged tile
  constexpr int SD = 3 * D + 1;
  const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
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

  const size_t rs = (size_t)H * D;  // row stride of [., H, D] tensors
  const TIn *K, *V;
  int n;
  if (f == 0) {
    K = text_k + (size_t)b * n_text * rs + (size_t)h * D;
    V = text_v + (size_t)b * n_text * rs + (size_t)h * D;
    n = n_text;
  } else {
    const size_t r0 = (size_t)b * T * N + (size_t)t * N;
    K = k + r0 * rs + (size_t)h * D;
    V = v + r0 * rs + (size_t)h * D;
    n = N;
  }
  // per-frame gate (scales A and W at the end) or per-token gates (fold into
  // the staged values)
  const float bt = beta_tok ? 1.f : beta[bh * (T + 1) + f];
  const float* btok = beta_tok ? beta + bh * ((size_t)n_text + (size_t)T * N) +
                                     (f == 0 ? 0 : (size_t)n_text + (size_t)t * N)
                               : nullptr;

  extern __shared__ float smem[];
  float* aug = smem;              // [D][SD]
  float* Ks = aug + D * SD;       // [BN][D]
  float* Vs = Ks + BN * D;        // [BN][D]
  __shared__ float Bs[BN];

  const int ty = tid >> 4, tx = tid & 15;
  float accA[RT][CT], accW[RT][CT];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int m = 0; m < CT; ++m) accA[r][m] = accW[r][m] = 0.f;

  for (int n0 = 0; n0 < n; n0 += BN) {
    __syncthreads();
    for (int e = tid; e < BN * D; e += blockDim.x) {
      const int rr = e / D, cc = e % D;
      const bool ok = n0 + rr < n;
      Ks[e] = ok ? to_f(K[(size_t)(n0 + rr) * rs + cc]) : 0.f;
      Vs[e] = ok ? to_f(V[(size_t)(n0 + rr) * rs + cc]) : 0.f;
    }
    for (int rr = tid; rr < BN; rr += blockDim.x)
      Bs[rr] = (n0 + rr < n) ? (btok ? btok[n0 + rr] : 1.f) : 0.f;
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < BN; ++rr) {
      float a[RT], kk[CT], vv[CT];
      const float bn = Bs[rr];
#pragma unroll
      for (int r = 0; r < RT; ++r) a[r] = Ks[rr * D + ty * RT + r];
#pragma unroll
      for (int m = 0; m < CT; ++m) {
        kk[m] = Ks[rr * D + tx + 16 * m] * bn;
        vv[m] = Vs[rr * D + tx + 16 * m] * bn;
      }
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int m = 0; m < CT; ++m) {
          accA[r][m] = fmaf(a[r], kk[m], accA[r][m]);
          accW[r][m] = fmaf(a[r], vv[m], accW[r][m]);
        }
    }
  }
  __syncthreads();
  if (frozen) {  // frozen-state rule: X = I - beta A, W = beta W
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int i = ty * RT + r;
#pragma unroll
      for (int m = 0; m < CT; ++m) {
        const int j = tx + 16 * m;
        Mo[i * D + j] = (i == j ? 1.f : 0.f) - bt * accA[r][m];
        Ro[i * D + j] = bt * accW[r][m];
      }
    }
    return;
  }
  // [I + beta A | I | beta W]; video frames write beta W now and eliminate
  // the first two blocks only (-> X); the text frame also carries beta W
  // through (-> X beta W, its state)
  const int ncol = (f == 0) ? 3 * D : 2 * D;
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const int i = ty * RT + r;
#pragma unroll
    for (int m = 0; m < CT; ++m) {
      const int j = tx + 16 * m;
      aug[i * SD + j] = bt * accA[r][m] + (i == j ? 1.f : 0.f);
      aug[i * SD + 2 * D + j] = bt * accW[r][m];
      if (f >= 1) Ro[i * D + j] = bt * accW[r][m];
    }
  }
  for (int e = tid; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e % D;
    aug[i * SD + D + j] = (i == j) ? 1.f : 0.f;
  }

  // Gauss-Jordan without pivoting (I + A is symmetric positive definite with
  // eigenvalues >= 1).  Columns < p of the left block are already unit
  // vectors and stay unchanged.
  float* prow = Ks;  // 3D floats (Ks+Vs hold 2*BN*D >= 4D floats)
  float* pcol = Ks + 3 * D;
  const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  for (int p = 0; p < D; ++p) {
    __syncthreads();
    const float inv = 1.f / aug[p * SD + p];
    for (int j = p + tid; j < ncol; j += blockDim.x) prow[j] = aug[p * SD + j] * inv;
    for (int i = tid; i < D; i += blockDim.x) pcol[i] = aug[i * SD + p];
    __syncthreads();
    for (int i = warp; i < D; i += nwarps) {
      const float fi = pcol[i];
      float* row = aug + i * SD;
      if (i == p) {
        for (int j = p + lane; j < ncol; j += 32) row[j] = prow[j];
      } else {
        for (int j = p + lane; j < ncol; j += 32) row[j] = fmaf(-fi, prow[j], row[j]);
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e % D;
    Mo[e] = aug[i * SD + D + j];
    if (f == 0) Ro[e] = aug[i * SD + 2 * D + j];
  }
}

// ---------------------------------------------------------------------------
// S3: chunk composition.  Forward: frames s..e-1 in increasing order;
// reverse: e-1..s.  With M_t = X_t Diag(alpha_t):
//   (M, R) <- (X_t (Diag(alpha_t) M), X_t (Diag(alpha_t) R + W_t))      VDA
//   (M, R) <- (X_t (Diag(alpha_t) M), X_t (Diag(alpha_t) R) + W_t)      frozen
// starting from the first frame's (X_t Diag(alpha_t), X_t W_t) (frozen: W_t).
// Both products act on columns independently, so each CTA composes one
// 32-column slice of M and R (the whole X_t is staged once per frame).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
vda_chunk_compose_kernel(const float* __restrict__ Mf, const float* __restrict__ Rf,
                         const float* __restrict__ alpha, float* __restrict__ CM,
                         float* __restrict__ CR, int B, int H, int T, int C, bool frozen) {
  constexpr int RT = D / 32, SD = D + 1;
  const int cb = (blockIdx.x % (D / 32)) * 32;
  const int c = blockIdx.x / (D / 32);
  const int h = blockIdx.y;
  const int b = blockIdx.z >> 1, dir = blockIdx.z & 1;
  const int nc = (T + C - 1) / C;
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  const int s = c * C, e = min(T, (c + 1) * C);
  extern __shared__ float smem[];
  float* Mt = smem;            // [D][SD]  X_t
  float* Ma = Mt + D * SD;     // [D][32]  slice of the composed M
  float* Ra = Ma + D * 32;     // [D][32]  slice of the composed R

  const int nfr = e - s;
  for (int step = 0; step < nfr; ++step) {
    const int t = dir == 0 ? s + step : e - 1 - step;
    const float* Xg = Mf + (bh * (T + 1) + 1 + t) * mat;
    const float* Wg = Rf + (bh * (T + 1) + 1 + t) * mat;
    const float* al = alpha != nullptr ? alpha + (bh * T + t) * D : nullptr;
    __syncthreads();
    for (int q = tid; q < D * D; q += blockDim.x) Mt[(q / D) * SD + (q % D)] = Xg[q];
    // this thread's 4 x 4 block of the slices, before the products
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int i = ty * RT + r;
      const float ai = al != nullptr ? al[i] : 1.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = tx * 4 + m;
        const float w = Wg[i * D + cb + j];
        if (step == 0) {  // M = X_t Diag(alpha_t) (no product); R pre-product = W_t
          Ma[i * 32 + j] = Xg[i * D + cb + j] * (al != nullptr ? al[cb + j] : 1.f);
          Ra[i * 32 + j] = w;
        } else {
          Ma[i * 32 + j] *= ai;
          Ra[i * 32 + j] = frozen ? ai * Ra[i * 32 + j] : fmaf(ai, Ra[i * 32 + j], w);
        }
      }
    }
    if (step == 0 && frozen) continue;  // (X_t Diag(alpha_t), W_t): no product
    __syncthreads();
    const bool do_m = step > 0;
    float am[RT][4], ar[RT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int m = 0; m < 4; ++m) am[r][m] = ar[r][m] = 0.f;
    if (do_m) {
#pragma unroll 4
      for (int l = 0; l < D; ++l) {
        const float4 bm = *reinterpret_cast<const float4*>(Ma + l * 32 + tx * 4);
        const float4 br = *reinterpret_cast<const float4*>(Ra + l * 32 + tx * 4);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const float a = Mt[(ty * RT + r) * SD + l];
          am[r][0] = fmaf(a, bm.x, am[r][0]);
          am[r][1] = fmaf(a, bm.y, am[r][1]);
          am[r][2] = fmaf(a, bm.z, am[r][2]);
          am[r][3] = fmaf(a, bm.w, am[r][3]);
          ar[r][0] = fmaf(a, br.x, ar[r][0]);
          ar[r][1] = fmaf(a, br.y, ar[r][1]);
          ar[r][2] = fmaf(a, br.z, ar[r][2]);
          ar[r][3] = fmaf(a, br.w, ar[r][3]);
        }
      }
    } else {  // first frame: the R product only
#pragma unroll 4
      for (int l = 0; l < D; ++l) {
        const float4 br = *reinterpret_cast<const float4*>(Ra + l * 32 + tx * 4);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const float a = Mt[(ty * RT + r) * SD + l];
          ar[r][0] = fmaf(a, br.x, ar[r][0]);
          ar[r][1] = fmaf(a, br.y, ar[r][1]);
          ar[r][2] = fmaf(a, br.z, ar[r][2]);
          ar[r][3] = fmaf(a, br.w, ar[r][3]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int i = ty * RT + r;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = tx * 4 + m;
        if (do_m) Ma[i * 32 + j] = am[r][m];
        Ra[i * 32 + j] = frozen ? ar[r][m] + Wg[i * D + cb + j] : ar[r][m];
      }
    }
  }
  __syncthreads();
  // layout [2 (direction)][B][H][nc][D][D]
  float* CMo = CM + ((size_t)dir * B * H * nc + bh * nc + c) * mat;
  float* CRo = CR + ((size_t)dir * B * H * nc + bh * nc + c) * mat;
  for (int q = tid; q < D * 32; q += blockDim.x) {
    const int i = q >> 5, j = q & 31;
    CMo[i * D + cb + j] = Ma[q];
    CRo[i * D + cb + j] = Ra[q];
  }
}

// ---------------------------------------------------------------------------
// S4: bidirectional chunk scan over 32-column slices of the state.
// FS[j] = state after chunks < j (FS[0] = init), GS[j] = state after chunks
// >= j (GS[nc] = init); init = S_text / 2 (or S_text, text_full).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
vda_chunk_scan_kernel(const float* __restrict__ Rf, const float* __restrict__ CM,
                      const float* __restrict__ CR, float* __restrict__ FS,
                      float* __restrict__ GS, int B, int H, int T, int C, float init_scale) {
  constexpr int RT = D / 32, SD = D + 1;
  const int cb = blockIdx.x * 32, h = blockIdx.y, b = blockIdx.z >> 1, dir = blockIdx.z & 1;
  const int nc = (T + C - 1) / C;
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  extern __shared__ float smem[];
  float* Ms = smem;          // [D][SD]
  float* Ss = Ms + D * SD;   // [D][32]
  const float* St = Rf + (bh * (T + 1) + 0) * mat;  // text state
  for (int q = tid; q < D * 32; q += blockDim.x) {
    const int i = q >> 5, j = q & 31;
    Ss[q] = init_scale * St[i * D + cb + j];
  }
  float* OUT = dir == 0 ? FS : GS;
  const size_t dir_off = (size_t)dir * B * H * nc;
  const int j_first = dir == 0 ? 0 : nc;
  __syncthreads();
  for (int q = tid; q < D * 32; q += blockDim.x) {
    const int i = q >> 5, j = q & 31;
    OUT[(bh * (nc + 1) + j_first) * mat + i * D + cb + j] = Ss[q];
  }
  for (int step = 0; step < nc; ++step) {
    const int cc = dir == 0 ? step : nc - 1 - step;
    const float* Mg = CM + (dir_off + bh * nc + cc) * mat;
    const float* Rg = CR + (dir_off + bh * nc + cc) * mat;
    __syncthreads();
    for (int q = tid; q < D * D; q += blockDim.x) Ms[(q / D) * SD + (q % D)] = Mg[q];
    __syncthreads();
    float acc[RT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[r][m] = 0.f;
    for (int l = 0; l < D; ++l) {
      const float4 sv = *reinterpret_cast<const float4*>(Ss + l * 32 + tx * 4);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float a = Ms[(ty * RT + r) * SD + l];
        acc[r][0] = fmaf(a, sv.x, acc[r][0]);
        acc[r][1] = fmaf(a, sv.y, acc[r][1]);
        acc[r][2] = fmaf(a, sv.z, acc[r][2]);
        acc[r][3] = fmaf(a, sv.w, acc[r][3]);
      }
    }
    __syncthreads();
    const int jout = dir == 0 ? cc + 1 : cc;
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int i = ty * RT + r;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = tx * 4 + m;
        const float val = acc[r][m] + Rg[i * D + cb + j];
        Ss[i * 32 + j] = val;
        OUT[(bh * (nc + 1) + jout) * mat + i * D + cb + j] = val;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// S3+S4 for short clips: the bidirectional scan run directly over the frames,
// S <- X_t (Diag(alpha_t) S + W_t) (frozen-state rule: X_t Diag(alpha_t) S +
// W_t), keeping only the chunk-boundary states (FS[k] after the frames of
// chunks < k, GS[k] after the frames of chunks >= k).  It needs T sequential
// steps instead of ceil(T / C), but does one product per frame instead of the
// composition's two per frame plus the chunk scan, and reads the per-frame
// maps directly.  Anchor frames (no write) only decay: S <- Diag(alpha_t) S.
// One CTA per 32-column slice of S and direction.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256, 2)
vda_frame_scan_kernel(const float* __restrict__ Mf, const float* __restrict__ Rf,
                      const float* __restrict__ alpha, float* __restrict__ FS,
                      float* __restrict__ GS, int B, int H, int T, int C, float init_scale,
                      bool frozen) {
  constexpr int RT = D / 32, SD = D + 4;  // row stride keeps float4 stores aligned
  const int cb = blockIdx.x * 32, h = blockIdx.y, b = blockIdx.z >> 1, dir = blockIdx.z & 1;
  const int nc = (T + C - 1) / C;
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const size_t mat = (size_t)D * D;
  const size_t bh = (size_t)b * H + h;
  extern __shared__ float smem[];
  float* Ms = smem;          // [D][SD]
  float* Ss = Ms + D * SD;   // [D][32]
  const float* St = Rf + (bh * (T + 1) + 0) * mat;  // text state
  for (int q = tid; q < D * 32; q += blockDim.x) {
    const int i = q >> 5, j = q & 31;
    Ss[q] = init_scale * St[i * D + cb + j];
  }
  float* OUT = dir == 0 ? FS : GS;
  __syncthreads();
  {
    const int k0 = dir == 0 ? 0 : nc;
    for (int q = tid; q < D * 32; q += blockDim.x) {
      const int i = q >> 5, j = q & 31;
      OUT[(bh * (nc + 1) + k0) * mat + i * D + cb + j] = Ss[q];
    }
  }
  // X_t of the next frame is loaded into registers (D*D/4/256 float4 per
  // thread, all in flight at once) while the current frame's product runs
  constexpr int NV = D * D / 4 / 256;
  float4 mv[NV];
  auto frame_of = [&](int step) { return dir == 0 ? step : T - 1 - step; };
  auto is_anchor = [&](int t) { return t == 0 || t == T - 1; };
  auto load_m = [&](int t) {
    const float4* Mg = reinterpret_cast<const float4*>(Mf + (bh * (T + 1) + 1 + t) * mat);
#pragma unroll
    for (int k = 0; k < NV; ++k) mv[k] = Mg[tid + k * 256];
  };
  if (T > 0 && !is_anchor(frame_of(0))) load_m(frame_of(0));
  for (int step = 0; step < T; ++step) {
    const int t = frame_of(step);
    const bool anchor = is_anchor(t);
    const float* Rg = Rf + (bh * (T + 1) + 1 + t) * mat;
    float acc[RT][4];
    __syncthreads();
    if (anchor) {  // X_t = I, W_t = 0
      const float* al = alpha != nullptr ? alpha + (bh * T + t) * D : nullptr;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int i = ty * RT + r;
        const float a = al != nullptr ? al[i] : 1.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[r][m] = a * Ss[i * 32 + tx * 4 + m];
      }
      if (step + 1 < T && !is_anchor(frame_of(step + 1))) load_m(frame_of(step + 1));
    } else {
      // this thread's 4 x 4 block of the slice: Diag(alpha_t) S (+ W_t, VDA)
      const float* al = alpha != nullptr ? alpha + (bh * T + t) * D : nullptr;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const int i = ty * RT + r;
        const float a = al != nullptr ? al[i] : 1.f;
        float4 sv = *reinterpret_cast<const float4*>(Ss + i * 32 + tx * 4);
        if (frozen) {
          sv.x *= a; sv.y *= a; sv.z *= a; sv.w *= a;
        } else {
          const float4 wv = *reinterpret_cast<const float4*>(Rg + i * D + cb + tx * 4);
          sv.x = fmaf(a, sv.x, wv.x); sv.y = fmaf(a, sv.y, wv.y);
          sv.z = fmaf(a, sv.z, wv.z); sv.w = fmaf(a, sv.w, wv.w);
        }
        *reinterpret_cast<float4*>(Ss + i * 32 + tx * 4) = sv;
      }
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int q = tid + k * 256;
        const int i = q / (D / 4), c4 = q % (D / 4);
        *reinterpret_cast<float4*>(Ms + i * SD + 4 * c4) = mv[k];
      }
      __syncthreads();
      if (step + 1 < T && !is_anchor(frame_of(step + 1))) load_m(frame_of(step + 1));
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[r][m] = 0.f;
      // X_t is symmetric (the inverse of the symmetric I + beta A_t; the
      // frozen rule's I - beta A_t is symmetric too), so X_t[i][l] is read as
      // X_t[l][i]: this thread's RT rows at column l are RT consecutive floats
      // of row l, one vector load instead of RT scalar ones
#pragma unroll 4
      for (int l = 0; l < D; ++l) {
        const float4 sv = *reinterpret_cast<const float4*>(Ss + l * 32 + tx * 4);
        float xa[RT];
        if constexpr (RT == 4) {
          const float4 x4 = *reinterpret_cast<const float4*>(Ms + l * SD + ty * RT);
          xa[0] = x4.x; xa[1] = x4.y; xa[2] = x4.z; xa[3] = x4.w;
        } else if constexpr (RT == 2) {
          const float2 x2 = *reinterpret_cast<const float2*>(Ms + l * SD + ty * RT);
          xa[0] = x2.x; xa[1] = x2.y;
        } else {
          xa[0] = Ms[l * SD + ty];
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          acc[r][0] = fmaf(xa[r], sv.x, acc[r][0]);
          acc[r][1] = fmaf(xa[r], sv.y, acc[r][1]);
          acc[r][2] = fmaf(xa[r], sv.z, acc[r][2]);
          acc[r][3] = fmaf(xa[r], sv.w, acc[r][3]);
        }
      }
      if (frozen) {
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          const int i = ty * RT + r;
          const float4 rv = *reinterpret_cast<const float4*>(Rg + i * D + cb + tx * 4);
          acc[r][0] += rv.x;
          acc[r][1] += rv.y;
          acc[r][2] += rv.z;
          acc[r][3] += rv.w;
        }
      }
    }
    __syncthreads();
    // chunk boundary reached after this frame: forward after the last frame of
    // chunk k-1 (k = (t+1)/C, or nc after the last frame), reverse after the
    // first frame of chunk k = t/C
    int kout = -1;
    if (dir == 0) {
      if (t == T - 1) kout = nc;
      else if ((t + 1) % C == 0) kout = (t + 1) / C;
    } else if (t % C == 0) {
      kout = t / C;
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int i = ty * RT + r;
      *reinterpret_cast<float4*>(Ss + i * 32 + tx * 4) =
          make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      if (kout >= 0)
        *reinterpret_cast<float4*>(OUT + (bh * (nc + 1) + kout) * mat + i * D + cb + tx * 4) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    }
  }
}

// ---------------------------------------------------------------------------
// S6: readout with the decay bridge, per frame (CUDA cores, FP32).
// ---------------------------------------------------------------------------
template <int D, typename TIn>
__global__ void __launch_bounds__(256)
vda_readout_kernel(const TIn* __restrict__ q, const float* __restrict__ alpha,
                   const float* __restrict__ Rf, const float* __restrict__ FS,
                   const float* __restrict__ GS, float* __restrict__ o_l, int H, int T,
                   int N, int C, int R, float init_scale) {
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
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
  constexpr int NG = D / 32;  // float4 groups per thread
  const int tok = tid >> 3, cg = (tid & 7) * 4;
  const size_t rs = (size_t)H * D;
  const size_t row0 = (size_t)b * T * N + (size_t)t * N;
  for (int n0 = 0; n0 < N; n0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * D; e += blockDim.x) {
      const int rr = e / D, cc = e % D;
      Qs[rr * (D + 1) + cc] =
          (n0 + rr < N) ? to_f(q[(row0 + n0 + rr) * rs + (size_t)h * D + cc]) : 0.f;
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
    if (n0 + tok < N) {
      float* dst = o_l + (row0 + n0 + tok) * rs + (size_t)h * D;
#pragma unroll
      for (int g = 0; g < NG; ++g)
        *reinterpret_cast<float4*>(dst + cg + 32 * g) =
            make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    }
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
// Chunk composition + chunk scan, or the direct frame scan: whichever the
// wave-count model puts first (or the one a.scan_mode forces).  Sequential
// steps per CTA: composition 2 C - 1 products then nc scan steps; direct
// scan T products.  CTAs: the composition runs 2 B H nc (D / 32) of them,
// both scans 2 B H (D / 32); two CTAs per SM.
bool vda_frame_scan_route(const VdaArgs& a) {
  if (a.scan_mode != 0) return a.scan_mode == 1;
  const long long nc = (a.T + a.C - 1) / a.C;
  const long long slots = 2LL * sm_count();
  const long long cta_scan = 2LL * a.B * a.H * (a.D / 32);
  const long long cta_comp = cta_scan * nc;
  const long long waves_scan = (cta_scan + slots - 1) / slots;
  const long long waves_comp = (cta_comp + slots - 1) / slots;
  const long long cost_chunk = waves_comp * (2LL * a.C - 1) + waves_scan * nc;
  const long long cost_direct = waves_scan * (long long)a.T;
  return cost_direct <= cost_chunk;
}

template <int D, typename TIn>
static cudaError_t launch_vda_states_t(const VdaArgs& a, cudaStream_t st) {
  const int H = a.H, B = a.B, T = a.T, nc = (a.T + a.C - 1) / a.C;
  if (a.tc) {
    cudaError_t e = launch_frame_tc(a, st);
    if (e != cudaSuccess) return e;
  } else {
    const size_t sm = sizeof(float) * ((size_t)D * (3 * D + 1) + 2 * 16 * D);
    auto kern = vda_frame_solve_kernel<D, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(T + 1, H, B), 256, sm, st>>>(
        (const TIn*)a.k, (const TIn*)a.v, (const TIn*)a.text_k, (const TIn*)a.text_v, a.beta,
        a.alpha, a.Mf, a.Rf, H, T, a.N, a.n_text, a.beta_tok, a.frozen);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (vda_frame_scan_route(a)) {
    const size_t sm = sizeof(float) * ((size_t)D * (D + 4) + (size_t)D * 32);
    auto kern = vda_frame_scan_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(D / 32, H, 2 * B), 256, sm, st>>>(a.Mf, a.Rf, a.alpha, a.FS, a.GS, B, H, T, a.C,
                                                  a.init_scale, a.frozen);
    return cudaGetLastError();
  }
  {
    const size_t sm = sizeof(float) * ((size_t)D * (D + 1) + 2 * (size_t)D * 32);
    auto kern = vda_chunk_compose_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3((D / 32) * nc, H, 2 * B), 256, sm, st>>>(a.Mf, a.Rf, a.alpha, a.CM, a.CR, B, H,
                                                         T, a.C, a.frozen);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t sm = sizeof(float) * ((size_t)D * (D + 1) + (size_t)D * 32);
    auto kern = vda_chunk_scan_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    kern<<<dim3(D / 32, H, 2 * B), 256, sm, st>>>(a.Rf, a.CM, a.CR, a.FS, a.GS, B, H, T, a.C,
                                                  a.init_scale);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_vda_states(const VdaArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == VDN_BF16;
  switch (a.D) {
    case 32: return bf ? launch_vda_states_t<32, __nv_bfloat16>(a, st) : launch_vda_states_t<32, float>(a, st);
    case 64: return bf ? launch_vda_states_t<64, __nv_bfloat16>(a, st) : launch_vda_states_t<64, float>(a, st);
    case 128: return bf ? launch_vda_states_t<128, __nv_bfloat16>(a, st) : launch_vda_states_t<128, float>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <int D, typename TIn>
static cudaError_t launch_readout_t(const VdaArgs& a, const void* q, float* o_l,
                                   cudaStream_t st) {
  const size_t sm = sizeof(float) * ((size_t)D * D + 32 * (D + 1));
  auto kern = vda_readout_kernel<D, TIn>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.T, a.H, a.B), 256, sm, st>>>((const TIn*)q, a.alpha, a.Rf, a.FS, a.GS, o_l,
                                             a.H, a.T, a.N, a.C, a.R, a.init_scale);
  return cudaGetLastError();
}

cudaError_t launch_vda_readout_simt(const VdaArgs& a, const void* q, float* o_l,
                                    cudaStream_t st) {
  const bool bf = a.dtype == VDN_BF16;
  switch (a.D) {
    case 32: return bf ? launch_readout_t<32, __nv_bfloat16>(a, q, o_l, st) : launch_readout_t<32, float>(a, q, o_l, st);
    case 64: return bf ? launch_readout_t<64, __nv_bfloat16>(a, q, o_l, st) : launch_readout_t<64, float>(a, q, o_l, st);
    case 128: return bf ? launch_readout_t<128, __nv_bfloat16>(a, q, o_l, st) : launch_readout_t<128, float>(a, q, o_l, st);
  }
  return cudaErrorInvalidValue;
}

// Copy the per-query-chunk boundary states out of FS/GS:
// F[c] = FS[max(0, c-R)], G[c] = GS[min(nc, c+R+1)].
__global__ void gather_boundary_kernel(const float* __restrict__ FS, const float* __restrict__ GS,
                                       float* __restrict__ F, float* __restrict__ G, int nc,
                                       int R, size_t mat) {
  const int c = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int jf = max(0, c - R), jr = min(nc, c + R + 1);
  const float* fs = FS + (bh * (nc + 1) + jf) * mat;
  const float* gs = GS + (bh * (nc + 1) + jr) * mat;
  for (size_t e = threadIdx.x; e < mat; e += blockDim.x) {
    if (F) F[(bh * nc + c) * mat + e] = fs[e];
    if (G) G[(bh * nc + c) * mat + e] = gs[e];
  }
}

cudaError_t launch_gather_boundary(const VdaArgs& a, float* F, float* G, cudaStream_t st) {
  const int nc = (a.T + a.C - 1) / a.C;
  gather_boundary_kernel<<<dim3(nc, a.B * a.H), 256, 0, st>>>(a.FS, a.GS, F, G, nc, a.R,
                                                              (size_t)a.D * a.D);
  return cudaGetLastError();
}

}  // namespace vdn
