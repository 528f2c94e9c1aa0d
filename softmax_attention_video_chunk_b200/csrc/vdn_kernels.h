// Internal launch interface between the C ABI layer and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/vdn.h"

namespace vdn {

struct VdaArgs {
  int B, H, T, N, D, C, R, n_text;
  vdn_dtype dtype;
  float init_scale;  // 0.5 (text counted once over the two scans) or 1
  const void *k, *v, *text_k, *text_v;
  const float *beta, *alpha;
  // workspace: per-frame transitions [B][H][T+1][D][D]; chunk maps
  // [2][B][H][nc][D][D]; boundary states [B][H][nc+1][D][D]
  float *Mf, *Rf, *CM, *CR, *FS, *GS;
  bool tc;      // frame statistics on the tensor cores (bf16, d in {64, 128})
  bool beta_tok;  // beta per token: [B][H][n_text + L]
  bool frozen;    // frozen-state rule: M = (I - A) Diag(alpha), R = W (no inverse)
  int scan_mode;  // 0: chosen from the shape; 1: scan over frames; 2: compose chunks
  int* status;  // device status word
};

cudaError_t launch_frame_tc(const VdaArgs& a, cudaStream_t st);

cudaError_t launch_vda_states(const VdaArgs& a, cudaStream_t st);
// true: launch_vda_states runs the direct frame scan (2 kernels in all);
// false: chunk composition + chunk scan (3 kernels in all)
bool vda_frame_scan_route(const VdaArgs& a);
cudaError_t launch_vda_readout_simt(const VdaArgs& a, const void* q, float* o_l, cudaStream_t st);
cudaError_t launch_gather_boundary(const VdaArgs& a, float* F, float* G, cudaStream_t st);

struct AttnArgs {
  int B, H, T, N, D, C, R;
  vdn_dtype dtype;
  float scale;
  const void *q, *k, *v;
  int n_text_keys;                  // text tokens joining the Softmax keys (0: none)
  const void *text_k, *text_v;      // [B, n_text, H, D]
  const void* text_q = nullptr;     // text queries [B, n_text, H, D]: dense text rows
};
cudaError_t launch_attn_simt(const AttnArgs& a, float* o_s, cudaStream_t st);

struct ProjArgs {
  int B, H, L, D, D_out;
  vdn_dtype dtype, out_dtype;
  float eps;
  const float *o_s, *o_l;  // [B*L, H*D] fp32
  const void *gates;       // [2][B*L][H*D]
  const void *W_soft, *W_lin;  // [H*D][D_out]
  float* rinv;             // [B*L*H] scratch
  void* out;
};
cudaError_t launch_proj_simt(const ProjArgs& a, cudaStream_t st);

// VDA-Prep (linear-branch feature map); k == nullptr skips K/V, q == nullptr Q.
struct PrepArgs {
  int B, H, T, gh, gw, D;
  bool bf16;
  float eps;
  const void *q, *k, *v;                         // [B, T*gh*gw, H, D]
  const float *wk_s, *wk_t, *wv_s, *wv_t;        // [H*D][9], [H*D][5]
  void *q_out, *k_out, *v_out;                   // [B, T*gh*gw, H, D]
  int* status;
};
cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st);

}  // namespace vdn
