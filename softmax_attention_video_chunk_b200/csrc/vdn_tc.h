// Internal interface of the tensor-core (tcgen05 / TMA) path.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/vdn.h"
#include "vdn_kernels.h"

namespace vdn {

struct TcSizes {
  size_t vt_bytes, wt_bytes, x_bytes;
};

struct TcAttnArgs {
  int B, H, T, N, D, C, R, L, Lp;
  float scale;
  const void *q, *k, *v;  // bf16 [B, L, H, D]
  __half* vt;             // fp16 [B*H][D][Lp], V transposed (keys contiguous)
  int* status;            // device status word
  int n_text_keys;        // text tokens joining the Softmax keys (0: none)
  int ntp;                // n_text_keys rounded up to 64
  const void *text_k, *text_v;  // bf16 [B, n_text, H, D]
  __half* vt_text;        // fp16 [B*H][D][ntp], text V transposed
  const void* text_q = nullptr;  // bf16 [B, n_text, H, D]: text queries (dense rows)
  int kv_split = 1;              // text rows: key tiles split over this many CTAs
  float* part = nullptr;         // [kv_split][B*n_text*H][D] partial outputs
  float* ml = nullptr;           // [kv_split][B*n_text*H][2] running max and sum
};

struct TcFwdArgs {
  int B, H, T, N, D, L, D_out;
  vdn_dtype out_dtype;
  float eps;
  const void* gates;           // bf16 [2][B][L][H][D]
  const void *W_soft, *W_lin;  // bf16 [H*D][D_out]
  __half* wt;                  // fp16 [D_out][2*H*D]
  __half* x;                   // fp16 [B*L][2*H*D] = [g_s*o_s | g_l*RMS(o_l)]
  // MXFP8 projection: when xq != nullptr the Softmax and readout epilogues
  // write x as E4M3 codes [B*L][2*H*D] and its UE8M0 scales (atom layout of
  // mx_scale_bytes) instead of fp16
  uint8_t* xq = nullptr;
  uint8_t* sfa = nullptr;
  void* out;                   // [B*L][D_out]
  const void* q;
  VdaArgs vda;
  int* status;
};

bool use_tc(const vdn_params& p);
TcSizes tc_sizes(const vdn_params& p);
TcAttnArgs tc_attn_args(const vdn_params& p, const AttnArgs& a, void* vt, int* status);
TcFwdArgs tc_fwd_args(const vdn_params& p, const VdaArgs& va, const TcAttnArgs& t,
                      const void* W_soft, const void* W_lin, const void* gates, void* out,
                      void* wt, void* x);

cudaError_t launch_convert_v(const TcAttnArgs& t, cudaStream_t st);
cudaError_t launch_convert_w(const TcFwdArgs& f, cudaStream_t st);
// fused != nullptr: epilogue writes g_s * o_s as fp16 into f->x; else o_s fp32.
cudaError_t launch_attn_tc(const TcAttnArgs& t, const TcFwdArgs* fused, float* o_s,
                           cudaStream_t st);
cudaError_t launch_readout_tc(const TcFwdArgs& f, cudaStream_t st);
cudaError_t launch_gemm_tc(const TcFwdArgs& f, cudaStream_t st);

// MXFP8 projection (k_mxfp8.cu)
size_t mx_scale_bytes(long long rows_padded, int cols);
cudaError_t launch_mx_quant(const __half* x, uint8_t* codes, uint8_t* scales, long long rows,
                            long long rows_padded, int cols, cudaStream_t st);
cudaError_t launch_mx_gemm(const uint8_t* xq, const uint8_t* sfa, const uint8_t* wq,
                           const uint8_t* sfb, void* out, vdn_dtype out_dtype, int M, int Nout,
                           int K, int* status, cudaStream_t st);

}  // namespace vdn
