// C ABI of libvdn: argument validation, workspace layout, launch sequence.
//
// The call sequence follows the pages' forward (method section of "Video
// DeltaNet: A Video-Native Hybrid Attention for Livestream Video
// Generation"): the VDA state path (frame statistics -> Gauss-Jordan solve ->
// chunk composition -> bidirectional chunk scan), the window+anchor Softmax,
// the linear readout with its decay bridge, then the gated dual output
// projection.  Every step runs in this library's kernels; PyTorch (or any
// caller) only provides device memory and the stream.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "vdn_common.cuh"
#include "vdn_kernels.h"
#include "vdn_tc.h"

namespace vdn {

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t status, Mf, Rf, CM, CR, FS, GS;   // VDA state path
  size_t o_s, o_l, rinv;                   // CUDA-core path intermediates
  size_t vt, wt, x;                        // tensor-core path operands
  size_t xq, sfa, wq, sfb;                 // MXFP8 projection operands and scales
  size_t vda_end;                          // end of the VDA state-path prefix
  size_t total;
};

static WsLayout layout(const vdn_params& p) {
  WsLayout w;
  memset(&w, 0, sizeof(w));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t B = p.B, H = p.H, T = p.T, d = p.d_k;
  const size_t L = (size_t)p.T * p.N;
  const size_t nc = (p.T + p.chunk - 1) / p.chunk;
  const size_t mat = d * d * sizeof(float);
  w.status = take(256);
  w.Mf = take(B * H * (T + 1) * mat);
  w.Rf = take(B * H * (T + 1) * mat);
  w.CM = take(2 * B * H * nc * mat);
  w.CR = take(2 * B * H * nc * mat);
  w.FS = take(B * H * (nc + 1) * mat);
  w.GS = take(B * H * (nc + 1) * mat);
  w.vda_end = off;
  if (use_tc(p)) {
    TcSizes s = tc_sizes(p);
    w.vt = take(s.vt_bytes);
    w.wt = take(s.wt_bytes);
    w.x = take(s.x_bytes);
    if (p.flags & VDN_FLAG_PROJ_MXFP8) {
      const size_t K = 2 * H * d, M = B * L, No = p.D_out;
      w.xq = take(M * K);
      w.sfa = take(mx_scale_bytes((long long)M, (int)K));
      w.wq = take(No * K);
      w.sfb = take(mx_scale_bytes((long long)((No + 255) / 256 * 256), (int)K));
    }
  } else {
    w.o_s = take(B * L * H * d * sizeof(float));
    w.o_l = take(B * L * H * d * sizeof(float));
    w.rinv = take(B * L * H * sizeof(float));
  }
  w.total = off;
  return w;
}

static vdn_status validate_params(const vdn_params* p) {
  if (p == nullptr) return VDN_ERR_INVALID_ARG;
  if (p->flags & ~(unsigned)(VDN_FLAG_TEXT_FULL | VDN_FLAG_SIMT | VDN_FLAG_TEXT_SOFTMAX |
                             VDN_FLAG_BETA_PER_TOKEN | VDN_FLAG_FROZEN_STATE |
                             VDN_FLAG_SCAN_FRAMES | VDN_FLAG_SCAN_CHUNKS |
                             VDN_FLAG_PROJ_MXFP8))
    return VDN_ERR_INVALID_ARG;
  if ((p->flags & VDN_FLAG_SCAN_FRAMES) && (p->flags & VDN_FLAG_SCAN_CHUNKS))
    return VDN_ERR_INVALID_ARG;
  if ((p->dtype != VDN_F32 && p->dtype != VDN_BF16) ||
      (p->out_dtype != VDN_F32 && p->out_dtype != VDN_BF16))
    return VDN_ERR_DTYPE;
  if (p->B < 1 || p->H < 1 || p->T < 1 || p->N < 1 || p->n_text < 0 || p->chunk < 1 ||
      p->window_radius < 0 || p->D_out < 1)
    return VDN_ERR_SHAPE;
  if (p->d_k != p->d_v) return VDN_ERR_UNSUPPORTED;
  if (p->d_k != 32 && p->d_k != 64 && p->d_k != 128) return VDN_ERR_UNSUPPORTED;
  if (p->D_out % 8 != 0) return VDN_ERR_SHAPE;
  if (!(p->softmax_scale >= 0.f) || isinf(p->softmax_scale)) return VDN_ERR_INVALID_ARG;
  if (!(p->rms_eps >= 0.f) || isinf(p->rms_eps)) return VDN_ERR_INVALID_ARG;
  // index ranges: tokens and grid sizes
  const double L = (double)p->T * p->N;
  if (L > 2147483647.0 / 2) return VDN_ERR_SHAPE;
  if ((double)p->B * L * p->H * p->d_k > 9.0e15) return VDN_ERR_SHAPE;
  if (p->H > 65535 || p->B > 32767 || p->T + 1 > 2147483647 / 2) return VDN_ERR_SHAPE;
  return VDN_OK;
}

static inline bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

static vdn_status check_ptr(const void* ptr, bool required) {
  if (ptr == nullptr) return required ? VDN_ERR_INVALID_ARG : VDN_OK;
  return aligned16(ptr) ? VDN_OK : VDN_ERR_ALIGNMENT;
}

// Bytes of the workspace prefix the VDA state path uses (status word,
// per-frame transitions, chunk maps, boundary states).
size_t vda_scratch_bytes(const vdn_params& p) { return layout(p).vda_end; }

vdn_status boundary_states_impl(const vdn_params* p, const void* k, const void* v,
                                const float* beta, const float* alpha, const void* text_k,
                                const void* text_v, float* F, float* G, void* workspace,
                                vdn_stream_t stream);

int sm_count();

static vdn_status validate_prep(const vdn_prep_params* p) {
  if (p == nullptr) return VDN_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->T < 1 || p->grid_h < 1 || p->grid_w < 1) return VDN_ERR_SHAPE;
  if (p->d != 32 && p->d != 64 && p->d != 128) return VDN_ERR_UNSUPPORTED;
  if (p->spatial_taps != 3 || p->temporal_taps != 5) return VDN_ERR_UNSUPPORTED;
  if (p->dtype != VDN_F32 && p->dtype != VDN_BF16) return VDN_ERR_DTYPE;
  if (!(p->l2_eps >= 0.f) || p->l2_eps > 1.f) return VDN_ERR_INVALID_ARG;
  // the TMA frame coordinate and the grid extents are 32-bit
  if ((long long)p->B * p->T > (1ll << 30) || (long long)p->grid_h * p->grid_w > (1ll << 30))
    return VDN_ERR_SHAPE;
  // launch grid: y = grid rows, z = (batch, head, K or V)
  if (p->grid_h > 65535 || 2LL * p->B * p->H > 65535) return VDN_ERR_SHAPE;
  return VDN_OK;
}

static vdn_status check_ws(const vdn_params* p, const void* ws, size_t ws_bytes) {
  const WsLayout w = layout(*p);
  if (ws == nullptr || ws_bytes < w.total) return VDN_ERR_WORKSPACE;
  if (((uintptr_t)ws & 255u) != 0) return VDN_ERR_ALIGNMENT;
  return VDN_OK;
}

#define VDN_TRY(expr)                        \
  do {                                       \
    vdn_status _s = (expr);                  \
    if (_s != VDN_OK) return _s;             \
  } while (0)

#define VDN_CUDA(expr)                                   \
  do {                                                   \
    if ((expr) != cudaSuccess) return VDN_ERR_CUDA;      \
  } while (0)

// The projection out = x [W_soft; W_lin] of f.B * f.L rows from the fp16
// operand f.x and W^T (converted into f.wt here): fp16 tcgen05 GEMM, or with
// VDN_FLAG_PROJ_MXFP8 both operands quantised to MXFP8 and the block-scaled
// fp8 GEMM.  With f.xq set, the epilogues have already written x in MXFP8.
static cudaError_t launch_projection(const vdn_params* p, const TcFwdArgs& f, char* ws,
                                     const WsLayout& w, cudaStream_t st) {
  cudaError_t e = launch_convert_w(f, st);
  if (e != cudaSuccess) return e;
  if (!(p->flags & VDN_FLAG_PROJ_MXFP8)) return launch_gemm_tc(f, st);
  const long long M = (long long)f.B * f.L;
  const int K = 2 * f.H * f.D, No = f.D_out;
  uint8_t *xq = (uint8_t*)(ws + w.xq), *sfa = (uint8_t*)(ws + w.sfa);
  uint8_t *wq = (uint8_t*)(ws + w.wq), *sfb = (uint8_t*)(ws + w.sfb);
  if (f.xq == nullptr &&
      (e = launch_mx_quant(f.x, xq, sfa, M, (M + 127) / 128 * 128, K, st)) != cudaSuccess)
    return e;
  if ((e = launch_mx_quant(f.wt, wq, sfb, No, (No + 255) / 256 * 256, K, st)) != cudaSuccess)
    return e;
  return launch_mx_gemm(xq, sfa, wq, sfb, f.out, f.out_dtype, (int)M, No, K, f.status, st);
}

static VdaArgs vda_args(const vdn_params* p, const void* k, const void* v, const float* beta,
                        const float* alpha, const void* text_k, const void* text_v, char* ws) {
  const WsLayout w = layout(*p);
  VdaArgs a;
  a.B = p->B; a.H = p->H; a.T = p->T; a.N = p->N; a.D = p->d_k; a.C = p->chunk;
  a.R = p->window_radius; a.n_text = p->n_text; a.dtype = p->dtype;
  a.init_scale = (p->flags & VDN_FLAG_TEXT_FULL) ? 1.f : 0.5f;
  a.k = k; a.v = v; a.text_k = text_k; a.text_v = text_v; a.beta = beta; a.alpha = alpha;
  a.Mf = (float*)(ws + w.Mf); a.Rf = (float*)(ws + w.Rf);
  a.CM = (float*)(ws + w.CM); a.CR = (float*)(ws + w.CR);
  a.FS = (float*)(ws + w.FS); a.GS = (float*)(ws + w.GS);
  a.tc = use_tc(*p);
  a.beta_tok = (p->flags & VDN_FLAG_BETA_PER_TOKEN) != 0;
  a.frozen = (p->flags & VDN_FLAG_FROZEN_STATE) != 0;
  a.scan_mode = (p->flags & VDN_FLAG_SCAN_FRAMES) ? 1 : ((p->flags & VDN_FLAG_SCAN_CHUNKS) ? 2 : 0);
  a.status = (int*)(ws + w.status);
  return a;
}

static AttnArgs attn_args(const vdn_params* p, const void* q, const void* k, const void* v,
                          const void* text_k, const void* text_v) {
  AttnArgs a;
  a.B = p->B; a.H = p->H; a.T = p->T; a.N = p->N; a.D = p->d_k; a.C = p->chunk;
  a.R = p->window_radius; a.dtype = p->dtype;
  a.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.f / sqrtf((float)p->d_k);
  a.q = q; a.k = k; a.v = v;
  a.n_text_keys = (p->flags & VDN_FLAG_TEXT_SOFTMAX) ? p->n_text : 0;
  a.text_k = text_k; a.text_v = text_v;
  return a;
}

static vdn_status common_inputs(const vdn_params* p, const void* q, const void* k, const void* v,
                                const float* beta, const float* alpha, const void* text_k,
                                const void* text_v, bool need_q) {
  VDN_TRY(check_ptr(q, need_q));
  VDN_TRY(check_ptr(k, true));
  VDN_TRY(check_ptr(v, true));
  VDN_TRY(check_ptr(beta, true));
  VDN_TRY(check_ptr(alpha, false));
  VDN_TRY(check_ptr(text_k, p->n_text > 0));
  VDN_TRY(check_ptr(text_v, p->n_text > 0));
  return VDN_OK;
}

}  // namespace vdn

using namespace vdn;

extern "C" {

int vdn_abi_version(void) { return VDN_ABI_VERSION; }

const char* vdn_status_string(vdn_status s) {
  switch (s) {
    case VDN_OK: return "VDN_OK";
    case VDN_ERR_INVALID_ARG: return "VDN_ERR_INVALID_ARG: missing pointer or invalid flag/value";
    case VDN_ERR_SHAPE: return "VDN_ERR_SHAPE: size out of range";
    case VDN_ERR_DTYPE: return "VDN_ERR_DTYPE: unsupported dtype";
    case VDN_ERR_ALIGNMENT: return "VDN_ERR_ALIGNMENT: pointer not 16-byte aligned (workspace: 256)";
    case VDN_ERR_WORKSPACE: return "VDN_ERR_WORKSPACE: workspace missing or too small";
    case VDN_ERR_CUDA: return "VDN_ERR_CUDA: CUDA runtime error";
    case VDN_ERR_TIMEOUT: return "VDN_ERR_TIMEOUT: bounded device wait expired";
    case VDN_ERR_UNSUPPORTED: return "VDN_ERR_UNSUPPORTED: configuration not served";
    case VDN_ERR_RANGE: return "VDN_ERR_RANGE: value outside the range of an fp16 operand";
  }
  return "VDN_ERR_UNKNOWN";
}

vdn_status vdn_params_init(vdn_params* p, int B, int H, int T, int N, int d, int n_text,
                           vdn_dtype dtype) {
  if (p == nullptr) return VDN_ERR_INVALID_ARG;
  memset(p, 0, sizeof(*p));
  p->B = B; p->H = H; p->T = T; p->N = N; p->d_k = d; p->d_v = d; p->n_text = n_text;
  p->D_out = H * d; p->chunk = 5; p->window_radius = 1; p->dtype = dtype;
  p->out_dtype = VDN_F32; p->softmax_scale = 0.f; p->rms_eps = 1e-6f; p->flags = 0;
  return validate_params(p);
}

vdn_status vdn_workspace_bytes(const vdn_params* p, size_t* bytes) {
  if (bytes == nullptr) return VDN_ERR_INVALID_ARG;
  VDN_TRY(validate_params(p));
  *bytes = layout(*p).total;
  return VDN_OK;
}

vdn_status vdn_vda_boundary_states(const vdn_params* p, const void* k, const void* v,
                                   const float* beta, const float* alpha, const void* text_k,
                                   const void* text_v, float* F, float* G, void* workspace,
                                   size_t workspace_bytes, vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  VDN_TRY(common_inputs(p, nullptr, k, v, beta, alpha, text_k, text_v, false));
  VDN_TRY(check_ptr(F, false));
  VDN_TRY(check_ptr(G, false));
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  VdaArgs a = vda_args(p, k, v, beta, alpha, text_k, text_v, ws);
  VDN_CUDA(launch_vda_states(a, st));
  if (F != nullptr || G != nullptr) VDN_CUDA(launch_gather_boundary(a, F, G, st));
  return VDN_OK;
}

}  // extern "C"

namespace vdn {
// The boundary-state path of vdn_vda_boundary_states_noalloc: the same
// launches as vdn_vda_boundary_states on a scratch region whose first
// vda_scratch_bytes(*p) bytes are usable (checked by the caller).
vdn_status boundary_states_impl(const vdn_params* p, const void* k, const void* v,
                                const float* beta, const float* alpha, const void* text_k,
                                const void* text_v, float* F, float* G, void* workspace,
                                vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  VDN_TRY(common_inputs(p, nullptr, k, v, beta, alpha, text_k, text_v, false));
  VDN_TRY(check_ptr(F, false));
  VDN_TRY(check_ptr(G, false));
  if (workspace == nullptr) return VDN_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  VdaArgs a = vda_args(p, k, v, beta, alpha, text_k, text_v, ws);
  VDN_CUDA(launch_vda_states(a, st));
  if (F != nullptr || G != nullptr) VDN_CUDA(launch_gather_boundary(a, F, G, st));
  return VDN_OK;
}
}  // namespace vdn

extern "C" {

vdn_status vdn_hybrid_attn_branches(const vdn_params* p, const void* q, const void* k,
                                    const void* v, const float* beta, const float* alpha,
                                    const void* text_k, const void* text_v, float* o_soft,
                                    float* o_lin, void* workspace, size_t workspace_bytes,
                                    vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  VDN_TRY(common_inputs(p, q, k, v, beta, alpha, text_k, text_v, true));
  VDN_TRY(check_ptr(o_soft, false));
  VDN_TRY(check_ptr(o_lin, false));
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const WsLayout w = layout(*p);
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  const bool tc = use_tc(*p);
  if (o_lin != nullptr) {
    VdaArgs a = vda_args(p, k, v, beta, alpha, text_k, text_v, ws);
    VDN_CUDA(launch_vda_states(a, st));
    VDN_CUDA(launch_vda_readout_simt(a, q, o_lin, st));
  }
  if (o_soft != nullptr) {
    AttnArgs a = attn_args(p, q, k, v, text_k, text_v);
    if (tc) {
      TcAttnArgs t = tc_attn_args(*p, a, ws + w.vt, (int*)(ws + w.status));
      VDN_CUDA(launch_convert_v(t, st));
      VDN_CUDA(launch_attn_tc(t, nullptr, o_soft, st));
    } else {
      VDN_CUDA(launch_attn_simt(a, o_soft, st));
    }
  }
  return VDN_OK;
}

}  // extern "C"

namespace vdn {
// The forward with the linear branch reading its own q_l, k_l, v_l (equal to
// q, k, v unless the caller passes the linear feature map's outputs).
static vdn_status fwd_impl(const vdn_params* p, const void* q, const void* k, const void* v,
                           const void* q_l, const void* k_l, const void* v_l, const float* beta,
                           const float* alpha, const void* text_k, const void* text_v,
                           const void* W_o_soft, const void* W_o_lin, const void* gates,
                           void* out, void* workspace, size_t workspace_bytes,
                           vdn_stream_t stream, const vdn_stage_events* ev) {
  VDN_TRY(validate_params(p));
  if ((p->flags & VDN_FLAG_PROJ_MXFP8) && !use_tc(*p)) return VDN_ERR_UNSUPPORTED;
  VDN_TRY(common_inputs(p, q, k, v, beta, alpha, text_k, text_v, true));
  VDN_TRY(check_ptr(q_l, true));
  VDN_TRY(check_ptr(k_l, true));
  VDN_TRY(check_ptr(v_l, true));
  VDN_TRY(check_ptr(W_o_soft, true));
  VDN_TRY(check_ptr(W_o_lin, true));
  VDN_TRY(check_ptr(gates, true));
  VDN_TRY(check_ptr(out, true));
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  if (ev != nullptr)
    for (int i = 0; i <= VDN_STAGES; ++i)
      if (ev->events[i] == nullptr) return VDN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  auto mark = [&](int i) -> cudaError_t {
    return ev ? cudaEventRecord((cudaEvent_t)ev->events[i], st) : cudaSuccess;
  };
  char* ws = (char*)workspace;
  const WsLayout w = layout(*p);
  VDN_CUDA(mark(0));
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  VdaArgs va = vda_args(p, k_l, v_l, beta, alpha, text_k, text_v, ws);
  AttnArgs aa = attn_args(p, q, k, v, text_k, text_v);
  if (use_tc(*p)) {
    TcAttnArgs t = tc_attn_args(*p, aa, ws + w.vt, (int*)(ws + w.status));
    TcFwdArgs f = tc_fwd_args(*p, va, t, W_o_soft, W_o_lin, gates, out, ws + w.wt, ws + w.x);
    f.q = q_l;  // the readout's queries
    if (p->flags & VDN_FLAG_PROJ_MXFP8) {
      // the Softmax and readout epilogues write x in MXFP8; scale bytes of
      // the rows past B*L in the last 128-row group read as the smallest scale
      f.xq = (uint8_t*)(ws + w.xq);
      f.sfa = (uint8_t*)(ws + w.sfa);
      const long long M = (long long)f.B * f.L;
      const int K = 2 * f.H * f.D;
      if (M % 128 != 0) {
        const size_t group = (size_t)(K / 128) * 512u;
        VDN_CUDA(cudaMemsetAsync(f.sfa + (size_t)(M / 128) * group, 0, group, st));
      }
    }
    VDN_CUDA(launch_vda_states(va, st));
    VDN_CUDA(mark(1));
    VDN_CUDA(launch_convert_v(t, st));
    VDN_CUDA(mark(2));
    VDN_CUDA(launch_attn_tc(t, &f, nullptr, st));
    VDN_CUDA(mark(3));
    VDN_CUDA(launch_readout_tc(f, st));
    VDN_CUDA(mark(4));
    VDN_CUDA(launch_projection(p, f, ws, w, st));
    VDN_CUDA(mark(5));
    return VDN_OK;
  }
  float* o_s = (float*)(ws + w.o_s);
  float* o_l = (float*)(ws + w.o_l);
  VDN_CUDA(launch_vda_states(va, st));
  VDN_CUDA(mark(1));
  VDN_CUDA(mark(2));
  VDN_CUDA(launch_attn_simt(aa, o_s, st));
  VDN_CUDA(mark(3));
  VDN_CUDA(launch_vda_readout_simt(va, q_l, o_l, st));
  VDN_CUDA(mark(4));
  ProjArgs pa;
  pa.B = p->B; pa.H = p->H; pa.L = p->T * p->N; pa.D = p->d_k; pa.D_out = p->D_out;
  pa.dtype = p->dtype; pa.out_dtype = p->out_dtype; pa.eps = p->rms_eps;
  pa.o_s = o_s; pa.o_l = o_l; pa.gates = gates; pa.W_soft = W_o_soft; pa.W_lin = W_o_lin;
  pa.rinv = (float*)(ws + w.rinv); pa.out = out;
  VDN_CUDA(launch_proj_simt(pa, st));
  VDN_CUDA(mark(5));
  return VDN_OK;
}

}  // namespace vdn

extern "C" {

vdn_status vdn_hybrid_attn_fwd_staged(const vdn_params* p, const void* q, const void* k,
                                      const void* v, const float* beta, const float* alpha,
                                      const void* text_k, const void* text_v,
                                      const void* W_o_soft, const void* W_o_lin,
                                      const void* gates, void* out, void* workspace,
                                      size_t workspace_bytes, vdn_stream_t stream,
                                      const vdn_stage_events* ev) {
  return fwd_impl(p, q, k, v, q, k, v, beta, alpha, text_k, text_v, W_o_soft, W_o_lin, gates,
                  out, workspace, workspace_bytes, stream, ev);
}

vdn_status vdn_hybrid_attn_fwd_split(const vdn_params* p, const void* q, const void* k,
                                     const void* v, const void* q_lin, const void* k_lin,
                                     const void* v_lin, const float* beta, const float* alpha,
                                     const void* text_k, const void* text_v,
                                     const void* W_o_soft, const void* W_o_lin,
                                     const void* gates, void* out, void* workspace,
                                     size_t workspace_bytes, vdn_stream_t stream,
                                     const vdn_stage_events* ev) {
  return fwd_impl(p, q, k, v, q_lin, k_lin, v_lin, beta, alpha, text_k, text_v, W_o_soft,
                  W_o_lin, gates, out, workspace, workspace_bytes, stream, ev);
}

vdn_status vdn_hybrid_attn_fwd(const vdn_params* p, const void* q, const void* k, const void* v,
                               const float* beta, const float* alpha, const void* text_k,
                               const void* text_v, const void* W_o_soft, const void* W_o_lin,
                               const void* gates, void* out, void* workspace,
                               size_t workspace_bytes, vdn_stream_t stream) {
  return vdn_hybrid_attn_fwd_staged(p, q, k, v, beta, alpha, text_k, text_v, W_o_soft, W_o_lin,
                                    gates, out, workspace, workspace_bytes, stream, nullptr);
}

vdn_status vdn_hybrid_attn_operand(const vdn_params* p, const void* q, const void* k,
                                   const void* v, const float* beta, const float* alpha,
                                   const void* text_k, const void* text_v, const void* gates,
                                   void* x, void* workspace, size_t workspace_bytes,
                                   vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  if (!use_tc(*p)) return VDN_ERR_UNSUPPORTED;
  VDN_TRY(common_inputs(p, q, k, v, beta, alpha, text_k, text_v, true));
  VDN_TRY(check_ptr(gates, true));
  VDN_TRY(check_ptr(x, true));
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const WsLayout w = layout(*p);
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  VdaArgs va = vda_args(p, k, v, beta, alpha, text_k, text_v, ws);
  AttnArgs aa = attn_args(p, q, k, v, text_k, text_v);
  TcAttnArgs t = tc_attn_args(*p, aa, ws + w.vt, (int*)(ws + w.status));
  // the fused Softmax and readout epilogues write straight into the caller's x
  TcFwdArgs f = tc_fwd_args(*p, va, t, nullptr, nullptr, gates, nullptr, ws + w.wt, x);
  f.q = q;
  VDN_CUDA(launch_vda_states(va, st));
  VDN_CUDA(launch_convert_v(t, st));
  VDN_CUDA(launch_attn_tc(t, &f, nullptr, st));
  VDN_CUDA(launch_readout_tc(f, st));
  return VDN_OK;
}

vdn_status vdn_output_projection(const vdn_params* p, long long rows, const void* x,
                                 const void* W_o_soft, const void* W_o_lin, void* out,
                                 void* workspace, size_t workspace_bytes, vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  if (!use_tc(*p)) return VDN_ERR_UNSUPPORTED;
  if (rows < 1 || rows > 2147483647LL / 2) return VDN_ERR_SHAPE;
  VDN_TRY(check_ptr(x, true));
  VDN_TRY(check_ptr(W_o_soft, true));
  VDN_TRY(check_ptr(W_o_lin, true));
  VDN_TRY(check_ptr(out, true));
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const WsLayout w = layout(*p);
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  TcFwdArgs f;
  memset(&f, 0, sizeof(f));
  f.B = 1; f.L = (int)rows; f.H = p->H; f.D = p->d_k; f.T = 1; f.N = (int)rows;
  f.D_out = p->D_out; f.out_dtype = p->out_dtype; f.eps = p->rms_eps;
  f.W_soft = W_o_soft; f.W_lin = W_o_lin; f.wt = (__half*)(ws + w.wt);
  f.x = (__half*)const_cast<void*>(x); f.out = out; f.status = (int*)(ws + w.status);
  if (p->flags & VDN_FLAG_PROJ_MXFP8) {
    // the scale and code regions of the workspace are sized for B*T*N rows
    if (rows > (long long)p->B * p->T * p->N) return VDN_ERR_WORKSPACE;
  }
  VDN_CUDA(launch_projection(p, f, ws, w, st));
  return VDN_OK;
}

vdn_status vdn_hybrid_attn_fwd_host(const vdn_params* p, const vdn_host_inputs* hin,
                                    void* host_out, vdn_host_slot* slot, void* workspace,
                                    size_t workspace_bytes, vdn_stream_t copy_in,
                                    vdn_stream_t compute, vdn_stream_t copy_out,
                                    size_t* h2d_bytes, size_t* d2h_bytes) {
  VDN_TRY(validate_params(p));
  if (hin == nullptr || slot == nullptr || host_out == nullptr) return VDN_ERR_INVALID_ARG;
  VDN_TRY(check_ws(p, workspace, workspace_bytes));
  const size_t es = p->dtype == VDN_BF16 ? 2 : 4;
  const size_t B = p->B, H = p->H, L = (size_t)p->T * p->N, d = p->d_k, nt = p->n_text;
  const size_t act = B * L * H * d * es;
  const size_t beta_n = (p->flags & VDN_FLAG_BETA_PER_TOKEN) ? B * H * (nt + L)
                                                              : B * H * (p->T + 1);
  struct Copy {
    void* dst;
    const void* src;
    size_t bytes;
    bool required;
  };
  const Copy cp[10] = {
      {slot->q, hin->q, act, true},
      {slot->k, hin->k, act, true},
      {slot->v, hin->v, act, true},
      {slot->beta, hin->beta, beta_n * 4, true},
      {slot->alpha, hin->alpha, B * H * p->T * d * 4, false},
      {slot->text_k, hin->text_k, B * nt * H * d * es, nt > 0},
      {slot->text_v, hin->text_v, B * nt * H * d * es, nt > 0},
      {slot->W_o_soft, hin->W_o_soft, H * d * (size_t)p->D_out * es, true},
      {slot->W_o_lin, hin->W_o_lin, H * d * (size_t)p->D_out * es, true},
      {slot->gates, hin->gates, 2 * act, true},
  };
  for (const Copy& c : cp) {
    if (c.required && (c.src == nullptr || c.dst == nullptr)) return VDN_ERR_INVALID_ARG;
    if ((c.src == nullptr) != (c.dst == nullptr)) return VDN_ERR_INVALID_ARG;
    VDN_TRY(check_ptr(c.dst, false));
  }
  VDN_TRY(check_ptr(slot->out, true));
  const size_t out_bytes = B * L * (size_t)p->D_out * (p->out_dtype == VDN_BF16 ? 2 : 4);
  cudaStream_t s_in = (cudaStream_t)copy_in, s_cmp = (cudaStream_t)compute,
               s_out = (cudaStream_t)copy_out;
  cudaEvent_t* ev = reinterpret_cast<cudaEvent_t*>(slot->events);
  if (!slot->used)
    for (int i = 0; i < 3; ++i) {
      if (ev[i] == nullptr &&
          cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess)
        return VDN_ERR_CUDA;
    }
  cudaEvent_t uploaded = ev[0], inputs_read = ev[1], out_copied = ev[2];
  // uploads: once the previous forward on this slot has read its inputs
  if (slot->used) VDN_CUDA(cudaStreamWaitEvent(s_in, inputs_read, 0));
  size_t h2d = 0;
  for (const Copy& c : cp) {
    if (c.src == nullptr) continue;
    VDN_CUDA(cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s_in));
    h2d += c.bytes;
  }
  VDN_CUDA(cudaEventRecord(uploaded, s_in));
  // forward: once uploaded and the previous download of this slot's out is done
  VDN_CUDA(cudaStreamWaitEvent(s_cmp, uploaded, 0));
  if (slot->used) VDN_CUDA(cudaStreamWaitEvent(s_cmp, out_copied, 0));
  VDN_TRY(fwd_impl(p, slot->q, slot->k, slot->v, slot->q, slot->k, slot->v, slot->beta,
                   slot->alpha, slot->text_k, slot->text_v, slot->W_o_soft, slot->W_o_lin,
                   slot->gates, slot->out, workspace, workspace_bytes, compute, nullptr));
  VDN_CUDA(cudaEventRecord(inputs_read, s_cmp));
  // download
  VDN_CUDA(cudaStreamWaitEvent(s_out, inputs_read, 0));
  VDN_CUDA(cudaMemcpyAsync(host_out, slot->out, out_bytes, cudaMemcpyDeviceToHost, s_out));
  VDN_CUDA(cudaEventRecord(out_copied, s_out));
  slot->used = 1;
  if (h2d_bytes != nullptr) *h2d_bytes = h2d;
  if (d2h_bytes != nullptr) *d2h_bytes = out_bytes;
  return VDN_OK;
}

vdn_status vdn_mxfp8_quantize(const void* x, long long rows, long long rows_padded, int cols,
                              void* codes, void* scales, size_t scales_bytes,
                              vdn_stream_t stream) {
  if (rows < 1 || rows_padded < rows || rows_padded > (1LL << 40) || cols < 128 ||
      cols % 128 != 0)
    return VDN_ERR_SHAPE;
  VDN_TRY(check_ptr(x, true));
  VDN_TRY(check_ptr(codes, true));
  VDN_TRY(check_ptr(scales, true));
  if (scales_bytes < mx_scale_bytes(rows_padded, cols)) return VDN_ERR_WORKSPACE;
  VDN_CUDA(launch_mx_quant((const __half*)x, (uint8_t*)codes, (uint8_t*)scales, rows,
                           rows_padded, cols, (cudaStream_t)stream));
  return VDN_OK;
}

vdn_status vdn_host_slot_release(vdn_host_slot* slot) {
  if (slot == nullptr) return VDN_OK;
  cudaEvent_t* ev = reinterpret_cast<cudaEvent_t*>(slot->events);
  vdn_status st = VDN_OK;
  for (int i = 0; i < 3; ++i) {
    if (ev[i] != nullptr && cudaEventDestroy(ev[i]) != cudaSuccess) st = VDN_ERR_CUDA;
    ev[i] = nullptr;
  }
  slot->used = 0;
  return st;
}

vdn_status vdn_prep_params_init(vdn_prep_params* p, int B, int H, int T, int grid_h,
                                int grid_w, int d, vdn_dtype dtype) {
  if (p == nullptr) return VDN_ERR_INVALID_ARG;
  memset(p, 0, sizeof(*p));
  p->B = B; p->H = H; p->T = T; p->grid_h = grid_h; p->grid_w = grid_w; p->d = d;
  p->spatial_taps = 3; p->temporal_taps = 5; p->dtype = dtype; p->l2_eps = 1e-6f;
  return validate_prep(p);
}

vdn_status vdn_vda_prep(const vdn_prep_params* p, const void* q, const void* k, const void* v,
                        const float* wk_s, const float* wk_t, const float* wv_s,
                        const float* wv_t, void* q_out, void* k_out, void* v_out,
                        void* workspace, size_t workspace_bytes, vdn_stream_t stream) {
  VDN_TRY(validate_prep(p));
  const bool has_q = q != nullptr || q_out != nullptr;
  const bool has_kv = k != nullptr || v != nullptr || k_out != nullptr || v_out != nullptr ||
                      wk_s != nullptr || wk_t != nullptr || wv_s != nullptr || wv_t != nullptr;
  if (!has_q && !has_kv) return VDN_ERR_INVALID_ARG;
  if (has_q) {
    VDN_TRY(check_ptr(q, true));
    VDN_TRY(check_ptr(q_out, true));
  }
  if (has_kv) {
    const void* need[8] = {k, v, k_out, v_out, wk_s, wk_t, wv_s, wv_t};
    for (const void* ptr : need) VDN_TRY(check_ptr(ptr, true));
    // the convolution reads neighbours: no output may overlap an input
    const size_t n = (size_t)p->B * p->T * p->grid_h * p->grid_w * p->H * p->d *
                     (p->dtype == VDN_BF16 ? 2 : 4);
    auto overlap = [n](const void* a, const void* b) {
      const char *x = (const char*)a, *y = (const char*)b;
      return x < y + n && y < x + n;
    };
    const void* outs[2] = {k_out, v_out};
    const void* ins[2] = {k, v};
    for (const void* o : outs)
      for (const void* i : ins)
        if (overlap(o, i)) return VDN_ERR_INVALID_ARG;
    if (overlap(k_out, v_out)) return VDN_ERR_INVALID_ARG;
  }
  if (workspace == nullptr || workspace_bytes < VDN_PREP_WORKSPACE_BYTES)
    return VDN_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return VDN_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaMemsetAsync(workspace, 0, sizeof(int), st));
  PrepArgs a;
  a.B = p->B; a.H = p->H; a.T = p->T; a.gh = p->grid_h; a.gw = p->grid_w; a.D = p->d;
  a.bf16 = p->dtype == VDN_BF16; a.eps = p->l2_eps;
  a.q = has_q ? q : nullptr; a.q_out = has_q ? q_out : nullptr;
  a.k = has_kv ? k : nullptr; a.v = v; a.k_out = k_out; a.v_out = v_out;
  a.wk_s = wk_s; a.wk_t = wk_t; a.wv_s = wv_s; a.wv_t = wv_t;
  a.status = (int*)workspace;
  VDN_CUDA(launch_prep(a, st));
  return VDN_OK;
}

vdn_status vdn_text_query_attn(const vdn_params* p, const void* text_q, const void* k,
                               const void* v, const void* text_k, const void* text_v,
                               float* o_text, void* workspace, size_t workspace_bytes,
                               vdn_stream_t stream) {
  VDN_TRY(validate_params(p));
  if (p->n_text < 1) return VDN_ERR_SHAPE;
  const void* need[6] = {text_q, k, v, text_k, text_v, o_text};
  for (const void* ptr : need) VDN_TRY(check_ptr(ptr, true));
  vdn_params pt = *p;  // the text tokens join the keys (their V^T in the workspace)
  pt.flags |= VDN_FLAG_TEXT_SOFTMAX;
  VDN_TRY(check_ws(&pt, workspace, workspace_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const WsLayout w = layout(pt);
  VDN_CUDA(cudaMemsetAsync(ws, 0, 256, st));
  AttnArgs a = attn_args(&pt, nullptr, k, v, text_k, text_v);
  a.text_q = text_q;
  if (use_tc(pt)) {
    TcAttnArgs t = tc_attn_args(pt, a, ws + w.vt, (int*)(ws + w.status));
    // split the keys of the few text-row CTAs until the grid covers the GPU
    // twice; the partial results live in the (here unused) operand region x
    const int tiles = (int)((pt.T * (size_t)pt.N + 127) / 128 + (pt.n_text + 127) / 128);
    const long long base = (long long)((pt.n_text + 255) / 256) * pt.B * pt.H;
    int split = (int)((2LL * sm_count() + base - 1) / base);
    split = split < 1 ? 1 : (split > 16 ? 16 : split);
    if (split > tiles / 2) split = tiles / 2 > 1 ? tiles / 2 : 1;
    const size_t rows = (size_t)pt.B * pt.n_text * pt.H;
    while (split > 1 && (size_t)split * rows * (pt.d_k + 2) * sizeof(float) > w.total - w.x)
      --split;
    if (split > 1) {
      t.kv_split = split;
      t.part = (float*)(ws + w.x);
      t.ml = t.part + (size_t)split * rows * pt.d_k;
    }
    VDN_CUDA(launch_convert_v(t, st));
    VDN_CUDA(launch_attn_tc(t, nullptr, o_text, st));
  } else {
    VDN_CUDA(launch_attn_simt(a, o_text, st));
  }
  return VDN_OK;
}

vdn_status vdn_forward_launches(const vdn_params* p, int* launches) {
  VDN_TRY(validate_params(p));
  if (launches == nullptr) return VDN_ERR_INVALID_ARG;
  if ((p->flags & VDN_FLAG_PROJ_MXFP8) && !use_tc(*p)) return VDN_ERR_UNSUPPORTED;
  VdaArgs va;
  memset(&va, 0, sizeof(va));
  va.B = p->B; va.H = p->H; va.T = p->T; va.D = p->d_k; va.C = p->chunk;
  va.scan_mode = (p->flags & VDN_FLAG_SCAN_FRAMES) ? 1 : ((p->flags & VDN_FLAG_SCAN_CHUNKS) ? 2 : 0);
  int n = vda_frame_scan_route(va) ? 2 : 3;
  if (use_tc(*p))  // V^T conversion (text V^T too when text keys join), Softmax, readout, W^T, GEMM
    n += 4 + ((p->flags & VDN_FLAG_PROJ_MXFP8) ? 2 : 1) +
         (((p->flags & VDN_FLAG_TEXT_SOFTMAX) && p->n_text > 0) ? 1 : 0);
  else
    n += 4;
  *launches = n;
  return VDN_OK;
}

vdn_status vdn_device_status(const vdn_params* p, void* workspace, vdn_stream_t stream) {
  if (p != nullptr) VDN_TRY(validate_params(p));
  if (workspace == nullptr) return VDN_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaStreamSynchronize(st));
  int word = 0;
  VDN_CUDA(cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost));
  VDN_CUDA(cudaMemset(workspace, 0, sizeof(int)));
  if (word & kDevTimeout) return VDN_ERR_TIMEOUT;
  if (word & kDevRange) return VDN_ERR_RANGE;
  return VDN_OK;
}

}  // extern "C"
