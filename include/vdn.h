/*
 * vdn.h -- C ABI of libvdn, the sm_100a (B200) implementation of the Video
 * DeltaNet hybrid attention forward for video-to-video interactions.
 *
 * Source of every operation: "Video DeltaNet: A Video-Native Hybrid Attention
 * for Livestream Video Generation" (Xi et al.):
 *   - Softmax branch: the paragraph of the method on the local window (exact
 *     Softmax inside a chunk-aligned window of 2*window_radius+1 chunks, plus
 *     the two boundary anchors: every frame sees all tokens of the first and
 *     last latent frame, and those two frames see the whole clip; a key frame
 *     counts once).
 *   - Linear branch: the paragraph on bidirectional linear attention (a
 *     forward and a reverse scan over the frames outside the query's window,
 *     anchors excluded, both initialised from a text-summary state, readouts
 *     added; a channel-wise decay bridge across the skipped window span) and
 *     the Video Delta Attention paragraphs (per-frame joint update
 *     S_t = (I + A_t)^-1 (Diag(alpha_t) S_{t-1} + W_t), A_t = beta_t K_t^T K_t,
 *     W_t = beta_t K_t^T V_t, solved in key-channel space, FP32 state).
 *   - Output: the paragraph on the two output gates (sigmoid gate on the
 *     Softmax readout, RMS norm + sigmoid gate on the linear readout, two
 *     separate output projections whose results are added).
 *   - Implementation section ("Chunk-wise scans", "Small-matrix inverse"):
 *     per-frame affine transitions composed per chunk and scanned in both
 *     directions; only chunk-boundary states are kept.
 *
 * Conventions shared by every entry point
 *   - Sizes: L = T*N video tokens per batch item, token index t*N + n
 *     (frame-major).  n_chunks = ceil(T / chunk).  Anchors = frames {0, T-1}.
 *   - Layouts (row-major, innermost last):
 *       q, k, v            [B, L, H, d]      dtype params.dtype
 *       text_k, text_v     [B, n_text, H, d] dtype params.dtype
 *       beta               [B, H, 1+T]       float32; [.,.,0] is the text frame
 *                          ([B, H, n_text+L] with VDN_FLAG_BETA_PER_TOKEN)
 *       alpha              [B, H, T, d_k]    float32 in [0,1], or NULL (= 1)
 *       W_o_soft, W_o_lin  [H*d_v, D_out]    dtype params.dtype; y = x W
 *       gates              [2, B, L, H, d_v] dtype params.dtype, post-sigmoid;
 *                                            [0] Softmax gate, [1] linear gate
 *       out                [B, L, D_out]     dtype params.out_dtype
 *   - Ownership: the caller owns every buffer (device memory unless stated).
 *     The library never allocates or frees device memory; all scratch comes
 *     from the caller's workspace (size from vdn_workspace_bytes).
 *   - Alignment: every pointer must be 16-byte aligned; the workspace 256-byte
 *     aligned (any cudaMalloc / PyTorch allocation is).
 *   - Asynchrony: compute entry points validate arguments on the host, then
 *     enqueue kernels on `stream` and return without synchronising.  VDN_OK
 *     means "enqueued".  Device-side conditions (a bounded wait that expired,
 *     a value outside the range of an internal fp16 operand) are recorded in
 *     a status word inside the workspace, which every compute call clears when
 *     it starts; read it with vdn_device_status after the call.
 *   - Errors: a failed validation returns before any launch and leaves every
 *     output untouched.  No exceptions cross the ABI.  The library keeps no
 *     global state except a per-device attribute cache; calls on different
 *     streams with different workspaces may run concurrently.
 *   - Supported: d_k == d_v in {32, 64, 128}, chunk >= 1, window_radius >= 0,
 *     T >= 1, N >= 1, n_text >= 0, D_out a multiple of 8.  Tensor-core
 *     kernels serve dtype BF16 with d in {64, 128} (Q K^T in bf16; P, V, the
 *     gated branch outputs and W in fp16; FP32 accumulation, FP32 state);
 *     every other case, and VDN_FLAG_SIMT, runs exact-FP32 CUDA-core kernels.
 *   - Range (tensor-core path): |v|, |W_o_*| and |gate * branch output| must
 *     stay below 65504 (fp16); an overflow sets VDN_ERR_RANGE.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VDN_ABI_VERSION 1

#if defined(__GNUC__)
#define VDN_API __attribute__((visibility("default")))
#else
#define VDN_API
#endif

typedef enum vdn_status {
  VDN_OK = 0,
  VDN_ERR_INVALID_ARG = 1, /* NULL where a pointer is required, bad enum/flag */
  VDN_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  VDN_ERR_DTYPE = 3,       /* unsupported dtype combination */
  VDN_ERR_ALIGNMENT = 4,   /* a pointer is not 16-byte aligned */
  VDN_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than required */
  VDN_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  VDN_ERR_TIMEOUT = 7,     /* a bounded device-side wait expired */
  VDN_ERR_UNSUPPORTED = 8, /* valid request that this build does not serve */
  VDN_ERR_RANGE = 9        /* an input value overflowed an internal fp16 operand */
} vdn_status;

typedef enum vdn_dtype { VDN_F32 = 0, VDN_BF16 = 1 } vdn_dtype;

/* Binary-compatible with cudaStream_t / CUstream; NULL = legacy default stream. */
typedef struct CUstream_st *vdn_stream_t;

/* params.flags */
#define VDN_FLAG_TEXT_FULL (1u << 0) /* both scans start from S_text (not S_text/2) */
#define VDN_FLAG_SIMT (1u << 1)      /* force the exact-FP32 CUDA-core kernels */
/* Video queries also attend every text token in the Softmax branch, under one
 * normaliser with their visible video keys (method section: the text keeps
 * its Softmax path while the linear memory also summarises it).  Needs n_text > 0. */
#define VDN_FLAG_TEXT_SOFTMAX (1u << 2)
/* One write gate per token instead of per frame (the pages' beta_{t,i}): beta
 * is then [B, H, n_text + L] float32, the n_text text tokens first, then the
 * video tokens in token order.  On the tensor-core path the frame statistics
 * use sqrt(beta_i)-scaled fp16 copies of the key/value tiles. */
#define VDN_FLAG_BETA_PER_TOKEN (1u << 3)
/* Comparison mode: every frame update follows the frozen-state (SANA-WM)
 * batched rule of the Video Delta Attention section instead of VDA's: all
 * token corrections are evaluated at the same decayed state,
 * S_t = (I - A_t) Diag(alpha_t) S_{t-1} + W_t (no inverse; the text frame
 * likewise, S_text = W_text).  Keys are taken as given: SANA-WM's frame-size
 * key scaling, whose factor the pages lost, is left to the caller. */
#define VDN_FLAG_FROZEN_STATE (1u << 4)
/* How the bidirectional scan (implementation section, "Chunk-wise scans") is
 * evaluated.  By default the library picks, from the problem's shape, either
 * the composition of each chunk's frame maps followed by a scan over chunks,
 * or a scan straight over the frames that keeps only the chunk-boundary
 * states (fewer products, more sequential steps: the better choice for short
 * clips).  Both give the same states up to FP32 rounding.  These flags force
 * one of them (setting both is VDN_ERR_INVALID_ARG). */
#define VDN_FLAG_SCAN_FRAMES (1u << 5)
#define VDN_FLAG_SCAN_CHUNKS (1u << 6)
/* Reduced-precision mode of the output projections (implementation section:
 * MXFP8 for the output GEMM): the fp16 operands x = [g_s o_s | g_l RMS(o_l)]
 * and [W_o_soft; W_o_lin] are quantised to MXFP8 -- blocks of 32 elements
 * along the contraction dimension share a power-of-two scale 2^e,
 * e = floor(log2 max|v|) - 8 (stored as e + 127), elements v / 2^e rounded to
 * E4M3 (ties to even, saturating at +-448) -- and multiplied on the block-
 * scaled fp8 tensor cores with FP32 accumulation.  In the forward, the
 * Softmax and readout epilogues quantise their rows of x in registers (the
 * same fp16 values, the same codes and scales as vdn_mxfp8_quantize), so x
 * never reaches memory in fp16; vdn_output_projection quantises the x it is
 * given.  Tensor-core path only (else VDN_ERR_UNSUPPORTED).  Its error against the exact projection is that
 * of the format (about 4% of the output RMS, up to about 25% at single
 * outputs), far above the default path's; see vdn_mxfp8_quantize for the
 * exact quantisation. */
#define VDN_FLAG_PROJ_MXFP8 (1u << 7)

typedef struct vdn_params {
  int B;             /* batch */
  int H;             /* heads */
  int T;             /* latent frames */
  int N;             /* tokens per frame */
  int d_k, d_v;      /* head dims (must be equal) */
  int n_text;        /* text tokens summarised into the initial state */
  int D_out;         /* output width of both projections */
  int chunk;         /* frames per chunk (5 on the pages: one VAE temporal unit) */
  int window_radius; /* chunks on each side of the query chunk (1 on the pages) */
  vdn_dtype dtype;     /* q, k, v, text_k, text_v, W_o_*, gates */
  vdn_dtype out_dtype; /* out */
  float softmax_scale; /* 0 => 1/sqrt(d_k) */
  float rms_eps;       /* epsilon of the linear-readout RMS norm (pages: unstated; 1e-6) */
  unsigned flags;      /* VDN_FLAG_* */
} vdn_params;

/* ABI version of the loaded library (VDN_ABI_VERSION). */
VDN_API int vdn_abi_version(void);

/* Static string for a status code; never NULL. */
VDN_API const char *vdn_status_string(vdn_status s);

/* Fills `p` with the pages' defaults for the given sizes: chunk 5,
 * window_radius 1, D_out = H*d, softmax_scale 0, rms_eps 1e-6, flags 0. */
VDN_API vdn_status vdn_params_init(vdn_params *p, int B, int H, int T, int N, int d,
                           int n_text, vdn_dtype dtype);

/* Workspace bytes needed by vdn_hybrid_attn_fwd, vdn_hybrid_attn_branches
 * and vdn_vda_boundary_states for these params (one size serves all three).
 * Host only; validates `p` like the compute calls. */
VDN_API vdn_status vdn_workspace_bytes(const vdn_params *p, size_t *bytes);

/* The whole hybrid attention forward:
 *   o_s = window+anchor Softmax(q, k, v)                          [B,L,H,d_v]
 *   o_l = q^T S_fwd + q^T S_rev (VDA scans, text-initialised)      [B,L,H,d_v]
 *   out = concat_h(g_s * o_s) W_o_soft + concat_h(g_l * RMS(o_l)) W_o_lin
 * alpha may be NULL (no decay).  n_text may be 0 (text_k/text_v may then be
 * NULL; S_text = 0).  Everything else is required. */
VDN_API vdn_status vdn_hybrid_attn_fwd(const vdn_params *p, const void *q, const void *k,
                               const void *v, const float *beta, const float *alpha,
                               const void *text_k, const void *text_v,
                               const void *W_o_soft, const void *W_o_lin,
                               const void *gates, void *out, void *workspace,
                               size_t workspace_bytes, vdn_stream_t stream);

/* Number of kernel launches that vdn_hybrid_attn_fwd enqueues for `p`
 * (host only; the status-word clear is a memset, not counted).  The state
 * path takes 2 kernels (frame statistics + solve, then the direct scan over
 * frames) or 3 (frame statistics + solve, chunk composition, chunk scan): the
 * library picks the route from the shape and the device's SM count unless
 * VDN_FLAG_SCAN_FRAMES / VDN_FLAG_SCAN_CHUNKS forces it.  Then, on the
 * tensor-core path: V^T conversion (a second one for the text values when
 * VDN_FLAG_TEXT_SOFTMAX adds text keys), Softmax, readout, W^T conversion and the
 * GEMM (with VDN_FLAG_PROJ_MXFP8: the quantisation of W^T and the block-
 * scaled GEMM, x arriving quantised from the epilogues); on the CUDA-core
 * path: Softmax, readout, RMS factors, projection.
 * Validates `p` like the compute calls; `launches` must not be NULL
 * (VDN_ERR_INVALID_ARG). */
VDN_API vdn_status vdn_forward_launches(const vdn_params *p, int *launches);

/* Stage boundaries recorded by vdn_hybrid_attn_fwd_staged. */
#define VDN_STAGES 5 /* VDA states, operand conversion, Softmax, readout, projection */
typedef struct vdn_stage_events {
  void *events[VDN_STAGES + 1]; /* cudaEvent_t handles created by the caller */
} vdn_stage_events;

/* Same computation and arguments as vdn_hybrid_attn_fwd, and records
 * events[0] before the first kernel and events[i] after stage i on `stream`:
 * 1 VDA state path (frame statistics + solve, then the bidirectional scan),
 * 2 V^T conversion to fp16 (empty on the CUDA-core path), 3 window+anchor
 * Softmax, 4 linear readout (+ RMS norm and gate on the tensor-core path),
 * 5 output projection (W^T conversion, with VDN_FLAG_PROJ_MXFP8 the MXFP8
 * quantisation of W^T, and the GEMM; x is quantised inside stages 3 and 4).  Used for live per-stage timing
 * with cudaEventElapsedTime.  `ev` may be NULL (no events). */
VDN_API vdn_status vdn_hybrid_attn_fwd_staged(const vdn_params *p, const void *q, const void *k,
                                      const void *v, const float *beta, const float *alpha,
                                      const void *text_k, const void *text_v,
                                      const void *W_o_soft, const void *W_o_lin,
                                      const void *gates, void *out, void *workspace,
                                      size_t workspace_bytes, vdn_stream_t stream,
                                      const vdn_stage_events *ev);

/* vdn_hybrid_attn_fwd_staged with the linear branch reading its own inputs:
 * the method feeds the linear branch from the same projections through its
 * own feature map (vdn_vda_prep), while the Softmax branch keeps q, k, v.
 *  - q, k, v: Softmax branch inputs, as for vdn_hybrid_attn_fwd.
 *  - q_lin, k_lin, v_lin: [B, L, H, d] dtype params.dtype, the linear branch's
 *    queries (readout), keys and values (frame statistics).  Passing q, k, v
 *    again gives exactly vdn_hybrid_attn_fwd_staged.
 *  - text_k, text_v serve both branches; every other argument, the workspace
 *    size and the events as vdn_hybrid_attn_fwd_staged. */
VDN_API vdn_status vdn_hybrid_attn_fwd_split(const vdn_params *p, const void *q, const void *k,
                                     const void *v, const void *q_lin, const void *k_lin,
                                     const void *v_lin, const float *beta, const float *alpha,
                                     const void *text_k, const void *text_v,
                                     const void *W_o_soft, const void *W_o_lin,
                                     const void *gates, void *out, void *workspace,
                                     size_t workspace_bytes, vdn_stream_t stream,
                                     const vdn_stage_events *ev);

/* ---- The forward in two halves (head-sharded, Ulysses-style execution) -----
 * The implementation section of the paper shards VDA by attention head over
 * GPUs (Ulysses).  Every step of the forward is independent per head except
 * the output projection, which contracts over heads.  These two calls split
 * the forward at that point, so that a rank can compute the operand of its
 * heads, exchange it (an all-to-all from head shards to token shards), and
 * project its own tokens with the whole W:
 *   vdn_hybrid_attn_fwd == vdn_hybrid_attn_operand + vdn_output_projection
 * (bit for bit, on the same inputs).  Tensor-core path only (dtype BF16,
 * d in {64, 128}, no VDN_FLAG_SIMT); otherwise VDN_ERR_UNSUPPORTED. */

/* x: [B, L, 2, H, d_v] fp16 (IEEE binary16), caller-owned, 16-byte aligned:
 *   x[b, l, 0, h, :] = g_s * o_s          (gated Softmax readout)
 *   x[b, l, 1, h, :] = g_l * RMS(o_l)     (gated, RMS-normalised linear readout)
 * i.e. the rows of the operand [g_s o_s | g_l RMS(o_l)] of the two output
 * projections.  Other arguments, workspace and errors as vdn_hybrid_attn_fwd
 * (W_o_* are not needed); values beyond the fp16 range set VDN_ERR_RANGE. */
VDN_API vdn_status vdn_hybrid_attn_operand(const vdn_params *p, const void *q, const void *k,
                                           const void *v, const float *beta, const float *alpha,
                                           const void *text_k, const void *text_v,
                                           const void *gates, void *x, void *workspace,
                                           size_t workspace_bytes, vdn_stream_t stream);

/* out[r, :] = x[r, 0, :, :] W_o_soft + x[r, 1, :, :] W_o_lin for r < rows:
 * x [rows, 2, H, d_v] fp16 as vdn_hybrid_attn_operand writes it (any set of
 * rows, e.g. one token shard holding every head), W_o_* [H*d_v, D_out] in
 * params.dtype, out [rows, D_out] in params.out_dtype.  Only H, d, D_out, the
 * dtypes and flags of `p` matter here (the rest is validated as usual); the
 * workspace is one of vdn_workspace_bytes(p).  rows in 1 .. 2^30 (else
 * VDN_ERR_SHAPE). */
VDN_API vdn_status vdn_output_projection(const vdn_params *p, long long rows, const void *x,
                                         const void *W_o_soft, const void *W_o_lin, void *out,
                                         void *workspace, size_t workspace_bytes,
                                         vdn_stream_t stream);

/* MXFP8 quantisation (the VDN_FLAG_PROJ_MXFP8 rule) of a row-major fp16
 * (IEEE binary16) matrix x [rows, cols], cols a multiple of 128, in blocks of
 * 32 along each row:
 *  - codes [rows, cols] uint8: the E4M3 elements (1 sign, 4 exponent bits of
 *    bias 7, 3 mantissa bits);
 *  - scales: the shared exponents e + 127 (UE8M0) in 512-byte atoms, one per
 *    128 rows x 128 columns: scale of row r, block j (columns 32j .. 32j+31) at
 *    byte ((r / 128) * (cols / 128) + j / 4) * 512 + 16 (r % 32)
 *    + 4 ((r % 128) / 32) + j % 4.  scales_bytes must hold
 *    ceil(rows_padded / 128) * (cols / 128) * 512 bytes; rows in
 *    [rows, rows_padded) get the smallest scale (e = -127).
 * This is the layout the block-scaled tensor cores read.  Device pointers,
 * 16-byte aligned; asynchronous on `stream`. */
VDN_API vdn_status vdn_mxfp8_quantize(const void *x, long long rows, long long rows_padded,
                                      int cols, void *codes, void *scales, size_t scales_bytes,
                                      vdn_stream_t stream);

/* ---- End to end from host memory ------------------------------------------
 * One forward whose inputs and output live in host memory: the call enqueues
 * the host -> device copies of every input, the forward, and the device ->
 * host copy of `out`, ordered by CUDA events, on three caller streams.  It
 * allocates no device memory: the device buffers of one step (a "slot") and
 * the workspace are the caller's.  Alternating two slots lets the uploads of
 * step i+1 and the download of step i-1 overlap the forward of step i; the
 * events in the slot keep a slot's buffers from being overwritten while a
 * previous step still reads them. */
typedef struct vdn_host_inputs {
  /* host pointers, same layouts and dtypes as vdn_hybrid_attn_fwd; pinned
   * (page-locked) memory for asynchronous copies.  alpha may be NULL, and
   * text_k / text_v when n_text == 0. */
  const void *q, *k, *v;
  const float *beta, *alpha;
  const void *text_k, *text_v, *W_o_soft, *W_o_lin, *gates;
} vdn_host_inputs;

typedef struct vdn_host_slot {
  /* device buffers of one step (caller-owned, sizes of the layouts above);
   * alpha NULL when the host alpha is NULL */
  void *q, *k, *v;
  float *beta, *alpha;
  void *text_k, *text_v, *W_o_soft, *W_o_lin, *gates, *out;
  /* library-managed: zero-initialise the struct before its first use and
   * release it with vdn_host_slot_release; three cudaEvent_t handles
   * (uploaded, inputs read by the forward, output copied back) created on the
   * slot's first use */
  void *events[3];
  int used;
} vdn_host_slot;

/* host_in: host inputs of this step; host_out: host memory for out
 * [B, L, D_out] (out_dtype); slot: device buffers for this step; workspace as
 * vdn_hybrid_attn_fwd.  copy_in / compute / copy_out: streams of the uploads,
 * the forward and the download (they may all be the same stream).  On return
 * *h2d_bytes and *d2h_bytes (each may be NULL) hold the bytes copied each way.
 * Asynchronous: host_out is complete once copy_out reaches this point (for
 * instance after cudaStreamSynchronize(copy_out)); host_in and the slot must
 * stay untouched until then.  No source in the paper: the pages' serving stack
 * moves data between host and GPU, and this is the library's form of it.
 * Validation as vdn_hybrid_attn_fwd, plus every host and slot pointer the
 * layouts require (VDN_ERR_INVALID_ARG). */
VDN_API vdn_status vdn_hybrid_attn_fwd_host(const vdn_params *p, const vdn_host_inputs *host_in,
                                            void *host_out, vdn_host_slot *slot,
                                            void *workspace, size_t workspace_bytes,
                                            vdn_stream_t copy_in, vdn_stream_t compute,
                                            vdn_stream_t copy_out, size_t *h2d_bytes,
                                            size_t *d2h_bytes);

/* Destroys the events of a slot (after its last step has completed); the
 * caller frees the slot's device buffers.  NULL is a no-op. */
VDN_API vdn_status vdn_host_slot_release(vdn_host_slot *slot);

/* ---- VDA-Prep: the linear branch's feature map ----------------------------
 * "Video DeltaNet" method (the linear branch applies its own feature map to
 * the pretrained projections: a separable short convolution of K and V -- a
 * depthwise spatial filter and a five-tap temporal filter -- then SiLU, and L2
 * normalisation of Q and K) and implementation ("Fused VDA kernels",
 * VDA-Prep).  Computed, in FP32:
 *   k_l = L2(SiLU(conv_t(conv_s(k)))),  v_l = SiLU(conv_t(conv_s(v))),
 *   q_l = L2(q),   L2(x) = x / sqrt(sum_d x^2 + l2_eps) per (token, head).
 * conv_s: depthwise 3x3 cross-correlation over the frame's row-major
 * grid_h x grid_w token grid (token n = y * grid_w + x), zero padding;
 * conv_t: depthwise 5 taps over frames t-2 .. t+2, zero padding at the clip
 * ends.  Video tokens only (text tokens have no grid).  Outputs are rounded
 * once to dtype. */
typedef struct vdn_prep_params {
  int B, H, T;          /* batch, heads, latent frames */
  int grid_h, grid_w;   /* tokens per frame N = grid_h * grid_w */
  int d;                /* head dim: 32, 64 or 128 */
  int spatial_taps;     /* 3 (the only size served) */
  int temporal_taps;    /* 5 (the only size served) */
  vdn_dtype dtype;      /* of q, k, v and of the outputs */
  float l2_eps;         /* default 1e-6 */
} vdn_prep_params;

/* Workspace of vdn_vda_prep: its device status word. */
#define VDN_PREP_WORKSPACE_BYTES 256u

/* Fills defaults (3x3 spatial, 5 temporal taps, l2_eps 1e-6) and validates. */
VDN_API vdn_status vdn_prep_params_init(vdn_prep_params *p, int B, int H, int T, int grid_h,
                                        int grid_w, int d, vdn_dtype dtype);

/*  - q, k, v: [B, T*grid_h*grid_w, H, d] dtype, device.  Either group may be
 *    skipped: q = q_out = NULL skips Q; k, v, k_out, v_out and the four
 *    filters all NULL skips K/V.
 *  - wk_s, wv_s: float32 [H*d][3][3] spatial filters of K and V (channel
 *    c = h*d + i, then filter row, then column); wk_t, wv_t: float32
 *    [H*d][5] temporal filters (tap j weighs frame t + j - 2).
 *  - q_out, k_out, v_out: [B, T*grid_h*grid_w, H, d] dtype.  k_out and v_out
 *    must not overlap k, v or each other (VDN_ERR_INVALID_ARG); q_out may be q.
 *  - workspace: >= VDN_PREP_WORKSPACE_BYTES bytes of device memory, 256-byte
 *    aligned; holds the device status word (read it with
 *    vdn_device_status(NULL, workspace, stream)).
 *  - Other conventions as the forward: 16-byte aligned pointers, validation
 *    before any launch, asynchronous on `stream`. */
VDN_API vdn_status vdn_vda_prep(const vdn_prep_params *p, const void *q, const void *k,
                                const void *v, const float *wk_s, const float *wk_t,
                                const float *wv_s, const float *wv_t, void *q_out, void *k_out,
                                void *v_out, void *workspace, size_t workspace_bytes,
                                vdn_stream_t stream);

/* Text tokens as queries: the text rows of the joint Softmax with text
 * (method section: the text keeps its Softmax path).  Every text query
 * attends every video key and every text key under one normaliser, with no
 * mask:  o_text[i] = softmax_j(scale * q_i . k_j) v_j  over j in
 * [video tokens; text tokens].
 *  - text_q: [B, n_text, H, d] dtype params.dtype (the text tokens' queries);
 *    k, v: [B, L, H, d]; text_k, text_v: [B, n_text, H, d].
 *  - o_text: float32 [B, n_text, H, d_v], caller-owned.
 *  - Needs n_text >= 1 (else VDN_ERR_SHAPE).  The workspace must hold
 *    vdn_workspace_bytes of the same params with VDN_FLAG_TEXT_SOFTMAX set
 *    (the transposed text values live there).  Runs the tensor-core kernel
 *    for bf16 with d in {64, 128}, the FP32 kernel otherwise (or with
 *    VDN_FLAG_SIMT).  Other conventions as vdn_hybrid_attn_fwd. */
VDN_API vdn_status vdn_text_query_attn(const vdn_params *p, const void *text_q, const void *k,
                                       const void *v, const void *text_k, const void *text_v,
                                       float *o_text, void *workspace, size_t workspace_bytes,
                                       vdn_stream_t stream);

/* The two branch readouts before gating and projection, float32
 * [B, L, H, d_v]: o_soft = Softmax branch, o_lin = linear branch before its
 * RMS norm.  Either output pointer may be NULL to skip that branch. */
VDN_API vdn_status vdn_hybrid_attn_branches(const vdn_params *p, const void *q, const void *k,
                                    const void *v, const float *beta, const float *alpha,
                                    const void *text_k, const void *text_v,
                                    float *o_soft, float *o_lin, void *workspace,
                                    size_t workspace_bytes, vdn_stream_t stream);

/* The chunk-boundary states of the VDA scans, float32 [B, H, n_chunks, d_k, d_v]:
 * F[c] = forward state read by query chunk c (after every frame before its
 * window), G[c] = reverse state (after every frame after its window), before
 * the per-frame decay bridge.  Either output may be NULL. */
VDN_API vdn_status vdn_vda_boundary_states(const vdn_params *p, const void *k, const void *v,
                                   const float *beta, const float *alpha,
                                   const void *text_k, const void *text_v, float *F,
                                   float *G, void *workspace, size_t workspace_bytes,
                                   vdn_stream_t stream);

/* Size of the static device array used by vdn_vda_boundary_states_noalloc. */
#define VDN_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */

/* vdn_vda_boundary_states without workspace: same kernels, same results, for
 * callers that cannot allocate device memory (a host framework that owns all
 * allocations, a plugin with no allocator, code that must not call cudaMalloc
 * while a stream is captured).  The paper has no counterpart; this is a
 * deployment convenience of the library.
 *  - Scratch lives in a static __device__ array of VDN_NOALLOC_SCRATCH_BYTES
 *    inside the library; each GPU that loads the library keeps it until exit.
 *    Nothing is allocated or freed by this call.
 *  - Problems whose state-path scratch exceeds that size return
 *    VDN_ERR_WORKSPACE.  The scratch is about
 *    4 * d*d * B*H * (2*(T+1) + 6*ceil(T/chunk) + 2) bytes: e.g. B*H = 8,
 *    T = 40, d = 64 needs 17 MiB and fits; the 768p workload does not.
 *  - Every call looks up the array's device address on the current device
 *    (a table read once the library is loaded there; nothing is cached, so a
 *    context destroyed and re-created by cudaDeviceReset is handled).  The
 *    first call on a device may load the library's module there: make it
 *    before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents:
 *    calls that overlap on the GPU (unordered streams or threads) race.  Order
 *    them on one stream.
 *  - Device-side conditions (VDN_ERR_TIMEOUT, VDN_ERR_RANGE) go to a status
 *    word at the start of the array, cleared when each call starts: read it
 *    with vdn_noalloc_device_status.
 *  - Other conventions as vdn_vda_boundary_states; no workspace arguments. */
VDN_API vdn_status vdn_vda_boundary_states_noalloc(const vdn_params *p, const void *k,
                                                   const void *v, const float *beta,
                                                   const float *alpha, const void *text_k,
                                                   const void *text_v, float *F, float *G,
                                                   vdn_stream_t stream);

/* Status of the last vdn_vda_boundary_states_noalloc call on the current
 * device: synchronises `stream`, then reads and clears the status word in the
 * library's static array (VDN_OK, VDN_ERR_TIMEOUT or VDN_ERR_RANGE).  Like
 * that entry point it has no counterpart in the paper and allocates nothing.
 * A status word is shared by every no-allocation call on the device: read it
 * after the call whose status you want, before the next one is enqueued. */
VDN_API vdn_status vdn_noalloc_device_status(vdn_stream_t stream);

/* Synchronises `stream`, then reads and clears the device status word that
 * the last compute call on this workspace left (VDN_OK, VDN_ERR_TIMEOUT or
 * VDN_ERR_RANGE).  `workspace` must be the one passed to that call.  `p` may
 * be NULL (it is only validated when given). */
VDN_API vdn_status vdn_device_status(const vdn_params *p, void *workspace, vdn_stream_t stream);

/* Self-test of failure detection, without a fault or a hang.
 * Every pipelined kernel of this library bounds its waits on shared-memory
 * barriers by time: on expiry it records VDN_ERR_TIMEOUT in the device status
 * word, the other warps of the block leave through an abort flag, and the
 * block frees its tensor memory and exits.  This call enqueues one block that
 * runs that sequence on a barrier nothing ever arrives at.
 *  - workspace: any workspace of this library (device memory, 256-byte
 *    aligned); only its status word is written.  It is cleared first, so
 *    vdn_device_status afterwards returns VDN_ERR_TIMEOUT.
 *  - limit_us: the wait limit, 100 us .. 1 s (else VDN_ERR_INVALID_ARG).  The
 *    block ends within about twice this limit.
 *  - The GPU context stays usable; later calls run normally. */
VDN_API vdn_status vdn_selftest_bounded_wait(void *workspace, unsigned int limit_us,
                                             vdn_stream_t stream);

/* Self-test of the exponential that the tensor-core Softmax kernel evaluates
 * on the FMA pipe for a share of its P = 2^x values (to relieve the MUFU
 * pipe): y[i] = 2^x[i] by a Cody-Waite split x = n + f, n = round(x), and a
 * degree-4 minimax polynomial for 2^f (relative error below 3e-6), with x
 * clamped below at -125 (so every x <= -125 gives 2^-125, which is zero once
 * rounded to the fp16 P operand).  Valid for x <= 64.
 *  - x, y: float32 device arrays of n elements (y may be x); asynchronous on
 *    `stream`; VDN_ERR_INVALID_ARG for NULL pointers. */
VDN_API vdn_status vdn_selftest_exp2(const float *x, float *y, size_t n, vdn_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VDN_H_ */
