/*
 * vit.h -- C ABI of libvit, a B200 (sm_100a) implementation of the vision
 * transformer encoder hot path of an OCR vision-language model:
 *
 *   27 x [ LayerNorm -> QKV GEMM + bias -> 2D RoPE -> bidirectional
 *          multi-head attention -> output projection + bias + residual ->
 *          LayerNorm -> fc1 + bias -> GELU(tanh) -> fc2 + bias + residual ]
 *   followed by the 2x2 spatial merge.
 *
 * Source of the method: KLiteInfer README (PaddleOCR-VL 0.9B vision tower),
 * intro bullet "多模态全流程自研" (SigLIP ViT, 27 layers, 2D RoPE, bidirectional
 * attention, 2x2 spatial merge), section "精度与性能" (27 layers x 3900 tokens
 * of batched GEMMs) and section "架构", paragraph "视觉算子" (row-major batched
 * tokens; GEMM + bias, bidirectional attention, LayerNorm, 2D RoPE, 2x2
 * spatial merge).  The prefix K/V segment follows the LightX2V NeoPP README,
 * section "KV file layout" (online layout [layers, 2, seq, kv_heads, d]).
 *
 * Around the stack: patch embedding and bilinear position-table
 * interpolation (the steps before it), a CUDA-graph capture of any sequence
 * of calls, and an MXFP8 block-scaled linear layer (E4M3 codes, one E8M0
 * scale per 32 elements) with its quantiser.
 *
 * Conventions (all entry points):
 *  - Every tensor pointer is a DEVICE pointer owned by the caller, unless the
 *    parameter name ends in _host.  The library never allocates or frees
 *    device memory, except one 16-byte status word per context (allocated
 *    by vit_init, freed by vit_destroy).
 *  - Activations are row-major [tokens, features] with contiguous rows.
 *    Weights use the [out_features, in_features] row-major layout.
 *  - Element type of every floating tensor = vit_config.dtype (fp32 or bf16);
 *    the MXFP8 entry points take byte codes and scales as documented there.
 *    bf16 runs tcgen05 tensor-core kernels with fp32 accumulation; fp32 runs
 *    SIMT FFMA kernels (no TF32).
 *  - Streams are passed as void* (a cudaStream_t; NULL = legacy stream).  All
 *    work is enqueued asynchronously on that stream.
 *  - All argument and shape checks happen before anything is launched; on an
 *    error status nothing was launched and outputs are untouched.  A failed
 *    launch returns VIT_ERR_CUDA.  Faults detected inside a kernel (a bounded
 *    wait that ran out, an index out of range) set the context's device
 *    status word, read by vit_get_last_device_status().
 *  - Pointers passed to bf16 entry points must be 16-byte aligned, and row
 *    pitches (features x element size) multiples of 16 bytes.
 *  - A context may be used from several host threads and streams at once as
 *    long as each concurrent call has its own workspace.
 */
#ifndef VIT_H_
#define VIT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VIT_API __attribute__((visibility("default")))
#else
#define VIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VIT_OK = 0,
  VIT_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum      */
  VIT_ERR_SHAPE = 2,         /* inconsistent sizes (odd merge grid, T != sum) */
  VIT_ERR_UNSUPPORTED = 3,   /* valid but not implemented (head_dim 96, non-sm_100 device) */
  VIT_ERR_WORKSPACE = 4,     /* workspace missing or too small              */
  VIT_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed        */
  VIT_ERR_TIMEOUT = 6,       /* a kernel's bounded wait ran out (device status) */
  VIT_ERR_DEVICE_BOUNDS = 7  /* a kernel's index check failed (device status) */
} vit_status;

typedef enum { VIT_F32 = 0, VIT_BF16 = 1 } vit_dtype;

/* vit_config.flags */
#define VIT_FLAG_NO_ROPE 0x1u   /* layers skip 2D RoPE                        */
#define VIT_FLAG_NO_MLP  0x2u   /* layers stop after the attention residual   */

typedef struct {
  int hidden;        /* C = heads * head_dim                                 */
  int heads;         /* H                                                    */
  int head_dim;      /* d: 64 (fp32 only), 72 or 128                         */
  int mlp;           /* F, MLP width (ignored with VIT_FLAG_NO_MLP)          */
  float ln_eps;      /* LayerNorm epsilon (biased variance), e.g. 1e-6       */
  float rope_theta;  /* 2D RoPE base, e.g. 10000                             */
  vit_dtype dtype;
  unsigned flags;
} vit_config;

/* One layer's parameters; all device pointers of cfg.dtype.
 * w_qkv [3C, C] (output rows: Q heads 0..H-1, then K, then V; d each),
 * w_o [C, C], w_fc1 [F, C], w_fc2 [C, F]; biases and LayerNorm vectors 1-D.
 * The ln2 / fc pointers may be NULL with VIT_FLAG_NO_MLP.
 *
 * LayerNorm folded into the projection after it (bf16 only; see
 * vit_fold_layernorm): when qkv_fold is not NULL, w_qkv must be the folded
 * weight W_qkv diag(ln1_g) and qkv_fold points to fp32 [2][3C] = (s, c) of
 * that fold; ln1_g, ln1_b and b_qkv are then not read (may be NULL).  The
 * layer then launches no LayerNorm: the QKV GEMM reads the raw x and its
 * epilogue applies the normalisation.  fc1_fold likewise for LN2 and fc1
 * (fp32 [2][F]; ln2_g, ln2_b, b_fc1 not read).  Both NULL: the plain layer. */
typedef struct {
  const void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o;
  const void *ln2_g, *ln2_b, *w_fc1, *b_fc1, *w_fc2, *b_fc2;
  const void *qkv_fold, *fc1_fold;
} vit_layer_weights;

/* Packed variable-length sequences (images).  Tokens of sequence s are rows
 * cu_seqlens[s] .. cu_seqlens[s+1]-1; attention never crosses sequences
 * (block-diagonal mask).  pos_rc[t] = (row, col) of token t in its image
 * grid (NULL: no RoPE).  prefix_kv, if not NULL, holds per sequence P keys
 * and values used as given (no RoPE) in front of the sequence's own keys:
 * layout [n_seqs, 2 (K then V), prefix_len, kv_heads, head_dim]; query head h
 * reads prefix head h / (heads / kv_heads). */
typedef struct {
  int total_tokens;            /* T = cu_seqlens[n_seqs]                     */
  int n_seqs;                  /* >= 1                                       */
  int max_seqlen;              /* >= every sequence length                   */
  const int32_t *cu_seqlens;   /* device [n_seqs + 1], cu_seqlens[0] = 0     */
  const int32_t *pos_rc;       /* device [T, 2] or NULL                      */
  const void *prefix_kv;       /* device, see above, or NULL                 */
  int prefix_len;              /* P (0 when prefix_kv is NULL)               */
  int kv_heads;                /* heads of prefix_kv (0 means = heads)       */
} vit_seqs;

typedef struct vit_ctx vit_ctx;

/* Creates a context for one device.  Checks that the device is sm_100,
 * validates cfg (hidden = heads*head_dim, head_dim in {64,72,128} with 64
 * fp32-only, mlp > 0 unless VIT_FLAG_NO_MLP) and allocates the 16-byte
 * device status word.  *out receives the context (NULL on error). */
VIT_API vit_status vit_init(const vit_config *cfg, int device, vit_ctx **out);

/* Frees the context and its status word.  NULL is ignored. */
VIT_API void vit_destroy(vit_ctx *ctx);

/* Bytes of device workspace vit_layer_forward / vit_encoder_forward need for
 * total_tokens tokens (256-byte aligned base required). */
VIT_API size_t vit_workspace_bytes(const vit_ctx *ctx, int total_tokens);

/* Folds each pre-LayerNorm into the projection that reads its output
 * (KLiteInfer README, 架构 / 视觉算子: LayerNorm, then GEMM + bias, over
 * the same rows).  For a row x with mean m and r = 1/sqrt(var + eps):
 *   LN(x) W^T + b = r (x W'^T - m s) + c,
 *   W' = W diag(gamma),  s_n = sum_k W'_nk,  c = b + W beta,
 * an exact identity; the folded GEMM needs only each row's m and r, which
 * the kernel that wrote the row supplies (see vit_layer_weights), so the
 * LayerNorm kernel and its round trip through memory disappear.
 * Rounding: W' is rounded once to bf16 (in place of the LayerNorm output);
 * s is summed from the rounded W' and c from W and beta, in fp32.
 *   in       the layer's plain weights (ln1_g, ln1_b, w_qkv, b_qkv read for
 *            the QKV fold; ln2_g, ln2_b, w_fc1, b_fc1 for the fc1 fold)
 *   w_qkv_out  [3C, C] bf16 folded weight (may equal in->w_qkv: in place)
 *   qkv_fold   fp32 [2][3C]: s, then c
 *   w_fc1_out  [F, C] bf16 (may equal in->w_fc1),  fc1_fold fp32 [2][F]
 * Either output pair may be NULL to skip that fold (both NULL: nothing is
 * done).  bf16 contexts only (else VIT_ERR_UNSUPPORTED); pointers 16-byte
 * aligned.  Weights of a model are folded once, when they are loaded; the
 * caller then fills a vit_layer_weights with w_qkv = w_qkv_out,
 * qkv_fold = qkv_fold, and so on. */
VIT_API vit_status vit_fold_layernorm(vit_ctx *ctx, const vit_layer_weights *in,
                                      void *w_qkv_out, void *qkv_fold, void *w_fc1_out,
                                      void *fc1_fold, void *stream);

/* One pre-LN encoder layer (reading: x1 = x + Wo Attn(RoPE(Wqkv LN1(x))) + bo;
 * y = x1 + W2 GELU(W1 LN2(x1) + b1) + b2).  x, y: [T, C]; y may not alias x.
 * With VIT_FLAG_NO_MLP y = x1 (DiT-style attention half-layer). */
VIT_API vit_status vit_layer_forward(vit_ctx *ctx, const vit_layer_weights *w,
                             const void *x, void *y, const vit_seqs *seqs,
                             void *workspace, size_t ws_bytes, void *stream);

/* vit_layer_forward without a workspace argument, for callers that cannot
 * allocate device memory when they run a layer: for example a runtime that
 * has already handed all device memory to its own pool, or a latency-critical
 * sequence that must not call cudaMalloc/cudaFree (which can block and
 * synchronise the device).  The pages describe no such call; it exists only
 * for those callers.
 *
 * The layer's intermediates live in one fixed 32 MiB array compiled into the
 * library (a static __device__ array; every GPU that loads the library holds
 * it until the process exits).  The call allocates nothing: no cudaMalloc,
 * cudaFree or allocating library routine.  The caller still passes x, y and
 * the weights, as for vit_layer_forward.
 *  - Size limit: the layer's intermediates (LayerNorm output, qkv, attention
 *    output, x1, MLP hidden, row statistics; no split-attention scratch,
 *    which this call never uses) must fit in 32 MiB: up to 1,227 tokens at
 *    hidden 1152 / MLP 4304.  Larger calls return VIT_ERR_WORKSPACE before
 *    anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, once per device) and keeps it; make that first
 *    call before any stream capture.  The kept address belongs to the
 *    device's primary context: after cudaDeviceReset on that device (which
 *    reloads the library's device code) the process must not call this
 *    entry point again on that device.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents.  Nothing in it has to start at zero (every intermediate is
 *    written before it is read), so nothing is cleared.  Calls whose work
 *    overlaps on the GPU (different streams, no ordering between them) race
 *    on the array: order them, e.g. issue them on one stream.
 *  - Launch counts are kept as for every call; no timing events are created
 *    during this call even when profiling is enabled. */
VIT_API vit_status vit_layer_forward_noalloc(vit_ctx *ctx, const vit_layer_weights *w,
                                             const void *x, void *y, const vit_seqs *seqs,
                                             void *stream);

/* The stack of n_layers layers; layers is a HOST array of n_layers weight
 * structs (device pointers inside).  Intermediate activations live in the
 * workspace; x is read only; y [T, C] receives the last layer's output. */
VIT_API vit_status vit_encoder_forward(vit_ctx *ctx, const vit_layer_weights *layers,
                               int n_layers, const void *x, void *y,
                               const vit_seqs *seqs, void *workspace,
                               size_t ws_bytes, void *stream);

/* ---- CUDA graphs of library calls --------------------------------------
 * Stream capture, so a whole stack (and the merge) replays with one launch.
 * vit_graph_begin returns a stream owned by the context; enqueue any calls of
 * this context on it (their arguments are checked as usual), then
 * vit_graph_end instantiates the captured work into *out.  Every pointer
 * and size passed while capturing is baked into the graph: each launch
 * re-runs the same kernels on the same buffers, which the caller keeps
 * alive and may refill between launches.  One capture per context at a
 * time (else VIT_ERR_INVALID_ARG); a failed capture returns VIT_ERR_CUDA
 * and leaves *out NULL.  The pages have no counterpart: their runtime
 * launches op by op without CUDA graphs (KLiteInfer README, section
 * 已知限制与后续).
 * vit_graph_kernels: this library's kernel launches in one replay. */
typedef struct vit_graph vit_graph;
VIT_API vit_status vit_graph_begin(vit_ctx *ctx, void **capture_stream);
VIT_API vit_status vit_graph_end(vit_ctx *ctx, vit_graph **out);
VIT_API vit_status vit_graph_launch(vit_graph *g, void *stream);
VIT_API long long vit_graph_kernels(const vit_graph *g);
VIT_API void vit_graph_destroy(vit_graph *g);

/* Bidirectional multi-head attention over packed sequences ("视觉算子":
 * softmax(Q K^T * scale) V per head and sequence).  qkv [T, 3, H, d]
 * (the QKV projection's output layout), o [T, H, d].  With seqs->pos_rc the
 * kernel rotates Q and K by 2D RoPE as it loads them, every key tile once
 * per query-tile pair that reads it: a convenience for unrotated inputs,
 * about six times slower at head_dim 72 (3900 tokens: 733 against 121 us)
 * than rotating once (vit_rope2d, or the layer's QKV epilogue) and calling
 * without positions.  scale <= 0 selects 1/sqrt(d). */
VIT_API vit_status vit_attention(vit_ctx *ctx, const void *qkv, void *o,
                         const vit_seqs *seqs, float scale, void *stream);

/* 2x2 spatial merge (intro bullet: Projector, 2x2 spatial merge).  Per image
 * with grid (rows, cols), both even: output token (R, Q) = concat of input
 * tokens (2R,2Q), (2R,2Q+1), (2R+1,2Q), (2R+1,2Q+1).  x [T, channels],
 * y [T/4, 4*channels]; images packed in order.  grids_hw_host: HOST int32
 * [n_images, 2] = (rows, cols).  Odd sides -> VIT_ERR_SHAPE.  Bit-exact. */
VIT_API vit_status vit_spatial_merge_2x2(vit_ctx *ctx, const void *x, void *y,
                                 const int32_t *grids_hw_host, int n_images,
                                 int channels, void *stream);

/* Writes cu_seqlens [n_images+1] and pos_rc [T, 2] (row-major tokens,
 * positions restarting at (0,0) per image) for packed image grids given on
 * the HOST ([n_images, 2] = rows, cols; n_images <= 1024). */
VIT_API vit_status vit_positions_from_grids(vit_ctx *ctx, const int32_t *grids_hw_host,
                                    int n_images, int32_t *cu_seqlens,
                                    int32_t *pos_rc, void *stream);

/* ---- before the encoder: patch embedding + interpolated positions -------
 * KLiteInfer README: section 精度与性能 (patch embedding, the first compared
 * stage) and section 架构, paragraph 视觉算子 (bilinear position-embedding
 * interpolation).  The pages give no patch or table size; both are
 * parameters here.
 *   pixels     images packed in order, image i [3, rows_i*patch,
 *              cols_i*patch], channels first, ctx dtype
 *   grids      HOST int32 [n_images, 2] = (rows, cols) in patches
 *   w_pe       [C, 3*patch*patch]: a stride-patch Conv2d weight [C, 3, patch,
 *              patch], flattened in (channel, y, x) order; b_pe [C]
 *   pos_table  [table_h, table_w, C]
 *   y          [T, C], T = sum rows*cols; token r*cols + c of image i
 * y = patch(t) . w_pe^T + b_pe + table resized bilinearly (half-pixel
 * centres, as PyTorch's align_corners = false) to (rows, cols) at (r, c).
 * 1 <= patch <= 32, n_images <= 1024, C % 8 == 0; b_pe, pos_table, y and the
 * workspace 16-byte aligned.  Workspace:
 * vit_embed_workspace_bytes (patches, padded weight, interpolated table).
 * Launches: one for the GEMM's operands (patch rows and resized position
 * rows), one that pads w_pe to the GEMM's layout (see
 * vit_patch_embed_padded, which skips it), and the GEMM, whose epilogue adds
 * b_pe and the position rows. */
VIT_API size_t vit_embed_workspace_bytes(const vit_ctx *ctx, int total_tokens, int patch);
VIT_API vit_status vit_patch_embed(vit_ctx *ctx, const void *pixels,
                                   const int32_t *grids_hw_host, int n_images, int patch,
                                   const void *w_pe, const void *b_pe, const void *pos_table,
                                   int table_h, int table_w, void *y, void *workspace,
                                   size_t ws_bytes, void *stream);
/* The GEMM's weight layout: w_pad [C, Kp], Kp = vit_patch_kp(patch) = 3 p^2
 * rounded up to a multiple of 8 (a TMA row must be a multiple of 16 bytes),
 * columns 3p^2 .. Kp-1 zero.  vit_pad_patch_weight writes it from w_pe
 * [C, 3 p^2] once (a model constant, as a loader would prepare it);
 * vit_patch_embed_padded is vit_patch_embed with that weight, one launch
 * fewer per call.  vit_patch_kp returns 0 for a patch outside 1..32;
 * w_pad 16-byte aligned; same workspace as vit_patch_embed. */
VIT_API int vit_patch_kp(int patch);
VIT_API vit_status vit_pad_patch_weight(vit_ctx *ctx, const void *w_pe, int patch, void *w_pad,
                                        void *stream);
VIT_API vit_status vit_patch_embed_padded(vit_ctx *ctx, const void *pixels,
                                          const int32_t *grids_hw_host, int n_images, int patch,
                                          const void *w_pad, const void *b_pe,
                                          const void *pos_table, int table_h, int table_w,
                                          void *y, void *workspace, size_t ws_bytes,
                                          void *stream);
/* The interpolation alone: y [T, C] = resized pos_table per image (as above). */
VIT_API vit_status vit_pos_interp(vit_ctx *ctx, const void *pos_table, int table_h, int table_w,
                                  const int32_t *grids_hw_host, int n_images, void *y,
                                  void *stream);

/* ---- projector after the merge ------------------------------------------
 * The KLiteInfer README's intro bullet names the projector only as the 2x2
 * spatial merge (vit_spatial_merge_2x2).  For models that follow the merge
 * with a LayerNorm and a two-layer GELU MLP mapping the merged tokens to the
 * decoder's width, this call runs that composition with caller-chosen
 * widths:
 *   y = GELU_tanh(LN(x) W1^T + b1) W2^T + b2
 * x [M, d_in] (merged tokens, d_in = 4C), LayerNorm over d_in (biased
 * variance, eps = cfg.ln_eps), W1 [d_hidden, d_in], W2 [d_out, d_hidden],
 * y [M, d_out].  Launches: the LayerNorm (a block per row above 4096
 * columns), then two GEMMs (vit_linear's kernels, bias + GELU and bias
 * epilogues).  Workspace: vit_projector_workspace_bytes (LN output and the
 * hidden activations, 256-byte aligned).  bf16: d_in, d_hidden, d_out
 * multiples of 8; d_in <= 16384.  No trained projector is available, so
 * parity is with the fp64 composition only. */
typedef struct {
  const void *ln_g, *ln_b;  /* [d_in] */
  const void *w1, *b1;      /* [d_hidden, d_in], [d_hidden] */
  const void *w2, *b2;      /* [d_out, d_hidden], [d_out] */
} vit_projector_weights;
VIT_API size_t vit_projector_workspace_bytes(const vit_ctx *ctx, int M, int d_in, int d_hidden);
VIT_API vit_status vit_projector(vit_ctx *ctx, const vit_projector_weights *w, const void *x,
                                 void *y, int M, int d_in, int d_hidden, int d_out,
                                 void *workspace, size_t ws_bytes, void *stream);

/* ---- single steps of the layer, exposed for step-level use and testing --- */

/* LayerNorm over the last axis ("视觉算子": LayerNorm), biased variance,
 * y = (x - mean)/sqrt(var + eps) * gamma + beta.  x, y [rows, cols];
 * y may alias x.  cols a multiple of 4, at most 16384 (rows of up to 4096
 * columns take one warp each, wider rows one block each), else
 * VIT_ERR_UNSUPPORTED. */
VIT_API vit_status vit_layernorm(vit_ctx *ctx, const void *x, void *y,
                         const void *gamma, const void *beta, int rows,
                         int cols, float eps, void *stream);

/* Epilogues of vit_linear */
typedef enum {
  VIT_EPI_BIAS = 0,           /* y = x W^T + b                               */
  VIT_EPI_BIAS_GELU = 1,      /* y = GELU_tanh(x W^T + b)                    */
  VIT_EPI_BIAS_RESIDUAL = 2   /* y = residual + x W^T + b (residual [M, N])  */
} vit_epilogue;

/* GEMM + bias with a fused epilogue ("视觉算子": GEMM + bias).  x [M, K],
 * w [N, K], bias [N] (may be NULL), residual [M, N] for
 * VIT_EPI_BIAS_RESIDUAL, y [M, N].  bf16: K and N multiples of 8. */
VIT_API vit_status vit_linear(vit_ctx *ctx, const void *x, const void *w,
                      const void *bias, const void *residual, void *y, int M,
                      int N, int K, vit_epilogue epi, void *stream);

/* 2D RoPE in place on the Q and K parts of qkv [T, 3, H, d] (intro bullet
 * "2D RoPE"): dims [0, d/2) rotate by row, [d/2, d) by column; within a
 * half of width h, dim j pairs with j + h/2 at frequency
 * theta^(-2j/h). */
VIT_API vit_status vit_rope2d(vit_ctx *ctx, void *qkv, const int32_t *pos_rc,
                      int total_tokens, void *stream);

/* ---- MXFP8 (block-scaled 8-bit) linear layer ----
 * The pages name 8-bit inference as a next step without fixing a format (the
 * NEO++ launcher page lists fp8 variants of its dense checkpoints; KLiteInfer
 * README, section "已知限制与后续": FP16 / INT8 after CUDA Graph and operator
 * fusion).  The format here is OCP Microscaling v1.0 MXFP8: E4M3 elements
 * (bias 7, max 448, no infinity), one E8M0 scale 2^(s-127) per 32
 * consecutive elements of a row.  bf16 contexts only.
 *
 * codes  : [rows, vit_mx8_row_bytes(K)] bytes, element (r, k) at
 *          r * row_bytes + k (bytes past K are never read).
 * scales : vit_mx8_scale_bytes(rows, K) bytes of 512-byte blocks, block
 *          (rb, kb) = rows [128 rb, 128 rb + 128) x columns [128 kb, 128 kb +
 *          128) at (rb * ceil(K/128) + kb) * 512; inside it the scale of row
 *          128 rb + r0 + 32 r1 (r0 < 32, r1 < 4) and of its 32-column group j
 *          (< 4) at byte 16 r0 + 4 r1 + j (the tensor core's scale-copy
 *          shape).  Bytes of rows or groups past the matrix hold 127 (2^0).
 * All buffers belong to the caller; device pointers 16-byte aligned. */
VIT_API size_t vit_mx8_row_bytes(int K);
VIT_API size_t vit_mx8_scale_bytes(int rows, int K);

/* x bf16 [rows, K] (row stride K) -> codes, scales.  Per 32-element group:
 * X = floor(log2 max|x|) - 8 clamped to [-127, 127] (-127 for an all-zero
 * group), code = E4M3(x / 2^X) rounded to nearest even, magnitudes above 448
 * clamped to 448.  Errors: VIT_ERR_INVALID_ARG (null or misaligned pointer,
 * negative size), VIT_ERR_UNSUPPORTED (fp32 context). */
VIT_API vit_status vit_mx8_quantize(vit_ctx *ctx, const void *x, int rows, int K,
                                    void *codes, void *scales, void *stream);

/* LayerNorm straight to MXFP8: codes, scales = vit_mx8_quantize(bf16 of
 * vit_layernorm(x, gamma, beta)), bit for bit, in one launch (the FP8
 * layer's LayerNorms).  x bf16 [rows, cols], gamma / beta [cols], eps as
 * vit_layernorm.  cols a multiple of 4, at most 1536 (VIT_ERR_UNSUPPORTED
 * beyond, or in an fp32 context); errors otherwise as vit_mx8_quantize. */
VIT_API vit_status vit_layernorm_mx8(vit_ctx *ctx, const void *x, const void *gamma,
                                     const void *beta, int rows, int cols, float eps, void *codes,
                                     void *scales, void *stream);

/* y bf16 [M, N] = epi(deq(A) deq(W)^T + bias) with A = (a_codes, a_scales)
 * [M, K] and W = (w_codes, w_scales) [N, K] (a PyTorch Linear weight,
 * quantised along K); bias bf16 [N] or NULL; residual bf16 [M, N] for
 * VIT_EPI_BIAS_RESIDUAL.  fp32 accumulation on the tensor core (block-scaled
 * MMA).  N a multiple of 8.  Errors as vit_linear. */
VIT_API vit_status vit_linear_mx8(vit_ctx *ctx, const void *a_codes, const void *a_scales,
                                  const void *w_codes, const void *w_scales, const void *bias,
                                  const void *residual, void *y, int M, int N, int K,
                                  vit_epilogue epi, void *stream);

/* ---- FP8 encoder layers ------------------------------------------------
 * The encoder layer with its four projections (QKV, output, fc1, fc2) in
 * MXFP8 (reading: the pages list fp8 variants of dense checkpoints and put
 * FP16 / INT8 on the KLiteInfer road map, without a format; OCP MX v1.0
 * MXFP8 E4M3 is taken).  Per projection the input activation is quantised
 * along K (vit_mx8_quantize's rule: the bf16 activation, quantised) and
 * multiplied with the weight's codes by the block-scaled tensor-core GEMM
 * (vit_linear_mx8); LayerNorm, RoPE (a pass over the projection output),
 * attention, GELU and the residual adds are those of the bf16 layer.  The
 * quantisation is fused where the producer holds whole 32-element groups:
 * the two LayerNorms write MXFP8 directly (hidden <= 1536), and fc1's
 * epilogue writes GELU's output as MXFP8 for fc2; the attention output has
 * its own pass (its 72-wide heads split the groups).  Nine launches per
 * layer.  Weights are quantised once by the caller with vit_mx8_quantize
 * (w_* [out, in] along in); the LayerNorm vectors and biases stay bf16.
 * bf16 contexts only.
 * Workspace: vit_workspace_bytes_mx8 (the bf16 layer's buffers plus two
 * quantised activations, K = hidden and K = MLP width).  Errors as vit_encoder_forward; the folded
 * LayerNorm and prefix K/V are not supported here (VIT_ERR_UNSUPPORTED). */
typedef struct {
  const void *ln1_g, *ln1_b, *b_qkv, *b_o, *ln2_g, *ln2_b, *b_fc1, *b_fc2;  /* bf16 */
  const void *w_qkv_codes, *w_qkv_scales, *w_o_codes, *w_o_scales;
  const void *w_fc1_codes, *w_fc1_scales, *w_fc2_codes, *w_fc2_scales;
} vit_layer_weights_mx8;
VIT_API size_t vit_workspace_bytes_mx8(const vit_ctx *ctx, int total_tokens);
VIT_API vit_status vit_encoder_forward_mx8(vit_ctx *ctx, const vit_layer_weights_mx8 *layers,
                                           int n_layers, const void *x, void *y,
                                           const vit_seqs *seqs, void *workspace,
                                           size_t ws_bytes, void *stream);

/* ---- launch accounting and per-kernel timing ---- */

/* Kernel kinds counted by the context (one count per kernel launch). */
typedef enum {
  VIT_K_LAYERNORM = 0, VIT_K_GEMM_QKV = 1, VIT_K_ROPE = 2, VIT_K_ATTENTION = 3,
  VIT_K_GEMM_OUT = 4, VIT_K_GEMM_FC1 = 5, VIT_K_GEMM_FC2 = 6, VIT_K_MERGE = 7,
  VIT_K_POSITIONS = 8, VIT_K_GEMM = 9, /* vit_linear, the patch projection */
  VIT_K_EMBED = 10, /* patch extraction, weight padding, position interpolation */
  VIT_K_MX8_QUANTIZE = 11, VIT_K_GEMM_MX8 = 12, /* vit_mx8_quantize, vit_linear_mx8 */
  VIT_K_ROWSTATS = 13, /* row statistics of a stack's input (folded LayerNorm) */
  VIT_K_FOLD = 14,     /* vit_fold_layernorm */
  VIT_K_COUNT = 15
} vit_kernel_kind;

/* enable != 0: every later kernel launch of this context is bracketed by two
 * CUDA events recorded on its stream (host-side objects, no device memory);
 * enable == 0 stops recording.  Not thread-safe while enabled. */
VIT_API vit_status vit_profile_enable(vit_ctx *ctx, int enable);

/* For kernel kind `kind`: *launches = launches since the last reset (always
 * counted), *total_ms = summed device time of the launches recorded while
 * profiling was enabled (synchronises on the recorded events).  reset != 0
 * clears the counts and recorded events of every kind after reading. */
VIT_API vit_status vit_profile_read(vit_ctx *ctx, int kind, long long *launches,
                                    double *total_ms, int reset);

/* ---- status ---- */

/* Synchronises the device, reads the context's device status word, clears
 * it and returns VIT_OK, VIT_ERR_TIMEOUT or VIT_ERR_DEVICE_BOUNDS (or
 * VIT_ERR_CUDA when the device reports an error). */
VIT_API vit_status vit_get_last_device_status(vit_ctx *ctx);

/* Fault injection for tests of the bounded waits; the pages have no
 * counterpart.  With bytes > 0, every later one-CTA GEMM launch of this
 * context (vit_linear with at most 128 rows always takes that kernel)
 * announces `bytes` more per pipeline stage than its copies deliver, so the
 * stage barrier never completes.  The kernel's waits are bounded (2 s): it
 * winds down, waits for its copies, frees its tensor memory and records
 * VIT_ERR_TIMEOUT, which vit_get_last_device_status() returns; the context
 * stays usable.  bytes = 0 (the default) turns the injection off; values
 * above 65536 return VIT_ERR_INVALID_ARG. */
VIT_API vit_status vit_debug_lost_tx(vit_ctx *ctx, unsigned bytes);

/* Static string for a status code. */
VIT_API const char *vit_status_string(vit_status s);

/* Library version string, e.g. "libvit 0.1 sm_100a". */
VIT_API const char *vit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VIT_H_ */
