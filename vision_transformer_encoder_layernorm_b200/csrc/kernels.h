// kernels.h -- launchers of libvit's kernels (internal; the public ABI is
// include/vit.h).  Every launcher enqueues on the given stream and returns
// the launch status; argument validation happens in vit_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <stdlib.h>

#include <algorithm>

#include "common.cuh"

namespace vit {

constexpr int kF32 = 0;
constexpr int kBF16 = 1;

// Per-image table passed by value (__grid_constant__) to the merge and
// positions kernels; a call covers at most kMaxImagesPerLaunch images.
constexpr int kMaxImagesPerLaunch = 256;
struct ImageEntry {
  int rows, cols;
  int base;  // first token of the image in the packed sequence
};
struct ImageTable {
  ImageEntry img[kMaxImagesPerLaunch];
};

// Rotation frequencies divided by pi, wpi[j] = theta^(-2j/h) / pi for
// j < d/4, h = d/2 (computed on the host in fp64).  Kernels evaluate the
// rotation as sincospif(p * wpi[j]), whose argument reduction is exact.
struct RopeFreqs {
  float wpi[32];
};

// Sequence description shared by the attention kernels.
struct SeqArgs {
  int total_tokens, n_seqs, max_seqlen;
  const int32_t *cu_seqlens;
  const int32_t *pos;      // [T, 2] or null
  const void *prefix_kv;   // [S, 2, P, Hkv, d] or null
  int prefix_len, kv_heads;
};

cudaError_t launch_layernorm(int dtype, const void *x, void *y, const void *g, const void *b,
                             int rows, int cols, float eps, cudaStream_t st);
// LayerNorm of bf16 rows straight to MXFP8 codes and scales (layout as
// launch_mx8_quantize; the bf16-rounded LayerNorm quantised); cols % 4 == 0,
// cols <= 1536.
cudaError_t launch_layernorm_mx8(const void *x, const void *g, const void *b, int rows, int cols,
                                 float eps, uint8_t *codes, uint8_t *scales, cudaStream_t st);
cudaError_t launch_merge2x2(const ImageTable &tab, int n_images, const void *x, void *y,
                            size_t row_bytes, long long max_out_tokens, cudaStream_t st);
cudaError_t launch_positions(const ImageTable &tab, int n_images, int cu_offset_index,
                             int max_tokens, int32_t *cu, int32_t *pos, cudaStream_t st);
cudaError_t launch_rope2d(int dtype, void *qkv, const int32_t *pos, int T, int H, int d,
                          const RopeFreqs &fr, cudaStream_t st);

// patch embedding inputs (k_embed.cu)
cudaError_t launch_embed_inputs(int dtype, const ImageTable &tab, int n_images,
                                long long max_tokens, const void *px, void *patches, int p, int kp,
                                const void *table, int gh, int gw, int C, void *pos,
                                cudaStream_t st);
cudaError_t launch_pad_cols(int dtype, const void *w, void *out, int n, int k, int kp,
                            cudaStream_t st);
cudaError_t launch_pos_interp(int dtype, const ImageTable &tab, int n_images, long long max_tokens,
                              const void *table, int gh, int gw, int C, void *y, cudaStream_t st);

// Epilogue codes: an operation (the low two bits; 0-2 match vit_epilogue)
// and two flags.
constexpr int kEpiBias = 0;
constexpr int kEpiGelu = 1;
constexpr int kEpiResidual = 2;
constexpr int kEpiRope = 3;  // bias, then 2D RoPE on columns < rot_cols (QKV projection)
constexpr int kEpiOpMask = 3;
// LayerNorm folded into this GEMM: A is the raw row x (length K), the weight
// was folded to w' = w diag(gamma), and the epilogue forms
// rstd (acc - mean s) + c in place of acc + bias (see EpiArgs).
constexpr int kEpiLn = 4;
// The output rows' statistics, per slice of the columns one epilogue warp
// writes, go to EpiArgs::stats_out (for a later kEpiLn GEMM on this output).
constexpr int kEpiStats = 8;
// MXFP8 output (MXFP8 GEMM only): each 32-column chunk of a row, rounded to
// bf16, is quantised as launch_mx8_quantize does; codes go to y viewed as
// bytes with row stride q_row_bytes, scales to q_scales (its 512-byte blocks,
// padding entries 127)
constexpr int kEpiQuant = 16;

// Per-row statistics of a row's column slices: slice j covers columns
// [j w, min((j + 1) w, n)); entry (mean, M2) = mean of the slice and the sum
// of squared deviations from it.  A row's slices merge (Chan's pairwise
// update) into the row's mean and biased variance M2 / n.
struct SliceStats {
  float2 *p;   // [rows][parts]
  int parts;   // ceil(n / w)
  int w;       // slice width (columns)
};

// Epilogue operands of the tensor-core GEMMs (passed by value, __grid_constant__).
struct EpiArgs {
  const __nv_bfloat16 *bias;  // [N] or null; not read with kEpiLn
  const __nv_bfloat16 *res;   // [M, N] residual (kEpiResidual)
  __nv_bfloat16 *y;           // [M, N] output
  // kEpiLn: fp32 [2][N]: s = row sums of the folded weight, c = b + w beta;
  // stats_in: slice statistics of the rows of A (row length K)
  const float *ln_sc;
  SliceStats stats_in;
  float ln_eps;
  // kEpiStats: slice statistics of the (bf16-rounded) output rows, slice
  // width = half the tile width (gemm_stats_width)
  SliceStats stats_out;
  // kEpiQuant: scales of the MXFP8 output, row stride of its codes, and its
  // 128-column blocks
  uint8_t *q_scales;
  size_t q_row_bytes;
  int q_kblocks;
};

// Arguments of the RoPE epilogue: the GEMM's tile width is 2 * head_dim so
// each epilogue warp holds whole heads; output columns [0, rot_cols) (Q and
// K) are rotated by the row's position pos[row] = (r, c).
struct RopeEpi {
  const int32_t *pos;
  int rot_cols;
  int head_dim;
  RopeFreqs fr;
};

// SIMT GEMM (fp32 FFMA; fp32 or bf16 storage): y = epi(x w^T + b).
cudaError_t launch_gemm_simt(int dtype, const void *x, const void *w, const void *b,
                             const void *res, void *y, int M, int N, int K, int epi,
                             cudaStream_t st);

// SIMT attention (fp32 math; fp32 or bf16 storage).
cudaError_t launch_attention_simt(int dtype, const void *qkv, void *o, const SeqArgs &s, int H,
                                  int d, float scale, const RopeFreqs &fr, int *status,
                                  cudaStream_t st);

// tcgen05 GEMM, bf16 in / bf16 out, fp32 accumulation in TMEM.
struct GemmPlan;
// lost_tx: fault injection for the watchdog tests (0 in normal use): the
// one-CTA kernel's stage barriers expect this many bytes more than arrive.
// With kEpiStats, ea.stats_out.w must equal gemm_stats_width(M, N, K).
cudaError_t launch_gemm_tc(const void *x, const void *w, const EpiArgs &ea, int M, int N, int K,
                           int epi, int num_sms, cudaStream_t st, int *status,
                           const RopeEpi *rope = nullptr, uint32_t lost_tx = 0);
// Slice width of the row statistics a kEpiStats GEMM of this shape writes.
int gemm_stats_width(int M, int N, int K, int num_sms);

// Row statistics of x [rows, cols] bf16 in slices of 64 columns.
constexpr int kRowStatsWidth = 64;
cudaError_t launch_rowstats(const void *x, float2 *out, int rows, int cols, cudaStream_t st);
// LayerNorm folded into the following projection w [n, k] (bias b [n], LN
// gamma/beta [k]): w_out = bf16(w diag(gamma)), sc = fp32 [2][n]:
// s = row sums of w_out, c = b + w beta.
cudaError_t launch_fold_ln(const void *w, const void *gamma, const void *beta, const void *b,
                           void *w_out, float *sc, int n, int k, cudaStream_t st);

// tcgen05 flash attention, bf16, head_dim 72 or 128.
// Split (stream-K) attention schedule: most CTAs it uses, and the bytes of
// partial rows each of them needs in the workspace.
int attn_split_max_ctas();
bool attn_split_possible(int T, int H, int grid);
bool attn_split_enabled();
size_t attn_split_part_bytes();
cudaError_t launch_attention_tc(const void *qkv, void *o, const SeqArgs &s, int H, int d,
                                float scale, const RopeFreqs &fr, int num_sms, int *status,
                                float *part, int *cnt,
                                cudaStream_t st);

// Launches `kern` with programmatic dependent launch allowed (and a cluster
// of cluster_x CTAs when cluster_x > 1).  Kernels launched this way call
// pdl_wait() before touching global memory.  VIT_NO_PDL=1 in the environment
// turns the attribute off (plain stream order).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, unsigned cluster_x, Args... args) {
  static const bool pdl_off = [] {
    const char *e = getenv("VIT_NO_PDL");
    return e != nullptr && e[0] == '1';
  }();
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (!pdl_off) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Driver entry point for cuTensorMapEncodeTiled (resolved once).
CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                              uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz);

}  // namespace vit
