// vit_api.cu -- the C ABI of include/vit.h: argument validation (always
// before any launch), workspace carving, and the order of kernel launches for
// one encoder layer and for the stack.
//
// Layer (pre-LN reading of the KLiteInfer README, "视觉算子" op list):
//   h  = LN1(x)                      layernorm kernel
//   qkv = h Wqkv^T + bqkv            GEMM (bias epilogue; bf16: + 2D RoPE on Q, K)
//   qkv[Q,K] = RoPE2D(qkv[Q,K])      fp32 mode: rope kernel, in place (workspace)
//   a  = Attn(qkv)                   attention kernel (varlen, prefix)
//   x1 = x + a Wo^T + bo             GEMM (bias + residual epilogue)
//   h  = LN2(x1)                     layernorm kernel
//   g  = GELU(h W1^T + b1)           GEMM (bias + GELU epilogue)
//   y  = x1 + g W2^T + b2            GEMM (bias + residual epilogue)
// bf16 runs the tcgen05 GEMM / attention kernels, fp32 the SIMT ones.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include <new>

#include "../../include/vit.h"
#include "kernels.h"
#include "mx8.h"

// Launch accounting: a count per kernel kind, and (while enabled) a pair of
// CUDA events around every launch.
struct VitProfiler {
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  bool on = false;
  long long launches[VIT_K_COUNT] = {};
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void clear() {
    for (auto &r : recs) {
      pool.push_back(r.a);
      pool.push_back(r.b);
    }
    recs.clear();
    for (auto &l : launches) l = 0;
  }
  void destroy() {
    clear();
    for (auto e : pool) cudaEventDestroy(e);
    pool.clear();
  }
};

struct vit_ctx {
  vit_config cfg;
  int device;
  int num_sms;
  int *d_status;  // 4 ints; [0] = first error code recorded by a kernel
  vit::RopeFreqs fr;
  VitProfiler prof;
  // stream capture in progress (vit_graph_begin .. vit_graph_end)
  cudaStream_t cap_stream = nullptr;
  bool cap_prof_on = false;
  long long cap_launches0 = 0;
  // fault injection (vit_debug_lost_tx): extra bytes the one-CTA GEMM's
  // stage barriers wait for; 0 in normal use
  uint32_t debug_lost_tx = 0;
};

struct vit_graph {
  cudaGraphExec_t exec = nullptr;
  int device = 0;
  long long kernels = 0;  // library kernel launches captured
};

namespace {

using namespace vit;

struct DeviceGuard {
  int prev = -1;
  bool changed = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
      changed = cudaSetDevice(dev) == cudaSuccess;
    }
  }
  ~DeviceGuard() {
    if (changed) cudaSetDevice(prev);
  }
};

inline size_t esize(const vit_config &c) { return c.dtype == VIT_F32 ? 4 : 2; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

vit_status cuda_status(cudaError_t e) { return e == cudaSuccess ? VIT_OK : VIT_ERR_CUDA; }

// Runs one kernel launch `f` of kind `kind` with launch accounting.
template <class F>
cudaError_t counted(vit_ctx *ctx, int kind, cudaStream_t st, F &&f) {
  VitProfiler &p = ctx->prof;
  p.launches[kind]++;
  if (!p.on) return f();
  cudaEvent_t a = p.get(), b = p.get();
  cudaEventRecord(a, st);
  const cudaError_t e = f();
  cudaEventRecord(b, st);
  p.recs.push_back({kind, a, b});
  return e;
}

vit_status check_seqs(const vit_ctx *ctx, const vit_seqs *s, bool allow_prefix) {
  if (!s) return VIT_ERR_INVALID_ARG;
  if (s->total_tokens < 0 || s->n_seqs < 1 || s->max_seqlen < 0) return VIT_ERR_INVALID_ARG;
  if (s->total_tokens > 0 && (!s->cu_seqlens || s->max_seqlen < 1)) return VIT_ERR_INVALID_ARG;
  if (s->max_seqlen > s->total_tokens) return VIT_ERR_SHAPE;
  if (s->prefix_kv) {
    if (!allow_prefix) return VIT_ERR_INVALID_ARG;
    if (s->prefix_len <= 0) return VIT_ERR_SHAPE;
    const int hkv = s->kv_heads > 0 ? s->kv_heads : ctx->cfg.heads;
    if (hkv > ctx->cfg.heads || ctx->cfg.heads % hkv) return VIT_ERR_SHAPE;
    if (ctx->cfg.dtype == VIT_BF16 && !aligned16(s->prefix_kv)) return VIT_ERR_INVALID_ARG;
  } else if (s->prefix_len != 0) {
    return VIT_ERR_INVALID_ARG;
  }
  return VIT_OK;
}

SeqArgs to_seq_args(const vit_seqs *s, bool with_pos) {
  SeqArgs a;
  a.total_tokens = s->total_tokens;
  a.n_seqs = s->n_seqs;
  a.max_seqlen = s->max_seqlen;
  a.cu_seqlens = s->cu_seqlens;
  a.pos = with_pos ? s->pos_rc : nullptr;
  a.prefix_kv = s->prefix_kv;
  a.prefix_len = s->prefix_kv ? s->prefix_len : 0;
  a.kv_heads = s->kv_heads;
  return a;
}

EpiArgs epi_args(const void *b, const void *res, void *y) {
  EpiArgs ea{};
  ea.bias = static_cast<const __nv_bfloat16 *>(b);
  ea.res = static_cast<const __nv_bfloat16 *>(res);
  ea.y = static_cast<__nv_bfloat16 *>(y);
  return ea;
}

// y = epi(x w^T ...): the SIMT kernel for fp32 contexts (plain epilogues
// only), the tcgen05 kernel for bf16.
cudaError_t run_linear(vit_ctx *ctx, int kind, const void *x, const void *w, const EpiArgs &ea,
                       int M, int N, int K, int epi, cudaStream_t st,
                       const RopeEpi *rope = nullptr) {
  return counted(ctx, kind, st, [&] {
    if (ctx->cfg.dtype == VIT_F32) {
      if (epi & ~kEpiOpMask) return cudaErrorInvalidValue;
      return launch_gemm_simt(kF32, x, w, ea.bias, ea.res, ea.y, M, N, K, epi, st);
    }
    return launch_gemm_tc(x, w, ea, M, N, K, epi, ctx->num_sms, st, ctx->d_status, rope,
                          ctx->debug_lost_tx);
  });
}

cudaError_t run_attention(vit_ctx *ctx, const void *qkv, void *o, const SeqArgs &s, float scale,
                          cudaStream_t st, float *part = nullptr, int *cnt = nullptr) {
  const vit_config &c = ctx->cfg;
  return counted(ctx, VIT_K_ATTENTION, st, [&] {
    if (c.dtype == VIT_F32)
      return launch_attention_simt(kF32, qkv, o, s, c.heads, c.head_dim, scale, ctx->fr,
                                   ctx->d_status, st);
    return launch_attention_tc(qkv, o, s, c.heads, c.head_dim, scale, ctx->fr, ctx->num_sms,
                               ctx->d_status, part, cnt, st);
  });
}

struct Workspace {
  void *h, *qkv, *attn, *x1, *g, *act[2];
  void *part, *cnt;  // split attention: partial rows and per-item counters (or null)
  // slice statistics of the layer input x and of x1 (folded LayerNorms, bf16)
  float2 *stats_x, *stats_x1;
};

// Most slices a row's statistics take: the narrowest slice written is 64
// columns (the row-statistics kernel, and the half tile of the narrowest
// GEMM tile, 128 columns)
inline int max_stat_parts(int C) { return (C + 63) / 64; }

// Whether slice statistics of the layer input are in ws.stats_x, and their
// slice width.
struct StatsState {
  bool valid = false;
  int w = 0;
};

// CTAs of the split attention schedule whose scratch the workspace holds
// for T tokens (bf16 at head_dim 72, large enough to split; 0 = none)
int split_ctas(const vit_ctx *ctx, int T) {
  if (ctx->cfg.dtype != VIT_BF16 || ctx->cfg.head_dim != 72 || !attn_split_enabled()) return 0;
  const int g = std::min(ctx->num_sms, attn_split_max_ctas());
  return attn_split_possible(T, ctx->cfg.heads, g) ? g : 0;
}

size_t workspace_layout(const vit_config &c, int T, Workspace *w, void *base, int sk_ctas) {
  const size_t es = esize(c);
  const size_t C = size_t(c.hidden);
  const size_t F = (c.flags & VIT_FLAG_NO_MLP) ? 0 : size_t(c.mlp);
  const size_t st = c.dtype == VIT_BF16 ? size_t(T) * max_stat_parts(c.hidden) * sizeof(float2) : 0;
  constexpr int kSlots = 11;
  const size_t sizes[kSlots] = {T * C * es, T * 3 * C * es, T * C * es, T * C * es,
                                T * F * es, T * C * es, T * C * es,
                                size_t(sk_ctas) * attn_split_part_bytes(), size_t(sk_ctas) * 4,
                                st, st};
  size_t off = 0;
  void *ptrs[kSlots];
  for (int i = 0; i < kSlots; ++i) {
    ptrs[i] = sizes[i] && base ? static_cast<char *>(base) + off : nullptr;
    off += align256(sizes[i]);
  }
  if (w) {
    w->h = ptrs[0]; w->qkv = ptrs[1]; w->attn = ptrs[2]; w->x1 = ptrs[3]; w->g = ptrs[4];
    w->act[0] = ptrs[5]; w->act[1] = ptrs[6]; w->part = ptrs[7]; w->cnt = ptrs[8];
    w->stats_x = static_cast<float2 *>(ptrs[9]);
    w->stats_x1 = static_cast<float2 *>(ptrs[10]);
  }
  return off;
}

vit_status check_layer_weights(const vit_config &c, const vit_layer_weights *w) {
  if (!w) return VIT_ERR_INVALID_ARG;
  auto ok = [&](const void *p) { return p && (c.dtype != VIT_BF16 || aligned16(p)); };
  const bool no_mlp = (c.flags & VIT_FLAG_NO_MLP) != 0;
  if ((w->qkv_fold || (w->fc1_fold && !no_mlp)) && c.dtype != VIT_BF16) return VIT_ERR_UNSUPPORTED;
  // a folded LayerNorm leaves its gamma, beta and the projection's bias unread
  const void *need[4] = {w->w_qkv, w->w_o, w->b_o, w->qkv_fold ? w->qkv_fold : w->b_qkv};
  for (const void *p : need)
    if (!ok(p)) return VIT_ERR_INVALID_ARG;
  if (!w->qkv_fold && !(ok(w->ln1_g) && ok(w->ln1_b))) return VIT_ERR_INVALID_ARG;
  if (!no_mlp) {
    const void *mlp[4] = {w->w_fc1, w->w_fc2, w->b_fc2, w->fc1_fold ? w->fc1_fold : w->b_fc1};
    for (const void *p : mlp)
      if (!ok(p)) return VIT_ERR_INVALID_ARG;
    if (!w->fc1_fold && !(ok(w->ln2_g) && ok(w->ln2_b))) return VIT_ERR_INVALID_ARG;
  }
  return VIT_OK;
}

// One layer; all arguments already validated.  xs: whether ws.stats_x holds
// the slice statistics of x (updated to those of y when out_stats, i.e. the
// next layer folds its first LayerNorm; else cleared).
vit_status layer_impl(vit_ctx *ctx, const vit_layer_weights *w, const void *x, void *y,
                      const vit_seqs *seqs, const Workspace &ws, cudaStream_t st, StatsState &xs,
                      bool out_stats) {
  const vit_config &c = ctx->cfg;
  const int T = seqs->total_tokens, C = c.hidden, F = c.mlp;
  const int dt = c.dtype == VIT_F32 ? kF32 : kBF16;
  const bool rope = !(c.flags & VIT_FLAG_NO_ROPE) && seqs->pos_rc != nullptr;
  const bool no_mlp = (c.flags & VIT_FLAG_NO_MLP) != 0;
  const float scale = 1.0f / sqrtf(float(c.head_dim));
  auto ln = [&](const void *in, const void *g, const void *b) {
    return counted(ctx, VIT_K_LAYERNORM, st, [&] {
      return launch_layernorm(dt, in, ws.h, g, b, T, C, c.ln_eps, st);
    });
  };
  auto slices = [&](float2 *p, int width) { return SliceStats{p, (C + width - 1) / width, width}; };
  // ---- LN1 + QKV (+ RoPE).  bf16: the QKV GEMM rotates Q and K in its
  // epilogue (tiles of whole heads); fp32: a separate RoPE pass.  With the
  // first LayerNorm folded, the GEMM reads x itself and normalises in its
  // epilogue from x's slice statistics.
  const bool fused_rope = rope && dt == kBF16 && (c.head_dim == 72 || c.head_dim == 128);
  RopeEpi re{};
  if (fused_rope) {
    re.pos = seqs->pos_rc;
    re.rot_cols = 2 * C;
    re.head_dim = c.head_dim;
    re.fr = ctx->fr;
  }
  int epi_q = fused_rope ? kEpiRope : kEpiBias;
  EpiArgs eq = epi_args(w->b_qkv, nullptr, ws.qkv);
  const void *a_qkv = ws.h;
  if (w->qkv_fold) {
    if (!xs.valid) {
      if (counted(ctx, VIT_K_ROWSTATS, st,
                  [&] { return launch_rowstats(x, ws.stats_x, T, C, st); }))
        return VIT_ERR_CUDA;
      xs.valid = true;
      xs.w = kRowStatsWidth;
    }
    eq.bias = nullptr;
    eq.ln_sc = static_cast<const float *>(w->qkv_fold);
    eq.stats_in = slices(ws.stats_x, xs.w);
    eq.ln_eps = c.ln_eps;
    epi_q |= kEpiLn;
    a_qkv = x;
  } else if (ln(x, w->ln1_g, w->ln1_b)) {
    return VIT_ERR_CUDA;
  }
  if (run_linear(ctx, VIT_K_GEMM_QKV, a_qkv, w->w_qkv, eq, T, 3 * C, C, epi_q, st,
                 fused_rope ? &re : nullptr))
    return VIT_ERR_CUDA;
  if (rope && !fused_rope && counted(ctx, VIT_K_ROPE, st, [&] {
        return launch_rope2d(dt, ws.qkv, seqs->pos_rc, T, c.heads, c.head_dim, ctx->fr, st);
      }))
    return VIT_ERR_CUDA;
  // ---- attention
  const SeqArgs sa = to_seq_args(seqs, false);
  if (run_attention(ctx, ws.qkv, ws.attn, sa, scale, st, static_cast<float *>(ws.part),
                    static_cast<int *>(ws.cnt)))
    return VIT_ERR_CUDA;
  // ---- out-projection + residual; it writes the slice statistics of its
  // output when a folded LayerNorm reads that output next
  const bool fold2 = !no_mlp && w->fc1_fold != nullptr;
  const bool stats_o = no_mlp ? out_stats : fold2;
  EpiArgs eo = epi_args(w->b_o, x, no_mlp ? y : ws.x1);
  int epi_o = kEpiResidual, w_o = 0;
  if (stats_o) {
    w_o = gemm_stats_width(T, C, C, ctx->num_sms);
    eo.stats_out = slices(no_mlp ? ws.stats_x : ws.stats_x1, w_o);
    epi_o |= kEpiStats;
  }
  if (run_linear(ctx, VIT_K_GEMM_OUT, ws.attn, w->w_o, eo, T, C, C, epi_o, st))
    return VIT_ERR_CUDA;
  if (no_mlp) {
    xs.valid = out_stats;
    xs.w = w_o;
    return VIT_OK;
  }
  // ---- LN2 + fc1 + GELU
  EpiArgs e1 = epi_args(w->b_fc1, nullptr, ws.g);
  int epi_1 = kEpiGelu;
  const void *a_fc1 = ws.h;
  if (fold2) {
    e1.bias = nullptr;
    e1.ln_sc = static_cast<const float *>(w->fc1_fold);
    e1.stats_in = slices(ws.stats_x1, w_o);
    e1.ln_eps = c.ln_eps;
    epi_1 |= kEpiLn;
    a_fc1 = ws.x1;
  } else if (ln(ws.x1, w->ln2_g, w->ln2_b)) {
    return VIT_ERR_CUDA;
  }
  if (run_linear(ctx, VIT_K_GEMM_FC1, a_fc1, w->w_fc1, e1, T, F, C, epi_1, st))
    return VIT_ERR_CUDA;
  // ---- fc2 + residual (+ the next layer's input statistics)
  EpiArgs e2 = epi_args(w->b_fc2, ws.x1, y);
  int epi_2 = kEpiResidual, w_2 = 0;
  if (out_stats) {
    w_2 = gemm_stats_width(T, C, F, ctx->num_sms);
    e2.stats_out = slices(ws.stats_x, w_2);
    epi_2 |= kEpiStats;
  }
  if (run_linear(ctx, VIT_K_GEMM_FC2, ws.g, w->w_fc2, e2, T, C, F, epi_2, st))
    return VIT_ERR_CUDA;
  xs.valid = out_stats;
  xs.w = w_2;
  return VIT_OK;
}

// sk_ctas: CTAs of the split attention schedule whose scratch the caller's
// workspace layout holds (split_ctas(), or 0 where the split is never used)
vit_status check_layer_call(vit_ctx *ctx, const void *x, void *y, const vit_seqs *seqs,
                            void *workspace, size_t ws_bytes, int sk_ctas) {
  if (!ctx) return VIT_ERR_INVALID_ARG;
  vit_status s = check_seqs(ctx, seqs, true);
  if (s != VIT_OK) return s;
  if (seqs->total_tokens == 0) return VIT_OK;  // nothing is read or written
  if (!x || !y || x == y) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype == VIT_BF16 && (!aligned16(x) || !aligned16(y))) return VIT_ERR_INVALID_ARG;
  if (seqs->total_tokens > 0 && !(ctx->cfg.flags & VIT_FLAG_NO_ROPE) && !seqs->pos_rc)
    return VIT_ERR_INVALID_ARG;
  const size_t need = workspace_layout(ctx->cfg, seqs->total_tokens, nullptr, nullptr, sk_ctas);
  if (!workspace || ws_bytes < need) return VIT_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return VIT_ERR_WORKSPACE;
  return VIT_OK;
}

}  // namespace

// ---------------------------------------------------------------- embedding helpers
namespace {

int embed_kp(int patch) { return (3 * patch * patch + 7) & ~7; }  // TMA rows: 16-byte multiples

// Validates the image grids (host) and packs them into launch tables of at
// most kMaxImagesPerLaunch images; returns the total token count (or < 0).
long long embed_tokens(const int32_t *grids, int n_images) {
  if (!grids || n_images < 1 || n_images > 1024) return -1;
  long long t = 0;
  for (int i = 0; i < n_images; ++i) {
    const int r = grids[2 * i], c = grids[2 * i + 1];
    if (r <= 0 || c <= 0) return -2;
    t += (long long)r * c;
  }
  return t > INT32_MAX ? -2 : t;
}

template <class F>
cudaError_t for_image_tables(const int32_t *grids, int n_images, F &&f) {
  long long base = 0;
  for (int i0 = 0; i0 < n_images; i0 += kMaxImagesPerLaunch) {
    const int n = std::min(kMaxImagesPerLaunch, n_images - i0);
    ImageTable tab;
    long long max_t = 0;
    for (int i = 0; i < n; ++i) {
      const int r = grids[2 * (i0 + i)], c = grids[2 * (i0 + i) + 1];
      tab.img[i].rows = r;
      tab.img[i].cols = c;
      tab.img[i].base = int(base);
      base += (long long)r * c;
      max_t = std::max(max_t, (long long)r * c);
    }
    const cudaError_t e = f(tab, n, max_t);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

extern "C" {

const char *vit_status_string(vit_status s) {
  switch (s) {
    case VIT_OK: return "VIT_OK";
    case VIT_ERR_INVALID_ARG: return "VIT_ERR_INVALID_ARG";
    case VIT_ERR_SHAPE: return "VIT_ERR_SHAPE";
    case VIT_ERR_UNSUPPORTED: return "VIT_ERR_UNSUPPORTED";
    case VIT_ERR_WORKSPACE: return "VIT_ERR_WORKSPACE";
    case VIT_ERR_CUDA: return "VIT_ERR_CUDA";
    case VIT_ERR_TIMEOUT: return "VIT_ERR_TIMEOUT";
    case VIT_ERR_DEVICE_BOUNDS: return "VIT_ERR_DEVICE_BOUNDS";
  }
  return "VIT_ERR_UNKNOWN";
}

// ---------------------------------------------------------------- CUDA graphs
// Stream capture of any sequence of this library's calls: the caller enqueues
// them on the stream vit_graph_begin returns; vit_graph_end instantiates the
// captured work (launches keep their programmatic-dependent-launch edges).
// Per-launch profiling events are off during the capture.

static long long total_launches(const vit_ctx *ctx) {
  long long n = 0;
  for (long long l : ctx->prof.launches) n += l;
  return n;
}

vit_status vit_graph_begin(vit_ctx *ctx, void **capture_stream) {
  if (!ctx || !capture_stream) return VIT_ERR_INVALID_ARG;
  *capture_stream = nullptr;
  if (ctx->cap_stream) return VIT_ERR_INVALID_ARG;  // one capture at a time per context
  DeviceGuard g(ctx->device);
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return VIT_ERR_CUDA;
  // relaxed: the launch paths may query or set function attributes while capturing
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return VIT_ERR_CUDA;
  }
  ctx->cap_stream = cs;
  ctx->cap_prof_on = ctx->prof.on;
  ctx->prof.on = false;
  ctx->cap_launches0 = total_launches(ctx);
  *capture_stream = cs;
  return VIT_OK;
}

vit_status vit_graph_end(vit_ctx *ctx, vit_graph **out) {
  if (!ctx || !out) return VIT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!ctx->cap_stream) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(ctx->cap_stream, &graph);
  cudaStreamDestroy(ctx->cap_stream);
  ctx->cap_stream = nullptr;
  ctx->prof.on = ctx->cap_prof_on;
  const long long kernels = total_launches(ctx) - ctx->cap_launches0;
  if (e != cudaSuccess || graph == nullptr) {
    if (graph) cudaGraphDestroy(graph);
    return VIT_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ei != cudaSuccess) return VIT_ERR_CUDA;
  vit_graph *gr = new (std::nothrow) vit_graph;
  if (!gr) {
    cudaGraphExecDestroy(exec);
    return VIT_ERR_CUDA;
  }
  gr->exec = exec;
  gr->device = ctx->device;
  gr->kernels = kernels;
  *out = gr;
  return VIT_OK;
}

vit_status vit_graph_launch(vit_graph *g, void *stream) {
  if (!g) return VIT_ERR_INVALID_ARG;
  DeviceGuard dg(g->device);
  return cuda_status(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)));
}

long long vit_graph_kernels(const vit_graph *g) { return g ? g->kernels : 0; }

void vit_graph_destroy(vit_graph *g) {
  if (!g) return;
  DeviceGuard dg(g->device);
  cudaGraphExecDestroy(g->exec);
  delete g;
}

const char *vit_version(void) { return "libvit 0.1 sm_100a"; }

vit_status vit_init(const vit_config *cfg, int device, vit_ctx **out) {
  if (!out) return VIT_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg) return VIT_ERR_INVALID_ARG;
  const vit_config &c = *cfg;
  if (c.dtype != VIT_F32 && c.dtype != VIT_BF16) return VIT_ERR_INVALID_ARG;
  if (c.hidden <= 0 || c.heads <= 0 || c.head_dim <= 0) return VIT_ERR_INVALID_ARG;
  if (c.heads * c.head_dim != c.hidden) return VIT_ERR_SHAPE;
  if (!(c.flags & VIT_FLAG_NO_MLP) && c.mlp <= 0) return VIT_ERR_INVALID_ARG;
  if (!(c.ln_eps >= 0.f) || !(c.rope_theta > 0.f)) return VIT_ERR_INVALID_ARG;
  if (c.flags & ~(VIT_FLAG_NO_ROPE | VIT_FLAG_NO_MLP)) return VIT_ERR_INVALID_ARG;
  const bool hd_ok = c.dtype == VIT_F32 ? (c.head_dim == 64 || c.head_dim == 72 || c.head_dim == 128)
                                        : (c.head_dim == 72 || c.head_dim == 128);
  if (!hd_ok) return VIT_ERR_UNSUPPORTED;
  if (c.hidden % 8 || (!(c.flags & VIT_FLAG_NO_MLP) && c.mlp % 8)) return VIT_ERR_UNSUPPORTED;
  if (c.hidden > 4096) return VIT_ERR_UNSUPPORTED;  // LayerNorm keeps a row in registers
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return VIT_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return VIT_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return VIT_ERR_UNSUPPORTED;
  DeviceGuard g(device);
  vit_ctx *ctx = new vit_ctx;
  ctx->cfg = c;
  ctx->device = device;
  ctx->num_sms = prop.multiProcessorCount;
  ctx->d_status = nullptr;
  if (cudaMalloc(&ctx->d_status, 4 * sizeof(int)) != cudaSuccess ||
      cudaMemset(ctx->d_status, 0, 4 * sizeof(int)) != cudaSuccess) {
    if (ctx->d_status) cudaFree(ctx->d_status);
    delete ctx;
    return VIT_ERR_CUDA;
  }
  const int h = c.head_dim / 2;
  memset(&ctx->fr, 0, sizeof(ctx->fr));
  for (int j = 0; j < c.head_dim / 4 && j < 32; ++j)
    ctx->fr.wpi[j] = float(pow(double(c.rope_theta), -2.0 * j / h) / M_PI);
  *out = ctx;
  return VIT_OK;
}

void vit_destroy(vit_ctx *ctx) {
  if (!ctx) return;
  {
    DeviceGuard g(ctx->device);
    ctx->prof.destroy();
    if (ctx->d_status) cudaFree(ctx->d_status);
  }
  delete ctx;
}

size_t vit_workspace_bytes(const vit_ctx *ctx, int total_tokens) {
  if (!ctx || total_tokens < 0) return 0;
  return workspace_layout(ctx->cfg, total_tokens, nullptr, nullptr, split_ctas(ctx, total_tokens));
}

vit_status vit_fold_layernorm(vit_ctx *ctx, const vit_layer_weights *in, void *w_qkv_out,
                              void *qkv_fold, void *w_fc1_out, void *fc1_fold, void *stream) {
  if (!ctx || !in) return VIT_ERR_INVALID_ARG;
  const vit_config &c = ctx->cfg;
  if (c.dtype != VIT_BF16) return VIT_ERR_UNSUPPORTED;
  const bool do_qkv = w_qkv_out || qkv_fold, do_fc1 = w_fc1_out || fc1_fold;
  if ((do_qkv && !(w_qkv_out && qkv_fold)) || (do_fc1 && !(w_fc1_out && fc1_fold)))
    return VIT_ERR_INVALID_ARG;
  if (do_fc1 && (c.flags & VIT_FLAG_NO_MLP)) return VIT_ERR_INVALID_ARG;
  const void *qkv_in[6] = {in->ln1_g, in->ln1_b, in->w_qkv, in->b_qkv, w_qkv_out, qkv_fold};
  const void *fc1_in[6] = {in->ln2_g, in->ln2_b, in->w_fc1, in->b_fc1, w_fc1_out, fc1_fold};
  for (int i = 0; i < 6; ++i) {
    if (do_qkv && (!qkv_in[i] || !aligned16(qkv_in[i]))) return VIT_ERR_INVALID_ARG;
    if (do_fc1 && (!fc1_in[i] || !aligned16(fc1_in[i]))) return VIT_ERR_INVALID_ARG;
  }
  if (!do_qkv && !do_fc1) return VIT_OK;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int C = c.hidden;
  if (do_qkv && counted(ctx, VIT_K_FOLD, st, [&] {
        return launch_fold_ln(in->w_qkv, in->ln1_g, in->ln1_b, in->b_qkv, w_qkv_out,
                              static_cast<float *>(qkv_fold), 3 * C, C, st);
      }))
    return VIT_ERR_CUDA;
  if (do_fc1 && counted(ctx, VIT_K_FOLD, st, [&] {
        return launch_fold_ln(in->w_fc1, in->ln2_g, in->ln2_b, in->b_fc1, w_fc1_out,
                              static_cast<float *>(fc1_fold), c.mlp, C, st);
      }))
    return VIT_ERR_CUDA;
  return VIT_OK;
}

vit_status vit_layer_forward(vit_ctx *ctx, const vit_layer_weights *w, const void *x, void *y,
                             const vit_seqs *seqs, void *workspace, size_t ws_bytes,
                             void *stream) {
  vit_status s = check_layer_call(ctx, x, y, seqs, workspace, ws_bytes,
                                  seqs ? split_ctas(ctx, seqs->total_tokens) : 0);
  if (s != VIT_OK) return s;
  if ((s = check_layer_weights(ctx->cfg, w)) != VIT_OK) return s;
  if (seqs->total_tokens == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  Workspace ws;
  workspace_layout(ctx->cfg, seqs->total_tokens, &ws, workspace, split_ctas(ctx, seqs->total_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the split attention's counters start at zero; each launch leaves them so
  if (ws.cnt && cudaMemsetAsync(ws.cnt, 0, size_t(split_ctas(ctx, seqs->total_tokens)) * 4, st) != cudaSuccess)
    return VIT_ERR_CUDA;
  StatsState xs;
  return layer_impl(ctx, w, x, y, seqs, ws, st, xs, false);
}

vit_status vit_encoder_forward(vit_ctx *ctx, const vit_layer_weights *layers, int n_layers,
                               const void *x, void *y, const vit_seqs *seqs, void *workspace,
                               size_t ws_bytes, void *stream) {
  vit_status s = check_layer_call(ctx, x, y, seqs, workspace, ws_bytes,
                                  seqs ? split_ctas(ctx, seqs->total_tokens) : 0);
  if (s != VIT_OK) return s;
  if (!layers || n_layers < 1) return VIT_ERR_INVALID_ARG;
  for (int i = 0; i < n_layers; ++i)
    if ((s = check_layer_weights(ctx->cfg, &layers[i])) != VIT_OK) return s;
  if (seqs->total_tokens == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  Workspace ws;
  workspace_layout(ctx->cfg, seqs->total_tokens, &ws, workspace, split_ctas(ctx, seqs->total_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the split attention's counters start at zero; each launch leaves them so
  if (ws.cnt && cudaMemsetAsync(ws.cnt, 0, size_t(split_ctas(ctx, seqs->total_tokens)) * 4, st) != cudaSuccess)
    return VIT_ERR_CUDA;
  StatsState xs;  // slice statistics of each layer's input, when a folded LN reads them
  for (int i = 0; i < n_layers; ++i) {
    const void *in = i == 0 ? x : ws.act[(i - 1) & 1];
    void *out = i == n_layers - 1 ? y : ws.act[i & 1];
    const bool next_folds = i + 1 < n_layers && layers[i + 1].qkv_fold != nullptr;
    if ((s = layer_impl(ctx, &layers[i], in, out, seqs, ws, st, xs, next_folds)) != VIT_OK)
      return s;
  }
  return VIT_OK;
}

vit_status vit_attention(vit_ctx *ctx, const void *qkv, void *o, const vit_seqs *seqs,
                         float scale, void *stream) {
  if (!ctx) return VIT_ERR_INVALID_ARG;
  vit_status s = check_seqs(ctx, seqs, true);
  if (s != VIT_OK) return s;
  if (seqs->total_tokens == 0) return VIT_OK;  // nothing is read or written
  if (!qkv || !o) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype == VIT_BF16 && (!aligned16(qkv) || !aligned16(o))) return VIT_ERR_INVALID_ARG;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf(float(ctx->cfg.head_dim));
  DeviceGuard g(ctx->device);
  const SeqArgs sa = to_seq_args(seqs, true);
  return cuda_status(run_attention(ctx, qkv, o, sa, scale, static_cast<cudaStream_t>(stream)));
}

vit_status vit_layernorm(vit_ctx *ctx, const void *x, void *y, const void *gamma,
                         const void *beta, int rows, int cols, float eps, void *stream) {
  if (!ctx || !x || !y || !gamma || !beta || rows < 0 || cols <= 0 || !(eps >= 0.f))
    return VIT_ERR_INVALID_ARG;
  if (cols % 4 || cols > 16384) return VIT_ERR_UNSUPPORTED;
  const size_t a = esize(ctx->cfg) * 4;
  const void *ps[4] = {x, y, gamma, beta};
  for (const void *p : ps)
    if (reinterpret_cast<uintptr_t>(p) % a) return VIT_ERR_INVALID_ARG;
  if (rows == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(counted(ctx, VIT_K_LAYERNORM, st, [&] {
    return launch_layernorm(ctx->cfg.dtype == VIT_F32 ? kF32 : kBF16, x, y, gamma, beta, rows,
                            cols, eps, st);
  }));
}

vit_status vit_linear(vit_ctx *ctx, const void *x, const void *w, const void *bias,
                      const void *residual, void *y, int M, int N, int K, vit_epilogue epi,
                      void *stream) {
  if (!ctx || !x || !w || !y || M < 0 || N <= 0 || K <= 0) return VIT_ERR_INVALID_ARG;
  if (epi != VIT_EPI_BIAS && epi != VIT_EPI_BIAS_GELU && epi != VIT_EPI_BIAS_RESIDUAL)
    return VIT_ERR_INVALID_ARG;
  if (epi == VIT_EPI_BIAS_RESIDUAL && !residual) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype == VIT_BF16) {
    if (K % 8 || N % 8) return VIT_ERR_UNSUPPORTED;
    const void *ps[5] = {x, w, bias, residual, y};
    for (const void *p : ps)
      if (p && !aligned16(p)) return VIT_ERR_INVALID_ARG;
  }
  if (M == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  return cuda_status(run_linear(ctx, VIT_K_GEMM, x, w,
                                epi_args(bias, epi == VIT_EPI_BIAS_RESIDUAL ? residual : nullptr, y),
                                M, N, K, int(epi), static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- projector
size_t vit_projector_workspace_bytes(const vit_ctx *ctx, int M, int d_in, int d_hidden) {
  if (!ctx || M < 0 || d_in <= 0 || d_hidden <= 0) return 0;
  const size_t e = esize(ctx->cfg);
  return align256(size_t(M) * d_in * e) + align256(size_t(M) * d_hidden * e);
}

vit_status vit_projector(vit_ctx *ctx, const vit_projector_weights *w, const void *x, void *y,
                         int M, int d_in, int d_hidden, int d_out, void *workspace,
                         size_t ws_bytes, void *stream) {
  if (!ctx || !w || !x || !y || M < 0 || d_in <= 0 || d_hidden <= 0 || d_out <= 0)
    return VIT_ERR_INVALID_ARG;
  const void *need[6] = {w->ln_g, w->ln_b, w->w1, w->b1, w->w2, w->b2};
  const bool bf16 = ctx->cfg.dtype == VIT_BF16;
  const size_t al = bf16 ? 16 : esize(ctx->cfg) * 4;
  for (const void *p : need)
    if (!p || reinterpret_cast<uintptr_t>(p) % al) return VIT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % al || reinterpret_cast<uintptr_t>(y) % al || x == y)
    return VIT_ERR_INVALID_ARG;
  if (d_in % 4 || d_in > 16384) return VIT_ERR_UNSUPPORTED;
  if (bf16 && (d_in % 8 || d_hidden % 8 || d_out % 8)) return VIT_ERR_UNSUPPORTED;
  if (M == 0) return VIT_OK;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      ws_bytes < vit_projector_workspace_bytes(ctx, M, d_in, d_hidden))
    return VIT_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dt = bf16 ? kBF16 : kF32;
  char *h = static_cast<char *>(workspace);
  char *hid = h + align256(size_t(M) * d_in * esize(ctx->cfg));
  if (counted(ctx, VIT_K_LAYERNORM, st, [&] {
        return launch_layernorm(dt, x, h, w->ln_g, w->ln_b, M, d_in, ctx->cfg.ln_eps, st);
      }))
    return VIT_ERR_CUDA;
  if (run_linear(ctx, VIT_K_GEMM, h, w->w1, epi_args(w->b1, nullptr, hid), M, d_hidden, d_in,
                 kEpiGelu, st))
    return VIT_ERR_CUDA;
  return cuda_status(run_linear(ctx, VIT_K_GEMM, hid, w->w2, epi_args(w->b2, nullptr, y), M,
                                d_out, d_hidden, kEpiBias, st));
}

// ---------------------------------------------------------------- embedding
size_t vit_embed_workspace_bytes(const vit_ctx *ctx, int total_tokens, int patch) {
  if (!ctx || total_tokens < 0 || patch < 1 || patch > 32) return 0;
  const size_t e = esize(ctx->cfg), kp = size_t(embed_kp(patch)), C = size_t(ctx->cfg.hidden);
  return align256(size_t(total_tokens) * kp * e) + align256(C * kp * e) +
         align256(size_t(total_tokens) * C * e);
}

vit_status vit_pos_interp(vit_ctx *ctx, const void *pos_table, int table_h, int table_w,
                          const int32_t *grids_hw_host, int n_images, void *y, void *stream) {
  if (!ctx || !pos_table || !y || table_h < 1 || table_w < 1) return VIT_ERR_INVALID_ARG;
  const long long T = embed_tokens(grids_hw_host, n_images);
  if (T == -1) return VIT_ERR_INVALID_ARG;
  if (T < 0) return VIT_ERR_SHAPE;
  const int C = ctx->cfg.hidden;
  if (C % 8) return VIT_ERR_UNSUPPORTED;
  if (!aligned16(pos_table) || !aligned16(y)) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dt = ctx->cfg.dtype == VIT_F32 ? kF32 : kBF16;
  return cuda_status(for_image_tables(grids_hw_host, n_images, [&](const ImageTable &tab, int n,
                                                                  long long max_t) {
    return counted(ctx, VIT_K_EMBED, st, [&] {
      return launch_pos_interp(dt, tab, n, max_t, pos_table, table_h, table_w, C, y, st);
    });
  }));
}

// The embedding with a weight already in the GEMM's [C, Kp] layout: one
// launch for both GEMM operands (patch rows and resized position rows), then
// the GEMM, whose residual epilogue adds the bias and the position rows.
static vit_status patch_embed_impl(vit_ctx *ctx, const void *pixels, const int32_t *grids_hw_host,
                                   int n_images, int patch, const void *w_pad, const void *b_pe,
                                   const void *pos_table, int table_h, int table_w, void *y,
                                   void *workspace, size_t ws_bytes, bool pad_from,
                                   const void *w_pe, void *stream) {
  if (!ctx || !pixels || !w_pe || !b_pe || !pos_table || !y || !workspace || table_h < 1 ||
      table_w < 1 || patch < 1 || patch > 32)
    return VIT_ERR_INVALID_ARG;
  const long long T = embed_tokens(grids_hw_host, n_images);
  if (T == -1) return VIT_ERR_INVALID_ARG;
  if (T < 0) return VIT_ERR_SHAPE;
  const int C = ctx->cfg.hidden;
  if (C % 8) return VIT_ERR_UNSUPPORTED;
  if (ws_bytes < vit_embed_workspace_bytes(ctx, int(T), patch)) return VIT_ERR_WORKSPACE;
  {
    const void *ps[4] = {b_pe, pos_table, y, workspace};
    for (const void *q : ps)
      if (!aligned16(q)) return VIT_ERR_INVALID_ARG;
    if (!pad_from && !aligned16(w_pad)) return VIT_ERR_INVALID_ARG;
  }
  const size_t e = esize(ctx->cfg);
  const int k = 3 * patch * patch, kp = embed_kp(patch);
  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  void *patches = wsb;
  void *w_ws = wsb + align256(size_t(T) * kp * e);
  void *pos = static_cast<uint8_t *>(w_ws) + align256(size_t(C) * kp * e);
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dt = ctx->cfg.dtype == VIT_F32 ? kF32 : kBF16;
  cudaError_t err = for_image_tables(grids_hw_host, n_images, [&](const ImageTable &tab, int n,
                                                                 long long max_t) {
    return counted(ctx, VIT_K_EMBED, st, [&] {
      return launch_embed_inputs(dt, tab, n, max_t, pixels, patches, patch, kp, pos_table, table_h,
                                 table_w, C, pos, st);
    });
  });
  if (err != cudaSuccess) return VIT_ERR_CUDA;
  if (pad_from) {
    if (counted(ctx, VIT_K_EMBED, st, [&] { return launch_pad_cols(dt, w_pe, w_ws, C, k, kp, st); }))
      return VIT_ERR_CUDA;
    w_pad = w_ws;
  }
  // tokens = patches . w_pad^T + b_pe + interpolated table (residual epilogue)
  return cuda_status(run_linear(ctx, VIT_K_GEMM, patches, w_pad, epi_args(b_pe, pos, y), int(T), C,
                                kp, kEpiResidual, st));
}

vit_status vit_patch_embed(vit_ctx *ctx, const void *pixels, const int32_t *grids_hw_host,
                           int n_images, int patch, const void *w_pe, const void *b_pe,
                           const void *pos_table, int table_h, int table_w, void *y,
                           void *workspace, size_t ws_bytes, void *stream) {
  return patch_embed_impl(ctx, pixels, grids_hw_host, n_images, patch, nullptr, b_pe, pos_table,
                          table_h, table_w, y, workspace, ws_bytes, true, w_pe, stream);
}

vit_status vit_patch_embed_padded(vit_ctx *ctx, const void *pixels, const int32_t *grids_hw_host,
                                  int n_images, int patch, const void *w_pad, const void *b_pe,
                                  const void *pos_table, int table_h, int table_w, void *y,
                                  void *workspace, size_t ws_bytes, void *stream) {
  return patch_embed_impl(ctx, pixels, grids_hw_host, n_images, patch, w_pad, b_pe, pos_table,
                          table_h, table_w, y, workspace, ws_bytes, false, w_pad, stream);
}

int vit_patch_kp(int patch) { return patch < 1 || patch > 32 ? 0 : embed_kp(patch); }

vit_status vit_pad_patch_weight(vit_ctx *ctx, const void *w_pe, int patch, void *w_pad,
                                void *stream) {
  if (!ctx || !w_pe || !w_pad || patch < 1 || patch > 32) return VIT_ERR_INVALID_ARG;
  if (!aligned16(w_pad)) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int dt = ctx->cfg.dtype == VIT_F32 ? kF32 : kBF16;
  return cuda_status(counted(ctx, VIT_K_EMBED, st, [&] {
    return launch_pad_cols(dt, w_pe, w_pad, ctx->cfg.hidden, 3 * patch * patch, embed_kp(patch), st);
  }));
}

// ---------------------------------------------------------------- MXFP8
size_t vit_mx8_row_bytes(int K) { return K < 0 ? 0 : mx8_row_bytes(K); }
size_t vit_mx8_scale_bytes(int rows, int K) {
  return rows < 0 || K < 0 ? 0 : mx8_scale_bytes(rows, K);
}

vit_status vit_mx8_quantize(vit_ctx *ctx, const void *x, int rows, int K, void *codes,
                            void *scales, void *stream) {
  if (!ctx || !x || !codes || !scales || rows < 0 || K < 0) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype != VIT_BF16) return VIT_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return VIT_ERR_INVALID_ARG;
  if (rows == 0 || K == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(counted(ctx, VIT_K_MX8_QUANTIZE, st, [&] {
    return launch_mx8_quantize(x, rows, K, static_cast<uint8_t *>(codes),
                               static_cast<uint8_t *>(scales), st);
  }));
}

vit_status vit_layernorm_mx8(vit_ctx *ctx, const void *x, const void *gamma, const void *beta,
                             int rows, int cols, float eps, void *codes, void *scales,
                             void *stream) {
  if (!ctx || !x || !gamma || !beta || !codes || !scales || rows < 0 || cols < 0)
    return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype != VIT_BF16 || cols % 4 || cols > 1536) return VIT_ERR_UNSUPPORTED;
  const void *ps[5] = {x, gamma, beta, codes, scales};
  for (const void *q : ps)
    if (!aligned16(q)) return VIT_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(counted(ctx, VIT_K_LAYERNORM, st, [&] {
    return launch_layernorm_mx8(x, gamma, beta, rows, cols, eps, static_cast<uint8_t *>(codes),
                                static_cast<uint8_t *>(scales), st);
  }));
}

vit_status vit_linear_mx8(vit_ctx *ctx, const void *a_codes, const void *a_scales,
                          const void *w_codes, const void *w_scales, const void *bias,
                          const void *residual, void *y, int M, int N, int K, vit_epilogue epi,
                          void *stream) {
  if (!ctx || !a_codes || !a_scales || !w_codes || !w_scales || !y || M < 0 || N <= 0 || K <= 0)
    return VIT_ERR_INVALID_ARG;
  if (epi != VIT_EPI_BIAS && epi != VIT_EPI_BIAS_GELU && epi != VIT_EPI_BIAS_RESIDUAL)
    return VIT_ERR_INVALID_ARG;
  if (epi == VIT_EPI_BIAS_RESIDUAL && !residual) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype != VIT_BF16) return VIT_ERR_UNSUPPORTED;
  if (N % 8) return VIT_ERR_UNSUPPORTED;
  const void *ps[7] = {a_codes, a_scales, w_codes, w_scales, bias, residual, y};
  for (const void *p : ps)
    if (p && !aligned16(p)) return VIT_ERR_INVALID_ARG;
  if (M == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(counted(ctx, VIT_K_GEMM_MX8, st, [&] {
    return launch_gemm_mx8(static_cast<const uint8_t *>(a_codes),
                           static_cast<const uint8_t *>(a_scales),
                           static_cast<const uint8_t *>(w_codes),
                           static_cast<const uint8_t *>(w_scales), bias,
                           epi == VIT_EPI_BIAS_RESIDUAL ? residual : nullptr, y, M, N, K, int(epi),
                           ctx->num_sms, ctx->d_status, st);
  }));
}

// ---------------------------------------------------------------- FP8 layers
namespace {

// the bf16 layer's workspace, then two quantised activations: the inputs of
// the QKV, out and fc1 projections (K = hidden), and fc1's output, written
// quantised by its epilogue as fc2's input (K = MLP width)
size_t mx8_act_bytes(int T, int K) {
  return align256(size_t(T) * mx8_row_bytes(K)) + align256(mx8_scale_bytes(T, K));
}
size_t mx8_extra(const vit_config &c, int T) {
  return mx8_act_bytes(T, c.hidden) +
         ((c.flags & VIT_FLAG_NO_MLP) ? size_t(0) : mx8_act_bytes(T, c.mlp));
}

vit_status check_layer_weights_mx8(const vit_config &c, const vit_layer_weights_mx8 *w) {
  if (!w) return VIT_ERR_INVALID_ARG;
  const void *need[8] = {w->ln1_g, w->ln1_b, w->b_qkv, w->b_o,
                         w->w_qkv_codes, w->w_qkv_scales, w->w_o_codes, w->w_o_scales};
  for (const void *p : need)
    if (!p || !aligned16(p)) return VIT_ERR_INVALID_ARG;
  if (!(c.flags & VIT_FLAG_NO_MLP)) {
    const void *mlp[8] = {w->ln2_g, w->ln2_b, w->b_fc1, w->b_fc2,
                          w->w_fc1_codes, w->w_fc1_scales, w->w_fc2_codes, w->w_fc2_scales};
    for (const void *p : mlp)
      if (!p || !aligned16(p)) return VIT_ERR_INVALID_ARG;
  }
  return VIT_OK;
}

// One FP8 layer (all arguments validated).  aq / asc: quantised activation.
vit_status layer_mx8_impl(vit_ctx *ctx, const vit_layer_weights_mx8 *w, const void *x, void *y,
                          const vit_seqs *seqs, const Workspace &ws, uint8_t *aq, uint8_t *asc,
                          uint8_t *gq, uint8_t *gsc, cudaStream_t st) {
  const vit_config &c = ctx->cfg;
  const int T = seqs->total_tokens, C = c.hidden, F = c.mlp;
  const bool rope = !(c.flags & VIT_FLAG_NO_ROPE) && seqs->pos_rc != nullptr;
  const bool no_mlp = (c.flags & VIT_FLAG_NO_MLP) != 0;
  const float scale = 1.0f / sqrtf(float(c.head_dim));
  auto quant = [&](const void *a, int K) {
    return counted(ctx, VIT_K_MX8_QUANTIZE, st,
                   [&] { return launch_mx8_quantize(a, T, K, aq, asc, st); });
  };
  // LayerNorm straight to MXFP8 (one launch) where the row fits a warp's
  // registers, else LayerNorm then the quantiser
  auto ln_q = [&](const void *in, const void *g, const void *b) {
    if (C <= 1536)
      return counted(ctx, VIT_K_LAYERNORM, st, [&] {
        return launch_layernorm_mx8(in, g, b, T, C, c.ln_eps, aq, asc, st);
      });
    cudaError_t e = counted(ctx, VIT_K_LAYERNORM, st, [&] {
      return launch_layernorm(kBF16, in, ws.h, g, b, T, C, c.ln_eps, st);
    });
    return e != cudaSuccess ? e : quant(ws.h, C);
  };
  auto gemm = [&](int kind, const uint8_t *a, const uint8_t *asf, const void *wc, const void *wsc,
                  const void *b, const void *res, void *out, int N, int K, int epi,
                  uint8_t *out_sc = nullptr) {
    return counted(ctx, kind, st, [&] {
      return launch_gemm_mx8(a, asf, static_cast<const uint8_t *>(wc),
                             static_cast<const uint8_t *>(wsc), b, res, out, T, N, K, epi,
                             ctx->num_sms, ctx->d_status, st, out_sc);
    });
  };
  if (ln_q(x, w->ln1_g, w->ln1_b) ||
      gemm(VIT_K_GEMM_QKV, aq, asc, w->w_qkv_codes, w->w_qkv_scales, w->b_qkv, nullptr, ws.qkv,
           3 * C, C, kEpiBias))
    return VIT_ERR_CUDA;
  if (rope && counted(ctx, VIT_K_ROPE, st, [&] {
        return launch_rope2d(kBF16, ws.qkv, seqs->pos_rc, T, c.heads, c.head_dim, ctx->fr, st);
      }))
    return VIT_ERR_CUDA;
  const SeqArgs sa = to_seq_args(seqs, false);
  if (run_attention(ctx, ws.qkv, ws.attn, sa, scale, st)) return VIT_ERR_CUDA;
  if (quant(ws.attn, C) || gemm(VIT_K_GEMM_OUT, aq, asc, w->w_o_codes, w->w_o_scales, w->b_o, x,
                                no_mlp ? y : ws.x1, C, C, kEpiResidual))
    return VIT_ERR_CUDA;
  if (no_mlp) return VIT_OK;
  // fc1's epilogue writes GELU(.) as MXFP8 codes and scales: fc2's input
  if (ln_q(ws.x1, w->ln2_g, w->ln2_b) ||
      gemm(VIT_K_GEMM_FC1, aq, asc, w->w_fc1_codes, w->w_fc1_scales, w->b_fc1, nullptr, gq, F, C,
           kEpiGelu | kEpiQuant, gsc) ||
      gemm(VIT_K_GEMM_FC2, gq, gsc, w->w_fc2_codes, w->w_fc2_scales, w->b_fc2, ws.x1, y, C, F,
           kEpiResidual))
    return VIT_ERR_CUDA;
  return VIT_OK;
}

}  // namespace

size_t vit_workspace_bytes_mx8(const vit_ctx *ctx, int total_tokens) {
  if (!ctx || total_tokens < 0 || ctx->cfg.dtype != VIT_BF16) return 0;
  return workspace_layout(ctx->cfg, total_tokens, nullptr, nullptr, 0) +
         mx8_extra(ctx->cfg, total_tokens);
}

vit_status vit_encoder_forward_mx8(vit_ctx *ctx, const vit_layer_weights_mx8 *layers,
                                   int n_layers, const void *x, void *y, const vit_seqs *seqs,
                                   void *workspace, size_t ws_bytes, void *stream) {
  if (!ctx) return VIT_ERR_INVALID_ARG;
  if (ctx->cfg.dtype != VIT_BF16) return VIT_ERR_UNSUPPORTED;
  vit_status s = check_layer_call(ctx, x, y, seqs, workspace, ws_bytes, 0);
  if (s != VIT_OK) return s;
  if (seqs->prefix_kv) return VIT_ERR_UNSUPPORTED;
  if (!layers || n_layers < 1) return VIT_ERR_INVALID_ARG;
  for (int i = 0; i < n_layers; ++i)
    if ((s = check_layer_weights_mx8(ctx->cfg, &layers[i])) != VIT_OK) return s;
  const int T = seqs->total_tokens;
  if (T == 0) return VIT_OK;
  if (ws_bytes < vit_workspace_bytes_mx8(ctx, T)) return VIT_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  Workspace ws;
  const size_t base = workspace_layout(ctx->cfg, T, &ws, workspace, 0);
  const int C = ctx->cfg.hidden, F = ctx->cfg.mlp;
  uint8_t *aq = static_cast<uint8_t *>(workspace) + base;
  uint8_t *asc = aq + align256(size_t(T) * mx8_row_bytes(C));
  uint8_t *gq = aq + mx8_act_bytes(T, C);  // used only with the MLP
  uint8_t *gsc = gq + align256(size_t(T) * mx8_row_bytes(F));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < n_layers; ++i) {
    const void *in = i == 0 ? x : ws.act[(i - 1) & 1];
    void *out = i == n_layers - 1 ? y : ws.act[i & 1];
    if ((s = layer_mx8_impl(ctx, &layers[i], in, out, seqs, ws, aq, asc, gq, gsc, st)) != VIT_OK)
      return s;
  }
  return VIT_OK;
}

vit_status vit_rope2d(vit_ctx *ctx, void *qkv, const int32_t *pos_rc, int total_tokens,
                      void *stream) {
  if (!ctx || !qkv || !pos_rc || total_tokens < 0) return VIT_ERR_INVALID_ARG;
  if (total_tokens == 0) return VIT_OK;
  DeviceGuard g(ctx->device);
  const vit_config &c = ctx->cfg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(counted(ctx, VIT_K_ROPE, st, [&] {
    return launch_rope2d(c.dtype == VIT_F32 ? kF32 : kBF16, qkv, pos_rc, total_tokens, c.heads,
                         c.head_dim, ctx->fr, st);
  }));
}

vit_status vit_spatial_merge_2x2(vit_ctx *ctx, const void *x, void *y,
                                 const int32_t *grids_hw_host, int n_images, int channels,
                                 void *stream) {
  if (!ctx || !x || !y || !grids_hw_host || n_images < 0 || channels <= 0)
    return VIT_ERR_INVALID_ARG;
  long long total = 0;
  for (int i = 0; i < n_images; ++i) {
    const int r = grids_hw_host[2 * i], c = grids_hw_host[2 * i + 1];
    if (r <= 0 || c <= 0) return VIT_ERR_SHAPE;
    if (r % 2 || c % 2) return VIT_ERR_SHAPE;
    total += (long long)r * c;
  }
  if (total > INT32_MAX) return VIT_ERR_SHAPE;
  const size_t row_bytes = size_t(channels) * esize(ctx->cfg);
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  long long base = 0;
  for (int i0 = 0; i0 < n_images; i0 += kMaxImagesPerLaunch) {
    const int n = std::min(kMaxImagesPerLaunch, n_images - i0);
    ImageTable tab;
    long long max_out = 0;
    for (int i = 0; i < n; ++i) {
      const int r = grids_hw_host[2 * (i0 + i)], c = grids_hw_host[2 * (i0 + i) + 1];
      tab.img[i].rows = r;
      tab.img[i].cols = c;
      tab.img[i].base = int(base);
      base += (long long)r * c;
      max_out = std::max(max_out, (long long)(r / 2) * (c / 2));
    }
    if (counted(ctx, VIT_K_MERGE, st,
                [&] { return launch_merge2x2(tab, n, x, y, row_bytes, max_out, st); }))
      return VIT_ERR_CUDA;
  }
  return VIT_OK;
}

vit_status vit_positions_from_grids(vit_ctx *ctx, const int32_t *grids_hw_host, int n_images,
                                    int32_t *cu_seqlens, int32_t *pos_rc, void *stream) {
  if (!ctx || !grids_hw_host || !cu_seqlens || !pos_rc || n_images < 1 || n_images > 1024)
    return VIT_ERR_INVALID_ARG;
  long long total = 0;
  for (int i = 0; i < n_images; ++i) {
    const int r = grids_hw_host[2 * i], c = grids_hw_host[2 * i + 1];
    if (r <= 0 || c <= 0) return VIT_ERR_SHAPE;
    total += (long long)r * c;
  }
  if (total > INT32_MAX) return VIT_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(pos_rc) & 7u) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  long long base = 0;
  for (int i0 = 0; i0 < n_images; i0 += kMaxImagesPerLaunch) {
    const int n = std::min(kMaxImagesPerLaunch, n_images - i0);
    ImageTable tab;
    int max_tok = 0;
    for (int i = 0; i < n; ++i) {
      const int r = grids_hw_host[2 * (i0 + i)], c = grids_hw_host[2 * (i0 + i) + 1];
      tab.img[i].rows = r;
      tab.img[i].cols = c;
      tab.img[i].base = int(base);
      base += (long long)r * c;
      max_tok = std::max(max_tok, r * c);
    }
    if (counted(ctx, VIT_K_POSITIONS, st, [&] {
          return launch_positions(tab, n, i0, max_tok, cu_seqlens, pos_rc, st);
        }))
      return VIT_ERR_CUDA;
  }
  return VIT_OK;
}

vit_status vit_profile_enable(vit_ctx *ctx, int enable) {
  if (!ctx) return VIT_ERR_INVALID_ARG;
  ctx->prof.on = enable != 0;
  return VIT_OK;
}

vit_status vit_profile_read(vit_ctx *ctx, int kind, long long *launches, double *total_ms,
                            int reset) {
  if (!ctx || kind < 0 || kind >= VIT_K_COUNT) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  double ms = 0.0;
  for (auto &r : ctx->prof.recs) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return VIT_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return VIT_ERR_CUDA;
    ms += t;
  }
  if (launches) *launches = ctx->prof.launches[kind];
  if (total_ms) *total_ms = ms;
  if (reset) ctx->prof.clear();
  return VIT_OK;
}

vit_status vit_debug_lost_tx(vit_ctx *ctx, unsigned bytes) {
  if (!ctx || bytes > 65536u) return VIT_ERR_INVALID_ARG;  // keeps the tx count in range
  ctx->debug_lost_tx = bytes;
  return VIT_OK;
}

vit_status vit_get_last_device_status(vit_ctx *ctx) {
  if (!ctx) return VIT_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return VIT_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};
  if (cudaMemcpy(h, ctx->d_status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return VIT_ERR_CUDA;
  if (cudaMemset(ctx->d_status, 0, sizeof(h)) != cudaSuccess) return VIT_ERR_CUDA;
  if (h[0] == kDevTimeout) return VIT_ERR_TIMEOUT;
  if (h[0] == kDevBounds) return VIT_ERR_DEVICE_BOUNDS;
  return VIT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation layer call
// vit_layer_forward_noalloc: the same layer as vit_layer_forward, with its
// scratch (the intermediate activations) in a fixed array compiled into the
// library instead of a caller-provided workspace.
#include <map>
#include <mutex>

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB, per device

// Device-side scratch of the no-allocation call.  Its name in host code is a
// host stand-in, not a device address: host code only ever passes the
// address returned by cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_layer_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
std::map<int, void *> g_scratch_addr;  // device ordinal -> device address of g_layer_scratch

// Resolves the scratch's device address on the current device (the caller
// made ctx->device current), once per device.
vit_status static_scratch(int device, void **out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  auto it = g_scratch_addr.find(device);
  if (it != g_scratch_addr.end()) {
    *out = it->second;
    return VIT_OK;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_layer_scratch) != cudaSuccess || p == nullptr)
    return VIT_ERR_CUDA;
  g_scratch_addr[device] = p;
  *out = p;
  return VIT_OK;
}

}  // namespace

extern "C" vit_status vit_layer_forward_noalloc(vit_ctx *ctx, const vit_layer_weights *w,
                                                const void *x, void *y, const vit_seqs *seqs,
                                                void *stream) {
  if (!ctx || !seqs) return VIT_ERR_INVALID_ARG;
  if (seqs->total_tokens < 0) return VIT_ERR_INVALID_ARG;
  // size check first, against the fixed scratch, before any device work
  if (workspace_layout(ctx->cfg, seqs->total_tokens, nullptr, nullptr, 0) > kStaticScratchBytes)
    return VIT_ERR_WORKSPACE;
  DeviceGuard g(ctx->device);
  void *scratch = nullptr;
  vit_status s = static_scratch(ctx->device, &scratch);
  if (s != VIT_OK) return s;
  // the layout below holds no split-attention scratch (part and cnt stay
  // null, so attention takes the whole-item schedule): size it the same way
  if ((s = check_layer_call(ctx, x, y, seqs, scratch, kStaticScratchBytes, 0)) != VIT_OK) return s;
  if ((s = check_layer_weights(ctx->cfg, w)) != VIT_OK) return s;
  if (seqs->total_tokens == 0) return VIT_OK;
  Workspace ws;
  workspace_layout(ctx->cfg, seqs->total_tokens, &ws, scratch, 0);
  // launch counts only: no timing events are created during this call
  const bool prof_on = ctx->prof.on;
  ctx->prof.on = false;
  StatsState xs;
  s = layer_impl(ctx, w, x, y, seqs, ws, static_cast<cudaStream_t>(stream), xs, false);
  ctx->prof.on = prof_on;
  return s;
}
