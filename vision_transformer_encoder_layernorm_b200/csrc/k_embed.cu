// k_embed.cu -- the steps before the encoder: patch extraction for the patch
// embedding GEMM, and the bilinear interpolation of the position table.
//
// KLiteInfer README, section "精度与性能" (patch embedding is the first of
// the compared stages) and section "架构", paragraph "视觉算子" (bilinear
// position-embedding interpolation).  Image i is [3, rows*p, cols*p],
// channels first, packed after image i-1; its tokens are its patches in
// row-major order, token t of the packed sequence starting at base(i).  A
// token's patch is flattened in (channel, y, x) order, as a Conv2d weight
// [C, 3, p, p] is, so the embedding is one GEMM against the weight viewed as
// [C, 3*p*p].  The table [gh, gw, C] is resized to (rows, cols) with
// half-pixel centres (PyTorch's bilinear default, align_corners = false).
#include "kernels.h"

namespace vit {

// Tokens per block of the operand kernel below.
constexpr int kTokPerBlock = 4;

// w [N, K] -> w_pad [N, Kp], zero columns K..Kp-1; block per row
template <typename T>
__global__ void __launch_bounds__(256) pad_cols_kernel(const T *__restrict__ w, T *__restrict__ out,
                                                        int k, int kp) {
  pdl_trigger();
  pdl_wait();
  const T *src = w + (long long)blockIdx.x * k;
  T *dst = out + (long long)blockIdx.x * kp;
  for (int col = threadIdx.x; col < kp; col += blockDim.x)
    dst[col] = col < k ? src[col] : from_f32<T>(0.0f);
}

// ---------------------------------------------------------------- position table
// Source index of output i of n along an axis of g table entries, with
// half-pixel centres: s = (i + 1/2) g / n - 1/2 = ((2i + 1) g - n) / (2n),
// clamped below at 0.  Integer floor, so the neighbours are exact.
__device__ __forceinline__ void bilinear_axis(int i, int n, int g, int &i0, int &i1, float &w1) {
  const long long num = (2LL * i + 1) * g - n, den = 2LL * n;
  if (num <= 0) {
    i0 = 0;
    w1 = 0.0f;
  } else {
    i0 = int(num / den);
    w1 = float(num - den * i0) / float(den);
  }
  i1 = min(i0 + 1, g - 1);
}

template <typename T>
struct Vec8;  // eight elements, one or two aligned 16-byte loads
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *q, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4 *>(q);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16_lo(w[i]);
      f[2 * i + 1] = bf16_hi(w[i]);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *q, const float (&f)[8]) {
    *reinterpret_cast<uint4 *>(q) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                               pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float *q, float (&f)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(q), b = *reinterpret_cast<const float4 *>(q + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  static __device__ __forceinline__ void store(float *q, const float (&f)[8]) {
    *reinterpret_cast<float4 *>(q) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4 *>(q + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
};

// y[base(i) + r*cols + c, :] = bilinear(table)[r, c, :]; block (token, image),
// one thread per 8 channels (C % 8 == 0), fp32 arithmetic.
template <typename T>
__global__ void __launch_bounds__(128) pos_interp_kernel(const __grid_constant__ ImageTable tab,
                                                          const T *__restrict__ table, int gh,
                                                          int gw, int C, T *__restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const ImageEntry im = tab.img[blockIdx.y];
  const int tok = blockIdx.x;
  if (tok >= im.rows * im.cols) return;
  const int r = tok / im.cols, c = tok - r * im.cols;
  int y0, y1, x0, x1;
  float wy, wx;
  bilinear_axis(r, im.rows, gh, y0, y1, wy);
  bilinear_axis(c, im.cols, gw, x0, x1, wx);
  const T *t00 = table + ((long long)y0 * gw + x0) * C, *t01 = table + ((long long)y0 * gw + x1) * C;
  const T *t10 = table + ((long long)y1 * gw + x0) * C, *t11 = table + ((long long)y1 * gw + x1) * C;
  T *out = y + (long long)(im.base + tok) * C;
  for (int ch = threadIdx.x * 8; ch < C; ch += blockDim.x * 8) {
    float a[8], b[8], d[8], f[8], o[8];
    Vec8<T>::load(t00 + ch, a);
    Vec8<T>::load(t01 + ch, b);
    Vec8<T>::load(t10 + ch, d);
    Vec8<T>::load(t11 + ch, f);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float top = (1.0f - wx) * a[u] + wx * b[u];
      const float bot = (1.0f - wx) * d[u] + wx * f[u];
      o[u] = (1.0f - wy) * top + wy * bot;
    }
    Vec8<T>::store(out + ch, o);
  }
}

// ---------------------------------------------------------------- both inputs of the GEMM
// One launch for the embedding GEMM's operands: block (x, image) covers
// kTokPerBlock tokens of the image and writes their patch rows (patches
// [T, Kp], zero padded) and their resized position rows (pos [T, C]).  A
// patch row is 3p runs of p pixels (one per channel and pixel row); with
// bf16 pixels and an even p a run moves as p/2 four-byte words (a run starts
// at an even element of an image row, and at an even element of the patch
// row, and the pixels start at a four-byte boundary: `words`), otherwise
// element by element.  Position rows as pos_interp_kernel:
// 16-byte table loads, fp32 blend.
template <typename T>
__global__ void __launch_bounds__(256) embed_inputs_kernel(const __grid_constant__ ImageTable tab,
                                                            const T *__restrict__ px,
                                                            T *__restrict__ patches, int p, int kp,
                                                            int words, const T *__restrict__ table,
                                                            int gh, int gw, int C,
                                                            T *__restrict__ pos) {
  pdl_trigger();
  pdl_wait();
  const ImageEntry im = tab.img[blockIdx.y];
  const int n_tok = im.rows * im.cols;
  const int tok0 = blockIdx.x * kTokPerBlock;
  if (tok0 >= n_tok) return;
  const int nt = min(kTokPerBlock, n_tok - tok0);
  const int pp = p * p, k3 = 3 * pp;
  const int W = im.cols * p, Hh = im.rows * p;
  const T *img = px + (long long)im.base * k3;
  // patch rows: work unit = (token, run); then the padding columns
  const int runs = 3 * p;
  for (int u = threadIdx.x; u < nt * runs; u += blockDim.x) {
    const int tt = u / runs, run = u - tt * runs;
    const int tok = tok0 + tt;
    const int r = tok / im.cols, c = tok - r * im.cols;
    const int ch = run / p, y = run - ch * p;
    const T *src = img + ((long long)ch * Hh + (long long)r * p + y) * W + (long long)c * p;
    T *dst = patches + (long long)(im.base + tok) * kp + ch * pp + y * p;
    if (words) {  // all of the run's loads in flight before its stores (p <= 32)
      const uint32_t *s4 = reinterpret_cast<const uint32_t *>(src);
      uint32_t *d4 = reinterpret_cast<uint32_t *>(dst);
      const int nw = p / 2;
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < nw) w[i] = __ldg(s4 + i);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < nw) d4[i] = w[i];
    } else {
      for (int i = 0; i < p; ++i) dst[i] = src[i];
    }
  }
  const int pad = kp - k3;
  for (int u = threadIdx.x; u < nt * pad; u += blockDim.x) {
    const int tt = u / pad;
    patches[(long long)(im.base + tok0 + tt) * kp + k3 + (u - tt * pad)] = from_f32<T>(0.0f);
  }
  // position rows: work unit = (token, 8 channels)
  const int c8 = C / 8;
  for (int u = threadIdx.x; u < nt * c8; u += blockDim.x) {
    const int tt = u / c8, ch = (u - tt * c8) * 8;
    const int tok = tok0 + tt;
    const int r = tok / im.cols, c = tok - r * im.cols;
    int y0, y1, x0, x1;
    float wy, wx;
    bilinear_axis(r, im.rows, gh, y0, y1, wy);
    bilinear_axis(c, im.cols, gw, x0, x1, wx);
    float a[8], b[8], d[8], f[8], o[8];
    Vec8<T>::load(table + ((long long)y0 * gw + x0) * C + ch, a);
    Vec8<T>::load(table + ((long long)y0 * gw + x1) * C + ch, b);
    Vec8<T>::load(table + ((long long)y1 * gw + x0) * C + ch, d);
    Vec8<T>::load(table + ((long long)y1 * gw + x1) * C + ch, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float top = (1.0f - wx) * a[e] + wx * b[e];
      const float bot = (1.0f - wx) * d[e] + wx * f[e];
      o[e] = (1.0f - wy) * top + wy * bot;
    }
    Vec8<T>::store(pos + (long long)(im.base + tok) * C + ch, o);
  }
}

cudaError_t launch_embed_inputs(int dtype, const ImageTable &tab, int n_images,
                                long long max_tokens, const void *px, void *patches, int p, int kp,
                                const void *table, int gh, int gw, int C, void *pos,
                                cudaStream_t st) {
  if (n_images == 0 || max_tokens == 0) return cudaSuccess;
  const dim3 grid(unsigned((max_tokens + kTokPerBlock - 1) / kTokPerBlock), n_images);
  if (dtype == kF32)
    return launch_pdl(embed_inputs_kernel<float>, grid, dim3(256), 0, st, 1, tab,
                      static_cast<const float *>(px), static_cast<float *>(patches), p, kp, 0,
                      static_cast<const float *>(table), gh, gw, C, static_cast<float *>(pos));
  const int words = (p % 2 == 0 && (reinterpret_cast<uintptr_t>(px) & 3) == 0) ? 1 : 0;
  return launch_pdl(embed_inputs_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, 1, tab,
                    static_cast<const __nv_bfloat16 *>(px), static_cast<__nv_bfloat16 *>(patches),
                    p, kp, words, static_cast<const __nv_bfloat16 *>(table), gh, gw, C,
                    static_cast<__nv_bfloat16 *>(pos));
}

cudaError_t launch_pad_cols(int dtype, const void *w, void *out, int n, int k, int kp,
                            cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (dtype == kF32)
    return launch_pdl(pad_cols_kernel<float>, dim3(n), dim3(256), 0, st, 1,
                      static_cast<const float *>(w), static_cast<float *>(out), k, kp);
  return launch_pdl(pad_cols_kernel<__nv_bfloat16>, dim3(n), dim3(256), 0, st, 1,
                    static_cast<const __nv_bfloat16 *>(w), static_cast<__nv_bfloat16 *>(out), k, kp);
}

cudaError_t launch_pos_interp(int dtype, const ImageTable &tab, int n_images, long long max_tokens,
                              const void *table, int gh, int gw, int C, void *y, cudaStream_t st) {
  if (n_images == 0 || max_tokens == 0) return cudaSuccess;
  const dim3 grid(unsigned(max_tokens), n_images);
  if (dtype == kF32)
    return launch_pdl(pos_interp_kernel<float>, grid, dim3(128), 0, st, 1, tab,
                      static_cast<const float *>(table), gh, gw, C, static_cast<float *>(y));
  return launch_pdl(pos_interp_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, 1, tab,
                    static_cast<const __nv_bfloat16 *>(table), gh, gw, C,
                    static_cast<__nv_bfloat16 *>(y));
}

}  // namespace vit
