// k_rows.cu -- HBM-bound row kernels: LayerNorm, 2x2 spatial merge,
// positions from image grids, and in-place 2D RoPE on Q/K.
//
// KLiteInfer README, section "架构", paragraph "视觉算子": LayerNorm over
// row-major batched tokens, 2D RoPE, 2x2 spatial merge.  The pages' LayerNorm
// is one block per row with a two-pass reduction; here one warp owns a row,
// holds it in registers (one HBM read, one write) and reduces with shuffles.
#include <cuda_fp8.h>

#include "kernels.h"

namespace vit {

// ---------------------------------------------------------------- LayerNorm
template <typename T>
struct Vec4;  // four elements, one aligned load
template <>
struct Vec4<float> {
  using raw = float4;
  static __device__ __forceinline__ void unpack(const raw &r, float (&f)[4]) {
    f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
  }
  static __device__ __forceinline__ raw pack(const float (&f)[4]) {
    return make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <>
struct Vec4<__nv_bfloat16> {
  using raw = uint2;
  static __device__ __forceinline__ void unpack(const raw &r, float (&f)[4]) {
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
  }
  static __device__ __forceinline__ raw pack(const float (&f)[4]) {
    return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
  }
};

// One warp per row; lane l holds vectors l, l+32, l+64, ... (MAXV at most).
// gamma and beta, the same for every row, are staged once per block in
// shared memory while the rows are being loaded.
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) layernorm_warp_kernel(
    const T *__restrict__ x, T *__restrict__ y, const T *__restrict__ gamma,
    const T *__restrict__ beta, int rows, int cols, float eps) {
  using V = Vec4<T>;
  using R = typename V::raw;
  extern __shared__ __align__(16) unsigned char ln_smem[];
  pdl_trigger();
  pdl_wait();
  const int nvec = cols >> 2;  // cols % 4 == 0 checked by the host
  R *sg = reinterpret_cast<R *>(ln_smem);
  R *sb = sg + nvec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  const bool active = row < rows;
  const R *xr = reinterpret_cast<const R *>(x + size_t(active ? row : 0) * cols);
  float v[MAXV][4];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (active && c < nvec) {
      V::unpack(xr[c], v[i]);
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
    }
  }
  const R *gr = reinterpret_cast<const R *>(gamma);
  const R *br = reinterpret_cast<const R *>(beta);
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    sg[i] = __ldg(gr + i);
    sb[i] = __ldg(br + i);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) s += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / float(cols);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[i][e] - mean;
        q += d * d;
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = 1.0f / sqrtf(q / float(cols) + eps);
  __syncthreads();
  if (!active) return;
  R *yr = reinterpret_cast<R *>(y + size_t(row) * cols);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
      float g[4], b[4], o[4];
      V::unpack(sg[c], g);
      V::unpack(sb[c], b);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = (v[i][e] - mean) * rstd * g[e] + b[e];
      yr[c] = V::pack(o);
    }
  }
}

// Rows wider than a warp holds (cols > 4096, e.g. the 4C = 4608 columns of
// merged tokens): one block of 256 threads per row, thread t holding the
// 4-element vectors t, t + 256, ... (MAXV at most); the mean, then the
// centred variance, are reduced over the block (warp shuffles, then the 8
// warp partials through shared memory, summed in a fixed order).
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) layernorm_block_kernel(
    const T *__restrict__ x, T *__restrict__ y, const T *__restrict__ gamma,
    const T *__restrict__ beta, int rows, int cols, float eps) {
  using V = Vec4<T>;
  using R = typename V::raw;
  __shared__ float red[2][8];
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = cols >> 2;
  const R *xr = reinterpret_cast<const R *>(x + size_t(row) * cols);
  float v[MAXV][4];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = threadIdx.x + 256 * i;
    if (c < nvec) {
      V::unpack(xr[c], v[i]);
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) s += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[0][warp] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[0][w];
  const float mean = tot / float(cols);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    if (threadIdx.x + 256 * i < nvec) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[i][e] - mean;
        q = fmaf(d, d, q);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (lane == 0) red[1][warp] = q;
  __syncthreads();
  float qt = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) qt += red[1][w];
  const float rstd = 1.0f / sqrtf(qt / float(cols) + eps);
  R *yr = reinterpret_cast<R *>(y + size_t(row) * cols);
  const R *gr = reinterpret_cast<const R *>(gamma);
  const R *br = reinterpret_cast<const R *>(beta);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = threadIdx.x + 256 * i;
    if (c < nvec) {
      float g[4], b[4], o[4];
      V::unpack(__ldg(gr + c), g);
      V::unpack(__ldg(br + c), b);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = (v[i][e] - mean) * rstd * g[e] + b[e];
      yr[c] = V::pack(o);
    }
  }
}

// LayerNorm whose output goes straight to MXFP8 (bf16 only): the row is
// normalised exactly as layernorm_warp_kernel does, each result rounded to
// bf16 -- the value the plain kernel would store -- and then quantised as
// mx8_quantize_kernel does (X = floor(log2 amax) - 8 per 32-element group,
// clamped to [-127, 127]; E4M3 codes of x 2^-X, nearest even, saturating).
// Lane l holds 4-element vectors l, l + 32, ..., so a group is 8 lanes'
// vectors of one iteration and its amax takes three shuffles.  The grid
// covers the scale blocks' padded rows: a warp past the last row writes its
// padding scale bytes (127) and stops; every row writes the padding bytes
// of groups past the last column.
template <int MAXV>
__global__ void __launch_bounds__(256) layernorm_mx8_kernel(
    const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ gamma,
    const __nv_bfloat16 *__restrict__ beta, int rows, int cols, float eps,
    uint8_t *__restrict__ codes, uint8_t *__restrict__ scales, size_t row_bytes, int k_blocks) {
  using V = Vec4<__nv_bfloat16>;
  using R = V::raw;
  extern __shared__ __align__(16) unsigned char ln_smem[];
  pdl_trigger();
  pdl_wait();
  const int nvec = cols >> 2;
  const int groups = (cols + 31) / 32, pgroups = 4 * k_blocks;
  R *sg = reinterpret_cast<R *>(ln_smem);
  R *sb = sg + nvec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  const bool active = row < rows;
  auto scale_at = [&](int g) -> uint8_t & {
    const int rb = row >> 7, rr = row & 127, kb = g >> 2, jj = g & 3;
    return scales[(size_t(rb) * k_blocks + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + jj];
  };
  const R *xr = reinterpret_cast<const R *>(x + size_t(active ? row : 0) * cols);
  float v[MAXV][4];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (active && c < nvec) {
      V::unpack(xr[c], v[i]);
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
    }
  }
  const R *gr = reinterpret_cast<const R *>(gamma);
  const R *br = reinterpret_cast<const R *>(beta);
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    sg[i] = __ldg(gr + i);
    sb[i] = __ldg(br + i);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) s += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / float(cols);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[i][e] - mean;
        q += d * d;
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = 1.0f / sqrtf(q / float(cols) + eps);
  __syncthreads();
  if (row >= (rows + 127) / 128 * 128) return;
  if (!active) {  // a padding row of the last row block
    for (int g = lane; g < pgroups; g += 32) scale_at(g) = 127;
    return;
  }
  for (int g = groups + lane; g < pgroups; g += 32) scale_at(g) = 127;
  uint32_t *cr = reinterpret_cast<uint32_t *>(codes + size_t(row) * row_bytes);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    if (32 * i >= nvec) break;  // the same for the whole warp
    const int c = lane + 32 * i;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    if (c < nvec) {
      float g[4], b[4];
      V::unpack(sg[c], g);
      V::unpack(sb[c], b);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = (v[i][e] - mean) * rstd * g[e] + b[e];
      V::unpack(V::pack(o), o);  // the bf16 value the plain kernel stores
    }
    float amax = fmaxf(fmaxf(fabsf(o[0]), fabsf(o[1])), fmaxf(fabsf(o[2]), fabsf(o[3])));
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const int ef = int(__float_as_uint(amax) >> 23) & 0xFF;
    const int X = ef == 0 ? -127 : min(max(ef - 127 - 8, -127), 127);
    const float inv = __uint_as_float(uint32_t(127 - X) << 23);
    if (c < nvec) {
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(o[0] * inv, o[1] * inv),
                                                   __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(o[2] * inv, o[3] * inv),
                                                   __NV_SATFINITE, __NV_E4M3);
      cr[c] = (lo & 0xFFFFu) | ((hi & 0xFFFFu) << 16);
      if ((lane & 7) == 0) scale_at(c >> 3) = uint8_t(X + 127);
    }
  }
}

cudaError_t launch_layernorm_mx8(const void *x, const void *g, const void *b, int rows, int cols,
                                 float eps, uint8_t *codes, uint8_t *scales, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int nvec = cols / 4;
  if (cols % 4 || nvec > 32 * 12) return cudaErrorInvalidValue;
  const int warps = 8;
  const int prows = (rows + 127) / 128 * 128;
  dim3 grid((prows + warps - 1) / warps), block(32 * warps);
  const size_t smem = 2 * size_t(nvec) * sizeof(uint2);
  auto xp = static_cast<const __nv_bfloat16 *>(x);
  auto gp = static_cast<const __nv_bfloat16 *>(g);
  auto bp = static_cast<const __nv_bfloat16 *>(b);
  const size_t rb = (size_t(cols) + 15) / 16 * 16;
  const int kb = (cols + 127) / 128;
  if (nvec <= 32 * 4)
    return launch_pdl(layernorm_mx8_kernel<4>, grid, block, smem, st, 1, xp, gp, bp, rows, cols,
                      eps, codes, scales, rb, kb);
  if (nvec <= 32 * 9)
    return launch_pdl(layernorm_mx8_kernel<9>, grid, block, smem, st, 1, xp, gp, bp, rows, cols,
                      eps, codes, scales, rb, kb);
  return launch_pdl(layernorm_mx8_kernel<12>, grid, block, smem, st, 1, xp, gp, bp, rows, cols,
                    eps, codes, scales, rb, kb);
}

template <typename T>
cudaError_t launch_layernorm_t(const void *x, void *y, const void *g, const void *b, int rows,
                               int cols, float eps, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (cols > 4096) {  // a block per row (cols <= 16384, checked by the caller)
    auto k = layernorm_block_kernel<T, 16>;
    return launch_pdl(k, dim3(rows), dim3(256), 0, st, 1, static_cast<const T *>(x),
                      static_cast<T *>(y), static_cast<const T *>(g), static_cast<const T *>(b),
                      rows, cols, eps);
  }
  const int warps = 8;
  dim3 grid((rows + warps - 1) / warps), block(32 * warps);
  const int nvec = cols / 4;
  const size_t smem = 2 * size_t(nvec) * sizeof(typename Vec4<T>::raw);
  auto xp = static_cast<const T *>(x);
  auto yp = static_cast<T *>(y);
  auto gp = static_cast<const T *>(g);
  auto bp = static_cast<const T *>(b);
  if (nvec <= 32 * 4)
    return launch_pdl(layernorm_warp_kernel<T, 4>, grid, block, smem, st, 1, xp, yp, gp, bp, rows, cols, eps);
  else if (nvec <= 32 * 9)
    return launch_pdl(layernorm_warp_kernel<T, 9>, grid, block, smem, st, 1, xp, yp, gp, bp, rows, cols, eps);
  else if (nvec <= 32 * 12)
    return launch_pdl(layernorm_warp_kernel<T, 12>, grid, block, smem, st, 1, xp, yp, gp, bp, rows, cols, eps);
  else if (nvec <= 32 * 24)
    return launch_pdl(layernorm_warp_kernel<T, 24>, grid, block, smem, st, 1, xp, yp, gp, bp, rows, cols, eps);
  else
    return launch_pdl(layernorm_warp_kernel<T, 32>, grid, block, smem, st, 1, xp, yp, gp, bp, rows, cols, eps);
  return cudaGetLastError();
}

cudaError_t launch_layernorm(int dtype, const void *x, void *y, const void *g, const void *b,
                             int rows, int cols, float eps, cudaStream_t st) {
  return dtype == kF32 ? launch_layernorm_t<float>(x, y, g, b, rows, cols, eps, st)
                       : launch_layernorm_t<__nv_bfloat16>(x, y, g, b, rows, cols, eps, st);
}

// ---------------------------------------------------------------- LayerNorm folded into a GEMM
// With the LayerNorm folded into the projection that follows it, the
// projection reads the raw row x and forms
//   LN(x) w^T + b = rstd (x w'^T - mean s) + c,
//   w' = w diag(gamma), s_n = sum_k w'_nk, c = b + w beta,
// so only the row's mean and rstd are needed, as slice statistics: these
// come from the epilogue of the GEMM that wrote x (kEpiStats), or, for a
// stack's input, from this kernel.

// Row statistics of x [rows, cols] (bf16) in slices of kRowStatsWidth = 64
// columns: (mean, sum of squared deviations) per slice.  One warp per row;
// lane l holds 4-element vectors l, l + 32, ... (vector c = columns
// [4c, 4c + 4)), so for a fixed i lanes 0-15 hold slice 2i and lanes 16-31
// slice 2i + 1; each half-warp reduces its slice with shuffles, two passes
// over the registers.
template <int MAXV>
__global__ void __launch_bounds__(256) rowstats_kernel(const __nv_bfloat16 *__restrict__ x,
                                                       float2 *__restrict__ out, int rows,
                                                       int cols) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;  // whole warps only
  const int nvec = cols >> 2, parts = (cols + kRowStatsWidth - 1) / kRowStatsWidth;
  const uint2 *xr = reinterpret_cast<const uint2 *>(x + size_t(row) * cols);
  float v[MAXV][4];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
      const uint2 r = xr[c];
      v[i][0] = bf16_lo(r.x); v[i][1] = bf16_hi(r.x); v[i][2] = bf16_lo(r.y); v[i][3] = bf16_hi(r.y);
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    const int j = 2 * i + (lane >> 4);  // this half-warp's slice
    const int n = min(kRowStatsWidth, cols - j * kRowStatsWidth);  // <= 0: past the row
    float s = (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
#pragma unroll
    for (int o = 8; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / float(max(n, 1));
    float q = 0.f;
    if (c < nvec) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[i][e] - mean;
        q = fmaf(d, d, q);
      }
    }
#pragma unroll
    for (int o = 8; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if ((lane & 15) == 0 && n > 0) out[size_t(row) * parts + j] = make_float2(mean, q);
  }
}

cudaError_t launch_rowstats(const void *x, float2 *out, int rows, int cols, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((rows + warps - 1) / warps), block(32 * warps);
  const int nvec = cols / 4;
  auto xp = static_cast<const __nv_bfloat16 *>(x);
  if (nvec <= 32 * 4) return launch_pdl(rowstats_kernel<4>, grid, block, 0, st, 1, xp, out, rows, cols);
  if (nvec <= 32 * 9) return launch_pdl(rowstats_kernel<9>, grid, block, 0, st, 1, xp, out, rows, cols);
  if (nvec <= 32 * 12) return launch_pdl(rowstats_kernel<12>, grid, block, 0, st, 1, xp, out, rows, cols);
  if (nvec <= 32 * 24) return launch_pdl(rowstats_kernel<24>, grid, block, 0, st, 1, xp, out, rows, cols);
  return launch_pdl(rowstats_kernel<32>, grid, block, 0, st, 1, xp, out, rows, cols);
}

// The folded weight and its vectors, one warp per output row n, 8 columns
// per lane step: w_out = bf16(w * gamma) (a product of two bf16 values is
// exact in fp32, so this is a single rounding), s = sum of w_out as stored,
// c = b + sum_k w * beta, both accumulated in fp32 and reduced in a fixed
// shuffle order.  w_out may be w itself: each element is read before the
// same thread overwrites it.
__global__ void __launch_bounds__(256) fold_ln_kernel(
    const __nv_bfloat16 *w, const __nv_bfloat16 *__restrict__ gamma,
    const __nv_bfloat16 *__restrict__ beta, const __nv_bfloat16 *__restrict__ b,
    __nv_bfloat16 *w_out, float *__restrict__ sc, int n, int k) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= n) return;
  const uint4 *wr = reinterpret_cast<const uint4 *>(w + size_t(row) * k);
  uint4 *wo = reinterpret_cast<uint4 *>(w_out + size_t(row) * k);
  const uint4 *gr = reinterpret_cast<const uint4 *>(gamma);
  const uint4 *br = reinterpret_cast<const uint4 *>(beta);
  float s = 0.f, c = 0.f;
  for (int u = lane; u < k / 8; u += 32) {
    const uint4 wv = wr[u], gv = __ldg(gr + u), bv = __ldg(br + u);
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
    const uint32_t gg[4] = {gv.x, gv.y, gv.z, gv.w};
    const uint32_t bb[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t oo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float w0 = bf16_lo(ww[e]), w1 = bf16_hi(ww[e]);
      oo[e] = pack_bf16x2(w0 * bf16_lo(gg[e]), w1 * bf16_hi(gg[e]));
      s += bf16_lo(oo[e]) + bf16_hi(oo[e]);
      c = fmaf(w0, bf16_lo(bb[e]), c);
      c = fmaf(w1, bf16_hi(bb[e]), c);
    }
    wo[u] = make_uint4(oo[0], oo[1], oo[2], oo[3]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) {
    sc[row] = s;
    sc[n + row] = c + (b != nullptr ? __bfloat162float(b[row]) : 0.f);
  }
}

cudaError_t launch_fold_ln(const void *w, const void *gamma, const void *beta, const void *b,
                           void *w_out, float *sc, int n, int k, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  return launch_pdl(fold_ln_kernel, dim3((n + warps - 1) / warps), dim3(32 * warps), 0, st, 1,
                    static_cast<const __nv_bfloat16 *>(w), static_cast<const __nv_bfloat16 *>(gamma),
                    static_cast<const __nv_bfloat16 *>(beta), static_cast<const __nv_bfloat16 *>(b),
                    static_cast<__nv_bfloat16 *>(w_out), sc, n, k);
}

// ---------------------------------------------------------------- 2x2 merge
// One warp builds one merged token: the four source tokens' rows (each
// `units_per_token` units of U: 16 bytes, or 4 / 2 bytes when the row is
// not a multiple of 16 bytes) are concatenated in window order.  A lane
// issues up to kMergeBatch loads before its stores, so each warp keeps
// several kilobytes in flight; the index arithmetic is done once per token.
// blockIdx.y = image, blockIdx.x * warps + warp = merged token of the image.
constexpr int kMergeBatch = 16;

template <typename U>
__global__ void __launch_bounds__(128) merge2x2_kernel(const __grid_constant__ ImageTable tab,
                                                       const U *__restrict__ x,
                                                       U *__restrict__ y, int units_per_token) {
  pdl_trigger();
  pdl_wait();
  const ImageEntry im = tab.img[blockIdx.y];
  const int half_w = im.cols >> 1;
  const int out_tokens = (im.rows >> 1) * half_w;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int o = blockIdx.x * (blockDim.x >> 5) + warp; o < out_tokens;
       o += gridDim.x * (blockDim.x >> 5)) {
    const int R = o / half_w, Q = o - R * half_w;
    const long long top = im.base + (long long)(2 * R) * im.cols + 2 * Q;  // top-left source token
    // source token of window part p: top + (p >> 1) * cols + (p & 1)
    U *dst = y + ((long long)(im.base / 4) + o) * 4 * units_per_token;
    const int n = 4 * units_per_token;
    // flattened unit i = part * units_per_token + u, walked 32 at a time
    int part = 0, u = lane;
    while (part < 4 && u >= units_per_token) { u -= units_per_token; ++part; }
    for (int i0 = lane; i0 < n; i0 += 32 * kMergeBatch) {
      U v[kMergeBatch];
      int pk[kMergeBatch], uk[kMergeBatch];
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        pk[k] = part;
        uk[k] = u;
        if (part < 4)
          v[k] = x[(top + (long long)(part >> 1) * im.cols + (part & 1)) * units_per_token + u];
        u += 32;
        while (part < 4 && u >= units_per_token) { u -= units_per_token; ++part; }
      }
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k)
        if (pk[k] < 4) dst[pk[k] * units_per_token + uk[k]] = v[k];
    }
  }
}

cudaError_t launch_merge2x2(const ImageTable &tab, int n_images, const void *x, void *y,
                            size_t row_bytes, long long max_out_tokens, cudaStream_t st) {
  if (n_images == 0 || max_out_tokens == 0) return cudaSuccess;
  const int threads = 128, warps = threads / 32;
  const int bx = int(std::min<long long>((max_out_tokens + warps - 1) / warps, 65535));
  if (row_bytes % 16 == 0)
    return launch_pdl(merge2x2_kernel<uint4>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                      static_cast<const uint4 *>(x), static_cast<uint4 *>(y), int(row_bytes / 16));
  if (row_bytes % 4 == 0)
    return launch_pdl(merge2x2_kernel<uint32_t>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                      static_cast<const uint32_t *>(x), static_cast<uint32_t *>(y),
                      int(row_bytes / 4));
  return launch_pdl(merge2x2_kernel<uint16_t>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                    static_cast<const uint16_t *>(x), static_cast<uint16_t *>(y),
                    int(row_bytes / 2));
}

// ---------------------------------------------------------------- positions
__global__ void positions_kernel(const __grid_constant__ ImageTable tab, int n_images,
                                 int cu_offset_index, int32_t *__restrict__ cu,
                                 int32_t *__restrict__ pos) {
  const ImageEntry im = tab.img[blockIdx.y];
  const int n = im.rows * im.cols;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    cu[cu_offset_index + blockIdx.y + 1] = int32_t(im.base + n);
    if (blockIdx.y == 0 && cu_offset_index == 0) cu[0] = 0;
  }
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
    const int r = t / im.cols;
    const int c = t - r * im.cols;
    reinterpret_cast<int2 *>(pos)[im.base + t] = make_int2(r, c);
  }
}

cudaError_t launch_positions(const ImageTable &tab, int n_images, int cu_offset_index,
                             int max_tokens, int32_t *cu, int32_t *pos, cudaStream_t st) {
  if (n_images == 0) return cudaSuccess;
  const int threads = 256;
  int bx = std::max(1, std::min((max_tokens + threads - 1) / threads, 1024));
  positions_kernel<<<dim3(bx, n_images), threads, 0, st>>>(tab, n_images, cu_offset_index, cu,
                                                            pos);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- 2D RoPE
// In place on the Q and K parts of qkv [T, 3, H, d].  One thread rotates one
// half-head (d/2 contiguous elements: dims [0, d/2) by the row, [d/2, d) by
// the column; dim j pairs with j + d/4), read and written with 8-byte vector
// accesses.  The cos/sin of a block's tokens are computed once into shared
// memory (2 axes x d/4 frequencies per token) and shared by its 2*H Q/K heads.
template <typename T>
struct Vec8B;  // 8 bytes of T
template <>
struct Vec8B<__nv_bfloat16> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *f) {
    const uint2 r = *reinterpret_cast<const uint2 *>(p);
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float *f) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
  }
};
template <>
struct Vec8B<float> {
  static constexpr int N = 2;
  static __device__ __forceinline__ void load(const float *p, float *f) {
    const float2 r = *reinterpret_cast<const float2 *>(p);
    f[0] = r.x; f[1] = r.y;
  }
  static __device__ __forceinline__ void store(float *p, const float *f) {
    *reinterpret_cast<float2 *>(p) = make_float2(f[0], f[1]);
  }
};

template <typename T, int HALF>
__global__ void __launch_bounds__(256) rope2d_kernel(T *__restrict__ qkv,
                                                     const int32_t *__restrict__ pos, int T_,
                                                     int H, int tok_per_block,
                                                     const __grid_constant__ RopeFreqs fr) {
  constexpr int Q4 = HALF / 2;  // pairs per half-head
  using V = Vec8B<T>;
  extern __shared__ float2 cs[];  // [tok_per_block][2][Q4] = (cos, sin)
  pdl_trigger();
  pdl_wait();
  const int tok0 = blockIdx.x * tok_per_block;
  const int n_cs = tok_per_block * 2 * Q4;
  for (int i = threadIdx.x; i < n_cs; i += blockDim.x) {
    const int t = tok0 + i / (2 * Q4);
    const int r = i % (2 * Q4);
    const int axis = r / Q4, j = r % Q4;
    float sn = 0.f, c = 1.f;
    if (t < T_) sincospif(float(pos[2 * t + axis]) * fr.wpi[j], &sn, &c);
    cs[i] = make_float2(c, sn);
  }
  __syncthreads();
  const int units = 4 * H;  // (Q|K) x head x axis per token
  const int lt = threadIdx.x / units, u = threadIdx.x % units;
  const int t = tok0 + lt;
  if (lt >= tok_per_block || t >= T_) return;
  const int axis = u & 1, h = (u >> 1) % H, part = u / (2 * H);
  const int d = 2 * HALF;
  T *p = qkv + (size_t)t * 3 * H * d + (size_t)part * H * d + (size_t)h * d + axis * HALF;
  float v[HALF];
#pragma unroll
  for (int i = 0; i < HALF; i += V::N) V::load(p + i, v + i);
  const float2 *tc = cs + (lt * 2 + axis) * Q4;
#pragma unroll
  for (int j = 0; j < Q4; ++j) {
    const float2 k = tc[j];
    const float a = v[j], b = v[j + Q4];
    v[j] = a * k.x - b * k.y;
    v[j + Q4] = b * k.x + a * k.y;
  }
#pragma unroll
  for (int i = 0; i < HALF; i += V::N) V::store(p + i, v + i);
}

template <typename T>
static cudaError_t launch_rope_t(void *qkv, const int32_t *pos, int T_, int H, int d,
                                 const RopeFreqs &fr, cudaStream_t st) {
  const int units = 4 * H;
  const int tpb = std::max(1, 256 / units);
  const int threads = tpb * units;
  if (threads > 1024) return cudaErrorInvalidValue;
  const int blocks = (T_ + tpb - 1) / tpb;
  const size_t smem = sizeof(float2) * tpb * 2 * (d / 4);
  T *q = static_cast<T *>(qkv);
  switch (d) {
    case 64: return launch_pdl(rope2d_kernel<T, 32>, dim3(blocks), dim3(threads), smem, st, 1, q, pos, T_, H, tpb, fr);
    case 72: return launch_pdl(rope2d_kernel<T, 36>, dim3(blocks), dim3(threads), smem, st, 1, q, pos, T_, H, tpb, fr);
    case 128: return launch_pdl(rope2d_kernel<T, 64>, dim3(blocks), dim3(threads), smem, st, 1, q, pos, T_, H, tpb, fr);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rope2d(int dtype, void *qkv, const int32_t *pos, int T_, int H, int d,
                          const RopeFreqs &fr, cudaStream_t st) {
  if (T_ == 0) return cudaSuccess;
  return dtype == kF32 ? launch_rope_t<float>(qkv, pos, T_, H, d, fr, st)
                       : launch_rope_t<__nv_bfloat16>(qkv, pos, T_, H, d, fr, st);
}

}  // namespace vit
