// k_rows.cu -- HBM-bound row kernels: LayerNorm, 2x2 spatial merge,
// positions from image grids, and in-place 2D RoPE on Q/K.
//
// KLiteInfer README, section "架构", paragraph "视觉算子": LayerNorm over
// row-major batched tokens, 2D RoPE, 2x2 spatial merge.  The pages' LayerNorm
// is one block per row with a two-pass reduction; here one warp owns a row,
// holds it in registers (one HBM read, one write) and reduces with shuffles.
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
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) layernorm_warp_kernel(
    const T *__restrict__ x, T *__restrict__ y, const T *__restrict__ gamma,
    const T *__restrict__ beta, int rows, int cols, float eps) {
  using V = Vec4<T>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const int nvec = cols >> 2;  // cols % 4 == 0 checked by the host
  const typename V::raw *xr = reinterpret_cast<const typename V::raw *>(x + size_t(row) * cols);
  float v[MAXV][4];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
      V::unpack(xr[c], v[i]);
      s += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
    } else {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
    }
  }
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
  const typename V::raw *gr = reinterpret_cast<const typename V::raw *>(gamma);
  const typename V::raw *br = reinterpret_cast<const typename V::raw *>(beta);
  typename V::raw *yr = reinterpret_cast<typename V::raw *>(y + size_t(row) * cols);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nvec) {
      float g[4], b[4], o[4];
      V::unpack(gr[c], g);
      V::unpack(br[c], b);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = (v[i][e] - mean) * rstd * g[e] + b[e];
      yr[c] = V::pack(o);
    }
  }
}

template <typename T>
cudaError_t launch_layernorm_t(const void *x, void *y, const void *g, const void *b, int rows,
                               int cols, float eps, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((rows + warps - 1) / warps), block(32 * warps);
  const int nvec = cols / 4;
  auto xp = static_cast<const T *>(x);
  auto yp = static_cast<T *>(y);
  auto gp = static_cast<const T *>(g);
  auto bp = static_cast<const T *>(b);
  if (nvec <= 32 * 4)
    layernorm_warp_kernel<T, 4><<<grid, block, 0, st>>>(xp, yp, gp, bp, rows, cols, eps);
  else if (nvec <= 32 * 12)
    layernorm_warp_kernel<T, 12><<<grid, block, 0, st>>>(xp, yp, gp, bp, rows, cols, eps);
  else
    layernorm_warp_kernel<T, 32><<<grid, block, 0, st>>>(xp, yp, gp, bp, rows, cols, eps);
  return cudaGetLastError();
}

cudaError_t launch_layernorm(int dtype, const void *x, void *y, const void *g, const void *b,
                             int rows, int cols, float eps, cudaStream_t st) {
  return dtype == kF32 ? launch_layernorm_t<float>(x, y, g, b, rows, cols, eps, st)
                       : launch_layernorm_t<__nv_bfloat16>(x, y, g, b, rows, cols, eps, st);
}

// ---------------------------------------------------------------- 2x2 merge
// One thread copies one 16-byte unit (or one element-sized unit when the
// token row is not a multiple of 16 bytes).  blockIdx.y = image.
template <typename U>
__global__ void merge2x2_kernel(const __grid_constant__ ImageTable tab, const U *__restrict__ x,
                                U *__restrict__ y, int units_per_token) {
  const ImageEntry im = tab.img[blockIdx.y];
  const int half_w = im.cols >> 1;
  const long long out_tokens = (long long)(im.rows >> 1) * half_w;
  const long long total = out_tokens * 4 * units_per_token;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long o = i / (4 * units_per_token);
    const int rem = int(i - o * 4 * units_per_token);
    const int part = rem / units_per_token;  // 0 TL, 1 TR, 2 BL, 3 BR
    const int u = rem - part * units_per_token;
    const int R = int(o / half_w), Q = int(o - (long long)R * half_w);
    const long long src_tok =
        im.base + (long long)(2 * R + (part >> 1)) * im.cols + (2 * Q + (part & 1));
    const long long dst_tok = im.base / 4 + o;
    y[dst_tok * 4 * units_per_token + part * units_per_token + u] =
        x[src_tok * units_per_token + u];
  }
}

cudaError_t launch_merge2x2(const ImageTable &tab, int n_images, const void *x, void *y,
                            size_t row_bytes, long long max_out_tokens, cudaStream_t st) {
  if (n_images == 0 || max_out_tokens == 0) return cudaSuccess;
  const int threads = 256;
  if (row_bytes % 16 == 0) {
    const int upt = int(row_bytes / 16);
    long long units = max_out_tokens * 4 * upt;
    int bx = int(std::min<long long>((units + threads - 1) / threads, 4096));
    merge2x2_kernel<uint4><<<dim3(bx, n_images), threads, 0, st>>>(
        tab, static_cast<const uint4 *>(x), static_cast<uint4 *>(y), upt);
  } else if (row_bytes % 4 == 0) {
    const int upt = int(row_bytes / 4);
    long long units = max_out_tokens * 4 * upt;
    int bx = int(std::min<long long>((units + threads - 1) / threads, 4096));
    merge2x2_kernel<uint32_t><<<dim3(bx, n_images), threads, 0, st>>>(
        tab, static_cast<const uint32_t *>(x), static_cast<uint32_t *>(y), upt);
  } else {
    const int upt = int(row_bytes / 2);
    long long units = max_out_tokens * 4 * upt;
    int bx = int(std::min<long long>((units + threads - 1) / threads, 4096));
    merge2x2_kernel<uint16_t><<<dim3(bx, n_images), threads, 0, st>>>(
        tab, static_cast<const uint16_t *>(x), static_cast<uint16_t *>(y), upt);
  }
  return cudaGetLastError();
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
// In place on the Q and K parts of qkv [T, 3, H, d].  One thread per
// (token, Q|K, head, half, pair).
template <typename T>
__global__ void rope2d_kernel(T *__restrict__ qkv, const int32_t *__restrict__ pos, int T_,
                              int H, int d, const __grid_constant__ RopeFreqs fr) {
  const int quarter = d >> 2;                  // pairs per half
  const long long per_tok = 2LL * H * 2 * quarter;
  const long long total = (long long)T_ * per_tok;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = int(i / per_tok);
    int r = int(i - (long long)t * per_tok);
    const int j = r % quarter;
    r /= quarter;
    const int axis = r & 1;
    r >>= 1;
    const int h = r % H;
    const int part = r / H;  // 0 Q, 1 K
    const float p = float(pos[2 * t + axis]);
    float sn, cs;
    sincospif(p * fr.wpi[j], &sn, &cs);
    T *base = qkv + (size_t)t * 3 * H * d + (size_t)part * H * d + (size_t)h * d + axis * 2 * quarter;
    const float a = to_f32(base[j]), b = to_f32(base[j + quarter]);
    base[j] = from_f32<T>(a * cs - b * sn);
    base[j + quarter] = from_f32<T>(b * cs + a * sn);
  }
}

cudaError_t launch_rope2d(int dtype, void *qkv, const int32_t *pos, int T_, int H, int d,
                          const RopeFreqs &fr, cudaStream_t st) {
  if (T_ == 0) return cudaSuccess;
  const long long total = (long long)T_ * 2 * H * (d / 2);
  const int threads = 256;
  const int blocks = int(std::min<long long>((total + threads - 1) / threads, 148LL * 16));
  if (dtype == kF32)
    rope2d_kernel<float><<<blocks, threads, 0, st>>>(static_cast<float *>(qkv), pos, T_, H, d, fr);
  else
    rope2d_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(static_cast<__nv_bfloat16 *>(qkv),
                                                            pos, T_, H, d, fr);
  return cudaGetLastError();
}

}  // namespace vit
