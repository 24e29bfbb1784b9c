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

template <typename T>
cudaError_t launch_layernorm_t(const void *x, void *y, const void *g, const void *b, int rows,
                               int cols, float eps, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
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

// ---------------------------------------------------------------- 2x2 merge
// One thread copies one 16-byte unit (or one element-sized unit when the
// token row is not a multiple of 16 bytes).  blockIdx.y = image.
template <typename U>
__global__ void merge2x2_kernel(const __grid_constant__ ImageTable tab, const U *__restrict__ x,
                                U *__restrict__ y, int units_per_token) {
  pdl_trigger();
  pdl_wait();
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
    return launch_pdl(merge2x2_kernel<uint4>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                      static_cast<const uint4 *>(x), static_cast<uint4 *>(y), upt);
  } else if (row_bytes % 4 == 0) {
    const int upt = int(row_bytes / 4);
    long long units = max_out_tokens * 4 * upt;
    int bx = int(std::min<long long>((units + threads - 1) / threads, 4096));
    return launch_pdl(merge2x2_kernel<uint32_t>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                      static_cast<const uint32_t *>(x), static_cast<uint32_t *>(y), upt);
  } else {
    const int upt = int(row_bytes / 2);
    long long units = max_out_tokens * 4 * upt;
    int bx = int(std::min<long long>((units + threads - 1) / threads, 4096));
    return launch_pdl(merge2x2_kernel<uint16_t>, dim3(bx, n_images), dim3(threads), 0, st, 1, tab,
                      static_cast<const uint16_t *>(x), static_cast<uint16_t *>(y), upt);
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
