// k_simt.cu -- fp32-arithmetic SIMT kernels: GEMM + bias with fused
// epilogues, and bidirectional varlen attention.  These carry the fp32 mode
// of the library (the reference engine runs its vision tower in fp32 with TF32
// disabled, KLiteInfer README, "视觉算子": GEMM + bias via cuBLAS with TF32 off),
// so every product here is an IEEE fp32 FFMA.
#include "kernels.h"

namespace vit {

// ---------------------------------------------------------------- GEMM
// y[M,N] = epi(x[M,K] . w[N,K]^T + b).  64x64 tile, 16-deep k slices, 256
// threads, 4x4 outputs per thread at stride 16 (conflict-free smem reads).
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T *__restrict__ x,
                                                        const T *__restrict__ w,
                                                        const T *__restrict__ bias,
                                                        const T *__restrict__ res,
                                                        T *__restrict__ y, int M, int N, int K,
                                                        int epi) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int idx = threadIdx.x + 256 * l;  // 0..1023 over a 64x16 slice
      const int r = idx >> 4, c = idx & 15;
      const int gk = k0 + c;
      const int gm = m0 + r, gn = n0 + r;
      As[c][r] = (gm < M && gk < K) ? to_f32(x[(size_t)gm * K + gk]) : 0.f;
      Ws[c][r] = (gn < N && gk < K) ? to_f32(w[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      float v = acc[i][j] + (bias ? to_f32(bias[gn]) : 0.f);
      if (epi == kEpiGelu) v = gelu_tanh_f32(v);
      if (epi == kEpiResidual) v += to_f32(res[(size_t)gm * N + gn]);
      y[(size_t)gm * N + gn] = from_f32<T>(v);
    }
  }
}

cudaError_t launch_gemm_simt(int dtype, const void *x, const void *w, const void *b,
                             const void *res, void *y, int M, int N, int K, int epi,
                             cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  if (dtype == kF32)
    gemm_simt_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float *>(x), static_cast<const float *>(w),
        static_cast<const float *>(b), static_cast<const float *>(res), static_cast<float *>(y),
        M, N, K, epi);
  else
    gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w),
        static_cast<const __nv_bfloat16 *>(b), static_cast<const __nv_bfloat16 *>(res),
        static_cast<__nv_bfloat16 *>(y), M, N, K, epi);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- attention
// One CTA = 64 query rows of one (sequence, head); one thread per query row.
// Key tiles of 32 (prefix keys first, then the sequence's own keys) are
// staged in shared memory; 2D RoPE is applied to Q and own K as they are
// staged when pos is given.  Online softmax in fp32 with expf.
constexpr int kSimtQ = 64, kSimtK = 32;

template <typename T, int D>
__device__ __forceinline__ void stage_rows(float *dst, int ld, const T *src_base, size_t pitch,
                                           int n_rows, int valid_rows, const int32_t *pos_rows,
                                           const RopeFreqs &fr) {
  // Each work unit is one rotation pair (dims d1, d1 + D/4) of one row.
  constexpr int Q4 = D / 4;
  for (int idx = threadIdx.x; idx < n_rows * (D / 2); idx += blockDim.x) {
    const int r = idx / (D / 2);
    const int i = idx - r * (D / 2);
    const int axis = i / Q4, j = i - axis * Q4;
    const int d1 = axis * (D / 2) + j, d2 = d1 + Q4;
    float a = 0.f, b = 0.f;
    if (r < valid_rows) {
      const T *row = src_base + (size_t)r * pitch;
      a = to_f32(row[d1]);
      b = to_f32(row[d2]);
      if (pos_rows) {
        float sn, cs;
        sincospif(float(pos_rows[2 * r + axis]) * fr.wpi[j], &sn, &cs);
        const float a2 = a * cs - b * sn, b2 = b * cs + a * sn;
        a = a2;
        b = b2;
      }
    }
    dst[r * ld + d1] = a;
    dst[r * ld + d2] = b;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kSimtQ) attention_simt_kernel(const T *__restrict__ qkv,
                                                                T *__restrict__ o, SeqArgs s,
                                                                int H, float scale,
                                                                const __grid_constant__ RopeFreqs fr) {
  extern __shared__ float smem[];
  constexpr int LD = D + 1;
  float *Qs = smem;
  float *Ks = Qs + kSimtQ * LD;
  float *Vs = Ks + kSimtK * LD;
  const int seq = blockIdx.z, h = blockIdx.y;
  const int start = s.cu_seqlens[seq];
  const int len = s.cu_seqlens[seq + 1] - start;
  const int q0 = blockIdx.x * kSimtQ;
  if (q0 >= len) return;
  const int C = H * D;
  const size_t pitch = 3 * (size_t)C;
  const int qrows = min(kSimtQ, len - q0);
  stage_rows<T, D>(Qs, LD, qkv + (size_t)(start + q0) * pitch + (size_t)h * D, pitch, kSimtQ,
                   qrows, s.pos ? s.pos + 2 * (start + q0) : nullptr, fr);

  const int P = s.prefix_kv ? s.prefix_len : 0;
  const int Hkv = s.kv_heads > 0 ? s.kv_heads : H;
  const int hk = h / (H / Hkv);
  const int r = threadIdx.x;
  float acc[D];
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int nkeys = P + len;
  for (int k0 = 0; k0 < nkeys; k0 += kSimtK) {
    __syncthreads();
    // stage up to 32 keys: prefix part [k0, min(P, k0+32)), own part after it
    const int pk = max(0, min(P, k0 + kSimtK) - k0);
    if (pk > 0) {
      const T *pbase = static_cast<const T *>(s.prefix_kv);
      const size_t pp = (size_t)Hkv * D;
      const T *kb = pbase + ((size_t)(seq * 2 + 0) * P + k0) * pp + (size_t)hk * D;
      const T *vb = pbase + ((size_t)(seq * 2 + 1) * P + k0) * pp + (size_t)hk * D;
      stage_rows<T, D>(Ks, LD, kb, pp, pk, pk, nullptr, fr);
      stage_rows<T, D>(Vs, LD, vb, pp, pk, pk, nullptr, fr);
    }
    if (pk < kSimtK) {
      const int own0 = k0 + pk - P;  // first own key of this tile
      const int nown = kSimtK - pk;
      const int valid = max(0, min(nown, len - own0));
      const T *kb = qkv + (size_t)(start + own0) * pitch + C + (size_t)h * D;
      const T *vb = qkv + (size_t)(start + own0) * pitch + 2 * (size_t)C + (size_t)h * D;
      stage_rows<T, D>(Ks + pk * LD, LD, kb, pitch, nown, valid,
                       s.pos ? s.pos + 2 * (start + own0) : nullptr, fr);
      stage_rows<T, D>(Vs + pk * LD, LD, vb, pitch, nown, valid, nullptr, fr);
    }
    __syncthreads();
    const int kvalid = min(kSimtK, nkeys - k0);
    float sc[kSimtK];
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < kSimtK; ++c) {
      float dot = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) dot = fmaf(Qs[r * LD + e], Ks[c * LD + e], dot);
      sc[c] = (c < kvalid) ? dot * scale : -INFINITY;
      mt = fmaxf(mt, sc[c]);
    }
    const float mn = fmaxf(m, mt);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
    l *= alpha;
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] *= alpha;
#pragma unroll
    for (int c = 0; c < kSimtK; ++c) {
      const float p = (c < kvalid) ? expf(sc[c] - mn) : 0.f;
      l += p;
#pragma unroll
      for (int e = 0; e < D; ++e) acc[e] = fmaf(p, Vs[c * LD + e], acc[e]);
    }
    m = mn;
  }
  if (r < qrows) {
    T *orow = o + (size_t)(start + q0 + r) * C + (size_t)h * D;
    const float inv = 1.0f / l;
#pragma unroll
    for (int e = 0; e < D; ++e) orow[e] = from_f32<T>(acc[e] * inv);
  }
}

template <typename T, int D>
static cudaError_t launch_attn_simt_td(const void *qkv, void *o, const SeqArgs &s, int H,
                                       float scale, const RopeFreqs &fr, cudaStream_t st) {
  const size_t smem = sizeof(float) * (kSimtQ + 2 * kSimtK) * (D + 1);
  auto kern = attention_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((s.max_seqlen + kSimtQ - 1) / kSimtQ, H, s.n_seqs);
  kern<<<grid, kSimtQ, smem, st>>>(static_cast<const T *>(qkv), static_cast<T *>(o), s, H, scale,
                                   fr);
  return cudaGetLastError();
}

cudaError_t launch_attention_simt(int dtype, const void *qkv, void *o, const SeqArgs &s, int H,
                                  int d, float scale, const RopeFreqs &fr, int *status,
                                  cudaStream_t st) {
  (void)status;
  if (s.total_tokens == 0 || s.max_seqlen == 0) return cudaSuccess;
  if (dtype == kF32) {
    if (d == 64) return launch_attn_simt_td<float, 64>(qkv, o, s, H, scale, fr, st);
    if (d == 72) return launch_attn_simt_td<float, 72>(qkv, o, s, H, scale, fr, st);
    return launch_attn_simt_td<float, 128>(qkv, o, s, H, scale, fr, st);
  }
  if (d == 64) return launch_attn_simt_td<__nv_bfloat16, 64>(qkv, o, s, H, scale, fr, st);
  if (d == 72) return launch_attn_simt_td<__nv_bfloat16, 72>(qkv, o, s, H, scale, fr, st);
  return launch_attn_simt_td<__nv_bfloat16, 128>(qkv, o, s, H, scale, fr, st);
}

}  // namespace vit
