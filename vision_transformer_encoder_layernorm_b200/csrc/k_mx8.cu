// k_mx8.cu -- bf16 -> MXFP8 quantisation (OCP Microscaling v1.0: E4M3
// elements, one E8M0 scale per 32 consecutive elements of a row).
//
// The pages point at 8-bit inference (the NEO++ launcher page's fp8
// checkpoints; KLiteInfer README, "已知限制与后续": FP16 / INT8 next) without
// a format; this is the block-scaled format the tensor core's kind::mxf8f6f4
// MMA consumes.  One thread per 32-element group:
//   X = floor(log2(amax)) - 8 (8 = exponent of E4M3's largest normal, 448),
//       clamped to [-127, 127]; an all-zero group gets -127;
//   code = E4M3(x * 2^-X), round to nearest even, saturating at +-448.
// x * 2^-X is exact in fp32 (a power-of-two rescale that stays in range for
// every bf16 input), so the conversion decides exactly as an fp64 reference.
// The scale byte X + 127 is written straight into the 512-byte blocks the
// GEMM copies into tensor memory (layout in mx8.h); the threads run over the
// blocks' whole padded shape, and those past the rows or groups write the
// padding byte 127 (2^0), so no separate fill is needed.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "kernels.h"
#include "mx8.h"

namespace vit {

__global__ void __launch_bounds__(256) mx8_quantize_kernel(const __nv_bfloat16 *__restrict__ x,
                                                           int rows, int K, size_t row_bytes,
                                                           int k_blocks, uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ scales) {
  pdl_trigger();
  pdl_wait();
  const int groups = (K + 31) / 32, pgroups = 4 * k_blocks, prows = (rows + 127) / 128 * 128;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)prows * pgroups) return;
  const int r = int(gid / pgroups), j = int(gid - (long long)r * pgroups);
  if (r >= rows || j >= groups) {  // a padding entry of the scale blocks
    const int rb = r >> 7, rr = r & 127, kb = j >> 2, jj = j & 3;
    scales[(size_t(rb) * k_blocks + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + jj] = 127;
    return;
  }
  const int k0 = j * 32, n = min(32, K - k0);
  const __nv_bfloat16 *xr = x + size_t(r) * K + k0;
  float v[32];
  if (n == 32 && (K % 8) == 0) {  // 16-byte aligned: row start r*K*2 and k0*2 are multiples of 16
    const uint4 *p = reinterpret_cast<const uint4 *>(xr);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(p + q);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
        v[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = i < n ? __bfloat162float(xr[i]) : 0.f;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  // floor(log2(amax)) from the exponent field; zero and subnormal amax
  // (below 2^-126) give X below -127, i.e. the clamp
  const int ef = int(__float_as_uint(amax) >> 23) & 0xFF;
  const int X = ef == 0 ? -127 : min(max(ef - 127 - 8, -127), 127);
  const float inv = __uint_as_float(uint32_t(127 - X) << 23);  // 2^-X (X <= 120 for bf16 inputs)
  uint32_t packed[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 f = make_float2(v[4 * q + 2 * h] * inv, v[4 * q + 2 * h + 1] * inv);
      const uint32_t pair = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);  // .x low byte
      word |= (pair & 0xFFFFu) << (16 * h);
    }
    packed[q] = word;
  }
  uint8_t *cr = codes + size_t(r) * row_bytes + k0;
  if (n == 32) {  // k0 is a multiple of 32 and row_bytes of 16: 16-byte aligned
    reinterpret_cast<uint4 *>(cr)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    reinterpret_cast<uint4 *>(cr)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  } else {
    for (int i = 0; i < n; ++i) cr[i] = uint8_t(packed[i >> 2] >> (8 * (i & 3)));
  }
  const int rb = r >> 7, rr = r & 127, kb = j >> 2, jj = j & 3;
  scales[(size_t(rb) * k_blocks + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + jj] =
      uint8_t(X + 127);
}

cudaError_t launch_mx8_quantize(const void *x, int rows, int K, uint8_t *codes, uint8_t *scales,
                                cudaStream_t st) {
  if (rows == 0 || K == 0) return cudaSuccess;
  const long long threads = (long long)((rows + 127) / 128 * 128) * (4 * ((K + 127) / 128));
  const int block = 256;
  const long long grid = (threads + block - 1) / block;
  if (grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  return launch_pdl(mx8_quantize_kernel, dim3(unsigned(grid)), dim3(block), 0, st, 1,
                    static_cast<const __nv_bfloat16 *>(x), rows, K, mx8_row_bytes(K),
                    (K + 127) / 128, codes, scales);
}

}  // namespace vit
