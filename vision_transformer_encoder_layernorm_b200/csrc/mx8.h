// mx8.h -- host-side declarations of the MXFP8 (block-scaled E4M3) kernels.
//
// Layouts (OCP Microscaling v1.0, MXFP8 with E4M3 elements):
//   codes  [rows, mx8_row_bytes(K)] uint8, element (r, k) at r * row_bytes + k;
//          bytes at k >= K are never read.
//   scales one E8M0 byte (2^(s-127)) per 32 consecutive elements of a row,
//          stored in 512-byte blocks, one per (128-row block, 128-column
//          block), block (rb, kb) at (rb * ceil(K/128) + kb) * 512.  Inside a
//          block, row r = r0 + 32*r1 (r0 < 32, r1 < 4) and 32-element group
//          j (< 4) sit at byte 16*r0 + 4*r1 + j: the shape the tensor core's
//          scale copy takes (32 lanes x 16 bytes, each lane holding 4 rows'
//          scale words).  Bytes of rows >= rows or groups past K hold 127.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace vit {

inline size_t mx8_row_bytes(int K) { return (size_t(K) + 15) / 16 * 16; }
inline size_t mx8_scale_bytes(int rows, int K) {
  return size_t((rows + 127) / 128) * size_t((K + 127) / 128) * 512;
}

// bf16 [rows, K] (row stride K) -> codes and scales.
cudaError_t launch_mx8_quantize(const void *x, int rows, int K, uint8_t *codes, uint8_t *scales,
                                cudaStream_t st);

// y[M, N] (bf16) = epi(deq(A) . deq(W)^T + b): A codes/scales [M, K], W
// codes/scales [N, K]; epi as launch_gemm_tc (bias, GELU, residual).  With
// kEpiGelu | kEpiQuant the output is MXFP8 instead: codes to y [M,
// mx8_row_bytes(N)] and scales to y_scales [mx8_scale_bytes(M, N)].
cudaError_t launch_gemm_mx8(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *w_codes,
                            const uint8_t *w_scales, const void *b, const void *res, void *y, int M,
                            int N, int K, int epi, int num_sms, int *status, cudaStream_t st,
                            uint8_t *y_scales = nullptr);

}  // namespace vit
