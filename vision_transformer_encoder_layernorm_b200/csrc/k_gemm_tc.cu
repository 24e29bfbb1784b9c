// k_gemm_tc.cu -- tcgen05 GEMM with fused epilogues for the dense
// projections of the encoder layer (QKV, output projection, fc1, fc2).
//
// KLiteInfer README, "视觉算子": the projections are GEMM + bias over
// row-major batched tokens (cuBLAS fp32 there).  Here: y = epi(x w^T + b) with
// bf16 operands, fp32 accumulation in tensor memory, and bias, GELU(tanh) or
// the residual add applied on the way out of TMEM.
//
// Structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: 128x64 tile of x and BNx64 tile of w per stage,
//               128-byte swizzled, into a STAGES-deep shared-memory ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (128 x BN x 16)
//               into one of two TMEM accumulators and commits stage releases.
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time (thread = row),
//               bias / GELU / residual in fp32, bf16 stores.
// The two accumulators let the epilogue of tile i overlap the main loop of
// tile i+1.  Every wait is bounded (see mbar_wait); on a timeout the kernel
// drains its in-flight copies, frees TMEM and reports through `status`.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace vit {

namespace gemm {
constexpr int BM = 128;
constexpr int BK = 64;                     // one 128-byte swizzle atom of bf16
constexpr int kThreads = 192;
constexpr uint32_t kATileBytes = BM * BK * 2;  // 16 KB

template <int BN>
struct Cfg {
  static constexpr uint32_t kBTileBytes = BN * BK * 2;
  static constexpr uint32_t kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kStages = (BN >= 256) ? 4 : 6;
  static constexpr uint32_t kTmemCols = (2 * BN <= 256) ? 256 : 512;
  // ring + barriers/bookkeeping + 1 KB alignment slack
  static constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN);
};

struct __align__(8) Bars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float gelu_fast(float u) {
  const float k0 = 0.7978845608028654f, k1 = 0.044715f;
  return 0.5f * u * (1.0f + tanh_fast(k0 * fmaf(k1 * u, u * u, u)));
}

// Waits bounded by time only (used while draining after an abort).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;  // 200 ms
  }
}

}  // namespace gemm

template <int BN, int EPI>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __nv_bfloat16 *__restrict__ bias, const __nv_bfloat16 *__restrict__ res,
                   __nv_bfloat16 *__restrict__ y, int M, int N, int K, int *status) {
  using namespace gemm;
  using CF = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + size_t(CF::kStages) * CF::kStageBytes);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int k_blocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, CF::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;  // per stage: last fill parity
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t *sa = smem + size_t(stage) * CF::kStageBytes;
          mbar_arrive_expect_tx(&bars->full[stage], CF::kStageBytes);
          tma_load_2d(sa, &tmA, &bars->full[stage], kb * BK, mb * BM);
          tma_load_2d(sa + kATileBytes, &tmB, &bars->full[stage], kb * BK, nb * BN);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // make sure no TMA write into this CTA's shared memory is still in flight
        for (int s = 0; s < CF::kStages; ++s)
          if (issued_mask & (1u << s)) drain_wait(&bars->full[s], (issued_parity >> s) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool any_mma = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int a = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&bars->acc_empty[a], aphase ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + uint32_t(a * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&bars->full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + size_t(stage) * CF::kStageBytes);
          const uint32_t sb = sa + kATileBytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = smem_desc(sa + k * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(sb + k * 32, 16, 1024, 2);
            mma_bf16_ss(d_tmem, ad, bd, CF::kIdesc, (kb | k) != 0);
          }
          any_mma = true;
          mma_commit(&bars->empty[stage]);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&bars->acc_full[a]);
      }
      if (!ok && any_mma) {
        // wait until every MMA issued so far has finished before TMEM is freed
        mma_commit(&bars->drain);
        drain_wait(&bars->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
    const int row_in_tile = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int a = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!mbar_wait(&bars->acc_full[a], aphase, abort_flag)) break;
      tc_fence_after();
      const int row = mb * BM + row_in_tile;
      const bool row_ok = row < M;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + (uint32_t(quarter * 32) << 16) + uint32_t(a * BN + c * 32), r);
        tmem_ld_wait();
        const int col0 = nb * BN + c * 32;
        if (!row_ok || col0 >= N) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if (bias != nullptr) {
          const uint4 *bp = reinterpret_cast<const uint4 *>(bias + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (col0 + 8 * q < N) {
              const uint4 b4 = __ldg(bp + q);
              v[8 * q + 0] += bf16_lo(b4.x); v[8 * q + 1] += bf16_hi(b4.x);
              v[8 * q + 2] += bf16_lo(b4.y); v[8 * q + 3] += bf16_hi(b4.y);
              v[8 * q + 4] += bf16_lo(b4.z); v[8 * q + 5] += bf16_hi(b4.z);
              v[8 * q + 6] += bf16_lo(b4.w); v[8 * q + 7] += bf16_hi(b4.w);
            }
          }
        }
        if (EPI == kEpiGelu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_fast(v[i]);
        }
        if (EPI == kEpiResidual) {
          const uint4 *rp = reinterpret_cast<const uint4 *>(res + size_t(row) * N + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (col0 + 8 * q < N) {
              const uint4 r4 = __ldg(rp + q);
              v[8 * q + 0] += bf16_lo(r4.x); v[8 * q + 1] += bf16_hi(r4.x);
              v[8 * q + 2] += bf16_lo(r4.y); v[8 * q + 3] += bf16_hi(r4.y);
              v[8 * q + 4] += bf16_lo(r4.z); v[8 * q + 5] += bf16_hi(r4.z);
              v[8 * q + 6] += bf16_lo(r4.w); v[8 * q + 7] += bf16_hi(r4.w);
            }
          }
        }
        uint4 *yp = reinterpret_cast<uint4 *>(y + size_t(row) * N + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (col0 + 8 * q < N) {
            uint4 o;
            o.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
            o.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
            o.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
            o.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
            yp[q] = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, CF::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report_status(status, kDevTimeout);
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                              uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  if (g_encode == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        fn == nullptr)
      return CUDA_ERROR_NOT_FOUND;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int BN, int EPI>
static cudaError_t launch_bn(const CUtensorMap &ta, const CUtensorMap &tb, const void *b,
                             const void *res, void *y, int M, int N, int K, int num_sms,
                             int *status, cudaStream_t st) {
  using CF = gemm::Cfg<BN>;
  auto kern = gemm_tc_kernel<BN, EPI>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CF::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + BN - 1) / BN);
  const int grid = std::max(1, std::min(tiles, num_sms));
  kern<<<grid, gemm::kThreads, CF::kSmemBytes, st>>>(
      ta, tb, static_cast<const __nv_bfloat16 *>(b), static_cast<const __nv_bfloat16 *>(res),
      static_cast<__nv_bfloat16 *>(y), M, N, K, status);
  return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_epi(int epi, const CUtensorMap &ta, const CUtensorMap &tb,
                              const void *b, const void *res, void *y, int M, int N, int K,
                              int num_sms, int *status, cudaStream_t st) {
  switch (epi) {
    case kEpiGelu:
      return launch_bn<BN, kEpiGelu>(ta, tb, b, res, y, M, N, K, num_sms, status, st);
    case kEpiResidual:
      return launch_bn<BN, kEpiResidual>(ta, tb, b, res, y, M, N, K, num_sms, status, st);
    default:
      return launch_bn<BN, kEpiBias>(ta, tb, b, res, y, M, N, K, num_sms, status, st);
  }
}

// Tile width: the narrower tile wins when it needs fewer full waves of
// output tiles (makespan ~ waves x tile width).
static int choose_bn(int M, int N, int num_sms) {
  const int mt = (M + gemm::BM - 1) / gemm::BM;
  long best_cost = -1;
  int best = 256;
  for (int bn : {256, 128}) {
    const long tiles = long(mt) * ((N + bn - 1) / bn);
    const long waves = (tiles + num_sms - 1) / num_sms;
    const long cost = waves * bn;
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = bn; }
  }
  return best;
}

cudaError_t launch_gemm_tc(const void *x, const void *w, const void *b, const void *res, void *y,
                           int M, int N, int K, int epi, int num_sms, int *status,
                           cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const int bn = choose_bn(M, N, num_sms);
  CUtensorMap ta, tb;
  if (encode_tensor_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, uint64_t(K) * 2,
                           gemm::BK, gemm::BM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, uint64_t(K) * 2,
                           gemm::BK, bn, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (bn == 256) return launch_epi<256>(epi, ta, tb, b, res, y, M, N, K, num_sms, status, st);
  return launch_epi<128>(epi, ta, tb, b, res, y, M, N, K, num_sms, status, st);
}

}  // namespace vit
