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
//   warps 2-9   epilogue: two warps per TMEM lane quarter (thread = row), each
//               draining half of the tile's columns 32 at a time; each warp
//               stages its bias half in shared memory, residual loads are
//               overlapped with the TMEM load; fp32 math, bf16 stores.
// The two accumulators let the epilogue of tile i overlap the main loop of
// tile i+1.  Every wait is bounded (see mbar_wait); on a timeout the kernel
// drains its in-flight copies, frees TMEM and reports through `status`.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>

#include <atomic>

#include <cuda_fp8.h>

#include "kernels.h"
#include "mx8.h"
#include "sm100.cuh"
#include "sm100_mx8.cuh"

namespace vit {

namespace gemm {
constexpr int BM = 128;
constexpr int BK = 64;                     // one 128-byte swizzle atom of bf16
constexpr int kThreads = 320;   // 2 role warps + 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr uint32_t kATileBytes = BM * BK * 2;  // 16 KB

constexpr size_t kSmemLimit = 232448;  // dynamic shared memory of one CTA (227 KB)

// Shared memory after the operand ring, counted from the barrier block:
// barriers and bias slots (3 KB) -- with a folded LayerNorm (no bias) the
// LayerNorm's slots take the place of the bias slots, right after the
// barriers -- then one output staging buffer per epilogue warp: a 32 x 32
// chunk (64-byte swizzled), or for a RoPE tile one head of 32 rows x HD
// columns.  A LayerNorm slot holds s and c of the warp's columns: half a
// non-RoPE tile (<= 128 columns) or two heads of 72 / one of 128.
constexpr uint32_t kLnSlotBytes = 1152;
constexpr uint32_t kLnSlotsOffset = 256;
template <int EPI, int TS>
struct EpiSmem {
  static constexpr bool kRope = (EPI & 3) == 3;
  static constexpr int kHD = kRope ? (TS == 216 ? 72 : TS / 2) : 0;
  static constexpr uint32_t kBufBytes = kRope ? uint32_t(32 * kHD * 2) : 2048u;
  static constexpr uint32_t kLnBytes = (EPI & 4) ? kEpiWarps * kLnSlotBytes : 0u;
  static constexpr uint32_t kBufOff =
      (EPI & 4) ? (kLnSlotsOffset + kLnBytes + 1023u) / 1024u * 1024u : 3072u;
  static constexpr uint32_t kAfterRing = kBufOff + kEpiWarps * kBufBytes;
};

// Operand ring of a GEMM variant: as many stages (at most 8) as fit next to
// the epilogue's shared memory.  PAIR: a CTA holds half of the tile's W rows.
template <int BN, int EPI, int TS, bool PAIR>
struct Cfg {
  using ES = EpiSmem<EPI, TS>;
  static constexpr uint32_t kBRows = PAIR ? BN / 2 : BN;
  static constexpr uint32_t kStageBytes = kATileBytes + kBRows * BK * 2;
  static constexpr int kFit = int((kSmemLimit - 1024 - ES::kAfterRing) / kStageBytes);
  static constexpr int kStages = kFit > 8 ? 8 : kFit;
  static constexpr uint32_t kTmemCols = (2 * BN <= 256) ? 256 : 512;
  // ring + 1 KB alignment slack + barriers, slots and staging buffers
  static constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 + ES::kAfterRing;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(PAIR ? 256 : BM, BN);
  static_assert(kStages >= 2 && kStageBytes % 1024 == 0, "operand ring");
};

struct __align__(16) Bars {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= kLnSlotsOffset, "barrier block overlaps the LayerNorm slots");

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

// Mean and 1/sqrt(var + eps) of row `row` of a LayerNorm input of K
// columns, from its slice statistics (mean_j, M2_j) over slices of n_j
// columns: mean = sum_j n_j mean_j / K, M2 = sum_j M2_j + sum_j n_j
// (mean_j - mean)^2 (the two-pass form of Chan's merge).  Rows of up to
// kStatRegs slices are loaded at once into registers (all loads in flight
// together); longer rows take a loop over L1.
constexpr int kStatRegs = 20;
__device__ __forceinline__ void ln_row_stats(const EpiArgs &ea, int row, int K, float &mu,
                                             float &rstd) {
  const SliceStats &st = ea.stats_in;
  const float2 *p = st.p + size_t(row) * st.parts;
  const int last = st.parts - 1;
  const float wf = float(st.w), nl = float(K - last * st.w);
  float mean, m2 = 0.f, dev = 0.f;
  if (st.parts <= kStatRegs) {
    float2 e[kStatRegs];
#pragma unroll
    for (int j = 0; j < kStatRegs; ++j) e[j] = j < st.parts ? __ldg(p + j) : make_float2(0.f, 0.f);
    float s = 0.f, ml = 0.f, m2l = 0.f;
#pragma unroll
    for (int j = 0; j < kStatRegs; ++j) {
      if (j < last) s += e[j].x;
      if (j == last) {
        ml = e[j].x;
        m2l = e[j].y;
      }
    }
    mean = fmaf(wf, s, nl * ml) / float(K);
#pragma unroll
    for (int j = 0; j < kStatRegs; ++j)
      if (j < last) {
        const float d = e[j].x - mean;
        m2 += e[j].y;
        dev = fmaf(d, d, dev);
      }
    const float dl = ml - mean;
    m2 += m2l + fmaf(wf, dev, nl * dl * dl);
  } else {
    float s = 0.f;
#pragma unroll 6
    for (int j = 0; j < last; ++j) s += __ldg(p + j).x;
    mean = fmaf(wf, s, nl * __ldg(p + last).x) / float(K);
#pragma unroll 6
    for (int j = 0; j < last; ++j) {
      const float2 e = __ldg(p + j);
      const float d = e.x - mean;
      m2 += e.y;
      dev = fmaf(d, d, dev);
    }
    const float2 el = __ldg(p + last);
    const float dl = el.x - mean;
    m2 += el.y + fmaf(wf, dev, nl * dl * dl);
  }
  mu = mean;
  rstd = 1.0f / sqrtf(m2 / float(K) + ea.ln_eps);
}

using gemm::kLnSlotBytes;
using gemm::kLnSlotsOffset;

// Stages s and c of NSEG column segments of `ncols` columns each, starting
// at col0[k] (fp32 [2][N] at ea.ln_sc), into slot + k * 2 ncols: s, then c;
// columns past N read as zero.  Every load is issued before the first
// shared-memory store.  Warp-level only (the slot is private to the warp).
template <int NSEG, int MAXV>
__device__ __forceinline__ void stage_ln_cols(float *slot, const EpiArgs &ea,
                                              const int (&col0)[NSEG], int nseg, int ncols, int N,
                                              int lane) {
  float4 sv[NSEG][MAXV], cv[NSEG][MAXV];
#pragma unroll
  for (int k = 0; k < NSEG; ++k)
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
      const int i = lane + 32 * m;
      const int c = col0[k] + 4 * i;
      const bool in = k < nseg && i < ncols / 4 && c < N;
      sv[k][m] = in ? __ldg(reinterpret_cast<const float4 *>(ea.ln_sc + c))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      cv[k][m] = in ? __ldg(reinterpret_cast<const float4 *>(ea.ln_sc + N + c))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
  for (int k = 0; k < NSEG; ++k)
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
      const int i = lane + 32 * m;
      if (k < nseg && i < ncols / 4) {
        reinterpret_cast<float4 *>(slot + k * 2 * ncols)[i] = sv[k][m];
        reinterpret_cast<float4 *>(slot + k * 2 * ncols + ncols)[i] = cv[k][m];
      }
    }
}

// Running (count, mean, M2) of a row slice, merged chunk by chunk.
struct RunStats {
  float n = 0.f, mean = 0.f, m2 = 0.f;
  __device__ __forceinline__ void merge(float nb, float mb, float m2b) {
    const float nn = n + nb;
    const float f = nb / nn;
    const float d = mb - mean;
    mean = fmaf(d, f, mean);
    m2 += m2b + d * d * n * f;
    n = nn;
  }
};

// One 32-column slice of one output row: fp32 accumulators r, then either
// + bias (from shared memory) or, with the LayerNorm folded in,
// rstd (r - mu s) + c (s, c already loaded); then the epilogue op (GELU, or
// + residual rv, already loaded); the 32 results rounded to bf16 in o.
// With kEpiStats and `valid` (the row and the chunk exist), adds the mean
// and M2 of the stored values of the chunk's columns below N to `rs`.
template <int EPI>
__device__ __forceinline__ void compute_chunk(const uint32_t (&r)[32], int col0, int N, bool valid,
                                              const __nv_bfloat16 *bias_s, const uint4 (&rv)[4],
                                              const float4 (&sv)[8], const float4 (&cv)[8],
                                              float mu, float rstd, uint4 (&o)[4], RunStats &rs) {
  constexpr int OP = EPI & kEpiOpMask;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if constexpr ((EPI & kEpiLn) != 0) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float sq[4] = {sv[q].x, sv[q].y, sv[q].z, sv[q].w};
      const float cq[4] = {cv[q].x, cv[q].y, cv[q].z, cv[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * q + e] = fmaf(rstd, fmaf(-mu, sq[e], v[4 * q + e]), cq[e]);
    }
  } else {
    const uint4 *bp = reinterpret_cast<const uint4 *>(bias_s);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 b4 = bp[q];
      v[8 * q + 0] += bf16_lo(b4.x); v[8 * q + 1] += bf16_hi(b4.x);
      v[8 * q + 2] += bf16_lo(b4.y); v[8 * q + 3] += bf16_hi(b4.y);
      v[8 * q + 4] += bf16_lo(b4.z); v[8 * q + 5] += bf16_hi(b4.z);
      v[8 * q + 6] += bf16_lo(b4.w); v[8 * q + 7] += bf16_hi(b4.w);
    }
  }
  if constexpr (OP == kEpiGelu) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gemm::gelu_fast(v[i]);
  }
  if constexpr (OP == kEpiResidual) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 r4 = rv[q];
      v[8 * q + 0] += bf16_lo(r4.x); v[8 * q + 1] += bf16_hi(r4.x);
      v[8 * q + 2] += bf16_lo(r4.y); v[8 * q + 3] += bf16_hi(r4.y);
      v[8 * q + 4] += bf16_lo(r4.z); v[8 * q + 5] += bf16_hi(r4.z);
      v[8 * q + 6] += bf16_lo(r4.w); v[8 * q + 7] += bf16_hi(r4.w);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    o[q].x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    o[q].y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    o[q].z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    o[q].w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
  }
  if constexpr ((EPI & kEpiStats) != 0) {
    if (valid) {
      // statistics of the values as stored: the next GEMM multiplies these
      float w[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        w[8 * q + 0] = bf16_lo(o[q].x); w[8 * q + 1] = bf16_hi(o[q].x);
        w[8 * q + 2] = bf16_lo(o[q].y); w[8 * q + 3] = bf16_hi(o[q].y);
        w[8 * q + 4] = bf16_lo(o[q].z); w[8 * q + 5] = bf16_hi(o[q].z);
        w[8 * q + 6] = bf16_lo(o[q].w); w[8 * q + 7] = bf16_hi(o[q].w);
      }
      const int nq = min(4, (N - col0) >> 3);  // valid 8-column groups (>= 1)
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq)
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += w[8 * q + e];
      const float nb = float(8 * nq);
      const float mb = sum / nb;
      float m2 = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float d = w[8 * q + e] - mb;
            m2 = fmaf(d, d, m2);
          }
      rs.merge(nb, mb, m2);
    }
  }
}

// Stages one warp's 32 x 32 chunk (thread = row `lane`, 64 bytes each) in
// its 64-byte-swizzled buffer and stores it with one TMA copy at (col0,
// row0); rows past M and columns past N are not written.  The buffer is
// reused only after the previous copy has read it.
__device__ __forceinline__ void stage_store_chunk(uint8_t *buf, const CUtensorMap *tm_y,
                                                  const uint4 (&o)[4], int lane, int col0,
                                                  int row0, bool any) {
  if (lane == 0) bulk_wait_group_read<0>();
  __syncwarp();
  uint8_t *rowp = buf + lane * 64;
  const int sw = (lane >> 1) & 3;  // 64-byte swizzle: 16-byte unit u ^ ((row >> 1) & 3)
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4 *>(rowp + ((q ^ sw) << 4)) = o[q];
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && any) {
    tma_store_2d(tm_y, buf, col0, row0);
    bulk_commit_group();
  }
}

// kEpiQuant: one thread's 32-column chunk of row `row` (bf16 values o) as
// one MXFP8 group -- X = floor(log2 amax) - 8 clamped to [-127, 127], E4M3
// codes of x 2^-X (nearest even, saturating) -- codes to ea.y viewed as
// bytes, the scale byte into ea.q_scales' 512-byte blocks.  Threads of the
// blocks' padding (rows past M, groups past N inside the last 128-column
// block) write the padding scale 127.
__device__ __forceinline__ void quant_store_chunk(const uint4 (&o)[4], const EpiArgs &ea, int row,
                                                  int M, int col0, int N) {
  if (row >= (M + 127) / 128 * 128 || col0 >= (N + 127) / 128 * 128) return;
  const int g = col0 >> 5, rr = row & 127;
  uint8_t &sc = ea.q_scales[(size_t(row >> 7) * ea.q_kblocks + (g >> 2)) * 512 + (rr & 31) * 16 +
                            (rr >> 5) * 4 + (g & 3)];
  if (row >= M || col0 >= N) {
    sc = 127;
    return;
  }
  const int n = min(32, N - col0);
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {o[q].x, o[q].y, o[q].z, o[q].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e] = bf16_lo(w[e]);
      v[8 * q + 2 * e + 1] = bf16_hi(w[e]);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, i < n ? fabsf(v[i]) : 0.f);
  const int ef = int(__float_as_uint(amax) >> 23) & 0xFF;
  const int X = ef == 0 ? -127 : min(max(ef - 127 - 8, -127), 127);
  const float inv = __uint_as_float(uint32_t(127 - X) << 23);
  uint32_t packed[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * q] * inv, v[4 * q + 1] * inv),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(v[4 * q + 2] * inv, v[4 * q + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    packed[q] = (lo & 0xFFFFu) | ((hi & 0xFFFFu) << 16);
  }
  uint8_t *cr = reinterpret_cast<uint8_t *>(ea.y) + size_t(row) * ea.q_row_bytes + col0;
  if (n == 32) {  // q_row_bytes % 16 == 0 and col0 % 32 == 0: 16-byte aligned
    reinterpret_cast<uint4 *>(cr)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    reinterpret_cast<uint4 *>(cr)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  } else {
    for (int i = 0; i < n; ++i) cr[i] = uint8_t(packed[i >> 2] >> (8 * (i & 3)));
  }
  sc = uint8_t(X + 127);
}

// Epilogue of one accumulator (one output tile) by the 8 epilogue warps:
// epilogue warp e (= warp - 2) drains TMEM lane quarter (warp & 3), i.e. one
// row per thread (rows row0 .. row0 + 31 of the warp), and column half
// (e >> 2) of the tile.  The warp's half of the tile bias was staged in its
// shared-memory slot (bias_w).  mu / rstd: the row's LayerNorm statistics
// (kEpiLn), s and c in the warp's ln_slot.  STAGED: results go through the
// warp's staging buffer `ebuf` and TMA stores (tensor map tm_y); otherwise
// each thread stores its row directly.
template <int BN, int EPI, int TS = BN, bool STAGED = true>
__device__ __forceinline__ void epilogue_tile(uint32_t tmem_acc, int warp, int lane, int row,
                                              int M, int n0, int N, const RopeEpi &re,
                                              const __nv_bfloat16 *bias_w, const EpiArgs &ea,
                                              float mu, float rstd, const float *ln_slot,
                                              uint8_t *ebuf, const CUtensorMap *tm_y) {
  constexpr int kChunks = BN / 64;  // 32-column chunks per half
  constexpr int OP = EPI & kEpiOpMask;
  const int quarter = warp & 3, half = (warp - 2) >> 2;
  const bool row_ok = row < M;
  const int row0 = row - lane;  // the warp's first row
  __nv_bfloat16 *__restrict__ y = ea.y;
  if constexpr (OP == kEpiRope) {
    // whole heads: the tile holds HPT heads of HD columns (TS = HPT * HD;
    // the MMA width BN may round TS up); warp `half` of a lane quarter takes
    // heads half, half + 2, ...: bias (or the folded LayerNorm), then the 2D
    // rotation of Q/K pairs (j, j + HD/4) in each half of the head, in fp32
    constexpr int HPT = TS == 216 ? 3 : 2, HD = TS / HPT, Q4 = HD / 4, NF = HD / 32;
    static_assert(HPT * HD == TS && TS <= BN, "RoPE tile of whole heads");
#pragma unroll 1
    for (int hh = half; hh < HPT; hh += 2) {
      const int col0 = n0 + hh * HD;
      const uint32_t base = tmem_acc + (uint32_t(quarter * 32) << 16) + uint32_t(hh * HD);
      uint32_t r[NF][32];
      uint32_t r8[8];
      __syncwarp();
#pragma unroll
      for (int c = 0; c < NF; ++c) tmem_ld32(base + c * 32, r[c]);
      if (HD % 32) tmem_ld8(base + NF * 32, r8);
      tmem_ld_wait();
      const bool valid = row_ok && col0 < N;
      float v[HD];
#pragma unroll
      for (int i = 0; i < HD; ++i) {
        const uint32_t bits = i < NF * 32 ? r[i / 32][i % 32] : r8[i - NF * 32];
        v[i] = __uint_as_float(bits);
      }
      if constexpr ((EPI & kEpiLn) != 0) {
        // the head's s and c, staged in the warp's slot (the k-th head of the
        // warp at k * 2 HD: s, then c)
        const float4 *sp = reinterpret_cast<const float4 *>(ln_slot + (hh >> 1) * 2 * HD);
        const float4 *cp = sp + HD / 4;
#pragma unroll
        for (int u = 0; u < HD / 4; ++u) {
          const float4 s4 = sp[u], c4 = cp[u];
          v[4 * u + 0] = fmaf(rstd, fmaf(-mu, s4.x, v[4 * u + 0]), c4.x);
          v[4 * u + 1] = fmaf(rstd, fmaf(-mu, s4.y, v[4 * u + 1]), c4.y);
          v[4 * u + 2] = fmaf(rstd, fmaf(-mu, s4.z, v[4 * u + 2]), c4.z);
          v[4 * u + 3] = fmaf(rstd, fmaf(-mu, s4.w, v[4 * u + 3]), c4.w);
        }
      } else if (ea.bias != nullptr && col0 < N) {  // the head's bias (broadcast loads)
        const uint4 *bp = reinterpret_cast<const uint4 *>(ea.bias + col0);
#pragma unroll
        for (int u = 0; u < HD / 8; ++u) {
          const uint4 b4 = __ldg(bp + u);
          const uint32_t bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[8 * u + 2 * e] += bf16_lo(bb[e]);
            v[8 * u + 2 * e + 1] += bf16_hi(bb[e]);
          }
        }
      }
      if (valid && col0 < re.rot_cols) {
        const int2 pr = reinterpret_cast<const int2 *>(re.pos)[row];
#pragma unroll
        for (int axis = 0; axis < 2; ++axis) {
          const float p = float(axis == 0 ? pr.x : pr.y);
#pragma unroll
          for (int j = 0; j < Q4; ++j) {
            float sn, cs;
            sincospif(p * re.fr.wpi[j], &sn, &cs);
            const float a = v[axis * (HD / 2) + j], b = v[axis * (HD / 2) + Q4 + j];
            v[axis * (HD / 2) + j] = a * cs - b * sn;
            v[axis * (HD / 2) + Q4 + j] = b * cs + a * sn;
          }
        }
      }
      if constexpr (STAGED) {
        // one head of the warp's 32 rows through the staging buffer
        // (unswizzled rows of HD columns), then one TMA copy
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        uint4 *rowp = reinterpret_cast<uint4 *>(ebuf + lane * (HD * 2));
#pragma unroll
        for (int u = 0; u < HD / 8; ++u)
          rowp[u] = make_uint4(pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                               pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                               pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                               pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < M && col0 < N) {
          tma_store_2d(tm_y, ebuf, col0, row0);
          bulk_commit_group();
        }
      } else if (valid) {
        uint4 *yp = reinterpret_cast<uint4 *>(y + size_t(row) * N + col0);
#pragma unroll
        for (int u = 0; u < HD / 8; ++u)
          yp[u] = make_uint4(pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                             pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                             pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                             pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
      }
    }
  } else {
    RunStats rs;
#pragma unroll 1
    for (int i = 0; i < kChunks; ++i) {
      const int c = half * kChunks + i;
      const int col0 = n0 + c * 32;
      const bool ok = row_ok && col0 < N;
      uint32_t r[32];
      __syncwarp();
      tmem_ld32(tmem_acc + (uint32_t(quarter * 32) << 16) + uint32_t(c * 32), r);
      // operands of the epilogue, in flight together with the TMEM load
      uint4 rv[4] = {};
      if (OP == kEpiResidual && ok) {
        const uint4 *rp = reinterpret_cast<const uint4 *>(ea.res + size_t(row) * N + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) rv[q] = (col0 + 8 * q < N) ? __ldg(rp + q) : make_uint4(0, 0, 0, 0);
      }
      float4 sv[8], cv[8];
      if constexpr ((EPI & kEpiLn) != 0) {  // this chunk's s and c from the warp's slot
        const float4 *sp = reinterpret_cast<const float4 *>(ln_slot + i * 32);
        const float4 *cp = reinterpret_cast<const float4 *>(ln_slot + BN / 2 + i * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          sv[q] = sp[q];
          cv[q] = cp[q];
        }
      }
      tmem_ld_wait();
      uint4 o[4];
      compute_chunk<EPI>(r, col0, N, ok, bias_w + i * 32, rv, sv, cv, mu, rstd, o, rs);
      if constexpr ((EPI & kEpiQuant) != 0) {
        quant_store_chunk(o, ea, row, M, col0, N);
      } else if constexpr (STAGED) {
        stage_store_chunk(ebuf, tm_y, o, lane, col0, row0, row0 < M && col0 < N);
      } else if (ok) {
        uint4 *yp = reinterpret_cast<uint4 *>(y + size_t(row) * N + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (col0 + 8 * q < N) yp[q] = o[q];
      }
    }
    if constexpr ((EPI & kEpiStats) != 0) {
      // this warp's slice of the row: columns [n0 + half BN/2, + BN/2)
      const int c0 = n0 + half * (BN / 2);
      if (row_ok && c0 < N)
        ea.stats_out.p[size_t(row) * ea.stats_out.parts + c0 / (BN / 2)] = make_float2(rs.mean, rs.m2);
    }
  }
}

// Each epilogue warp stages the bias of its own column half of the tile
// [n0 + half*BN/2, n0 + (half+1)*BN/2) in its own shared-memory slot (zeros
// past N or without bias).  Only the warp itself reads the slot, so warp-level
// synchronisation suffices (no barrier across epilogue warps, which could not
// be left safely if a bounded wait ran out).
template <int BN>
__device__ __forceinline__ void stage_bias_warp(__nv_bfloat16 *bias_w, const __nv_bfloat16 *bias,
                                                int n0, int N, int warp, int lane) {
  const int half = (warp - 2) >> 2;
  __syncwarp();  // previous tile's reads of the slot are done
  if (lane < BN / 16) {
    const int col = n0 + half * (BN / 2) + lane * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (bias != nullptr && col < N) v = __ldg(reinterpret_cast<const uint4 *>(bias + col));
    reinterpret_cast<uint4 *>(bias_w)[lane] = v;
  }
  __syncwarp();
}

template <int BN, int EPI>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ EpiArgs ea,
                   int M, int N, int K, int *status, const __grid_constant__ RopeEpi re,
                   uint32_t lost_tx) {
  using namespace gemm;
  using CF = Cfg<BN, EPI, BN, false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + size_t(CF::kStages) * CF::kStageBytes);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int k_blocks = (K + BK - 1) / BK;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kEpiWarps);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, CF::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_wait();  // inputs of this GEMM are written by the previous kernel

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
          // lost_tx > 0 only under fault injection (vit_debug_lost_tx): the
          // stage then waits for bytes no copy delivers, and the bounded
          // waits end the kernel with VIT_ERR_TIMEOUT
          mbar_arrive_expect_tx(&bars->full[stage], CF::kStageBytes + lost_tx);
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
    const int row_in_tile = (warp & 3) * 32 + lane;
    __nv_bfloat16 *bias_w = reinterpret_cast<__nv_bfloat16 *>(bars + 1) + (warp - 2) * 128;
    int it = 0;
    float *ln_slot = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + kLnSlotsOffset +
                                               (warp - 2) * kLnSlotBytes);
    uint8_t *ebuf = reinterpret_cast<uint8_t *>(bars) + CF::ES::kBufOff + (warp - 2) * CF::ES::kBufBytes;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int a = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      const int row = mb * BM + row_in_tile;
      float mu = 0.f, rstd = 0.f;  // LayerNorm statistics of the row (kEpiLn)
      if constexpr ((EPI & kEpiLn) != 0) {
        __syncwarp();  // the previous tile's reads of the slot are done
        const int c0[1] = {nb * BN + ((warp - 2) >> 2) * (BN / 2)};
        stage_ln_cols<1, (BN / 2 / 4 + 31) / 32>(ln_slot, ea, c0, 1, BN / 2, N, lane);
        if (row < M) ln_row_stats(ea, row, K, mu, rstd);
        __syncwarp();
      } else {
        stage_bias_warp<BN>(bias_w, ea.bias, nb * BN, N, warp, lane);
      }
      if (!mbar_wait(&bars->acc_full[a], aphase, abort_flag)) break;
      tc_fence_after();
      epilogue_tile<BN, EPI>(tmem + uint32_t(a * BN), warp, lane, row, M, nb * BN, N, re,
                             bias_w, ea, mu, rstd, ln_slot, ebuf, &tmY);
      tc_fence_before();
      __syncwarp();
      // the accumulator's TMEM reads are complete (tcgen05.wait::ld): a
      // relaxed arrival, which does not wait for the tile's stores
      if (lane == 0) mbar_arrive_relaxed(&bars->acc_empty[a]);
    }
    if (lane == 0) bulk_wait_group<0>();  // the TMA stores have completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, CF::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report_status(status, kDevTimeout);
}

// ---------------------------------------------------------------- CTA-pair GEMM
// The same GEMM with 256-row output tiles computed by a pair of CTAs (a
// cluster of 2 on two SMs) through tcgen05.mma.cta_group::2: each CTA loads
// its own 128 rows of x and half of the tile's BN rows of w, the leader CTA
// (rank 0) issues one M = 256 MMA that reads both CTAs' shared memory, and
// each CTA's TMEM receives its 128 output rows.  Per SM this halves the w
// bytes per FLOP compared with a 128 x BN tile on one SM.
//   - full[s] lives in the leader and counts both CTAs' TMA bytes;
//   - empty[s] and acc_full[a] are signalled in both CTAs by one multicast
//     tcgen05.commit of the leader;
//   - acc_empty[a] lives in the leader and collects the 8 epilogue warps of
//     both CTAs (remote arrivals from the peer).
// No load uses cluster multicast.
template <int BN, int EPI, int TS = BN>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ EpiArgs ea,
                    int M, int N, int K, int *status, const __grid_constant__ RopeEpi re) {
  using namespace gemm;
  using CF = Cfg<BN, EPI, TS, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + size_t(CF::kStages) * CF::kStageBytes);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  // tiles step TS columns (TS <= BN, the MMA width: a RoPE tile of three
  // 72-wide heads computes 224 columns and keeps 216)
  const int num_m = (M + 2 * BM - 1) / (2 * BM), num_n = (N + TS - 1) / TS;
  const int num_tiles = num_m * num_n;
  const int k_blocks = (K + BK - 1) / BK;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], 2 * kEpiWarps);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars->tmem_base, CF::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_wait();  // inputs of this GEMM are written by the previous kernel

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t *sa = smem + size_t(stage) * CF::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&bars->full[stage], 2 * CF::kStageBytes);
          const uint32_t full_leader = map_to_cta(&bars->full[stage], 0);
          tma_load_2d_pair(sa, &tmA, full_leader, kb * BK, mb * 2 * BM + int(rank) * BM);
          tma_load_2d_pair(sa + kATileBytes, &tmB, full_leader, kb * BK,
                           nb * TS + int(rank) * (BN / 2));
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        if (leader) {
          for (int s = 0; s < CF::kStages; ++s)
            if (issued_mask & (1u << s)) drain_wait(&bars->full[s], (issued_parity >> s) & 1);
        } else {
          // the peer's copies complete on the leader's barriers: give them time
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 2000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true, any_mma = false;
      for (int tile = pair; tile < num_tiles && ok; tile += n_pairs, ++it) {
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
            mma_bf16_ss_pair(d_tmem, ad, bd, CF::kIdesc, (kb | k) != 0);
          }
          any_mma = true;
          mma_commit_pair_mc(&bars->empty[stage], 0x3);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair_mc(&bars->acc_full[a], 0x3);
      }
      if (!ok && any_mma) {
        mma_commit_pair_mc(&bars->drain, 0x1);
        drain_wait(&bars->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int row_in_tile = int(rank) * BM + (warp & 3) * 32 + lane;
    __nv_bfloat16 *bias_w = reinterpret_cast<__nv_bfloat16 *>(bars + 1) + (warp - 2) * 128;
    int it = 0;
    float *ln_slot = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + kLnSlotsOffset +
                                               (warp - 2) * kLnSlotBytes);
    uint8_t *ebuf = reinterpret_cast<uint8_t *>(bars) + CF::ES::kBufOff + (warp - 2) * CF::ES::kBufBytes;
    for (int tile = pair; tile < num_tiles; tile += n_pairs, ++it) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int a = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      const int row = mb * 2 * BM + row_in_tile;
      float mu = 0.f, rstd = 0.f;  // LayerNorm statistics of the row (kEpiLn)
      if constexpr ((EPI & kEpiLn) != 0) {
        __syncwarp();  // the previous tile's reads of the slot are done
        const int half = (warp - 2) >> 2;
        if constexpr ((EPI & kEpiOpMask) == kEpiRope) {
          // the warp's heads half, half + 2, ... of the tile, each [s HD | c HD]
          constexpr int HPT = TS == 216 ? 3 : 2, HD = TS / HPT;
          constexpr int NSEG = (HPT + 1) / 2;
          int c0[NSEG];
#pragma unroll
          for (int k = 0; k < NSEG; ++k) c0[k] = nb * TS + (half + 2 * k) * HD;
          stage_ln_cols<NSEG, (HD / 4 + 31) / 32>(ln_slot, ea, c0, (HPT - half + 1) / 2, HD, N,
                                                  lane);
        } else {
          const int c0[1] = {nb * TS + half * (BN / 2)};
          stage_ln_cols<1, (BN / 2 / 4 + 31) / 32>(ln_slot, ea, c0, 1, BN / 2, N, lane);
        }
        if (row < M) ln_row_stats(ea, row, K, mu, rstd);
        __syncwarp();
      } else if constexpr ((EPI & kEpiOpMask) != kEpiRope) {
        stage_bias_warp<BN>(bias_w, ea.bias, nb * TS, N, warp, lane);
      }
      if (!mbar_wait(&bars->acc_full[a], aphase, abort_flag)) break;
      tc_fence_after();
      epilogue_tile<BN, EPI, TS>(tmem + uint32_t(a * BN), warp, lane, row, M, nb * TS, N, re,
                                 bias_w, ea, mu, rstd, ln_slot, ebuf, &tmY);
      tc_fence_before();
      __syncwarp();
      // the accumulator's TMEM reads are complete (tcgen05.wait::ld): a
      // relaxed arrival, which does not wait for the tile's stores
      if (lane == 0) mbar_arrive_cluster_relaxed(map_to_cta(&bars->acc_empty[a], 0));
    }
    if (lane == 0) bulk_wait_group<0>();  // the TMA stores have completed
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while the pair's MMAs may still read its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, CF::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report_status(status, kDevTimeout);
}

// ---------------------------------------------------------------- host side
constexpr int kMaxDevices = 64;  // per-device caches of launch properties

// cuTensorMapEncodeTiled, resolved once per process (thread-safe static init)
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                              uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
                              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int BN, int EPI>
static cudaError_t launch_bn(const CUtensorMap &ta, const CUtensorMap &tb,
                             const CUtensorMap &ty, const EpiArgs &ea,
                             int M, int N, int K, int num_sms, int *status, cudaStream_t st,
                             const RopeEpi &re, uint32_t lost_tx) {
  using CF = gemm::Cfg<BN, EPI, BN, false>;
  auto kern = gemm_tc_kernel<BN, EPI>;
  const size_t smem = CF::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + BN - 1) / BN);
  const int grid = std::max(1, std::min(tiles, num_sms));
  return launch_pdl(kern, dim3(grid), dim3(gemm::kThreads), smem, st, 1, ta, tb, ty, ea, M, N, K,
                    status, re, lost_tx);
}

// the epilogue combinations the library launches: plain bias, GELU and
// residual; LayerNorm folded into bias or GELU; residual with row statistics
template <int BN>
static cudaError_t launch_epi(int epi, const CUtensorMap &ta, const CUtensorMap &tb,
                             const CUtensorMap &ty,
                              const EpiArgs &ea, int M, int N, int K, int num_sms, int *status,
                              cudaStream_t st, uint32_t lost_tx) {
  const RopeEpi none{};
  switch (epi) {
    case kEpiBias:
      return launch_bn<BN, kEpiBias>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none, lost_tx);
    case kEpiGelu:
      return launch_bn<BN, kEpiGelu>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none, lost_tx);
    case kEpiResidual:
      return launch_bn<BN, kEpiResidual>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none, lost_tx);
    case kEpiBias | kEpiLn:
      return launch_bn<BN, kEpiBias | kEpiLn>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none,
                                              lost_tx);
    case kEpiGelu | kEpiLn:
      return launch_bn<BN, kEpiGelu | kEpiLn>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none,
                                              lost_tx);
    case kEpiResidual | kEpiStats:
      return launch_bn<BN, kEpiResidual | kEpiStats>(ta, tb, ty, ea, M, N, K, num_sms, status, st,
                                                     none, lost_tx);
    default:
      return cudaErrorInvalidValue;
  }
}

template <int BN, int EPI, int TS = BN>
static cudaError_t launch_pair(const CUtensorMap &ta, const CUtensorMap &tb,
                             const CUtensorMap &ty, const EpiArgs &ea,
                               int M, int N, int K, int num_sms, int *status, cudaStream_t st,
                               const RopeEpi &re) {
  using CF = gemm::Cfg<BN, EPI, TS, true>;
  auto kern = gemm_tc2_kernel<BN, EPI, TS>;
  const size_t smem = CF::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // SM pairs that can hold one CTA pair each (clusters live inside a GPC),
  // queried once per device and kernel (0 = not yet known; concurrent first
  // calls compute the same value)
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  int max_clusters = dev < kMaxDevices ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (max_clusters <= 0) {
    cfg.gridDim = dim3(2 * (num_sms / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_clusters = n;
    if (dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
  }
  const int tiles = ((M + 2 * gemm::BM - 1) / (2 * gemm::BM)) * ((N + TS - 1) / TS);
  return launch_pdl(kern, dim3(2 * std::max(1, std::min(tiles, max_clusters))),
                    dim3(gemm::kThreads), smem, st, 2, ta, tb, ty, ea, M, N, K, status, re);
}

template <int BN>
static cudaError_t launch_pair_epi(int epi, const CUtensorMap &ta, const CUtensorMap &tb,
                             const CUtensorMap &ty,
                                   const EpiArgs &ea, int M, int N, int K, int num_sms,
                                   int *status, cudaStream_t st) {
  const RopeEpi none{};
  switch (epi) {
    case kEpiBias:
      return launch_pair<BN, kEpiBias>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none);
    case kEpiGelu:
      return launch_pair<BN, kEpiGelu>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none);
    case kEpiResidual:
      return launch_pair<BN, kEpiResidual>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none);
    case kEpiBias | kEpiLn:
      return launch_pair<BN, kEpiBias | kEpiLn>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none);
    case kEpiGelu | kEpiLn:
      return launch_pair<BN, kEpiGelu | kEpiLn>(ta, tb, ty, ea, M, N, K, num_sms, status, st, none);
    case kEpiResidual | kEpiStats:
      return launch_pair<BN, kEpiResidual | kEpiStats>(ta, tb, ty, ea, M, N, K, num_sms, status, st,
                                                       none);
    default:
      return cudaErrorInvalidValue;
  }
}

// GEMM variant = (CTAs per MMA, tile width).  Cost model: output tiles are
// processed in rounds over the SMs (or SM pairs); per 64-deep k-block an SM
// spends max(MMA clocks, operand bytes / kIngestBytesPerClk).  The per-SM
// operand ingest rate is the measured limiter of these GEMMs (their tensor
// pipe idles while shared memory waits for TMA data), so the pair variant,
// which loads half of w per SM, usually wins.
struct GemmVariant {
  int pair, bn;
};
constexpr double kIngestBytesPerClk = 45.0;

static GemmVariant choose_variant(int M, int N, int K, int num_sms) {
  if (const char *f = getenv("VIT_GEMM_TILE")) {  // e.g. "2x192": tuning and tests
    int p = 0, bn = 0;
    if (sscanf(f, "%dx%d", &p, &bn) == 2 && (p == 1 || p == 2) &&
        (bn == 128 || bn == 256 || (p == 2 && bn == 192)))
      return {p, bn};
  }
  const GemmVariant cands[5] = {{1, 128}, {1, 256}, {2, 128}, {2, 192}, {2, 256}};
  const int kb = (K + gemm::BK - 1) / gemm::BK;
  double best = -1;
  GemmVariant pick = {1, 128};
  for (const auto &v : cands) {
    if (v.pair == 2 && M <= gemm::BM) continue;  // a single row tile: no pair to share
    const long tiles = long((M + v.pair * gemm::BM - 1) / (v.pair * gemm::BM)) *
                       ((N + v.bn - 1) / v.bn);
    const long units = num_sms / v.pair;
    const long rounds = (tiles + units - 1) / units;
    const double mma = 2.0 * v.bn;
    const double ingest = (16384.0 + 128.0 * v.bn / v.pair) / kIngestBytesPerClk;
    const double cost = double(rounds) * kb * std::max(mma, ingest);
    if (best < 0 || cost < best) { best = cost; pick = v; }
  }
  return pick;
}

int gemm_stats_width(int M, int N, int K, int num_sms) {
  return choose_variant(M, N, K, num_sms).bn / 2;
}

cudaError_t launch_gemm_tc(const void *x, const void *w, const EpiArgs &ea, int M, int N, int K,
                           int epi, int num_sms, cudaStream_t st, int *status,
                           const RopeEpi *rope, uint32_t lost_tx) {
  if (M == 0 || N == 0) return cudaSuccess;
  GemmVariant v = choose_variant(M, N, K, num_sms);
  const int op = epi & kEpiOpMask;
  if (op == kEpiRope) {  // tiles of whole heads on a CTA pair: 3 x 72 (MMA N = 224) or 2 x 128
    if (rope == nullptr || (rope->head_dim != 72 && rope->head_dim != 128) || (epi & kEpiStats))
      return cudaErrorInvalidValue;
    v = {2, rope->head_dim == 72 ? 224 : 256};
  }
  if ((epi & kEpiStats) && (ea.stats_out.p == nullptr || ea.stats_out.w != v.bn / 2 ||
                            ea.stats_out.parts != (N + v.bn / 2 - 1) / (v.bn / 2)))
    return cudaErrorInvalidValue;
  if ((epi & kEpiLn) && (ea.ln_sc == nullptr || ea.stats_in.p == nullptr || ea.stats_in.w <= 0 ||
                         ea.stats_in.parts != (K + ea.stats_in.w - 1) / ea.stats_in.w))
    return cudaErrorInvalidValue;
  const int b_rows = v.pair == 2 ? v.bn / 2 : v.bn;
  CUtensorMap ta, tb, ty;
  // output stores: 32-row boxes of 32 columns (64-byte swizzled staging) or,
  // for RoPE tiles, of one head
  if (op == kEpiRope) {
    if (encode_tensor_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ea.y, N, M, uint64_t(N) * 2,
                             rope->head_dim, 32, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else if (encode_tensor_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ea.y, N, M,
                                  uint64_t(N) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B) !=
             CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  if (encode_tensor_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, uint64_t(K) * 2,
                           gemm::BK, gemm::BM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, uint64_t(K) * 2,
                           gemm::BK, b_rows, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (op == kEpiRope) {
    const bool ln = (epi & kEpiLn) != 0;
    if (v.bn == 224)
      return ln ? launch_pair<224, kEpiRope | kEpiLn, 216>(ta, tb, ty, ea, M, N, K, num_sms, status, st,
                                                           *rope)
                : launch_pair<224, kEpiRope, 216>(ta, tb, ty, ea, M, N, K, num_sms, status, st, *rope);
    return ln ? launch_pair<256, kEpiRope | kEpiLn, 256>(ta, tb, ty, ea, M, N, K, num_sms, status, st,
                                                         *rope)
              : launch_pair<256, kEpiRope, 256>(ta, tb, ty, ea, M, N, K, num_sms, status, st, *rope);
  }
  if (v.pair == 2) {
    if (v.bn == 256) return launch_pair_epi<256>(epi, ta, tb, ty, ea, M, N, K, num_sms, status, st);
    if (v.bn == 192) return launch_pair_epi<192>(epi, ta, tb, ty, ea, M, N, K, num_sms, status, st);
    return launch_pair_epi<128>(epi, ta, tb, ty, ea, M, N, K, num_sms, status, st);
  }
  if (v.bn == 256)
    return launch_epi<256>(epi, ta, tb, ty, ea, M, N, K, num_sms, status, st, lost_tx);
  return launch_epi<128>(epi, ta, tb, ty, ea, M, N, K, num_sms, status, st, lost_tx);
}

// ---------------------------------------------------------------- MXFP8 GEMM
// The same persistent structure as gemm_tc_kernel with E4M3 operands and E8M0
// block scales (OCP Microscaling v1.0): per 128-column k-block, the producer
// brings a 128x128-byte tile of A codes and a BNx128 tile of W codes (the
// same 128-byte swizzle atom as 64 bf16), plus the 512-byte scale blocks of
// A's 128 rows and W's BN rows.  The MMA lane copies the scale blocks into
// TMEM (tcgen05.cp, one copy per 128 rows), then issues four K = 32 block-
// scaled MMAs; MMA k reads byte k of each row's scale word.  The scale
// columns are rewritten every k-block: the tensor core runs copies and MMAs
// of one thread in issue order.
namespace gemm {
constexpr int kMxBK = 128;                      // E4M3 elements (bytes) per k-block
constexpr uint32_t kMxATileBytes = BM * kMxBK;  // 16 KB
constexpr uint32_t kMxSfBlock = 512;            // scales of 128 rows x 128 columns
template <int BN>
struct CfgMx {
  static constexpr uint32_t kBTileBytes = BN * kMxBK;
  static constexpr int kSfbBlocks = BN / 128;
  static constexpr uint32_t kSfOff = kMxATileBytes + kBTileBytes;
  static constexpr uint32_t kStageBytes = kSfOff + kMxSfBlock * (1 + kSfbBlocks);
  static constexpr int kStages = 6;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSfaCol = 2 * BN;      // 4 columns
  static constexpr uint32_t kSfbCol = 2 * BN + 4;  // 4 columns per 128 rows of W
  // ring + 1 KB alignment slack + barriers and bias slots (3 KB) + the
  // epilogue warps' 2 KB output staging buffers
  static constexpr uint32_t kBufOff = 3072;
  static constexpr size_t kSmemBytes =
      size_t(kStages) * kStageBytes + 1024 + kBufOff + kEpiWarps * 2048;
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1 KB alignment of the swizzled tiles");
  static_assert(kSfbCol + 4 * kSfbBlocks <= kTmemCols, "TMEM columns");
  static_assert(kStages <= 8, "barrier slots");
};
}  // namespace gemm

template <int BN, int EPI>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gemm_mx8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const uint8_t *__restrict__ sfa,
                    const uint8_t *__restrict__ sfb, const __grid_constant__ EpiArgs ea, int M,
                    int N, int K, int *status) {
  using namespace gemm;
  using CF = CfgMx<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + size_t(CF::kStages) * CF::kStageBytes);
  volatile int *abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int k_blocks = (K + kMxBK - 1) / kMxBK;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kEpiWarps);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, CF::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t *sa = smem + size_t(stage) * CF::kStageBytes;
          mbar_arrive_expect_tx(&bars->full[stage], CF::kStageBytes);
          tma_load_2d(sa, &tmA, &bars->full[stage], kb * kMxBK, mb * BM);
          tma_load_2d(sa + kMxATileBytes, &tmB, &bars->full[stage], kb * kMxBK, nb * BN);
          bulk_load(sa + CF::kSfOff, sfa + (size_t(mb) * k_blocks + kb) * kMxSfBlock, kMxSfBlock,
                    &bars->full[stage]);
#pragma unroll
          for (int i = 0; i < CF::kSfbBlocks; ++i)
            bulk_load(sa + CF::kSfOff + kMxSfBlock * (1 + i),
                      sfb + (size_t(nb * CF::kSfbBlocks + i) * k_blocks + kb) * kMxSfBlock,
                      kMxSfBlock, &bars->full[stage]);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
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
      const uint32_t sfa_t = tmem + CF::kSfaCol, sfb_t = tmem + CF::kSfbCol;
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
          const uint32_t sb = sa + kMxATileBytes;
          const uint32_t ssf = sa + CF::kSfOff;
          tmem_cp_32x128b_x4(sfa_t, smem_desc(ssf, 0, 128, 0));
#pragma unroll
          for (int i = 0; i < CF::kSfbBlocks; ++i)
            tmem_cp_32x128b_x4(sfb_t + 4 * i, smem_desc(ssf + kMxSfBlock * (1 + i), 0, 128, 0));
#pragma unroll
          for (int k = 0; k < kMxBK / 32; ++k) {
            const uint64_t ad = smem_desc(sa + k * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(sb + k * 32, 16, 1024, 2);
            mma_mx8_ss(d_tmem, ad, bd, idesc_mx8(BM, BN, k, k), sfa_t | (uint32_t(k) << 30),
                       sfb_t | (uint32_t(k) << 30), (kb | k) != 0);
          }
          any_mma = true;
          mma_commit(&bars->empty[stage]);
          if (++stage == CF::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&bars->acc_full[a]);
      }
      if (!ok && any_mma) {
        mma_commit(&bars->drain);
        drain_wait(&bars->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int row_in_tile = (warp & 3) * 32 + lane;
    __nv_bfloat16 *bias_w = reinterpret_cast<__nv_bfloat16 *>(bars + 1) + (warp - 2) * 128;
    uint8_t *ebuf = reinterpret_cast<uint8_t *>(bars) + CF::kBufOff + (warp - 2) * 2048;
    const RopeEpi none{};
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int a = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      stage_bias_warp<BN>(bias_w, ea.bias, nb * BN, N, warp, lane);
      if (!mbar_wait(&bars->acc_full[a], aphase, abort_flag)) break;
      tc_fence_after();
      const int row = mb * BM + row_in_tile;
      epilogue_tile<BN, EPI>(tmem + uint32_t(a * BN), warp, lane, row, M, nb * BN, N, none,
                             bias_w, ea, 0.f, 0.f, nullptr, ebuf, &tmY);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&bars->acc_empty[a]);  // TMEM reads complete
    }
    if (lane == 0) bulk_wait_group<0>();  // the TMA stores have completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, CF::kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report_status(status, kDevTimeout);
}

template <int BN, int EPI>
static cudaError_t launch_mx8_bn(const CUtensorMap &ta, const CUtensorMap &tb,
                                 const CUtensorMap &ty, const uint8_t *sfa,
                                 const uint8_t *sfb, const EpiArgs &ea, int M, int N, int K,
                                 int num_sms, int *status, cudaStream_t st) {
  using CF = gemm::CfgMx<BN>;
  auto kern = gemm_mx8_kernel<BN, EPI>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CF::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + BN - 1) / BN);
  const int grid = std::max(1, std::min(tiles, num_sms));
  return launch_pdl(kern, dim3(grid), dim3(gemm::kThreads), CF::kSmemBytes, st, 1, ta, tb, ty,
                    sfa, sfb, ea, M, N, K, status);
}

cudaError_t launch_gemm_mx8(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *w_codes,
                            const uint8_t *w_scales, const void *b, const void *res, void *y, int M,
                            int N, int K, int epi, int num_sms, int *status, cudaStream_t st,
                            uint8_t *y_scales) {
  if (M == 0 || N == 0) return cudaSuccess;
  constexpr int BN = 128;
  if ((epi & kEpiQuant) && (epi != (kEpiGelu | kEpiQuant) || y_scales == nullptr))
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (encode_tensor_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K, M, mx8_row_bytes(K),
                           gemm::kMxBK, gemm::BM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K, N, mx8_row_bytes(K),
                           gemm::kMxBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  CUtensorMap ty;  // output stores: 32 x 32 boxes, 64-byte swizzled staging
  if (encode_tensor_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, uint64_t(N) * 2, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  EpiArgs ea{};
  ea.bias = static_cast<const __nv_bfloat16 *>(b);
  ea.res = static_cast<const __nv_bfloat16 *>(res);
  ea.y = static_cast<__nv_bfloat16 *>(y);
  ea.q_scales = y_scales;
  ea.q_row_bytes = mx8_row_bytes(N);
  ea.q_kblocks = (N + 127) / 128;
  switch (epi) {
    case kEpiGelu:
      return launch_mx8_bn<BN, kEpiGelu>(ta, tb, ty, a_scales, w_scales, ea, M, N, K, num_sms, status,
                                         st);
    case kEpiGelu | kEpiQuant:
      return launch_mx8_bn<BN, kEpiGelu | kEpiQuant>(ta, tb, ty, a_scales, w_scales, ea, M, N, K,
                                                     num_sms, status, st);
    case kEpiResidual:
      return launch_mx8_bn<BN, kEpiResidual>(ta, tb, ty, a_scales, w_scales, ea, M, N, K, num_sms,
                                             status, st);
    default:
      return launch_mx8_bn<BN, kEpiBias>(ta, tb, ty, a_scales, w_scales, ea, M, N, K, num_sms, status,
                                         st);
  }
}

}  // namespace vit
