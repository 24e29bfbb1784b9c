// k_attn_tc.cu -- bidirectional flash attention on tcgen05 for bf16 packed
// sequences, head_dim 72 or 128, with an optional prefix K/V segment and
// optional 2D RoPE applied to Q and K as they are loaded.
//
// KLiteInfer README, "视觉算子": bidirectional attention over batched tokens,
// done there as two strided-batched SGEMMs around a softmax kernel (the score
// matrix goes through HBM).  Here scores never leave the SM: S = Q K^T is
// accumulated in tensor memory, the softmax runs in registers (one thread per
// query row, online max/sum), P is written back into the same TMEM columns as
// bf16 and consumed as the A operand of O += P V, with O also in TMEM.
// Prefix K/V (LightX2V NeoPP README, "KV file layout": [2, seq, kv_heads, d]
// per layer) is read through its own TMA descriptors as the first key tiles.
//
// CTA = (sequence, head, two 128-row query tiles), 20 warps:
//   0        TMA producer (Q tiles once, then K and V tiles through a ring)
//   1        TMEM allocator; one lane issues all tcgen05.mma
//   2-3      (ROPE only) rotate each own-key K tile in shared memory
//   4-11     softmax of query tile 0, 12-19 of query tile 1: two threads per
//            query row, one per 64-column half of the score row; the pair
//            swaps partial row maxima through shared memory each key tile
// Four softmax warps per SM sub-partition keep the exp unit, the FMA and the
// integer pipes fed while a warp waits on a TMEM load or a barrier.
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,..), O1 [384,..).
// head_dim 72 is computed as 80 (4 MMA k-steps from a 64-column 128B-swizzled
// chunk, 1 from a 16-column 32B-swizzled chunk); Q's columns 72..79 are zeroed
// in shared memory so the neighbouring head's values there contribute 0.
#include "kernels.h"
#include "sm100.cuh"

namespace vit {
namespace attn {

constexpr int kBlockQ = 128;
constexpr int kBlockK = 128;

template <int HD>
struct Cfg {
  static constexpr int HDP = HD == 72 ? 80 : 128;            // padded head_dim
  static constexpr uint32_t kChunk0 = 128 * 128;              // 128 rows x 64 bf16
  static constexpr uint32_t kChunk1 = HD == 72 ? 128 * 32 : 128 * 128;
  static constexpr uint32_t kTile = kChunk0 + kChunk1;        // one operand tile
  static constexpr int kStages = HD == 72 ? 4 : 2;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = 2 * kTile;
  static constexpr uint32_t kVOff = kKOff + kStages * kTile;
  static constexpr uint32_t kBarOff = kVOff + kStages * kTile;
  static constexpr uint32_t kXOff = kBarOff + 512;             // row-max exchange [2][2][128] f32
  static constexpr size_t kSmem = size_t(kXOff) + 2048 + 1024;
  static constexpr uint32_t kTmemS = 0, kTmemO = 256;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, kBlockK, 0, 0);
  static constexpr uint32_t kIdescPV0 = idesc_bf16_f32(128, HD == 72 ? 64 : 128, 0, 1);
  static constexpr uint32_t kIdescPV1 = idesc_bf16_f32(128, 16, 0, 1);
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t q_ready[2];
  uint64_t k_full[4], v_full[4], kv_empty[4], k_ready[4];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t xchg[2][4];  // per (query tile, lane quarter): the 64 threads of a row pair
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");
constexpr int kThreads = 640;

struct Params {
  int H, C, Hkv, P, n_pairs;
  float scale_log2;      // softmax scale * log2(e)
  const int32_t *cu;
  const int32_t *pos;
  __nv_bfloat16 *o;
  int *status;
};

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;
  }
}

// Byte offset of logical 16-byte unit u (0..HDP/8-1) of row r inside an
// operand tile: chunk 0 (units 0..7) is 128B-swizzled, chunk 1 is 32B-swizzled
// (head_dim 72, units 8..9) or 128B-swizzled (head_dim 128, units 8..15).
template <int HD>
__device__ __forceinline__ uint32_t unit_offset(int r, int u) {
  using CF = Cfg<HD>;
  if (u < 8) return uint32_t(r * 128 + ((u ^ (r & 7)) << 4));
  const int v = u - 8;
  if (HD == 72) return CF::kChunk0 + uint32_t(r * 32 + ((v ^ ((r >> 2) & 1)) << 4));
  return CF::kChunk0 + uint32_t(r * 128 + ((v ^ (r & 7)) << 4));
}

// Rotates row r of an operand tile in place by 2D RoPE at position (pr, pc):
// dims [0, HD/2) by pr, [HD/2, HD) by pc; in a half, dim j pairs with j+HD/4.
// fr.wpi[j] = theta^(-2j/(HD/2)) / pi.
template <int HD>
__device__ __forceinline__ void rope_row_smem(uint8_t *tile, int r, int pr, int pc,
                                              const RopeFreqs &fr) {
  constexpr int Q4 = HD / 4;
  // one axis at a time: the 16-byte units holding dims [axis HD/2, axis HD/2 + HD/2)
  // (head_dim 72: unit 4 holds the end of the row half and the start of the
  // column half, and is read back after the first axis wrote it)
#pragma unroll
  for (int axis = 0; axis < 2; ++axis) {
    constexpr int kUnits = (HD / 2 + 7) / 8 + (HD % 16 ? 1 : 0);
    const int u0 = (axis * (HD / 2)) / 8;
    uint32_t w[kUnits * 4];
#pragma unroll
    for (int k = 0; k < kUnits; ++k) {
      if (u0 + k >= HD / 8) continue;
      const uint4 v = *reinterpret_cast<const uint4 *>(tile + unit_offset<HD>(r, u0 + k));
      w[4 * k + 0] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
    }
    const float p = float(axis == 0 ? pr : pc);
#pragma unroll
    for (int j = 0; j < Q4; ++j) {
      const int d1 = axis * (HD / 2) + j - u0 * 8, d2 = d1 + Q4;  // dims relative to unit u0
      float sn, cs;
      sincospif(p * fr.wpi[j], &sn, &cs);
      const uint32_t w1 = w[d1 >> 1], w2 = w[d2 >> 1];
      const float a = (d1 & 1) ? bf16_hi(w1) : bf16_lo(w1);
      const float b = (d2 & 1) ? bf16_hi(w2) : bf16_lo(w2);
      const float a2 = a * cs - b * sn, b2 = b * cs + a * sn;
      const uint32_t ha = __bfloat16_as_ushort(__float2bfloat16_rn(a2));
      const uint32_t hb = __bfloat16_as_ushort(__float2bfloat16_rn(b2));
      w[d1 >> 1] = (d1 & 1) ? ((w1 & 0xFFFFu) | (ha << 16)) : ((w1 & 0xFFFF0000u) | ha);
      const uint32_t w2n = w[d2 >> 1];
      w[d2 >> 1] = (d2 & 1) ? ((w2n & 0xFFFFu) | (hb << 16)) : ((w2n & 0xFFFF0000u) | hb);
    }
#pragma unroll
    for (int k = 0; k < kUnits; ++k) {
      if (u0 + k >= HD / 8) continue;
      *reinterpret_cast<uint4 *>(tile + unit_offset<HD>(r, u0 + k)) =
          make_uint4(w[4 * k + 0], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
  }
}

// A bounded mbarrier wait whose outcome is the same for all 32 lanes (the
// warp-collective TMEM accesses and votes that follow need a converged warp).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Normalises one half of a finished output row (O / l) and stores it as bf16:
// half 0 writes the first ceil(HD/16) 16-byte units of the row, half 1 the
// rest.  head_dim 72 reads l from O column 72 (accumulated by the tensor core);
// head_dim 128 gets it from the caller.  orow == nullptr: load only (row past
// the sequence end; the TMEM loads are warp-collective).
template <int HD, int HALF>
__device__ __forceinline__ void store_o_half(uint32_t o_addr, float l_sum, __nv_bfloat16 *orow) {
  constexpr int NU = HD / 8;
  constexpr int U0 = HALF ? (NU + 1) / 2 : 0, U1 = HALF ? NU : (NU + 1) / 2;
  constexpr int C0 = (U0 * 8) / 16, C1 = (U1 * 8 - 1) / 16;  // 16-column TMEM chunks used
  uint32_t ov[Cfg<HD>::HDP / 16][16];
  __syncwarp();
#pragma unroll
  for (int c = C0; c <= C1; ++c) tmem_ld16(o_addr + c * 16, ov[c]);
  if constexpr (HD == 72 && C1 < 4) tmem_ld16(o_addr + 64, ov[4]);
  tmem_ld_wait();
  float l = l_sum;
  if constexpr (HD == 72) l = __uint_as_float(ov[4][8]);
  const float inv = 1.0f / l;
  const uint64_t inv2 = f2_pack(inv, inv);
  if (orow == nullptr) return;
#pragma unroll
  for (int u = U0; u < U1; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = u * 8 + 2 * e;
      float a, b;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(ov[col / 16][col % 16]),
                               __uint_as_float(ov[col / 16][col % 16 + 1])),
                       inv2),
                a, b);
      w[e] = pack_bf16x2(a, b);
    }
    *reinterpret_cast<uint4 *>(orow + u * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace attn

template <int HD, bool ROPE>
__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_x0,
                        const __grid_constant__ CUtensorMap tm_x1,
                        const __grid_constant__ CUtensorMap tm_p0,
                        const __grid_constant__ CUtensorMap tm_p1, const attn::Params prm,
                        const __grid_constant__ RopeFreqs fr) {
  using namespace attn;
  using CF = Cfg<HD>;
  constexpr int NS = CF::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + CF::kBarOff);
  volatile int *abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_trigger();
  pdl_wait();
  // ---- work item: pairs of query tiles, longest sequences' last pairs first
  const int S = gridDim.x / (prm.n_pairs * prm.H);
  const int b = blockIdx.x;
  const int pair = prm.n_pairs - 1 - b / (prm.H * S);
  const int rem = b % (prm.H * S);
  const int seq = rem % S, h = rem / S;
  const int seg0 = prm.cu[seq];
  const int len = prm.cu[seq + 1] - seg0;
  const int q0 = pair * 2 * kBlockQ;
  if (q0 >= len) return;  // uniform across the CTA, before any barrier or TMEM use
  const int n_tiles_q = (len - q0 > kBlockQ) ? 2 : 1;
  const int n_pre = prm.P > 0 ? (prm.P + kBlockK - 1) / kBlockK : 0;
  const int n_kv = n_pre + (len + kBlockK - 1) / kBlockK;
  const int hk = h / (prm.H / prm.Hkv);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_ready[t], 128);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 256);
      mbar_init(&bars->o_done[t], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&bars->xchg[t][q], 64);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->k_ready[s], 64);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // key tile j -> (map, column of head's chunk 0, first row, valid keys)
  auto kv_coords = [&](int j, bool is_v, int &row, int &col, bool &prefix, int &nvalid) {
    if (j < n_pre) {
      prefix = true;
      row = (seq * 2 + (is_v ? 1 : 0)) * prm.P + j * kBlockK;
      col = hk * HD;
      nvalid = min(kBlockK, prm.P - j * kBlockK);
    } else {
      prefix = false;
      const int jj = j - n_pre;
      row = seg0 + jj * kBlockK;
      col = (is_v ? 2 : 1) * prm.C + h * HD;
      nvalid = min(kBlockK, len - jj * kBlockK);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      mbar_arrive_expect_tx(&bars->q_full, n_tiles_q * CF::kTile);
      for (int t = 0; t < n_tiles_q; ++t) {
        uint8_t *qt = smem + CF::kQOff + t * CF::kTile;
        const int row = seg0 + q0 + t * kBlockQ;
        tma_load_2d(qt, &tm_x0, &bars->q_full, h * HD, row);
        tma_load_2d(qt + CF::kChunk0, &tm_x1, &bars->q_full, h * HD + 64, row);
      }
      bool ok = true;
      uint32_t issued = 0, issued_par = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NS;
        const uint32_t f = (j / NS) & 1;
        if (!mbar_wait(&bars->kv_empty[st], f ^ 1, abort_flag)) { ok = false; break; }
        int row, col, nvalid;
        bool pre;
        uint8_t *kt = smem + CF::kKOff + st * CF::kTile;
        uint8_t *vt = smem + CF::kVOff + st * CF::kTile;
        kv_coords(j, false, row, col, pre, nvalid);
        mbar_arrive_expect_tx(&bars->k_full[st], CF::kTile);
        tma_load_2d(kt, pre ? &tm_p0 : &tm_x0, &bars->k_full[st], col, row);
        tma_load_2d(kt + CF::kChunk0, pre ? &tm_p1 : &tm_x1, &bars->k_full[st], col + 64, row);
        kv_coords(j, true, row, col, pre, nvalid);
        mbar_arrive_expect_tx(&bars->v_full[st], CF::kTile);
        tma_load_2d(vt, pre ? &tm_p0 : &tm_x0, &bars->v_full[st], col, row);
        tma_load_2d(vt + CF::kChunk0, pre ? &tm_p1 : &tm_x1, &bars->v_full[st], col + 64, row);
        issued |= 1u << st;
        issued_par = (issued_par & ~(1u << st)) | (f << st);
      }
      if (!ok) {
        drain_wait(&bars->q_full, 0);
        for (int s = 0; s < NS; ++s)
          if (issued & (1u << s)) {
            drain_wait(&bars->k_full[s], (issued_par >> s) & 1);
            drain_wait(&bars->v_full[s], (issued_par >> s) & 1);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true, any = false;
      const uint32_t sq = smem_u32(smem + CF::kQOff);
      const uint32_t sk = smem_u32(smem + CF::kKOff);
      const uint32_t sv = smem_u32(smem + CF::kVOff);
      // S_t = Q_t K_j^T over HDP/16 k-steps
      auto issue_s = [&](int t, int st) {
        const uint32_t qa = sq + t * CF::kTile, ka = sk + st * CF::kTile;
        const uint32_t d = tmem + CF::kTmemS + t * 128;
#pragma unroll
        for (int k = 0; k < CF::HDP / 16; ++k) {
          uint64_t ad, bd;
          if (k < 4) {
            ad = smem_desc(qa + k * 32, 16, 1024, 2);
            bd = smem_desc(ka + k * 32, 16, 1024, 2);
          } else if (HD == 72) {
            ad = smem_desc(qa + CF::kChunk0, 16, 256, 6);
            bd = smem_desc(ka + CF::kChunk0, 16, 256, 6);
          } else {
            ad = smem_desc(qa + CF::kChunk0 + (k - 4) * 32, 16, 1024, 2);
            bd = smem_desc(ka + CF::kChunk0 + (k - 4) * 32, 16, 1024, 2);
          }
          mma_bf16_ss(d, ad, bd, CF::kIdescS, k > 0);
        }
      };
      // O_t += P_t V_j; P_t is bf16 in TMEM (S_t's first 64 columns)
      auto issue_pv = [&](int t, int st, bool acc) {
        const uint32_t va = sv + st * CF::kTile;
        const uint32_t p = tmem + CF::kTmemS + t * 128;
        const uint32_t d = tmem + CF::kTmemO + t * 128;
#pragma unroll
        for (int k = 0; k < kBlockK / 16; ++k) {
          const uint32_t accf = (acc || k > 0) ? 1u : 0u;
          if (HD == 72) {
            mma_bf16_ts(d, p + k * 8, smem_desc(va + k * 2048, 16384, 1024, 2), CF::kIdescPV0,
                        accf);
            mma_bf16_ts(d + 64, p + k * 8, smem_desc(va + CF::kChunk0 + k * 512, 4096, 256, 6),
                        CF::kIdescPV1, accf);
          } else {
            mma_bf16_ts(d, p + k * 8, smem_desc(va + k * 2048, 16384, 1024, 2), CF::kIdescPV0,
                        accf);
          }
        }
      };
      auto wait_k = [&](int j) -> bool {
        const int st = j % NS;
        const uint32_t f = (j / NS) & 1;
        return ROPE ? mbar_wait(&bars->k_ready[st], f, abort_flag)
                    : mbar_wait(&bars->k_full[st], f, abort_flag);
      };
      do {
        for (int t = 0; t < n_tiles_q; ++t)
          if (!mbar_wait(&bars->q_ready[t], 0, abort_flag)) { ok = false; break; }
        if (!ok || !wait_k(0)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < n_tiles_q; ++t) {
          issue_s(t, 0);
          mma_commit(&bars->s_full[t]);
        }
        any = true;
        for (int j = 0; j < n_kv && ok; ++j) {
          const int st = j % NS;
          const uint32_t f = (j / NS) & 1;
          if (!mbar_wait(&bars->v_full[st], f, abort_flag)) { ok = false; break; }
          for (int t = 0; t < n_tiles_q; ++t) {
            if (!mbar_wait(&bars->p_full[t], j & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, st, j > 0);
            mma_commit(&bars->o_done[t]);
            if (j + 1 < n_kv) {
              if (!wait_k(j + 1)) { ok = false; break; }
              // S_t(j+1) overwrites P_t(j): wait until O_t += P_t V_j has finished
              if (!mbar_wait(&bars->o_done[t], j & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              issue_s(t, (j + 1) % NS);
              mma_commit(&bars->s_full[t]);
            }
          }
          mma_commit(&bars->kv_empty[st]);
        }
      } while (false);
      if (!ok && any) {
        mma_commit(&bars->drain);
        drain_wait(&bars->drain, 0);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 4;
    const int t = sw >> 3;               // query tile of this warp
    const int half = (sw >> 2) & 1;      // which 64 of the 128 score columns
    const int quarter = warp & 3;        // TMEM lane quarter
    const int r = quarter * 32 + lane;   // query row inside the tile
    if (t < n_tiles_q) {
      const int qrow = q0 + t * kBlockQ + r;  // row inside the sequence
      bool ok = true;
      if (half == 0) {
        ok = mbar_wait(&bars->q_full, 0, abort_flag);
        if (ok) {
          uint8_t *qt = smem + CF::kQOff + t * CF::kTile;
          if (ROPE && qrow < len)
            rope_row_smem<HD>(qt, r, prm.pos[2 * (seg0 + qrow)], prm.pos[2 * (seg0 + qrow) + 1], fr);
          if (HD == 72)  // zero the 8 padding columns 72..79 (logical unit 9)
            *reinterpret_cast<uint4 *>(qt + unit_offset<HD>(r, 9)) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
        }
        mbar_arrive(&bars->q_ready[t]);
      }
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t lane_base = uint32_t(quarter * 32) << 16;
      const uint32_t s_addr = tmem + lane_base + CF::kTmemS + t * 128;
      const uint32_t o_addr = tmem + lane_base + CF::kTmemO + t * 128;
      float *xv = reinterpret_cast<float *>(smem + CF::kXOff) + t * 256;  // [half][row]
      uint64_t *xb = &bars->xchg[t][quarter];
      const float sl2 = prm.scale_log2;
      // head_dim 72: the softmax denominator is accumulated by the tensor core
      // as O column 72 -- V's first padding column is set to 1.0 before each
      // P.V -- so the row sum costs no instruction here and sums exactly the
      // bf16 P the numerator uses.  That also lets P be rounded toward zero
      // (one byte permute per pair): the rounding's mean cancels between
      // numerator and denominator and its spread equals round-to-nearest's.
      // head_dim 128 sums in registers and rounds P to nearest.
      constexpr bool kSumByMma = (HD == 72);
      // pairs of this thread's 64 exponentials that run on the FMA pipe
      // instead of the special-function unit (8 of 32: a 25% share)
      constexpr int kPolyPairs = 8;
      constexpr int kOC = CF::HDP / 16;         // 16-column chunks of O
      constexpr int kOCHalf = (kOC + 1) / 2;   // rescaled by half 0; the rest by half 1
      const int oc_lo = half ? kOCHalf : 0, oc_hi = half ? kOC : kOCHalf;
      float m = -INFINITY;
      uint64_t l2[2] = {0, 0};  // packed partial row sums (head_dim 128)
      for (int j = 0; j < n_kv && ok; ++j) {
        if (!warp_wait(&bars->s_full[t], j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int nvalid = (j < n_pre ? min(kBlockK, prm.P - j * kBlockK)
                                      : min(kBlockK, len - (j - n_pre) * kBlockK)) -
                           half * 64;  // valid keys among this thread's 64 columns
        uint32_t s[2][32];
        __syncwarp();
        tmem_ld32(s_addr + half * 64, s[0]);
        tmem_ld32(s_addr + half * 64 + 32, s[1]);
        tmem_ld_wait();
        if (nvalid < 64) {  // keys past the sequence end: -inf, so p = 0
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i >= nvalid) s[c][i] = 0xFF800000u;
        }
        float mc[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float a = __uint_as_float(s[c][0]);
#pragma unroll
          for (int i = 1; i < 31; i += 2)
            a = fmax3(a, __uint_as_float(s[c][i]), __uint_as_float(s[c][i + 1]));
          mc[c] = fmaxf(a, __uint_as_float(s[c][31]));
        }
        // swap partial maxima with the thread that holds the row's other half
        // (its P columns overlap this half's S columns, so the swap also
        // orders this thread's TMEM loads before the partner's P stores)
        xv[half * 128 + r] = fmaxf(mc[0], mc[1]) * sl2;
        tc_fence_before();
        mbar_arrive(xb);
        if (!warp_wait(xb, j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float m_tile = fmaxf(xv[r], xv[128 + r]);
        const bool grow = __any_sync(0xffffffffu, m_tile > m + 8.0f);
        if (j == 0) {
          m = m_tile;
        } else if (grow) {
          // rescale O (and the row sum) only when the running max grew by
          // more than 8 in log2 units; otherwise keep the stale max
          const bool mine = m_tile > m + 8.0f;
          const float m_new = mine ? m_tile : m;
          const float factor = mine ? ex2_approx(m - m_new) : 1.0f;
          const uint64_t f2 = f2_pack(factor, factor);
          if (!warp_wait(&bars->o_done[t], (j - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kOC; ++c) {
            if (c < oc_lo || c >= oc_hi) continue;
            uint32_t v[16];
            __syncwarp();
            tmem_ld16(o_addr + c * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float a, b;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), f2),
                        a, b);
              v[2 * i] = __float_as_uint(a);
              v[2 * i + 1] = __float_as_uint(b);
            }
            tmem_st16(o_addr + c * 16, v);
          }
          tmem_st_wait();
          if (!kSumByMma)
#pragma unroll
            for (int k = 0; k < 2; ++k) l2[k] = f2_mul(l2[k], f2);
          m = m_new;
        }
        // p = 2^(s*scale*log2e - m) two at a time; bf16 P of keys
        // [64 half, 64 half + 64) into S columns [32 half, 32 half + 32)
        const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t xa = f2_fma(
                f2_pack(__uint_as_float(s[c][2 * i]), __uint_as_float(s[c][2 * i + 1])), sc2, nm2);
            float p0, p1;
            if (c * 16 + i < kPolyPairs) {  // this share of the exponentials runs on the FMA pipe
              exp2_poly_x2(xa, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(xa, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            if (kSumByMma) {
              pk[i] = pack_bf16x2_trunc(p0, p1);
            } else {
              l2[i & 1] = f2_add(l2[i & 1], f2_pack(p0, p1));
              pk[i] = pack_bf16x2_alu(p0, p1);
            }
          }
          tmem_st16(s_addr + half * 32 + c * 16, pk);
        }
        if (kSumByMma && t == 0 && half == 0) {
          // ones in V's column 72 of this key tile (the first padding column)
          const int st = j % NS;
          if (!warp_wait(&bars->v_full[st], (j / NS) & 1, abort_flag)) { ok = false; break; }
          *reinterpret_cast<uint16_t *>(smem + CF::kVOff + st * CF::kTile + unit_offset<HD>(r, 9)) =
              0x3F80u;  // bf16 1.0
          fence_proxy_async_smem();
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t]);
      }
      // epilogue: O / l -> bf16 rows of o [T, H, HD], each thread its half of the row
      if (ok && warp_wait(&bars->o_done[t], (n_kv - 1) & 1, abort_flag)) {
        tc_fence_after();
        float l = 0.0f;
        bool have_l = true;
        if (!kSumByMma) {  // add the two halves' partial sums
          float a, b, c2, d2;
          f2_unpack(l2[0], a, b);
          f2_unpack(l2[1], c2, d2);
          xv[half * 128 + r] = (a + b) + (c2 + d2);
          mbar_arrive(xb);
          have_l = warp_wait(xb, n_kv & 1, abort_flag);
          l = xv[r] + xv[128 + r];
        }
        if (have_l) {
          __nv_bfloat16 *orow =
              qrow < len ? prm.o + size_t(seg0 + qrow) * prm.C + size_t(h) * HD : nullptr;
          if (half == 0)
            store_o_half<HD, 0>(o_addr, l, orow);
          else
            store_o_half<HD, 1>(o_addr, l, orow);
        }
      }
    }
  } else if (ROPE && warp < 4) {
    // ------------------------------------------------------------ K rotation
    // warps 2-3; thread rotates key rows r and r + 64 of each own-key tile
    const int r0 = (warp - 2) * 32 + lane;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j % NS;
      const uint32_t f = (j / NS) & 1;
      if (!mbar_wait(&bars->k_full[st], f, abort_flag)) break;
      if (j >= n_pre) {
#pragma unroll 1
        for (int r = r0; r < kBlockK; r += 64) {
          const int key = (j - n_pre) * kBlockK + r;
          if (key < len)
            rope_row_smem<HD>(smem + CF::kKOff + st * CF::kTile, r, prm.pos[2 * (seg0 + key)],
                              prm.pos[2 * (seg0 + key) + 1], fr);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&bars->k_ready[st]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bars->abort_flag) report_status(prm.status, kDevTimeout);
}

// ---------------------------------------------------------------- host side
template <int HD, bool ROPE>
static cudaError_t launch_hd(const CUtensorMap *maps, const attn::Params &prm, int grid,
                             const RopeFreqs &fr, cudaStream_t st) {
  using CF = attn::Cfg<HD>;
  auto kern = attention_tc_kernel<HD, ROPE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CF::kSmem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(attn::kThreads), CF::kSmem, st, 1, maps[0], maps[1],
                    maps[2], maps[3], prm, fr);
}

cudaError_t launch_attention_tc(const void *qkv, void *o, const SeqArgs &s, int H, int d,
                                float scale, const RopeFreqs &fr, int num_sms, int *status,
                                cudaStream_t st) {
  (void)num_sms;
  if (s.total_tokens == 0 || s.max_seqlen == 0) return cudaSuccess;
  const int C = H * d;
  const int Hkv = s.kv_heads > 0 ? s.kv_heads : H;
  const int P = s.prefix_kv ? s.prefix_len : 0;
  CUtensorMap maps[4];
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool small = (d == 72);
  // qkv viewed as [T, 3C]
  if (encode_tensor_map_2d(&maps[0], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, 64, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&maps[1], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, small ? 16 : 64,
                           128, small ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (P > 0) {
    // prefix viewed as [S * 2 * P, Hkv * d]
    const uint64_t rows = uint64_t(s.n_seqs) * 2 * P;
    if (encode_tensor_map_2d(&maps[2], BF, s.prefix_kv, uint64_t(Hkv) * d, rows,
                             uint64_t(Hkv) * d * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    if (encode_tensor_map_2d(&maps[3], BF, s.prefix_kv, uint64_t(Hkv) * d, rows,
                             uint64_t(Hkv) * d * 2, small ? 16 : 64, 128,
                             small ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    maps[2] = maps[0];
    maps[3] = maps[1];
  }
  attn::Params prm;
  prm.H = H;
  prm.C = C;
  prm.Hkv = Hkv;
  prm.P = P;
  prm.n_pairs = (s.max_seqlen + 2 * attn::kBlockQ - 1) / (2 * attn::kBlockQ);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu = s.cu_seqlens;
  prm.pos = s.pos;
  prm.o = static_cast<__nv_bfloat16 *>(o);
  prm.status = status;
  const int grid = prm.n_pairs * H * s.n_seqs;
  const bool rope = s.pos != nullptr;
  if (d == 72)
    return rope ? launch_hd<72, true>(maps, prm, grid, fr, st)
                : launch_hd<72, false>(maps, prm, grid, fr, st);
  return rope ? launch_hd<128, true>(maps, prm, grid, fr, st)
              : launch_hd<128, false>(maps, prm, grid, fr, st);
}

}  // namespace vit
