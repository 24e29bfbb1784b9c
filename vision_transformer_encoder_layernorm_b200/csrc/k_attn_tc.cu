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
// Persistent: one CTA per SM walks a static list of work items = (sequence,
// head, two 128-row query tiles), full pairs first, round-robin over CTAs;
// every barrier phase is counted across items.  20 warps:
//   0        TMA producer (Q tiles once, then K and V tiles through a ring)
//   1, 2     MMA issuers of query tiles 0 and 1 (one lane each; warp 1 also
//            owns the TMEM allocation): each follows its own tile's
//            softmax, so neither tile's MMAs wait behind the other's
//   3        prepares each item's Q tiles (head_dim 72: zero the padding
//            columns; ROPE: rotate) and each key tile (ROPE: rotate own-key
//            K rows; head_dim 72: ones in V's column 72, the row sums), so
//            the next item's first S overlaps the softmax epilogue
//   4-11     softmax of query tile 0, 12-19 of query tile 1: two threads per
//            query row, one per half of the key tile's score columns; each
//            also reads the other half's scores from TMEM for the row max
// Per query tile t, TMEM holds S_t (fp32 scores of one key tile), P_t (bf16
// probabilities, its own columns) and O_t.  Because P does not overwrite S,
// the MMA warp issues S_t(j+1) = Q_t K_{j+1}^T as soon as the softmax threads
// have loaded S_t(j) into registers: the tensor core computes the next key
// tile's scores while the exponentials of this one run, and O_t += P_t V_j
// follows when P_t(j) is stored.  To fit 2 x (S + P + O) in the 512 TMEM
// columns a key tile has 112 keys at head_dim 72 and 80 at head_dim 128.
// head_dim 72 is computed as 80 (4 MMA k-steps from a 64-column 128B-swizzled
// chunk, 1 from a 16-column 32B-swizzled chunk); Q's columns 72..79 are zeroed
// in shared memory so the neighbouring head's values there contribute 0.
#include <cstdlib>
#include <type_traits>
#include <vector>

#include "kernels.h"
#include "sm100.cuh"

namespace vit {
namespace attn {

constexpr int kBlockQ = 128;
constexpr int kThreads = 640;
constexpr int kRegsLow = 64, kRegsHigh = 104;  // warpgroup 0 / softmax warpgroups

__host__ __device__ constexpr uint32_t round_up_1k(uint32_t x) { return (x + 1023u) & ~1023u; }

template <int HD>
struct Cfg {
  static constexpr int HDP = HD == 72 ? 80 : 128;            // padded head_dim
  static constexpr int BK = HD == 72 ? 112 : 80;             // keys per key tile
  static constexpr int HC = BK / 2;                          // score columns per softmax thread
  static constexpr uint32_t kQChunk0 = kBlockQ * 128;        // 128 rows x 64 bf16
  static constexpr uint32_t kQChunk1 = HD == 72 ? kBlockQ * 32 : kBlockQ * 128;
  static constexpr uint32_t kQTile = kQChunk0 + kQChunk1;
  static constexpr uint32_t kKChunk0 = BK * 128;             // multiple of 1024
  static constexpr uint32_t kKChunk1 = HD == 72 ? BK * 32 : BK * 128;
  static constexpr uint32_t kKTile = round_up_1k(kKChunk0 + kKChunk1);
  // head_dim 72: V is stored as five 16-column 32B-swizzled chunks so that
  // one N = 80 MMA per k-step covers it (head_dim 128: as K, two 64-column
  // 128B-swizzled chunks, one N = 128 MMA)
  static constexpr uint32_t kVChunk = HD == 72 ? BK * 32 : BK * 128;
  static constexpr int kVChunks = HD == 72 ? 5 : 2;
  static constexpr int kStages = HD == 72 ? 5 : 3;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = 2 * kQTile;
  static constexpr uint32_t kVOff = kKOff + kStages * kKTile;
  static constexpr uint32_t kBarOff = kVOff + kStages * kKTile;
  static constexpr uint32_t kXOff = kBarOff + 512;             // row-max exchange [2][2][2][128] f32
  static constexpr size_t kSmem = size_t(kXOff) + 4096 + 1024;
  // TMEM columns (16-aligned): S0, S1, P0, P1, O0, O1
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = BK;
  static constexpr uint32_t kTmemP0 = 2 * BK, kTmemP1 = (2 * BK + BK / 2 + 15) / 16 * 16;
  static constexpr uint32_t kTmemO0 = HD == 72 ? 352 : 256, kTmemO1 = kTmemO0 + (HD == 72 ? 80 : 128);
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, HDP, 0, 1);
  __host__ __device__ static constexpr uint32_t tmem_s(int t) { return t ? kTmemS1 : kTmemS0; }
  __host__ __device__ static constexpr uint32_t tmem_p(int t) { return t ? kTmemP1 : kTmemP0; }
  __host__ __device__ static constexpr uint32_t tmem_o(int t) { return t ? kTmemO1 : kTmemO0; }
};
static_assert(Cfg<72>::kVChunks * Cfg<72>::kVChunk <= Cfg<72>::kKTile &&
                  Cfg<128>::kVChunks * Cfg<128>::kVChunk <= Cfg<128>::kKTile,
              "V tile");
static_assert(Cfg<72>::kSmem <= 232448 && Cfg<128>::kSmem <= 232448, "shared memory");
static_assert(Cfg<72>::kTmemP1 + Cfg<72>::BK / 2 <= Cfg<72>::kTmemO0 && Cfg<72>::kTmemO1 + 80 <= 512,
              "TMEM layout, head_dim 72");
static_assert(Cfg<128>::kTmemP1 + Cfg<128>::BK / 2 <= Cfg<128>::kTmemO0 &&
                  Cfg<128>::kTmemO1 + 128 <= 512,
              "TMEM layout, head_dim 128");

struct __align__(8) Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t q_ready[2];
  uint64_t k_full[5], v_full[5], kv_empty[5], k_ready[5], v_ready[5];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint64_t xchg[2][4];  // per (query tile, lane quarter): the 64 threads of a row pair
  uint64_t part_done;   // split units: all softmax warps wrote their partial rows
  uint64_t part_flag[2];  // split units: the counter was read (per tile)
  uint64_t drain[2];
  int part_last;        // split units: this CTA combines the parts
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block overflows its slot");

struct Params {
  int H, C, Hkv, P, n_pairs, n_seqs;
  int tpi;               // query tiles per item: 2, or 1 when the items would not fill the SMs
  int snake;             // packed sequences: items by descending length, dealt out in a snake
  float scale_log2;      // softmax scale * log2(e)
  const int32_t *cu;
  const int32_t *pos;
  __nv_bfloat16 *o;
  int *status;
  float *part;           // split work: per CTA 2 slots x 2 tiles x 128 rows x kPartStride fp32
  int *cnt;              // split work: parts finished, per item (indexed by its first CTA)
};

// Split (stream-K) schedule, head_dim 72, one sequence: CTA c processes the
// key tiles from position (bw[c], bj[c]) up to (bw[c+1], bj[c+1]) of the
// item list (item, key tile), in item order.  n == 0: whole items
// round-robin instead.
constexpr int kMaxSkCtas = 160;
// a partial row: O columns 0..79 (72 = row sum), the running max at column
// kPartM; the stride keeps every row 16-byte aligned for the vector stores
constexpr int kPartStride = 84, kPartM = 80;
static_assert((kPartStride * 4) % 16 == 0 && kPartM % 4 == 0 && 72 % 4 == 0,
              "partial rows, the max and the row sum must sit at 16-byte boundaries");
struct SkTable {
  int n;
  int bw[kMaxSkCtas + 1], bj[kMaxSkCtas + 1];
};

// One work item: query tiles [q0, q0 + tpi * 128) of head h of sequence seq.
struct Item {
  int seq, h, hk, seg0, len, q0, n_tiles_q, n_kv;
};

// Work item w (pairs in ascending order, so a sequence's last, partial pair
// comes after all full ones); false if the pair lies past the sequence end.
__device__ __forceinline__ bool decode_item(int w, const Params &prm, int bk, Item &it) {
  const int per_pair = prm.H * prm.n_seqs;
  const int pair = w / per_pair, rem = w - pair * per_pair;
  it.seq = rem % prm.n_seqs;
  it.h = rem / prm.n_seqs;
  it.hk = it.h / (prm.H / prm.Hkv);
  it.seg0 = prm.cu[it.seq];
  it.len = prm.cu[it.seq + 1] - it.seg0;
  it.q0 = pair * prm.tpi * kBlockQ;
  if (it.q0 >= it.len) return false;
  it.n_tiles_q = (prm.tpi == 2 && it.len - it.q0 > kBlockQ) ? 2 : 1;
  const int n_pre = prm.P > 0 ? (prm.P + bk - 1) / bk : 0;
  it.n_kv = n_pre + (it.len + bk - 1) / bk;
  return true;
}

// Packed sequences of different lengths (snake schedule): the items are
// listed by descending sequence length (a sequence's items pair-major, heads
// inner) and dealt to the CTAs in a snake, round r going 0..G-1 for even r
// and G-1..0 for odd r, so the long items spread evenly and the short ones
// fill in behind them.  The CTA's warp 0 builds the order in shared
// memory: ord[i] = i-th longest sequence, pre[i] = items before it.
constexpr int kMaxSnakeSeqs = 64;
struct SnakeTab {
  int len[kMaxSnakeSeqs];
  int ord[kMaxSnakeSeqs];
  int pre[kMaxSnakeSeqs + 1];
};

// Warp 0: each lane ranks sequences lane and lane + 32 by length
// (descending, ties by index), then lane 0 sums the items in that order.
__device__ __forceinline__ void build_snake(const Params &prm, SnakeTab *tab, int lane) {
  const int n = prm.n_seqs;
  for (int i = lane; i < n; i += 32) tab->len[i] = prm.cu[i + 1] - prm.cu[i];
  __syncwarp();
  for (int i = lane; i < n; i += 32) {
    const int li = tab->len[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const int lj = tab->len[j];
      rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    tab->ord[rank] = i;
  }
  __syncwarp();
  if (lane == 0) {
    tab->pre[0] = 0;
    for (int i = 0; i < n; ++i)
      tab->pre[i + 1] =
          tab->pre[i] + (tab->len[tab->ord[i]] + 2 * kBlockQ - 1) / (2 * kBlockQ) * prm.H;
  }
}

// Item w of the snake order (always a real item).
__device__ __forceinline__ void decode_snake(int w, const Params &prm, const SnakeTab &tab, int bk,
                                             Item &it) {
  int i = 0;
  while (tab.pre[i + 1] <= w) ++i;
  const int local = w - tab.pre[i];
  const int pair = local / prm.H;
  it.seq = tab.ord[i];
  it.h = local - pair * prm.H;
  it.hk = it.h / (prm.H / prm.Hkv);
  it.seg0 = prm.cu[it.seq];
  it.len = tab.len[it.seq];
  it.q0 = pair * 2 * kBlockQ;
  it.n_tiles_q = (it.len - it.q0 > kBlockQ) ? 2 : 1;
  const int n_pre = prm.P > 0 ? (prm.P + bk - 1) / bk : 0;
  it.n_kv = n_pre + (it.len + bk - 1) / bk;
}

// A work unit: key tiles [j0, j1) of item w.
struct Unit {
  Item it;
  int w, j0, j1;
  bool whole;
};

// k-th unit of this CTA: 0 = no more units, 1 = unit, 2 = nothing to do for
// this k (an empty pair slot)
__device__ __forceinline__ int get_unit(int k, const Params &prm, const SkTable &sk, int bk,
                                        Unit &u, const SnakeTab *snake) {
  const int c = blockIdx.x;
  if (prm.snake) {
    const int G = gridDim.x;
    u.w = k * G + ((k & 1) ? G - 1 - c : c);
    if (u.w >= snake->pre[prm.n_seqs]) return 0;  // rounds only grow: no more items
    decode_snake(u.w, prm, *snake, bk, u.it);
    u.j0 = 0;
    u.j1 = u.it.n_kv;
    u.whole = true;
    return 1;
  }
  if (sk.n == 0) {
    u.w = c + k * gridDim.x;
    if (u.w >= prm.n_pairs * prm.H * prm.n_seqs) return 0;
    if (!decode_item(u.w, prm, bk, u.it)) return 2;
    u.j0 = 0;
    u.j1 = u.it.n_kv;
    u.whole = true;
    return 1;
  }
  u.w = sk.bw[c] + k;
  const int last = sk.bj[c + 1] > 0 ? sk.bw[c + 1] : sk.bw[c + 1] - 1;
  if (u.w > last) return 0;
  if (!decode_item(u.w, prm, bk, u.it)) return 2;
  u.j0 = u.w == sk.bw[c] ? sk.bj[c] : 0;
  u.j1 = u.w == sk.bw[c + 1] ? sk.bj[c + 1] : u.it.n_kv;
  if (u.j1 <= u.j0) return 2;
  u.whole = u.j0 == 0 && u.j1 == u.it.n_kv;
  return 1;
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;
  }
}

// Byte offset of logical 16-byte unit u (0..HDP/8-1) of row r inside an
// operand tile whose chunk 0 takes chunk0 bytes: chunk 0 (units 0..7) is
// 128B-swizzled, chunk 1 is 32B-swizzled (head_dim 72, units 8..9) or
// 128B-swizzled (head_dim 128, units 8..15).
template <int HD>
__device__ __forceinline__ uint32_t unit_offset(int r, int u, uint32_t chunk0) {
  if (u < 8) return uint32_t(r * 128 + ((u ^ (r & 7)) << 4));
  const int v = u - 8;
  if (HD == 72) return chunk0 + uint32_t(r * 32 + ((v ^ ((r >> 2) & 1)) << 4));
  return chunk0 + uint32_t(r * 128 + ((v ^ (r & 7)) << 4));
}

// Rotates row r of an operand tile in place by 2D RoPE at position (pr, pc):
// dims [0, HD/2) by pr, [HD/2, HD) by pc; in a half, dim j pairs with j+HD/4.
// fr.wpi[j] = theta^(-2j/(HD/2)) / pi.
template <int HD>
__device__ __forceinline__ void rope_row_smem(uint8_t *tile, uint32_t chunk0, int r, int pr,
                                              int pc, const RopeFreqs &fr) {
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
      const uint4 v = *reinterpret_cast<const uint4 *>(tile + unit_offset<HD>(r, u0 + k, chunk0));
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
      *reinterpret_cast<uint4 *>(tile + unit_offset<HD>(r, u0 + k, chunk0)) =
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

// Maximum of the first `nvalid` of N consecutive TMEM columns of this
// thread's lane (N % 4 == 0): all N columns in one load round trip (one
// tcgen05.wait::ld), then two independent chains of 3-input maxima.
template <int N>
__device__ __forceinline__ float tmem_rowmax(uint32_t addr, int nvalid) {
  static_assert(N <= 56 && N % 8 == 0, "row width");
  uint32_t q[N];
  __syncwarp();
  tmem_ld_cols<N>(addr, q);
  tmem_ld_wait();
  if (nvalid < N) {
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (i >= nvalid) q[i] = 0xFF800000u;
  }
  float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
  for (int i = 0; i + 3 < N; i += 4) {
    a0 = fmax3(a0, __uint_as_float(q[i]), __uint_as_float(q[i + 1]));
    a1 = fmax3(a1, __uint_as_float(q[i + 2]), __uint_as_float(q[i + 3]));
  }
  return fmaxf(a0, a1);
}

// Partial rows of a split item: this half's O columns (fp32, unnormalised;
// column 72 holds the row sum) and, from half 0, the running max m.
template <int HD, int HALF>
__device__ __forceinline__ void store_o_part(uint32_t o_addr, float *row, float m) {
  constexpr int NC = Cfg<HD>::HDP / 16;
  constexpr int C0 = HALF ? (NC + 1) / 2 : 0, C1 = HALF ? NC : (NC + 1) / 2;
  uint32_t ov[NC][16];
  __syncwarp();
#pragma unroll
  for (int c = C0; c < C1; ++c) tmem_ld16(o_addr + c * 16, ov[c]);
  tmem_ld_wait();
#pragma unroll
  for (int c = C0; c < C1; ++c)
#pragma unroll
    for (int i = 0; i < 16; i += 4)
      *reinterpret_cast<float4 *>(row + c * 16 + i) =
          make_float4(__uint_as_float(ov[c][i]), __uint_as_float(ov[c][i + 1]),
                      __uint_as_float(ov[c][i + 2]), __uint_as_float(ov[c][i + 3]));
  if (HALF == 0) row[kPartM] = m;
}

// Combines the parts of a split item held by CTAs c0..c1 for row r:
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (l_s = O_s
// column 72); this half's 16-byte units of the output row, bf16.
// Partial rows of CTA cc's part of item w, query tile t (slot 0: the CTA's
// first unit, 1: its last).
__device__ __forceinline__ const float *part_rows(const float *part, const SkTable &sk, int cc,
                                                 int w, int t) {
  return part + ((size_t(cc) * 2 + (w == sk.bw[cc] ? 0 : 1)) * 2 + t) * kBlockQ * kPartStride;
}

template <int HD, int HALF>
__device__ __noinline__ void combine_parts(const float *part, const SkTable &sk, int w, int t,
                                           int c0, int c1, int r, __nv_bfloat16 *orow) {
  constexpr int NU = HD / 8;
  constexpr int U0 = HALF ? (NU + 1) / 2 : 0, U1 = HALF ? NU : (NU + 1) / 2;
  constexpr int NV = (U1 - U0) * 2;  // float4 vectors of this half's output columns
  // rows of the other CTAs' parts: 16-byte loads through L2 (ld.global.cg)
  auto rowv = [&](int cc) {
    return reinterpret_cast<const float4 *>(part_rows(part, sk, cc, w, t) + size_t(r) * kPartStride);
  };
  float M = -INFINITY;
  for (int c = c0; c <= c1; ++c) M = fmaxf(M, __ldcg(rowv(c) + kPartM / 4).x);
  float acc[NV * 4], l = 0.0f;
#pragma unroll
  for (int i = 0; i < NV * 4; ++i) acc[i] = 0.0f;
  for (int c = c0; c <= c1; ++c) {
    const float4 *v = rowv(c);
    float4 d[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) d[i] = __ldcg(v + U0 * 2 + i);
    const float e = ex2_approx(__ldcg(v + kPartM / 4).x - M);
    l += e * __ldcg(v + HD / 4).x;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      acc[4 * i] += e * d[i].x;
      acc[4 * i + 1] += e * d[i].y;
      acc[4 * i + 2] += e * d[i].z;
      acc[4 * i + 3] += e * d[i].w;
    }
  }
  if (orow == nullptr) return;
  const float inv = 1.0f / l;
#pragma unroll
  for (int u = U0; u < U1; ++u) {
    const float *a = acc + (u - U0) * 8;
    *reinterpret_cast<uint4 *>(orow + u * 8) =
        make_uint4(pack_bf16x2(a[0] * inv, a[1] * inv), pack_bf16x2(a[2] * inv, a[3] * inv),
                   pack_bf16x2(a[4] * inv, a[5] * inv), pack_bf16x2(a[6] * inv, a[7] * inv));
  }
}

}  // namespace attn

template <int HD, bool ROPE>
__global__ void __launch_bounds__(attn::kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q0,
                        const __grid_constant__ CUtensorMap tm_q1,
                        const __grid_constant__ CUtensorMap tm_k0,
                        const __grid_constant__ CUtensorMap tm_k1,
                        const __grid_constant__ CUtensorMap tm_p0,
                        const __grid_constant__ CUtensorMap tm_p1, const attn::Params prm,
                        const __grid_constant__ RopeFreqs fr,
                        const __grid_constant__ attn::SkTable sk) {
  using namespace attn;
  using CF = Cfg<HD>;
  constexpr int NS = CF::kStages;
  constexpr int BK = CF::BK;
  constexpr int HC = CF::HC;
  constexpr bool kPrep = ROPE || HD == 72;  // warp 3 has Q / K / V tiles to touch up
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + CF::kBarOff);
  volatile int *abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_trigger();
  pdl_wait();
  const int n_pre = prm.P > 0 ? (prm.P + BK - 1) / BK : 0;

  // the snake order's table sits in the row-sum exchange region, unused at
  // head_dim 72 (the only persistent kernel that takes the snake schedule)
  SnakeTab *snake = reinterpret_cast<SnakeTab *>(smem + CF::kXOff);
  static_assert(sizeof(SnakeTab) <= 4096, "snake table");
  if (warp == 0 && prm.snake) build_snake(prm, snake, lane);
  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->q_empty[t], 1);
      mbar_init(&bars->q_ready[t], 32);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_free[t], 256);
      mbar_init(&bars->p_full[t], 256);
      mbar_init(&bars->o_done[t], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&bars->xchg[t][q], 64);
      mbar_init(&bars->drain[t], 1);
      mbar_init(&bars->part_flag[t], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 2);  // one commit per query tile (tile 0 twice if alone)
      mbar_init(&bars->k_ready[s], 32);
      mbar_init(&bars->v_ready[s], 32);
    }
    mbar_init(&bars->part_done, 16);  // lane 0 of each softmax warp (tile 0 twice when alone)
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
  // registers: 640 threads x 96 at launch; warps 0-3 (one warpgroup) give
  // back 32 each, the four softmax warpgroups take 8 more:
  // 128 x 64 + 512 x 104 = 640 x 96
  static_assert(128 * kRegsLow + 512 * kRegsHigh <= kThreads * 96, "register split");

  // key tile j of an item -> (prefix?, column of the head's chunk 0, first row)
  auto kv_coords = [&](const Item &it, int j, bool is_v, int &row, int &col, bool &prefix) {
    if (j < n_pre) {
      prefix = true;
      row = (it.seq * 2 + (is_v ? 1 : 0)) * prm.P + j * BK;
      col = it.hk * HD;
    } else {
      prefix = false;
      row = it.seg0 + (j - n_pre) * BK;
      col = (is_v ? 2 : 1) * prm.C + it.h * HD;
    }
  };

  if (warp < 4) {
  regs_dec<kRegsLow>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      bool ok = true;
      uint32_t J = 0;                 // key tiles loaded so far (ring position)
      uint32_t act[2] = {0, 0};       // items in which each query tile was active
      uint32_t issued = 0, issued_par = 0, q_issued = 0;
      for (int k = 0; ok; ++k) {
        Unit u;
        const int gu = get_unit(k, prm, sk, BK, u, snake);
        if (gu == 0) break;
        if (gu == 2) continue;
        const Item &it = u.it;
        // Q tiles: loaded here only when warp 3 has no touch-ups to do; else
        // warp 3 loads them, so this thread never waits for an item's Q
        // buffer to be free and keeps the K/V ring full across items
        for (int t = 0; !kPrep && t < it.n_tiles_q; ++t) {
          // the previous unit's S MMAs of this tile have finished reading Q_t
          if (act[t] > 0 && !mbar_wait(&bars->q_empty[t], (act[t] - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *qt = smem + CF::kQOff + t * CF::kQTile;
          const int row = it.seg0 + it.q0 + t * kBlockQ;
          mbar_arrive_expect_tx(&bars->q_full[t], CF::kQTile);
          tma_load_2d(qt, &tm_q0, &bars->q_full[t], it.h * HD, row);
          tma_load_2d(qt + CF::kQChunk0, &tm_q1, &bars->q_full[t], it.h * HD + 64, row);
          q_issued = (q_issued & ~(3u << (2 * t))) | ((1u | ((act[t] & 1) << 1)) << (2 * t));
          ++act[t];
        }
        for (int j = u.j0; j < u.j1 && ok; ++j, ++J) {
          const int st = J % NS;
          const uint32_t f = (J / NS) & 1;
          if (!mbar_wait(&bars->kv_empty[st], f ^ 1, abort_flag)) { ok = false; break; }
          int row, col;
          bool pre;
          uint8_t *kt = smem + CF::kKOff + st * CF::kKTile;
          uint8_t *vt = smem + CF::kVOff + st * CF::kKTile;
          kv_coords(it, j, false, row, col, pre);
          mbar_arrive_expect_tx(&bars->k_full[st], CF::kKChunk0 + CF::kKChunk1);
          tma_load_2d(kt, pre ? &tm_p0 : &tm_k0, &bars->k_full[st], col, row);
          tma_load_2d(kt + CF::kKChunk0, pre ? &tm_p1 : &tm_k1, &bars->k_full[st], col + 64, row);
          kv_coords(it, j, true, row, col, pre);
          mbar_arrive_expect_tx(&bars->v_full[st], CF::kVChunks * CF::kVChunk);
          if (HD == 72) {
#pragma unroll
            for (int c = 0; c < CF::kVChunks; ++c)
              tma_load_2d(vt + c * CF::kVChunk, pre ? &tm_p1 : &tm_k1, &bars->v_full[st],
                          col + 16 * c, row);
          } else {
            tma_load_2d(vt, pre ? &tm_p0 : &tm_k0, &bars->v_full[st], col, row);
            tma_load_2d(vt + CF::kVChunk, pre ? &tm_p1 : &tm_k1, &bars->v_full[st], col + 64, row);
          }
          issued |= 1u << st;
          issued_par = (issued_par & ~(1u << st)) | (f << st);
        }
      }
      if (!ok) {  // wait (bounded) for the copies still in flight before the CTA exits
        for (int t = 0; t < 2; ++t)
          if (q_issued & (1u << (2 * t))) drain_wait(&bars->q_full[t], (q_issued >> (2 * t + 1)) & 1);
        for (int s = 0; s < NS; ++s)
          if (issued & (1u << s)) {
            drain_wait(&bars->k_full[s], (issued_par >> s) & 1);
            drain_wait(&bars->v_full[s], (issued_par >> s) & 1);
          }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    const int t = warp - 1;  // query tile served by this warp
    if (elect_one()) {
      bool ok = true, any = false;
      const uint32_t qa = smem_u32(smem + CF::kQOff + t * CF::kQTile);
      const uint32_t k_ring = smem_u32(smem + CF::kKOff);
      const uint32_t sv = smem_u32(smem + CF::kVOff);
      const uint32_t s_tm = tmem + CF::tmem_s(t), p_tm = tmem + CF::tmem_p(t),
                     o_tm = tmem + CF::tmem_o(t);
      // S_t = Q_t K_j^T over HDP/16 k-steps
      auto issue_s = [&](int st) {
        const uint32_t ka = k_ring + st * CF::kKTile;
#pragma unroll
        for (int k = 0; k < CF::HDP / 16; ++k) {
          uint64_t ad, bd;
          if (k < 4) {
            ad = smem_desc(qa + k * 32, 16, 1024, 2);
            bd = smem_desc(ka + k * 32, 16, 1024, 2);
          } else if (HD == 72) {
            ad = smem_desc(qa + CF::kQChunk0, 16, 256, 6);
            bd = smem_desc(ka + CF::kKChunk0, 16, 256, 6);
          } else {
            ad = smem_desc(qa + CF::kQChunk0 + (k - 4) * 32, 16, 1024, 2);
            bd = smem_desc(ka + CF::kKChunk0 + (k - 4) * 32, 16, 1024, 2);
          }
          mma_bf16_ss(s_tm, ad, bd, CF::kIdescS, k > 0);
        }
      };
      // O_t += P_t V_j; P_t is bf16 in its own TMEM columns (2 keys per column)
      auto issue_pv = [&](int st, bool acc) {
        const uint32_t va = sv + st * CF::kKTile;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint32_t accf = (acc || k > 0) ? 1u : 0u;
          // V is the MN-major B operand: 16 keys (rows) per k-step, the
          // column chunks kVChunk bytes apart along N
          const uint64_t bd = HD == 72 ? smem_desc(va + k * 512, CF::kVChunk, 256, 6)
                                       : smem_desc(va + k * 2048, CF::kVChunk, 1024, 2);
          mma_bf16_ts(o_tm, p_tm + k * 8, bd, CF::kIdescPV, accf);
        }
      };
      auto wait_k = [&](uint32_t J) -> bool {
        const int st = J % NS;
        const uint32_t f = (J / NS) & 1;
        return ROPE ? mbar_wait(&bars->k_ready[st], f, abort_flag)
                    : mbar_wait(&bars->k_full[st], f, abort_flag);
      };
      uint32_t J = 0;     // ring position (key tiles of all items so far)
      uint32_t tc = 0;    // key tiles processed by this query tile so far
      uint32_t act = 0;   // items in which this query tile was active
      for (int k = 0; ok; ++k) {
        Unit u;
        const int gu = get_unit(k, prm, sk, BK, u, snake);
        if (gu == 0) break;
        if (gu == 2) continue;
        const Item &it = u.it;
        const int n_kv = u.j1 - u.j0;  // key tiles of this unit
        if (t >= it.n_tiles_q) {  // tile 0's issuer commits this tile's share of kv_empty
          J += n_kv;
          continue;
        }
        const bool alone = it.n_tiles_q == 1;
        // Q_t loaded and prepared; S_t of the previous item loaded by the softmax
        if (!mbar_wait(kPrep ? &bars->q_ready[t] : &bars->q_full[t], act & 1, abort_flag) ||
            (tc > 0 && !mbar_wait(&bars->s_free[t], (tc - 1) & 1, abort_flag)) || !wait_k(J)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(J % NS);
        mma_commit(&bars->s_full[t]);
        if (n_kv == 1) mma_commit(&bars->q_empty[t]);
        any = true;
        for (int j = 0; j < n_kv; ++j) {
          const uint32_t Jj = J + j, tj = tc + j;
          const int st = Jj % NS;
          // S_t(j+1) as soon as the softmax threads hold S_t(j) in registers
          if (j + 1 < n_kv) {
            if (!wait_k(Jj + 1) || !mbar_wait(&bars->s_free[t], tj & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s((Jj + 1) % NS);
            mma_commit(&bars->s_full[t]);
            if (j + 2 == n_kv) mma_commit(&bars->q_empty[t]);  // last S of the item: Q_t free after it
          }
          if (!mbar_wait(HD == 72 ? &bars->v_ready[st] : &bars->v_full[st], (Jj / NS) & 1, abort_flag) ||
              !mbar_wait(&bars->p_full[t], tj & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(st, j > 0);  // j counts this unit's tiles
          mma_commit(&bars->o_done[t]);
          mma_commit(&bars->kv_empty[st]);  // this tile is done with K_j and V_j
          if (alone) mma_commit(&bars->kv_empty[st]);
        }
        J += n_kv;
        tc += n_kv;
        ++act;
      }
      if (!ok && any) {
        mma_commit(&bars->drain[t]);
        drain_wait(&bars->drain[t], 0);
      }
    }
  } else if (warp == 3 && kPrep) {
    // ------------------------------------------------------------ Q loads, Q, K, V touch-ups
    // lane 0 loads each item's Q tiles as soon as the previous item's last S
    // has read the buffer; the warp then prepares them.  Thread handles rows
    // lane, lane + 32, ... of each tile
    uint32_t J = 0;
    uint32_t act[2] = {0, 0};
    uint32_t q_issued = 0;  // lane 0: per tile, a load in flight and its parity
    bool ok = true;
    for (int k = 0; ok; ++k) {
      Unit u;
      const int gu = get_unit(k, prm, sk, BK, u, snake);
      if (gu == 0) break;
      if (gu == 2) continue;
      const Item &it = u.it;
      for (int t = 0; t < it.n_tiles_q; ++t) {
        int okq = 1;
        if (lane == 0) {
          // the previous unit's S MMAs of this tile have finished reading Q_t
          if (act[t] > 0) okq = mbar_wait(&bars->q_empty[t], (act[t] - 1) & 1, abort_flag);
          if (okq) {
            uint8_t *qt = smem + CF::kQOff + t * CF::kQTile;
            const int row = it.seg0 + it.q0 + t * kBlockQ;
            mbar_arrive_expect_tx(&bars->q_full[t], CF::kQTile);
            tma_load_2d(qt, &tm_q0, &bars->q_full[t], it.h * HD, row);
            tma_load_2d(qt + CF::kQChunk0, &tm_q1, &bars->q_full[t], it.h * HD + 64, row);
            q_issued = (q_issued & ~(3u << (2 * t))) | ((1u | ((act[t] & 1) << 1)) << (2 * t));
          }
        }
        if (!__shfl_sync(0xffffffffu, okq, 0)) { ok = false; break; }
        if (!mbar_wait(&bars->q_full[t], act[t] & 1, abort_flag)) { ok = false; break; }
        if (lane == 0) q_issued &= ~(1u << (2 * t));  // landed
        uint8_t *qt = smem + CF::kQOff + t * CF::kQTile;
#pragma unroll 1
        for (int r = lane; r < kBlockQ; r += 32) {
          const int qrow = it.q0 + t * kBlockQ + r;
          if (ROPE && qrow < it.len)
            rope_row_smem<HD>(qt, CF::kQChunk0, r, prm.pos[2 * (it.seg0 + qrow)],
                              prm.pos[2 * (it.seg0 + qrow) + 1], fr);
          if (HD == 72)  // zero the 8 padding columns 72..79 (logical unit 9)
            *reinterpret_cast<uint4 *>(qt + unit_offset<HD>(r, 9, CF::kQChunk0)) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->q_ready[t]);
        ++act[t];
      }
      for (int j = u.j0; j < u.j1 && ok; ++j, ++J) {
        const int st = J % NS;
        const uint32_t f = (J / NS) & 1;
        if (ROPE) {
          if (!mbar_wait(&bars->k_full[st], f, abort_flag)) { ok = false; break; }
          if (j >= n_pre) {
#pragma unroll 1
            for (int r = lane; r < BK; r += 32) {
              const int key = (j - n_pre) * BK + r;
              if (key < it.len)
                rope_row_smem<HD>(smem + CF::kKOff + st * CF::kKTile, CF::kKChunk0, r,
                                  prm.pos[2 * (it.seg0 + key)], prm.pos[2 * (it.seg0 + key) + 1], fr);
            }
            fence_proxy_async_smem();
          }
          mbar_arrive(&bars->k_ready[st]);
        }
        if (HD == 72) {
          // V's column 72 (16-byte unit 1 of the fifth 32B-swizzled chunk) = 1.0:
          // O column 72 then accumulates the softmax row sum on the tensor core
          if (!mbar_wait(&bars->v_full[st], f, abort_flag)) { ok = false; break; }
          uint8_t *vt = smem + CF::kVOff + st * CF::kKTile + 4 * CF::kVChunk;
#pragma unroll
          for (int r = lane; r < BK; r += 32)
            *reinterpret_cast<uint16_t *>(vt + r * 32 + ((1 ^ ((r >> 2) & 1)) << 4)) = 0x3F80u;
          fence_proxy_async_smem();
          mbar_arrive(&bars->v_ready[st]);
        }
      }
    }
    if (!ok && lane == 0) {  // Q copies still in flight land before the CTA exits
      for (int t = 0; t < 2; ++t)
        if (q_issued & (1u << (2 * t))) drain_wait(&bars->q_full[t], (q_issued >> (2 * t + 1)) & 1);
    }
  }
  } else {  // warps 4-19
  regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax
    const int sw = warp - 4;
    const int t = sw >> 3;               // query tile of this warp
    const int half = (sw >> 2) & 1;      // which half of the key tile's score columns
    const int quarter = warp & 3;        // TMEM lane quarter
    const int r = quarter * 32 + lane;   // query row inside the tile
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + CF::tmem_s(t) + half * HC;
    const uint32_t s_other = tmem + lane_base + CF::tmem_s(t) + (half ^ 1) * HC;
    const uint32_t p_addr = tmem + lane_base + CF::tmem_p(t) + half * (HC / 2);
    const uint32_t o_addr = tmem + lane_base + CF::tmem_o(t);
    float *xv = reinterpret_cast<float *>(smem + CF::kXOff) + t * 256;  // [phase&1][t][half][row]
    uint64_t *xb = &bars->xchg[t][quarter];
    const float sl2 = prm.scale_log2;
    // head_dim 72: the softmax denominator is accumulated by the tensor core
    // as O column 72 -- warp 3 sets V's first padding column to 1.0 before
    // each P.V -- so the row sum costs no instruction here and sums exactly the
    // bf16 P the numerator uses.  That also lets P be rounded toward zero
    // (one byte permute per pair): the rounding's mean cancels between
    // numerator and denominator and its spread equals round-to-nearest's.
    // head_dim 128 sums in registers and rounds P to nearest.
    constexpr bool kSumByMma = (HD == 72);
    // pairs of this thread's HC exponentials that run on the FMA pipe
    // instead of the special-function unit (about a tenth)
    constexpr int kPolyPairs = HC / 16;
    constexpr int kOC = CF::HDP / 16;         // 16-column chunks of O
    constexpr int kOCHalf = (kOC + 1) / 2;   // rescaled by half 0; the rest by half 1
    const int oc_lo = half ? kOCHalf : 0, oc_hi = half ? kOC : kOCHalf;
    bool ok = true;
    uint32_t tc = 0;    // key tiles processed by this query tile so far
    uint32_t xc = 0;    // row-pair exchanges so far
    uint32_t act = 0;   // units in which this query tile was active
    uint32_t pc = 0;    // split units in which this query tile was active
    uint32_t pd = 0;    // split units (tile 0: phases of part_done)
    for (int k = 0; ok; ++k) {
      Unit u;
      const int gu = get_unit(k, prm, sk, BK, u, snake);
      if (gu == 0) break;
      if (gu == 2) continue;
      const Item &it = u.it;
      if (t >= it.n_tiles_q) continue;
      const int n_kv = u.j1 - u.j0, len = it.len;  // n_kv: this unit's key tiles
      const int qrow = it.q0 + t * kBlockQ + r;  // row inside the sequence
      float m = -INFINITY;
      uint64_t l2[2] = {0, 0};  // packed partial row sums (head_dim 128)
      for (int j = 0; j < n_kv; ++j) {
        const uint32_t tj = tc + j;
        if (!warp_wait(&bars->s_full[t], tj & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int ja = u.j0 + j;  // key tile of the item
        const int nv_tile = ja < n_pre ? min(BK, prm.P - ja * BK) : min(BK, len - (ja - n_pre) * BK);
        const int nvalid = nv_tile - half * HC;  // valid keys among this thread's columns
        // the row max needs the other half's scores too: read them from TMEM
        // and keep only their maximum (cheaper than a hand-off between the
        // two threads of the row)
        const float m_other = tmem_rowmax<HC>(s_other, nv_tile - (half ^ 1) * HC);
        uint32_t s[HC];
        __syncwarp();
        tmem_ld_cols<HC>(s_addr, s);
        tmem_ld_wait();
        tc_fence_before();
        // S_t may now be overwritten by the next key tile: the loads are
        // complete (tcgen05.wait::ld), so the arrival is relaxed and does not
        // wait for this thread's output stores of the previous item
        mbar_arrive_relaxed(&bars->s_free[t]);
        if (nvalid < HC) {  // keys past the sequence end: -inf, so p = 0
#pragma unroll
          for (int i = 0; i < HC; ++i)
            if (i >= nvalid) s[i] = 0xFF800000u;
        }
        float a0 = __uint_as_float(s[0]), a1 = __uint_as_float(s[1]);
#pragma unroll
        for (int i = 2; i + 3 < HC; i += 4) {
          a0 = fmax3(a0, __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
          a1 = fmax3(a1, __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
        }
        if constexpr ((HC - 2) % 4 != 0)
          a0 = fmax3(a0, __uint_as_float(s[HC - 2]), __uint_as_float(s[HC - 1]));
        const float m_tile = fmax3(a0, a1, m_other) * sl2;
        // The row max only matters when it grows by more than 8 (log2 units)
        // over the running max m: then O (and the row sum) is rescaled.
        // Otherwise m stays (stale) and the final O / l division absorbs it
        // exactly.  (Starting the exponentials with m before the partner's
        // max arrives measured slower.)
        if (j == 0) {
          m = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m + 8.0f)) {
          const bool mine = m_tile > m + 8.0f;
          const float m_new = mine ? m_tile : m;
          const float factor = mine ? ex2_approx(m - m_new) : 1.0f;
          const uint64_t f2 = f2_pack(factor, factor);
          if (!warp_wait(&bars->o_done[t], (tj - 1) & 1, abort_flag)) { ok = false; break; }
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
        // p = 2^(s*scale*log2e - m) two at a time, packed bf16 pairs; stored
        // to P_t in two pieces (the first once O_t += P_t V_{j-1} has read
        // the previous P_t, which by then has normally finished)
        constexpr int NP = HC / 2, NP0 = NP >= 16 ? 16 : NP;
        uint32_t pk[NP];
        const uint64_t sc2 = f2_pack(sl2, sl2);
        auto exp_pairs = [&](auto i0c, auto i1c) {
          constexpr int i0 = decltype(i0c)::value, i1 = decltype(i1c)::value;
          const uint64_t nm2 = f2_pack(-m, -m);
          uint64_t lsum[2] = {0, 0};
#pragma unroll
          for (int i = i0; i < i1; ++i) {
            const uint64_t xa =
                f2_fma(f2_pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), sc2, nm2);
            float p0, p1;
            if (i < kPolyPairs) {  // this share of the exponentials runs on the FMA pipe
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
              lsum[i & 1] = f2_add(lsum[i & 1], f2_pack(p0, p1));
              pk[i] = pack_bf16x2_alu(p0, p1);
            }
          }
          return f2_add(lsum[0], lsum[1]);
        };
        const uint64_t part0 =
            exp_pairs(std::integral_constant<int, 0>{}, std::integral_constant<int, NP0>{});
        if (!kSumByMma) l2[0] = f2_add(l2[0], part0);
        if (j > 0 && !warp_wait(&bars->o_done[t], (tj - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        tmem_st_cols<NP0>(p_addr, pk);
        if constexpr (NP > NP0) {
          const uint64_t part1 =
              exp_pairs(std::integral_constant<int, NP0>{}, std::integral_constant<int, NP>{});
          if (!kSumByMma) l2[1] = f2_add(l2[1], part1);
          tmem_st_cols<NP - NP0>(p_addr + NP0, pk + NP0);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows of o [T, H, HD], each thread its half of the row
      if (!warp_wait(&bars->o_done[t], (tc + n_kv - 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float l = 0.0f;
      if (!kSumByMma) {  // add the two halves' partial sums
        float a, b, c2, d2;
        f2_unpack(l2[0], a, b);
        f2_unpack(l2[1], c2, d2);
        float *xj = xv + (xc & 1) * 512;
        xj[half * 128 + r] = (a + b) + (c2 + d2);
        mbar_arrive(xb);
        if (!warp_wait(xb, xc & 1, abort_flag)) { ok = false; break; }
        l = xj[r] + xj[128 + r];
      }
      __nv_bfloat16 *orow =
          qrow < len ? prm.o + size_t(it.seg0 + qrow) * prm.C + size_t(it.h) * HD : nullptr;
      if constexpr (HD == 72) {
        if (!u.whole) {
          // part of a split item: unnormalised O (column 72 = row sum) and the
          // running max go to this CTA's slot; the last part to finish
          // combines all parts of the item
          const int c = blockIdx.x;
          float *mine = const_cast<float *>(part_rows(prm.part, sk, c, u.w, t)) + size_t(r) * kPartStride;
          if (half == 0)
            store_o_part<HD, 0>(o_addr, mine, m);
          else
            store_o_part<HD, 1>(o_addr, mine, m);
          __syncwarp();
          if (lane == 0) mbar_arrive_cnt(&bars->part_done, it.n_tiles_q == 1 ? 2u : 1u);
          // first and last CTA holding a part of this item
          int c0 = c, c1 = c;
          while (c0 > 0 && !(sk.bw[c0] < u.w || (sk.bw[c0] == u.w && sk.bj[c0] == 0))) --c0;
          while (c1 + 1 < sk.n && (sk.bw[c1 + 1] < u.w || (sk.bw[c1 + 1] == u.w && sk.bj[c1 + 1] < it.n_kv)))
            ++c1;
          if (warp == 4 && lane == 0) {
            bool okp = mbar_wait(&bars->part_done, pd & 1, abort_flag);
            int last = 0;
            if (okp) {
              // part_done ordered every thread's partial rows before this
              // point; the GPU-scope fence releases them (cumulatively)
              // before the count
              __threadfence();
              const int old = atomicAdd(prm.cnt + c0, 1);
              last = old == c1 - c0;
              if (last) {
                prm.cnt[c0] = 0;  // every part has arrived: ready for the next launch
                __threadfence();  // order the other parts' rows before the reads below
              }
            }
            bars->part_last = last;
            for (int tt = 0; tt < it.n_tiles_q; ++tt) mbar_arrive(&bars->part_flag[tt]);
          }
          ++pd;
          if (!warp_wait(&bars->part_flag[t], pc & 1, abort_flag)) { ok = false; break; }
          ++pc;
          if (*reinterpret_cast<volatile int *>(&bars->part_last)) {
            // the counting thread's fence acquired the other parts' rows and
            // part_flag passed that on; they are read through L2
            if (half == 0)
              combine_parts<HD, 0>(prm.part, sk, u.w, t, c0, c1, r, orow);
            else
              combine_parts<HD, 1>(prm.part, sk, u.w, t, c0, c1, r, orow);
          }
          tc += n_kv;
          ++act;
          continue;
        }
      }
      if (half == 0)
        store_o_half<HD, 0>(o_addr, l, orow);
      else
        store_o_half<HD, 1>(o_addr, l, orow);
      tc += n_kv;
      xc += kSumByMma ? 0 : 1;  // the head_dim 128 epilogue swaps the halves' row sums
      ++act;
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
                             const RopeFreqs &fr, const attn::SkTable &sk, cudaStream_t st) {
  using CF = attn::Cfg<HD>;
  auto kern = attention_tc_kernel<HD, ROPE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(CF::kSmem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(attn::kThreads), CF::kSmem, st, 1, maps[0], maps[1],
                    maps[2], maps[3], maps[4], maps[5], prm, fr, sk);
}

int attn_split_max_ctas() { return attn::kMaxSkCtas; }

// The split schedule is opt-in (VIT_ATTN_SPLIT=1): it balances the SMs, but
// the partial rows' round trip and the combine cost more than the balance
// gains at the c2 size (measured 139 against 126 us per launch).
bool attn_split_enabled() {
  static const bool on = [] {
    const char *e = getenv("VIT_ATTN_SPLIT");
    return e != nullptr && atoi(e) != 0;
  }();
  return on;
}

// Whether one sequence of T tokens (no prefix) takes the split schedule at
// head_dim 72 on `grid` CTAs: the same size rules as build_split_table.
bool attn_split_possible(int T, int H, int grid) {
  constexpr int BK = attn::Cfg<72>::BK;
  const long long n_kv = (T + BK - 1) / BK;
  const long long n_pairs = (T + 2 * attn::kBlockQ - 1) / (2 * attn::kBlockQ);
  if (grid <= 0 || grid > attn::kMaxSkCtas || n_kv < 8) return false;
  return n_pairs * H * 4 * n_kv / grid >= 8 * 3;  // upper bound of the real weight
}
size_t attn_split_part_bytes() { return size_t(2) * 2 * attn::kBlockQ * attn::kPartStride * 4; }

// Split schedule for one sequence at head_dim 72 (see SkTable): equal shares
// of the key-tile work (a tile of a two-query-tile item weighs 4, of a
// one-tile item 3, their measured cost ratio), boundaries snapped to item
// edges when within 3 tiles of one.  false: use whole items.
static bool build_split_table(const SeqArgs &s, int H, int n_pairs, int grid, attn::SkTable &sk) {
  constexpr int BK = attn::Cfg<72>::BK;
  const int len = s.total_tokens, P = s.prefix_kv ? s.prefix_len : 0;
  const int n_pre = P > 0 ? (P + BK - 1) / BK : 0;
  const int n_kv = n_pre + (len + BK - 1) / BK;
  const int N = n_pairs * H;
  if (grid > attn::kMaxSkCtas || n_kv < 8) return false;
  std::vector<long long> cum(N + 1, 0);
  for (int w = 0; w < N; ++w) {
    const int q0 = (w / H) * 2 * attn::kBlockQ;
    const int tw = len - q0 > attn::kBlockQ ? 4 : 3;
    cum[w + 1] = cum[w] + (long long)tw * n_kv;
  }
  const long long W = cum[N];
  if (W / grid < 8 * 3) return false;  // shares of at least ~8 key tiles
  sk.n = grid;
  int w = 0;
  for (int c = 0; c <= grid; ++c) {
    const long long B = (long long)c * W / grid;
    while (w < N && cum[w + 1] <= B) ++w;
    int bw = w, bj = 0;
    if (w < N && c < grid) {
      const long long tw = (cum[w + 1] - cum[w]) / n_kv;
      bj = int((B - cum[w] + tw - 1) / tw);
      if (bj < 3) bj = 0;
      if (bj > n_kv - 3) bj = n_kv;
      if (bj >= n_kv) {
        bw = w + 1;
        bj = 0;
      }
    } else {
      bw = N;
      bj = 0;
    }
    sk.bw[c] = bw;
    sk.bj[c] = bj;
  }
  for (int c = 0; c < grid; ++c)  // every share non-empty
    if (!(sk.bw[c] < sk.bw[c + 1] || (sk.bw[c] == sk.bw[c + 1] && sk.bj[c] < sk.bj[c + 1])))
      return false;
  return true;
}

cudaError_t launch_attention_tc(const void *qkv, void *o, const SeqArgs &s, int H, int d,
                                float scale, const RopeFreqs &fr, int num_sms, int *status,
                                float *part, int *cnt, cudaStream_t st) {
  if (s.total_tokens == 0 || s.max_seqlen == 0) return cudaSuccess;
  const int C = H * d;
  const int Hkv = s.kv_heads > 0 ? s.kv_heads : H;
  const int P = s.prefix_kv ? s.prefix_len : 0;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool small = (d == 72);
  const uint32_t bk = small ? attn::Cfg<72>::BK : attn::Cfg<128>::BK;
  const uint32_t w1 = small ? 16 : 64;  // inner box of a tile's second chunk
  const auto sw1 = small ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  // maps: Q chunk 0/1 (128-row boxes), K/V chunk 0/1 (key-tile boxes), prefix chunk 0/1
  CUtensorMap maps[6];
  bool good = true;
  // qkv viewed as [T, 3C]
  good &= encode_tensor_map_2d(&maps[0], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, 64,
                               attn::kBlockQ, CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS;
  good &= encode_tensor_map_2d(&maps[1], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, w1,
                               attn::kBlockQ, sw1) == CUDA_SUCCESS;
  good &= encode_tensor_map_2d(&maps[2], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, 64, bk,
                               CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS;
  good &= encode_tensor_map_2d(&maps[3], BF, qkv, 3ull * C, s.total_tokens, 6ull * C, w1, bk,
                               sw1) == CUDA_SUCCESS;
  if (P > 0) {
    // prefix viewed as [S * 2 * P, Hkv * d]
    const uint64_t rows = uint64_t(s.n_seqs) * 2 * P;
    good &= encode_tensor_map_2d(&maps[4], BF, s.prefix_kv, uint64_t(Hkv) * d, rows,
                                 uint64_t(Hkv) * d * 2, 64, bk, CU_TENSOR_MAP_SWIZZLE_128B) ==
            CUDA_SUCCESS;
    good &= encode_tensor_map_2d(&maps[5], BF, s.prefix_kv, uint64_t(Hkv) * d, rows,
                                 uint64_t(Hkv) * d * 2, w1, bk, sw1) == CUDA_SUCCESS;
  } else {
    maps[4] = maps[2];
    maps[5] = maps[3];
  }
  if (!good) return cudaErrorInvalidValue;
  attn::Params prm;
  prm.H = H;
  prm.C = C;
  prm.Hkv = Hkv;
  prm.P = P;
  // Items of one query tile when even those fit in one round over the SMs
  // (short sequences: twice the CTAs at work, each tile's softmax without a
  // second tile beside it); else pairs sharing each K/V tile.
  const long long single_items =
      (long long)((s.max_seqlen + attn::kBlockQ - 1) / attn::kBlockQ) * H * s.n_seqs;
  prm.tpi = single_items <= num_sms ? 1 : 2;
  prm.n_pairs = (s.max_seqlen + prm.tpi * attn::kBlockQ - 1) / (prm.tpi * attn::kBlockQ);
  prm.snake = 0;  // set below for packed sequences on the persistent kernel
  prm.n_seqs = s.n_seqs;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu = s.cu_seqlens;
  prm.pos = s.pos;
  prm.o = static_cast<__nv_bfloat16 *>(o);
  prm.status = status;
  prm.part = part;
  prm.cnt = cnt;
  const int n_items = prm.n_pairs * H * s.n_seqs;
  // persistent (one CTA per SM walking the items) or one CTA per item
  static const int grid_mode = [] {
    const char *e = getenv("VIT_ATTN_GRID");
    return e ? atoi(e) : 0;
  }();
  const bool persistent = grid_mode == 1 || (grid_mode == 0 && d == 72);
  int grid = (persistent && n_items > num_sms) ? num_sms : n_items;
  attn::SkTable sk;
  sk.n = 0;
  if (d == 72 && s.n_seqs == 1 && part && cnt && persistent && prm.tpi == 2 &&
      attn_split_enabled() &&
      !build_split_table(s, H, prm.n_pairs, std::min(num_sms, attn::kMaxSkCtas), sk))
    sk.n = 0;
  if (sk.n) grid = sk.n;
  // several sequences of (possibly) different lengths: the snake schedule
  if (d == 72 && persistent && sk.n == 0 && prm.tpi == 2 && s.n_seqs > 1 &&
      s.n_seqs <= attn::kMaxSnakeSeqs && n_items > grid)
    prm.snake = 1;
  const bool rope = s.pos != nullptr;
  if (d == 72)
    return rope ? launch_hd<72, true>(maps, prm, grid, fr, sk, st)
                : launch_hd<72, false>(maps, prm, grid, fr, sk, st);
  return rope ? launch_hd<128, true>(maps, prm, grid, fr, sk, st)
              : launch_hd<128, false>(maps, prm, grid, fr, sk, st);
}

}  // namespace vit
