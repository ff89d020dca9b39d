// Fused attention forward for sm_100a: O = softmax(scale * Q K^T, mask) V and the
// per-row log-sum-exp, computed tile by tile with a running row max m and running
// exp-sum l so the N x N score matrix never leaves the SM.
//
// Method: tiling of Q/K/V into blocks kept on chip, the blockwise softmax that
// keeps (m, l) per row and rescales the partial output when m grows, and fusion of
// matmul + softmax + weighted sum into one kernel ("FlashAttention优化Transformer显存
// 与计算效率", sections 2.2.1-2.2.3); fp32 softmax accumulation with bf16 inputs
// and outputs (same page, section 3.2); causal masking (ms-swift FA2/3 page, FA3
// feature list). The LSE output is what the backward pass recomputes from.
//
// B200 design (not the pages' A100/H100 tiling):
//  * a work unit = one (batch, head) and 256 query rows held as two 128-row tiles;
//    the kernel is persistent: one CTA per SM takes units one after another (the
//    first one by block index, the rest from a per-launch ticket counter), so the
//    next unit's Q and K/V loads and first Q K^T products run while the current
//    unit's last products and epilogue finish, instead of every unit paying its
//    pipeline fill and drain on an otherwise idle SM;
//  * the producer warp streams K_j and V_j (128 x d bf16) through a ring of shared-memory
//    stages with TMA (128-byte swizzle) and mbarrier full/empty pairs; the ring runs
//    on across units, and the producer hands each unit to the other roles through a
//    small shared-memory ring with its decoded (batch, head, row block), skipping units
//    with nothing to do (past the end of a shorter sequence);
//  * one MMA warp per Q tile issues tcgen05.mma from one thread: S_t = Q_t K_j^T into
//    TMEM (fp32, 128 lanes x 128 columns per tile), then O_t += P_t V_j with P_t read
//    straight from TMEM (bf16, two keys per column: the P of keys [32g, 32g + 32) over
//    S_t columns [32g, 32g + 16), the column group's own); with two
//    issuing warps the tensor pipe keeps work queued while either one waits on a
//    barrier or a commit;
//  * the softmax warps (four groups of four, each group taking 32 of the 128 key
//    columns of every row, one TMEM lane per row) work on one Q tile at a time
//    (tile 0, then tile 1, per key tile), so all of them keep the exponential unit
//    busy while the tensor pipe computes the other tile's products; exponentials are
//    computed against the current reference max and redone only in the rare steps
//    where a row grew past it; P is published to the tile's MMA warp per 64-key half;
//  * TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,256+d) O_1 [256+d,256+2d).
//    Between units, Q_t is reloaded once the unit's last Q_t K^T has executed and O_t
//    is overwritten (the next unit's first P V) once the epilogue has read it.
#pragma once

#include <math.h>

#include <type_traits>

#include "ptx.cuh"

namespace fa {

struct FwdParams {
  int B, H, N;        // N: sequence length (dense) or the largest one (variable length)
  int num_qblocks;    // ceil(N / 256): units per (batch, head)
  int num_units;      // num_qblocks * B * H
  int head_group;     // heads scheduled together (divides B*H), for L2 reuse of K/V
  int window_left;    // keys visible to query i: [i - window_left, i + window_right];
  int window_right;   // -1 = unbounded on that side (causal: window_right = 0)
  float scale_log2;   // scale * log2(e)
  const int* cu_seqlens;  // NULL: dense [B, N] rows; else [B + 1] token offsets
  int total;          // variable length: tokens in the packed tensors
  long long o_rs;     // elements between consecutive rows (tokens) of out
  uint16_t* out;      // dense: row (b, n) at (b*N + n)*o_rs; variable: token t at t*o_rs
  float* lse;         // dense [B, H, N]; variable [H, total]; fp32, natural log
  unsigned int* ticket;  // zero at launch; unit gridDim.x + k goes to the k-th request
};

// The softmax of a 128-row tile is split over kFwdGroups groups of four warps, each
// taking 128 / kFwdGroups key columns of every row; more groups put more warps on the
// exponential unit at once.
#ifndef FA_FWD_COL_GROUPS
#define FA_FWD_COL_GROUPS 4
#endif
constexpr int kFwdGroups = FA_FWD_COL_GROUPS;
constexpr int kFwdCols = 128 / kFwdGroups;  // key columns per group
constexpr int kFwdSoftmaxWarps = 4 * kFwdGroups;
// Warp roles: softmax warps first, then the TMA producer, then one MMA-issuing warp
// per Q tile. Each tile's products come from their own warp, so one warp's waits and
// commits never leave the tensor pipe without work from the other.
constexpr int kFwdProducerWarp = kFwdSoftmaxWarps;
constexpr int kFwdMmaWarp = kFwdSoftmaxWarps + 1;  // tile t: kFwdMmaWarp + t
constexpr int kFwdThreads = 32 * (kFwdSoftmaxWarps + 3);
static_assert(kFwdGroups == 2 || kFwdGroups == 4, "2 or 4 column groups");
constexpr int kFwdUnitSlots = 4;  // units published ahead of the consumers

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 6;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barrier indices
  static constexpr int kQFull = 0;                      // [2]
  static constexpr int kQEmpty = 2;                     // [2] the unit's last Q_t K^T executed
  static constexpr int kKVFull = 4;                     // [kStages]
  static constexpr int kKVEmpty = 4 + kStages;          // [kStages]
  static constexpr int kSFull = 4 + 2 * kStages;        // [2]
  static constexpr int kPHalf = kSFull + 2;             // [2 tiles][2 key halves]
  static constexpr int kOFinal = kPHalf + 4;            // [2]
  static constexpr int kOFree = kOFinal + 2;            // [2] epilogue has read O_t
  static constexpr int kUnitFull = kOFree + 2;          // [kFwdUnitSlots]
  static constexpr int kUnitEmpty = kUnitFull + kFwdUnitSlots;  // [kFwdUnitSlots]
  static constexpr int kDrain = kUnitEmpty + kFwdUnitSlots;     // [2] one per MMA warp
  static constexpr int kNumBars = kDrain + 2;
  // Exchange between the column groups of a row: maxima [tile][group][128] fp32
  // (exact steps only) and exp-sums [tile][group][128] fp32 (epilogue).
  static constexpr int kXMaxOff = kBarOff + kNumBars * 8;
  static constexpr int kXSumOff = kXMaxOff + 2 * kFwdGroups * 128 * 4;
  static constexpr int kMiscOff = kXSumOff + 2 * kFwdGroups * 128 * 4;
  // kMiscOff: TMEM base, abort flag, then the unit ring: kFwdUnitSlots slots of four
  // ints (unit index or -1 to end, batch, head, row block).
  static constexpr int kBytes = kMiscOff + 16 + 16 * kFwdUnitSlots;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kThreads = kFwdThreads;
  static constexpr uint32_t kTmemCols = 512;
};

// Site ids for timeout reports.
enum : unsigned int {
  kSiteFwdProducer = 0x101,
  kSiteFwdMma = 0x102,
  kSiteFwdSoftmax = 0x103,
  kSiteFwdSeqlens = 0x104
};

// One work unit: (batch, head) and 256 query rows as two 128-row tiles.
struct FwdUnit {
  int b, h;
  int seq0, seqlen, tb;    // first token, length, batch coordinate of the tensor maps
  int row0[2], ka[2], nkv[2];
  int J0, nkv_max;         // key tiles streamed: [J0, J0 + nkv_max); 0 = nothing to do
};

// Work order: heads are taken in groups of head_group so the units in flight share a
// few heads' K/V in L2; within a group the heaviest causal row blocks come first.
// A unit of a variable-length batch that lies past its sequence, or whose cu_seqlens
// entries are invalid (reported once, by the producer), has nkv_max = 0.
// The unit's (batch, head, 256-row block): the integer divisions of the decoding, done
// once per unit by the producer and handed to the other roles through shared memory.
struct FwdUnitId {
  int b, h, qb;
};
__device__ __forceinline__ FwdUnitId fwd_unit_id(const FwdParams& p, int u) {
  const int G = p.head_group;
  const int per_group = G * p.num_qblocks;
  const int grp = u / per_group;
  const int rem = u % per_group;
  const int bh = grp * G + rem % G;
  return FwdUnitId{bh / p.H, bh % p.H, p.num_qblocks - 1 - rem / G};
}

// The rest of the decoding, from the unit's (batch, head, row block).
template <bool CAUSAL, bool GENERAL>
__device__ __forceinline__ FwdUnit fwd_unit(const FwdParams& p, FwdUnitId id, bool report_bad) {
  FwdUnit w;
  const int qb = id.qb;
  w.b = id.b;
  w.h = id.h;
  w.seq0 = 0;
  w.seqlen = p.N;
  w.tb = w.b;
  w.nkv_max = 0;
  if (GENERAL && p.cu_seqlens != nullptr) {
    const int s0 = __ldg(p.cu_seqlens + w.b), s1 = __ldg(p.cu_seqlens + w.b + 1);
    w.seq0 = s0;
    w.seqlen = s1 - s0;
    w.tb = 0;
    if (s0 < 0 || w.seqlen < 0 || w.seqlen > p.N || s1 > p.total) {
      if (report_bad && qb == 0 && w.h == 0) report(kDevBadInput, kSiteFwdSeqlens, w.b);
      return w;
    }
  }
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);
  // Key tiles [ka[t], kb[t]] reach at least one row of Q tile t: rows [r, r + 128)
  // see keys [r - wl, r + 127 + wr] within [0, L).
  int kb[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    w.row0[t] = qb * 256 + t * 128;
    const int lo = wl < 0 ? 0 : max(0, w.row0[t] - wl);
    const int hi = wr < 0 ? w.seqlen - 1 : min(w.seqlen - 1, w.row0[t] + 127 + wr);
    w.ka[t] = lo / 128;
    kb[t] = hi < 0 ? -1 : hi / 128;
    w.nkv[t] = (w.row0[t] < w.seqlen && lo <= hi) ? kb[t] - w.ka[t] + 1 : 0;
  }
  w.J0 = w.nkv[0] > 0 ? (w.nkv[1] > 0 ? min(w.ka[0], w.ka[1]) : w.ka[0]) : w.ka[1];
  const int J1 = w.nkv[1] > 0 ? (w.nkv[0] > 0 ? max(kb[0], kb[1]) : kb[1]) : kb[0];
  w.nkv_max = (w.nkv[0] > 0 || w.nkv[1] > 0) ? J1 - w.J0 + 1 : 0;
  return w;
}

// GENERAL = false compiles the plain dense case (no sequence offsets, no window,
// CAUSAL fixed) with every window and varlen test folded away; GENERAL = true reads
// the window and cu_seqlens from the parameters (CAUSAL is then unused).
template <int D, bool CAUSAL, bool GENERAL>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_u32);
  const uint32_t sQ = base + L::kQOff;
  const uint32_t sKV = base + L::kKVOff;
  const uint32_t bar0 = base + L::kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 16);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = warp_id();
  const int lane = lane_id();
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(L::kQFull + t), 1);
      mbar_init(BAR(L::kQEmpty + t), 1);
      mbar_init(BAR(L::kSFull + t), 1);
      // One arrival per softmax thread whose columns fall in the key half.
      mbar_init(BAR(L::kPHalf + 2 * t + 0), 64 * kFwdGroups);  // keys 0-63
      mbar_init(BAR(L::kPHalf + 2 * t + 1), 64 * kFwdGroups);  // keys 64-127
      mbar_init(BAR(L::kOFinal + t), 1);
      mbar_init(BAR(L::kOFree + t), kFwdSoftmaxWarps);  // one arrival per softmax warp
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(L::kKVFull + s), 1);
      mbar_init(BAR(L::kKVEmpty + s), 2);  // one arrival per MMA warp
    }
    for (int s = 0; s < kFwdUnitSlots; ++s) {
      mbar_init(BAR(L::kUnitFull + s), 1);
      mbar_init(BAR(L::kUnitEmpty + s), kFwdSoftmaxWarps + 2);  // every consumer warp
    }
    mbar_init(BAR(L::kDrain + 0), 1);
    mbar_init(BAR(L::kDrain + 1), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Consumers read the k-th unit of this CTA from slot k % kFwdUnitSlots (index -1 ends
  // the loop). Returns false on an abort (every role then leaves its loop).
  auto next_unit = [&](int k, int* u, FwdUnitId* id) -> bool {
    const int slot = k % kFwdUnitSlots;
    const bool w = __all_sync(0xffffffffu, wait_bar(BAR(L::kUnitFull + slot), (k / kFwdUnitSlots) & 1,
                                                    abort_flag, warp >= kFwdMmaWarp ? kSiteFwdMma : kSiteFwdSoftmax));
    if (!w) return false;
    const volatile int* e = unit_ring + 4 * slot;
    *u = e[0];
    *id = FwdUnitId{e[1], e[2], e[3]};
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(L::kUnitEmpty + slot));
    return true;
  };

  if (warp == kFwdProducerWarp) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;                // ring items issued, over all units
      int qloads[2] = {0, 0};    // Q tile loads issued, per tile
      bool ok = true;
      int u = static_cast<int>(blockIdx.x);
      for (int k = 0; ok; ++k) {
        // Units with nothing to do (past the end of a shorter sequence) are skipped here;
        // the other roles never see them.
        FwdUnitId id{};
        FwdUnit w{};
        for (; u < p.num_units; u = static_cast<int>(gridDim.x + atomicAdd(p.ticket, 1u))) {
          id = fwd_unit_id(p, u);
          w = fwd_unit<CAUSAL, GENERAL>(p, id, true);
          if (w.nkv_max > 0) break;
        }
        // Publish unit k (or the end) once its slot has been read by every consumer.
        const int slot = k % kFwdUnitSlots;
        if (!wait_bar(BAR(L::kUnitEmpty + slot), ((k / kFwdUnitSlots) & 1) ^ 1u, abort_flag, kSiteFwdProducer))
          break;
        const bool last = u >= p.num_units;
        volatile int* e = unit_ring + 4 * slot;
        e[0] = last ? -1 : u;
        e[1] = id.b;
        e[2] = id.h;
        e[3] = id.qb;
        mbar_arrive(BAR(L::kUnitFull + slot));
        if (last) break;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || w.nkv[t] == 0) continue;
          // The previous unit's last Q_t K^T must have read this Q tile.
          if (qloads[t] > 0 &&
              !wait_bar(BAR(L::kQEmpty + t), (qloads[t] - 1) & 1, abort_flag, kSiteFwdProducer)) {
            ok = false;
            continue;
          }
          mbar_arrive_expect_tx(BAR(L::kQFull + t), L::kTileBytes);
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(sQ + t * L::kTileBytes + bx * 16384, &tmQ, BAR(L::kQFull + t), bx * 64, w.h,
                        w.seq0 + w.row0[t], w.tb);
          ++qloads[t];
        }
        for (int j = 0; j < w.nkv_max && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            const int s = it % L::kStages;
            const uint32_t ph = (it / L::kStages) & 1;
            if (!wait_bar(BAR(L::kKVEmpty + s), ph ^ 1u, abort_flag, kSiteFwdProducer)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(BAR(L::kKVFull + s), L::kTileBytes);
            const CUtensorMap* m = kv ? &tmV : &tmK;
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_4d(sKV + s * L::kTileBytes + bx * 16384, m, BAR(L::kKVFull + s), bx * 64, w.h,
                          w.seq0 + (w.J0 + j) * 128, w.tb);
            ++it;
          }
        }
        u = static_cast<int>(gridDim.x + atomicAdd(p.ticket, 1u));
      }
      // Never leave the CTA with copies in flight.
      for (int k = max(0, it - L::kStages); k < it; ++k)
        drain_wait(BAR(L::kKVFull + k % L::kStages), (k / L::kStages) & 1);
      for (int t = 0; t < 2; ++t)
        if (qloads[t] > 0) drain_wait(BAR(L::kQFull + t), (qloads[t] - 1) & 1);
    }
  } else if (warp == kFwdMmaWarp || warp == kFwdMmaWarp + 1) {
    // ------------------------------------------------------------ MMA issuers
    // Warp kFwdMmaWarp + t issues every product of Q tile t, from one thread:
    // S_t = Q_t K_j^T into TMEM columns [128 t, 128 t + 128), then O_t += P_t V_j with
    // P_t read back from the same columns (bf16, two keys per column; keys [32g, 32g + 32)
    // in columns [32g, 32g + 16)), in two key
    // halves so the first half's products start while the softmax warps finish the
    // second. A ring stage is free once both warps have arrived on its empty
    // barrier: a warp that reads the stage commits after its last product on it, a
    // warp that does not (its tile's range ends earlier or starts later) arrives once
    // the stage is loaded, which keeps both arrivals in the phase of that load. The
    // whole warp runs the loop (its operands stay warp-uniform) and elect.sync picks
    // the issuing lane; every wait result is made uniform across the warp before it
    // steers control.
    // The tile index is a template constant in each warp's copy of the loop, so the
    // unit's per-tile fields are indexed statically.
    auto mma_role = [&](auto tile) {
      constexpr int t = decltype(tile)::value;
      constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQt = sQ + t * L::kTileBytes;
      const uint32_t tS = tmem + t * 128;
      const uint32_t tO = tmem + 256 + t * D;
      bool ok = true;
      int x = 0;         // ring items consumed, over all units
      int qwaits = 0;    // Q_t loads waited for
      int steps = 0;     // key steps of tile t done, over all units (P-half parities)
      int ouses = 0;     // units whose O_t was produced (epilogue reads them)
      auto issue_qk = [&](int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint64_t ad = sdesc_sw128(sQt + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKV + s * L::kTileBytes + koff, 16, 1024);
          umma_ss_w(tS, ad, bd, kIdQK, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V for keys [64*half, 64*half + 64) of the tile.
      auto issue_pv_half = [&](int s, int half, bool acc) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = half * 4 + k4;
          const uint64_t bd = sdesc_sw128(sKV + s * L::kTileBytes + kk * 2048, 16384, 1024);
          umma_ts_w(tO, tS + 32 * (kk >> 1) + 8 * (kk & 1), bd, kIdPV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto item_wait = [&](int xi) {
        return __all_sync(0xffffffffu, wait_bar(BAR(L::kKVFull + xi % L::kStages), (xi / L::kStages) & 1,
                                                abort_flag, kSiteFwdMma));
      };
      // Releases ring items [x, to) that this tile does not read.
      auto skip_items = [&](int to) {
        for (; x < to && ok; ++x) {
          ok = item_wait(x);
          if (ok && lane == 0) mbar_arrive(BAR(L::kKVEmpty + x % L::kStages));
        }
      };
      for (int k = 0; ok; ++k) {
        int u = -1;
        FwdUnitId id;
        if (!(ok = next_unit(k, &u, &id)) || u < 0) break;
        const FwdUnit w = fwd_unit<CAUSAL, GENERAL>(p, id, false);
        const int x0 = x;  // first ring item of this unit; item x0 + 2r (+1) = K (V) of key tile J0 + r
        const int n = w.nkv[t];
        const int a = n > 0 ? w.ka[t] - w.J0 : w.nkv_max;
        skip_items(x0 + 2 * a);
        if (n > 0 && ok) {
          ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull + t), qwaits & 1, abort_flag, kSiteFwdMma));
          ++qwaits;
          if (ok) ok = item_wait(x);
          if (ok) {
            tc_fence_after();
            issue_qk(x % L::kStages);
            umma_commit_w(BAR(L::kSFull + t));
            if (n == 1) umma_commit_w(BAR(L::kQEmpty + t));
            umma_commit_w(BAR(L::kKVEmpty + x % L::kStages));
          }
          for (int i = 0; i < n && ok; ++i) {  // i-th key tile of this Q tile
            const int iv = x0 + 2 * (a + i) + 1, ik = iv + 1;
            const int sv = iv % L::kStages, sk = ik % L::kStages;
            ok = item_wait(iv);
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kPHalf + 2 * t + 0), steps & 1, abort_flag, kSiteFwdMma));
            // The first P V of a unit overwrites O_t: the previous unit's epilogue must
            // have read it.
            if (ok && i == 0 && ouses > 0)
              ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kOFree + t), (ouses - 1) & 1, abort_flag, kSiteFwdMma));
            if (!ok) break;
            tc_fence_after();
            issue_pv_half(sv, 0, i > 0);
            if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kPHalf + 2 * t + 1), steps & 1, abort_flag, kSiteFwdMma))))
              break;
            ++steps;
            tc_fence_after();
            issue_pv_half(sv, 1, i > 0);
            const bool more = i + 1 < n;
            if (more) {
              if (!(ok = item_wait(ik))) break;
              tc_fence_after();
              issue_qk(sk);
              umma_commit_w(BAR(L::kSFull + t));
              if (i + 2 == n) umma_commit_w(BAR(L::kQEmpty + t));  // last Q_t K^T of the unit
            } else {
              umma_commit_w(BAR(L::kOFinal + t));
            }
            umma_commit_w(BAR(L::kKVEmpty + sv));
            if (more) umma_commit_w(BAR(L::kKVEmpty + sk));
          }
          if (ok) ++ouses;
          x = x0 + 2 * (a + n);
        }
        // Ring loads after this tile's last key tile.
        skip_items(x0 + 2 * w.nkv_max);
      }
      // Let every issued MMA finish before TMEM can be released.
      umma_commit_w(BAR(L::kDrain + t));
      drain_wait(BAR(L::kDrain + t), 0);
    };
    if (warp == kFwdMmaWarp)
      mma_role(std::integral_constant<int, 0>{});
    else
      mma_role(std::integral_constant<int, 1>{});
  } else {
    // ------------------------------------------------------------ softmax warps
    // The softmax warps work on one Q tile at a time (tile 0, then tile 1, for every
    // key tile j). Group g (warps 4g..4g+3) takes key columns [g*C, g*C + C),
    // C = 128 / kFwdGroups, of each of the 128 rows (one TMEM lane per row), so all
    // softmax warps share the exponential unit on one tile while the tensor pipe runs
    // the other tile's products. Column groups of a row meet in shared memory only
    // on exact steps (row maxima) and at the end (exp-sums).
    constexpr int C = kFwdCols;
    constexpr int NTQ = 32 * kFwdGroups;  // threads of one lane quarter (named barriers)
    const int grp = warp >> 2;
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    // Named barriers of this lane quarter: 1-4 for the per-tile vote and max exchange,
    // 5-8 for the epilogue's exp-sum exchange (0 is __syncthreads).
    const int kBarVote = 1 + wq, kBarEpi = 5 + wq;
    const float sl2 = p.scale_log2;
    float* xmax = reinterpret_cast<float*>(smem + L::kXMaxOff);
    float* xsum = reinterpret_cast<float*>(smem + L::kXSumOff);
    // Phase parities over all units: bit t = parity of the key steps of tile t done
    // (S-full barrier), bit 2 + t = parity of the units of tile t finished (O-final).
    uint32_t par = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u = -1;
      // The warps of a lane quarter share named barriers, so they take the same
      // decision even if an abort lands while some of them are still waiting.
      FwdUnitId id;
      ok = named_bar_and(kBarVote, NTQ, next_unit(k, &u, &id));
      if (!ok || u < 0) break;
      const FwdUnit w = fwd_unit<CAUSAL, GENERAL>(p, id, false);
      const int seqlen = w.seqlen;
      float m[2] = {-INFINITY, -INFINITY};  // running row max per tile (log2 units)
      float l[2] = {0.f, 0.f};              // running exp-sum over this group's columns
      for (int jr = 0; jr < w.nkv_max && ok; ++jr) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int i = jr - (w.ka[t] - w.J0);  // step index within this Q tile's key tiles
          if (i < 0 || i >= w.nkv[t]) continue;  // uniform over the CTA
          const int j = w.J0 + jr;               // key tile
          const int row_g = w.row0[t] + r;
          const int row0t = w.row0[t];
          const uint32_t tS = tmem + t * 128 + lane_off;
          const uint32_t tO = tmem + 256 + t * D + lane_off;
          const bool w_ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kSFull + t), ((par >> t) + i) & 1,
                                                            abort_flag, kSiteFwdSoftmax));
          tc_fence_after();
          float x[C];
          {
            uint32_t s0[32];
#pragma unroll
            for (int q32 = 0; q32 < C / 32; ++q32) {
              tmem_ld32(tS + C * grp + 32 * q32, s0);
              tmem_wait_ld();
              reg_fence32(s0);
#pragma unroll
              for (int c = 0; c < 32; ++c) x[32 * q32 + c] = __uint_as_float(s0[c]);
            }
          }
          tc_fence_before();  // the loads above precede the barrier that lets P be stored
          const int kbase = j * 128 + C * grp;  // key index of this group's column 0
          // A tile needs per-element masking if it reaches past the sequence or outside
          // the window of some row of the Q tile (causal: the diagonal tile).
          const int k0 = j * 128;
          const bool masked = (k0 + 128 > seqlen) || (wl >= 0 && k0 < row0t + 127 - wl) ||
                              (wr >= 0 && k0 + 127 > row0t + wr);
          if (masked) {
            // Diagonal or tail tile: scale first, then mask to -inf.
            const int lim = wr < 0 ? seqlen - 1 : min(row_g + wr, seqlen - 1);
            const int first = wl < 0 ? 0 : row_g - wl;
#pragma unroll
            for (int c = 0; c < C; ++c)
              x[c] = (kbase + c > lim || kbase + c < first) ? -INFINITY : x[c] * sl2;
          }
          // x holds raw scores (unmasked tile) or scaled, masked scores (masked tile).
          // exps(ms): p = 2^(x*sl2 - ms) (resp. 2^(x - ms)) for this group's C columns,
          // their sum into rsum, and bf16 P (two keys per 32-bit word) into pk. store_p()
          // writes pk to TMEM over the first 16 of this group's own 32 S columns, which
          // only this group has read, so P can be stored before the vote; the P V products
          // read the four groups' P from those columns.
          float rsum = 0.f;
          uint32_t pk[C / 32][16];
          auto exps = [&](float ms) {
            const float nms = -ms;
            float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ch = 0; ch < C / 32; ++ch) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = ch * 32 + 2 * i;
                float a = x[c], bb = x[c + 1];
                if (masked) {
                  a -= ms;
                  bb -= ms;
                } else {
                  fma2(a, bb, a, bb, sl2, sl2, nms, nms);
                }
                a = ex2_approx(a);
                bb = ex2_approx(bb);
                add2(rs[2 * (i & 1)], rs[2 * (i & 1) + 1], rs[2 * (i & 1)], rs[2 * (i & 1) + 1], a, bb);
                pk[ch][i] = pack_bf16x2(a, bb);
              }
            }
            rsum = (rs[0] + rs[1]) + (rs[2] + rs[3]);
          };
          auto store_p = [&]() {
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < C / 32; ++ch) tmem_st16(tS + C * grp + ch * 16, pk[ch]);
          };
          // Fast path: exponentiate against the current reference max. If this group's
          // exponentials of every row sum to at most 256, none of them exceeds 2^8, so P
          // is final (p <= 256 stays exact enough in fp32 and bf16, and O / l stays exact
          // because both use the same reference). The check costs one compare on a sum
          // that is needed anyway, instead of a running max over every score. The choice
          // is made per TMEM lane quarter: the groups of a row are the G warps of one
          // quarter (same SMSP), and rows of different quarters never exchange anything.
          // It is uniform over those warps (j and the scale's sign are), so they all reach
          // the same named barriers; an abort is folded into the vote and forces the exact
          // path, which ends it. A NaN or infinite sum fails the compare and also goes
          // exact.
          bool exact = (i == 0) || !(sl2 >= 0.f);
          if (!exact) {
            exps(m[t]);
            store_p();  // own columns: no other group reads them, so no need to wait for the vote
            exact = named_bar_or(kBarVote, NTQ, !w_ok || !(rsum <= 256.f));
            if (!exact) l[t] += rsum;
          }
          if (exact) {
            tmem_wait_st();  // a speculative P from the fast path lands before the exact one
            // Exact path (first tile, negative scale, a grown row, or an abort): the
            // column groups exchange their maxima, move the reference, rescale O, and
            // (re)do the exponentials.
            float mx_grp;
            {
              float acc[8];
              const bool up = masked || sl2 >= 0.f;
#pragma unroll
              for (int a8 = 0; a8 < 8; ++a8) acc[a8] = up ? -INFINITY : INFINITY;
              if (up) {
#pragma unroll
                for (int c = 0; c < C; c += 2) acc[(c >> 1) & 7] = max3f(acc[(c >> 1) & 7], x[c], x[c + 1]);
                const float mxr = fmaxf(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], max3f(acc[5], acc[6], acc[7])));
                mx_grp = masked ? mxr : mxr * sl2;
              } else {
#pragma unroll
                for (int c = 0; c < C; c += 2) acc[(c >> 1) & 7] = min3f(acc[(c >> 1) & 7], x[c], x[c + 1]);
                mx_grp = fminf(min3f(acc[0], acc[1], acc[2]), min3f(acc[3], acc[4], min3f(acc[5], acc[6], acc[7]))) * sl2;
              }
            }
            float* xm = xmax + t * (128 * kFwdGroups);
            xm[grp * 128 + r] = mx_grp;
            ok = named_bar_and(kBarVote, NTQ, w_ok);
            if (!ok) break;
            float mx = mx_grp;
#pragma unroll
            for (int g2 = 0; g2 < kFwdGroups; ++g2) mx = fmaxf(mx, xm[g2 * 128 + r]);
            const float m_new = fmaxf(m[t], mx);
            if (__any_sync(0xffffffffu, m_new > m[t] + 8.f)) {
              // 0 while the row has seen no visible key (m = -inf; this also covers a row
              // whose keys so far were all outside its window: -inf - -inf must not give NaN).
              const float alpha = m[t] == -INFINITY ? 0.f : ex2_approx(m[t] - m_new);
              l[t] *= alpha;
              m[t] = m_new;
              if (i > 0) {
                // Rescale this group's D/G columns of the row's partial output before this
                // tile's products accumulate into it (PV_t(j-1) completed before S_t(j)).
#pragma unroll
                for (int cc = 0; cc < D / kFwdGroups / 16; ++cc) {
                  uint32_t o[16];
                  tmem_ld16(tO + grp * (D / kFwdGroups) + cc * 16, o);
                  tmem_wait_ld();
                  reg_fence16(o);
#pragma unroll
                  for (int c = 0; c < 16; c += 2) {
                    float a0, a1;
                    mul2(a0, a1, __uint_as_float(o[c]), __uint_as_float(o[c + 1]), alpha, alpha);
                    o[c] = __float_as_uint(a0);
                    o[c + 1] = __float_as_uint(a1);
                  }
                  tmem_st16(tO + grp * (D / kFwdGroups) + cc * 16, o);
                }
              }
            }
            // The exchange slots are reused at the next exact step of this tile only
            // after every thread has read them.
            named_bar_sync(kBarVote, NTQ);
            exps(m[t] == -INFINITY ? 0.f : m[t]);
            l[t] += rsum;
            store_p();
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(BAR(L::kPHalf + 2 * t + (grp * C) / 64));
        }
      }
      // Epilogue per tile: O / l and the LSE. Each group writes its D/G output columns.
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (w.nkv[t] == 0) continue;  // uniform over the CTA
        const uint32_t ofin = (par >> (2 + t)) & 1u;
        par ^= ((static_cast<uint32_t>(w.nkv[t]) & 1u) << t) | (1u << (2 + t));
        // Every softmax thread reaches the barrier below, aborted or not; the AND
        // carries the abort so all of them leave together.
        bool w_ok = ok;
        if (w_ok) w_ok = wait_bar(BAR(L::kOFinal + t), ofin, abort_flag, kSiteFwdSoftmax);
        w_ok = __all_sync(0xffffffffu, w_ok);
        float* xs = xsum + t * (128 * kFwdGroups);
        xs[grp * 128 + r] = l[t];
        ok = named_bar_and(kBarEpi, NTQ, w_ok);
        if (!ok) continue;
        float lt = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < kFwdGroups; ++g2) lt += xs[g2 * 128 + r];
        // The exp-sum slots are reused by the next unit's epilogue only after every
        // thread of the quarter has read them.
        named_bar_sync(kBarEpi, NTQ);
        tc_fence_after();
        const int row_g = w.row0[t] + r;
        constexpr int DG = D / kFwdGroups;  // output columns of this group
        const uint32_t tO = tmem + 256 + t * D + lane_off + grp * DG;
        const float inv_l = (lt > 0.f) ? 1.f / lt : 0.f;
        const bool row_ok = row_g < seqlen;
        const long long tok = (GENERAL && p.cu_seqlens != nullptr ? static_cast<long long>(w.seq0)
                                                                  : static_cast<long long>(w.b) * p.N) +
                              row_g;
        uint16_t* orow = p.out + tok * p.o_rs + w.h * D + grp * DG;
        // Each thread writes its own row, so a warp's store touches 32 rows: one 32-byte
        // store per 16 columns (when the rows allow it) halves those scattered pieces.
        const bool wide = ((reinterpret_cast<uintptr_t>(p.out) | static_cast<uintptr_t>(p.o_rs * 2)) & 31u) == 0;
#pragma unroll
        for (int cc = 0; cc < DG / 16; ++cc) {
          uint32_t o[16];
          tmem_ld16(tO + cc * 16, o);
          tmem_wait_ld();
          reg_fence16(o);
          uint32_t pk[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
          if (row_ok) {
            if (wide) {
              st_global_v8(orow + cc * 16, pk);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + cc * 16);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
        // O_t has been read: the next unit's first P V may overwrite it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(L::kOFree + t));
        if (row_ok && grp == 0) {
          const float lse = (lt > 0.f) ? (m[t] + log2f(lt)) * 0.69314718055994531f : -INFINITY;
          if (GENERAL && p.cu_seqlens != nullptr)
            p.lse[static_cast<size_t>(w.h) * p.total + tok] = lse;
          else
            p.lse[(static_cast<size_t>(w.b) * p.H + w.h) * p.N + row_g] = lse;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
#undef BAR
}

}  // namespace fa
