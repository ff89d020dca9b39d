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
//  * one CTA = one (batch, head) and 256 query rows held as two 128-row tiles;
//  * warp 8 streams K_j and V_j (128 x d bf16) through a ring of shared-memory
//    stages with TMA (128-byte swizzle) and mbarrier full/empty pairs;
//  * warp 9 issues tcgen05.mma from one thread: S_t = Q_t K_j^T into TMEM
//    (fp32, 128 lanes x 128 columns per tile), then O_t += P_t V_j with P_t read
//    straight from TMEM (bf16 packed over the first 64 columns of S_t);
//  * warps 0-7 do the softmax of one Q tile at a time (tile 0, then tile 1, per key
//    tile): warps 0-3 take key columns 0-63 and warps 4-7 columns 64-127 of the
//    same 128 rows (one TMEM lane per row), so all eight warps keep the exponential
//    unit busy while the MMA warp computes the other tile's products; both halves
//    read the whole row of scores for the row max, and each half publishes its P
//    columns to the MMA warp as soon as they are stored;
//  * TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,256+d) O_1 [256+d,256+2d).
#pragma once

#include <math.h>

#include "ptx.cuh"

namespace fa {

struct FwdParams {
  int B, H, N;
  int num_qblocks;   // ceil(N / 256): CTAs per (batch, head)
  int head_group;    // heads scheduled together (divides B*H), for L2 reuse of K/V
  int nkv_total;     // ceil(N / 128): key tiles per head
  float scale_log2;  // scale * log2(e)
  uint16_t* out;     // [B, N, H, d] bf16
  float* lse;        // [B, H, N] fp32, natural log
};

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 6;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barrier indices
  static constexpr int kQFull = 0;                      // [2]
  static constexpr int kKVFull = 2;                     // [kStages]
  static constexpr int kKVEmpty = 2 + kStages;          // [kStages]
  static constexpr int kSFull = 2 + 2 * kStages;        // [2]
  static constexpr int kPHalf = kSFull + 2;             // [2 tiles][2 key halves]
  static constexpr int kOFinal = kPHalf + 4;            // [2]
  static constexpr int kDrain = kOFinal + 2;            // [1]
  static constexpr int kNumBars = kDrain + 1;
  // Exchange between the two column halves of a row: maxima [tile][half][128] fp32
  // (exact steps only) and exp-sums [tile][half][128] fp32 (epilogue).
  static constexpr int kXMaxOff = kBarOff + kNumBars * 8;
  static constexpr int kXSumOff = kXMaxOff + 2 * 2 * 128 * 4;
  static constexpr int kMiscOff = kXSumOff + 2 * 2 * 128 * 4;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
};

// Of every 16 exponential pairs of an unmasked tile, this many use the FMA-pipe
// polynomial (exp2_poly2) instead of the MUFU unit.
#ifndef FA_FWD_POLY_PAIRS
#define FA_FWD_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = FA_FWD_POLY_PAIRS;

// Site ids for timeout reports.
enum : unsigned int { kSiteFwdProducer = 0x101, kSiteFwdMma = 0x102, kSiteFwdSoftmax = 0x103 };

// Max / min of 128 values held as two 64-element halves, with 8 independent
// accumulators so the reduction is 10 dependent steps deep instead of 64.
__device__ __forceinline__ float row_max128(const float (&x)[64], const float (&y)[64]) {
  float acc[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) acc[a] = fmaxf(x[a], y[a]);
#pragma unroll
  for (int c = 8; c < 64; c += 8)
#pragma unroll
    for (int a = 0; a < 8; ++a) acc[a] = max3f(acc[a], x[c + a], y[c + a]);
  return fmaxf(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], max3f(acc[5], acc[6], acc[7])));
}
__device__ __forceinline__ float row_min128(const float (&x)[64], const float (&y)[64]) {
  float acc[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) acc[a] = fminf(x[a], y[a]);
#pragma unroll
  for (int c = 8; c < 64; c += 8)
#pragma unroll
    for (int a = 0; a < 8; ++a) acc[a] = min3f(acc[a], x[c + a], y[c + a]);
  return fminf(min3f(acc[0], acc[1], acc[2]), min3f(acc[3], acc[4], min3f(acc[5], acc[6], acc[7])));
}

// Trace slot of (role, key tile, event) for the traced CTA (block 0).
#define FA_FWD_TR(role, j, e) ((((role) * 128 + ((j) & 127)) * 8) + (e))

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
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
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = warp_id();
  const int lane = lane_id();

  // Work unit: heads are taken in groups of head_group so the CTAs in flight share
  // a few heads' K/V in L2; within a group the heaviest causal row blocks come first.
  const int G = p.head_group;
  const int per_group = G * p.num_qblocks;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int rem = static_cast<int>(blockIdx.x) % per_group;
  const int qb = p.num_qblocks - 1 - rem / G;
  const int bh = grp * G + rem % G;
  const int b = bh / p.H;
  const int h = bh % p.H;
  int row0[2], nkv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    row0[t] = qb * 256 + t * 128;
    const bool valid = row0[t] < p.N;
    nkv[t] = !valid ? 0 : (CAUSAL ? min(row0[t] / 128 + 1, p.nkv_total) : p.nkv_total);
  }
  const int nkv_max = max(nkv[0], nkv[1]);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(L::kQFull + t), 1);
      mbar_init(BAR(L::kSFull + t), 1);
      mbar_init(BAR(L::kPHalf + 2 * t + 0), 128);
      mbar_init(BAR(L::kPHalf + 2 * t + 1), 128);
      mbar_init(BAR(L::kOFinal + t), 1);
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(L::kKVFull + s), 1);
      mbar_init(BAR(L::kKVEmpty + s), 1);
    }
    mbar_init(BAR(L::kDrain), 1);
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

  if (warp == 8) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < 2; ++t) {
        if (nkv[t] == 0) continue;
        mbar_arrive_expect_tx(BAR(L::kQFull + t), L::kTileBytes);
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_4d(sQ + t * L::kTileBytes + bx * 16384, &tmQ, BAR(L::kQFull + t), bx * 64, h,
                      row0[t], b);
      }
      int it = 0;
      for (int j = 0; j < nkv_max; ++j) {
        bool stop = false;
        for (int kv = 0; kv < 2; ++kv) {
          const int s = it % L::kStages;
          const uint32_t ph = (it / L::kStages) & 1;
          if (!wait_bar(BAR(L::kKVEmpty + s), ph ^ 1u, abort_flag, kSiteFwdProducer)) {
            stop = true;
            break;
          }
          FA_TRACE_EVENT(blockIdx.x == 0, FA_FWD_TR(3, j, kv));
          mbar_arrive_expect_tx(BAR(L::kKVFull + s), L::kTileBytes);
          const CUtensorMap* m = kv ? &tmV : &tmK;
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(sKV + s * L::kTileBytes + bx * 16384, m, BAR(L::kKVFull + s), bx * 64, h,
                        j * 128, b);
          ++it;
        }
        if (stop) break;
      }
      // Never leave the CTA with copies in flight.
      for (int k = max(0, it - L::kStages); k < it; ++k)
        drain_wait(BAR(L::kKVFull + k % L::kStages), (k / L::kStages) & 1);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0) drain_wait(BAR(L::kQFull + t), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, 0, 1);
      bool ok = true;
      auto issue_qk = [&](int t, int s) {
        const uint32_t dt = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint64_t ad = sdesc_sw128(sQ + t * L::kTileBytes + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKV + s * L::kTileBytes + koff, 16, 1024);
          umma_ss(dt, ad, bd, kIdQK, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V for keys [64*half, 64*half + 64) of the tile.
      auto issue_pv_half = [&](int t, int s, int half, bool acc) {
        const uint32_t dt = tmem + 256 + t * D;
        const uint32_t at = tmem + t * 128;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = half * 4 + k4;
          const uint64_t bd = sdesc_sw128(sKV + s * L::kTileBytes + kk * 2048, 16384, 1024);
          umma_ts(dt, at + kk * 8, bd, kIdPV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      for (int t = 0; t < 2 && ok; ++t)
        if (nkv[t] > 0) ok = wait_bar(BAR(L::kQFull + t), 0, abort_flag, kSiteFwdMma);
      if (ok) {
        // S_t for key tile 0 (ring load 0).
        ok = wait_bar(BAR(L::kKVFull + 0), 0, abort_flag, kSiteFwdMma);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            if (nkv[t] == 0) continue;
            issue_qk(t, 0);
            umma_commit(BAR(L::kSFull + t));
          }
          umma_commit(BAR(L::kKVEmpty + 0));
        }
      }
      for (int j = 0; j < nkv_max && ok; ++j) {
        const int iv = 2 * j + 1, ik = 2 * j + 2;
        const int sv = iv % L::kStages, sk = ik % L::kStages;
        if (!wait_bar(BAR(L::kKVFull + sv), (iv / L::kStages) & 1, abort_flag, kSiteFwdMma)) {
          ok = false;
          break;
        }
        FA_TRACE_EVENT(blockIdx.x == 0, FA_FWD_TR(0, j, 0));
        tc_fence_after();
        bool k_next = false;
        for (int t = 0; t < 2; ++t) {
          if (j >= nkv[t]) continue;
          // P_t arrives in two key halves; the first half's products start while the
          // softmax warpgroup is still exponentiating the second half.
          if (!wait_bar(BAR(L::kPHalf + 2 * t + 0), j & 1, abort_flag, kSiteFwdMma)) {
            ok = false;
            break;
          }
          FA_TRACE_EVENT(blockIdx.x == 0, FA_FWD_TR(0, j, 1 + 2 * t));
          tc_fence_after();
          issue_pv_half(t, sv, 0, j > 0);
          if (!wait_bar(BAR(L::kPHalf + 2 * t + 1), j & 1, abort_flag, kSiteFwdMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv_half(t, sv, 1, j > 0);
          if (j + 1 < nkv[t]) {
            if (!k_next) {
              if (!wait_bar(BAR(L::kKVFull + sk), (ik / L::kStages) & 1, abort_flag,
                            kSiteFwdMma)) {
                ok = false;
                break;
              }
              tc_fence_after();
              k_next = true;
            }
            issue_qk(t, sk);
            umma_commit(BAR(L::kSFull + t));
          } else {
            umma_commit(BAR(L::kOFinal + t));
          }
          FA_TRACE_EVENT(blockIdx.x == 0, FA_FWD_TR(0, j, 2 + 2 * t));
        }
        if (!ok) break;
        umma_commit(BAR(L::kKVEmpty + sv));
        if (k_next) umma_commit(BAR(L::kKVEmpty + sk));
      }
      // Let every issued MMA finish before TMEM can be released.
      umma_commit(BAR(L::kDrain));
      drain_wait(BAR(L::kDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // All eight warps work on one Q tile at a time (tile 0, then tile 1, for every
    // key tile j): warpgroup `half` takes key columns [64*half, 64*half + 64) of each
    // of the 128 rows, so the exponential unit is shared by two warps per SM
    // sub-partition while the MMA warp runs the other tile's products. The two
    // halves of a row both read the whole row of scores for the row max, and add
    // their exp-sums through shared memory at the end; P is published to the MMA
    // warp per half.
    const int half = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    float* xmax = reinterpret_cast<float*>(smem + L::kXMaxOff);
    float* xsum = reinterpret_cast<float*>(smem + L::kXSumOff);
    const bool tr = blockIdx.x == 0 && threadIdx.x == 0;
    float m[2] = {-INFINITY, -INFINITY};  // running row max per tile (log2 units)
    float l[2] = {0.f, 0.f};              // running exp-sum over this half's columns
    bool ok = true;
    for (int j = 0; j < nkv_max && ok; ++j) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (j >= nkv[t]) continue;  // uniform over the CTA
        const int row_g = row0[t] + r;
        const uint32_t tS = tmem + t * 128 + lane_off;
        const uint32_t tO = tmem + 256 + t * D + lane_off;
        const bool w_ok = __all_sync(0xffffffffu,
                                     wait_bar(BAR(L::kSFull + t), j & 1, abort_flag, kSiteFwdSoftmax));
        FA_TRACE_EVENT(tr, FA_FWD_TR(1 + t, j, 0));
        tc_fence_after();
        uint32_t s0[32], s1[32];
        tmem_ld32(tS + 64 * half, s0);
        tmem_ld32(tS + 64 * half + 32, s1);
        tmem_wait_ld();
        reg_fence32(s0);
        reg_fence32(s1);
        FA_TRACE_EVENT(tr, FA_FWD_TR(1 + t, j, 1));
        float x[64];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(s0[c]);
          x[32 + c] = __uint_as_float(s1[c]);
        }
        const int kbase = j * 128 + 64 * half;  // key index of column 0 of this half
        const bool masked = (CAUSAL && j * 128 == row0[t]) || (j * 128 + 128 > p.N);
        if (masked) {
          // Diagonal or tail tile: scale first, then mask to -inf.
          const int lim = CAUSAL ? min(row_g, p.N - 1) : p.N - 1;
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] = (kbase + c > lim) ? -INFINITY : x[c] * sl2;
        }
        // x holds raw scores (unmasked tile) or scaled, masked scores (masked tile).
        // exps(ms, mx_out): p = 2^(x*sl2 - ms) (resp. 2^(x - ms)) for this half's 64
        // columns, their sum, bf16 P into TMEM, and this half's max of the scaled
        // scores computed alongside on the ALU (8 independent accumulators).
        float rsum = 0.f;
        auto exps = [&](float ms, float& mx_out) {
          const float nms = -ms;
          float rs[4] = {0.f, 0.f, 0.f, 0.f};
          float acc[8];
#pragma unroll
          for (int a8 = 0; a8 < 8; ++a8) acc[a8] = -INFINITY;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = ch * 32 + 2 * i;
              float a = x[c], bb = x[c + 1];
              acc[i & 7] = max3f(acc[i & 7], a, bb);
              if (masked) {
                a -= ms;
                bb -= ms;
              } else {
                fma2(a, bb, a, bb, sl2, sl2, nms, nms);
              }
              if (!masked && i < kPolyPairs) {
                exp2_poly2(a, bb);  // FMA/ALU pipes
              } else {
                a = ex2_approx(a);  // MUFU
                bb = ex2_approx(bb);
              }
              add2(rs[2 * (i & 1)], rs[2 * (i & 1) + 1], rs[2 * (i & 1)], rs[2 * (i & 1) + 1], a, bb);
              pk[i] = pack_bf16x2(a, bb);
            }
            tmem_st16(tS + 32 * half + ch * 16, pk);
          }
          float mxr = fmaxf(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], max3f(acc[5], acc[6], acc[7])));
          mx_out = masked ? mxr : mxr * sl2;
          rsum = (rs[0] + rs[1]) + (rs[2] + rs[3]);
        };
        // Fast path: exponentiate against the current reference max while computing
        // this half's max; if no row of the tile grew past the reference by more than
        // 2^8, P is final (p <= 256 stays exact enough in fp32 and bf16, and O / l stays
        // exact because both use the same reference).
        // The fast/exact choice is uniform over all 256 softmax threads (j and the
        // scale's sign are), so every thread reaches the same named barriers; an
        // abort is folded into the vote and forces the exact path, which ends it.
        bool exact = (j == 0) || !(sl2 >= 0.f);
        float mx_half = -INFINITY;
        if (!exact) {
          exps(m[t], mx_half);
          exact = named_bar_or(1, 256, !w_ok || !(mx_half <= m[t] + 8.f));
          if (!exact) l[t] += rsum;
        }
        if (exact) {
          // Exact path (first tile, negative scale, a grown row, or an abort): the two
          // halves exchange their maxima, move the reference, rescale O, and (re)do
          // the exponentials.
          if (mx_half == -INFINITY) {
            float acc[8];
#pragma unroll
            for (int a8 = 0; a8 < 8; ++a8) acc[a8] = (sl2 >= 0.f || masked) ? -INFINITY : INFINITY;
            if (masked || sl2 >= 0.f) {
#pragma unroll
              for (int c = 0; c < 64; c += 2) acc[(c >> 1) & 7] = max3f(acc[(c >> 1) & 7], x[c], x[c + 1]);
              const float mxr = fmaxf(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], max3f(acc[5], acc[6], acc[7])));
              mx_half = masked ? mxr : mxr * sl2;
            } else {
#pragma unroll
              for (int c = 0; c < 64; c += 2) acc[(c >> 1) & 7] = min3f(acc[(c >> 1) & 7], x[c], x[c + 1]);
              mx_half = fminf(min3f(acc[0], acc[1], acc[2]), min3f(acc[3], acc[4], min3f(acc[5], acc[6], acc[7]))) * sl2;
            }
          }
          float* xm = xmax + t * 256;
          xm[half * 128 + r] = mx_half;
          ok = named_bar_and(1, 256, w_ok);
          if (!ok) break;
          const float mx = fmaxf(mx_half, xm[(half ^ 1) * 128 + r]);
          const float m_new = fmaxf(m[t], mx);
          if (__any_sync(0xffffffffu, m_new > m[t] + 8.f)) {
            const float alpha = ex2_approx(m[t] - m_new);  // 0 on the first tile (m = -inf)
            l[t] *= alpha;
            m[t] = m_new;
            if (j > 0) {
              // Rescale this half of the row's partial output before this tile's
              // products accumulate into it (PV_t(j-1) completed before S_t(j)).
#pragma unroll
              for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[16];
                tmem_ld16(tO + half * (D / 2) + cc * 16, o);
                tmem_wait_ld();
                reg_fence16(o);
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                  float a0, a1;
                  mul2(a0, a1, __uint_as_float(o[c]), __uint_as_float(o[c + 1]), alpha, alpha);
                  o[c] = __float_as_uint(a0);
                  o[c + 1] = __float_as_uint(a1);
                }
                tmem_st16(tO + half * (D / 2) + cc * 16, o);
              }
            }
          }
          // The exchange slots are reused at the next exact step of this tile only
          // after every thread has read them.
          named_bar_sync(1, 256);
          float unused;
          exps(m[t] == -INFINITY ? 0.f : m[t], unused);
          l[t] += rsum;
        }
        FA_TRACE_EVENT(tr, FA_FWD_TR(1 + t, j, 4));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(L::kPHalf + 2 * t + half));
        FA_TRACE_EVENT(tr, FA_FWD_TR(1 + t, j, 2));
      }
    }
    // Epilogue per tile: O / l and the LSE. Each half writes its D/2 output columns.
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (nkv[t] == 0) continue;  // uniform over the CTA
      // Every softmax thread reaches the barrier below, aborted or not; the AND
      // carries the abort so all 256 threads leave together.
      bool w_ok = ok;
      if (w_ok) w_ok = wait_bar(BAR(L::kOFinal + t), 0, abort_flag, kSiteFwdSoftmax);
      w_ok = __all_sync(0xffffffffu, w_ok);
      float* xs = xsum + t * 256;
      xs[half * 128 + r] = l[t];
      ok = named_bar_and(2, 256, w_ok);
      if (!ok) continue;
      const float lt = l[t] + xs[(half ^ 1) * 128 + r];
      tc_fence_after();
      const int row_g = row0[t] + r;
      const uint32_t tO = tmem + 256 + t * D + lane_off + half * (D / 2);
      const float inv_l = (lt > 0.f) ? 1.f / lt : 0.f;
      const bool row_ok = row_g < p.N;
      uint16_t* orow = p.out + ((static_cast<size_t>(b) * p.N + row_g) * p.H + h) * D + half * (D / 2);
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        reg_fence32(o);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (row_ok && half == 0) {
        const float lse = (lt > 0.f) ? (m[t] + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.N + row_g] = lse;
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
