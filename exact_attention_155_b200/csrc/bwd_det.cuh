// Deterministic attention backward for sm_100a: the same recomputation as bwd.cuh
// (P = exp(scale S - LSE), dV = P^T dO, dP = dO V^T, dS = P * (dP - D),
// dK = scale dS^T Q, dQ = scale dS K; the "重计算 / Recomputation" item of the
// ms-swift FA2/3 page), split into two kernels so that no CTA adds into another's
// output and every gradient element is written once: dQ, dK and dV are bitwise
// repeatable on the same inputs (the flash_attn `deterministic` flag of the MindSpore
// page's 常见问题与解决方案). It runs seven 128 x 128 tile products per (key tile,
// query tile) pair instead of the fused kernel's five, so it is the slower path.
//  * bwd_dkdv_kernel: one CTA per (batch, head, 128-key tile j). K_j and V_j stay in
//    shared memory; the CTA walks the query tiles i that see its keys with Q_i and
//    dO_i double-buffered. Scores are computed transposed (keys on TMEM lanes), so
//    P^T and dS^T are already the A operands of the two accumulating products and
//    both stay in TMEM:
//       S^T  = K Q_i^T      (TMEM cols [0,128), fp32; P^T bf16 over [0,64))
//       dP^T = V dO_i^T     (TMEM cols [128,256), fp32; dS^T bf16 over [128,192))
//       dV  += P^T dO_i     (A = P^T from TMEM)
//       dK  += dS^T Q_i     (A = dS^T from TMEM)
//    Warps 0-7 (one key row per thread, two warpgroups splitting the query columns)
//    turn S^T into P^T and dP^T into dS^T; warp 8 issues TMA; warp 9 issues
//    tcgen05.mma in the order dV(i), S^T(i+1), dK(i), dP^T(i+1), which keeps the
//    tensor pipe busy while the exponentials of the next query tile run.
//  * bwd_dq_kernel: one CTA per (batch, head, 128-query tile i). Q_i and dO_i stay
//    in shared memory and dQ_i accumulates in TMEM over the key tiles j that the
//    queries see, streamed through a ring of shared-memory stages:
//       S  = Q_i K_j^T      (TMEM, two buffers so S(j+2) is computed during dQ(j))
//       dP = dO_i V_j^T     (into the same buffer once S has been read)
//       dQ += dS K_j        (A = dS bf16 in TMEM over the dP buffer)
//    and dQ_i is written once, scaled, as bf16.
// Both read the per-row LSE (log2 units) and D written by bwd_pre_kernel.
#pragma once

#include <math.h>

#include "bwd.cuh"
#include "ptx.cuh"

namespace fa {

// SS product of two 128-row, K-major, 128-byte-swizzled bf16 tiles over the head dim:
// D[tmem] = A B^T with M = N = 128 (K = D).
template <int D>
__device__ __forceinline__ void bwd_issue_ss(uint32_t d_tmem, uint32_t a, uint32_t b) {
  constexpr uint32_t kId = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
    umma_ss_w(d_tmem, sdesc_sw128(a + koff, 16, 1024), sdesc_sw128(b + koff, 16, 1024), kId,
              kk > 0 ? 1u : 0u);
  }
}
// TS product accumulating into a 128 x D fp32 tile: D[tmem] (+)= A B with A a 128 x 128
// bf16 tile in TMEM and B a 128 x D tile in shared memory read MN-major (the contraction
// runs over B's 128 rows). A's values [64h, 64h + 64) sit two per column in columns
// [64h, 64h + 32) (h = 0, 1): each softmax warpgroup writes its half over the first half
// of the columns it read, which the other warpgroup never reads.
template <int D>
__device__ __forceinline__ void bwd_issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                             bool accumulate) {
  constexpr uint32_t kId = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_ts_w(d_tmem, a_tmem + 64 * (kk >> 2) + 8 * (kk & 3), sdesc_sw128(b + kk * 2048, 16384, 1024),
              kId, (accumulate || kk > 0) ? 1u : 0u);
}

// Converts 64 fp32 TMEM values of one row, scaled, to bf16 and stores them as 128
// contiguous bytes (8 x 16-byte stores).
// 64 consecutive values of one output row (a: the first 32, b: the next 32) x mul as
// bf16. Each thread writes its own row, so a warp's store touches 32 rows: with `wide`
// (dst 32-byte aligned) the row goes out in 32-byte pieces, half as many as 16-byte ones.
__device__ __forceinline__ void store_row64(uint16_t* dst, const uint32_t (&a)[32],
                                            const uint32_t (&b)[32], float mul, bool ok, bool wide) {
  if (!ok) return;
  if (wide) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint32_t* s = v < 2 ? a : b;
      const int o = (v & 1) * 16;
      uint32_t w8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        w8[e] = pack_bf16x2(__uint_as_float(s[o + 2 * e]) * mul, __uint_as_float(s[o + 2 * e + 1]) * mul);
      st_global_v8(dst + 16 * v, w8);
    }
    return;
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint32_t* s = v < 4 ? a : b;
    const int o = (v & 3) * 8;
    d4[v] = make_uint4(pack_bf16x2(__uint_as_float(s[o]) * mul, __uint_as_float(s[o + 1]) * mul),
                       pack_bf16x2(__uint_as_float(s[o + 2]) * mul, __uint_as_float(s[o + 3]) * mul),
                       pack_bf16x2(__uint_as_float(s[o + 4]) * mul, __uint_as_float(s[o + 5]) * mul),
                       pack_bf16x2(__uint_as_float(s[o + 6]) * mul, __uint_as_float(s[o + 7]) * mul));
  }
}

// Row stores can be 32 bytes wide when the base and the row stride keep rows 32-byte aligned.
__device__ __forceinline__ bool rows32(const uint16_t* base, long long row_stride) {
  return ((reinterpret_cast<uintptr_t>(base) | static_cast<uintptr_t>(row_stride * 2)) & 31u) == 0;
}

// =============================================================================
// dK / dV
// =============================================================================
template <int D>
struct BwdKVLayout {
  static constexpr int kTile = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kK = 0;
  static constexpr int kV = kTile;
  static constexpr int kQ0 = 2 * kTile;   // [2] Q_i tiles
  static constexpr int kDO0 = 4 * kTile;  // [2] dO_i tiles
  static constexpr int kVec = 6 * kTile;  // [2] x (lse2[128], D[128]) fp32, with Q_i
  static constexpr int kBar = kVec + 2 * 1024;
  static constexpr int kKVFull = 0;
  static constexpr int kQFull = 1;     // [2]
  static constexpr int kQEmpty = 3;    // [2]
  static constexpr int kDOFull = 5;    // [2]
  static constexpr int kDOEmpty = 7;   // [2]
  static constexpr int kSFull = 9;
  static constexpr int kDPFull = 10;
  static constexpr int kPFull = 11;    // 256 arrivals: P^T stored
  static constexpr int kDSFull = 12;   // 256 arrivals: dS^T stored
  static constexpr int kMmaDone = 13;
  static constexpr int kDrain = 14;
  static constexpr int kNumBars = 15;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kBytes <= 232448, "shared memory budget");
};

// GENERAL = false compiles the plain dense case (no sequence offsets, no window,
// CAUSAL fixed); GENERAL = true reads the window and cu_seqlens at run time.
template <int D, bool CAUSAL, bool GENERAL>
__global__ void __launch_bounds__(320, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams p) {
  using L = BwdKVLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {
    // The swizzled tiles need a 1024-byte aligned base; there is no slack to realign.
    if (threadIdx.x == 0) report(kDevTimeout, kSiteBwdSmemAlign, base);
    return;
  }
  const uint32_t sK = base + L::kK, sV = base + L::kV;
  const uint32_t bar0 = base + L::kBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = warp_id(), lane = lane_id();
  // Heads in groups of head_group (L2 reuse of Q and dO); within a group, key tile 0
  // (the most query tiles when causal) first.
  const int G = p.head_group;
  const int per_group = G * p.nqt;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int rem = static_cast<int>(blockIdx.x) % per_group;
  const int jt = rem / G;
  const int bh = grp * G + rem % G;
  const int b = bh / p.H, h = bh % p.H;
  long long tok0 = static_cast<long long>(b) * p.N;  // first token of the sequence
  int seqlen = p.N;
  if (GENERAL && !bwd_seq(p, b, &tok0, &seqlen)) return;  // reported by the preprocessing kernel
  const bool var = GENERAL && p.cu_seqlens != nullptr;
  const int tb = var ? 0 : b;                            // batch coordinate of the maps
  const int trow = var ? static_cast<int>(tok0) : 0;     // row coordinate of row 0
  if (jt * 128 >= seqlen) return;  // key tile past the end of a shorter sequence
  // Query tiles [it0, it0 + niter) see at least one key of this tile: keys
  // [k0, k1] are visible to queries [k0 - wr, k1 + wl] within [0, L).
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);
  const int k0 = jt * 128, k1 = min(seqlen, k0 + 128) - 1;
  const int qlo = wr < 0 ? 0 : max(0, k0 - wr);
  const int qhi = wl < 0 ? seqlen - 1 : min(seqlen - 1, k1 + wl);
  const int it0 = qlo / 128;
  const int niter = qhi / 128 - it0 + 1;  // >= 1: every key sees at least itself

  if (threadIdx.x == 0) {
    mbar_init(BAR(L::kKVFull), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(L::kQFull + s), 1);
      mbar_init(BAR(L::kQEmpty + s), 1);
      mbar_init(BAR(L::kDOFull + s), 1);
      mbar_init(BAR(L::kDOEmpty + s), 1);
    }
    mbar_init(BAR(L::kSFull), 1);
    mbar_init(BAR(L::kDPFull), 1);
    mbar_init(BAR(L::kPFull), 256);
    mbar_init(BAR(L::kDSFull), 256);
    mbar_init(BAR(L::kMmaDone), 1);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;
  auto sQ = [&](int n) { return base + L::kQ0 + static_cast<uint32_t>(n & 1) * L::kTile; };
  auto sDO = [&](int n) { return base + L::kDO0 + static_cast<uint32_t>(n & 1) * L::kTile; };

  if (warp == 8) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(BAR(L::kKVFull), 2 * L::kTile);
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_4d(sK + bx * 16384, &tmK, BAR(L::kKVFull), bx * 64, h, trow + jt * 128, tb);
        tma_load_4d(sV + bx * 16384, &tmV, BAR(L::kKVFull), bx * 64, h, trow + jt * 128, tb);
      }
      const float* lse2_h = p.lse2 + static_cast<size_t>(bh) * p.Np;
      const float* dvec_h = p.dvec + static_cast<size_t>(bh) * p.Np;
      int nq = 0, ndo = 0;  // loads issued
      for (int n = 0; n < niter; ++n) {
        const int it = it0 + n;
        const int s = n & 1;
        const uint32_t ph = ((n >> 1) & 1) ^ 1u;
        if (!wait_bar(BAR(L::kQEmpty + s), ph, abort_flag, kSiteBwdProducer)) break;
        mbar_arrive_expect_tx(BAR(L::kQFull + s), L::kTile + 1024);
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_4d(sQ(n) + bx * 16384, &tmQ, BAR(L::kQFull + s), bx * 64, h, trow + it * 128, tb);
        const uint32_t sv = base + L::kVec + s * 1024;
        bulk_load(sv, lse2_h + it * 128, 512, BAR(L::kQFull + s));
        bulk_load(sv + 512, dvec_h + it * 128, 512, BAR(L::kQFull + s));
        ++nq;
        if (!wait_bar(BAR(L::kDOEmpty + s), ph, abort_flag, kSiteBwdProducer)) break;
        mbar_arrive_expect_tx(BAR(L::kDOFull + s), L::kTile);
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_4d(sDO(n) + bx * 16384, &tmdO, BAR(L::kDOFull + s), bx * 64, h, trow + it * 128, tb);
        ++ndo;
      }
      // Never leave the CTA with copies in flight.
      for (int k = max(0, nq - 2); k < nq; ++k) drain_wait(BAR(L::kQFull + (k & 1)), (k >> 1) & 1);
      for (int k = max(0, ndo - 2); k < ndo; ++k) drain_wait(BAR(L::kDOFull + (k & 1)), (k >> 1) & 1);
      drain_wait(BAR(L::kKVFull), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs the issue loop (the operands stay warp-uniform); elect.sync
    // picks the lane that issues each tcgen05 instruction, and every wait result is
    // made uniform across the warp before it steers control. Issue order per query
    // tile n: dV(n), S^T(n+1), dK(n), dP^T(n+1). The exponentials of tile n+1 run
    // while dK(n) and dP^T(n+1) execute; the dS pass of tile n runs during dV(n) and
    // S^T(n+1). Products execute in issue order, so S^T(n+1) overwrites P^T(n) only
    // after dV(n) has read it, and dP^T(n+1) overwrites dS^T(n) only after dK(n).
    bool ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kKVFull), 0, abort_flag, kSiteBwdMma));
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull), 0, abort_flag, kSiteBwdMma));
    if (ok) {
      tc_fence_after();
      bwd_issue_ss<D>(tS, sK, sQ(0));
      umma_commit_w(BAR(L::kSFull));
      ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDOFull), 0, abort_flag, kSiteBwdMma));
    }
    if (ok) {
      tc_fence_after();
      bwd_issue_ss<D>(tDP, sV, sDO(0));
      umma_commit_w(BAR(L::kDPFull));
    }
    for (int n = 0; n < niter && ok; ++n) {
      const int s = n & 1;
      const bool more = n + 1 < niter;
      const uint32_t ph1 = ((n + 1) >> 1) & 1;
      // dV += P^T dO_n
      if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kPFull), n & 1, abort_flag, kSiteBwdMma)))) break;
      tc_fence_after();
      bwd_issue_ts<D>(tDV, tS, sDO(n), n > 0);
      umma_commit_w(BAR(L::kDOEmpty + s));
      // S^T(n+1) = K Q_{n+1}^T
      if (more) {
        if (!(ok = __all_sync(0xffffffffu,
                              wait_bar(BAR(L::kQFull + (s ^ 1)), ph1, abort_flag, kSiteBwdMma))))
          break;
        tc_fence_after();
        bwd_issue_ss<D>(tS, sK, sQ(n + 1));
        umma_commit_w(BAR(L::kSFull));
      }
      // dK += dS^T Q_n
      if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDSFull), n & 1, abort_flag, kSiteBwdMma)))) break;
      tc_fence_after();
      bwd_issue_ts<D>(tDK, tDP, sQ(n), n > 0);
      umma_commit_w(BAR(L::kQEmpty + s));
      // dP^T(n+1) = V dO_{n+1}^T
      if (more) {
        if (!(ok = __all_sync(0xffffffffu,
                              wait_bar(BAR(L::kDOFull + (s ^ 1)), ph1, abort_flag, kSiteBwdMma))))
          break;
        tc_fence_after();
        bwd_issue_ss<D>(tDP, sV, sDO(n + 1));
        umma_commit_w(BAR(L::kDPFull));
      }
    }
    if (ok) umma_commit_w(BAR(L::kMmaDone));
    umma_commit_w(BAR(L::kDrain));
    drain_wait(BAR(L::kDrain), 0);
  } else if (warp < 8) {
    // ------------------------------------ P^T and dS^T: one key row per thread; two
    // warpgroups split the 128 query columns of every tile (64 columns each).
    const int wq = warp & 3;
    const int half = warp >> 2;
    const int c0 = half * 64;  // first query column of this warpgroup
    const int r = wq * 32 + lane;
    const int key = jt * 128 + r;
    const bool key_ok = key < seqlen;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < niter; ++n) {
      const int it = it0 + n;
      const int s = n & 1;
      const float* vec = reinterpret_cast<const float*>(smem + L::kVec + s * 1024) + c0;
      ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kSFull), n & 1, abort_flag, kSiteBwdSoftmax));
      if (ok)
        ok = __all_sync(0xffffffffu,
                        wait_bar(BAR(L::kQFull + s), (n >> 1) & 1, abort_flag, kSiteBwdSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(tS + lane_off + c0, s0);
      tmem_ld32(tS + lane_off + c0 + 32, s1);
      tmem_wait_ld();
      reg_fence32(s0);
      reg_fence32(s1);
      // Local columns c in [qlo_c, qhi_c] are the queries that see this key (window
      // [key - wr, key + wl]); none if the key is past the sequence. Queries past the
      // sequence have lse2 = +inf, so their P is already 0.
      const int q0 = it * 128 + c0;
      const int qlo_c = !key_ok ? (1 << 30) : (wr < 0 ? -(1 << 30) : key - wr - q0);
      const int qhi_c = wl < 0 ? (1 << 30) : key + wl - q0;
      uint32_t pk[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const int c = 2 * c2;
        const uint32_t* src = c < 32 ? s0 : s1;
        const float e0 = ex2_approx(__uint_as_float(src[c & 31]) * sl2 - vec[c]);
        const float e1 = ex2_approx(__uint_as_float(src[(c + 1) & 31]) * sl2 - vec[c + 1]);
        const float p0 = (c < qlo_c || c > qhi_c) ? 0.f : e0;
        const float p1 = (c + 1 < qlo_c || c + 1 > qhi_c) ? 0.f : e1;
        pk[c2] = pack_bf16x2(p0, p1);
      }
      // P^T of queries [c0, c0 + 64) goes to columns [c0, c0 + 32), over S^T columns this
      // warpgroup has read and the other never reads.
      tc_fence_after();
      tmem_st32(tS + lane_off + c0, pk);  // P^T bf16: two queries per 32-bit column
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(L::kPFull));

      ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDPFull), n & 1, abort_flag, kSiteBwdSoftmax));
      if (!ok) break;
      tc_fence_after();
      const float* dvec = vec + 128;
      uint32_t dp0[32], dp1[32];
      tmem_ld32(tDP + lane_off + c0, dp0);
      tmem_ld32(tDP + lane_off + c0 + 32, dp1);
      tmem_wait_ld();
      reg_fence32(dp0);
      reg_fence32(dp1);
      uint32_t ds[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const uint32_t pp = pk[c2];
        const float p0 = __uint_as_float(pp << 16), p1 = __uint_as_float(pp & 0xFFFF0000u);
        const int c = 2 * c2;
        const uint32_t* dp = c < 32 ? dp0 : dp1;
        const float d0 = p0 * (__uint_as_float(dp[c & 31]) - dvec[c]);
        const float d1 = p1 * (__uint_as_float(dp[(c + 1) & 31]) - dvec[c + 1]);
        ds[c2] = pack_bf16x2(d0, d1);
      }
      // dS^T goes over dP^T the same way P^T goes over S^T.
      tc_fence_after();
      tmem_st32(tDP + lane_off + c0, ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(L::kDSFull));
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kMmaDone), 0, abort_flag, kSiteBwdSoftmax));
    if (ok) {
      // Epilogue: warpgroup 0 writes dV rows, warpgroup 1 writes dK rows (x scale).
      tc_fence_after();
      const uint32_t tsrc = (half == 0 ? tDV : tDK) + lane_off;
      const float mul = half == 0 ? 1.f : p.scale;
      uint16_t* dst = (half == 0 ? p.dv + (tok0 + key) * p.rs_dv : p.dk + (tok0 + key) * p.rs_dk) + h * D;
      const bool wide = half == 0 ? rows32(p.dv, p.rs_dv) : rows32(p.dk, p.rs_dk);
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t a[32], c[32];
        tmem_ld32(tsrc + cc * 64, a);
        tmem_ld32(tsrc + cc * 64 + 32, c);
        tmem_wait_ld();
        reg_fence32(a);
        reg_fence32(c);
        store_row64(dst + cc * 64, a, c, mul, key_ok, wide);
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

// =============================================================================
// dQ
// =============================================================================
template <int D>
struct BwdQLayout {
  static constexpr int kTile = 128 * D * 2;
  // K_j / V_j ring: five 32 KB stages at d = 128 (K_{j+2} loads while dQ(j) still
  // reads K_j), more at d = 64.
  static constexpr int kStages = (D == 128) ? 5 : 10;
  static constexpr int kQ = 0;
  static constexpr int kDO = kTile;
  static constexpr int kRing = 2 * kTile;
  static constexpr int kVec = kRing + kStages * kTile;  // lse2[128], D[128] fp32
  static constexpr int kBar = kVec + 1024;
  static constexpr int kQFull = 0;                   // Q, dO and the row vectors
  static constexpr int kKVFull = 1;                  // [kStages]
  static constexpr int kKVEmpty = 1 + kStages;       // [kStages]
  static constexpr int kSFull = 1 + 2 * kStages;     // [2] per S buffer
  static constexpr int kSFree = kSFull + 2;          // [2] 256 arrivals: S read
  static constexpr int kDPFull = kSFull + 4;         // [2]
  static constexpr int kDSFull = kSFull + 6;         // [2] 256 arrivals: dS stored
  static constexpr int kDQDone = kSFull + 8;
  static constexpr int kDrain = kSFull + 9;
  static constexpr int kNumBars = kDrain + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kThreads = 320;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool CAUSAL, bool GENERAL>
__global__ void __launch_bounds__(320, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdParams p) {
  using L = BwdQLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) report(kDevTimeout, kSiteBwdSmemAlign, base);
    return;
  }
  const uint32_t sQ = base + L::kQ, sDO = base + L::kDO, sRing = base + L::kRing;
  const uint32_t bar0 = base + L::kBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = warp_id(), lane = lane_id();
  // Heads in groups of head_group (their K and V stay in L2 while their CTAs run);
  // within a group the query tiles with the most key tiles (causal) come first.
  const int G = p.head_group;
  const int per_group = G * p.nqt;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int rem = static_cast<int>(blockIdx.x) % per_group;
  const int qt = p.nqt - 1 - rem / G;
  const int bh = grp * G + rem % G;
  const int b = bh / p.H, h = bh % p.H;
  long long tok0 = static_cast<long long>(b) * p.N;
  int seqlen = p.N;
  if (GENERAL && !bwd_seq(p, b, &tok0, &seqlen)) return;  // reported by the preprocessing kernel
  const bool var = GENERAL && p.cu_seqlens != nullptr;
  const int tb = var ? 0 : b;
  const int trow = var ? static_cast<int>(tok0) : 0;
  const int r0 = qt * 128;
  if (r0 >= seqlen) return;  // query tile past the end of a shorter sequence
  // Key tiles [ka, ka + nk) reach at least one row of this tile: rows [r0, r0 + 128)
  // see keys [r0 - wl, r0 + 127 + wr] within [0, L); every row sees itself, so nk >= 1.
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);
  const int lo = wl < 0 ? 0 : max(0, r0 - wl);
  const int hi = wr < 0 ? seqlen - 1 : min(seqlen - 1, r0 + 127 + wr);
  const int ka = lo / 128;
  const int nk = hi / 128 - ka + 1;

  if (threadIdx.x == 0) {
    mbar_init(BAR(L::kQFull), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR(L::kKVFull + s), 1);
      mbar_init(BAR(L::kKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(L::kSFull + t), 1);
      mbar_init(BAR(L::kSFree + t), 256);
      mbar_init(BAR(L::kDPFull + t), 1);
      mbar_init(BAR(L::kDSFull + t), 256);
    }
    mbar_init(BAR(L::kDQDone), 1);
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
  const uint32_t tDQ = tmem + 256;  // S / dP / dS buffers at [0,128) and [128,256)
  // Ring item x is K (x even) or V (x odd) of key tile ka + x / 2.
  auto stage = [&](int x) { return sRing + static_cast<uint32_t>(x % L::kStages) * L::kTile; };

  if (warp == 8) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(BAR(L::kQFull), 2 * L::kTile + 1024);
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_4d(sQ + bx * 16384, &tmQ, BAR(L::kQFull), bx * 64, h, trow + r0, tb);
        tma_load_4d(sDO + bx * 16384, &tmdO, BAR(L::kQFull), bx * 64, h, trow + r0, tb);
      }
      bulk_load(base + L::kVec, p.lse2 + static_cast<size_t>(bh) * p.Np + r0, 512, BAR(L::kQFull));
      bulk_load(base + L::kVec + 512, p.dvec + static_cast<size_t>(bh) * p.Np + r0, 512, BAR(L::kQFull));
      int x = 0;
      for (; x < 2 * nk; ++x) {
        const int s = x % L::kStages;
        if (!wait_bar(BAR(L::kKVEmpty + s), ((x / L::kStages) & 1) ^ 1u, abort_flag, kSiteBwdQProducer))
          break;
        mbar_arrive_expect_tx(BAR(L::kKVFull + s), L::kTile);
        const CUtensorMap* m = (x & 1) ? &tmV : &tmK;
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_4d(stage(x) + bx * 16384, m, BAR(L::kKVFull + s), bx * 64, h,
                      trow + (ka + x / 2) * 128, tb);
      }
      // Never leave the CTA with copies in flight.
      for (int k = max(0, x - L::kStages); k < x; ++k)
        drain_wait(BAR(L::kKVFull + k % L::kStages), (k / L::kStages) & 1);
      drain_wait(BAR(L::kQFull), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    // Key tile i lives in S buffer i % 2: S(i), then dP(i) over it once S has been
    // read, then dS(i) stored over dP by the softmax warps. Issue order per key tile:
    // dQ += dS(i) K_i, dP(i + 1) (S(i + 1) is already in the other buffer), S(i + 2)
    // into buffer i % 2 (executed after dQ(i) has read dS(i)). The exponentials of
    // tile i + 1 run while dQ(i) and dP(i + 1) execute, and S(i + 2) is ready before
    // they end.
    auto kv_wait = [&](int x) {
      return __all_sync(0xffffffffu, wait_bar(BAR(L::kKVFull + x % L::kStages), (x / L::kStages) & 1,
                                              abort_flag, kSiteBwdQMma));
    };
    // dP(i) = dO V_i^T into S buffer i % 2, once the softmax warps have read S(i).
    auto issue_dp = [&](int i) {
      const int bf = i & 1;
      if (!__all_sync(0xffffffffu, wait_bar(BAR(L::kSFree + bf), (i >> 1) & 1, abort_flag, kSiteBwdQMma)))
        return false;
      if (!kv_wait(2 * i + 1)) return false;
      tc_fence_after();
      bwd_issue_ss<D>(tmem + 128 * bf, sDO, stage(2 * i + 1));
      umma_commit_w(BAR(L::kDPFull + bf));
      umma_commit_w(BAR(L::kKVEmpty + (2 * i + 1) % L::kStages));
      return true;
    };
    bool ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull), 0, abort_flag, kSiteBwdQMma));
    for (int i = 0; i < 2 && i < nk && ok; ++i) {
      if (!(ok = kv_wait(2 * i))) break;
      tc_fence_after();
      bwd_issue_ss<D>(tmem + 128 * i, sQ, stage(2 * i));
      umma_commit_w(BAR(L::kSFull + i));
    }
    if (ok) ok = issue_dp(0);
    for (int i = 0; i < nk && ok; ++i) {
      const int bf = i & 1;
      const uint32_t tSP = tmem + 128 * bf;
      // dQ += dS(i) K_i
      if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDSFull + bf), (i >> 1) & 1, abort_flag,
                                                  kSiteBwdQMma))))
        break;
      tc_fence_after();
      bwd_issue_ts<D>(tDQ, tSP, stage(2 * i), i > 0);
      umma_commit_w(BAR(L::kKVEmpty + (2 * i) % L::kStages));
      if (i + 1 < nk && !(ok = issue_dp(i + 1))) break;
      // S(i + 2) = Q K_{i+2}^T
      if (i + 2 < nk) {
        if (!(ok = kv_wait(2 * i + 4))) break;
        tc_fence_after();
        bwd_issue_ss<D>(tSP, sQ, stage(2 * i + 4));
        umma_commit_w(BAR(L::kSFull + bf));
      }
    }
    if (ok) umma_commit_w(BAR(L::kDQDone));
    umma_commit_w(BAR(L::kDrain));
    drain_wait(BAR(L::kDrain), 0);
  } else if (warp < 8) {
    // ------------------------------------ P and dS: one query row per thread; two
    // warpgroups split the 128 key columns of every key tile (64 columns each).
    const int wq = warp & 3;
    const int half = warp >> 2;
    const int c0 = half * 64;  // first key column of this warpgroup
    const int r = wq * 32 + lane;
    const int q = r0 + r;      // query row in the sequence
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull), 0, abort_flag, kSiteBwdQSoftmax));
    const float* vec = reinterpret_cast<const float*>(smem + L::kVec);
    const float lse2_r = ok ? vec[r] : 0.f;
    const float d_r = ok ? vec[128 + r] : 0.f;
    // Visible keys of this row: [q - wl, q + wr] within [0, L).
    const int klo = wl < 0 ? 0 : q - wl;
    const int khi = wr < 0 ? seqlen - 1 : min(q + wr, seqlen - 1);
    for (int i = 0; i < nk && ok; ++i) {
      const int bf = i & 1;
      const uint32_t ph = (i >> 1) & 1;
      const uint32_t tSP = tmem + 128 * bf + lane_off;
      const int k0 = (ka + i) * 128;
      ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kSFull + bf), ph, abort_flag, kSiteBwdQSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(tSP + c0, s0);
      tmem_ld32(tSP + c0 + 32, s1);
      tmem_wait_ld();
      reg_fence32(s0);
      reg_fence32(s1);
      tc_fence_before();
      mbar_arrive(BAR(L::kSFree + bf));  // dP(i) may now overwrite S(i)
      // A tile needs per-element masking if it reaches past the sequence or outside
      // the window of some row of the tile (causal: the diagonal tile).
      const bool masked = (k0 + 128 > seqlen) || (wl >= 0 && k0 < r0 + 127 - wl) ||
                          (wr >= 0 && k0 + 127 > r0 + wr);
      const int clo = klo - k0 - c0, chi = khi - k0 - c0;  // visible local columns
      uint32_t pk[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const int c = 2 * c2;
        const uint32_t* src = c < 32 ? s0 : s1;
        float e0 = ex2_approx(__uint_as_float(src[c & 31]) * sl2 - lse2_r);
        float e1 = ex2_approx(__uint_as_float(src[(c + 1) & 31]) * sl2 - lse2_r);
        if (masked) {
          e0 = (c < clo || c > chi) ? 0.f : e0;
          e1 = (c + 1 < clo || c + 1 > chi) ? 0.f : e1;
        }
        pk[c2] = pack_bf16x2(e0, e1);
      }
      ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDPFull + bf), ph, abort_flag, kSiteBwdQSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp0[32], dp1[32];
      tmem_ld32(tSP + c0, dp0);
      tmem_ld32(tSP + c0 + 32, dp1);
      tmem_wait_ld();
      reg_fence32(dp0);
      reg_fence32(dp1);
      uint32_t ds[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const uint32_t pp = pk[c2];
        const float p0 = __uint_as_float(pp << 16), p1 = __uint_as_float(pp & 0xFFFF0000u);
        const int c = 2 * c2;
        const uint32_t* dp = c < 32 ? dp0 : dp1;
        ds[c2] = pack_bf16x2(p0 * (__uint_as_float(dp[c & 31]) - d_r),
                             p1 * (__uint_as_float(dp[(c + 1) & 31]) - d_r));
      }
      // dS of keys [c0, c0 + 64) goes to columns [c0, c0 + 32), over dP columns this
      // warpgroup has read and the other never reads.
      tc_fence_after();
      tmem_st32(tSP + c0, ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(L::kDSFull + bf));
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDQDone), 0, abort_flag, kSiteBwdQSoftmax));
    if (ok) {
      // Epilogue: each warpgroup writes half of the row's d columns, x scale.
      tc_fence_after();
      constexpr int DH = D / 2;
      const uint32_t tsrc = tDQ + lane_off + half * DH;
      uint16_t* dst = p.dq + (tok0 + q) * p.rs_dq + h * D + half * DH;
      const bool row_ok = q < seqlen;
      const bool wide = rows32(p.dq, p.rs_dq);
#pragma unroll
      for (int cc = 0; cc < DH / 64; ++cc) {
        uint32_t a[32], c[32];
        tmem_ld32(tsrc + cc * 64, a);
        tmem_ld32(tsrc + cc * 64 + 32, c);
        tmem_wait_ld();
        reg_fence32(a);
        reg_fence32(c);
        store_row64(dst + cc * 64, a, c, p.scale, row_ok, wide);
      }
      if constexpr (DH == 32) {
        uint32_t a[32];
        tmem_ld32(tsrc, a);
        tmem_wait_ld();
        reg_fence32(a);
        if (row_ok && wide) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w8[e] = pack_bf16x2(__uint_as_float(a[16 * v + 2 * e]) * p.scale,
                                  __uint_as_float(a[16 * v + 2 * e + 1]) * p.scale);
            st_global_v8(dst + 16 * v, w8);
          }
        } else if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * v]) * p.scale, __uint_as_float(a[8 * v + 1]) * p.scale),
                               pack_bf16x2(__uint_as_float(a[8 * v + 2]) * p.scale, __uint_as_float(a[8 * v + 3]) * p.scale),
                               pack_bf16x2(__uint_as_float(a[8 * v + 4]) * p.scale, __uint_as_float(a[8 * v + 5]) * p.scale),
                               pack_bf16x2(__uint_as_float(a[8 * v + 6]) * p.scale, __uint_as_float(a[8 * v + 7]) * p.scale));
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
