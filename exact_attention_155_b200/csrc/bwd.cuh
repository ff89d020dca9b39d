// Attention backward for sm_100a with recomputation: the score matrix is rebuilt
// from Q, K and the forward's LSE tile by tile instead of being stored (the
// "重计算 / Recomputation" item of the ms-swift FA2/3 page and of section 三 of the
// Qwen flash_attn explainer). The gradient formulas are the analytic derivative of
// softmax(scale Q K^T) V:
//   P = exp(scale S - LSE), dV = P^T dO, dP = dO V^T, D_i = sum_c dO_ic O_ic,
//   dS = P * (dP - D), dK = scale dS^T Q, dQ = scale dS K.
//
// Kernels:
//  * bwd_pre_kernel: D per query row, the LSE converted to log2 units, zeroed fp32
//    dQ accumulator. Rows are padded to a multiple of 128 (LSE = +inf there, so the
//    recomputed P of a padded row is exactly 0).
//  * bwd_kernel: persistent, one CTA per SM. A work unit is one (batch, head, 128-key
//    tile); a CTA takes units one after another (the first by block index, the rest
//    from a per-call counter in the workspace), keeps K_j and V_j in shared memory for
//    the unit and walks the query tiles i (i >= j when causal). The next unit's K/V
//    loads, first S^T product and Q/dO loads run while the current unit's last
//    products, dK/dV epilogue and dQ reductions finish. Scores are
//    computed transposed (keys on TMEM lanes) so P^T and dS^T are already in the
//    A-operand orientation of dV += P^T dO and dK += dS^T Q:
//       S^T  = K Q_i^T        (TMEM cols [0,128), fp32; P^T bf16 over [0,32), [64,96))
//       dP^T = V dO_i^T       (TMEM cols [128,256), fp32)
//       dV  += P^T dO_i       (A from TMEM, TMEM cols [256,256+d))
//       dK  += dS^T Q_i       (A = dS^T in shared memory, TMEM [256+d,256+2d))
//       dQ_i = dS K           (A = the same shared buffer read MN-major,
//                              TMEM cols [128,128+d) once dP^T has been read)
//    Warps 0-7 (one key row per thread, two warpgroups splitting the query
//    columns) turn S^T into P^T and dP^T into dS^T; warps 8-11 drain dQ_i from TMEM
//    into the fp32 accumulator (shared-memory staging + bulk async reductions for
//    d = 128, vector atomics for d = 64); warp 12 takes the work units and issues
//    TMA; warp 13 issues tcgen05.mma.
//  * bwd_dq_convert_kernel: dq = bf16(accumulator).
// The fp32 reductions of dQ land in an order that is not fixed, so dQ may differ in
// its last bits between runs. bwd_det.cuh has the bitwise-repeatable alternative
// (separate dK/dV and dQ kernels, seven tile products per tile pair instead of five).
#pragma once

#include <math.h>

#include "ptx.cuh"

namespace fa {

struct BwdParams {
  int B, H, N, Np;      // N: sequence length (dense) or the largest one (variable length);
                        // Np = N rounded up to a multiple of 128
  int nqt;              // Np / 128: key tiles and query tiles per (batch, head)
  int head_group;       // heads scheduled together (divides B*H), for L2 reuse
  int num_units;        // fused kernel: nqt * B * H units of one (batch, head, key tile)
  unsigned int* ticket; // fused kernel: zeroed by bwd_pre_kernel; the k-th request for a
                        // unit gets unit gridDim.x + k
  int window_left;      // keys visible to query i: [i - window_left, i + window_right],
  int window_right;     // -1 = unbounded on that side (causal: window_right = 0)
  float scale;          // softmax scale
  float scale_log2;     // scale * log2(e)
  const int* cu_seqlens;  // NULL: dense rows (b, n); else [B + 1] token offsets
  int total;            // variable length: tokens in the packed tensors
  // Elements between consecutive rows (tokens) of each row-major [*, H, d] tensor.
  long long rs_o, rs_do, rs_dq, rs_dk, rs_dv;
  const uint16_t* out;  // forward output
  const uint16_t* dout;
  const float* lse;     // dense [B, H, N]; variable [H, total]; natural log
  float* dq_acc;        // [B, H, Np, d] fp32 (fused kernel only; null for bwd_det.cuh)
  float* lse2;          // [B, H, Np] log2 units (+inf on rows past the sequence)
  float* dvec;          // [B, H, Np] rowsum(dO * O)
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
};

enum : unsigned int {
  kSiteBwdProducer = 0x201,
  kSiteBwdMma = 0x202,
  kSiteBwdSoftmax = 0x203,
  kSiteBwdDrain = 0x204,
  kSiteBwdSeqlens = 0x205,
  kSiteBwdQProducer = 0x211,
  kSiteBwdQMma = 0x212,
  kSiteBwdQSoftmax = 0x213,
  kSiteBwdSmemAlign = 0x2FF
};

// First token and length of sequence b; false for an invalid cu_seqlens entry.
__device__ __forceinline__ bool bwd_seq(const BwdParams& p, int b, long long* tok0, int* len) {
  if (p.cu_seqlens == nullptr) {
    *tok0 = static_cast<long long>(b) * p.N;
    *len = p.N;
    return true;
  }
  const int s0 = __ldg(p.cu_seqlens + b), s1 = __ldg(p.cu_seqlens + b + 1);
  *tok0 = s0;
  *len = s1 - s0;
  return !(s0 < 0 || s1 < s0 || s1 - s0 > p.N || s1 > p.total);
}

struct BwdWorkspace {
  size_t dq_off, lse2_off, dvec_off, ticket_off, total;
};

inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

inline BwdWorkspace bwd_ws_layout(int B, int H, int N, int d) {
  const size_t Np = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t rows = static_cast<size_t>(B) * H * Np;
  BwdWorkspace w;
  w.dq_off = 0;
  w.lse2_off = round256(rows * d * sizeof(float));
  w.dvec_off = w.lse2_off + round256(rows * sizeof(float));
  w.ticket_off = w.dvec_off + round256(rows * sizeof(float));  // the fused kernel's unit counter
  w.total = w.ticket_off + 256;
  return w;
}

template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
  constexpr int TPR = D / 8;  // threads per row, 16 bytes each
  const long long gt = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long total = static_cast<long long>(p.B) * p.H * p.Np;
  const long long row = gt / TPR;
  const int sub = static_cast<int>(gt % TPR);
  const bool valid = row < total;
  const int i = valid ? static_cast<int>(row % p.Np) : 0;
  const long long bh = valid ? row / p.Np : 0;
  const int b = static_cast<int>(bh / p.H), h = static_cast<int>(bh % p.H);
  long long tok0 = 0;
  int len = 0;
  const bool seq_ok = valid && bwd_seq(p, b, &tok0, &len);
  if (valid && !seq_ok && i == 0 && sub == 0 && h == 0) report(kDevBadInput, kSiteBwdSeqlens, b);
  const bool real = seq_ok && i < len;
  if (gt == 0 && p.ticket != nullptr) *p.ticket = 0u;  // runs before the fused kernel on the stream
  float acc = 0.f;
  if (real) {
    const long long tok = tok0 + i;
    const uint4 o = __ldg(reinterpret_cast<const uint4*>(p.out + tok * p.rs_o + h * D + sub * 8));
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(p.dout + tok * p.rs_do + h * D + sub * 8));
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc = fmaf(__uint_as_float(ow[k] << 16), __uint_as_float(gw[k] << 16), acc);
      acc = fmaf(__uint_as_float(ow[k] & 0xFFFF0000u), __uint_as_float(gw[k] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (!valid) return;
  if (sub == 0) {
    float lse = INFINITY;
    if (real)
      lse = (p.cu_seqlens != nullptr ? p.lse[static_cast<size_t>(h) * p.total + tok0 + i]
                                     : p.lse[bh * p.N + i]) * 1.4426950408889634f;
    p.dvec[row] = real ? acc : 0.f;
    p.lse2[row] = lse;
  }
  if (p.dq_acc != nullptr) {  // the fused kernel's fp32 dQ accumulator
    float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D + sub * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const BwdParams p) {
  constexpr int TPR = D / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long total = static_cast<long long>(p.B) * p.N * p.H;
  const long long row = gt / TPR;  // (b, i, h) in output order
  if (row >= total) return;
  const int sub = static_cast<int>(gt % TPR);
  const int h = static_cast<int>(row % p.H);
  const long long bi = row / p.H;
  const int i = static_cast<int>(bi % p.N);
  const int b = static_cast<int>(bi / p.N);
  long long tok0 = 0;
  int len = 0;
  if (!bwd_seq(p, b, &tok0, &len) || i >= len) return;
  const float4* src = reinterpret_cast<const float4*>(
      p.dq_acc + ((static_cast<size_t>(b) * p.H + h) * p.Np + i) * D + sub * 8);
  const float4 a = src[0], c = src[1];
  uint4 o;
  o.x = pack_bf16x2(a.x, a.y);
  o.y = pack_bf16x2(a.z, a.w);
  o.z = pack_bf16x2(c.x, c.y);
  o.w = pack_bf16x2(c.z, c.w);
  *reinterpret_cast<uint4*>(p.dq + (tok0 + i) * p.rs_dq + h * D + sub * 8) = o;
}

// Unit indices the producer publishes ahead of the other roles, and the warps that
// read each one (the MMA warp, eight softmax warps, four dQ drain warps).
constexpr int kBwdUnitSlots = 4;
constexpr int kBwdUnitReaders = 13;

template <int D>
struct BwdLayout {
  static constexpr int kTile = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kQStages = 2;         // Q_i (+ lse2_i, D_i) double-buffered
  static constexpr int kK = 0;
  static constexpr int kV = kTile;
  static constexpr int kQ0 = 2 * kTile;                      // kQStages tiles
  static constexpr int kDO = kQ0 + kQStages * kTile;         // dO_i, single buffer
  static constexpr int kDS = kDO + kTile;                    // 128 x 128 bf16 dS^T
  static constexpr int kStage = kDS + 32768;                 // 2 x 16 KB dQ staging (d = 128)
  static constexpr int kStageBytes = (D == 128) ? 2 * 16384 : 0;
  static constexpr int kVec = kStage + kStageBytes;          // per Q stage: lse2[128], D[128]
  static constexpr int kBar = kVec + kQStages * 1024;
  static constexpr int kKVFull = 0;
  static constexpr int kQFull = 1;                   // [kQStages]
  static constexpr int kQEmpty = 1 + kQStages;       // [kQStages]
  static constexpr int kDOFull = 1 + 2 * kQStages;
  static constexpr int kDOEmpty = kDOFull + 1;
  static constexpr int kSFull = kDOFull + 2;
  static constexpr int kDPFull = kSFull + 1;
  static constexpr int kPFull = kSFull + 2;
  static constexpr int kDSFull = kSFull + 3;
  static constexpr int kDSFree = kSFull + 4;
  static constexpr int kDQFull = kSFull + 5;
  static constexpr int kDQFree = kSFull + 6;
  static constexpr int kMmaDone = kSFull + 7;
  static constexpr int kDrain = kSFull + 8;
  static constexpr int kKVEmpty = kDrain + 1;        // the unit's last products read K_j, V_j
  static constexpr int kUnitFull = kKVEmpty + 1;     // [kBwdUnitSlots]
  static constexpr int kUnitEmpty = kUnitFull + kBwdUnitSlots;  // [kBwdUnitSlots]
  static constexpr int kNumBars = kUnitEmpty + kBwdUnitSlots;
  // kMisc: TMEM base address, abort flag, then the unit ring (kBwdUnitSlots ints).
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 4 * kBwdUnitSlots;
  static constexpr int kThreads = 448;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kBytes <= 232448, "shared memory budget");
};


__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
               "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// One work unit of the fused kernel: (batch, head) and one 128-key tile.
struct BwdUnit {
  int b, h, bh, jt;
  long long tok0;  // first token of the sequence
  int seqlen;
  int tb, trow;    // batch and row coordinates of the sequence's row 0 in the tensor maps
  int it0, niter;  // query tiles [it0, it0 + niter) see a key of the tile; 0 = no work
};

// Work order: heads in groups of head_group (L2 reuse of Q/dO and the dQ accumulator);
// within a group, key tile 0 (the most query tiles when causal) first. A key tile past
// the end of a shorter sequence, or in a sequence whose cu_seqlens entries are invalid
// (reported by bwd_pre_kernel), has niter = 0.
template <bool CAUSAL, bool GENERAL>
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams& p, int u) {
  BwdUnit w;
  const int G = p.head_group;
  const int per_group = G * p.nqt;
  const int grp = u / per_group;
  const int rem = u % per_group;
  w.jt = rem / G;
  w.bh = grp * G + rem % G;
  w.b = w.bh / p.H;
  w.h = w.bh % p.H;
  w.tok0 = static_cast<long long>(w.b) * p.N;
  w.seqlen = p.N;
  w.it0 = 0;
  w.niter = 0;
  const bool var = GENERAL && p.cu_seqlens != nullptr;
  if (GENERAL && !bwd_seq(p, w.b, &w.tok0, &w.seqlen)) {
    w.tok0 = 0;
    w.seqlen = 0;
  }
  w.tb = var ? 0 : w.b;
  w.trow = var ? static_cast<int>(w.tok0) : 0;
  if (w.jt * 128 >= w.seqlen) return w;
  // Keys [k0, k1] are visible to queries [k0 - wr, k1 + wl] within [0, L).
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);
  const int k0 = w.jt * 128, k1 = min(w.seqlen, k0 + 128) - 1;
  const int qlo = wr < 0 ? 0 : max(0, k0 - wr);
  const int qhi = wl < 0 ? w.seqlen - 1 : min(w.seqlen - 1, k1 + wl);
  w.it0 = qlo / 128;
  w.niter = qhi / 128 - w.it0 + 1;  // >= 1: every key sees at least itself
  return w;
}

// GENERAL = false compiles the plain dense case (no sequence offsets, no window,
// CAUSAL fixed); GENERAL = true reads the window and cu_seqlens at run time.
template <int D, bool CAUSAL, bool GENERAL>
__global__ void __launch_bounds__(448, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {
    // The swizzled tiles need a 1024-byte aligned base; there is no slack to realign.
    if (threadIdx.x == 0) report(kDevTimeout, kSiteBwdSmemAlign, base);
    return;
  }
  const uint32_t sK = base + L::kK, sV = base + L::kV, sDS = base + L::kDS;
  const uint32_t bar0 = base + L::kBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

  const int warp = warp_id(), lane = lane_id();
  const int wl = GENERAL ? p.window_left : -1;
  const int wr = GENERAL ? p.window_right : (CAUSAL ? 0 : -1);

  if (threadIdx.x == 0) {
    mbar_init(BAR(L::kKVFull), 1);
    mbar_init(BAR(L::kKVEmpty), 1);
    for (int s = 0; s < kBwdUnitSlots; ++s) {
      mbar_init(BAR(L::kUnitFull + s), 1);
      mbar_init(BAR(L::kUnitEmpty + s), kBwdUnitReaders);  // one arrival per reading warp
    }
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(BAR(L::kQFull + s), 1);
      mbar_init(BAR(L::kQEmpty + s), 1);
    }
    mbar_init(BAR(L::kDOFull), 1);
    mbar_init(BAR(L::kDOEmpty), 1);
    mbar_init(BAR(L::kSFull), 1);
    mbar_init(BAR(L::kDPFull), 1);
    mbar_init(BAR(L::kPFull), 256);
    mbar_init(BAR(L::kDSFull), 256);
    mbar_init(BAR(L::kDSFree), 1);
    mbar_init(BAR(L::kDQFull), 1);
    mbar_init(BAR(L::kDQFree), 128);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tDQ = tmem + 128, tDV = tmem + 256,
                 tDK = tmem + 256 + D;

  // The reading warps take the k-th unit of this CTA from slot k % kBwdUnitSlots; -1
  // ends the loop. Returns false on an abort.
  auto next_unit = [&](int k, int* u, unsigned int site) -> bool {
    const int slot = k % kBwdUnitSlots;
    const bool got = __all_sync(0xffffffffu, wait_bar(BAR(L::kUnitFull + slot), (k / kBwdUnitSlots) & 1,
                                                      abort_flag, site));
    if (!got) return false;
    *u = unit_ring[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(L::kUnitEmpty + slot));
    return true;
  };

  if (warp == 12) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      // Loads issued over all units: K/V pairs, Q tiles (+ lse2, D) and dO tiles. The
      // Q ring stage and every phase parity follow these running counts.
      int nkv = 0, nq = 0, ndo = 0;
      bool ok = true;
      int u = static_cast<int>(blockIdx.x);
      for (int k = 0; ok; ++k) {
        // Units with nothing to do are skipped here; the other roles never see them.
        BwdUnit w{};
        for (; u < p.num_units; u = static_cast<int>(gridDim.x + atomicAdd(p.ticket, 1u))) {
          w = bwd_unit<CAUSAL, GENERAL>(p, u);
          if (w.niter > 0) break;
        }
        // Publish unit k (or the end) once its slot has been read by every reading warp.
        const int slot = k % kBwdUnitSlots;
        if (!wait_bar(BAR(L::kUnitEmpty + slot), ((k / kBwdUnitSlots) & 1) ^ 1u, abort_flag, kSiteBwdProducer))
          break;
        const bool last = u >= p.num_units;
        unit_ring[slot] = last ? -1 : u;
        mbar_arrive(BAR(L::kUnitFull + slot));
        if (last) break;
        // K_j and V_j replace the previous unit's once its last products have read them.
        if (nkv > 0 && !wait_bar(BAR(L::kKVEmpty), (nkv - 1) & 1, abort_flag, kSiteBwdProducer)) break;
        mbar_arrive_expect_tx(BAR(L::kKVFull), 2 * L::kTile);
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_4d(sK + bx * 16384, &tmK, BAR(L::kKVFull), bx * 64, w.h, w.trow + w.jt * 128, w.tb);
          tma_load_4d(sV + bx * 16384, &tmV, BAR(L::kKVFull), bx * 64, w.h, w.trow + w.jt * 128, w.tb);
        }
        ++nkv;
        const float* lse2_h = p.lse2 + static_cast<size_t>(w.bh) * p.Np;
        const float* dvec_h = p.dvec + static_cast<size_t>(w.bh) * p.Np;
        for (int n = 0; n < w.niter; ++n) {
          const int it = w.it0 + n;
          const int s = nq % L::kQStages;
          if (!wait_bar(BAR(L::kQEmpty + s), ((nq / L::kQStages) & 1) ^ 1u, abort_flag, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          const uint32_t sQ = base + L::kQ0 + s * L::kTile;
          mbar_arrive_expect_tx(BAR(L::kQFull + s), L::kTile + 1024);
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(sQ + bx * 16384, &tmQ, BAR(L::kQFull + s), bx * 64, w.h, w.trow + it * 128, w.tb);
          const uint32_t sv = base + L::kVec + s * 1024;
          bulk_load(sv, lse2_h + it * 128, 512, BAR(L::kQFull + s));
          bulk_load(sv + 512, dvec_h + it * 128, 512, BAR(L::kQFull + s));
          ++nq;
          if (!wait_bar(BAR(L::kDOEmpty), (ndo & 1) ^ 1u, abort_flag, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(BAR(L::kDOFull), L::kTile);
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(base + L::kDO + bx * 16384, &tmdO, BAR(L::kDOFull), bx * 64, w.h, w.trow + it * 128,
                        w.tb);
          ++ndo;
        }
        u = static_cast<int>(gridDim.x + atomicAdd(p.ticket, 1u));
      }
      // Never leave the CTA with copies in flight.
      for (int k = max(0, nq - L::kQStages); k < nq; ++k)
        drain_wait(BAR(L::kQFull + k % L::kQStages), (k / L::kQStages) & 1);
      if (ndo > 0) drain_wait(BAR(L::kDOFull), (ndo - 1) & 1);
      if (nkv > 0) drain_wait(BAR(L::kKVFull), (nkv - 1) & 1);
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs the issue loop (the operands stay warp-uniform); elect.sync
    // picks the lane that issues each tcgen05 instruction, and every wait result is
    // made uniform across the warp before it steers control.
    {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t kIdKV = idesc_bf16_f32(128, D, 0, 1);   // dV (A in TMEM), dK (A K-major)
      // d = 128: dQ^T = K^T dS^T (head dim on TMEM lanes, coalesced reductions);
      // d = 64:  dQ = dS K (queries on TMEM lanes).
      constexpr uint32_t kIdQ = (D == 128) ? idesc_bf16_f32(128, 128, 1, 1) : idesc_bf16_f32(128, D, 1, 1);
      auto q_addr = [&](int g) { return base + L::kQ0 + static_cast<uint32_t>(g % L::kQStages) * L::kTile; };
      const uint32_t sdO = base + L::kDO;
      auto issue_st = [&](int g) {  // S^T = K Q_g^T
        const uint32_t sQ = q_addr(g);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
          umma_ss_w(tS, sdesc_sw128(sK + koff, 16, 1024), sdesc_sw128(sQ + koff, 16, 1024), kIdS,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit_w(BAR(L::kSFull));
      };
      // g counts query tiles over all units of this CTA: it selects the Q ring stage and
      // gives the phase of every per-tile barrier; nu counts units (K/V loads, MMA-done).
      int g = 0, nu = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int u = -1;
        if (!(ok = next_unit(k, &u, kSiteBwdMma)) || u < 0) break;
        const BwdUnit w = bwd_unit<CAUSAL, GENERAL>(p, u);
        // S^T of the unit's first query tile. Its TMEM columns held P^T of the previous
        // tile, which the dV product issued before it (executed in order) has read.
        if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kKVFull), nu & 1, abort_flag, kSiteBwdMma)))) break;
        if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull + g % L::kQStages), (g / L::kQStages) & 1,
                                                    abort_flag, kSiteBwdMma))))
          break;
        tc_fence_after();
        issue_st(g);
        // Issue order per query tile: dP^T, dV, S^T(next), dQ, dK: dP^T overlaps the
        // exponentials of the tile, the dS pass overlaps dV and the next S^T, the next
        // tile's exponentials overlap dQ and dK, and the dQ drain overlaps dK.
        for (int n = 0; n < w.niter; ++n, ++g) {
          const int s = g % L::kQStages;
          const uint32_t sQ = q_addr(g);
          // dP^T = V dO^T, into the columns the previous dQ used once they were read out
          // (that dQ may belong to the previous unit). It does not need P, so the dS pass
          // can start as soon as P is done.
          if (g > 0) {
            if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDQFree), (g - 1) & 1, abort_flag, kSiteBwdMma)))) break;
          }
          if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDOFull), g & 1, abort_flag, kSiteBwdMma)))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
            umma_ss_w(tDP, sdesc_sw128(sV + koff, 16, 1024), sdesc_sw128(sdO + koff, 16, 1024), kIdS,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit_w(BAR(L::kDPFull));
          // dV += P^T dO. The unit's first dV overwrites the accumulator: the softmax
          // warps arrive on P-full only after their epilogue of the previous unit has
          // read dV and dK out of TMEM.
          if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kPFull), g & 1, abort_flag, kSiteBwdMma)))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts_w(tDV, tS + 64 * (kk >> 2) + 8 * (kk & 3), sdesc_sw128(sdO + kk * 2048, 16384, 1024), kIdKV,
                    (n > 0 || kk > 0) ? 1u : 0u);
          umma_commit_w(BAR(L::kDOEmpty));
          // S^T of the next tile: the S columns are free once dV (issued above, executed
          // in order) has read P; the dS pass keeps P in registers.
          if (n + 1 < w.niter) {
            if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull + (g + 1) % L::kQStages),
                                                        ((g + 1) / L::kQStages) & 1, abort_flag, kSiteBwdMma))))
              break;
            tc_fence_after();
            issue_st(g + 1);
          }
          if (!(ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDSFull), g & 1, abort_flag, kSiteBwdMma)))) break;
          tc_fence_after();
          // dQ first, so the drain reads it out of TMEM while dK runs.
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            if constexpr (D == 128)
              umma_ss_w(tDQ, sdesc_sw128(sK + kk * 2048, 16384, 1024),
                      sdesc_sw128(sDS + kk * 2048, 16384, 1024), kIdQ, kk > 0 ? 1u : 0u);
            else
              umma_ss_w(tDQ, sdesc_sw128(sDS + kk * 2048, 16384, 1024),
                      sdesc_sw128(sK + kk * 2048, 16384, 1024), kIdQ, kk > 0 ? 1u : 0u);
          }
          umma_commit_w(BAR(L::kDQFull));
          // The unit's last dQ (and dP^T before it) were the last reads of K_j and V_j.
          if (n + 1 == w.niter) umma_commit_w(BAR(L::kKVEmpty));
          // dK += dS^T Q
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss_w(tDK, sdesc_sw128(sDS + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024),
                    sdesc_sw128(sQ + kk * 2048, 16384, 1024), kIdKV, (n > 0 || kk > 0) ? 1u : 0u);
          umma_commit_w(BAR(L::kDSFree));
          umma_commit_w(BAR(L::kQEmpty + s));
        }
        if (!ok) break;
        umma_commit_w(BAR(L::kMmaDone));  // dV and dK of the unit are final
        ++nu;
      }
      umma_commit_w(BAR(L::kDrain));
      drain_wait(BAR(L::kDrain), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------ P^T and dS^T: one key row per thread; two
    // warpgroups split the 128 query columns of every tile (64 columns each).
    const int wq = warp & 3;
    const int half = warp >> 2;
    const int c0 = half * 64;  // first query column of this warpgroup
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    // g: query tiles over all units (stage and phases, as in the MMA warp); nu: units.
    int g = 0, nu = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u = -1;
      if (!(ok = next_unit(k, &u, kSiteBwdSoftmax)) || u < 0) break;
      const BwdUnit w = bwd_unit<CAUSAL, GENERAL>(p, u);
      const int key = w.jt * 128 + r;
      const bool key_ok = key < w.seqlen;
      const long long tok0 = w.tok0;
      for (int n = 0; n < w.niter; ++n, ++g) {
        const int it = w.it0 + n;
        const int s = g % L::kQStages;
        const float* vec = reinterpret_cast<const float*>(smem + L::kVec + s * 1024) + c0;
        ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kSFull), g & 1, abort_flag, kSiteBwdSoftmax));
        if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kQFull + s), (g / L::kQStages) & 1,
                                                     abort_flag, kSiteBwdSoftmax));
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
        // sequence have lse2 = +inf, so their P is already 0. Only tiles where some key of
        // the warp misses some of the 64 columns (the causal diagonal, window edges, the
        // sequence end) take the per-element test.
        const int q0 = it * 128 + c0;
        const int qlo_c = !key_ok ? (1 << 30) : (wr < 0 ? -(1 << 30) : key - wr - q0);
        const int qhi_c = wl < 0 ? (1 << 30) : key + wl - q0;
        const bool edge = __any_sync(0xffffffffu, qlo_c > 0 || qhi_c < 63);
        const float4* vec4 = reinterpret_cast<const float4*>(vec);  // 16-byte aligned (c0 = 0, 64)
        uint32_t pk[32];
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 lv = vec4[c4];
          const uint32_t* src = c4 < 8 ? s0 : s1;
          const int o = (4 * c4) & 31;
          float e0 = ex2_approx(__uint_as_float(src[o]) * sl2 - lv.x);
          float e1 = ex2_approx(__uint_as_float(src[o + 1]) * sl2 - lv.y);
          float e2 = ex2_approx(__uint_as_float(src[o + 2]) * sl2 - lv.z);
          float e3 = ex2_approx(__uint_as_float(src[o + 3]) * sl2 - lv.w);
          if (edge) {
            const int c = 4 * c4;
            e0 = (c < qlo_c || c > qhi_c) ? 0.f : e0;
            e1 = (c + 1 < qlo_c || c + 1 > qhi_c) ? 0.f : e1;
            e2 = (c + 2 < qlo_c || c + 2 > qhi_c) ? 0.f : e2;
            e3 = (c + 3 < qlo_c || c + 3 > qhi_c) ? 0.f : e3;
          }
          pk[2 * c4] = pack_bf16x2(e0, e1);
          pk[2 * c4 + 1] = pack_bf16x2(e2, e3);
        }
        // P^T of queries [c0, c0 + 64) goes to columns [c0, c0 + 32), the first half of the
        // S^T columns this warpgroup has just read and no other warpgroup reads, so it needs
        // no wait. (A warpgroup is never more than one tile ahead: S^T(n + 1) waits for
        // both warpgroups' P^T(n).)
        tc_fence_after();
        tmem_st32(tS + lane_off + c0, pk);  // P^T bf16: two queries per 32-bit column
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(L::kPFull));

        ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDPFull), g & 1, abort_flag, kSiteBwdSoftmax));
        if (ok && g > 0)
          ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kDSFree), (g - 1) & 1, abort_flag, kSiteBwdSoftmax));
        if (!ok) break;
        tc_fence_after();
        const float4* dvec4 = reinterpret_cast<const float4*>(vec + 128);
        uint32_t dp0[32], dp1[32];
        tmem_ld32(tDP + lane_off + c0, dp0);
        tmem_ld32(tDP + lane_off + c0 + 32, dp1);
        tmem_wait_ld();
        reg_fence32(dp0);
        reg_fence32(dp1);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t* dp = q == 0 ? dp0 : dp1;
          uint32_t w[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 dv = dvec4[q * 8 + c4];
            const uint32_t pa = pk[q * 16 + 2 * c4], pb = pk[q * 16 + 2 * c4 + 1];
            float d0, d1, d2, d3;
            add2(d0, d1, __uint_as_float(dp[4 * c4]), __uint_as_float(dp[4 * c4 + 1]), -dv.x, -dv.y);
            add2(d2, d3, __uint_as_float(dp[4 * c4 + 2]), __uint_as_float(dp[4 * c4 + 3]), -dv.z, -dv.w);
            mul2(d0, d1, d0, d1, __uint_as_float(pa << 16), __uint_as_float(pa & 0xFFFF0000u));
            mul2(d2, d3, d2, d3, __uint_as_float(pb << 16), __uint_as_float(pb & 0xFFFF0000u));
            w[2 * c4] = pack_bf16x2(d0, d1);
            w[2 * c4 + 1] = pack_bf16x2(d2, d3);
          }
          // Row r of the dS^T tile, queries c0 + q*32 .. +31 (box `half`), 128-byte swizzle.
          const uint32_t row_base = sDS + half * 16384 + r * 128;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int chunk = q * 4 + ch;
            st_shared_v4(row_base + ((chunk ^ (r & 7)) << 4), w[4 * ch], w[4 * ch + 1], w[4 * ch + 2],
                         w[4 * ch + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(L::kDSFull));
      }
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(L::kMmaDone), nu & 1, abort_flag, kSiteBwdSoftmax));
      if (!ok) break;
      ++nu;
      {
        // Epilogue: warpgroup 0 writes dV rows, warpgroup 1 writes dK rows (x scale). Each
        // thread writes its own key row, so a warp's store touches 32 rows: 32-byte
        // stores (when the rows allow them) halve the number of those scattered pieces,
        // which, not the arithmetic, is what the epilogue's time goes to.
        tc_fence_after();
        const uint32_t tsrc = (half == 0 ? tDV : tDK) + lane_off;
        const float mul = half == 0 ? 1.f : p.scale;
        uint16_t* dst = (half == 0 ? p.dv + (tok0 + key) * p.rs_dv : p.dk + (tok0 + key) * p.rs_dk) + w.h * D;
        const bool wide = (((reinterpret_cast<uintptr_t>(half == 0 ? p.dv : p.dk)) |
                            static_cast<uintptr_t>((half == 0 ? p.rs_dv : p.rs_dk) * 2)) & 31u) == 0;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tsrc + cc * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
          if (key_ok) {
            if (wide) {
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                uint32_t w8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  w8[e] = pack_bf16x2(__uint_as_float(o[16 * v + 2 * e]) * mul,
                                      __uint_as_float(o[16 * v + 2 * e + 1]) * mul);
                st_global_v8(dst + cc * 32 + 16 * v, w8);
              }
            } else {
              uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                d4[v] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * v]) * mul, __uint_as_float(o[8 * v + 1]) * mul),
                                   pack_bf16x2(__uint_as_float(o[8 * v + 2]) * mul, __uint_as_float(o[8 * v + 3]) * mul),
                                   pack_bf16x2(__uint_as_float(o[8 * v + 4]) * mul, __uint_as_float(o[8 * v + 5]) * mul),
                                   pack_bf16x2(__uint_as_float(o[8 * v + 6]) * mul, __uint_as_float(o[8 * v + 7]) * mul));
            }
          }
        }
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------- dQ drain
    // d = 128: TMEM holds dQ^T (lane = head-dim index j, column = query), so one warp
    // instruction reduces 32 consecutive floats of one dQ row (128 contiguous bytes).
    // d = 64: TMEM holds dQ (lane = query), one thread reduces its own row.
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sc = p.scale;
    int g = 0;  // query tiles over all units (phase of the dQ barriers)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u = -1;
      // All four drain warps take the same decision: they share named barriers below.
      ok = named_bar_and(1, 128, next_unit(k, &u, kSiteBwdDrain));
      if (!ok || u < 0) break;
      const BwdUnit w = bwd_unit<CAUSAL, GENERAL>(p, u);
      for (int n = 0; n < w.niter; ++n, ++g) {
        const int it = w.it0 + n;
        ok = wait_bar(BAR(L::kDQFull), g & 1, abort_flag, kSiteBwdDrain);
        // All four drain warps leave together.
        ok = named_bar_and(1, 128, ok);
        if (!ok) break;
        tc_fence_after();
        if constexpr (D == 128) {
          // Read all of dQ^T (128 queries for this thread's head-dim index r), free the
          // TMEM columns, then push 32-query chunks through shared memory with one
          // asynchronous 16 KB bulk reduction each (rows of the accumulator are
          // contiguous: [bh][query][d]).
          uint32_t o0[32], o1[32], o2[32], o3[32];
          tmem_ld32(tDQ + lane_off + 0, o0);
          tmem_ld32(tDQ + lane_off + 32, o1);
          tmem_ld32(tDQ + lane_off + 64, o2);
          tmem_ld32(tDQ + lane_off + 96, o3);
          tmem_wait_ld();
          reg_fence32(o0);
          reg_fence32(o1);
          reg_fence32(o2);
          reg_fence32(o3);
          tc_fence_before();
          mbar_arrive(BAR(L::kDQFree));
          float* gtile = p.dq_acc + (static_cast<size_t>(w.bh) * p.Np + static_cast<size_t>(it) * 128) * D;
          const bool leader = (warp == 8 && lane == 0);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t buf = base + L::kStage + (cc & 1) * 16384;
            if (leader) bulk_wait_read1();  // the reduction that used this buffer has read it
            named_bar_sync(1, 128);
            const uint32_t* src = cc == 0 ? o0 : (cc == 1 ? o1 : (cc == 2 ? o2 : o3));
#pragma unroll
            for (int i = 0; i < 32; ++i) st_shared_f32(buf + (i * 128 + r) * 4, __uint_as_float(src[i]) * sc);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
              bulk_reduce_add_f32(gtile + cc * 32 * D, buf, 16384);
              bulk_commit();
            }
          }
          continue;
        } else {
          const int qrow = it * 128 + r;
          float* dst = p.dq_acc + (static_cast<size_t>(w.bh) * p.Np + qrow) * D;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tDQ + lane_off + cc * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
            if (qrow < w.seqlen) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                red_add_v4(dst + cc * 32 + 4 * v, __uint_as_float(o[4 * v]) * sc,
                           __uint_as_float(o[4 * v + 1]) * sc, __uint_as_float(o[4 * v + 2]) * sc,
                           __uint_as_float(o[4 * v + 3]) * sc);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(BAR(L::kDQFree));
      }
    }
    if constexpr (D == 128) {
      if (warp == 8 && lane == 0) bulk_wait_all();  // reductions complete before exit
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
