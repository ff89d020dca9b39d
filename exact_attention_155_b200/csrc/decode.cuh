// KV-cache decode for sm_100a: one new query row per (batch, head) attends to the
// valid rows of a [B, Ncap, H, d] bf16 cache, optionally after appending this
// step's K/V row at index cache_seqlens[b] (flash_attn_with_kvcache in section
// 推理优化与KV缓存 of "FlashAttention与MindSpore 2.0全场景融合方案").
//
// The work is a matrix-vector product per head, bound by reading K and V once from
// HBM, so it runs on CUDA cores (no tensor-core reshaping). decode_kernel: grid
// (splits, H, B) where the `splits` CTAs of one (batch, head) form a thread-block
// cluster. Each CTA takes one contiguous chunk of keys; d/8 lanes share a cache row
// (16-byte coalesced loads), K and V rows of several steps are loaded together,
// and each lane group keeps a running (m, l, o) online-softmax state, so a step has
// no block-wide synchronisation. Warp states are combined with shuffles, CTA states
// in shared memory, and the cluster's CTA states in the leader CTA's shared memory
// (the stable combination of per-block (m, l) of section 2.2.2 of
// "FlashAttention优化Transformer显存与计算效率"). The CTA whose chunk holds the
// appended row writes that row into the cache and every CTA reads it from k_new /
// v_new, so no CTA reads a row another one writes.
#pragma once

#include <math.h>

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace fa {

namespace cg = cooperative_groups;

constexpr int kDecodeMaxSplits = 8;  // CTAs per (batch, head): one portable cluster

// Row steps per thread whose K and V loads are issued before any is consumed.
#ifndef FA_DECODE_STEPS_IN_FLIGHT
#define FA_DECODE_STEPS_IN_FLIGHT 4
#endif
// Target CTAs per SM when choosing the number of splits (one wave at 7 per SM).
#ifndef FA_DECODE_CTAS_PER_SM
#define FA_DECODE_CTAS_PER_SM 6
#endif

struct DecodeParams {
  const uint16_t* q;      // [B, 1, H, d]
  uint16_t* k_cache;      // [B, Ncap, H, d]
  uint16_t* v_cache;      // [B, Ncap, H, d]
  const int* seqlens;     // [B] valid rows before this step's append
  const uint16_t* k_new;  // [B, 1, H, d] or null
  const uint16_t* v_new;  // [B, 1, H, d] or null
  uint16_t* out;          // [B, 1, H, d]
  float* lse;             // [B, H] or null
  int B, H, Ncap, nsplit, chunk;
  float scale_log2;
  // Paged caches (decode_kernel<D, true>): k_cache / v_cache are [num_pages, page_size,
  // H, d]; row r of batch b is row r % page_size of page block_table[b][r / page_size].
  // Ncap = max_blocks * page_size is the logical capacity.
  const int* block_table;  // [B, max_blocks]
  int max_blocks, num_pages, page_shift;  // page_size = 1 << page_shift
};

enum : unsigned int { kSiteDecodeSeqlen = 0x301, kSiteDecodePage = 0x302 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Running (m, l, o) state of the online softmax: m in log2 units, l = sum 2^(s - m),
// o = sum 2^(s - m) v (unnormalised). Combining two states rescales both to the
// larger max (the stable block combination of section 2.2.2).
__device__ __forceinline__ void online_merge(float& m, float& l, float (&o)[8], float m2, float l2,
                                             const float (&o2)[8]) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // both empty
  const float c1 = (m == -INFINITY) ? 0.f : ex2_approx(m - mn);
  const float c2 = (m2 == -INFINITY) ? 0.f : ex2_approx(m2 - mn);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = o[i] * c1 + o2[i] * c2;
  m = mn;
}

// One CTA per (split, head, batch); the `splits` CTAs of a (batch, head) form one
// thread-block cluster and combine their partial states in the leader CTA's shared
// memory (distributed shared memory), so the whole step is a single launch with no
// global workspace.
template <int D, bool PAGED>
__global__ void __launch_bounds__(128) decode_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;     // lanes per cache row (16 bytes each)
  constexpr int RPW = 32 / LPR;  // rows per warp per step
  constexpr int U = FA_DECODE_STEPS_IN_FLIGHT;  // steps whose loads are issued together
  constexpr int RSTEP = 4 * RPW; // rows per CTA per step
  __shared__ float s_warp[4][D + 2];   // per-warp partial: o[D], m, l
  __shared__ float s_part[8][D + 2];   // leader only: per-CTA partials of the cluster

  cg::cluster_group cluster = cg::this_cluster();
  const int split = static_cast<int>(cluster.block_rank());
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane / LPR, sub = lane % LPR;
  const bool append = p.k_new != nullptr;

  // A length outside [0, Ncap] (or a full cache when appending) is reported through
  // the device status word; that batch entry then attends nothing and appends nothing.
  int L = p.seqlens[b];
  const bool bad = L < 0 || L > p.Ncap || (append && L >= p.Ncap);
  if (bad) {
    if (tid == 0 && split == 0 && h == 0) report(kDevBadInput, kSiteDecodeSeqlen, b);
    L = 0;
  }
  const bool do_append = append && !bad;
  const int Lt = L + (do_append ? 1 : 0);
  const int k0 = split * p.chunk;
  const int k1 = min(k0 + p.chunk, Lt);
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  const size_t row_stride = static_cast<size_t>(p.H) * D;  // elements between cache rows
  const size_t cache0 = PAGED ? static_cast<size_t>(h) * D
                              : (static_cast<size_t>(b) * p.Ncap * p.H + h) * D;
  const uint16_t* kc = p.k_cache + cache0 + sub * 8;
  const uint16_t* vc = p.v_cache + cache0 + sub * 8;
  // Element offset of cache row r from this (b, h)'s row 0 (contiguous) or from the
  // cache base (paged), or -1 for a page id outside [0, num_pages), which is reported
  // and never dereferenced.
  auto table_at = [&](int r) -> int {
    return __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + (r >> p.page_shift));
  };
  auto paged_off = [&](int pg, int r) -> long long {
    if (pg < 0 || pg >= p.num_pages) {
      report(kDevBadInput, kSiteDecodePage, b);
      return -1;
    }
    return ((static_cast<long long>(pg) << p.page_shift) + (r & ((1 << p.page_shift) - 1))) *
           static_cast<long long>(row_stride);
  };
  auto row_off = [&](int r) -> long long {
    if (!PAGED) return static_cast<long long>(r) * static_cast<long long>(row_stride);
    return paged_off(table_at(r), r);
  };
  const uint16_t* kn = append ? p.k_new + bh * D + sub * 8 : nullptr;
  const uint16_t* vn = append ? p.v_new + bh * D + sub * 8 : nullptr;

  // The CTA whose chunk holds the appended row persists it in the cache; every CTA
  // reads that row from k_new / v_new, never from the cache.
  if (do_append && L >= k0 && L < k1 && tid < LPR) {
    const long long ro = row_off(L);
    if (ro >= 0) {
      const size_t off = cache0 + static_cast<size_t>(ro) + tid * 8;
      *reinterpret_cast<uint4*>(p.k_cache + off) =
          *reinterpret_cast<const uint4*>(p.k_new + bh * D + tid * 8);
      *reinterpret_cast<uint4*>(p.v_cache + off) =
          *reinterpret_cast<const uint4*>(p.v_new + bh * D + tid * 8);
    }
  }

  float qf[8];
  {
    const uint4 qu = *reinterpret_cast<const uint4*>(p.q + bh * D + sub * 8);
    bf16x8_to_f32(qu, qf);
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] *= p.scale_log2;
  }

  float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;

  // Paged: the page ids of the next row step are read while this step's K/V loads are
  // in flight, so no K/V load waits on a block-table read.
  auto page_id = [&](int r) -> int { return r < k1 ? table_at(r) : 0; };
  int pg_next[U];
  if (PAGED) {
#pragma unroll
    for (int u = 0; u < U; ++u) pg_next[u] = page_id(k0 + warp * RPW + u * RSTEP + grp);
  }
  // Rows handled by this lane group: k0 + warp*RPW + grp + RSTEP*t, t = 0, 1, ...
  for (int base = k0 + warp * RPW; base < k1; base += U * RSTEP) {
    int pg[U];
    if (PAGED) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        pg[u] = pg_next[u];
        pg_next[u] = page_id(base + U * RSTEP + u * RSTEP + grp);
      }
    }
    uint4 kv[U], vv[U];
    bool live[U];  // row inside the chunk with a readable source
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = base + u * RSTEP + grp;
      kv[u] = make_uint4(0, 0, 0, 0);
      vv[u] = make_uint4(0, 0, 0, 0);
      live[u] = false;
      if (kb < k1) {
        const bool is_new = do_append && kb == L;
        const long long off = is_new ? 0 : PAGED ? paged_off(pg[u], kb) : row_off(kb);
        if (is_new || off >= 0) {
          live[u] = true;
          kv[u] = __ldg(reinterpret_cast<const uint4*>(is_new ? kn : kc + off));
          vv[u] = __ldg(reinterpret_cast<const uint4*>(is_new ? vn : vc + off));
        }
      }
    }
    float sc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float f[8];
      bf16x8_to_f32(kv[u], f);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(qf[i], f[i], acc);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      sc[u] = live[u] ? acc : -INFINITY;
    }
    float mx = sc[0];
#pragma unroll
    for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[u]);
    const float m_new = fmaxf(m, mx);
    if (m_new != -INFINITY) {
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float pu = ex2_approx(sc[u] - m_new);  // 0 for rows past the chunk
        float f[8];
        bf16x8_to_f32(vv[u], f);
        l += pu;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(pu, f[i], o[i]);
      }
      m = m_new;
    }
  }

  // Combine the RPW row groups of the warp (lanes with the same slice `sub`).
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
    float o2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o2[i] = __shfl_xor_sync(0xffffffffu, o[i], off);
    online_merge(m, l, o, m2, l2, o2);
  }
  if (grp == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s_warp[warp][sub * 8 + i] = o[i];
    if (sub == 0) {
      s_warp[warp][D] = m;
      s_warp[warp][D + 1] = l;
    }
  }
  __syncthreads();

  // CTA partial -> the leader CTA's shared memory.
  float* dst = cluster.map_shared_rank(&s_part[0][0], 0) + split * (D + 2);
  if (tid < D) {
    float mc = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mc = fmaxf(mc, s_warp[w][D]);
    float oc = 0.f, lc = 0.f;
    if (mc != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = s_warp[w][D];
        const float cw = (mw == -INFINITY) ? 0.f : ex2_approx(mw - mc);
        oc = fmaf(s_warp[w][tid], cw, oc);
        lc = fmaf(s_warp[w][D + 1], cw, lc);
      }
    }
    dst[tid] = oc;
    if (tid == 0) {
      dst[D] = mc;
      dst[D + 1] = lc;
    }
  }
  cluster.sync();

  if (split == 0 && tid < D) {
    const int S = static_cast<int>(cluster.num_blocks());
    float M = -INFINITY;
    for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, s_part[s2][D]);
    float O = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < S; ++s2) {
        const float ms = s_part[s2][D];
        const float c = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
        O = fmaf(s_part[s2][tid], c, O);
        Ls = fmaf(s_part[s2][D + 1], c, Ls);
      }
    }
    const float out = (Ls > 0.f) ? O / Ls : 0.f;
    const float nb = __shfl_down_sync(0xffffffffu, out, 1);
    if ((tid & 1) == 0)
      reinterpret_cast<uint32_t*>(p.out + bh * D)[tid >> 1] = pack_bf16x2(out, nb);
    if (tid == 0 && p.lse)
      p.lse[bh] = (Ls > 0.f) ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace fa
