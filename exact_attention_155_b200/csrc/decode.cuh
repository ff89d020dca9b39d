// KV-cache decode for sm_100a: one new query row per (batch, head) attends to the
// valid rows of a [B, Ncap, H, d] bf16 cache, optionally after appending this
// step's K/V row at index cache_seqlens[b] (flash_attn_with_kvcache in section
// 推理优化与KV缓存 of "FlashAttention与MindSpore 2.0全场景融合方案").
//
// The work is a matrix-vector product per head, bound by reading K and V once from
// HBM, so it runs on CUDA cores (no tensor-core reshaping):
//  * decode_split_kernel: grid (splits, H, B). Each CTA takes one contiguous chunk
//    of keys, reads each K and V row once with 16-byte coalesced loads (d/8 lanes
//    per row, several rows in flight per thread), keeps the chunk's scores in
//    shared memory, and writes a partial (o_s, lse_s) for its chunk. The CTA whose
//    chunk holds the appended row writes that row into the cache and uses k_new /
//    v_new directly, so no other CTA reads it.
//  * decode_merge_kernel: LSE = log sum_s exp(lse_s), O = sum_s exp(lse_s - LSE) o_s,
//    the stable combination of per-block (m, l) of the blockwise softmax (section
//    2.2.2 of "FlashAttention优化Transformer显存与计算效率").
// With a single split the split kernel writes the final bf16 output itself.
#pragma once

#include <math.h>

#include "ptx.cuh"

namespace fa {

constexpr int kDecodeMaxChunk = 2048;  // keys per split (scores live in shared memory)

struct DecodeParams {
  const uint16_t* q;      // [B, 1, H, d]
  uint16_t* k_cache;      // [B, Ncap, H, d]
  uint16_t* v_cache;      // [B, Ncap, H, d]
  const int* seqlens;     // [B] valid rows before this step's append
  const uint16_t* k_new;  // [B, 1, H, d] or null
  const uint16_t* v_new;  // [B, 1, H, d] or null
  uint16_t* out;          // [B, 1, H, d]
  float* lse;             // [B, H] or null
  float* part_o;          // [B, H, nsplit, d] (nsplit > 1)
  float* part_lse;        // [B, H, nsplit]    (nsplit > 1)
  int B, H, Ncap, nsplit, chunk;
  float scale_log2;
};

enum : unsigned int { kSiteDecodeSeqlen = 0x301 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(128) decode_split_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;     // lanes per cache row (16 bytes each)
  constexpr int RPW = 32 / LPR;  // rows per warp step
  constexpr int RPC = 4 * RPW;   // rows per CTA step
  constexpr int U = 4;           // row steps kept in flight per thread
  __shared__ float s_sc[kDecodeMaxChunk];
  __shared__ float s_red[4];
  __shared__ float s_o[4][D];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
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
  const int n = max(0, k1 - k0);
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  const size_t row_stride = static_cast<size_t>(p.H) * D;  // elements between cache rows
  const uint16_t* kc = p.k_cache + (static_cast<size_t>(b) * p.Ncap * p.H + h) * D + sub * 8;
  const uint16_t* vc = p.v_cache + (static_cast<size_t>(b) * p.Ncap * p.H + h) * D + sub * 8;
  const uint16_t* kn = append ? p.k_new + bh * D + sub * 8 : nullptr;
  const uint16_t* vn = append ? p.v_new + bh * D + sub * 8 : nullptr;

  // This chunk holds the appended row: persist it in the cache.
  if (do_append && L >= k0 && L < k1 && tid < LPR) {
    const size_t off = (static_cast<size_t>(b) * p.Ncap + L) * row_stride + h * D + tid * 8;
    *reinterpret_cast<uint4*>(p.k_cache + off) =
        *reinterpret_cast<const uint4*>(p.k_new + bh * D + tid * 8);
    *reinterpret_cast<uint4*>(p.v_cache + off) =
        *reinterpret_cast<const uint4*>(p.v_new + bh * D + tid * 8);
  }

  float qf[8];
  {
    const uint4 qu = *reinterpret_cast<const uint4*>(p.q + bh * D + sub * 8);
    bf16x8_to_f32(qu, qf);
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] *= p.scale_log2;
  }

  // Phase 1: scores (log2 units) of this chunk's keys.
  for (int base = k0 + warp * RPW; base < k1; base += U * RPC) {
    uint4 kv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = base + u * RPC + grp;
      kv[u] = make_uint4(0, 0, 0, 0);
      if (kb < k1) {
        const uint16_t* src = (do_append && kb == L) ? kn : kc + static_cast<size_t>(kb) * row_stride;
        kv[u] = __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float f[8];
      bf16x8_to_f32(kv[u], f);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(qf[i], f[i], acc);
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int kb = base + u * RPC + grp;
      if (sub == 0 && kb < k1) s_sc[kb - k0] = acc;
    }
  }
  __syncthreads();

  // Phase 2: chunk max and exp-sum.
  float mx = -INFINITY;
  for (int i = tid; i < n; i += 128) mx = fmaxf(mx, s_sc[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  const float m = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  const float ms = (m == -INFINITY) ? 0.f : m;
  __syncthreads();
  float sum = 0.f;
  for (int i = tid; i < n; i += 128) {
    const float e = ex2_approx(s_sc[i] - ms);
    s_sc[i] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_red[warp] = sum;
  __syncthreads();
  const float l = s_red[0] + s_red[1] + s_red[2] + s_red[3];

  // Phase 3: weighted sum of V rows.
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int base = k0 + warp * RPW; base < k1; base += U * RPC) {
    uint4 vv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = base + u * RPC + grp;
      vv[u] = make_uint4(0, 0, 0, 0);
      if (kb < k1) {
        const uint16_t* src = (do_append && kb == L) ? vn : vc + static_cast<size_t>(kb) * row_stride;
        vv[u] = __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = base + u * RPC + grp;
      const float w = (kb < k1) ? s_sc[kb - k0] : 0.f;
      float f[8];
      bf16x8_to_f32(vv[u], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, f[i], acc[i]);
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (grp == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s_o[warp][sub * 8 + i] = acc[i];
  }
  __syncthreads();

  const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
  const float lse_nat = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
  if (p.nsplit == 1) {
    if (tid < D / 2) {
      const int c = 2 * tid;
      const float o0 = (s_o[0][c] + s_o[1][c] + s_o[2][c] + s_o[3][c]) * inv_l;
      const float o1 = (s_o[0][c + 1] + s_o[1][c + 1] + s_o[2][c + 1] + s_o[3][c + 1]) * inv_l;
      reinterpret_cast<uint32_t*>(p.out + bh * D)[tid] = pack_bf16x2(o0, o1);
    }
    if (tid == 0 && p.lse) p.lse[bh] = lse_nat;
  } else {
    if (tid < D) {
      const float o = (s_o[0][tid] + s_o[1][tid] + s_o[2][tid] + s_o[3][tid]) * inv_l;
      p.part_o[(bh * p.nsplit + split) * D + tid] = o;
    }
    if (tid == 0) p.part_lse[bh * p.nsplit + split] = lse_nat;
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecodeParams p) {
  const size_t bh = blockIdx.x;
  const int tid = threadIdx.x;
  const float* pl = p.part_lse + bh * p.nsplit;
  float m = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) m = fmaxf(m, pl[s]);
  float tot = 0.f, acc = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < p.nsplit; ++s) {
      const float w = expf(pl[s] - m);
      tot += w;
      acc = fmaf(w, p.part_o[(bh * p.nsplit + s) * D + tid], acc);
    }
  }
  const float o = (tot > 0.f) ? acc / tot : 0.f;
  const float o_nb = __shfl_down_sync(0xffffffffu, o, 1);
  if ((tid & 1) == 0)
    reinterpret_cast<uint32_t*>(p.out + bh * D)[tid >> 1] = pack_bf16x2(o, o_nb);
  if (tid == 0 && p.lse) p.lse[bh] = (tot > 0.f) ? m + logf(tot) : -INFINITY;
}

}  // namespace fa
