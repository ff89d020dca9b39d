// LSE merge of two partial attention results over disjoint key sets, for attention
// split over sequence shards (ring attention: each device runs attention of its query
// shard against one key/value shard at a time and folds the result into a running
// output, as the ring sequence-parallel mode of "Flash-Attention 2/3在ms-swift中的集成与
// 性能提升" (section on distributed training) describes). The combination is the stable
// per-block (m, l) merge of section 2.2.2 of "FlashAttention优化Transformer显存与计算效率"
// in log space: LSE = log(e^lse_a + e^lse_p), O = e^(lse_a - LSE) O_a + e^(lse_p - LSE) O_p,
// with O_a, O_p each normalised over their own keys. HBM bound; one thread per 8 columns.
#pragma once

#include <math.h>

#include "ptx.cuh"

namespace fa {

struct MergeParams {
  float* o_acc;          // [B, N, H, d] fp32, running output (normalised)
  float* lse_acc;        // [B, H, N] fp32, running LSE (-inf: nothing merged yet)
  const uint16_t* o_part;  // [B, N, H, d] bf16 partial output
  const float* lse_part;   // [B, H, N] fp32 partial LSE
  uint16_t* out;         // [B, N, H, d] bf16 copy of the merged output, or null
  int B, N, H;
};

template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  constexpr int TPR = D / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long rows = static_cast<long long>(p.B) * p.N * p.H;
  const long long row = gt / TPR;  // (b, n, h) in [B, N, H] order
  if (row >= rows) return;
  const int sub = static_cast<int>(gt % TPR);
  const int h = static_cast<int>(row % p.H);
  const long long bn = row / p.H;
  const int n = static_cast<int>(bn % p.N);
  const int b = static_cast<int>(bn / p.N);
  const size_t li = (static_cast<size_t>(b) * p.H + h) * p.N + n;
  const float la = p.lse_acc[li], lp = p.lse_part[li];
  const float m = fmaxf(la, lp);
  float* oa = p.o_acc + row * D + sub * 8;
  float res[8];
  if (m == -INFINITY) {  // neither part has a visible key
#pragma unroll
    for (int i = 0; i < 8; ++i) res[i] = oa[i];
  } else {
    const float wa = la == -INFINITY ? 0.f : expf(la - m);
    const float wp = lp == -INFINITY ? 0.f : expf(lp - m);
    const float inv = 1.f / (wa + wp);
    const uint4 u = *reinterpret_cast<const uint4*>(p.o_part + row * D + sub * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p0 = __uint_as_float(w[i] << 16), p1 = __uint_as_float(w[i] & 0xFFFF0000u);
      res[2 * i] = (wa * oa[2 * i] + wp * p0) * inv;
      res[2 * i + 1] = (wa * oa[2 * i + 1] + wp * p1) * inv;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) oa[i] = res[i];
    // The row's TPR threads are consecutive lanes of one warp and all read lse_acc[li]
    // above; the write waits until every one of them has.
    const int lane = static_cast<int>(threadIdx.x & 31);
    const unsigned row_mask = (TPR == 32 ? 0xffffffffu : ((1u << TPR) - 1u)) << (lane - sub);
    __syncwarp(row_mask);
    if (sub == 0) p.lse_acc[li] = m + logf(wa + wp);
  }
  if (p.out != nullptr) {
    uint4 o;
    o.x = pack_bf16x2(res[0], res[1]);
    o.y = pack_bf16x2(res[2], res[3]);
    o.z = pack_bf16x2(res[4], res[5]);
    o.w = pack_bf16x2(res[6], res[7]);
    *reinterpret_cast<uint4*>(p.out + row * D + sub * 8) = o;
  }
}

}  // namespace fa
