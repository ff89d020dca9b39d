// Running fp32 sum of bf16 partial results, with an optional bf16 copy of the sum.
//
// Attention split over sequence shards (the ring sequence-parallel mode of
// "Flash-Attention 2/3在ms-swift中的集成与性能提升", section on distributed training)
// produces each gradient as a sum over shard pairs: with the whole row's LSE and
// output fixed by the forward, the recomputed backward of "ms-swift长文本训练优化，
// Flash-Attention显存省一半" (section 1.2) is linear in the key set, so dQ of a query
// shard is the sum of its terms against every key shard and dK, dV of a key shard the
// sum of their terms from every query shard. The partial terms arrive as bf16 and the
// sum is kept in fp32. HBM bound; one thread per 8 elements.
#pragma once

#include "ptx.cuh"

namespace fa {

struct AccumParams {
  float* acc;            // n fp32 (read, written)
  const uint16_t* part;  // n bf16 added to acc, or null (acc unchanged)
  uint16_t* out;         // n bf16 copy of the sum, or null
  long long n8;          // n / 8
};

__global__ void __launch_bounds__(256) accumulate_kernel(const AccumParams p) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= p.n8) return;
  float4* a = reinterpret_cast<float4*>(p.acc) + 2 * i;
  float4 a0 = a[0], a1 = a[1];
  if (p.part != nullptr) {
    const uint4 u = reinterpret_cast<const uint4*>(p.part)[i];
    // bf16 -> fp32 is exact: the 16 bits are the top half of the fp32 pattern.
    a0.x += __uint_as_float(u.x << 16);
    a0.y += __uint_as_float(u.x & 0xFFFF0000u);
    a0.z += __uint_as_float(u.y << 16);
    a0.w += __uint_as_float(u.y & 0xFFFF0000u);
    a1.x += __uint_as_float(u.z << 16);
    a1.y += __uint_as_float(u.z & 0xFFFF0000u);
    a1.z += __uint_as_float(u.w << 16);
    a1.w += __uint_as_float(u.w & 0xFFFF0000u);
    a[0] = a0;
    a[1] = a1;
  }
  if (p.out != nullptr) {
    uint4 o;
    o.x = pack_bf16x2(a0.x, a0.y);
    o.y = pack_bf16x2(a0.z, a0.w);
    o.z = pack_bf16x2(a1.x, a1.y);
    o.w = pack_bf16x2(a1.z, a1.w);
    reinterpret_cast<uint4*>(p.out)[i] = o;
  }
}

}  // namespace fa
