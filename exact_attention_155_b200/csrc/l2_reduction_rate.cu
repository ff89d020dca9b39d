// Standalone measurement (not part of libfa.so): throughput of bulk fp32 reductions
// (cp.reduce.async.bulk .add.f32) from shared memory into a 256 MiB global accumulator,
// the operation the backward kernel uses to add dQ blocks into its fp32 accumulator.
// 148 CTAs (one per SM) each reduce 16 KB chunks in a loop with 2, 4 or 8 staging
// buffers in flight. Build and run on a B200:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o l2_reduction_rate l2_reduction_rate.cu
//   ./l2_reduction_rate
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
template <int NB>
__global__ void __launch_bounds__(128) k(float* g, long long region_floats, int iters, long long* cyc) {
  extern __shared__ __align__(128) uint8_t sm[];
  for (int i = threadIdx.x; i < NB * 4096; i += 128) reinterpret_cast<float*>(sm)[i] = 1e-3f;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  long long t0 = clock64();
  if (threadIdx.x == 0) {
    for (int i = 0; i < iters; ++i) {
      if (i >= NB) {
        if (NB == 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        if (NB == 4) asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
        if (NB == 8) asm volatile("cp.async.bulk.wait_group.read 7;" ::: "memory");
      }
      const long long chunk = (static_cast<long long>(blockIdx.x) * iters + i) % (region_floats / 4096);
      float* dst = g + chunk * 4096;
      const uint32_t src = smem_u32(sm + (i % NB) * 16384);
      asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(16384) : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    cyc[blockIdx.x] = clock64() - t0;
  }
}
int main() {
  const long long region = 64ll << 20;  // 64 M floats = 256 MiB, like the dQ accumulator
  float* g; long long* cyc;
  cudaMalloc(&g, region * 4); cudaMemset(g, 0, region * 4); cudaMalloc(&cyc, 148 * 8);
  const int iters = 256;
  auto run = [&](auto kern, int nb, const char* name) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, nb * 16384);
    for (int rep = 0; rep < 2; ++rep) {
      cudaEvent_t a, b; cudaEventCreate(&a); cudaEventCreate(&b);
      cudaEventRecord(a);
      kern<<<148, 128, nb * 16384>>>(g, region, iters, cyc);
      cudaEventRecord(b);
      cudaError_t e = cudaDeviceSynchronize();
      float ms; cudaEventElapsedTime(&ms, a, b);
      long long h[148]; cudaMemcpy(h, cyc, sizeof(h), cudaMemcpyDeviceToHost);
      double avg = 0; for (int i = 0; i < 148; ++i) avg += h[i]; avg /= 148;
      double bytes = 148.0 * iters * 16384;
      if (rep) printf("%s: %.1f B/clk/SM, %.2f TB/s by events (%s)\n", name, iters * 16384.0 / avg, bytes / (ms * 1e-3) / 1e12, cudaGetErrorString(e));
    }
  };
  run(k<2>, 2, "2 buffers");
  run(k<4>, 4, "4 buffers");
  run(k<8>, 8, "8 buffers");
  return 0;
}
