// Probe: cycles per tcgen05.mma (kind::f16, SS, bf16 -> f32) for M = 64 / 128.
// One CTA, all operands zero in shared memory; D in TMEM columns [0, N).
// Build and run (from the repository root):
//   python -m block_sparse_attention_bsattn_b200.build --probes
//   block_sparse_attention_bsattn_b200/_build/probes/mma_rate
#include <cstdio>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "sm100_ptx.cuh"
using namespace bsattn;

__global__ void probe(int M, int N, int iters, long long* out) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bar = (uint64_t*)(sm + 49152);
  __shared__ uint32_t tbase;
  for (int i = threadIdx.x; i < 49152 / 4; i += blockDim.x) ((uint32_t*)sm)[i] = 0;
  if (threadIdx.x == 0) { mbar_init(bar, 1); fence_barrier_init(); }
  fence_proxy_async_smem();
  if (threadIdx.x / 32 == 1) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 32) {
    const uint32_t a = smem_u32(sm), b = smem_u32(sm + 16384);
    const uint32_t idesc = idesc_bf16_f32(M, N, 0, 0);
    volatile int ab = 0;
    // warm-up
    for (int i = 0; i < 64; ++i)
      mma_ss(tm, smem_desc(a + (i & 3) * 32, 16, 1024, 2), smem_desc(b + (i & 3) * 32, 16, 1024, 2), idesc, i > 0);
    mma_commit(bar);
    mbar_wait(bar, 0, (volatile int*)&ab, 1000000000ull);
    long long t0 = clock64();
    for (int i = 0; i < iters; ++i)
      mma_ss(tm, smem_desc(a + (i & 3) * 32, 16, 1024, 2), smem_desc(b + (i & 3) * 32, 16, 1024, 2), idesc, 1);
    mma_commit(bar);
    bool ok = mbar_wait(bar, 1, (volatile int*)&ab, 1000000000ull);
    long long t1 = clock64();
    out[0] = ok ? (t1 - t0) : -1;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x / 32 == 1) { tc_fence_after(); tmem_dealloc(tm, 512); }
}

int main() {
  long long* d; cudaMalloc(&d, 8);
  cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, 52 * 1024);
  const int iters = 4096;
  for (int M : {64, 128})
    for (int N : {64, 128, 256}) {
      probe<<<1, 128, 52 * 1024>>>(M, N, iters, d);
      cudaError_t e = cudaDeviceSynchronize();
      long long c = -2; cudaMemcpy(&c, d, 8, cudaMemcpyDeviceToHost);
      double fl = 2.0 * M * N * 16;
      printf("M=%d N=%d K=16: %s cycles/mma %.1f  flop/cycle %.0f\n", M, N, cudaGetErrorString(e),
             (double)c / iters, fl * iters / (double)c);
    }
  return 0;
}
