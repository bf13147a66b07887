// Probe: cost of reading S back from TMEM (tcgen05.ld 32x32b.x32 + wait) by
// 4 or 8 warps, the 128-element row max, and a 4-warp bar.red.
// Build and run (from the repository root):
//   python -m block_sparse_attention_bsattn_b200.build --probes
//   block_sparse_attention_bsattn_b200/_build/probes/tmem_rate
#include <cstdio>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "sm100_ptx.cuh"
using namespace bsattn;

__global__ void probe(int nwarps_ld, int iters, long long* out) {
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  const uint32_t lane_addr = tm + ((uint32_t)((warp % 4) * 32) << 16);
  float acc = 0.f;
  long long t_ld = 0, t_max = 0, t_bar = 0;
  if (warp < nwarps_ld) {
    for (int it = 0; it < iters; ++it) {
      long long c0 = clock64();
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 128; c += 32)
        tmem_ld32(lane_addr + (warp / 4) * 256 + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
      tmem_wait_ld();
      long long c1 = clock64();
      const float m = row_max<128>(reinterpret_cast<const float*>(r));
      long long c2 = clock64();
      const bool all = bar_red_and(1 + (warp / 4), 128, m < 1e30f);
      long long c3 = clock64();
      acc += m + (all ? 1.f : 0.f);
      t_ld += c1 - c0; t_max += c2 - c1; t_bar += c3 - c2;
    }
  }
  if (lane == 0 && warp < nwarps_ld) {
    out[warp * 3 + 0] = t_ld / iters;
    out[warp * 3 + 1] = t_max / iters;
    out[warp * 3 + 2] = t_bar / iters;
  }
  if (acc == 12345.f) out[63] = 1;   // keep the work
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tm, 512); }
}

int main() {
  long long* d; cudaMalloc(&d, 64 * 8);
  long long h[64];
  for (int nw : {4, 8}) {
    cudaMemset(d, 0, 64 * 8);
    probe<<<1, nw * 32>>>(nw, 200, d);
    cudaError_t e = cudaDeviceSynchronize();
    cudaMemcpy(h, d, 64 * 8, cudaMemcpyDeviceToHost);
    printf("%d warps (%s): ld+wait / max / bar.red cycles per tile, per warp:", nw, cudaGetErrorString(e));
    for (int w = 0; w < nw; ++w) printf(" [%lld %lld %lld]", h[w * 3], h[w * 3 + 1], h[w * 3 + 2]);
    printf("\n");
  }
  return 0;
}
