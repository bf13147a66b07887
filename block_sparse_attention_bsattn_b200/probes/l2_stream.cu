// Probe: aggregate L2 -> SM throughput of the prefill's K/V stream.
// Each CTA streams 64 KB steps (a 128x128 bf16 K tile and V tile, each as two
// 64-column 128B-swizzled TMA boxes, exactly like the prefill kernels) through
// a ring of `stages` steps; one thread issues and waits.  All coordinates are
// in range: x in {0, 64}, y = tile * 128 with tile < nk, z < heads.
// Build and run (from the repository root):
//   python -m block_sparse_attention_bsattn_b200.build --probes
//   block_sparse_attention_bsattn_b200/_build/probes/l2_stream
#include <cstdio>
#include <cstdint>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>
#include "sm100_ptx.cuh"
using namespace bsattn;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

__global__ void stream(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       int steps, int stages, int nk, int heads, int ctas_per_head, int halves_only,
                       int* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t bars[8];
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  volatile int abort = 0;
  const int z = (blockIdx.x / ctas_per_head) % heads;
  int j = (blockIdx.x * 37) % nk;
  const uint32_t step_bytes = halves_only ? 32768 : 65536;
  auto issue = [&](int s, int tile) {
    uint8_t* dst = sm + (size_t)s * step_bytes;
    mbar_arrive_expect_tx(&bars[s], step_bytes);
    if (halves_only) {  // K half-tile of 64 keys (both boxes) + V one box
      tma_load_3d(dst, &tk, &bars[s], 0, tile * 128, z);
      tma_load_3d(dst + 8192, &tk, &bars[s], 64, tile * 128, z);
      tma_load_3d(dst + 16384, &tv, &bars[s], 0, tile * 128, z);
    } else {
      tma_load_3d(dst, &tk, &bars[s], 0, tile * 128, z);
      tma_load_3d(dst + 16384, &tk, &bars[s], 64, tile * 128, z);
      tma_load_3d(dst + 32768, &tv, &bars[s], 0, tile * 128, z);
      tma_load_3d(dst + 49152, &tv, &bars[s], 64, tile * 128, z);
    }
  };
  int issued = 0;
  for (; issued < stages && issued < steps; ++issued) { issue(issued, j); j = (j + 1) % nk; }
  for (int done = 0; done < steps; ++done) {
    const int s = done % stages;
    const uint32_t par = (done / stages) & 1;
    if (!mbar_wait(&bars[s], par, &abort, 2000000000ull)) {
      atomicExch(err, 1);
      for (int d = done; d < issued; ++d)
        mbar_wait_drain(&bars[d % stages], (d / stages) & 1, 1000000000ull);
      return;
    }
    if (issued < steps) { issue(s, j); j = (j + 1) % nk; ++issued; }
  }
}

int main() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q);
  EncodeTiledFn enc = (EncodeTiledFn)ptr;
  const uint64_t D = 128, N = 32768, H = 8;
  const size_t bytes = D * N * H * 2;
  void *k, *v;
  cudaMalloc(&k, bytes); cudaMalloc(&v, bytes);
  cudaMemset(k, 0, bytes); cudaMemset(v, 0, bytes);
  CUtensorMap mk, mv;
  cuuint64_t dims[3] = {D, N, H};
  cuuint64_t str[2] = {D * 2, D * N * 2};
  cuuint32_t box[3] = {64, 128, 1}, box_half[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  int* err; cudaMalloc(&err, 4); cudaMemset(err, 0, 4);
  int nsm = 0; cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  struct Cfg { int ctas_mult, stages, heads, cph, halves; const char* what; };
  std::vector<Cfg> cfgs = {
      {1, 3, 1, 1 << 20, 0, "1 CTA/SM, 3 stages, one KV head (L2 resident)"},
      {1, 2, 1, 1 << 20, 0, "1 CTA/SM, 2 stages, one KV head"},
      {1, 3, 8, 19, 0, "1 CTA/SM, 3 stages, 8 KV heads (134 MB)"},
      {2, 1, 1, 1 << 20, 0, "2 CTA/SM, 1 stage each, one KV head"},
      {1, 3, 1, 1 << 20, 1, "1 CTA/SM, 3 stages of 32 KB (half K + half V), one KV head"},
      {1, 6, 1, 1 << 20, 1, "1 CTA/SM, 6 stages of 32 KB, one KV head"},
  };
  for (const Cfg& c : cfgs) {
    enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (c.halves) {
      // K: box of 64 rows (first half of the tile) x 64 columns, both column halves;
      // V: box 128 rows x 64 columns (one column half).
      enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, str, box_half, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    const int grid = nsm * c.ctas_mult;
    const int step_bytes = c.halves ? 32768 : 65536;
    const int smem = c.stages * step_bytes + 1024;
    cudaFuncSetAttribute(stream, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int steps = c.halves ? 4000 : 2000;
    for (int rep = 0; rep < 3; ++rep) {
      cudaEventRecord(e0);
      stream<<<grid, 32, smem>>>(mk, mv, steps, c.stages, 256, c.heads, c.cph, c.halves, err);
      cudaEventRecord(e1);
      cudaError_t e = cudaEventSynchronize(e1);
      float ms = 0; cudaEventElapsedTime(&ms, e0, e1);
      int he = 0; cudaMemcpy(&he, err, 4, cudaMemcpyDeviceToHost);
      double tot = (double)grid * steps * step_bytes;
      printf("%-62s grid %d: %s err=%d  %.3f ms  %.2f TB/s  %.0f cycles/step/CTA@1.965GHz\n", c.what, grid,
             cudaGetErrorString(e), he, ms, tot / ms / 1e9, ms * 1e-3 * 1.965e9 / steps);
    }
  }
  return 0;
}
