// The exact combine of a split-KV decode's splits (the splits themselves run
// in decode_sm100.cu).
//
// "BLASST: Dynamic Blocked Attention Sparsity via Softmax Thresholding",
// section 4.2: each split of a (batch, KV head) problem leaves its
// unnormalised O (fp32), its exponent shift and its row sum; the splits are
// merged by log-sum-exp.
// decode_combine_kernel: one CTA per (batch, query head): the merge into bf16
//   O and fp32 LSE.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

// One CTA per (batch, query head), one thread per output dimension.
__global__ void decode_combine_kernel(const CombineParams p) {
  const int64_t bh = blockIdx.x;
  const int dd = threadIdx.x;
  const float* m = p.ws_m + bh * p.splits;
  const float* l = p.ws_l + bh * p.splits;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, m[s]);
  float num = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      if (m[s] == -INFINITY) continue;
      const float w = fast_exp2(m[s] - M);
      den += w * l[s];
      num += w * p.ws_o[(bh * p.splits + s) * p.D + dd];
    }
  }
  const bool have = den > 0.f;
  p.o[bh * p.D + dd] = __float2bfloat16_rn(have ? num / den : 0.f);
  if (dd == 0 && p.lse) p.lse[bh] = have ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY;
}

cudaError_t launch_decode_combine(const CombineParams& p, int grid, int threads,
                                  cudaStream_t stream) {
  decode_combine_kernel<<<grid, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace bsattn
