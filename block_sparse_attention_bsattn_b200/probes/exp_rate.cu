// Probe: exponentials per SM clock for the forms a softmax pass can use on
// sm_100a: the special-function unit on fp32, on packed f16 pairs and on packed
// bf16 pairs, the prefill's fp32 pair step (scale FMA, two exponentials, bf16
// pack, row-sum add), the same step through packed f16, and the FMA-pipe
// exponential (exp2_fma2, no special-function unit).  One CTA per SM with 8 or
// 16 warps; each thread runs ITERS iterations over 16 independent values.
// Build and run (from the repository root):
//   python -m block_sparse_attention_bsattn_b200.build --probes
//   block_sparse_attention_bsattn_b200/_build/probes/exp_rate
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "sm100_ptx.cuh"
using namespace bsattn;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t ex2h2(uint32_t x) {
  uint32_t y;
  asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t ex2b2(uint32_t x) {
  uint32_t y;
  asm volatile("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t subh2(uint32_t a, uint32_t b) {
  uint32_t y;
  asm volatile("sub.f16x2 %0, %1, %2;" : "=r"(y) : "r"(a), "r"(b));
  return y;
}
__device__ __forceinline__ uint32_t subb2(uint32_t a, uint32_t b) {
  uint32_t y;
  asm volatile("sub.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(a), "r"(b));
  return y;
}
__device__ __forceinline__ uint32_t cvt_h2(float lo, float hi) {
  uint32_t y;
  asm volatile("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(y) : "f"(hi), "f"(lo));
  return y;
}
__device__ __forceinline__ float2 h2f(uint32_t h) {
  float a, b;
  asm volatile("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
               "cvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
               : "=f"(a), "=f"(b) : "r"(h));
  return make_float2(a, b);
}

__global__ void k_exp(int variant, int iters, float seed, uint32_t* sink, long long* cyc) {
  float v[16];
  uint32_t h[8];
  for (int i = 0; i < 16; ++i) v[i] = -0.01f * (threadIdx.x % 7 + i) - seed;
  for (int i = 0; i < 8; ++i) h[i] = cvt_h2(v[2 * i], v[2 * i + 1]);
  const uint32_t c15h = cvt_h2(1.5f, 1.5f);
  const uint32_t c15b = pack_bf16x2(1.5f, 1.5f);
  float acc = 0.f;
  uint32_t pk = 0;
  __syncthreads();
  const long long t0 = clock64();
  if (variant == 0) {          // 16 x ex2.f32 (a subtraction each keeps the values in range)
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = ex2f(v[i]) - 1.5f;
  } else if (variant == 1) {   // 8 x ex2.f16x2: 16 results
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = subh2(ex2h2(h[i]), c15h);
  } else if (variant == 2) {   // 8 x ex2.bf16x2: 16 results
    for (int i = 0; i < 8; ++i) h[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = subb2(ex2b2(h[i]), c15b);
  } else if (variant == 3) {   // the prefill's pair step, fp32
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 x = ffma2(make_float2(v[2 * i], v[2 * i + 1]), make_float2(0.9f, 0.9f),
                               make_float2(-0.1f, -0.1f));
        const float ea = ex2f(x.x), eb = ex2f(x.y);
        pk ^= pack_bf16x2(ea, eb);
        acc += ea + eb;
        v[2 * i] = ea - 1.5f;
        v[2 * i + 1] = eb - 1.5f;
      }
    }
  } else if (variant == 4) {   // the same step through packed f16 exponentials
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 x = ffma2(make_float2(v[2 * i], v[2 * i + 1]), make_float2(0.9f, 0.9f),
                               make_float2(-0.1f, -0.1f));
        const float2 e = h2f(ex2h2(cvt_h2(x.x, x.y)));
        pk ^= pack_bf16x2(e.x, e.y);
        acc += e.x + e.y;
        v[2 * i] = e.x - 1.5f;
        v[2 * i + 1] = e.y - 1.5f;
      }
    }
  } else if (variant == 5) {   // FMA-pipe exponential on pairs
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 e = exp2_fma2(make_float2(v[2 * i], v[2 * i + 1]));
        v[2 * i] = e.x - 1.5f;
        v[2 * i + 1] = e.y - 1.5f;
      }
    }
  }
  const long long t1 = clock64();
  for (int i = 0; i < 16; ++i) acc += v[i];
  for (int i = 0; i < 8; ++i) pk ^= h[i];
  if (__float_as_uint(acc) == 0x7f7f7f7fu && pk == 0x12345u) sink[0] = pk;   // keep the work
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

int main() {
  int nsm = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
  uint32_t* sink;
  long long* cyc;
  cudaMalloc(&sink, 4);
  cudaMalloc(&cyc, 8 * 1024);
  const int iters = 4096;
  const char* names[] = {"ex2.approx.ftz.f32", "ex2.approx.f16x2", "ex2.approx.ftz.bf16x2",
                         "pair step, fp32 (fma2, 2 ex2, pack, add)", "pair step via ex2.f16x2",
                         "exp2_fma2 (FMA pipe)"};
  for (int warps : {8, 16}) {
    for (int var = 0; var < 6; ++var) {
      k_exp<<<nsm, warps * 32>>>(var, 64, 0.5f, sink, cyc);   // warm-up
      cudaEvent_t e0, e1;
      cudaEventCreate(&e0);
      cudaEventCreate(&e1);
      cudaEventRecord(e0);
      k_exp<<<nsm, warps * 32>>>(var, iters, 0.5f, sink, cyc);
      cudaEventRecord(e1);
      const cudaError_t e = cudaEventSynchronize(e1);
      float ms = 0;
      cudaEventElapsedTime(&ms, e0, e1);
      long long c = 0;
      cudaMemcpy(&c, cyc, 8, cudaMemcpyDeviceToHost);
      const double results = 16.0 * iters * warps * 32;   // per CTA = per SM
      printf("%2d warps/SM  %-42s %s  %.3f ms  %lld cycles  %.2f exps/clk/SM\n", warps, names[var],
             cudaGetErrorString(e), ms, c, results / (double)c);
    }
  }
  return 0;
}
