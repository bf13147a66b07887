// Probe: how long one thread takes to issue the prefill's MMA groups on an
// idle tensor pipe, and how long they take to complete.  A group is one BMM1
// of the two-tile prefill kernel (8 tcgen05.mma of 128 x 128 x 16, A and B from
// shared memory, descriptors built per MMA as the kernel builds them), the
// same with the descriptors built before the clock starts, two BMM1s back to
// back (16 MMAs into two accumulators), and one BMM2 (8 MMAs with A from TMEM).
// Optionally eight more warps run FMA chains meanwhile (the softmax warps'
// share of the issue slots).  A second part times, right after one BMM1 and
// its commit, three shared-memory operations of the same thread: a try_wait
// on a barrier whose phase completed long before, a volatile load of a flag,
// and an arrive.  One CTA; all operands zero.
// Build and run (from the repository root):
//   python -m block_sparse_attention_bsattn_b200.build --probes
//   block_sparse_attention_bsattn_b200/_build/probes/mma_issue
#include <cstdio>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include "sm100_ptx.cuh"
using namespace bsattn;

constexpr int Q_HALF = 128 * 128;      // bytes of one 64-column box of a 128-row tile
constexpr int Q_BYTES = 2 * Q_HALF;    // one 128 x 128 bf16 tile
constexpr int SMEM = 3 * Q_BYTES + 1024 + 64;

__global__ void after_commit(int what, int reps, long long* out) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bar = (uint64_t*)(sm + 3 * Q_BYTES);          // MMA completion
  uint64_t* done = bar + 1;                              // completed once, at set-up
  uint64_t* sink = bar + 2;                              // arrivals only
  volatile int* flag = (volatile int*)(sm + 3 * Q_BYTES + 32);
  __shared__ uint32_t tbase;
  for (int i = threadIdx.x; i < 3 * Q_BYTES / 4; i += blockDim.x) ((uint32_t*)sm)[i] = 0;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init(done, 1);
    mbar_init(sink, (1 << 20) - 1);
    *flag = 1;
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  const int warp = threadIdx.x / 32;
  if (warp == 1) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 32) {
    mbar_arrive(done);   // phase 0 of `done` completes here
    const uint32_t q_addr = smem_u32(sm), k_addr = smem_u32(sm + 2 * Q_BYTES);
    constexpr uint32_t IDESC1 = idesc_bf16_f32(128, 128, 0, 0);
    volatile int ab = 0;
    long long s_op = 0, s_mma = 0;
    bool ok = true;
    for (int r = 0; r < reps + 4 && ok; ++r) {
      const long long t0 = clock64();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = q_addr + (kk / 4) * Q_HALF + (kk % 4) * 32;
        const uint32_t b = k_addr + (kk / 4) * Q_HALF + (kk % 4) * 32;
        mma_ss(tm, smem_desc(a, 16, 1024, 2), smem_desc(b, 16, 1024, 2), IDESC1, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar);
      const long long t1 = clock64();
      int v = 0;
      if (what == 0) v = mbar_try_wait(done, 0) ? 1 : 0;
      else if (what == 1) v = *flag;
      else if (what == 2) mbar_arrive(sink);
      else v = 1;
      const long long t2 = clock64();
      ok = mbar_wait(bar, r & 1, &ab, 1000000000ull);
      if (r >= 4) {
        s_op += t2 - t1;
        s_mma += t1 - t0;
      }
      if (v == 7) out[7] = 1;
    }
    out[0] = ok ? s_op / reps : -1;
    out[1] = ok ? s_mma / reps : -1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

__global__ void probe(int pattern, int busy, int reps, long long* out) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bar = (uint64_t*)(sm + 3 * Q_BYTES);
  volatile int* stop = (volatile int*)(sm + 3 * Q_BYTES + 16);
  __shared__ uint32_t tbase;
  for (int i = threadIdx.x; i < 3 * Q_BYTES / 4; i += blockDim.x) ((uint32_t*)sm)[i] = 0;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *stop = 0;
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  const int warp = threadIdx.x / 32;
  if (warp == 1) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (threadIdx.x == 32) {
    const uint32_t q_addr = smem_u32(sm), k_addr = smem_u32(sm + 2 * Q_BYTES);
    constexpr uint32_t IDESC1 = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC2 = idesc_bf16_f32(128, 128, 0, 1);
    volatile int ab = 0;
    uint64_t pa[8], pb[8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      pa[kk] = smem_desc(q_addr + (kk / 4) * Q_HALF + (kk % 4) * 32, 16, 1024, 2);
      pb[kk] = smem_desc(k_addr + (kk / 4) * Q_HALF + (kk % 4) * 32, 16, 1024, 2);
    }
    long long s_issue = 0, s_total = 0, m_issue = 1LL << 60, m_total = 1LL << 60;
    bool ok = true;
    for (int r = 0; r < reps + 4 && ok; ++r) {
      const int e = r & 1;
      const long long t0 = clock64();
      if (pattern == 0 || pattern == 2) {
        for (int g = 0; g < (pattern == 2 ? 2 : 1); ++g) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t a = q_addr + ((e + g) & 1) * Q_BYTES + (kk / 4) * Q_HALF + (kk % 4) * 32;
            const uint32_t b = k_addr + (kk / 4) * Q_HALF + (kk % 4) * 32;
            mma_ss(tm + 256 * g, smem_desc(a, 16, 1024, 2), smem_desc(b, 16, 1024, 2), IDESC1,
                   kk > 0 ? 1u : 0u);
          }
        }
      } else if (pattern == 1) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(tm, pa[kk], pb[kk], IDESC1, kk > 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t b = k_addr + kk * (16 * 128);
          mma_ts(tm + 128, tm + kk * 8, smem_desc(b, Q_HALF, 1024, 2), IDESC2, 1u);
        }
      }
      const long long t1 = clock64();
      mma_commit(bar);
      ok = mbar_wait(bar, r & 1, &ab, 1000000000ull);
      const long long t2 = clock64();
      if (r >= 4) {
        s_issue += t1 - t0;
        s_total += t2 - t0;
        m_issue = min(m_issue, t1 - t0);
        m_total = min(m_total, t2 - t0);
      }
    }
    out[0] = ok ? s_issue / reps : -1;
    out[1] = ok ? s_total / reps : -1;
    out[2] = m_issue;
    out[3] = m_total;
    *stop = 1;
  } else if (busy && warp >= 2) {
    // FMA chains until the issuer is done (bounded)
    float x = threadIdx.x * 1e-3f, y = 1.0001f;
    for (int i = 0; i < 4000000 && !*stop; ++i) {
#pragma unroll
      for (int j = 0; j < 16; ++j) x = fmaf(x, y, 1e-7f);
    }
    if (x == 12345.f) out[7] = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

int main() {
  long long* d;
  cudaMalloc(&d, 8 * 8);
  cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  cudaFuncSetAttribute(after_commit, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  const char* names[] = {"BMM1, 8 SS MMAs, descriptors built per MMA",
                         "BMM1, 8 SS MMAs, descriptors built before",
                         "two BMM1s back to back, 16 SS MMAs",
                         "BMM2, 8 TS MMAs (A from TMEM)"};
  for (int busy : {0, 1})
    for (int pat = 0; pat < 4; ++pat) {
      cudaMemset(d, 0, 64);
      probe<<<1, busy ? 320 : 64, SMEM>>>(pat, busy, 64, d);
      const cudaError_t e = cudaDeviceSynchronize();
      long long h[8];
      cudaMemcpy(h, d, 64, cudaMemcpyDeviceToHost);
      printf("%-46s %s %s: issue %lld (min %lld) cycles, issue to complete %lld (min %lld)\n",
             names[pat], busy ? "+ 8 FMA warps" : "alone        ", cudaGetErrorString(e), h[0], h[2],
             h[1], h[3]);
    }
  const char* ops[] = {"try_wait on a completed barrier", "volatile flag load", "mbarrier arrive",
                       "nothing"};
  for (int what = 0; what < 4; ++what) {
    cudaMemset(d, 0, 64);
    after_commit<<<1, 64, SMEM>>>(what, 64, d);
    const cudaError_t e = cudaDeviceSynchronize();
    long long h[8];
    cudaMemcpy(h, d, 64, cudaMemcpyDeviceToHost);
    printf("after a BMM1 and its commit: %-34s %s: %lld cycles (BMM1 issue + commit %lld)\n",
           ops[what], cudaGetErrorString(e), h[0], h[1]);
  }
  return 0;
}
