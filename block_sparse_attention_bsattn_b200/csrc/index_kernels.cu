// Block mask -> per-query-block CSR lists ("块稀疏Attention实战", section 2.3:
// the 0/1 block mask kept as an index of its non-zero blocks; section 3.3:
// the attention tiling loop walks that index instead of testing every block).
//
// Three small launches on the caller's stream (a fourth for the optional
// longest-first row order):
//   count: one warp per (mask head, query block) row counts the kept key
//          blocks (ballot over 32 columns at a time) into row_ptr[.. + i + 1];
//   scan:  one CTA turns the counts into absolute offsets (inclusive scan over
//          the flattened [mask_heads][nq + 1] array whose slot 0 of each head
//          holds 0) and writes nnz per head;
//   fill:  one warp per row writes the ascending column indices.
#include <cstdint>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

__device__ __forceinline__ bool keep_block(const IndexArgs& a, int h, int i, int j) {
  if (j >= a.nk) return false;
  if (a.causal && (int64_t)j * a.k_block > (int64_t)(i + 1) * a.q_block - 1) return false;
  return a.mask[((int64_t)h * a.nq + i) * a.nk + j] != 0;
}

__global__ void index_count_kernel(IndexArgs a) {
  const int warps = blockDim.x / 32;
  const int64_t row = (int64_t)blockIdx.x * warps + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= (int64_t)a.mask_heads * a.nq) return;
  const int h = (int)(row / a.nq), i = (int)(row % a.nq);
  int cnt = 0;
  for (int j0 = 0; j0 < a.nk; j0 += 32) {
    const bool k = keep_block(a, h, i, j0 + lane);
    cnt += __popc(__ballot_sync(0xffffffffu, k));
  }
  if (lane == 0) {
    a.row_ptr[(int64_t)h * (a.nq + 1) + i + 1] = cnt;
    if (i == 0) a.row_ptr[(int64_t)h * (a.nq + 1)] = 0;
  }
}

// Single CTA of 1024 threads: inclusive scan of n entries in chunks.
__global__ void __launch_bounds__(1024) index_scan_kernel(IndexArgs a) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry_s;
  const int64_t n = (int64_t)a.mask_heads * (a.nq + 1);
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += 1024) {
    const int64_t idx = base + tid;
    int32_t x = idx < n ? a.row_ptr[idx] : 0;
    // warp inclusive scan
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int32_t s = warp_sums[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += y;
      }
      warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int32_t carry = carry_s;
    const int32_t incl = x + (warp > 0 ? warp_sums[warp - 1] : 0) + carry;
    if (idx < n) a.row_ptr[idx] = incl;
    __syncthreads();
    if (tid == 1023) carry_s = incl;
    __syncthreads();
  }
  // per-head nnz and the capacity check
  for (int h = tid; h < a.mask_heads; h += 1024) {
    const int32_t s = a.row_ptr[(int64_t)h * (a.nq + 1)];
    const int32_t e = a.row_ptr[(int64_t)h * (a.nq + 1) + a.nq];
    a.nnz[h] = e - s;
  }
  if (tid == 0 && (int64_t)carry_s > a.capacity) report_status(a.status, kDevCapacity);
}

__global__ void index_fill_kernel(IndexArgs a) {
  const int warps = blockDim.x / 32;
  const int64_t row = (int64_t)blockIdx.x * warps + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= (int64_t)a.mask_heads * a.nq) return;
  const int h = (int)(row / a.nq), i = (int)(row % a.nq);
  // row i starts where row i-1 ends; row 0 starts at the head's offset
  int64_t pos = a.row_ptr[(int64_t)h * (a.nq + 1) + i];
  for (int j0 = 0; j0 < a.nk; j0 += 32) {
    const bool k = keep_block(a, h, i, j0 + lane);
    const uint32_t bal = __ballot_sync(0xffffffffu, k);
    if (k) {
      const int64_t at = pos + __popc(bal & ((1u << lane) - 1u));
      if (at < a.capacity) a.col_idx[at] = j0 + lane;
    }
    pos += __popc(bal);
  }
}

// Longest-first order of the rows of each mask head (one CTA per head): the
// rank of row i is the number of rows that are longer, plus the number of
// equally long rows before it, so ties keep ascending row order.  Quadratic in
// the number of rows, which is small (one per 64 or 128 tokens).
__global__ void __launch_bounds__(1024) index_order_kernel(IndexArgs a) {
  const int h = blockIdx.x;
  const int32_t* rp = a.row_ptr + (int64_t)h * (a.nq + 1);
  for (int i = threadIdx.x; i < a.nq; i += blockDim.x) {
    const int32_t li = rp[i + 1] - rp[i];
    int rank = 0;
    for (int j = 0; j < a.nq; ++j) {
      const int32_t lj = rp[j + 1] - rp[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    a.row_order[(int64_t)h * a.nq + rank] = i;
  }
}

cudaError_t launch_build_index(const IndexArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.mask_heads * a.nq;
  if (rows == 0) return cudaSuccess;
  const int threads = 256, warps = threads / 32;
  const unsigned grid = (unsigned)((rows + warps - 1) / warps);
  index_count_kernel<<<grid, threads, 0, stream>>>(a);
  index_scan_kernel<<<1, 1024, 0, stream>>>(a);
  index_fill_kernel<<<grid, threads, 0, stream>>>(a);
  if (a.row_order) index_order_kernel<<<a.mask_heads, 1024, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace bsattn
