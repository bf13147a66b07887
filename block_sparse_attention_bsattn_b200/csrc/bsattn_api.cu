// Host side of the C ABI declared in include/bsattn.h: argument validation,
// TMA tensor-map encoding (through the driver entry point, so the library
// needs no link-time libcuda), kernel attribute set-up and launches.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn.h"
#include "backward_internal.h"
#include "bsattn_internal.h"

namespace bsattn {

// ------------------------------------------------------------------ debug knobs
static unsigned long long g_wait_limit_ns = 2000000000ull;  // 2 s
static int g_inject_stall = 0;
static volatile int32_t* g_trace = nullptr;
static int g_trace_n = 0;

// ------------------------------------------------------------------ driver entry
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 tensor [Z][Y][X] (X contiguous) tiled in boxes of 64 x box_rows x 1
// with the 128-byte swizzle; out-of-range rows read as zero.
static bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t X, uint64_t Y,
                           uint64_t Z, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {X, Y, Z};
  cuuint64_t strides[2] = {X * 2, X * Y * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSATTN_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  return major == 10 ? BSATTN_OK : BSATTN_ERR_UNSUPPORTED;
}

static bool bad_lambda(float lambda) { return !(lambda >= 0.f && lambda <= 1.f); }

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace bsattn

using namespace bsattn;

extern "C" {

const char* bsattn_status_string(int status) {
  switch (status) {
    case BSATTN_OK: return "BSATTN_OK";
    case BSATTN_ERR_INVALID_ARG: return "BSATTN_ERR_INVALID_ARG";
    case BSATTN_ERR_UNSUPPORTED: return "BSATTN_ERR_UNSUPPORTED";
    case BSATTN_ERR_ALIGNMENT: return "BSATTN_ERR_ALIGNMENT";
    case BSATTN_ERR_CAPACITY: return "BSATTN_ERR_CAPACITY";
    case BSATTN_ERR_CUDA: return "BSATTN_ERR_CUDA";
    case BSATTN_ERR_DEVICE_TIMEOUT: return "BSATTN_ERR_DEVICE_TIMEOUT";
    default: return "BSATTN_UNKNOWN_STATUS";
  }
}

int bsattn_version(void) { return 100; }

int bsattn_debug_set(long long wait_limit_ns, int inject_stall) {
  if (wait_limit_ns <= 0) return BSATTN_ERR_INVALID_ARG;
  g_wait_limit_ns = (unsigned long long)wait_limit_ns;
  g_inject_stall = inject_stall ? 1 : 0;
  return BSATTN_OK;
}

int bsattn_debug_exp2(const float* d_x, float* d_y, int64_t n, cudaStream_t stream) {
  if (n < 0 || n > ((int64_t)1 << 32) || (n > 0 && (!d_x || !d_y))) return BSATTN_ERR_INVALID_ARG;
  return launch_exp2_check(d_x, d_y, n, stream) == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

int bsattn_debug_trace(int n, int32_t** host_view) {
  if (n < 0 || (n > 0 && !host_view)) return BSATTN_ERR_INVALID_ARG;
#ifndef BSATTN_TRACE
  // the shipped library has no trace markers compiled in and allocates nothing
  if (host_view) *host_view = nullptr;
  return n == 0 ? BSATTN_OK : BSATTN_ERR_UNSUPPORTED;
#else
  static int32_t* host_buf = nullptr;
  g_trace = nullptr;
  g_trace_n = 0;
  if (host_buf) {
    cudaFreeHost(host_buf);
    host_buf = nullptr;
  }
  if (n == 0) {
    if (host_view) *host_view = nullptr;
    return BSATTN_OK;
  }
  if (cudaHostAlloc(reinterpret_cast<void**>(&host_buf), sizeof(int32_t) * (size_t)n,
                    cudaHostAllocMapped) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  std::memset(host_buf, 0, sizeof(int32_t) * (size_t)n);
  void* dev = nullptr;
  if (cudaHostGetDevicePointer(&dev, host_buf, 0) != cudaSuccess) {
    cudaFreeHost(host_buf);
    host_buf = nullptr;
    return BSATTN_ERR_CUDA;
  }
  g_trace = static_cast<volatile int32_t*>(dev);
  g_trace_n = n;
  *host_view = host_buf;
  return BSATTN_OK;
#endif
}

int bsattn_build_index(const uint8_t* d_mask, int mask_heads, int nq_blocks, int nk_blocks,
                       int q_block, int k_block, int causal, int32_t* d_row_ptr,
                       int32_t* d_col_idx, int64_t col_capacity, int32_t* d_nnz,
                       int32_t* d_row_order, int32_t* d_status, cudaStream_t stream) {
  if (!d_mask || !d_row_ptr || !d_nnz || (!d_col_idx && col_capacity > 0))
    return BSATTN_ERR_INVALID_ARG;
  if (mask_heads < 1 || nq_blocks < 1 || nk_blocks < 1 || q_block < 1 || k_block < 1 ||
      col_capacity < 0)
    return BSATTN_ERR_INVALID_ARG;
  if ((int64_t)mask_heads * nq_blocks * nk_blocks > (int64_t)INT32_MAX)
    return BSATTN_ERR_UNSUPPORTED;
  if (int rc = check_device()) return rc;
  IndexArgs a{d_mask, mask_heads, nq_blocks, nk_blocks, q_block, k_block, causal ? 1 : 0,
              d_row_ptr, d_col_idx, col_capacity, d_nnz, d_row_order, d_status};
  return launch_build_index(a, stream) == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

int bsattn_fwd_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int N, int d, int block, float scale, int causal,
                       float lambda, const int32_t* row_ptr, const int32_t* col_idx,
                       const int32_t* row_order, int mask_heads, uint8_t* tile_status,
                       int32_t* d_status, cudaStream_t stream) {
  return bsattn_fwd_prefill_ex(q, k, v, o, lse, B, Hq, Hkv, N, d, block, scale, causal, lambda,
                               row_ptr, col_idx, row_order, mask_heads, tile_status, nullptr,
                               0u, d_status, stream);
}

int bsattn_fwd_prefill_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int N, int d, int block, float scale,
                          int causal, float lambda, const int32_t* row_ptr,
                          const int32_t* col_idx, const int32_t* row_order, int mask_heads,
                          uint8_t* tile_status, const int32_t* d_seq_lens, unsigned flags,
                          int32_t* d_status, cudaStream_t stream) {
  if (!q || !k || !v || !o) return BSATTN_ERR_INVALID_ARG;
  if (flags & ~(BSATTN_PREFILL_REVERSE | BSATTN_PREFILL_SKIP_V)) return BSATTN_ERR_INVALID_ARG;
  if (row_order && !row_ptr) return BSATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return BSATTN_ERR_INVALID_ARG;
  if (bad_lambda(lambda) || !std::isfinite(scale) || !(scale > 0.f)) return BSATTN_ERR_INVALID_ARG;
  if (row_ptr && (!col_idx || (mask_heads != 1 && mask_heads != Hq))) return BSATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSATTN_ERR_UNSUPPORTED;
  if (block != 64 && block != 128) return BSATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return BSATTN_ERR_ALIGNMENT;
  const int64_t nq = (N + block - 1) / block;
  const int64_t items = (int64_t)B * Hq * nq;
  if (items > INT32_MAX || (int64_t)B * Hq > INT32_MAX / 2) return BSATTN_ERR_UNSUPPORTED;
  if (int rc = check_device()) return rc;

  CUtensorMap tq, tk, tv;
  if (!encode_bf16_3d(&tq, q, d, N, (uint64_t)B * Hq, block) ||
      !encode_bf16_3d(&tk, k, d, N, (uint64_t)B * Hkv, block) ||
      !encode_bf16_3d(&tv, v, d, N, (uint64_t)B * Hkv, block))
    return BSATTN_ERR_CUDA;

  if (tile_status &&
      cudaMemsetAsync(tile_status, 0, (size_t)items * (size_t)nq, stream) != cudaSuccess)
    return BSATTN_ERR_CUDA;

  PrefillParams p{};
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.row_order = row_order;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.tile_status = tile_status;
  p.status = d_status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.nq = (int)nq;
  p.nk = (int)nq;
  p.mask_heads = mask_heads;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.use_skip = lambda > 0.f ? 1 : 0;
  p.thr_log2 = lambda > 0.f ? (float)std::log2((double)lambda) : -INFINITY;
  p.reverse = (flags & BSATTN_PREFILL_REVERSE) ? 1 : 0;
  p.skip_v = (flags & BSATTN_PREFILL_SKIP_V) ? 1 : 0;
  p.seq_lens = d_seq_lens;
  p.debug_stall = g_inject_stall;
  p.wait_limit_ns = g_wait_limit_ns;
  p.trace = g_trace;
  p.trace_n = g_trace_n;

  cudaError_t e;
  // Two query tiles share a CTA and its K/V stream when they walk the same
  // visit list: two query heads of one KV head (group size even), or, without
  // a block mask, two consecutive query tiles of one head.
  const bool pair_heads = block == 128 && (Hq / Hkv) % 2 == 0 && (!row_ptr || mask_heads == 1);
  const bool pair_tiles = block == 128 && !pair_heads && !row_ptr;
  if (pair_heads || pair_tiles) {
    p.pair_tiles = pair_tiles ? 1 : 0;
    const int64_t pitems = pair_heads ? items / 2 : (int64_t)B * Hq * ((nq + 1) / 2);
    e = d == 128 ? launch_prefill_pair<128>(tq, tk, tv, p, (int)pitems, stream)
                 : launch_prefill_pair<64>(tq, tk, tv, p, (int)pitems, stream);
    return e == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
  }
  // one query tile per CTA: the longest rows of every head first (about one
  // wave of them), then head by head
  {
    const int sms = sm_count();
    if (sms <= 0) return BSATTN_ERR_CUDA;
    const int64_t bh = (int64_t)B * Hq;
    p.lead_ranks = (int)std::min<int64_t>(nq, (sms + bh - 1) / bh);
  }
  if (d == 128 && block == 128) e = launch_prefill<128, 128>(tq, tk, tv, p, (int)items, stream);
  else if (d == 64 && block == 128) e = launch_prefill<64, 128>(tq, tk, tv, p, (int)items, stream);
  else if (d == 128 && block == 64) e = launch_prefill<128, 64>(tq, tk, tv, p, (int)items, stream);
  else e = launch_prefill<64, 64>(tq, tk, tv, p, (int)items, stream);
  return e == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

size_t bsattn_decode_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B < 1 || Hq < 1 || d < 1 || num_splits < 1) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  return rows * (size_t)d * 4 + rows * 4 * 2;
}

int bsattn_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int L, int d, int block, float scale, int causal,
                      float lambda, int num_splits, void* workspace, size_t workspace_bytes,
                      uint8_t* tile_status, int32_t* d_status, cudaStream_t stream) {
  return bsattn_fwd_decode_ex(q, k, v, o, lse, B, Hq, Hkv, L, d, block, scale, causal, lambda,
                              num_splits, workspace, workspace_bytes, tile_status, nullptr, 0u,
                              d_status, stream);
}

int bsattn_fwd_decode_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int Hq, int Hkv, int L, int d, int block, float scale, int causal,
                         float lambda, int num_splits, void* workspace, size_t workspace_bytes,
                         uint8_t* tile_status, const int32_t* d_seq_lens, unsigned flags,
                         int32_t* d_status, cudaStream_t stream) {
  (void)causal;
  if (!q || !k || !v || !o || !workspace) return BSATTN_ERR_INVALID_ARG;
  if (flags & ~BSATTN_DECODE_SINK_SEED) return BSATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || Hq % Hkv != 0 || num_splits < 1)
    return BSATTN_ERR_INVALID_ARG;
  if (bad_lambda(lambda) || !std::isfinite(scale) || !(scale > 0.f)) return BSATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSATTN_ERR_UNSUPPORTED;
  if (block != 64 && block != 128) return BSATTN_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  // the tensor-core kernel takes any group of up to 16 query heads
  if (G > 16) return BSATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(workspace))
    return BSATTN_ERR_ALIGNMENT;
  if (workspace_bytes < bsattn_decode_workspace_size(B, Hq, d, num_splits))
    return BSATTN_ERR_CAPACITY;
  const int T = (L + block - 1) / block;
  const int64_t grid = (int64_t)B * Hkv * num_splits;
  if (grid > INT32_MAX || (int64_t)B * Hq > INT32_MAX) return BSATTN_ERR_UNSUPPORTED;
  if (int rc = check_device()) return rc;

  CUtensorMap tk, tv;
  if (!encode_bf16_3d(&tk, k, d, L, (uint64_t)B * Hkv, block) ||
      !encode_bf16_3d(&tv, v, d, L, (uint64_t)B * Hkv, block))
    return BSATTN_ERR_CUDA;
  if (tile_status &&
      cudaMemsetAsync(tile_status, 0, (size_t)B * Hkv * (size_t)T, stream) != cudaSuccess)
    return BSATTN_ERR_CUDA;

  const size_t rows = (size_t)B * Hq * num_splits;
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.ws_o = static_cast<float*>(workspace);
  p.ws_m = p.ws_o + rows * d;
  p.ws_l = p.ws_m + rows;
  p.tile_status = tile_status;
  p.status = d_status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.L = L;
  p.T = T;
  p.splits = num_splits;
  p.chunk = (T + num_splits - 1) / num_splits;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.use_skip = lambda > 0.f ? 1 : 0;
  p.thr_log2 = lambda > 0.f ? (float)std::log2((double)lambda) : -INFINITY;
  p.sink_seed = (flags & BSATTN_DECODE_SINK_SEED) ? 1 : 0;
  p.seq_lens = d_seq_lens;
  p.wait_limit_ns = g_wait_limit_ns;
  p.trace = g_trace;
  p.trace_n = g_trace_n;

  CUtensorMap tq;
  if (!encode_bf16_3d(&tq, q, d, Hq, (uint64_t)B, 16)) return BSATTN_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return BSATTN_ERR_CUDA;
  const int tc_grid = (int)(grid < sms ? grid : sms);
  cudaError_t e = d == 128 ? launch_decode_tc<128>(tq, tk, tv, p, G, block, tc_grid, stream)
                           : launch_decode_tc<64>(tq, tk, tv, p, G, block, tc_grid, stream);
  if (e != cudaSuccess) return BSATTN_ERR_CUDA;
  CombineParams c{p.ws_o, p.ws_m, p.ws_l, static_cast<__nv_bfloat16*>(o), lse, num_splits, d};
  e = launch_decode_combine(c, B * Hq, d, stream);
  return e == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

size_t bsattn_bwd_prefill_workspace_size(int B, int Hq, int N, int block) {
  if (B < 1 || Hq < 1 || N < 1 || block < 1) return 0;
  const size_t rows = (size_t)B * Hq * (size_t)((N + block - 1) / block) * 128;
  return 2 * rows * sizeof(float);
}

int bsattn_bwd_prefill(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, const uint8_t* tile_status, void* dq,
                       void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int block,
                       float scale, int causal, const int32_t* d_seq_lens, void* workspace,
                       size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !tile_status || !dq || !dk || !dv || !workspace)
    return BSATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return BSATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return BSATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BSATTN_ERR_UNSUPPORTED;
  if (block != 128) return BSATTN_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, dout, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return BSATTN_ERR_ALIGNMENT;
  if (workspace_bytes < bsattn_bwd_prefill_workspace_size(B, Hq, N, block))
    return BSATTN_ERR_CAPACITY;
  const int64_t nq = (N + block - 1) / block;
  if ((int64_t)B * Hq * nq > INT32_MAX || (int64_t)B * Hq * nq * 128 * 32 / 256 > INT32_MAX)
    return BSATTN_ERR_UNSUPPORTED;
  if (int rc = check_device()) return rc;

  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bf16_3d(&tq, q, d, N, (uint64_t)B * Hq, 128) ||
      !encode_bf16_3d(&tk, k, d, N, (uint64_t)B * Hkv, 128) ||
      !encode_bf16_3d(&tv, v, d, N, (uint64_t)B * Hkv, 128) ||
      !encode_bf16_3d(&tdo, dout, d, N, (uint64_t)B * Hq, 128))
    return BSATTN_ERR_CUDA;
  const size_t rows = (size_t)B * Hq * (size_t)nq * 128;
  BackwardParams p{};
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.lse = lse;
  p.tile_status = tile_status;
  p.seq_lens = d_seq_lens;
  p.ws_lse2 = static_cast<float*>(workspace);
  p.ws_d = p.ws_lse2 + rows;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.status = d_status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.nq = (int)nq;
  p.nk = (int)nq;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.wait_limit_ns = g_wait_limit_ns;
  {
    const int sms = sm_count();
    if (sms <= 0) return BSATTN_ERR_CUDA;
    const int64_t bk = (int64_t)B * Hkv, bh = (int64_t)B * Hq;
    p.lead_k = causal ? (int)std::min<int64_t>(nq, (sms + bk - 1) / bk) : 0;
    p.lead_q = causal ? (int)std::min<int64_t>(nq, (sms + bh - 1) / bh) : 0;
  }
  p.debug_stall = g_inject_stall;
  const cudaError_t e = d == 128 ? launch_backward<128>(tq, tk, tv, tdo, p, stream)
                                 : launch_backward<64>(tq, tk, tv, tdo, p, stream);
  return e == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // extern "C"
