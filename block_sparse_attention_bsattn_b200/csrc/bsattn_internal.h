// Parameter blocks and launchers shared between the C-ABI layer
// (bsattn_api.cu) and the kernel translation units.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace bsattn {

struct IndexArgs {
  const uint8_t* mask;
  int mask_heads, nq, nk, q_block, k_block, causal;
  int32_t* row_ptr;
  int32_t* col_idx;
  int64_t capacity;
  int32_t* nnz;
  int32_t* row_order;  // optional: rows of each mask head, longest first
  int32_t* status;
};

struct PrefillParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* row_order;  // optional: work order of query tiles within a head
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  float* lse;
  uint8_t* tile_status;
  int32_t* status;
  int B, Hq, Hkv, N, nq, nk, mask_heads, causal;
  float scale_log2;  // softmax scale * log2(e): scores are kept in base-2 units
  float thr_log2;    // log2(lambda)
  int use_skip;      // lambda > 0
  int debug_stall;   // test hook: the query tile is withheld from the tensor core
  int pair_tiles;    // two-slot kernel: consecutive query tiles of one head
  int lead_ranks;    // one-tile kernel: rows of rank < lead_ranks of every head go first
  int reverse;       // visit each row's key tiles in descending order
  int skip_v;        // load V only for tiles some query tile keeps
  const int32_t* seq_lens;   // [B] valid tokens per sequence (key padding) or null
  unsigned long long wait_limit_ns;
  volatile int32_t* trace;  // debug: progress markers (host-visible memory) or null
  int trace_n;
};

struct DecodeParams {
  const __nv_bfloat16* q;
  float* ws_o;      // [B][Hq][S][D] unnormalised split outputs
  float* ws_m;      // [B][Hq][S]    split exponent shift (base-2 units)
  float* ws_l;      // [B][Hq][S]    split row sums
  uint8_t* tile_status;
  int32_t* status;
  int B, Hq, Hkv, L, T, splits, chunk;
  float scale_log2;
  float thr_log2;
  int use_skip;
  int sink_seed;    // splits after the first start from key tile 0's row max
  const int32_t* seq_lens;   // [B] cache lengths (splits cut each one's own tiles) or null
  unsigned long long wait_limit_ns;
  volatile int32_t* trace;
  int trace_n;
};

struct CombineParams {
  const float* ws_o;
  const float* ws_m;
  const float* ws_l;
  __nv_bfloat16* o;
  float* lse;
  int splits, D;
};

cudaError_t launch_build_index(const IndexArgs& a, cudaStream_t stream);
// y[i] = 2^x[i] through the prefill kernels' FMA-pipe exponential (test hook)
cudaError_t launch_exp2_check(const float* x, float* y, int64_t n, cudaStream_t stream);

template <int D, int BLK>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const PrefillParams& p, int grid, cudaStream_t stream);

template <int D>
cudaError_t launch_prefill_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const PrefillParams& p, int grid,
                                cudaStream_t stream);

template <int D>
cudaError_t launch_decode_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const DecodeParams& p, int G, int block, int grid,
                             cudaStream_t stream);

cudaError_t launch_decode_combine(const CombineParams& p, int grid, int threads,
                                  cudaStream_t stream);

}  // namespace bsattn
