// Parameter block and launcher of the backward kernels, shared between the
// C-ABI layer (bsattn_api.cu) and backward_sm100.cu.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace bsattn {

struct BackwardParams {
  const __nv_bfloat16* o;       // forward output [B][Hq][N][d]
  const __nv_bfloat16* dout;    // its gradient, same layout
  const float* lse;             // forward LSE [B][Hq][N] (natural log)
  const uint8_t* tile_status;   // forward tile status [B][Hq][nq][nk]; 2 = executed
  const int32_t* seq_lens;      // [B] valid tokens or null
  float* ws_lse2;               // [B][Hq][nq * 128]: LSE * log2(e), +inf without weight
  float* ws_d;                  // [B][Hq][nq * 128]: rowsum(dO * O)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int32_t* status;
  int B, Hq, Hkv, N, nq, nk, d, causal;
  // causal work order: the lead_k lowest key tiles of every KV head (dK/dV)
  // and the lead_q last query tiles of every head (dQ) -- the longest work
  // items, about one wave of them -- go first, all heads at once
  int lead_k, lead_q;
  int debug_stall;   // test hook: the resident tiles are never loaded
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D>
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BackwardParams& p, cudaStream_t stream);

}  // namespace bsattn
