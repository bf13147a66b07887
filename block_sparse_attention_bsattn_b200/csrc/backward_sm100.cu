// Block-sparse attention backward for sm_100a, for sparsity-aware training.
//
// What it computes ("BLASST: Dynamic Blocked Attention Sparsity via Softmax
// Thresholding", section 3.3: fine-tuning runs the forward with the skip, and
// the blocks it skipped receive no gradient because they were never
// computed): with the forward's executed tiles held fixed, for each query row
// r and each unmasked key c of an executed tile
//   P = exp(scale q.k - LSE),  dP = dO . v,  D = rowsum(dO * O),
//   dS = P (dP - D),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
// The forward's tile status (2 = executed) names the tiles; its LSE gives P
// without a second softmax pass.
//
// Three kernels:
//   bwd_rows_kernel  per query row: D and LSE * log2(e) (+inf for a row with no
//                    weight), padded to whole query tiles (CUDA cores).
//   bwd_dkdv_kernel  one CTA per (sequence, KV head, key tile): keys on the TMEM
//                    lanes.  For every executed (query head of the group, query
//                    tile) pair: S^T = K Q^T and dP^T = V dO^T (tcgen05, smem
//                    operands), then P^T and dS^T in bf16 over them, then
//                    dV += P^T dO and dK += dS^T Q (A from TMEM) accumulated in
//                    TMEM across all pairs; one bf16 write of dK and dV.
//   bwd_dq_kernel    one CTA per (sequence, query head, query tile): for every
//                    executed key tile S = Q K^T, dP = dO V^T, dS in bf16 over
//                    S, dQ += dS K accumulated in TMEM; one bf16 write of dQ.
// No atomics: each output tile has one writer.  Warps: 0 TMA producer (it also
// finds the executed tiles, 32 status bytes per ballot, and passes each one to
// the other roles through its stage), 1 MMA issuer, 4..11 the element-wise
// work: two warps per TMEM lane quarter, each owning half of the tile's
// columns and writing its bf16 results inside them.  Every wait is bounded
// in time.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "backward_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

// ------------------------------------------------------------------ rows
__global__ void __launch_bounds__(256) bwd_rows_kernel(const BackwardParams p) {
  const int64_t rows = (int64_t)p.B * p.Hq * p.nq * 128;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= rows) return;
  const int64_t per = (int64_t)p.nq * 128;
  const int64_t bh = w / per;
  const int t = (int)(w - bh * per);
  const int b = (int)(bh / p.Hq);
  const int len = p.seq_lens ? min(max(p.seq_lens[b], 0), p.N) : p.N;
  float acc = 0.f;
  if (t < p.N) {
    const __nv_bfloat16* orow = p.o + (bh * p.N + t) * p.d;
    const __nv_bfloat16* drow = p.dout + (bh * p.N + t) * p.d;
    for (int x = lane * 2; x < p.d; x += 64) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(orow + x));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(drow + x));
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    float l2 = INFINITY;   // no weight: P = exp2(s - inf) = 0
    if (t < len) {
      const float l = p.lse[bh * p.N + t];
      if (isfinite(l)) l2 = l * 1.4426950408889634f;
    }
    p.ws_lse2[w] = l2;
    p.ws_d[w] = acc;
  }
}

// ------------------------------------------------------------------ shared layout
template <int D>
struct BwdCfg {
  static constexpr int BLK = 128;
  static constexpr int HALVES = D / 64;
  static constexpr int T_HALF = BLK * 128;          // one 64-column box of a 128-row tile
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int VEC = 512;                   // 128 fp32
  // dK/dV kernel: K, V resident; two stages of (Q, dO, LSE2, D)
  static constexpr int KV_K = 0;
  static constexpr int KV_V = T_BYTES;
  static constexpr int KV_STG = 2 * T_BYTES;
  static constexpr int KV_STG_BYTES = 2 * T_BYTES + 2 * VEC;   // a multiple of 1024
  static constexpr int KV_BAR = KV_STG + 2 * KV_STG_BYTES;
  // at least 116 KB: one CTA per SM, since each holds all 512 TMEM columns
  static constexpr int KV_SMEM = KV_BAR + 512 + 1024 > 118784 ? KV_BAR + 512 + 1024 : 118784;
  // dQ kernel: Q, dO resident; two stages of (K, V)
  static constexpr int Q_Q = 0;
  static constexpr int Q_DO = T_BYTES;
  static constexpr int Q_STG = 2 * T_BYTES;
  static constexpr int Q_STG_BYTES = 2 * T_BYTES;
  static constexpr int Q_BAR = Q_STG + 2 * Q_STG_BYTES;
  static constexpr int Q_SMEM = Q_BAR + 512 + 1024 > 118784 ? Q_BAR + 512 + 1024 : 118784;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns
  static constexpr uint32_t ACC0 = 0;               // dK (dK/dV kernel) or dQ
  static constexpr uint32_t ACC1 = D;               // dV (dK/dV kernel)
  static constexpr uint32_t S_COL = 256;            // S or S^T, then P^T / dS in bf16
  static constexpr uint32_t DP_COL = 384;           // dP or dP^T, then dS^T in bf16
  static constexpr int THREADS = 384;              // 4 role warps + 8 element-wise warps
};

struct BwdBarriers {
  uint64_t res_full;           // resident tiles landed
  uint64_t st_full[2], st_empty[2];
  uint64_t s_full;             // S and dP of the current pair are in TMEM
  uint64_t p_ready;            // bf16 operands written back (4 warps)
  uint64_t acc_done;           // every MMA finished
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int meta[2][2];              // per stage: (head, query tile) / (key tile, -) or -1 = end
};

// TMEM column (relative to S or dP) of the bf16 pairs of K-step kk (16 of
// the 128 inner indices) of the element-wise results: the warps that own
// inner indices [64 h, 64 h + 64) write their 32 columns of pairs at 64 h,
// inside the 64 fp32 columns they alone read.
__device__ __forceinline__ uint32_t bf16_col(int kk) {
  return (uint32_t)((kk / 4) * 64 + (kk % 4) * 8);
}

// Producer's end-of-stream marker in stage t % 2 (no bytes: a plain arrive).
__device__ __forceinline__ bool bwd_end_marker(BwdBarriers* bars, int t, volatile int* abort,
                                               uint64_t lim) {
  const int st = t & 1;
  if (!mbar_wait(&bars->st_empty[st], ((t >> 1) & 1) ^ 1, abort, lim)) return false;
  bars->meta[st][0] = -1;
  mbar_arrive(&bars->st_full[st]);
  return true;
}

// ------------------------------------------------------------------ dK, dV
template <int D>
__global__ void __launch_bounds__(384, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BackwardParams p) {
  using C = BwdCfg<D>;
  static_assert(sizeof(BwdBarriers) <= 512, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::KV_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // work item: key tile j of (b, kvh); ascending j first (the longest causal columns)
  const int bkv = (int)(blockIdx.x / (unsigned)p.nk);
  const int j = (int)(blockIdx.x - (unsigned)bkv * p.nk);
  const int b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int len = p.seq_lens ? min(max(p.seq_lens[b], 0), p.N) : p.N;

  if (threadIdx.x == 0) {
    mbar_init(&bars->res_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_ready, 8);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t lim = p.wait_limit_ns;

  if (warp == 0) {
    // ======================================================== producer
    int t = 0;          // pairs issued
    bool ok = true;
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmDO);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::T_BYTES);
      for (int hf = 0; hf < C::HALVES; ++hf) {
        tma_load_3d(smem + C::KV_K + hf * C::T_HALF, &tmK, &bars->res_full, hf * 64, j * 128,
                    b * p.Hkv + kvh);
        tma_load_3d(smem + C::KV_V + hf * C::T_HALF, &tmV, &bars->res_full, hf * 64, j * 128,
                    b * p.Hkv + kvh);
      }
    }
    for (int hl = 0; hl < g && ok; ++hl) {
      const int h = kvh * g + hl;
      const uint8_t* col = p.tile_status + ((int64_t)(b * p.Hq + h) * p.nq) * p.nk + j;
      for (int i0 = p.causal ? j : 0; i0 < p.nq && ok; i0 += 32) {
        const int i = i0 + lane;
        const bool ex = i < p.nq && col[(int64_t)i * p.nk] == 2;
        unsigned m = __ballot_sync(0xffffffffu, ex);
        while (m) {
          const int ii = i0 + __ffs(m) - 1;
          m &= m - 1;
          const int st = t & 1;
          bool w_ok = true;
          if (lane == 0) {
            w_ok = mbar_wait(&bars->st_empty[st], ((t >> 1) & 1) ^ 1, abort, lim);
            if (w_ok) {
              bars->meta[st][0] = h;
              bars->meta[st][1] = ii;
              uint8_t* sb = smem + C::KV_STG + st * C::KV_STG_BYTES;
              mbar_arrive_expect_tx(&bars->st_full[st], 2 * C::T_BYTES + 2 * C::VEC);
              for (int hf = 0; hf < C::HALVES; ++hf) {
                tma_load_3d(sb + hf * C::T_HALF, &tmQ, &bars->st_full[st], hf * 64, ii * 128,
                            b * p.Hq + h);
                tma_load_3d(sb + C::T_BYTES + hf * C::T_HALF, &tmDO, &bars->st_full[st], hf * 64,
                            ii * 128, b * p.Hq + h);
              }
              const int64_t row0 = ((int64_t)(b * p.Hq + h) * p.nq + ii) * 128;
              bulk_load(sb + 2 * C::T_BYTES, p.ws_lse2 + row0, C::VEC, &bars->st_full[st]);
              bulk_load(sb + 2 * C::T_BYTES + C::VEC, p.ws_d + row0, C::VEC, &bars->st_full[st]);
            }
          }
          if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) {
            ok = false;
            break;
          }
          ++t;
        }
      }
    }
    if (lane == 0) {
      if (ok) ok = bwd_end_marker(bars, t, abort, lim);
      if (*abort) {
        // let every copy this thread started land before the CTA can exit
        mbar_wait_drain(&bars->res_full, 0, lim);
        for (int x = (t > 2 ? t - 2 : 0); x < t; ++x)
          mbar_wait_drain(&bars->st_full[x & 1], (x >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_addr = smem_u32(smem + C::KV_K);
      const uint32_t v_addr = smem_u32(smem + C::KV_V);
      bool ok = mbar_wait(&bars->res_full, 0, abort, lim);
      tc_fence_after();
      for (int t = 0; ok; ++t) {
        const int st = t & 1;
        if (!mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim)) break;
        tc_fence_after();
        if (*reinterpret_cast<volatile int*>(&bars->meta[st][0]) < 0) break;
        const uint32_t qa = smem_u32(smem + C::KV_STG + st * C::KV_STG_BYTES);
        const uint32_t da = qa + C::T_BYTES;
        // S^T = K Q^T and dP^T = V dO^T: keys on the rows, queries on the columns
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(tmem + C::S_COL, smem_desc(k_addr + off, 16, 1024, 2),
                 smem_desc(qa + off, 16, 1024, 2), IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(tmem + C::DP_COL, smem_desc(v_addr + off, 16, 1024, 2),
                 smem_desc(da + off, 16, 1024, 2), IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full);
        if (!mbar_wait(&bars->p_ready, t & 1, abort, lim)) break;
        tc_fence_after();
        // dV += P^T dO and dK += dS^T Q (scale folded into dS): A from TMEM,
        // B = the query-side tile read MN-major
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::ACC1, tmem + C::S_COL + bf16_col(kk),
                 smem_desc(da + kk * (16 * 128), C::T_HALF, 1024, 2), IDESC_O,
                 (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::ACC0, tmem + C::DP_COL + bf16_col(kk),
                 smem_desc(qa + kk * (16 * 128), C::T_HALF, 1024, 2), IDESC_O,
                 (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->st_empty[st]);
      }
      mma_commit(&bars->acc_done);
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else if (warp >= 4) {
    // ======================================================== element-wise warps
    // Two warps per TMEM lane quarter: warp half hc owns the query columns
    // [64 hc, 64 hc + 64) of its 32 key rows and writes their bf16 pairs at
    // column 64 hc, inside the columns only it reads.
    const int quarter = warp % 4;
    const int hc = (warp - 4) / 4;
    const int c = quarter * 32 + lane;           // key row of the tile
    const int key = j * 128 + c;
    const bool key_ok = key < len;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    int t = 0;
    bool ok = true;
    for (;; ++t) {
      const int st = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim))) {
        ok = false;
        break;
      }
      const int ii = *reinterpret_cast<volatile int*>(&bars->meta[st][1]);
      if (*reinterpret_cast<volatile int*>(&bars->meta[st][0]) < 0) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* lse2 =
          reinterpret_cast<const float*>(smem + C::KV_STG + st * C::KV_STG_BYTES + 2 * C::T_BYTES);
      const float* dvec = lse2 + 128;
      const int q0 = ii * 128;
      // a query tile after the key tile sees every key (causal), so only the
      // diagonal pair needs the per-element mask
      const bool diag = p.causal && ii == j;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * hc + 32 * cc;        // 32 query columns
        uint32_t s[32], dp[32];
        tmem_ld32(lane_addr + C::S_COL + c0, s);
        tmem_ld32(lane_addr + C::DP_COL + c0, dp);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int r = 0; r < 32; r += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c0 + r);
          const float4 d4 = *reinterpret_cast<const float4*>(dvec + c0 + r);
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const float2 lu = u == 0 ? make_float2(-l4.x, -l4.y) : make_float2(-l4.z, -l4.w);
            const float2 du = u == 0 ? make_float2(-d4.x, -d4.y) : make_float2(-d4.z, -d4.w);
            const float2 x = ffma2(make_float2(__uint_as_float(s[r + u]),
                                               __uint_as_float(s[r + u + 1])), sl2, lu);
            float2 pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            if (!key_ok) pv = make_float2(0.f, 0.f);
            if (diag) {
              if (key > q0 + c0 + r + u) pv.x = 0.f;
              if (key > q0 + c0 + r + u + 1) pv.y = 0.f;
            }
            const float2 g = fadd2(make_float2(__uint_as_float(dp[r + u]),
                                               __uint_as_float(dp[r + u + 1])), du);
            const float2 ds = ffma2(make_float2(pv.x * p.scale, pv.y * p.scale), g,
                                    make_float2(0.f, 0.f));
            pk[(r + u) / 2] = pack_bf16x2(pv.x, pv.y);
            dk[(r + u) / 2] = pack_bf16x2(ds.x, ds.y);
          }
        }
        tmem_st16(lane_addr + C::S_COL + 64 * hc + 16 * cc, pk);
        tmem_st16(lane_addr + C::DP_COL + 64 * hc + 16 * cc, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);
    }
    // ---- epilogue: the key tile's dK rows (warp half 0) and dV rows (half 1),
    // zero when no pair took part
    if (ok) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, abort, lim))) ok = false;
      tc_fence_after();
    }
    if (ok) {
      const bool in_buf = key < p.N;
      const int64_t row = ((int64_t)(b * p.Hkv + kvh) * p.N + key) * D;
      __nv_bfloat16* dst = (hc == 0 ? p.dk : p.dv) + row;
      const uint32_t col = hc == 0 ? C::ACC0 : C::ACC1;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        if (t > 0) {
          tmem_ld32(lane_addr + col + c0, r);
          tmem_wait_ld();
        }
        if (in_buf) {
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            w[x / 2] = t > 0 ? pack_bf16x2(__uint_as_float(r[x]), __uint_as_float(r[x + 1])) : 0u;
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort) report_status(p.status, kDevTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ dQ
template <int D>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BackwardParams p) {
  using C = BwdCfg<D>;
  static_assert(sizeof(BwdBarriers) <= 512, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::Q_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // work item: query tile i of (b, h); longest causal rows first
  const int bh = (int)(blockIdx.x / (unsigned)p.nq);
  const int r = (int)(blockIdx.x - (unsigned)bh * p.nq);
  const int i = p.causal ? p.nq - 1 - r : r;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int kvh = h / (p.Hq / p.Hkv);
  const int len = p.seq_lens ? min(max(p.seq_lens[b], 0), p.N) : p.N;

  if (threadIdx.x == 0) {
    mbar_init(&bars->res_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_ready, 8);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t lim = p.wait_limit_ns;

  if (warp == 0) {
    // ======================================================== producer
    int t = 0;
    bool ok = true;
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(&bars->res_full, 2 * C::T_BYTES);
      for (int hf = 0; hf < C::HALVES; ++hf) {
        tma_load_3d(smem + C::Q_Q + hf * C::T_HALF, &tmQ, &bars->res_full, hf * 64, i * 128,
                    b * p.Hq + h);
        tma_load_3d(smem + C::Q_DO + hf * C::T_HALF, &tmDO, &bars->res_full, hf * 64, i * 128,
                    b * p.Hq + h);
      }
    }
    const uint8_t* row = p.tile_status + ((int64_t)(b * p.Hq + h) * p.nq + i) * p.nk;
    const int jend = p.causal ? min(p.nk, i + 1) : p.nk;
    for (int j0 = 0; j0 < jend && ok; j0 += 32) {
      const int jj = j0 + lane;
      const bool ex = jj < jend && row[jj] == 2;
      unsigned m = __ballot_sync(0xffffffffu, ex);
      while (m) {
        const int j = j0 + __ffs(m) - 1;
        m &= m - 1;
        const int st = t & 1;
        bool w_ok = true;
        if (lane == 0) {
          w_ok = mbar_wait(&bars->st_empty[st], ((t >> 1) & 1) ^ 1, abort, lim);
          if (w_ok) {
            bars->meta[st][0] = j;
            uint8_t* sb = smem + C::Q_STG + st * C::Q_STG_BYTES;
            mbar_arrive_expect_tx(&bars->st_full[st], 2 * C::T_BYTES);
            for (int hf = 0; hf < C::HALVES; ++hf) {
              tma_load_3d(sb + hf * C::T_HALF, &tmK, &bars->st_full[st], hf * 64, j * 128,
                          b * p.Hkv + kvh);
              tma_load_3d(sb + C::T_BYTES + hf * C::T_HALF, &tmV, &bars->st_full[st], hf * 64,
                          j * 128, b * p.Hkv + kvh);
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        ++t;
      }
    }
    if (lane == 0) {
      if (ok) ok = bwd_end_marker(bars, t, abort, lim);
      if (*abort) {
        mbar_wait_drain(&bars->res_full, 0, lim);
        for (int x = (t > 2 ? t - 2 : 0); x < t; ++x)
          mbar_wait_drain(&bars->st_full[x & 1], (x >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + C::Q_Q);
      const uint32_t do_addr = smem_u32(smem + C::Q_DO);
      bool ok = mbar_wait(&bars->res_full, 0, abort, lim);
      tc_fence_after();
      for (int t = 0; ok; ++t) {
        const int st = t & 1;
        if (!mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim)) break;
        tc_fence_after();
        if (*reinterpret_cast<volatile int*>(&bars->meta[st][0]) < 0) break;
        const uint32_t ka = smem_u32(smem + C::Q_STG + st * C::Q_STG_BYTES);
        const uint32_t va = ka + C::T_BYTES;
        // S = Q K^T and dP = dO V^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(tmem + C::S_COL, smem_desc(q_addr + off, 16, 1024, 2),
                 smem_desc(ka + off, 16, 1024, 2), IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(tmem + C::DP_COL, smem_desc(do_addr + off, 16, 1024, 2),
                 smem_desc(va + off, 16, 1024, 2), IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full);
        if (!mbar_wait(&bars->p_ready, t & 1, abort, lim)) break;
        tc_fence_after();
        // dQ += dS K (scale folded into dS): A from TMEM, B = the K tile read MN-major
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::ACC0, tmem + C::S_COL + bf16_col(kk),
                 smem_desc(ka + kk * (16 * 128), C::T_HALF, 1024, 2), IDESC_O,
                 (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->st_empty[st]);
      }
      mma_commit(&bars->acc_done);
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else if (warp >= 4) {
    // ======================================================== element-wise warps
    // Two warps per TMEM lane quarter: warp half hc owns the key columns
    // [64 hc, 64 hc + 64) of its 32 query rows and writes their bf16 pairs at
    // column 64 hc, inside the columns only it reads.
    const int quarter = warp % 4;
    const int hc = (warp - 4) / 4;
    const int rr = quarter * 32 + lane;          // query row of the tile
    const int qpos = i * 128 + rr;
    const int64_t wrow = ((int64_t)(b * p.Hq + h) * p.nq + i) * 128 + rr;
    const float lse2 = p.ws_lse2[wrow];          // +inf for rows without weight
    const float dval = p.ws_d[wrow];
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 nl2 = make_float2(-lse2, -lse2);
    const float2 nd2 = make_float2(-dval, -dval);
    int t = 0;
    bool ok = true;
    for (;; ++t) {
      const int st = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim))) {
        ok = false;
        break;
      }
      const int j = *reinterpret_cast<volatile int*>(&bars->meta[st][0]);
      if (j < 0) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * 128;
      // a key tile before the query tile and inside the sequence needs no
      // per-element mask
      const bool masked = (p.causal && j == i) || k0 + 128 > len;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * hc + 32 * cc;        // 32 key columns
        uint32_t s[32], dp[32];
        tmem_ld32(lane_addr + C::S_COL + c0, s);
        tmem_ld32(lane_addr + C::DP_COL + c0, dp);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 y = ffma2(make_float2(__uint_as_float(s[x]), __uint_as_float(s[x + 1])),
                                 sl2, nl2);
          float2 pv = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          if (masked) {
            const int key = k0 + c0 + x;
            if (key >= len || (p.causal && key > qpos)) pv.x = 0.f;
            if (key + 1 >= len || (p.causal && key + 1 > qpos)) pv.y = 0.f;
          }
          const float2 g = fadd2(make_float2(__uint_as_float(dp[x]), __uint_as_float(dp[x + 1])),
                                 nd2);
          const float2 ds = ffma2(make_float2(pv.x * p.scale, pv.y * p.scale), g,
                                  make_float2(0.f, 0.f));
          dk[x / 2] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st16(lane_addr + C::S_COL + 64 * hc + 16 * cc, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);
    }
    // ---- epilogue: this query tile's dQ rows, columns [hc D/2, hc D/2 + D/2)
    // per warp half (zero when no key tile took part)
    if (ok) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, abort, lim))) ok = false;
      tc_fence_after();
    }
    if (ok) {
      const bool in_buf = qpos < p.N;
      __nv_bfloat16* dst = p.dq + ((int64_t)(b * p.Hq + h) * p.N + qpos) * D;
#pragma unroll
      for (int c0 = hc * (D / 2); c0 < hc * (D / 2) + D / 2; c0 += 32) {
        uint32_t rg[32];
        if (t > 0) {
          tmem_ld32(lane_addr + C::ACC0 + c0, rg);
          tmem_wait_ld();
        }
        if (in_buf) {
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            w[x / 2] = t > 0 ? pack_bf16x2(__uint_as_float(rg[x]), __uint_as_float(rg[x + 1])) : 0u;
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort) report_status(p.status, kDevTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ launchers
template <int D>
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BackwardParams& p, cudaStream_t stream) {
  using C = BwdCfg<D>;
  static_assert(C::KV_SMEM <= 232448 && C::Q_SMEM <= 232448, "shared memory budget");
  const int64_t rows = (int64_t)p.B * p.Hq * p.nq * 128;
  bwd_rows_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::KV_SMEM);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<(unsigned)(p.B * p.Hkv * p.nk), C::THREADS, C::KV_SMEM, stream>>>(
      tq, tk, tv, tdo, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::Q_SMEM);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<(unsigned)(p.B * p.Hq * p.nq), C::THREADS, C::Q_SMEM, stream>>>(tq, tk, tv,
                                                                                     tdo, p);
  return cudaGetLastError();
}

template cudaError_t launch_backward<128>(const CUtensorMap&, const CUtensorMap&,
                                          const CUtensorMap&, const CUtensorMap&,
                                          const BackwardParams&, cudaStream_t);
template cudaError_t launch_backward<64>(const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&,
                                         const BackwardParams&, cudaStream_t);

}  // namespace bsattn
