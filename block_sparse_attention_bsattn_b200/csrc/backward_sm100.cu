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
// work: two warps per TMEM lane quarter, each owning half of a half-tile's
// columns and writing its bf16 results inside them.  Every wait is bounded
// in time.
//
// Each pair (dK/dV) or key tile (dQ) is taken as two halves of 64 columns
// (queries, resp. keys) with their S and dP in one of two TMEM buffers, so
// the element-wise work on one half runs while the tensor core computes the
// other half's products: the first products of half h + 1 are issued before
// the second products of half h, which wait for its bf16 operands.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "backward_internal.h"
#include "sm100_ptx.cuh"
#include "umma_desc.cuh"

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
  // half-tile buffer b at BUF + 128 b: S (or S^T) of 64 columns, then its
  // bf16 P^T / dS at the same place; dP (or dP^T) 64 columns further on, then
  // dS^T in bf16
  static constexpr uint32_t BUF = 256;
  static constexpr uint32_t DPOFF = 64;
  static constexpr int THREADS = 384;              // 4 role warps + 8 element-wise warps
};

struct BwdBarriers {
  uint64_t res_full;           // resident tiles landed
  uint64_t st_full[2], st_empty[2];
  uint64_t s_full[2];          // per half-tile buffer: S and dP are in TMEM
  uint64_t p_ready[2];         // per buffer: bf16 operands written back (8 warps)
  uint64_t acc_done;           // every MMA finished
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int meta[2][2];              // per stage: (head, query tile) / (key tile, -) or -1 = end
};

// TMEM column (relative to S or dP of a half-tile buffer) of the bf16 pairs
// of K-step kk (16 of the half's 64 inner indices) of the element-wise
// results: the warps that own inner indices [32 h, 32 h + 32) write their 16
// columns of pairs at 32 h, inside the 32 fp32 columns they alone read.
__device__ __forceinline__ uint32_t bf16_col(int kk) {
  return (uint32_t)((kk / 2) * 32 + (kk % 2) * 8);
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

  // work item: key tile j of (b, kvh).  Causal: the lead_k lowest key tiles
  // (the longest columns) of every KV head first, all KV heads at once, so
  // that no KV head's longest columns start late and run on alone; then each
  // KV head's remaining tiles in ascending order, KV head by KV head (its
  // query-side tiles stay in L2 while its CTAs run)
  int bkv, j;
  {
    const int BK = p.B * p.Hkv;
    const int lead = p.lead_k;
    const unsigned x = blockIdx.x;
    if (x < (unsigned)(lead * BK)) {
      j = (int)(x / (unsigned)BK);
      bkv = (int)(x - (unsigned)j * BK);
    } else {
      const unsigned y = x - (unsigned)(lead * BK);
      const int rest = p.nk - lead;
      bkv = (int)(y / (unsigned)rest);
      j = lead + (int)(y - (unsigned)bkv * rest);
    }
  }
  const int b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int len = p.seq_lens ? min(max(p.seq_lens[b], 0), p.N) : p.N;

  if (threadIdx.x == 0) {
    mbar_init(&bars->res_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 8);
    }
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
    if (lane == 0 && !p.debug_stall) {
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
        if (!p.debug_stall) mbar_wait_drain(&bars->res_full, 0, lim);
        for (int x = (t > 2 ? t - 2 : 0); x < t; ++x)
          mbar_wait_drain(&bars->st_full[x & 1], (x >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_lo = udesc_lo(smem_u32(smem + C::KV_K), 16);
      const uint32_t v_lo = udesc_lo(smem_u32(smem + C::KV_V), 16);
      const uint32_t stg_lo = udesc_lo(smem_u32(smem + C::KV_STG), 16);
      const uint32_t stg_lo_mn = udesc_lo(smem_u32(smem + C::KV_STG), C::T_HALF);
      // S^T and dP^T of half x (queries 64 (x & 1) .. + 64 of the pair in
      // stage st): keys on the rows, the half's queries on the columns
      auto first = [&](int x, int st) {
        const uint32_t buf = tmem + C::BUF + 128u * (uint32_t)(x & 1);
        const uint32_t qd = udesc_step(stg_lo, st * C::KV_STG_BYTES + (x & 1) * 8192);
        const uint32_t dd = udesc_step(qd, C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(buf, udesc128(k_lo, off), udesc128(qd, off), IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(buf + C::DPOFF, udesc128(v_lo, off), udesc128(dd, off), IDESC_S,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[x & 1]);
      };
      // dV += P^T dO and dK += dS^T Q over half x (scale folded into dS): A
      // from TMEM, B = the half's rows of the query-side tiles read MN-major;
      // the stage is released after its second half
      auto second = [&](int x, int st) -> bool {
        if (!mbar_wait(&bars->p_ready[x & 1], (x >> 1) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint32_t buf = tmem + C::BUF + 128u * (uint32_t)(x & 1);
        const uint32_t qd = udesc_step(stg_lo_mn, st * C::KV_STG_BYTES + (x & 1) * 8192);
        const uint32_t dd = udesc_step(qd, C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk)
          mma_ts(tmem + C::ACC1, buf + bf16_col(kk), udesc128(dd, kk * (16 * 128)), IDESC_O,
                 (x > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk)
          mma_ts(tmem + C::ACC0, buf + C::DPOFF + bf16_col(kk), udesc128(qd, kk * (16 * 128)),
                 IDESC_O, (x > 0 || kk > 0) ? 1u : 0u);
        if (x & 1) mma_commit(&bars->st_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->res_full, 0, abort, lim);
      tc_fence_after();
      int x = 0;   // halves whose first products are issued
      for (int t = 0; ok; ++t) {
        const int st = t & 1;
        if (!mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (*reinterpret_cast<volatile int*>(&bars->meta[st][0]) < 0) break;
        for (int hh = 0; hh < 2 && ok; ++hh, ++x) {
          first(x, st);
          if (x > 0) ok = second(x - 1, hh ? st : st ^ 1);
        }
      }
      if (ok && x > 0) second(x - 1, ((x - 1) >> 1) & 1);
      mma_commit(&bars->acc_done);
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else if (warp >= 4) {
    // ======================================================== element-wise warps
    // Two warps per TMEM lane quarter: warp half hc owns the query columns
    // [32 hc, 32 hc + 32) of each half-tile for its 32 key rows and writes
    // their bf16 pairs at column 32 hc, inside the columns only it reads.
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
      const float* lse2 =
          reinterpret_cast<const float*>(smem + C::KV_STG + st * C::KV_STG_BYTES + 2 * C::T_BYTES);
      const float* dvec = lse2 + 128;
      // a query tile after the key tile sees every key (causal), so only the
      // diagonal pair needs the per-element mask
      const bool diag = p.causal && ii == j;
      for (int hh = 0; hh < 2 && ok; ++hh) {
        const int x = 2 * t + hh;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x & 1], (x >> 1) & 1, abort, lim))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t buf = lane_addr + C::BUF + 128u * (uint32_t)(x & 1);
        const int c0 = 64 * hh + 32 * hc;          // 32 query columns of the tile
        const int q0 = ii * 128 + c0;
        uint32_t s[32], dp[32];
        tmem_ld32(buf + 32 * hc, s);
        tmem_ld32(buf + C::DPOFF + 32 * hc, dp);
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
            const float2 xv = ffma2(make_float2(__uint_as_float(s[r + u]),
                                                __uint_as_float(s[r + u + 1])), sl2, lu);
            float2 pv = make_float2(fast_exp2(xv.x), fast_exp2(xv.y));
            if (!key_ok) pv = make_float2(0.f, 0.f);
            if (diag) {
              if (key > q0 + r + u) pv.x = 0.f;
              if (key > q0 + r + u + 1) pv.y = 0.f;
            }
            const float2 g = fadd2(make_float2(__uint_as_float(dp[r + u]),
                                               __uint_as_float(dp[r + u + 1])), du);
            const float2 ds = ffma2(make_float2(pv.x * p.scale, pv.y * p.scale), g,
                                    make_float2(0.f, 0.f));
            pk[(r + u) / 2] = pack_bf16x2(pv.x, pv.y);
            dk[(r + u) / 2] = pack_bf16x2(ds.x, ds.y);
          }
        }
        tmem_st16(buf + 32 * hc, pk);
        tmem_st16(buf + C::DPOFF + 32 * hc, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[x & 1]);
      }
      if (!ok) break;
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

  // work item: query tile i of (b, h), ranked r (causal: longest rows, the
  // last query tiles, first).  The lead_q best-ranked rows of every head go
  // first, all heads at once; then each head's remaining rows in rank order,
  // head by head
  int bh, r;
  {
    const int BH = p.B * p.Hq;
    const int lead = p.lead_q;
    const unsigned x = blockIdx.x;
    if (x < (unsigned)(lead * BH)) {
      r = (int)(x / (unsigned)BH);
      bh = (int)(x - (unsigned)r * BH);
    } else {
      const unsigned y = x - (unsigned)(lead * BH);
      const int rest = p.nq - lead;
      bh = (int)(y / (unsigned)rest);
      r = lead + (int)(y - (unsigned)bh * rest);
    }
  }
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
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 8);
    }
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
    if (lane == 0 && !p.debug_stall) {
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
        if (!p.debug_stall) mbar_wait_drain(&bars->res_full, 0, lim);
        for (int x = (t > 2 ? t - 2 : 0); x < t; ++x)
          mbar_wait_drain(&bars->st_full[x & 1], (x >> 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_lo = udesc_lo(smem_u32(smem + C::Q_Q), 16);
      const uint32_t do_lo = udesc_lo(smem_u32(smem + C::Q_DO), 16);
      const uint32_t stg_lo = udesc_lo(smem_u32(smem + C::Q_STG), 16);
      const uint32_t stg_lo_mn = udesc_lo(smem_u32(smem + C::Q_STG), C::T_HALF);
      // S and dP of half x (keys 64 (x & 1) .. + 64 of the key tile in stage st)
      auto first = [&](int x, int st) {
        const uint32_t buf = tmem + C::BUF + 128u * (uint32_t)(x & 1);
        const uint32_t kd = udesc_step(stg_lo, st * C::Q_STG_BYTES + (x & 1) * 8192);
        const uint32_t vd = udesc_step(kd, C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(buf, udesc128(q_lo, off), udesc128(kd, off), IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::T_HALF + (kk % 4) * 32;
          mma_ss(buf + C::DPOFF, udesc128(do_lo, off), udesc128(vd, off), IDESC_S,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[x & 1]);
      };
      // dQ += dS K over half x (scale folded into dS): A from TMEM, B = the
      // half's rows of the K tile read MN-major; the stage is released after
      // its second half
      auto second = [&](int x, int st) -> bool {
        if (!mbar_wait(&bars->p_ready[x & 1], (x >> 1) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint32_t buf = tmem + C::BUF + 128u * (uint32_t)(x & 1);
        const uint32_t kd = udesc_step(stg_lo_mn, st * C::Q_STG_BYTES + (x & 1) * 8192);
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk)
          mma_ts(tmem + C::ACC0, buf + bf16_col(kk), udesc128(kd, kk * (16 * 128)), IDESC_O,
                 (x > 0 || kk > 0) ? 1u : 0u);
        if (x & 1) mma_commit(&bars->st_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->res_full, 0, abort, lim);
      tc_fence_after();
      int x = 0;   // halves whose first products are issued
      for (int t = 0; ok; ++t) {
        const int st = t & 1;
        if (!mbar_wait(&bars->st_full[st], (t >> 1) & 1, abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (*reinterpret_cast<volatile int*>(&bars->meta[st][0]) < 0) break;
        for (int hh = 0; hh < 2 && ok; ++hh, ++x) {
          first(x, st);
          if (x > 0) ok = second(x - 1, hh ? st : st ^ 1);
        }
      }
      if (ok && x > 0) second(x - 1, ((x - 1) >> 1) & 1);
      mma_commit(&bars->acc_done);
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else if (warp >= 4) {
    // ======================================================== element-wise warps
    // Two warps per TMEM lane quarter: warp half hc owns the key columns
    // [32 hc, 32 hc + 32) of each half-tile for its 32 query rows and writes
    // their bf16 pairs at column 32 hc, inside the columns only it reads.
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
      for (int hh = 0; hh < 2 && ok; ++hh) {
        const int x = 2 * t + hh;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x & 1], (x >> 1) & 1, abort, lim))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t buf = lane_addr + C::BUF + 128u * (uint32_t)(x & 1);
        const int k0 = j * 128 + 64 * hh + 32 * hc;   // first of this warp's 32 keys
        // keys up to the query and inside the sequence need no per-element mask
        const bool masked = (p.causal && k0 + 31 > qpos) || k0 + 32 > len;
        uint32_t sv[32], dp[32];
        tmem_ld32(buf + 32 * hc, sv);
        tmem_ld32(buf + C::DPOFF + 32 * hc, dp);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int xx = 0; xx < 32; xx += 2) {
          const float2 y = ffma2(make_float2(__uint_as_float(sv[xx]), __uint_as_float(sv[xx + 1])),
                                 sl2, nl2);
          float2 pv = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          if (masked) {
            const int key = k0 + xx;
            if (key >= len || (p.causal && key > qpos)) pv.x = 0.f;
            if (key + 1 >= len || (p.causal && key + 1 > qpos)) pv.y = 0.f;
          }
          const float2 g = fadd2(make_float2(__uint_as_float(dp[xx]), __uint_as_float(dp[xx + 1])),
                                 nd2);
          const float2 ds = ffma2(make_float2(pv.x * p.scale, pv.y * p.scale), g,
                                  make_float2(0.f, 0.f));
          dk[xx / 2] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st16(buf + 32 * hc, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[x & 1]);
      }
      if (!ok) break;
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
