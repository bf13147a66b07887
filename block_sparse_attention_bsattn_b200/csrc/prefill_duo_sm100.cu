// Block-sparse prefill for two query tiles per CTA whose visit lists are
// their own: the tiles of a block mask that no two query tiles share (one
// query head per KV head, or one mask per head), 128-token tiles.
//
// Same method as the other prefill kernels ("BLASST: Dynamic Blocked
// Attention Sparsity via Softmax Thresholding", Algorithm 1 and section 4.1;
// "块稀疏Attention实战" section 3.3): per query tile, its visited key tiles in
// order, S = Q K^T for each, the row max, the skip test against the running
// max, and for kept tiles P = exp(S - m), the row sums and O += P V.
//
// Why two tiles: one query tile alone leaves the tensor core idle while its
// softmax runs and the softmax idle while its MMAs run; with two, the MMA
// warp works on one tile while the other's softmax runs (the ping-pong of
// the BLASST page's prefill kernel, Figure 3).  The two query tiles here do
// not share K/V tiles: each slot has its own stream, and the two streams are
// interleaved through one ring -- load t of slot A, load t of slot B, load
// t + 1 of slot A, ... -- until the shorter list ends.  Work items are taken
// in pairs from the work order (longest rows first when the index builder's
// row order is given), so the two lists of a CTA have nearly equal lengths.
//
// 12 warps in three warpgroups (setmaxnreg: 56 registers per thread for
// warpgroup 0, 224 for the two softmax warpgroups):
//   warp 0      TMA producer of both Q tiles and the K tile of each load of
//               the interleaved stream (ring of KST stages)
//   warp 2      TMA producer of the V tiles (ring of VST stages)
//   warp 1      TMEM owner and MMA issuer
//   warps 4..7  softmax of slot A, warps 8..11 of slot B: one thread per query
//               row; the skip decision is one barrier reduction (bar.red.and)
//               over the slot's four warps; lambda = 0 runs a variant without it
// TMEM: S_A [0,128)  O_A [128,128+d)  S_B [256,384)  O_B [384,384+d).
// BMM1: A = Q (smem, K-major, 128B swizzle), B = K tile (smem, K-major).
// BMM2: A = P (TMEM, bf16 over S), B = V tile (smem, MN-major).
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

template <int D>
struct DuoCfg {
  static constexpr int BLK = 128;
  static constexpr int KST = D == 128 ? 3 : 4;          // K ring stages
  static constexpr int VST = D == 128 ? 2 : 4;          // V ring stages
  static constexpr int HALVES = D / 64;                 // 64-column (128-byte) swizzle boxes
  static constexpr int Q_HALF = 128 * 128;
  static constexpr int T_HALF = BLK * 128;
  static constexpr int Q_BYTES = HALVES * Q_HALF;
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int Q_OFF = 0;                       // two query tiles
  static constexpr int K_OFF = Q_OFF + 2 * Q_BYTES;
  static constexpr int V_OFF = K_OFF + KST * T_BYTES;
  static constexpr int BAR_OFF = V_OFF + VST * T_BYTES;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr float TAU = 8.0f;                    // lazy-rescale slack (base 2)
  static constexpr int THREADS = 384;
  static constexpr int REG_LAUNCH = 168;
  static constexpr int REG_LOW = 56;
  static constexpr int REG_HIGH = 224;
};

struct DuoBarriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip_flag[2];
};

// One work item of the pair: (batch, query head, query tile) and its visit
// list (CSR row, truncated by the causal limit and the sequence length).
struct DuoSlot {
  int b, h, kvh, i, n, lenb;
  const int32_t* cols;
};

__device__ __forceinline__ DuoSlot duo_slot(const PrefillParams& p, int64_t x) {
  DuoSlot s;
  const int64_t items = (int64_t)p.B * p.Hq * p.nq;
  if (x >= items) {   // the second slot of the last CTA when the count is odd
    s.b = s.h = s.kvh = s.i = 0;
    s.n = -1;
    s.lenb = 0;
    s.cols = nullptr;
    return s;
  }
  const int bh = (int)(x / p.nq);
  const int r = (int)(x - (int64_t)bh * p.nq);
  s.b = bh / p.Hq;
  s.h = bh % p.Hq;
  s.kvh = s.h / (p.Hq / p.Hkv);
  const int mh = p.mask_heads == 1 ? 0 : s.h;
  if (p.row_order) s.i = p.row_order[(int64_t)mh * p.nq + r];
  else s.i = p.causal ? p.nq - 1 - r : r;
  s.lenb = p.seq_lens ? min(max(p.seq_lens[s.b], 0), p.N) : p.N;
  const int nkb = (s.lenb + 128 - 1) / 128;
  int n;
  s.cols = nullptr;
  if (p.row_ptr) {
    const int32_t s0 = p.row_ptr[(int64_t)mh * (p.nq + 1) + s.i];
    const int32_t s1 = p.row_ptr[(int64_t)mh * (p.nq + 1) + s.i + 1];
    s.cols = p.col_idx + s0;
    n = s1 - s0;
    if (p.causal)
      while (n > 0 && s.cols[n - 1] > s.i) --n;
    while (n > 0 && s.cols[n - 1] >= nkb) --n;
  } else {
    n = min(p.causal ? s.i + 1 : p.nk, nkb);
  }
  if (s.i * 128 >= s.lenb) n = 0;
  s.n = n;
  return s;
}

template <int D, bool VOTE>
__global__ void __launch_bounds__(384, 1)
    prefill_duo_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = DuoCfg<D>;
  constexpr int BLK = C::BLK;
  static_assert(sizeof(DuoBarriers) <= 512, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* k_smem = smem + C::K_OFF;
  uint8_t* v_smem = smem + C::V_OFF;
  DuoBarriers* bars = reinterpret_cast<DuoBarriers*>(smem + C::BAR_OFF);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const DuoSlot s0 = duo_slot(p, 2 * (int64_t)blockIdx.x);
  const DuoSlot s1 = duo_slot(p, 2 * (int64_t)blockIdx.x + 1);
  const int n0 = max(s0.n, 0), n1 = max(s1.n, 0);
  // interleaved stream: load 2t + e is tile t of slot e while both lists
  // last, then the longer list's tiles one by one
  const int mboth = min(n0, n1), ntot = n0 + n1, longer = n0 >= n1 ? 0 : 1;
  auto pos = [&](int e, int t) -> int { return t < mboth ? 2 * t + e : 2 * mboth + (t - mboth); };
  // key tile of slot e's t-th visit (ascending, or descending on request)
  auto col_at = [&](int e, int t) -> int {
    const int ne = e ? n1 : n0;
    const int32_t* cols = e ? s1.cols : s0.cols;
    const int u = p.reverse ? ne - 1 - t : t;
    return cols ? cols[u] : u;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_ready[s], 4);
      mbar_init(&bars->o_done[s], 1);
    }
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
  if (warp < 4) {
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 0 || warp == 2) {
      // ================================================ TMA producers: warp 0
      // loads Q and K, warp 2 loads V, each as far ahead as its own ring
      // allows (a K load waiting behind a V stage would reach the MMA warp
      // just when it is needed)
      const bool kw = warp == 0;
      if (lane == 0 && ntot > 0) {
        if (kw) {
          prefetch_tensormap(&tmQ);
          prefetch_tensormap(&tmK);
        } else {
          prefetch_tensormap(&tmV);
        }
        if (kw && !p.debug_stall) {
          mbar_arrive_expect_tx(&bars->q_full,
                                ((n0 > 0) + (n1 > 0)) * C::HALVES * BLK * 128);
          for (int hf = 0; hf < C::HALVES; ++hf) {
            if (n0 > 0)
              tma_load_3d(q_smem + hf * C::Q_HALF, &tmQ, &bars->q_full, hf * 64, s0.i * BLK,
                          s0.b * p.Hq + s0.h);
            if (n1 > 0)
              tma_load_3d(q_smem + C::Q_BYTES + hf * C::Q_HALF, &tmQ, &bars->q_full, hf * 64,
                          s1.i * BLK, s1.b * p.Hq + s1.h);
          }
        }
        const int NST = kw ? C::KST : C::VST;
        uint64_t* full = kw ? bars->k_full : bars->v_full;
        uint64_t* empty = kw ? bars->k_empty : bars->v_empty;
        uint8_t* ring = kw ? k_smem : v_smem;
        const CUtensorMap* map = kw ? &tmK : &tmV;
        int issued = 0;
        for (int x = 0; x < ntot; ++x) {
          const int e = x < 2 * mboth ? (x & 1) : longer;
          const int t = x < 2 * mboth ? (x >> 1) : mboth + (x - 2 * mboth);
          const int j = col_at(e, t);
          const int z = e ? s1.b * p.Hkv + s1.kvh : s0.b * p.Hkv + s0.kvh;
          const int st = x % NST;
          if (!mbar_wait(&empty[st], ((x / NST) & 1) ^ 1, abort, lim)) break;
          mbar_arrive_expect_tx(&full[st], C::T_BYTES);
          for (int hf = 0; hf < C::HALVES; ++hf)
            tma_load_3d(ring + st * C::T_BYTES + hf * C::T_HALF, map, &full[st], hf * 64, j * BLK,
                        z);
          ++issued;
        }
        if (*abort) {
          // let every copy this thread started land before the CTA can exit
          for (int x = (issued > NST ? issued - NST : 0); x < issued; ++x)
            mbar_wait_drain(&full[x % NST], (x / NST) & 1, lim);
          if (kw && !p.debug_stall) mbar_wait_drain(&bars->q_full, 0, lim);
        }
      }
    } else if (warp == 1) {
      // ======================================================== MMA issuer
      if (lane == 0 && ntot > 0) {
        constexpr uint32_t IDESC1 = idesc_bf16_f32(128, BLK, 0, 0);
        constexpr uint32_t IDESC2 = idesc_bf16_f32(128, D, 0, 1);
        const uint32_t q_addr = smem_u32(q_smem);
        const uint32_t k_addr = smem_u32(k_smem);
        const uint32_t v_addr = smem_u32(v_smem);
        bool ok = mbar_wait(&bars->q_full, 0, abort, lim);
        tc_fence_after();
        // S_e = Q_e K^T (K of stream load x) into TMEM columns [256 e, 256 e + 128);
        // the K stage is released when the product has read it
        auto bmm1 = [&](int e, int x) -> bool {
          const int ks = x % C::KST;
          if (!mbar_wait(&bars->k_full[ks], (x / C::KST) & 1, abort, lim)) return false;
          tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t a = q_addr + e * C::Q_BYTES + (kk / 4) * C::Q_HALF + (kk % 4) * 32;
            const uint32_t bb = k_addr + ks * C::T_BYTES + (kk / 4) * C::T_HALF + (kk % 4) * 32;
            mma_ss(tmem + 256 * e, smem_desc(a, 16, 1024, 2), smem_desc(bb, 16, 1024, 2), IDESC1,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[e]);
          mma_commit(&bars->k_empty[ks]);
          return true;
        };
        // O_e += P_e V (V of stream load x), P_e in TMEM over S_e
        auto bmm2 = [&](int e, int vs, int first) {
  #pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk) {
            const uint32_t bb = v_addr + vs * C::T_BYTES + kk * (16 * 128);
            mma_ts(tmem + 256 * e + 128, tmem + 256 * e + kk * 8, smem_desc(bb, C::T_HALF, 1024, 2),
                   IDESC2, (!first || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->o_done[e]);
        };
        if (ok && n0 > 0) ok = bmm1(0, pos(0, 0));
        if (ok && n1 > 0) ok = bmm1(1, pos(1, 0));
        int kept[2] = {0, 0};
        const int nmax = max(n0, n1);
        for (int t = 0; ok && t < nmax; ++t) {
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int ne = e ? n1 : n0;
            if (!ok || t >= ne) continue;
            // every tile is handed back once, so the phase parity is t's
            if (!mbar_wait(&bars->p_ready[e], t & 1, abort, lim)) { ok = false; break; }
            tc_fence_after();
            const int skip = VOTE ? *reinterpret_cast<volatile int*>(&bars->skip_flag[e]) : 0;
            const int x = pos(e, t);
            const int vs = x % C::VST;
            // V of this load has landed (a skipped tile's too: the stage is
            // only handed back after its copy completed)
            if (!mbar_wait(&bars->v_full[vs], (x / C::VST) & 1, abort, lim)) { ok = false; break; }
            tc_fence_after();
            if (!skip) {
              bmm2(e, vs, kept[e] == 0);
              ++kept[e];
            }
            // released by a commit in both cases, so the release arrives after
            // every earlier product has finished reading this stage
            mma_commit(&bars->v_empty[vs]);
            if (t + 1 < ne && !bmm1(e, pos(e, t + 1))) { ok = false; break; }
          }
        }
        mma_commit(&bars->drain);
        mbar_wait_drain(&bars->drain, 0, lim);
      }
    }
  } else {
    setmaxnreg_inc<C::REG_HIGH>();
    {
      // ======================================================== softmax warps
      const int e = (warp - 4) / 4;           // which slot
      const int sw = (warp - 4) % 4;
      const int quarter = warp % 4;
      const int row = quarter * 32 + lane;
      // this slot's values as scalars (a runtime index would put them in
      // local memory)
      const bool has = (e ? s1.n : s0.n) >= 0;   // the slot holds a work item
      const int ne = e ? n1 : n0;
      const int i = e ? s1.i : s0.i;
      const int h = e ? s1.h : s0.h;
      const int b = e ? s1.b : s0.b;
      const int lenb = e ? s1.lenb : s0.lenb;
      const int32_t* cols = e ? s1.cols : s0.cols;
      const int r0 = i * BLK;
      const int du = p.reverse ? -1 : 1;
      const int u0 = p.reverse ? ne - 1 : 0;
      const bool valid = r0 + row < lenb;    // votes, and gets an output
      const bool in_buf = has && r0 + row < p.N;
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const uint32_t s_col = 256 * e, o_col = 256 * e + 128;
      float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
      int kept = 0;
      bool ok = true;
      for (int t = 0; t < ne; ++t) {
        const int u = u0 + du * t;
        const int j = cols ? cols[u] : u;
        // a warp whose wait ran out does no more work but still meets the
        // slot's other warps at the vote barrier once per tile
        if (!ok || !__all_sync(0xffffffffu, mbar_wait(&bars->s_full[e], t & 1, abort, lim))) {
          ok = false;
          if (VOTE) bar_red_and(1 + e, 128, true);
          continue;
        }
        tc_fence_after();
        uint32_t r[BLK];
  #pragma unroll
        for (int c0 = 0; c0 < BLK; c0 += 32)
          tmem_ld32(lane_addr + s_col + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
        tmem_wait_ld();
        const int k0 = j * BLK;
        if (k0 + BLK > lenb || (p.causal && j == i)) {
          const int qpos = r0 + row;
  #pragma unroll
          for (int c = 0; c < BLK; ++c) {
            const int key = k0 + c;
            if (key >= lenb || (p.causal && key > qpos)) r[c] = __float_as_uint(-INFINITY);
          }
        }
        const float mt = row_max<BLK>(reinterpret_cast<const float*>(r)) * p.scale_log2;
        int skip = 0;
        if (VOTE) {
          const bool pass = !valid || (mt - m_run < p.thr_log2);
          skip = bar_red_and(1 + e, 128, pass) ? 1 : 0;
        }
        m_run = fmaxf(m_run, mt);
        if (sw == 0 && lane == 0 && p.tile_status && (unsigned)j < (unsigned)p.nk)
          p.tile_status[(((int64_t)b * p.Hq + h) * p.nq + i) * p.nk + j] = skip ? 1 : 2;
        if (!skip) {
          if (kept > 0) {
            // S_e holds this tile, so the previous kept tile's BMM2 (issued
            // before this tile's BMM1) has completed; its wait is immediate
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[e], (kept - 1) & 1, abort, lim))) {
              ok = false;
              continue;
            }
            tc_fence_after();
          }
          float alpha = 1.f;
          bool rescale = false;
          if (kept == 0) {
            m_ref = m_run;
          } else if (m_run > m_ref + C::TAU) {
            alpha = fast_exp2(m_ref - m_run);
            rescale = true;
            m_ref = m_run;
          }
          const float shift = (m_ref == -INFINITY) ? 0.f : m_ref;
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 sh2 = make_float2(-shift, -shift);
          float2 rs4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  #pragma unroll
          for (int c0 = 0; c0 < BLK; c0 += 32) {
            uint32_t pk[16];
  #pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float2 xx = ffma2(make_float2(__uint_as_float(r[c0 + c]),
                                                  __uint_as_float(r[c0 + c + 1])), sc2, sh2);
              const float2 pv = make_float2(fast_exp2(xx.x), fast_exp2(xx.y));
              rs4[(c / 2) & 3] = fadd2(rs4[(c / 2) & 3], pv);
              pk[c / 2] = pack_bf16x2(pv.x, pv.y);
            }
            tmem_st16(lane_addr + s_col + c0 / 2, pk);
          }
          const float2 rs2 = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
          l = l * alpha + (rs2.x + rs2.y);
          if (__any_sync(0xffffffffu, rescale)) {
  #pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ro[32];
              tmem_ld32(lane_addr + o_col + c0, ro);
              tmem_wait_ld();
  #pragma unroll
              for (int c = 0; c < 32; ++c) ro[c] = __float_as_uint(__uint_as_float(ro[c]) * alpha);
              tmem_st32(lane_addr + o_col + c0, ro);
            }
          }
          tmem_wait_st();
          ++kept;
        }
        if (VOTE && sw == 0 && lane == 0) bars->skip_flag[e] = skip;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[e]);
      }
      // ---- epilogue: O / l -> bf16 and the LSE; rows of a query tile that
      // visits nothing are written as zeros (LSE -inf)
      if (ok && kept > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[e], (kept - 1) & 1, abort, lim)))
          ok = false;
        tc_fence_after();
      }
      if (ok && has) {
        const int64_t orow = ((int64_t)b * p.Hq + h) * p.N + r0 + row;
        __nv_bfloat16* dst = p.o + orow * D;
        const bool have = valid && kept > 0 && l > 0.f;
        const float inv_l = have ? 1.f / l : 0.f;
  #pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ro[32];
          if (kept > 0) {
            tmem_ld32(lane_addr + o_col + c0, ro);
            tmem_wait_ld();
          }
          if (in_buf) {
            uint32_t w[16];
  #pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float a0 = have ? __uint_as_float(ro[c]) * inv_l : 0.f;
              const float a1 = have ? __uint_as_float(ro[c + 1]) * inv_l : 0.f;
              w[c / 2] = pack_bf16x2(a0, a1);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
  #pragma unroll
            for (int v = 0; v < 4; ++v)
              d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (in_buf && p.lse)
          p.lse[orow] = have ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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

template <int D, bool VOTE>
static cudaError_t launch_duo(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const PrefillParams& p, int grid, cudaStream_t stream) {
  using C = DuoCfg<D>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static_assert(128 * C::REG_LOW + 256 * C::REG_HIGH == C::THREADS * C::REG_LAUNCH,
                "register split must equal the launch allocation");
  cudaError_t e = cudaFuncSetAttribute(prefill_duo_kernel<D, VOTE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits until the block's pool has the registers; launch only
  // when the compiled kernel reserves the REG_LAUNCH the split is built on
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, prefill_duo_kernel<D, VOTE>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != C::REG_LAUNCH) return cudaErrorInvalidConfiguration;
  prefill_duo_kernel<D, VOTE><<<grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_prefill_duo(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const PrefillParams& p, int grid,
                               cudaStream_t stream) {
  return p.use_skip ? launch_duo<D, true>(tq, tk, tv, p, grid, stream)
                    : launch_duo<D, false>(tq, tk, tv, p, grid, stream);
}

template cudaError_t launch_prefill_duo<128>(const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const PrefillParams&, int,
                                             cudaStream_t);
template cudaError_t launch_prefill_duo<64>(const CUtensorMap&, const CUtensorMap&,
                                            const CUtensorMap&, const PrefillParams&, int,
                                            cudaStream_t);

}  // namespace bsattn
