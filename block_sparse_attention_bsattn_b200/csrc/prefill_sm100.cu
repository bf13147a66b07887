// Block-sparse attention prefill for sm_100a: tcgen05 tensor-core MMAs with
// TMEM accumulators, TMA-staged tiles, warp-specialised roles, and the BLASST
// skip test inside the online softmax.  Serves the cases the two-tile kernel
// does not: 64-token tiles, per-head block masks, odd GQA groups with a mask.
//
// What it computes ("BLASST: Dynamic Blocked Attention Sparsity via Softmax
// Thresholding", Algorithm 1 and section 4.1; "块稀疏Attention实战" section
// 3.3): for each query tile, the key tiles of its visit list are processed in
// order (ascending, or descending on request); every visited tile gets
// S = Q K^T (BMM1), its row max, and the skip test against the running max; a
// kept tile then gets P = exp(S - m) (CUDA cores), the row sums, and O += P V
// (BMM2).  A skipped tile costs one BMM1 and a row max.  Optional per-sequence
// lengths mask padding keys and rows.
//
// One CTA = one (batch, head, query tile) work item; 10 warps (11 with V
// skipping):
//   warp 0      TMA producer: K_j and V_j of every visited tile into 3-stage
//               rings (V is loaded for every visited tile, as the BLASST
//               prefill kernel does, unless V skipping is requested: then
//               warp 10 loads V for kept tiles only, from a decision queue);
//   warp 1      TMEM owner and MMA issuer (one elected lane): BMM1 of tile
//               t + 1 is issued before waiting for the softmax of tile t, so
//               the tensor core works while the softmax warps do;
//   warps 2..9  softmax, two warpgroups: each query row (TMEM lane) is shared
//               by one thread of each warpgroup, which own the low and the
//               high half of the score columns (and of the output columns).
//               They first write the query tile into TMEM (bf16 pairs).  Per
//               tile one shared-memory round exchanges the half-row maxima
//               and the warp votes (__all_sync per warp; a row passes iff both
//               halves pass); P = exp2 goes back to TMEM as bf16 over the
//               tile's S columns; lazy rescale of O; the epilogue.
// TMEM columns: S double buffer at [0,128) and [128,256), O at [256, 256+d),
// Q at [384, 384 + d/2).
// BMM1: A = Q (TMEM), B = K tile (smem, K-major, 128B swizzle).
// BMM2: A = P (TMEM), B = V tile (smem, MN-major, 128B swizzle).
// The query tile always occupies 128 MMA rows; with 64-token tiles rows
// 64..127 carry no data and their outputs are never read.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"
#include "umma_desc.cuh"

namespace bsattn {

// Exponentials of a kept tile: of every 8 column pairs, the last
// emu_pairs(d) go to the FMA and integer pipes (exp2_fma2) instead of the
// special-function unit, which the two softmax warpgroups share.  Measured
// best: 1 at d = 128 (Video-DiT 2.37 vs 2.43 ms; 3 is slower than none), 3 at
// d = 64, where each tile's products take half as long (multimodal DiT
// 0.100 vs 0.105 ms).
constexpr int emu_pairs(int d) { return d == 64 ? 3 : 1; }

template <int D, int BLK>
struct PrefillCfg {
  static constexpr int KST = 3;                    // K ring stages
  static constexpr int VST = 3;                    // V ring stages
  static constexpr int HALVES = D / 64;            // 64-column (128-byte) swizzle boxes
  static constexpr int T_HALF = BLK * 128;         // bytes per K/V box region
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KST * T_BYTES;
  static constexpr int XM_OFF = V_OFF + VST * T_BYTES;  // float [2][2][128] + [2][128]
  static constexpr int BAR_OFF = XM_OFF + 6 * 128 * 4;
  // + alignment slack; at least 116 KB so that one CTA (which holds all 512
  // TMEM columns) is resident per SM
  static constexpr int SMEM_USED = BAR_OFF + 512 + 1024;
  static constexpr int SMEM = SMEM_USED > 118784 ? SMEM_USED : 118784;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;             // S[b] at b * 128
  static constexpr uint32_t O_COL = 256;
  static constexpr uint32_t Q_COL = 384;           // Q tile, bf16 pairs (d/2 columns)
  static constexpr float TAU = 8.0f;               // lazy-rescale slack (base-2 units)
  static constexpr int DQ = 4;                     // decision queue (V skipping)
};

struct PrefillBarriers {
  uint64_t q_ready;      // Q written to TMEM by the softmax warps
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[3], v_empty[3];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_done;
  uint64_t drain;
  uint64_t vote_bar[2];
  uint64_t epi_bar;
  uint32_t tmem_base;
  uint64_t dq_full[4], dq_empty[4];   // decisions to the V producer (V skipping)
  int abort;
  int skip_flag[2];
  int vote[2][8];
  int dval[4];           // 1 = kept
};

// SKIPV: V tiles are loaded only for executed tiles, by an eleventh warp that
// reads each tile's decision from a queue (the page's prefill kernel loads
// every V tile; this is the option it names for memory-bound cases).
template <int D, int BLK, bool SKIPV>
__global__ void __launch_bounds__(SKIPV ? 352 : 320, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D, BLK>;
  static_assert(sizeof(PrefillBarriers) <= 512, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* k_smem = smem + C::K_OFF;
  uint8_t* v_smem = smem + C::V_OFF;
  PrefillBarriers* bars = reinterpret_cast<PrefillBarriers*>(smem + C::BAR_OFF);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work item.  Query tiles are ranked inside each head: by the index
  // builder's row order (longest rows first), else causal work longest first,
  // else ascending.  The lead_ranks best-ranked (longest) rows of every head
  // go first, all heads at once, so that no head's longest rows start late
  // and run on alone at the end of the launch; the rest go head by head (the
  // heads of one KV head are adjacent, so the CTAs resident at one time share
  // a K/V stream that stays in L2).
  int rank, bh;
  {
    const int BH = p.B * p.Hq;
    const int lead = p.lead_ranks;
    const int64_t x = blockIdx.x;
    if (x < (int64_t)lead * BH) {
      rank = (int)(x / BH);
      bh = (int)(x - (int64_t)rank * BH);
    } else {
      const int64_t y = x - (int64_t)lead * BH;
      bh = (int)(y / (p.nq - lead));
      rank = lead + (int)(y - (int64_t)bh * (p.nq - lead));
    }
  }
  int i;
  if (p.row_order) {
    const int mh_o = p.mask_heads == 1 ? 0 : bh % p.Hq;
    i = p.row_order[(int64_t)mh_o * p.nq + rank];
  } else if (p.causal) {
    i = p.nq - 1 - rank;
  } else {
    i = rank;
  }
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int kvh = h / (p.Hq / p.Hkv);
  // valid tokens of this sequence (key padding) and the key tiles holding them
  const int lenb = p.seq_lens ? min(max(p.seq_lens[b], 0), p.N) : p.N;
  const int nkb = (lenb + BLK - 1) / BLK;

  // ---- visit list
  const int32_t* cols = nullptr;
  int n;
  if (p.row_ptr) {
    const int mh = p.mask_heads == 1 ? 0 : h;
    const int32_t s0 = p.row_ptr[(int64_t)mh * (p.nq + 1) + i];
    const int32_t s1 = p.row_ptr[(int64_t)mh * (p.nq + 1) + i + 1];
    cols = p.col_idx + s0;
    n = s1 - s0;
    if (p.causal)
      while (n > 0 && cols[n - 1] > i) --n;
    while (n > 0 && cols[n - 1] >= nkb) --n;
  } else {
    n = min(p.causal ? i + 1 : p.nk, nkb);
  }
  if (i * BLK >= lenb) n = 0;   // a query tile of padding visits nothing
  // key tile of visit step t (ascending, or descending on request)
  auto col_at = [&](int t) -> int {
    const int u = p.reverse ? n - 1 - t : t;
    return cols ? cols[u] : u;
  };

  // debug trace: slot 16 + CTA = stage reached (set-up, pipeline, teardown);
  // CTA 0 also marks each warp's exit.  Nothing is recorded per tile: markers
  // on the MMA warp's path measured 5% slower in the two-tile kernel.
  const bool tr0 = blockIdx.x == 0;
  if (threadIdx.x == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, 1);

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_ready, 8);
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
      mbar_init(&bars->p_ready[s], 8);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->vote_bar[0], 8);
    mbar_init(&bars->vote_bar[1], 8);
    for (int x = 0; x < C::DQ; ++x) {
      mbar_init(&bars->dq_full[x], 1);
      mbar_init(&bars->dq_empty[x], 1);
    }
    mbar_init(&bars->epi_bar, 8);
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
  if (threadIdx.x == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, 2);

  if (warp == 0) {
    // ======================================================== TMA producer
    if (lane == 0 && n > 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int issued_k = 0, issued_v = 0;
      for (int t = 0; t < n; ++t) {
        const int j = col_at(t);
        const int ks = t % C::KST;
        if (!mbar_wait(&bars->k_empty[ks], ((t / C::KST) & 1) ^ 1, abort, lim)) break;
        mbar_arrive_expect_tx(&bars->k_full[ks], C::T_BYTES);
        for (int hf = 0; hf < C::HALVES; ++hf)
          tma_load_3d(k_smem + ks * C::T_BYTES + hf * C::T_HALF, &tmK, &bars->k_full[ks],
                      hf * 64, j * BLK, b * p.Hkv + kvh);
        ++issued_k;
        if (SKIPV) continue;   // warp 10 loads V
        const int vs = t % C::VST;
        if (!mbar_wait(&bars->v_empty[vs], ((t / C::VST) & 1) ^ 1, abort, lim)) break;
        // a skipped tile hands its V slot back without waiting for the tile:
        // the previous load into the slot must have landed before it is armed
        if (p.use_skip && t >= C::VST &&
            !mbar_wait(&bars->v_full[vs], ((t / C::VST) & 1) ^ 1, abort, lim))
          break;
        mbar_arrive_expect_tx(&bars->v_full[vs], C::T_BYTES);
        for (int hf = 0; hf < C::HALVES; ++hf)
          tma_load_3d(v_smem + vs * C::T_BYTES + hf * C::T_HALF, &tmV, &bars->v_full[vs],
                      hf * 64, j * BLK, b * p.Hkv + kvh);
        ++issued_v;
      }
      if (*abort) {
        // let every copy this thread started land before the CTA can exit
        for (int t = (issued_k > C::KST ? issued_k - C::KST : 0); t < issued_k; ++t)
          mbar_wait_drain(&bars->k_full[t % C::KST], (t / C::KST) & 1, lim);
        for (int t = (issued_v > C::VST ? issued_v - C::VST : 0); t < issued_v; ++t)
          mbar_wait_drain(&bars->v_full[t % C::VST], (t / C::VST) & 1, lim);
      } else if (p.use_skip && !SKIPV) {
        // V tiles of skipped tiles nobody waited for land before the CTA exits
        for (int t = (issued_v > C::VST ? issued_v - C::VST : 0); t < issued_v; ++t)
          mbar_wait_drain(&bars->v_full[t % C::VST], (t / C::VST) & 1, lim);
      }
    }
  } else if (SKIPV && warp == 10) {
    // ======================================================== V producer (V skipping)
    if (lane == 0 && n > 0) {
      prefetch_tensormap(&tmV);
      int vc = 0;   // V tiles loaded
      for (int t = 0; t < n; ++t) {
        const int dq = t % C::DQ;
        if (!mbar_wait(&bars->dq_full[dq], (t / C::DQ) & 1, abort, lim)) break;
        const bool need = *reinterpret_cast<volatile int*>(&bars->dval[dq]) != 0;
        mbar_arrive(&bars->dq_empty[dq]);
        if (!need) continue;
        const int vs = vc % C::VST;
        if (!mbar_wait(&bars->v_empty[vs], ((vc / C::VST) & 1) ^ 1, abort, lim)) break;
        mbar_arrive_expect_tx(&bars->v_full[vs], C::T_BYTES);
        const int j = col_at(t);
        for (int hf = 0; hf < C::HALVES; ++hf)
          tma_load_3d(v_smem + vs * C::T_BYTES + hf * C::T_HALF, &tmV, &bars->v_full[vs],
                      hf * 64, j * BLK, b * p.Hkv + kvh);
        ++vc;
      }
      if (*abort)
        for (int x = (vc > C::VST ? vc - C::VST : 0); x < vc; ++x)
          mbar_wait_drain(&bars->v_full[x % C::VST], (x / C::VST) & 1, lim);
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t IDESC1 = idesc_bf16_f32(128, BLK, 0, 0);
      constexpr uint32_t IDESC2 = idesc_bf16_f32(128, D, 0, 1);
      const uint64_t k_desc = smem_desc(smem_u32(k_smem), 16, 1024, 2);
      const uint64_t v_desc = smem_desc(smem_u32(v_smem), C::T_HALF, 1024, 2);
      bool ok = mbar_wait(&bars->q_ready, 0, abort, lim);
      tc_fence_after();
      auto issue_bmm1 = [&](int t) -> bool {
        const int ks = t % C::KST;
        if (!mbar_wait(&bars->k_full[ks], (t / C::KST) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + C::S_COL + (uint32_t)(t & 1) * 128u;
        const uint64_t kd = desc_add(k_desc, ks * C::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(d_tmem, tmem + C::Q_COL + kk * 8, desc_add(kd, (kk / 4) * C::T_HALF + (kk % 4) * 32),
                 IDESC1, kk > 0 ? 1u : 0u);
        mma_commit(&bars->s_full[t & 1]);
        mma_commit(&bars->k_empty[ks]);
        return true;
      };
      if (ok) ok = issue_bmm1(0);
      int kept = 0;
      for (int t = 0; ok && t < n; ++t) {
        if (t + 1 < n && !issue_bmm1(t + 1)) break;
        const int sb = t & 1;
        if (!mbar_wait(&bars->p_ready[sb], (t >> 1) & 1, abort, lim)) break;
        tc_fence_after();
        const int skip = *reinterpret_cast<volatile int*>(&bars->skip_flag[sb]);
        // V ring position: every visited tile's, or (V skipping) the kept ones'
        const int vi = SKIPV ? kept : t;
        const int vs = vi % C::VST;
        // a skipped tile does not wait for its V tile (see the producer)
        if (!skip && !mbar_wait(&bars->v_full[vs], (vi / C::VST) & 1, abort, lim)) break;
        tc_fence_after();
        if (!skip) {
          const uint32_t p_tmem = tmem + C::S_COL + (uint32_t)sb * 128u;
          const uint64_t vd = desc_add(v_desc, vs * C::T_BYTES);
#pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk)
            mma_ts(tmem + C::O_COL, p_tmem + kk * 8, desc_add(vd, kk * (16 * 128)), IDESC2,
                   (kept > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->o_done);
          mma_commit(&bars->v_empty[vs]);
          ++kept;
        } else if (!SKIPV) {
          mbar_arrive(&bars->v_empty[vs]);
        }
      }
      // all tcgen05 work issued by this thread must finish before TMEM is freed
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else {
    // ======================================================== softmax warps
    // Two warpgroups share every query row: warpgroup `half` owns the score
    // columns [half*CW, half*CW + CW) and the output columns
    // [half*OW, half*OW + OW) of the rows of its TMEM lane quarter.
    constexpr int CW = BLK / 2;
    constexpr int OW = D / 2;
    const int sw = warp - 2;                // 0..7
    const int half = sw / 4;
    const int quarter = warp % 4;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // query row inside the tile
    const int r0 = i * BLK;
    const bool in_tile = row < BLK;
    const bool valid = in_tile && (r0 + row < lenb);   // votes, and gets an output
    const bool in_buf = in_tile && (r0 + row < p.N);   // written (padding rows as zeros)
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + C::XM_OFF);   // [2][2][128]
    float* lx = xmax + 2 * 2 * 128;                               // [2][128]
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;          // l: this half's columns
    int kept = 0;
    bool ok = true;
    // Q row -> TMEM (the A operand of BMM1, bf16 pairs along d): warpgroup
    // `half` writes d in [half*OW, half*OW + OW); rows past N are zero
    if (n > 0 && in_tile) {
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          p.q + (((int64_t)b * p.Hq + h) * p.N + r0 + row) * D + half * OW);
#pragma unroll
      for (int c0 = 0; c0 < OW / 2; c0 += 16) {        // 16 columns = 32 bf16 = 4 x uint4
        uint32_t w[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = (r0 + row < p.N) ? qsrc[c0 / 4 + v] : make_uint4(0, 0, 0, 0);
          w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
        }
        tmem_st16(lane_addr + C::Q_COL + half * (OW / 2) + c0, w);
      }
      tmem_wait_st();
    }
    if (n > 0 && !p.debug_stall) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_ready);
    }
    for (int t = 0; t < n; ++t) {
      const int j = col_at(t);
      const int sb = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (t >> 1) & 1, abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[CW];
      float mh = -INFINITY;
      if (in_tile) {
        uint32_t r[CW];
#pragma unroll
        for (int c0 = 0; c0 < CW; c0 += 32)
          tmem_ld32(lane_addr + C::S_COL + sb * 128 + half * CW + c0,
                    *reinterpret_cast<uint32_t(*)[32]>(&r[c0]));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < CW; ++c) s[c] = __uint_as_float(r[c]);
        // element masks: keys past the end, and keys after the query (causal)
        const int k0 = j * BLK + half * CW;
        if (j * BLK + BLK > lenb || (p.causal && j == i)) {
          const int qpos = r0 + row;
#pragma unroll
          for (int c = 0; c < CW; ++c) {
            const int key = k0 + c;
            if (key >= lenb || (p.causal && key > qpos)) s[c] = -INFINITY;
          }
        }
        mh = row_max<CW>(s);
      }
      const float mth = mh * p.scale_log2;  // half-row max, base-2 units
      // The row passes iff both of its halves pass: max(a, b) - m < t exactly
      // when a - m < t and b - m < t.  One exchange round carries the warp
      // votes and the half-row maxima (needed for the running max).
      const bool pass = !valid || (mth - m_run < p.thr_log2);
      const bool wpass = __all_sync(0xffffffffu, pass);
      xmax[((t & 1) * 2 + half) * 128 + row] = mth;
      if (lane == 0) bars->vote[t & 1][sw] = wpass ? 1 : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->vote_bar[t & 1]);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->vote_bar[t & 1], (t >> 1) & 1, abort, lim))) {
        ok = false;
        break;
      }
      int skip = 0;
      if (p.use_skip) {
        volatile int* vv = bars->vote[t & 1];
        skip = vv[0] & vv[1] & vv[2] & vv[3] & vv[4] & vv[5] & vv[6] & vv[7];
      }
      if (SKIPV) {   // the decision to the V producer, before any exponential
        if (sw == 0 && lane == 0) {
          const int dq = t % C::DQ;
          if (mbar_wait(&bars->dq_empty[dq], ((t / C::DQ) & 1) ^ 1, abort, lim)) {
            bars->dval[dq] = skip ? 0 : 1;
            mbar_arrive(&bars->dq_full[dq]);
          }
        }
        if (__any_sync(0xffffffffu, *abort != 0)) {
          ok = false;
          break;
        }
      }
      const float mt = fmaxf(mth, xmax[((t & 1) * 2 + (half ^ 1)) * 128 + row]);
      m_run = fmaxf(m_run, mt);
      if (sw == 0 && lane == 0 && p.tile_status && (unsigned)j < (unsigned)p.nk)
        p.tile_status[(((int64_t)b * p.Hq + h) * p.nq + i) * p.nk + j] = skip ? 1 : 2;
      if (!skip) {
        // P of this tile goes to the other S buffer than the one the previous
        // kept tile's BMM2 may still be reading, so the exponentials need not
        // wait for that BMM2; only a rescale of O does (below).
        // exponent shift: set by the first kept tile, then moved only when the
        // running max exceeds it by more than TAU (O and l rescaled below);
        // both halves of a row compute the same shift
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
        if (in_tile) {
          // two columns per packed FMA and row-sum add
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 sh2 = make_float2(-shift, -shift);
          float2 rs4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
          for (int c0 = 0; c0 < CW; c0 += 32) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float2 x = ffma2(make_float2(s[c0 + c], s[c0 + c + 1]), sc2, sh2);
              const float2 pv = ((c / 2) % 8 >= 8 - emu_pairs(D))
                                    ? exp2_fma2(x)
                                    : make_float2(fast_exp2(x.x), fast_exp2(x.y));
              rs4[(c / 2) & 3] = fadd2(rs4[(c / 2) & 3], pv);
              pk[c / 2] = pack_bf16x2(pv.x, pv.y);
            }
            tmem_st16(lane_addr + C::S_COL + sb * 128 + (half * CW + c0) / 2, pk);
          }
          const float2 rs2 = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
          const float rs = rs2.x + rs2.y;
          l = l * alpha + rs;
          // rare: bring this half of the accumulated O to the new shift, once
          // every earlier kept tile's BMM2 has landed in it.  The wait is for
          // the newest BMM2 that can have been issued (this tile's needs this
          // warp's hand-over), so skipping the waits of earlier phases cannot
          // confuse the phase parity.
          if (__any_sync(0xffffffffu, rescale)) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, (kept - 1) & 1, abort, lim))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < OW; c0 += 32) {
              uint32_t ro[32];
              tmem_ld32(lane_addr + C::O_COL + half * OW + c0, ro);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) ro[c] = __float_as_uint(__uint_as_float(ro[c]) * alpha);
              tmem_st32(lane_addr + C::O_COL + half * OW + c0, ro);
            }
          }
          tmem_wait_st();
        }
        ++kept;
      }
      if (sw == 0 && lane == 0) bars->skip_flag[sb] = skip;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready[sb]);
    }

    // ---- epilogue: row sums of both halves, O / l -> bf16, LSE.  tcgen05.ld
    // is warp-collective, so every lane of a warp that owns tile rows loads;
    // only rows inside the sequence are stored.
    if (ok) {
      lx[half * 128 + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->epi_bar);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->epi_bar, 0, abort, lim))) ok = false;
    }
    if (ok && kept > 0) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, (kept - 1) & 1, abort, lim)))
        ok = false;
      tc_fence_after();
    }
    if (ok && in_tile) {
      const float lt = lx[row] + lx[128 + row];
      const int64_t orow = ((int64_t)b * p.Hq + h) * p.N + r0 + row;
      __nv_bfloat16* dst = p.o + orow * D + half * OW;
      const bool have = valid && kept > 0 && lt > 0.f;
      const float inv_l = have ? 1.f / lt : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < OW; c0 += 32) {
        uint32_t r[32];
        if (kept > 0) {
          tmem_ld32(lane_addr + C::O_COL + half * OW + c0, r);
          tmem_wait_ld();
        }
        if (in_buf) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float a0 = have ? __uint_as_float(r[c]) * inv_l : 0.f;
            const float a1 = have ? __uint_as_float(r[c + 1]) * inv_l : 0.f;
            w[c / 2] = pack_bf16x2(a0, a1);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (in_buf && half == 0 && p.lse)
        p.lse[orow] = have ? (m_ref + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ---- teardown
  if (lane == 0) trace_mark(p.trace, p.trace_n, tr0 ? 8 + warp : p.trace_n, 1);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, bars->abort ? 13 : 3);
  if (threadIdx.x == 0 && bars->abort) report_status(p.status, kDevTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
    if (lane == 0) trace_mark(p.trace, p.trace_n, 16 + blockIdx.x, bars->abort ? 14 : 4);
  }
}

template <int D, int BLK, bool SKIPV>
static cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const PrefillParams& p, int grid, cudaStream_t stream) {
  using C = PrefillCfg<D, BLK>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, BLK, SKIPV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, BLK, SKIPV><<<grid, SKIPV ? 352 : 320, C::SMEM, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D, int BLK>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const PrefillParams& p, int grid, cudaStream_t stream) {
  return p.skip_v ? launch_one<D, BLK, true>(tq, tk, tv, p, grid, stream)
                  : launch_one<D, BLK, false>(tq, tk, tv, p, grid, stream);
}

template cudaError_t launch_prefill<128, 128>(const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const PrefillParams&, int,
                                              cudaStream_t);
template cudaError_t launch_prefill<64, 128>(const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const PrefillParams&, int,
                                             cudaStream_t);
template cudaError_t launch_prefill<128, 64>(const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const PrefillParams&, int,
                                             cudaStream_t);
template cudaError_t launch_prefill<64, 64>(const CUtensorMap&, const CUtensorMap&,
                                            const CUtensorMap&, const PrefillParams&, int,
                                            cudaStream_t);

// The FMA-pipe exponential on its own, two elements per thread, so that it
// can be checked against its error bound.
__global__ void exp2_check_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 r = exp2_fma2(v);
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

cudaError_t launch_exp2_check(const float* x, float* y, int64_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  exp2_check_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace bsattn
