// Block-sparse prefill for two query tiles that walk the same K/V stream, so
// every K and V tile crosses L2 once for two query tiles:
//   heads mode  the same query tile of two query heads that share a KV head
//               (GQA group of even size, one visit list for the group);
//   tiles mode  two consecutive query tiles of one head when no block mask is
//               given (every key tile, or the causal prefix, which differs by
//               the diagonal tile only).  Each slot takes part in a range of
//               the stream's steps: a prefix in ascending visit order, a
//               suffix in descending order.
//
// Same method as prefill_sm100.cu ("BLASST: Dynamic Blocked Attention Sparsity
// via Softmax Thresholding", Algorithm 1 and section 4.1; "块稀疏Attention实战"
// section 3.3): per query tile, visited key tiles in order, S = Q K^T for each,
// the row max, the skip test against the running max, and for kept tiles
// P = exp(S - m), the row sums and O += P V.  The two slots' skip decisions
// are independent.  Optional: descending visit order, per-sequence lengths
// (key padding), V loads only for kept tiles.
//
// 12 warps in three warpgroups; warpgroup 0 hands registers to the two
// softmax warpgroups (setmaxnreg: 56 / 224 per thread):
//   warp 0      TMA producer: Q of both slots, then K_j (3-stage ring) and V_j
//               (2-stage ring)
//   warp 1      TMEM owner, MMA issuer.  The two query tiles ping-pong: after
//               slot A's P is ready its BMM2 and its next BMM1 are issued, then
//               slot B's, so the tensor core works on one slot while the other
//               slot's softmax runs.
//   warps 4..7  softmax of slot A, warps 8..11 softmax of slot B: one thread
//               per query row (TMEM lane); the slot's skip decision is one
//               barrier reduction (bar.red.and) over its four warps.  With
//               lambda = 0 a variant compiled without the vote runs.
//   warp 2      with V skipping only: the V producer (warp 3 idles).  The section on the
//               prefill kernel keeps every V load (the decision comes too late
//               to hide a conditional load's latency); as an option, a slot's
//               softmax sends each decision through a queue and V_j is loaded
//               only when some slot keeps tile j.
// TMEM: S_A [0,128)  O_A [128,256)  S_B [256,384)  O_B [384,512).
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

// (batch, KV head) streams the causal two-head schedule runs at one time.
// One: the CTAs resident together stream a single KV head's K/V, which stays
// in L2 (DRAM reads fall to the unique bytes, 0.4 GB instead of 9 GB for the
// 32-head, 32K-token prefill at a = 10) and the kernel is fastest; more
// streams at once measured equal or slower.
constexpr int KVG = 1;

// Exponentials of a kept tile in the variant with the skip vote: of every 8
// column pairs, the last one goes to the FMA and integer pipes (exp2_fma2)
// instead of the special-function unit, which the two slots' softmax warps
// share (1/8 and 2/8 measured best for the BLASST prefill, about 1.6 %
// faster; 3/8 and 4/8 slower; dense causal attention gained nothing at any
// share, so the variant without the vote keeps the unit for all of them).
constexpr int kEmuPairs = 1;

template <int D>
struct PairCfg {
  static constexpr int BLK = 128;
  static constexpr int KST = 3;
  static constexpr int VST = 2;
  static constexpr int HALVES = D / 64;
  static constexpr int Q_HALF = 128 * 128;
  static constexpr int T_HALF = BLK * 128;
  static constexpr int Q_BYTES = HALVES * Q_HALF;
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int Q_OFF = 0;                       // two heads
  static constexpr int K_OFF = Q_OFF + 2 * Q_BYTES;
  static constexpr int V_OFF = K_OFF + KST * T_BYTES;
  static constexpr int BAR_OFF = V_OFF + VST * T_BYTES;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr float TAU = 8.0f;
  static constexpr int DQ = 4;                          // decision queue (V skipping)
  static constexpr int THREADS = 384;                   // 3 warpgroups
  static constexpr int REG_LAUNCH = 168;                // 65536 / 384, rounded down to 8
  static constexpr int REG_LOW = 56;                    // warpgroup 0 after the split
  static constexpr int REG_HIGH = 224;                  // softmax warpgroups after the split
};

struct PairBarriers {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2];       // per head
  uint64_t p_ready[2];      // per head
  uint64_t o_done[2];       // per head
  uint64_t dq_full[2][4], dq_empty[2][4];   // per slot: decisions to the V producer
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip_flag[2];
  int dval[2][4];           // 1 = kept
};

// A shared-memory matrix descriptor (the layout of smem_desc) as its two
// 32-bit words: the low word holds the start address and the leading offset,
// the high word only constants (stride offset, version, swizzle), so the
// descriptor of a tile `off` bytes further on is the low word plus off / 16
// (addresses stay below 256 KB: no carry out of the 14-bit address field).
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo_bytes, uint32_t swizzle) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | ((swizzle & 0x7u) << 29);
}
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
__device__ __forceinline__ uint64_t desc_of(uint32_t lo, uint32_t hi) {
  return ((uint64_t)hi << 32) | lo;
}

template <int D, bool SKIPV, bool VOTE>
__global__ void __launch_bounds__(384, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PairCfg<D>;
  constexpr int BLK = C::BLK;
  static_assert(sizeof(PairBarriers) <= 512, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* k_smem = smem + C::K_OFF;
  uint8_t* v_smem = smem + C::V_OFF;
  PairBarriers* bars = reinterpret_cast<PairBarriers*>(smem + C::BAR_OFF);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work item -> two slots (head h_e, query tile i_e, visit length n_e)
  int b, hs[2], is[2], ns[2];
  const int32_t* cols = nullptr;
  int n;  // length of the shared K/V stream
  int lenb = p.N;   // valid tokens of this CTA's sequence (key padding)
  if (!p.pair_tiles) {
    const int PH = p.Hq / 2;
    int i, bp;
    if (p.row_order) {
      // KV-head-major like the causal order below, the builder's row order
      // (longest rows first) inside a KV head, its head pairs interleaved
      const int PPK = (p.Hq / p.Hkv) / 2;
      const int per_kv = p.nq * PPK;
      const int gi = (int)(blockIdx.x / (unsigned)per_kv);
      const int rem = (int)(blockIdx.x - (unsigned)gi * per_kv);
      i = p.row_order[rem / PPK];
      bp = gi * PPK + rem % PPK;
    } else if (p.causal) {
      // groups of KVG (batch, KV head) streams, one after another; inside a
      // group, longest query tile first across the group's head pairs
      const int PPK = (p.Hq / p.Hkv) / 2;              // head pairs per KV head
      const int BK = p.B * p.Hkv;
      const int per_kv = p.nq * PPK;
      const int gi = (int)(blockIdx.x / ((unsigned)per_kv * KVG));
      const int g0 = gi * KVG;
      const int gk = min(KVG, BK - g0);
      const int rem = (int)(blockIdx.x - (unsigned)gi * per_kv * KVG);
      i = p.nq - 1 - rem / (gk * PPK);
      const int within = rem % (gk * PPK);
      bp = (g0 + within / PPK) * PPK + within % PPK;
    } else {
      bp = (int)(blockIdx.x / p.nq);
      i = (int)(blockIdx.x % p.nq);
    }
    b = bp / PH;
    hs[0] = 2 * (bp % PH);
    hs[1] = hs[0] + 1;
    is[0] = is[1] = i;
    if (p.seq_lens) lenb = min(max(p.seq_lens[b], 0), p.N);
    const int nkb = (lenb + BLK - 1) / BLK;   // key tiles holding valid keys
    // visit list of mask head 0, shared by both heads
    if (p.row_ptr) {
      const int32_t s0 = p.row_ptr[i];
      const int32_t s1 = p.row_ptr[i + 1];
      cols = p.col_idx + s0;
      n = s1 - s0;
      if (p.causal)
        while (n > 0 && cols[n - 1] > i) --n;
      while (n > 0 && cols[n - 1] >= nkb) --n;
    } else {
      n = min(p.causal ? i + 1 : p.nk, nkb);
    }
    if (i * BLK >= lenb) n = 0;   // a query tile of padding visits nothing
    ns[0] = ns[1] = n;
  } else {
    const int NP = (p.nq + 1) / 2;
    int m, bh;
    if (p.causal) {  // head-major, longest pairs first: one head's K/V stays in L2
      bh = (int)(blockIdx.x / NP);
      m = NP - 1 - (int)(blockIdx.x % NP);
    } else {
      bh = (int)(blockIdx.x / NP);
      m = (int)(blockIdx.x % NP);
    }
    b = bh / p.Hq;
    hs[0] = hs[1] = bh % p.Hq;
    is[0] = 2 * m;
    is[1] = 2 * m + 1;
    if (p.seq_lens) lenb = min(max(p.seq_lens[b], 0), p.N);
    const int nkb = (lenb + BLK - 1) / BLK;
    ns[0] = is[0] * BLK < lenb ? min(p.causal ? is[0] + 1 : p.nk, nkb) : 0;
    ns[1] = is[1] * BLK < lenb ? min(p.causal ? is[1] + 1 : p.nk, nkb) : 0;
    n = max(ns[0], ns[1]);
  }
  const int kvh = hs[0] / (p.Hq / p.Hkv);
  // stream step t -> key tile (ascending, or descending on request); slot e
  // takes part in steps [tb[e], te[e]): a prefix of the stream in ascending
  // order, a suffix in descending order
  auto col_at = [&](int t) -> int {
    const int u = p.reverse ? n - 1 - t : t;
    return cols ? cols[u] : u;
  };
  int tb[2], te[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    tb[e] = p.reverse ? n - ns[e] : 0;
    te[e] = p.reverse ? n : ns[e];
  }


  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_ready[s], 4);
      mbar_init(&bars->o_done[s], 1);
      for (int x = 0; x < C::DQ; ++x) {
        mbar_init(&bars->dq_full[s][x], 1);
        mbar_init(&bars->dq_empty[s][x], 1);
      }
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
  // register split: warpgroup 0 (producers, MMA) gives registers to the two
  // softmax warpgroups.  128 * REG_LOW + 256 * REG_HIGH equals the 384 * 168
  // the block is launched with (the launcher checks the kernel's count).
  if (warp < 4) {
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 0) {
      // ======================================================== TMA producer
      if (lane == 0 && n > 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        if (!p.debug_stall) {
          mbar_arrive_expect_tx(&bars->q_full, 2 * C::HALVES * BLK * 128);
  #pragma unroll
          for (int e = 0; e < 2; ++e)
            for (int hf = 0; hf < C::HALVES; ++hf)
              tma_load_3d(q_smem + e * C::Q_BYTES + hf * C::Q_HALF, &tmQ, &bars->q_full, hf * 64,
                          is[e] * BLK, b * p.Hq + hs[e]);
        }
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
          // with the vote, a step that both slots skip hands its V slot back
          // without waiting for the tile: the previous load into the slot
          // must have landed before the slot is armed again
          if (VOTE && t >= C::VST &&
              !mbar_wait(&bars->v_full[vs], ((t / C::VST) & 1) ^ 1, abort, lim))
            break;
          mbar_arrive_expect_tx(&bars->v_full[vs], C::T_BYTES);
          for (int hf = 0; hf < C::HALVES; ++hf)
            tma_load_3d(v_smem + vs * C::T_BYTES + hf * C::T_HALF, &tmV, &bars->v_full[vs],
                        hf * 64, j * BLK, b * p.Hkv + kvh);
          ++issued_v;
        }
        if (*abort) {
          for (int t = (issued_k > C::KST ? issued_k - C::KST : 0); t < issued_k; ++t)
            mbar_wait_drain(&bars->k_full[t % C::KST], (t / C::KST) & 1, lim);
          for (int t = (issued_v > C::VST ? issued_v - C::VST : 0); t < issued_v; ++t)
            mbar_wait_drain(&bars->v_full[t % C::VST], (t / C::VST) & 1, lim);
          if (!p.debug_stall) mbar_wait_drain(&bars->q_full, 0, lim);
        } else if (VOTE && !SKIPV) {
          // V tiles of skipped steps nobody waited for land before the CTA exits
          for (int t = (issued_v > C::VST ? issued_v - C::VST : 0); t < issued_v; ++t)
            mbar_wait_drain(&bars->v_full[t % C::VST], (t / C::VST) & 1, lim);
        }
      }
    } else if (SKIPV && warp == 2) {
      // ======================================================== V producer (V skipping)
      if (lane == 0 && n > 0) {
        prefetch_tensormap(&tmV);
        int vc = 0;   // V tiles loaded
        bool ok = true;
        for (int t = 0; ok && t < n; ++t) {
          bool need = false;
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (t < tb[e] || t >= te[e]) continue;
            const int tl = t - tb[e];
            if (!mbar_wait(&bars->dq_full[e][tl % C::DQ], (tl / C::DQ) & 1, abort, lim)) {
              ok = false;
              break;
            }
            need = need || *reinterpret_cast<volatile int*>(&bars->dval[e][tl % C::DQ]) != 0;
            mbar_arrive(&bars->dq_empty[e][tl % C::DQ]);
          }
          if (!ok || !need) continue;
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
        constexpr uint32_t HI = desc_hi(1024, 2);
        const uint32_t q_lo = desc_lo(smem_u32(q_smem), 16);
        const uint32_t k_lo = desc_lo(smem_u32(k_smem), 16);
        const uint32_t v_lo = desc_lo(smem_u32(v_smem), C::T_HALF);
        bool ok = mbar_wait(&bars->q_full, 0, abort, lim);
        tc_fence_after();
        // S_e = Q_e K_t^T into TMEM columns [256 e, 256 e + 128)
        auto bmm1 = [&](int e, int t) {
          const uint32_t qa = q_lo + (uint32_t)e * (C::Q_BYTES / 16);
          const uint32_t ka = k_lo + (uint32_t)(t % C::KST) * (C::T_BYTES / 16);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk / 4) * C::Q_HALF + (kk % 4) * 32) / 16;
            const uint32_t ko = ((kk / 4) * C::T_HALF + (kk % 4) * 32) / 16;
            mma_ss(tmem + 256 * e, desc_of(qa + qo, HI), desc_of(ka + ko, HI), IDESC1,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[e]);
        };
        // O_e += P_e V, P_e in TMEM over S_e, V in ring slot vs
        auto bmm2 = [&](int e, int vs, int first) {
          const uint32_t va = v_lo + (uint32_t)vs * (C::T_BYTES / 16);
  #pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk)
            mma_ts(tmem + 256 * e + 128, tmem + 256 * e + kk * 8, desc_of(va + kk * (16 * 128) / 16, HI),
                   IDESC2, (!first || kk > 0) ? 1u : 0u);
          mma_commit(&bars->o_done[e]);
        };
        if (ok) {
          ok = mbar_wait(&bars->k_full[0], 0, abort, lim);
          tc_fence_after();
          if (ok) {
            if (tb[0] == 0 && te[0] > 0) bmm1(0, 0);
            if (tb[1] == 0 && te[1] > 0) bmm1(1, 0);
            mma_commit(&bars->k_empty[0]);
          }
        }
        int kept[2] = {0, 0};
        int vc = 0;   // V tiles loaded so far (V skipping: only the kept steps')
        for (int t = 0; ok && t < n; ++t) {
          const int vi = SKIPV ? vc : t;
          const int vs = vi % C::VST;
          bool v_ready = false;
          bool k_next = false;        // K_{t+1} waited for
          const bool more = t + 1 < n;
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (t >= tb[e] && t < te[e]) {   // this slot takes part in step t
              int skip = 0;
              if (VOTE) {
                if (!mbar_wait(&bars->p_ready[e], (t - tb[e]) & 1, abort, lim)) { ok = false; break; }
                tc_fence_after();
                skip = *reinterpret_cast<volatile int*>(&bars->skip_flag[e]);
              } else {
                // no skipping: every tile is kept and p_ready completes once per tile
                if (!mbar_wait(&bars->p_ready[e], kept[e] & 1, abort, lim)) { ok = false; break; }
                tc_fence_after();
              }
              if (!skip) {
                if (!v_ready) {
                  if (!mbar_wait(&bars->v_full[vs], (vi / C::VST) & 1, abort, lim)) { ok = false; break; }
                  tc_fence_after();
                  v_ready = true;
                }
                bmm2(e, vs, kept[e] == 0);
                ++kept[e];
              }
            }
            if (t + 1 >= tb[e] && t + 1 < te[e]) {
              if (!k_next) {   // first use of K_{t+1}
                const int ks = (t + 1) % C::KST;
                if (!mbar_wait(&bars->k_full[ks], ((t + 1) / C::KST) & 1, abort, lim)) { ok = false; break; }
                tc_fence_after();
                k_next = true;
              }
              bmm1(e, t + 1);
            }
          }
          if (!ok) break;
          if (more) mma_commit(&bars->k_empty[(t + 1) % C::KST]);
          // release V_t: consumed (or not needed) by both slots; with V skipping
          // a step that no slot keeps has no V tile.  With the vote, a step
          // that no slot keeps releases the slot at once, without waiting for
          // the tile to land (the producer waits for that before it loads the
          // slot again), so the MMA warp goes straight on to the next step.
          if (v_ready) {
            mma_commit(&bars->v_empty[vs]);
            ++vc;
          } else if (!SKIPV) {
            if (!VOTE && !mbar_wait(&bars->v_full[vs], (t / C::VST) & 1, abort, lim)) break;
            mbar_arrive(&bars->v_empty[vs]);
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
      const int e = (warp - 4) / 4;           // which slot of the pair
      const int sw = (warp - 4) % 4;
      const int quarter = warp % 4;
      const int row = quarter * 32 + lane;
      // this slot's values as scalars (a runtime index would put the arrays in
      // local memory)
      const int i = e ? is[1] : is[0];
      const int r0 = i * BLK;
      const int h = e ? hs[1] : hs[0];
      const int t_first = e ? tb[1] : tb[0];
      const int ne = (e ? te[1] : te[0]) - t_first;
      // key tile of this slot's t-th visit: u0 + du * t into the CSR row (or
      // the tile index itself without one)
      const int du = p.reverse ? -1 : 1;
      const int u0 = p.reverse ? n - 1 - t_first : t_first;
      const bool valid = r0 + row < lenb;    // votes, and gets an output
      const bool in_buf = r0 + row < p.N;    // written (padding rows as zeros)
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const uint32_t s_col = 256 * e, o_col = 256 * e + 128;
      float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
      int kept = 0;
      bool ok = true;
      for (int t = 0; t < ne; ++t) {       // t counts this slot's tiles
        const int u = u0 + du * t;
        const int j = cols ? cols[u] : u;
        // A warp whose wait ran out (ok false) does no more work, but it still
        // meets the slot's other warps at the vote barrier once per tile, so
        // no warp is ever left waiting there: nothing in the loop leaves it
        // early.
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
          // the slot's decision: every valid row of the query tile passes.  One
          // barrier reduction over the slot's four warps (named barrier 1 + e)
          const bool pass = !valid || (mt - m_run < p.thr_log2);
          skip = bar_red_and(1 + e, 128, pass) ? 1 : 0;
        }
        if (SKIPV) {   // the decision to the V producer, before any exponential
          if (sw == 0 && lane == 0) {
            const int dq = t % C::DQ;
            if (mbar_wait(&bars->dq_empty[e][dq], ((t / C::DQ) & 1) ^ 1, abort, lim)) {
              bars->dval[e][dq] = skip ? 0 : 1;
              mbar_arrive(&bars->dq_full[e][dq]);
            }
          }
          if (__any_sync(0xffffffffu, *abort != 0)) {
            ok = false;
            continue;
          }
        }
        m_run = fmaxf(m_run, mt);
        if (sw == 0 && lane == 0 && p.tile_status && (unsigned)j < (unsigned)p.nk)
          p.tile_status[(((int64_t)b * p.Hq + h) * p.nq + i) * p.nk + j] = skip ? 1 : 2;
        if (!skip) {
          if (kept > 0) {
            // S_e holds this tile, so BMM2 of the previous kept tile has finished
            // reading P; wait for it to land in O before O may be rescaled
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
          // P = exp2(S * scale_log2 - shift), two columns per packed FMA and
          // row-sum add, written back over S as bf16 pairs
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 sh2 = make_float2(-shift, -shift);
          float2 rs4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  #pragma unroll
          for (int c0 = 0; c0 < BLK; c0 += 32) {
            uint32_t pk[16];
  #pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float2 x = ffma2(make_float2(__uint_as_float(r[c0 + c]),
                                                 __uint_as_float(r[c0 + c + 1])), sc2, sh2);
              const float2 pv = (VOTE && (c / 2) % 8 >= 8 - kEmuPairs)
                                    ? exp2_fma2(x)
                                    : make_float2(fast_exp2(x.x), fast_exp2(x.y));
              rs4[(c / 2) & 3] = fadd2(rs4[(c / 2) & 3], pv);
              pk[c / 2] = pack_bf16x2(pv.x, pv.y);
            }
            tmem_st16(lane_addr + s_col + c0 / 2, pk);
          }
          const float2 rs2 = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
          const float rs = rs2.x + rs2.y;
          l = l * alpha + rs;
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
      // ---- epilogue
      if (ok && kept > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[e], (kept - 1) & 1, abort, lim)))
          ok = false;
        tc_fence_after();
      }
      if (ok) {
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

template <int D, bool SKIPV, bool VOTE>
static cudaError_t launch_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const PrefillParams& p, int grid,
                               cudaStream_t stream) {
  using C = PairCfg<D>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(prefill_pair_kernel<D, SKIPV, VOTE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  static_assert(128 * C::REG_LOW + 256 * C::REG_HIGH == C::THREADS * C::REG_LAUNCH,
                "register split must equal the launch allocation");
  // setmaxnreg.inc waits until the block's pool has the registers; launch only
  // when the compiled kernel reserves the REG_LAUNCH the split is built on
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, prefill_pair_kernel<D, SKIPV, VOTE>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != C::REG_LAUNCH) return cudaErrorInvalidConfiguration;
  prefill_pair_kernel<D, SKIPV, VOTE><<<grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_prefill_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const PrefillParams& p, int grid,
                                cudaStream_t stream) {
  // lambda = 0: a kernel without the vote (nothing is skipped, so V skipping
  // has nothing to skip either)
  if (!p.use_skip) return launch_pair<D, false, false>(tq, tk, tv, p, grid, stream);
  return p.skip_v ? launch_pair<D, true, true>(tq, tk, tv, p, grid, stream)
                  : launch_pair<D, false, true>(tq, tk, tv, p, grid, stream);
}

template cudaError_t launch_prefill_pair<128>(const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const PrefillParams&, int,
                                              cudaStream_t);
template cudaError_t launch_prefill_pair<64>(const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const PrefillParams&, int,
                                             cudaStream_t);

}  // namespace bsattn
