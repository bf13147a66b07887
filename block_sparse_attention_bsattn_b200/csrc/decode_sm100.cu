// Split-KV decode with the BLASST skip on the 5th-generation tensor core.
//
// "BLASST: Dynamic Blocked Attention Sparsity via Softmax Thresholding",
// section 4.2: decode is bound by HBM reads of the KV cache, so every K tile is
// streamed, the skip decision is taken right after the tile's scores, and the
// V tile is loaded only when the tile is kept; K loads run ahead so that the
// decision and the remaining V loads overlap.
//
// The g query heads that share one KV head form the query tile (g <= 16).  The
// products are laid out so that the 128 keys of a tile fill the 128 MMA rows:
//   BMM1  S^T[128 keys x 16] = K_tile[128 x d] . Q^T          (tcgen05, M=128, N=16)
//   BMM2  O^T[d x 16]       += V_tile^T[d x 128] . P^T[128 x 16]
// K and V tiles arrive by TMA with the 128-byte swizzle; K is the A operand
// (K-major), V^T the A operand read MN-major from the same tile layout, and
// Q^T / P^T the B operands (16 rows, K-major).  Query columns past g read
// neighbouring heads (or zeros past the tensor) and are ignored; the
// matching P^T rows stay zero.
//
// Persistent CTAs walk a static list of (batch, KV head, split) items; every
// role walks the same global tile sequence, so the K stream never drains
// between items.  7 warps:
//   warp 0      K producer: Q^T of each item, then its K tiles (3-stage ring)
//   warp 1      TMEM owner, MMA issuer: BMM1 up to LA tiles ahead, BMM2 of a
//               kept tile once its P^T and V have arrived
//   warps 2..5  one thread per key: scores from TMEM, tile max per query head
//               (warp shuffles, then one shared-memory slot per warp), the vote,
//               the running max, P^T = exp2(S - shift) as bf16, row sums, and
//               the per-item epilogue (one thread per output dimension)
//   warp 6      V producer: waits for each decision, loads V only for kept tiles
// The exponent shift is lazy: it moves only when the running max exceeds it by
// more than TAU (base 2); O^T and the row sums are then rescaled after every
// earlier P.V has completed.  Every wait is bounded in time.
// Key tiles of 64 tokens (KT = 64) use the same 128-row products: the tile
// fills rows 0..63 of its K buffer, the scores of rows 64..127 are ignored,
// and BMM2 runs over the tile's 64 keys only (4 K-steps), so no stale row
// of a V buffer is ever read.
// The softmax warps' per-column loops run over NC columns, g rounded up to a
// power of two and fixed at compile time (one instance per NC), and the
// per-warp tile max is a butterfly reduce-scatter.  Options: sink-seeded
// splits (an extra first step scores key tile 0 to start the running max)
// and per-sequence cache lengths (the splits cut each cache's own tiles).
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsattn_internal.h"
#include "sm100_ptx.cuh"

namespace bsattn {

template <int D, int KT>
struct DecTcCfg {
  static constexpr int BLK = 128;                 // MMA rows of BMM2 (output dims, padded)
  static constexpr int NQ = 16;                   // MMA N: query columns
  static constexpr int KST = 3;                   // K ring
  // V ring: with 64-token tiles two stages, so that two CTAs fit on an SM
  static constexpr int VST = KT == 64 ? 2 : 3;
  static constexpr int LA = 3;                    // BMM1 look-ahead (tiles)
  static constexpr int NS = LA + 1;               // S buffers in TMEM
  static constexpr int PB = 4;                    // P^T slots
  static constexpr int R = 8;                     // BMM2 completion ring (> PB)
  static constexpr int DQ = 8;                    // decision queue to the V producer
  static constexpr int HALVES = D / 64;
  static constexpr int T_HALF = KT * 128;         // one 64-column box of a tile
  static constexpr int T_BYTES = HALVES * T_HALF;
  static constexpr int Q_HALF = NQ * 128;         // 16 rows x 128 bytes
  static constexpr int Q_BYTES = HALVES * Q_HALF;
  static constexpr int P_HALF = NQ * 128;         // P^T: 16 rows x 64 keys
  static constexpr int P_BYTES = (KT / 64) * P_HALF;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KST * T_BYTES;
  static constexpr int Q_OFF = V_OFF + VST * T_BYTES;
  static constexpr int P_OFF = Q_OFF + 2 * 4096;  // two item buffers (d <= 128)
  static constexpr int RED_OFF = P_OFF + PB * P_BYTES;   // float [2][4][NQ] tile maxima
  static constexpr int LS_OFF = RED_OFF + 2 * 4 * NQ * 4; // float [2][4][NQ] row sums
  static constexpr int BAR_OFF = LS_OFF + 2 * 4 * NQ * 4;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr uint32_t S_COL = 0;            // S buffer b at b * 16
  static constexpr uint32_t O_COL = 64;           // O^T buffer e at 64 + e * 16
  static constexpr int THREADS = 224;
  static constexpr float TAU = 32.0f;
};

struct DecTcBarriers {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[3], v_empty[3];
  uint64_t s_full[4], s_empty[4];
  uint64_t p_ready[4];
  uint64_t o_done[8];
  uint64_t dec_full[8], dec_empty[8];
  uint64_t red_bar[2];
  uint64_t epi_full[2], epi_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int msg[4];        // per p_ready slot: 1 = kept (P^T written), 0 = skipped
  int dec[8];        // decision queue: kept flag
};

// NC: the query columns the softmax warps work on, G rounded up to a power of
// two, fixed at compile time so that the per-column work of the scores (the
// reduction, the vote, the exponentials) unrolls and interleaves
// With 64-token tiles and at most 8 query columns two CTAs share an SM
// (launch bounds cap the registers at 146 per thread).
template <int D, int NC, int KT>
__global__ void __launch_bounds__(224, (KT == 64 && NC <= 8) ? 2 : 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecodeParams p, int G) {
  using C = DecTcCfg<D, KT>;
  static_assert(KT == 64 || KT == 128, "key tile");
  constexpr int KT_BYTES = C::T_BYTES;             // bytes of one K or V tile
  static_assert(NC == 1 || NC == 2 || NC == 4 || NC == 8 || NC == 16, "columns");
  constexpr int LOG_NC = NC >= 16 ? 4 : NC >= 8 ? 3 : NC >= 4 ? 2 : NC >= 2 ? 1 : 0;
  static_assert(sizeof(DecTcBarriers) <= C::BAR_BYTES, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* k_smem = smem + C::K_OFF;
  uint8_t* v_smem = smem + C::V_OFF;
  uint8_t* q_smem = smem + C::Q_OFF;
  uint8_t* p_smem = smem + C::P_OFF;
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  float* lsum = reinterpret_cast<float*>(smem + C::LS_OFF);
  DecTcBarriers* bars = reinterpret_cast<DecTcBarriers*>(smem + C::BAR_OFF);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_items = p.B * p.Hkv * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->red_bar[s], 4);
      mbar_init(&bars->epi_full[s], 4);
      mbar_init(&bars->epi_free[s], 1);
    }
    for (int s = 0; s < C::KST; ++s) { mbar_init(&bars->k_full[s], 1); mbar_init(&bars->k_empty[s], 1); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(&bars->v_full[s], 1); mbar_init(&bars->v_empty[s], 1); }
    for (int s = 0; s < C::NS; ++s) { mbar_init(&bars->s_full[s], 1); mbar_init(&bars->s_empty[s], 4); }
    for (int s = 0; s < 4; ++s) mbar_init(&bars->p_ready[s], 4);
    for (int s = 0; s < C::R; ++s) mbar_init(&bars->o_done[s], 1);
    for (int s = 0; s < C::DQ; ++s) { mbar_init(&bars->dec_full[s], 1); mbar_init(&bars->dec_empty[s], 1); }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  // P^T rows past g are read by BMM2 and must stay zero
  for (int x = threadIdx.x; x < C::PB * C::P_BYTES / 16; x += C::THREADS)
    reinterpret_cast<uint4*>(p_smem)[x] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t lim = p.wait_limit_ns;

  // item n of this CTA -> (batch, kv head, split) and its tile stream: nt
  // steps; with sink seeding (sd = 1) step 0 scores key tile 0 only to start
  // the running max, and step t >= sd is key tile t0 + t - sd.  With cache
  // lengths the splits cut the sequence's own ceil(len / 128) tiles.
  auto len_of = [&](int b) { return p.seq_lens ? min(max(p.seq_lens[b], 0), p.L) : p.L; };
  auto item_of = [&](int n, int& b, int& kvh, int& split, int& t0, int& nt, int& sd) {
    const int it = blockIdx.x + n * gridDim.x;
    split = it % p.splits;
    const int bk = it / p.splits;
    b = bk / p.Hkv;
    kvh = bk % p.Hkv;
    int T = p.T, chunk = p.chunk;
    if (p.seq_lens) {
      T = (len_of(b) + KT - 1) / KT;
      chunk = T > 0 ? (T + p.splits - 1) / p.splits : 1;
    }
    t0 = split * chunk;
    nt = max(0, min(T, t0 + chunk) - t0);
    sd = (p.sink_seed && split > 0 && nt > 0) ? 1 : 0;
    nt += sd;
  };
  auto tile_of = [](int t0, int sd, int t) { return (sd && t == 0) ? 0 : t0 + t - sd; };
  const int my_items = blockIdx.x < n_items ? (n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == 0) {
    // ======================================================== K producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      int g = 0;  // global tile counter
      bool ok = true;
      for (int n = 0; ok && n < my_items; ++n) {
        int b, kvh, split, t0, nt, sd;
        item_of(n, b, kvh, split, t0, nt, sd);
        const int qs = n & 1;
        if (!mbar_wait(&bars->q_empty[qs], ((n >> 1) & 1) ^ 1, abort, lim)) break;
        mbar_arrive_expect_tx(&bars->q_full[qs], C::HALVES * C::Q_HALF);
        for (int hf = 0; hf < C::HALVES; ++hf)
          tma_load_3d(q_smem + qs * 4096 + hf * C::Q_HALF, &tmQ, &bars->q_full[qs], hf * 64,
                      kvh * G, b);
        for (int t = 0; t < nt; ++t, ++g) {
          const int ks = g % C::KST;
          if (!mbar_wait(&bars->k_empty[ks], ((g / C::KST) & 1) ^ 1, abort, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->k_full[ks], KT_BYTES);
          for (int hf = 0; hf < C::HALVES; ++hf)
            tma_load_3d(k_smem + ks * C::T_BYTES + hf * C::T_HALF, &tmK, &bars->k_full[ks],
                        hf * 64, tile_of(t0, sd, t) * KT, b * p.Hkv + kvh);
        }
      }
      if (*abort) {
        for (int x = max(0, g - C::KST); x < g; ++x)
          mbar_wait_drain(&bars->k_full[x % C::KST], (x / C::KST) & 1, lim);
      }
    }
  } else if (warp == 6) {
    // ======================================================== V producer
    if (lane == 0) {
      prefetch_tensormap(&tmV);
      int g = 0, kept = 0;
      bool ok = true;
      for (int n = 0; ok && n < my_items; ++n) {
        int b, kvh, split, t0, nt, sd;
        item_of(n, b, kvh, split, t0, nt, sd);
        for (int t = 0; t < nt; ++t, ++g) {
          const int dq = g % C::DQ;
          if (!mbar_wait(&bars->dec_full[dq], (g / C::DQ) & 1, abort, lim)) { ok = false; break; }
          const int keep = *reinterpret_cast<volatile int*>(&bars->dec[dq]);
          mbar_arrive(&bars->dec_empty[dq]);
          if (!keep) continue;
          const int vs = kept % C::VST;
          if (!mbar_wait(&bars->v_empty[vs], ((kept / C::VST) & 1) ^ 1, abort, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->v_full[vs], KT_BYTES);
          for (int hf = 0; hf < C::HALVES; ++hf)
            tma_load_3d(v_smem + vs * C::T_BYTES + hf * C::T_HALF, &tmV, &bars->v_full[vs],
                        hf * 64, tile_of(t0, sd, t) * KT, b * p.Hkv + kvh);
          ++kept;
        }
      }
      if (*abort) {
        for (int x = max(0, kept - C::VST); x < kept; ++x)
          mbar_wait_drain(&bars->v_full[x % C::VST], (x / C::VST) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ======================================================== MMA issuer
    if (lane == 0) {
      // BMM1 has one MMA row per key: M = 64 for 64-token tiles, whose
      // accumulator rows 16 q + i (i < 16) sit in TMEM lane 32 q + i
      constexpr uint32_t IDESC1 = idesc_bf16_f32(KT, C::NQ, 0, 0);
      constexpr uint32_t IDESC2 = idesc_bf16_f32(128, C::NQ, 1, 0);
      const uint32_t k_addr = smem_u32(k_smem), v_addr = smem_u32(v_smem);
      const uint32_t q_addr = smem_u32(q_smem), p_addr = smem_u32(p_smem);
      // BMM1 stream state (runs up to LA tiles ahead of the BMM2 stream)
      int n1 = 0, t1 = 0, g1 = 0, nt1 = -1;
      int b_, kvh_, split_, t0_, sd_;
      bool ok = true;
      auto issue_next_bmm1 = [&]() -> int {  // 1 issued, 0 nothing left, -1 abort
        while (true) {
          if (nt1 < 0) {
            if (n1 >= my_items) return 0;
            item_of(n1, b_, kvh_, split_, t0_, nt1, sd_);
            t1 = 0;
            if (!mbar_wait(&bars->q_full[n1 & 1], (n1 >> 1) & 1, abort, lim)) return -1;
            tc_fence_after();
          }
          if (t1 < nt1) break;
          // item finished: its Q^T buffer may be refilled once these MMAs complete
          mma_commit(&bars->q_empty[n1 & 1]);
          ++n1;
          nt1 = -1;
        }
        const int ks = g1 % C::KST, sb = g1 % C::NS;
        if (!mbar_wait(&bars->k_full[ks], (g1 / C::KST) & 1, abort, lim)) return -1;
        if (!mbar_wait(&bars->s_empty[sb], ((g1 / C::NS) & 1) ^ 1, abort, lim)) return -1;
        tc_fence_after();
        const uint32_t qb = q_addr + (n1 & 1) * 4096;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a = k_addr + ks * C::T_BYTES + (kk / 4) * C::T_HALF + (kk % 4) * 32;
          const uint32_t bq = qb + (kk / 4) * C::Q_HALF + (kk % 4) * 32;
          mma_ss(tmem + C::S_COL + sb * 16, smem_desc(a, 16, 1024, 2), smem_desc(bq, 16, 1024, 2),
                 IDESC1, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->k_empty[ks]);
        ++t1;
        ++g1;
        return 1;
      };
      // prime the look-ahead
      for (int x = 0; ok && x < C::LA; ++x)
        if (issue_next_bmm1() < 0) ok = false;
      int g = 0, kept = 0;
      for (int n = 0; ok && n < my_items; ++n) {
        int b, kvh, split, t0, nt, sd;
        item_of(n, b, kvh, split, t0, nt, sd);
        int kept_item = 0;
        for (int t = 0; t < nt; ++t, ++g) {
          if (issue_next_bmm1() < 0) { ok = false; break; }
          const int pq = g % 4;
          if (!mbar_wait(&bars->p_ready[pq], (g / 4) & 1, abort, lim)) { ok = false; break; }
          tc_fence_after();
          if (!*reinterpret_cast<volatile int*>(&bars->msg[pq])) continue;
          const int vs = kept % C::VST, ps = kept % C::PB;
          if (!mbar_wait(&bars->v_full[vs], (kept / C::VST) & 1, abort, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t o_tmem = tmem + C::O_COL + (n & 1) * 16;
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk) {
            const uint32_t a = v_addr + vs * C::T_BYTES + kk * (16 * 128);
            const uint32_t bp = p_addr + ps * C::P_BYTES + (kk / 4) * C::P_HALF + (kk % 4) * 32;
            mma_ss(o_tmem, smem_desc(a, D == 128 ? C::T_HALF : 0, 1024, 2),
                   smem_desc(bp, 16, 1024, 2), IDESC2, (kept_item > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->o_done[kept % C::R]);
          mma_commit(&bars->v_empty[vs]);
          ++kept;
          ++kept_item;
        }
        if (!ok) break;
      }
      mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, lim);
    }
  } else {
    // ======================================================== score / softmax warps
    const int sw = warp - 2;                      // 0..3 -> TMEM lane quarter (warp % 4)
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;          // TMEM lane
    // key of the tile in this lane (BMM1 row): with 64-token tiles lanes
    // 16..31 of each quarter hold no key (KT marks them)
    const int key = KT == 128 ? row : (lane < 16 ? quarter * 16 + lane : KT);
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float thr = p.thr_log2;
    int g = 0, kept = 0;
    bool ok = true;
    for (int n = 0; ok && n < my_items; ++n) {
      int b, kvh, split, t0, nt, sd;
      item_of(n, b, kvh, split, t0, nt, sd);
      const int lenb = len_of(b);
      float m_run[NC], m_ref[NC], lp[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) { m_run[c] = -INFINITY; m_ref[c] = -INFINITY; lp[c] = 0.f; }
      int kept_item = 0;
      for (int t = 0; t < nt; ++t, ++g) {
        const int sb = g % C::NS;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (g / C::NS) & 1, abort, lim))) { ok = false; break; }
        tc_fence_after();
        uint32_t r[16];
        {
          // 32x32b.x16: this thread's key row, the 16 query columns
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
              "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
              : "r"(lane_addr + C::S_COL + sb * 16));
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
        const int jt = tile_of(t0, sd, t);
        const bool seed = sd && t == 0;
        const bool key_ok = key < KT && jt * KT + key < lenb;
        float s[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) s[c] = (key_ok && c < G) ? __uint_as_float(r[c]) : -INFINITY;
        // tile max per query column.  Inside the warp a butterfly that halves
        // the columns a lane holds at each exchange (NC - 1 shuffles, then a
        // plain reduction over the remaining lane bits) leaves lane l with the
        // maximum of column l >> (5 - log2 NC); across the four warps through
        // one shared-memory slot per warp and column.
        float* rr = red + (g & 1) * 4 * C::NQ;
        {
          float v[NC];
#pragma unroll
          for (int c = 0; c < NC; ++c) v[c] = s[c];
#pragma unroll
          for (int k = 0; k < LOG_NC; ++k) {
            const int w = NC >> (k + 1);
            const bool up = (lane >> (4 - k)) & 1;
#pragma unroll
            for (int i = 0; i < w; ++i) {
              const float send = up ? v[i] : v[i + w];
              const float keep = up ? v[i + w] : v[i];
              v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16 >> k));
            }
          }
#pragma unroll
          for (int off = 16 >> LOG_NC; off > 0; off >>= 1)
            v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], off));
          if ((lane & ((32 >> LOG_NC) - 1)) == 0) rr[sw * C::NQ + (lane >> (5 - LOG_NC))] = v[0];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->red_bar[g & 1]);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->red_bar[g & 1], (g >> 1) & 1, abort, lim))) { ok = false; break; }
        bool all_pass = true;
        float mt[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float m = fmaxf(fmaxf(rr[c], rr[C::NQ + c]), fmaxf(rr[2 * C::NQ + c], rr[3 * C::NQ + c]));
          mt[c] = m * p.scale_log2;
          if (c < G) all_pass = all_pass && (mt[c] - m_run[c] < thr);
        }
        // the seed step only starts the running max: never kept, not a visit
        const bool skip = seed || (p.use_skip && all_pass);
#pragma unroll
        for (int c = 0; c < NC; ++c) m_run[c] = fmaxf(m_run[c], mt[c]);
        // the decision goes to the V producer and (for tile status) to memory
        if (sw == 0 && lane == 0) {
          const int dq = g % C::DQ;
          if (!mbar_wait(&bars->dec_empty[dq], ((g / C::DQ) & 1) ^ 1, abort, lim)) {
            // abort is raised; the warp-uniform check below stops every warp
          } else {
            bars->dec[dq] = skip ? 0 : 1;
            mbar_arrive(&bars->dec_full[dq]);
          }
          if (p.tile_status && !seed)
            p.tile_status[(int64_t)(b * p.Hkv + kvh) * p.T + jt] = skip ? 1 : 2;
        }
        if (__any_sync(0xffffffffu, *abort != 0)) { ok = false; break; }
        if (!skip) {
          // the P^T slot of kept tile `kept` was last read by BMM2 of kept - PB
          if (kept >= C::PB) {
            const int pk = kept - C::PB;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[pk % C::R], (pk / C::R) & 1, abort, lim))) { ok = false; break; }
          }
          bool rescale = false;
          float alpha[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) alpha[c] = 1.f;
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            if (c >= G) continue;
            if (kept_item == 0) {
              m_ref[c] = m_run[c];
            } else if (m_run[c] > m_ref[c] + C::TAU) {
              alpha[c] = fast_exp2(m_ref[c] - m_run[c]);
              m_ref[c] = m_run[c];
              rescale = true;
            }
          }
          if (rescale) {
            // every earlier P.V of this item must have landed before O^T moves
            const int pk = kept - 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[pk % C::R], (pk / C::R) & 1, abort, lim))) { ok = false; break; }
            tc_fence_after();
            uint32_t o[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]),
                  "=r"(o[6]), "=r"(o[7]), "=r"(o[8]), "=r"(o[9]), "=r"(o[10]), "=r"(o[11]),
                  "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
                : "r"(lane_addr + C::O_COL + (n & 1) * 16));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c]);
            tmem_st16(lane_addr + C::O_COL + (n & 1) * 16, o);
            tmem_wait_st();
#pragma unroll
            for (int c = 0; c < NC; ++c) lp[c] *= alpha[c];
          }
          // P^T[c][key] = exp2(S * scale_log2 - shift) as bf16, 128-byte swizzle
          uint8_t* ps = p_smem + (kept % C::PB) * C::P_BYTES + (key / 64) * C::P_HALF;
          if (key < KT) {   // a lane without a key writes nothing
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              const float sh = m_ref[c] == -INFINITY ? 0.f : m_ref[c];
              const float pv = fast_exp2(fmaf(s[c], p.scale_log2, -sh));
              lp[c] += pv;
              const int kk = key % 64;
              *reinterpret_cast<__nv_bfloat16*>(ps + c * 128 + ((((kk >> 3) ^ (c & 7))) << 4) +
                                                (kk & 7) * 2) = __float2bfloat16_rn(pv);
            }
          }
          fence_proxy_async_smem();
          ++kept;
          ++kept_item;
        }
        if (sw == 0 && lane == 0) bars->msg[g % 4] = skip ? 0 : 1;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready[g % 4]);
      }
      if (!ok) break;
      // ---- item epilogue: O^T lanes are output dimensions
      if (kept_item > 0) {
        const int pk = kept - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[pk % C::R], (pk / C::R) & 1, abort, lim))) { ok = false; break; }
        tc_fence_after();
      }
      uint32_t o[16];
      if (kept_item > 0) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]),
              "=r"(o[6]), "=r"(o[7]), "=r"(o[8]), "=r"(o[9]), "=r"(o[10]), "=r"(o[11]),
              "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
            : "r"(lane_addr + C::O_COL + (n & 1) * 16));
        tmem_wait_ld();
      }
      // row sums: reduce the per-key partials over the 128 keys.  lsum is
      // double-buffered by item parity; warp 0 frees a buffer once it has
      // read it (epi_free), and the others fill it (epi_full).
      float* rl = lsum + (n & 1) * 4 * C::NQ;
      if (n >= 2 &&
          !__all_sync(0xffffffffu, mbar_wait(&bars->epi_free[n & 1], ((n >> 1) & 1) ^ 1, abort, lim))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (c >= G) break;
        float x = lp[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) rl[sw * C::NQ + c] = x;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->epi_full[n & 1]);
      const int64_t base = ((int64_t)b * p.Hq + (int64_t)kvh * G) * p.splits + split;
      const int dim = row;                         // O^T lane = output dimension
      if (dim < D) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (c >= G) break;
          p.ws_o[(base + (int64_t)c * p.splits) * D + dim] = kept_item > 0 ? __uint_as_float(o[c]) : 0.f;
        }
      }
      if (sw == 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->epi_full[n & 1], (n >> 1) & 1, abort, lim))) {
          ok = false;
          break;
        }
        if (lane < G) {
          const float l = rl[lane] + rl[C::NQ + lane] + rl[2 * C::NQ + lane] + rl[3 * C::NQ + lane];
          float mr = -INFINITY;
#pragma unroll
          for (int c = 0; c < NC; ++c)
            if (c == lane) mr = m_ref[c];
          p.ws_l[base + (int64_t)lane * p.splits] = kept_item > 0 ? l : 0.f;
          p.ws_m[base + (int64_t)lane * p.splits] = kept_item > 0 ? mr : -INFINITY;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->epi_free[n & 1]);
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

template <int D, int NC, int KT>
static cudaError_t launch_decode_tc_nc(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const DecodeParams& p, int G, int grid,
                                       cudaStream_t stream) {
  using C = DecTcCfg<D, KT>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<D, NC, KT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_tc_kernel<D, NC, KT>,
                           cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  // `grid` is one CTA per SM (or fewer items); with 64-token tiles and at
  // most 8 query columns two CTAs per SM (their shared memory, registers
  // under the launch bounds and 2 x 128 TMEM columns fit).  CTAs never wait
  // for one another, so a CTA that found no room would simply start later.
  const int n_items = p.B * p.Hkv * p.splits;
  if (KT == 64 && NC <= 8) grid = grid * 2 < n_items ? grid * 2 : n_items;
  decode_tc_kernel<D, NC, KT><<<grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, p, G);
  return cudaGetLastError();
}

template <int D, int KT>
static cudaError_t launch_decode_tc_kt(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const DecodeParams& p, int G, int grid,
                                       cudaStream_t stream) {
  if (G <= 1) return launch_decode_tc_nc<D, 1, KT>(tq, tk, tv, p, G, grid, stream);
  if (G <= 2) return launch_decode_tc_nc<D, 2, KT>(tq, tk, tv, p, G, grid, stream);
  if (G <= 4) return launch_decode_tc_nc<D, 4, KT>(tq, tk, tv, p, G, grid, stream);
  if (G <= 8) return launch_decode_tc_nc<D, 8, KT>(tq, tk, tv, p, G, grid, stream);
  return launch_decode_tc_nc<D, 16, KT>(tq, tk, tv, p, G, grid, stream);
}

template <int D>
cudaError_t launch_decode_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const DecodeParams& p, int G, int block, int grid,
                             cudaStream_t stream) {
  return block == 64 ? launch_decode_tc_kt<D, 64>(tq, tk, tv, p, G, grid, stream)
                     : launch_decode_tc_kt<D, 128>(tq, tk, tv, p, G, grid, stream);
}

template cudaError_t launch_decode_tc<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                           const DecodeParams&, int, int, int, cudaStream_t);
template cudaError_t launch_decode_tc<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                          const DecodeParams&, int, int, int, cudaStream_t);

}  // namespace bsattn
